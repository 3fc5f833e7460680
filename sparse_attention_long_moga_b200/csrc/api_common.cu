// Host-side status handling shared by all entry points.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace moga {

static thread_local char t_last_error[512] = "";

moga_status fail(moga_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

moga_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  t_last_error[0] = 0;
  return MOGA_OK;
}

}  // namespace moga

extern "C" const char* moga_last_error(void) { return moga::t_last_error; }

extern "C" const char* moga_version(void) {
#ifdef MOGA_DEBUG
  return "moga-b200 0.2 (sm_100a, checking build: device-side index checks)";
#else
  return "moga-b200 0.2 (sm_100a)";
#endif
}

extern "C" moga_status moga_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return moga::fail(MOGA_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  int code = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&code, moga::g_device_error, sizeof(int));
  if (e != cudaSuccess) return moga::fail(MOGA_ERR_CUDA, "read device error word: %s", cudaGetErrorString(e));
  if (code != 0) {
    e = cudaMemcpyToSymbol(moga::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return moga::fail(MOGA_ERR_CUDA, "clear device error word: %s", cudaGetErrorString(e));
    return moga::fail(static_cast<moga_status>(code), "device reported error code %d", code);
  }
  return MOGA_OK;
}
