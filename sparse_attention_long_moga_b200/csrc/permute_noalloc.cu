// moga_permute_noalloc: the stable group permute with its scratch held in a
// fixed device array owned by the library, for callers that cannot allocate.
//
// moga_permute() takes a caller-provided workspace.  Some callers have no way
// to provide one at the moment they run the layer: code executing inside a
// host callback or a plugin of another runtime whose memory is owned by that
// runtime, programs built on a static, pre-planned device-memory budget in
// which cudaMalloc during inference is forbidden (a cudaMalloc there may also
// synchronise the device), and callers that cannot reach any allocator
// (C callers without torch).  This entry point needs nothing but the inputs
// and outputs: the tile histograms and tile offsets live in
// g_permute_scratch below.
//
// Limits and sharing rules:
//   * N <= kNoAllocMaxTokens (4,194,304 tokens) and 1 <= M <= 32;
//     larger N is rejected with MOGA_ERR_WORKSPACE before any launch.
//   * The array (512 KiB) exists on every GPU that loads the library, for the
//     life of the process.
//   * All calls on a device share the one array and it keeps the previous
//     call's contents.  Every entry this call reads is written by this call
//     first (the histogram kernel writes all tile x group counts, the scan
//     writes all offsets), so nothing has to start at zero.  Two calls whose
//     kernels overlap on the GPU (different streams, or different host
//     threads) race on the array: serialise them.
//   * The first call on a device looks up the array's device address with
//     cudaGetSymbolAddress (with that device current) and caches it; make
//     that first call before any stream capture.  The cache lives as long as
//     the process and is never refreshed: after cudaDeviceReset() (or any
//     other teardown of the primary context) the cached address is stale, so
//     the entry point must not be called again in that process.
#include <mutex>

#include "common.cuh"

namespace moga {
namespace noalloc_detail {

constexpr int64_t kNoAllocMaxTokens = 4194304;
constexpr int kMaxTiles = (int)(kNoAllocMaxTokens / permute_detail::kTile);   // 2048
constexpr int kScratchInts = 2 * kMaxTiles * 32;                                // hist + offsets

// File-scope scratch.  In host code this name is only a stand-in: its device
// address comes from cudaGetSymbolAddress.
static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
static int32_t* g_scratch_ptr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

static moga_status scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_permute_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(MOGA_ERR_UNSUPPORTED, "moga_permute_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess || !p)
      return fail(MOGA_ERR_CUDA, "moga_permute_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOGA_OK;
}

}  // namespace noalloc_detail
}  // namespace moga

extern "C" moga_status moga_permute_noalloc(const int32_t* group_id, int64_t N, int32_t M, int32_t* perm,
                                            int32_t* cu_seqlens, int32_t* counts, int32_t* max_seqlen,
                                            void* stream) {
  using namespace moga;
  using namespace moga::permute_detail;
  using namespace moga::noalloc_detail;
  if (!group_id || !perm || !cu_seqlens || !counts || !max_seqlen)
    return fail(MOGA_ERR_INVALID_ARG, "moga_permute_noalloc: null pointer");
  if (N <= 0) return fail(MOGA_ERR_INVALID_ARG, "moga_permute_noalloc: N=%lld", (long long)N);
  if (N > kNoAllocMaxTokens)
    return fail(MOGA_ERR_WORKSPACE, "moga_permute_noalloc: N=%lld exceeds the built-in scratch limit of %lld tokens",
                (long long)N, (long long)kNoAllocMaxTokens);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_permute_noalloc: M=%d not in [1, 32]", M);
  int32_t* scratch = nullptr;
  moga_status st = scratch_for_current_device(&scratch);
  if (st != MOGA_OK) return st;
  return run_permute<32>(group_id, (int)N, M, (int)N, M, perm, cu_seqlens, counts, max_seqlen, scratch,
                         static_cast<cudaStream_t>(stream));
}
