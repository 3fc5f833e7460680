// Three-way mean (fp32 accumulator -> bf16 output) and the group-balancing loss.
//
// Mean: each token receives one dynamic (MoGA) and two static (window group,
// frame) outputs and the layer returns their average (MoGA note, flowchart
// and key design 4).  The accumulator already holds the sum of the three.
// Loss: L_gb = alpha * M * sum_i F_i * P_i (MoGA note, key design 3), with
// F_i = counts_i / N and P_i the mean of p(i|x) over all N tokens.
#include "common.cuh"

namespace moga {
namespace mean_detail {

constexpr int kThreads = 256;

// 8 elements per thread per step: two 16-byte loads, one 16-byte store.
__global__ void __launch_bounds__(kThreads)
mean3_kernel(const float4* __restrict__ acc, uint4* __restrict__ out, int64_t n8) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldcs(acc + 2 * i);
    const float4 b = __ldcs(acc + 2 * i + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat16 lo = __float2bfloat16_rn(v[2 * j] / 3.0f);
      const __nv_bfloat16 hi = __float2bfloat16_rn(v[2 * j + 1] / 3.0f);
      w[j] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    __stcs(out + i, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

__global__ void mean3_tail_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ out,
                                  int64_t start, int64_t n) {
  const int64_t i = start + threadIdx.x;
  if (i < n) out[i] = __float2bfloat16_rn(acc[i] / 3.0f);
}

// One block of 8 warps: warp w sums the route partials of blocks w, w+8, ...
// in fp64 (lane = group), then the warps are combined in a fixed order.
__global__ void __launch_bounds__(256)
balance_loss_kernel(const int32_t* __restrict__ counts, const float* __restrict__ partial, int blocks, int N,
                    int M, float alpha, double* __restrict__ loss) {
  __shared__ double part[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double s = 0.0;
  if (lane < M)
    for (int b = warp; b < blocks; b += 8) s += (double)partial[(size_t)b * M + lane];
  part[warp][lane] = s;
  __syncthreads();
  if (warp == 0) {
    double fp = 0.0;
    if (lane < M) {
      double tot = 0.0;
      for (int w = 0; w < 8; ++w) tot += part[w][lane];
      fp = ((double)counts[lane] / (double)N) * (tot / (double)N);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) fp += __shfl_xor_sync(0xffffffffu, fp, off);
    if (lane == 0) *loss = (double)alpha * (double)M * fp;
  }
}

}  // namespace mean_detail

int route_blocks(int64_t N, int M);

}  // namespace moga

extern "C" moga_status visual_attn_mean(const float* o_acc, int64_t n_elems, void* out, void* stream) {
  using namespace moga;
  using namespace moga::mean_detail;
  if (!o_acc || !out) return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean: null pointer");
  if (n_elems <= 0) return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean: n_elems=%lld", (long long)n_elems);
  if ((reinterpret_cast<uintptr_t>(o_acc) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean: pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n8 = n_elems / 8;
  if (n8 > 0) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = ceil_div((int)std::min<int64_t>(n8, INT32_MAX / 2), kThreads);
    const int blocks = (int)std::min<int64_t>(want, (int64_t)sms * 16);
    mean3_kernel<<<blocks, kThreads, 0, s>>>(reinterpret_cast<const float4*>(o_acc), static_cast<uint4*>(out), n8);
    moga_status st = check_launch("visual_attn_mean");
    if (st != MOGA_OK) return st;
  }
  if (n8 * 8 < n_elems) {
    mean3_tail_kernel<<<1, 32, 0, s>>>(o_acc, static_cast<__nv_bfloat16*>(out), n8 * 8, n_elems);
    return check_launch("visual_attn_mean/tail");
  }
  return MOGA_OK;
}

extern "C" moga_status moga_balance_loss(const int32_t* counts, const void* route_ws, int64_t N, int32_t M,
                                         float alpha, double* loss, void* stream) {
  using namespace moga;
  if (!counts || !route_ws || !loss) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: M=%d not in [1, 32]", M);
  mean_detail::balance_loss_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, static_cast<const float*>(route_ws), route_blocks(N, M), (int)N, M, alpha, loss);
  return check_launch("moga_balance_loss");
}
