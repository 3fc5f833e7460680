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

// One block of 1024 threads.  The partials form a [rows][M] fp32 array; with
// S = M * floor(1024 / M), thread t < S sums the elements t, t + S, t + 2S, ...
// (all of group t % M) in fp64; the per-thread sums are then folded per group
// in a fixed order (32 strided slices, then the 32 slice sums), so the result
// does not depend on scheduling.
__global__ void __launch_bounds__(1024)
balance_loss_kernel(const int32_t* __restrict__ counts, const float* __restrict__ partial, int rows, int N,
                    int M, int B, float alpha, double* __restrict__ loss) {
  __shared__ double part[1024];
  __shared__ double slice[32][32];
  const int t = threadIdx.x;
  const int R = 1024 / M;            // per-thread sums per group
  const int S = R * M;
  const int64_t n = (int64_t)rows * M;
  double s = 0.0;
  if (t < S) {
    double s1 = 0.0;
    int64_t i = t;
    for (; i + S < n; i += 2 * (int64_t)S) {
      s += (double)partial[i];
      s1 += (double)partial[i + S];
    }
    if (i < n) s += (double)partial[i];
    s += s1;
  }
  part[t] = s;
  __syncthreads();
  // slice j of group m: per-thread sums r = j, j + 32, ... (thread r * M + m)
  const int m = t & 31, j = t >> 5;
  if (m < M) {
    double a = 0.0;
    for (int r = j; r < R; r += 32) a += part[r * M + m];
    slice[j][m] = a;
  }
  __syncthreads();
  if (t < 32) {
    double fp = 0.0;
    if (t < M) {
      double tot = 0.0;
      for (int jj = 0; jj < 32; ++jj) tot += slice[jj][t];
      int cnt = 0;   // tokens of group t over the B videos of a batch
      for (int b = 0; b < B; ++b) cnt += counts[b * M + t];
      fp = ((double)cnt / (double)N) * (tot / (double)N);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) fp += __shfl_xor_sync(0xffffffffu, fp, off);
    if (t == 0) *loss = (double)alpha * (double)M * fp;
  }
}

// Training forward: the three branch outputs kept apart (for the backward);
// out = bf16_rn((a + b) + c) / 3), 4 elements per thread per step.
__global__ void __launch_bounds__(kThreads)
mean3_sep_kernel(const float4* __restrict__ a, const float4* __restrict__ b, const float4* __restrict__ c,
                 uint2* __restrict__ out, int64_t n4) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n4; i += stride) {
    const float4 x = __ldcs(a + i), y = __ldcs(b + i), z = __ldcs(c + i);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(((x.x + y.x) + z.x) / 3.0f, ((x.y + y.y) + z.y) / 3.0f);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(((x.z + y.z) + z.z) / 3.0f, ((x.w + y.w) + z.w) / 3.0f);
    __stcs(out + i, make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi)));
  }
}

}  // namespace mean_detail

int route_partial_rows(int64_t N);

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

extern "C" moga_status visual_attn_mean3(const float* o_moga, const float* o_win, const float* o_frame,
                                         int64_t n_elems, void* out, void* stream) {
  using namespace moga;
  using namespace moga::mean_detail;
  if (!o_moga || !o_win || !o_frame || !out) return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean3: null pointer");
  if (n_elems <= 0 || n_elems % 4) return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean3: n_elems=%lld", (long long)n_elems);
  const uintptr_t al = reinterpret_cast<uintptr_t>(o_moga) | reinterpret_cast<uintptr_t>(o_win) |
                       reinterpret_cast<uintptr_t>(o_frame) | reinterpret_cast<uintptr_t>(out);
  if (al & 15) return fail(MOGA_ERR_INVALID_ARG, "visual_attn_mean3: pointers must be 16-byte aligned");
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n4 = n_elems / 4;
  const int blocks = (int)std::min<int64_t>(ceil_div((int)std::min<int64_t>(n4, INT32_MAX / 2), kThreads),
                                            (int64_t)sms * 16);
  mean3_sep_kernel<<<blocks, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(o_moga), reinterpret_cast<const float4*>(o_win),
      reinterpret_cast<const float4*>(o_frame), static_cast<uint2*>(out), n4);
  return check_launch("visual_attn_mean3");
}

extern "C" moga_status moga_balance_loss(const int32_t* counts, const void* route_ws, int64_t N, int32_t M,
                                         float alpha, double* loss, void* stream) {
  using namespace moga;
  if (!counts || !route_ws || !loss) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss: M=%d not in [1, 32]", M);
  mean_detail::balance_loss_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, static_cast<const float*>(route_ws), route_partial_rows(N), (int)N, M, 1, alpha, loss);
  return check_launch("moga_balance_loss");
}

extern "C" moga_status moga_balance_loss_batched(const int32_t* counts, int32_t B, const void* route_ws,
                                                 int64_t N, int32_t M, float alpha, double* loss, void* stream) {
  using namespace moga;
  if (!counts || !route_ws || !loss) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_batched: null pointer");
  if (N <= 0 || N > INT32_MAX || B < 1 || N % B != 0)
    return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_batched: N=%lld, B=%d", (long long)N, B);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_batched: M=%d not in [1, 32]", M);
  mean_detail::balance_loss_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, static_cast<const float*>(route_ws), route_partial_rows(N), (int)N, M, B, alpha, loss);
  return check_launch("moga_balance_loss_batched");
}

// One rank's share of L_gb under sequence parallelism: F_i from the counts of
// all N tokens (every rank holds them after the routing all-gather), P_i
// summed over this rank's n_local tokens only (its router workspace), both
// normalised by N.  The sum of the ranks' shares is L_gb.
extern "C" moga_status moga_balance_loss_part(const int32_t* counts, const void* route_ws, int64_t n_local,
                                              int64_t N, int32_t M, float alpha, double* loss, void* stream) {
  using namespace moga;
  if (!counts || !route_ws || !loss) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_part: null pointer");
  if (N <= 0 || N > INT32_MAX || n_local <= 0 || n_local > N)
    return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_part: n_local=%lld, N=%lld", (long long)n_local,
                (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_balance_loss_part: M=%d not in [1, 32]", M);
  mean_detail::balance_loss_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, static_cast<const float*>(route_ws), route_partial_rows(n_local), (int)N, M, 1, alpha, loss);
  return check_launch("moga_balance_loss_part");
}
