// Backward of the router (MoGA note, key designs 1 and 3: the gate
// p(g(x)|x) scales the MoGA output and the balancing loss reads the mean
// routing probabilities; g(x) = argmax and the counts F_i carry no gradient).
//
// Per token t with p = softmax(r) (saved by the training forward) and
//   u[m] = dgate[t] * [m == g_t] + dloss * alpha * M * F_m / N,  F_m = counts[m] / N,
//   dr[m] = p[m] * (u[m] - sum_i u_i p_i),
// the gradients are  dx[t] = dr W_r^T,  dW_r = sum_t x_t^T dr_t,
// dbias = sum_t dr_t.
//
// route_bwd_kernel: grid (token blocks, 256-column slices of d), one thread
// per column k of x: it keeps W_r[k][:] in registers, walks the block's
// tokens in chunks of 32 (dr of the chunk computed once into shared memory),
// writes dx[t][k] (coalesced over k) and accumulates x[t][k] * dr[t][:] for
// dW_r.  Per-block partial sums of dW_r (and of dr for the bias) go to the
// workspace and route_bwd_reduce adds them in a fixed order.  HBM-bound:
// one read of x and one fp32 write of dx.
#include <algorithm>

#include "common.cuh"

namespace moga {
namespace route_bwd_detail {

constexpr int kThreads = 256;
constexpr int kMaxBlocks = 64;   // token blocks (bounds the partial-sum workspace)

inline int token_blocks(int64_t N) { return (int)std::min<int64_t>(kMaxBlocks, (N + 31) / 32); }
inline int tokens_per_block(int64_t N) {
  const int nb = token_blocks(N);
  return (int)(((N + nb - 1) / nb + 31) / 32 * 32);
}
inline size_t ws_align(size_t x) { return (x + 255) / 256 * 256; }
inline size_t ws_bytes_needed(int64_t N, int d, int M) {
  const int nb = token_blocks(N);
  return ws_align((size_t)nb * d * M * 4) + ws_align((size_t)nb * M * 4);
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

template <typename T, int MP>
__global__ void __launch_bounds__(kThreads)
route_bwd_kernel(const T* __restrict__ x, const T* __restrict__ w_r, int N, int d, int M, int tpb,
                 const int32_t* __restrict__ g, const float* __restrict__ probs, const float* __restrict__ dgate,
                 const int32_t* __restrict__ counts, float loss_coef, float* __restrict__ dx,
                 float* __restrict__ part_w, float* __restrict__ part_b) {
  __shared__ float dr[32][MP];
  __shared__ float floss[MP];   // dloss * alpha * M * F_m / N
  const int tid = threadIdx.x;
  const int k = blockIdx.y * kThreads + tid;
  const bool col = k < d;
  if (tid < MP) floss[tid] = tid < M ? loss_coef * (float)__ldg(counts + tid) : 0.f;
  float w[MP], acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    w[m] = (col && m < M) ? to_f32(w_r[(size_t)k * M + m]) : 0.f;
    acc[m] = 0.f;
  }
  float bsum = 0.f;   // thread m < M: sum of dr[:, m] over the block (bias)
  const int t0 = blockIdx.x * tpb, t1 = min(N, t0 + tpb);
  __syncthreads();
  for (int c0 = t0; c0 < t1; c0 += 32) {
    if (tid < 32) {
      const int t = c0 + tid;
      float pr[MP], u[MP];
      float dot = 0.f;
      if (t < t1) {
        const int gt = __ldg(g + t);
        const float dg = __ldg(dgate + t);
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          pr[m] = m < M ? __ldg(probs + (size_t)t * M + m) : 0.f;
          u[m] = floss[m] + (m == gt ? dg : 0.f);
          dot = fmaf(u[m], pr[m], dot);
        }
      } else {
#pragma unroll
        for (int m = 0; m < MP; ++m) pr[m] = u[m] = 0.f;
      }
#pragma unroll
      for (int m = 0; m < MP; ++m) dr[tid][m] = pr[m] * (u[m] - dot);
    }
    __syncthreads();
    if (blockIdx.y == 0 && tid < M) {
      const int n = min(32, t1 - c0);
      for (int tt = 0; tt < n; ++tt) bsum += dr[tt][tid];
    }
    if (col) {
      const int n = min(32, t1 - c0);
      for (int tt = 0; tt < n; ++tt) {
        const int t = c0 + tt;
        const float xv = to_f32(x[(size_t)t * d + k]);
        float dxv = 0.f;
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          acc[m] = fmaf(xv, dr[tt][m], acc[m]);
          dxv = fmaf(dr[tt][m], w[m], dxv);
        }
        dx[(size_t)t * d + k] = dxv;
      }
    }
    __syncthreads();
  }
  if (col)
#pragma unroll
    for (int m = 0; m < MP; ++m)
      if (m < M) part_w[((size_t)blockIdx.x * d + k) * M + m] = acc[m];
  if (blockIdx.y == 0 && tid < M) part_b[blockIdx.x * M + tid] = bsum;
}

// dw_r[k][m] = sum over token blocks in order; dbias likewise
__global__ void __launch_bounds__(256)
route_bwd_reduce(const float* __restrict__ part_w, const float* __restrict__ part_b, int nb, int dm, int M,
                 float* __restrict__ dw_r, float* __restrict__ dbias) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i < dm) {
    float s = 0.f;
    for (int b = 0; b < nb; ++b) s += part_w[(size_t)b * dm + i];
    dw_r[i] = s;
  }
  if (dbias != nullptr && blockIdx.x == 0 && threadIdx.x < M) {
    float s = 0.f;
    for (int b = 0; b < nb; ++b) s += part_b[b * M + threadIdx.x];
    dbias[threadIdx.x] = s;
  }
}

template <typename T, int MP>
static moga_status launch_mp(const void* x, const void* w_r, int N, int d, int M, const int32_t* g,
                             const float* probs, const float* dgate, const int32_t* counts, float loss_coef, float* dx,
                             float* part_w, float* part_b, cudaStream_t s) {
  const dim3 grid(token_blocks(N), ceil_div(d, kThreads));
  route_bwd_kernel<T, MP><<<grid, kThreads, 0, s>>>(static_cast<const T*>(x), static_cast<const T*>(w_r), N, d, M,
                                                     tokens_per_block(N), g, probs, dgate, counts, loss_coef, dx,
                                                     part_w, part_b);
  return check_launch("moga_route_bwd");
}

template <typename T>
static moga_status launch_t(const void* x, const void* w_r, int N, int d, int M, const int32_t* g, const float* probs,
                            const float* dgate, const int32_t* counts, float loss_coef, float* dx, float* part_w,
                            float* part_b, cudaStream_t s) {
  if (M <= 8) return launch_mp<T, 8>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, part_w, part_b, s);
  if (M <= 16) return launch_mp<T, 16>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, part_w, part_b, s);
  return launch_mp<T, 32>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, part_w, part_b, s);
}

}  // namespace route_bwd_detail
}  // namespace moga

extern "C" size_t moga_route_bwd_ws_bytes(int64_t N, int32_t d, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32 || d <= 0) return 0;
  return moga::route_bwd_detail::ws_bytes_needed(N, d, M);
}

extern "C" moga_status moga_route_bwd(const void* x, const void* w_r, moga_dtype dt, int64_t N, int32_t d, int32_t M,
                                      const int32_t* group_id, const float* probs, const float* dgate,
                                      const int32_t* counts, float alpha, float dloss, float* dx, float* dw_r,
                                      float* dbias, void* ws, size_t ws_bytes, void* stream) {
  using namespace moga;
  using namespace moga::route_bwd_detail;
  if (!x || !w_r || !group_id || !probs || !dgate || !counts || !dx || !dw_r || !ws)
    return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: M=%d not in [1, 32]", M);
  if (d <= 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: d=%d", d);
  if (dt != MOGA_F32 && dt != MOGA_BF16) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: bad dtype %d", (int)dt);
  if (ws_bytes < ws_bytes_needed(N, d, M))
    return fail(MOGA_ERR_WORKSPACE, "moga_route_bwd: workspace %zu < %zu bytes", ws_bytes, ws_bytes_needed(N, d, M));
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: workspace not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nb = token_blocks(N);
  float* part_w = static_cast<float*>(ws);
  float* part_b = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_align((size_t)nb * d * M * 4));
  // d(alpha M sum_i F_i P_i) / d p_t[m] = alpha M F_m / N,  F_m = counts[m] / N
  const float loss_coef = (float)((double)dloss * alpha * M / ((double)N * (double)N));
  moga_status st = dt == MOGA_BF16
                       ? launch_t<__nv_bfloat16>(x, w_r, (int)N, d, M, group_id, probs, dgate, counts, loss_coef, dx,
                                                 part_w, part_b, s)
                       : launch_t<float>(x, w_r, (int)N, d, M, group_id, probs, dgate, counts, loss_coef, dx, part_w,
                                         part_b, s);
  if (st != MOGA_OK) return st;
  const int dm = d * M;
  route_bwd_reduce<<<ceil_div(dm, 256), 256, 0, s>>>(part_w, part_b, nb, dm, M, dw_r, dbias);
  return check_launch("moga_route_bwd/reduce");
}
