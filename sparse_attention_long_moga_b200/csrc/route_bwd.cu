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
// Three kernels, deterministic (every sum in a fixed order):
//   route_dr_kernel    one thread per token: dr[t] (padded to MP floats) into
//                      the workspace, and per-block sums of dr for dbias
//   route_bwd_kernel   grid (token blocks, column slices), C = 32 / MP columns
//                      per thread with W_r[k][:] in registers; streams its
//                      tokens, reading x with C-wide vector loads, writing dx
//                      (fp32, C-wide stores) and accumulating x[t][k] dr[t][:]
//                      for dW_r.  The dr row of a token is the same address
//                      for every thread (a broadcast load).  HBM-bound: one
//                      read of x and one fp32 write of dx.
//   route_bwd_reduce   adds the per-block partials of dW_r (and of dbias) in a
//                      fixed order
#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"

namespace moga {
namespace route_bwd_detail {

constexpr long long kTimeoutCycles = kWaitLimitCycles;

constexpr int kDrThreads = 256;   // route_dr_kernel: tokens per block
constexpr int kThreads = 128;     // route_bwd_kernel: threads per block
constexpr int kMaxBlocks = 512;   // token blocks (bounds the dW_r partials)
constexpr int kMinTokens = 128;   // tokens per block at least (amortises the partial write)

inline int mp_of(int M) { return M <= 8 ? 8 : (M <= 16 ? 16 : 32); }
inline int token_blocks(int64_t N) {
  return (int)std::min<int64_t>(kMaxBlocks, (N + kMinTokens - 1) / kMinTokens);
}
inline int tokens_per_block(int64_t N) {
  const int nb = token_blocks(N);
  return (int)((N + nb - 1) / nb);
}
inline int dr_blocks(int64_t N) { return (int)((N + kDrThreads - 1) / kDrThreads); }
inline size_t ws_align(size_t x) { return (x + 255) / 256 * 256; }
// workspace: dr [N][MP] | dbias partials [dr_blocks][M] | dW_r partials [nb][d][M]
inline size_t ws_dr_bytes(int64_t N, int M) { return ws_align((size_t)N * mp_of(M) * 4); }
inline size_t ws_pb_bytes(int64_t N, int M) { return ws_align((size_t)dr_blocks(N) * M * 4); }
inline size_t ws_bytes_needed(int64_t N, int d, int M) {
  return ws_dr_bytes(N, M) + ws_pb_bytes(N, M) + ws_align((size_t)token_blocks(N) * d * M * 4);
}

template <int MP>
__global__ void __launch_bounds__(kDrThreads)
route_dr_kernel(int N, int M, const int32_t* __restrict__ g, const float* __restrict__ probs,
                const float* __restrict__ dgate, const int32_t* __restrict__ counts, float loss_coef,
                float* __restrict__ dr, float* __restrict__ part_b) {
  __shared__ float floss[MP];   // dloss * alpha * M * F_m / N
  __shared__ float wsum[kDrThreads / 32][MP];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < MP) floss[tid] = tid < M ? loss_coef * (float)__ldg(counts + tid) : 0.f;
  __syncthreads();
  const int t = blockIdx.x * kDrThreads + tid;
  float r[MP];
  if (t < N) {
    const int gt = __ldg(g + t);
    const float dg = __ldg(dgate + t);
    float pr[MP], u[MP], dot = 0.f;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      pr[m] = m < M ? __ldg(probs + (size_t)t * M + m) : 0.f;
      u[m] = floss[m] + (m == gt ? dg : 0.f);
      dot = fmaf(u[m], pr[m], dot);
    }
#pragma unroll
    for (int m = 0; m < MP; ++m) r[m] = pr[m] * (u[m] - dot);
    float4* dst = reinterpret_cast<float4*>(dr + (size_t)t * MP);
#pragma unroll
    for (int m4 = 0; m4 < MP / 4; ++m4) dst[m4] = make_float4(r[4 * m4], r[4 * m4 + 1], r[4 * m4 + 2], r[4 * m4 + 3]);
  } else {
#pragma unroll
    for (int m = 0; m < MP; ++m) r[m] = 0.f;
  }
  // block sum of dr for dbias: warp tree, then the warps in order
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    float v = r[m];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    if (lane == 0) wsum[warp][m] = v;
  }
  __syncthreads();
  if (tid < M) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kDrThreads / 32; ++w) acc += wsum[w][tid];
    part_b[blockIdx.x * M + tid] = acc;
  }
}

// Shared-memory layout of route_bwd_kernel: a ring of stages, each holding the
// CTA's column slice of kTok token rows of x and those tokens' dr rows.
template <typename T, int MP>
struct Ring {
  static constexpr int kC = 32 / MP;                        // columns per thread
  static constexpr int kCols = kThreads * kC;               // columns per CTA
  static constexpr int kRowBytes = kCols * (int)sizeof(T);  // one token's slice of x
  static constexpr int kTok = 8;                            // tokens per stage
  static constexpr int kStages = std::max(2, std::min(16, 65536 / (kTok * kRowBytes)));
  static constexpr int kX = 0;
  static constexpr int kDr = kX + kStages * kTok * kRowBytes;
  static constexpr int kBar = kDr + kStages * kTok * MP * 4;   // full[kStages], empty[kStages]
  static constexpr int kMisc = kBar + 16 * kStages;
  static constexpr int kBytes = kMisc + 16;
};

__device__ __forceinline__ void cols_from_smem(const __nv_bfloat16* p, float* v, int c) {
  if (c == 4) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
  } else if (c == 2) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(p);
    v[0] = __low2float(a); v[1] = __high2float(a);
  } else {
    v[0] = __bfloat162float(*p);
  }
}
__device__ __forceinline__ void cols_from_smem(const float* p, float* v, int c) {
  if (c == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else if (c == 2) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    v[0] = a.x; v[1] = a.y;
  } else {
    v[0] = *p;
  }
}
template <int C>
__device__ __forceinline__ void store_cols(float* p, const float* v) {
  if constexpr (C == 4) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  } else if constexpr (C == 2) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
  } else {
    __stcs(p, v[0]);
  }
}
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

// grid (token blocks, column slices of Ring::kCols), kThreads compute threads
// (warps 0-3) + one producer warp.  The producer streams the block's tokens
// through the ring with bulk copies (one per token row slice, one for the dr
// rows of the stage), so the bytes in flight do not depend on registers.
template <typename T, int MP>
__global__ void __launch_bounds__(kThreads + 32)
route_bwd_kernel(const T* __restrict__ x, const T* __restrict__ w_r, int N, int d, int M, int tpb,
                 const float* __restrict__ dr, float* __restrict__ dx, float* __restrict__ part_w,
                 long long timeout) {
  using R = Ring<T, MP>;
  constexpr int C = R::kC;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = tc::smem_u32(smem);
  auto full = [&](int s) { return sbase + R::kBar + 8u * (uint32_t)s; };
  auto empty = [&](int s) { return sbase + R::kBar + 8u * (uint32_t)(R::kStages + s); };
  volatile int* abort_flag = reinterpret_cast<int*>(smem + R::kMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_base = blockIdx.y * R::kCols;
  const int ncols = min(R::kCols, d - k_base);   // a multiple of 8 (d is)
  const int t0 = blockIdx.x * tpb, t1 = min(N, t0 + tpb);
  const int n_chunks = t1 > t0 ? (t1 - t0 + R::kTok - 1) / R::kTok : 0;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < R::kStages; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), kThreads / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kThreads / 32) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int last[R::kStages];
      for (int s = 0; s < R::kStages; ++s) last[s] = -1;
      const uint32_t row_bytes = (uint32_t)ncols * (uint32_t)sizeof(T);
      for (int j = 0; j < n_chunks; ++j) {
        const int s = j % R::kStages;
        if (!tc::mbar_wait(empty(s), ((j / R::kStages) & 1) ^ 1, abort_flag, timeout)) break;
        const int tb = t0 + j * R::kTok, nt = min(R::kTok, t1 - tb);
        tc::mbar_arrive_expect_tx(full(s), (uint32_t)nt * (row_bytes + MP * 4));
        for (int i = 0; i < nt; ++i)
          tc::bulk_load(sbase + R::kX + (uint32_t)((s * R::kTok + i) * R::kRowBytes),
                        x + (size_t)(tb + i) * d + k_base, row_bytes, full(s));
        tc::bulk_load(sbase + R::kDr + (uint32_t)(s * R::kTok * MP * 4), dr + (size_t)tb * MP,
                      (uint32_t)(nt * MP * 4), full(s));
        last[s] = j;
      }
      for (int s = 0; s < R::kStages; ++s)
        if (last[s] >= 0) tc::mbar_drain(full(s), (last[s] / R::kStages) & 1, timeout);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------------------------ compute
  const int kl = threadIdx.x * C;   // this thread's columns within the slice
  const bool active = kl < ncols;
  const int k0 = k_base + kl;
  float w[C][MP], acc[C][MP];
#pragma unroll
  for (int c = 0; c < C; ++c)
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      w[c][m] = (active && m < M) ? to_f32(w_r[(size_t)(k0 + c) * M + m]) : 0.f;
      acc[c][m] = 0.f;
    }
  for (int j = 0; j < n_chunks; ++j) {
    const int s = j % R::kStages;
    if (!__all_sync(0xffffffffu, tc::mbar_wait(full(s), (j / R::kStages) & 1, abort_flag, timeout))) break;
    const int tb = t0 + j * R::kTok, nt = min(R::kTok, t1 - tb);
    const T* xs = reinterpret_cast<const T*>(smem + R::kX + (s * R::kTok) * R::kRowBytes) + kl;
    const float4* drs = reinterpret_cast<const float4*>(smem + R::kDr + s * R::kTok * MP * 4);
    if (active) {
#pragma unroll 2
      for (int i = 0; i < nt; ++i) {
        float xv[C], r[MP];
        cols_from_smem(xs + i * (R::kRowBytes / (int)sizeof(T)), xv, C);
#pragma unroll
        for (int m4 = 0; m4 < MP / 4; ++m4) {
          const float4 q = drs[i * (MP / 4) + m4];
          r[4 * m4] = q.x; r[4 * m4 + 1] = q.y; r[4 * m4 + 2] = q.z; r[4 * m4 + 3] = q.w;
        }
        float o[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
          float sum = 0.f;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            sum = fmaf(r[m], w[c][m], sum);
            acc[c][m] = fmaf(xv[c], r[m], acc[c][m]);
          }
          o[c] = sum;
        }
        store_cols<C>(dx + (size_t)(tb + i) * d + k0, o);
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(empty(s));
  }
  if (active)
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
      for (int m = 0; m < MP; ++m)
        if (m < M) part_w[((size_t)blockIdx.x * d + k0 + c) * M + m] = acc[c][m];
}

// out[i] = sum over b of part[b][i], b < nrows: dW_r from the token blocks'
// partials, dbias from the dr blocks'.  Block (32 x 8): lane x owns column i,
// row y sums the partials b = y, y + 8, ... (four independent chains), then
// the eight row sums are added in row order.  Fixed order throughout, so the
// result is deterministic.
constexpr int kRedRows = 8;
__global__ void __launch_bounds__(32 * kRedRows)
route_bwd_reduce(const float* __restrict__ part, int nrows, int ncols, float* __restrict__ out) {
  __shared__ float rows[kRedRows][32];
  const int x = threadIdx.x, y = threadIdx.y;
  const int i = blockIdx.x * 32 + x;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (i < ncols) {
    int b = y;
    for (; b + 3 * kRedRows < nrows; b += 4 * kRedRows)
#pragma unroll
      for (int j = 0; j < 4; ++j) a[j] += __ldg(part + (size_t)(b + j * kRedRows) * ncols + i);
    for (; b < nrows; b += kRedRows) a[0] += __ldg(part + (size_t)b * ncols + i);
  }
  rows[y][x] = (a[0] + a[1]) + (a[2] + a[3]);
  __syncthreads();
  if (y == 0 && i < ncols) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < kRedRows; ++r) s += rows[r][x];
    out[i] = s;
  }
}

template <typename T, int MP>
static moga_status launch_mp(const void* x, const void* w_r, int N, int d, int M, const int32_t* g,
                             const float* probs, const float* dgate, const int32_t* counts, float loss_coef, float* dx,
                             float* dr, float* part_b, float* part_w, cudaStream_t s) {
  route_dr_kernel<MP><<<dr_blocks(N), kDrThreads, 0, s>>>(N, M, g, probs, dgate, counts, loss_coef, dr, part_b);
  moga_status st = check_launch("moga_route_bwd/dr");
  if (st != MOGA_OK) return st;
  using R = Ring<T, MP>;
  const cudaError_t e = cudaFuncSetAttribute(route_bwd_kernel<T, MP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             R::kBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_route_bwd: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  const dim3 grid(token_blocks(N), ceil_div(d, R::kCols));
  route_bwd_kernel<T, MP><<<grid, kThreads + 32, R::kBytes, s>>>(static_cast<const T*>(x), static_cast<const T*>(w_r),
                                                                  N, d, M, tokens_per_block(N), dr, dx, part_w,
                                                                  kTimeoutCycles);
  return check_launch("moga_route_bwd");
}

template <typename T>
static moga_status launch_t(const void* x, const void* w_r, int N, int d, int M, const int32_t* g, const float* probs,
                            const float* dgate, const int32_t* counts, float loss_coef, float* dx, float* dr,
                            float* part_b, float* part_w, cudaStream_t s) {
  if (M <= 8) return launch_mp<T, 8>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, dr, part_b, part_w, s);
  if (M <= 16) return launch_mp<T, 16>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, dr, part_b, part_w, s);
  return launch_mp<T, 32>(x, w_r, N, d, M, g, probs, dgate, counts, loss_coef, dx, dr, part_b, part_w, s);
}

}  // namespace route_bwd_detail
}  // namespace moga

extern "C" size_t moga_route_bwd_ws_bytes(int64_t N, int32_t d, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32 || d <= 0 || d % 8 != 0) return 0;
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
  if (d <= 0 || d % 8 != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: d=%d must be a positive multiple of 8", d);
  if (dt != MOGA_F32 && dt != MOGA_BF16) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: bad dtype %d", (int)dt);
  if (ws_bytes < ws_bytes_needed(N, d, M))
    return fail(MOGA_ERR_WORKSPACE, "moga_route_bwd: workspace %zu < %zu bytes", ws_bytes, ws_bytes_needed(N, d, M));
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: workspace not 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dx)) & 15)
    return fail(MOGA_ERR_INVALID_ARG, "moga_route_bwd: x and dx must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  float* dr = reinterpret_cast<float*>(w8);
  float* part_b = reinterpret_cast<float*>(w8 + ws_dr_bytes(N, M));
  float* part_w = reinterpret_cast<float*>(w8 + ws_dr_bytes(N, M) + ws_pb_bytes(N, M));
  // d(alpha M sum_i F_i P_i) / d p_t[m] = alpha M F_m / N,  F_m = counts[m] / N
  const float loss_coef = (float)((double)dloss * alpha * M / ((double)N * (double)N));
  moga_status st = dt == MOGA_BF16
                       ? launch_t<__nv_bfloat16>(x, w_r, (int)N, d, M, group_id, probs, dgate, counts, loss_coef, dx,
                                                 dr, part_b, part_w, s)
                       : launch_t<float>(x, w_r, (int)N, d, M, group_id, probs, dgate, counts, loss_coef, dx, dr,
                                         part_b, part_w, s);
  if (st != MOGA_OK) return st;
  const int dm = d * M;
  route_bwd_reduce<<<ceil_div(dm, 32), dim3(32, kRedRows), 0, s>>>(part_w, token_blocks(N), dm, dw_r);
  if (dbias != nullptr) route_bwd_reduce<<<1, dim3(32, kRedRows), 0, s>>>(part_b, dr_blocks(N), M, dbias);
  return check_launch("moga_route_bwd/reduce");
}
