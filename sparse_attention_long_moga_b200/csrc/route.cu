// Router kernel: r = x . W_r (+ bias), p = softmax(r), g = argmax p, gate = p_g,
// plus per-chunk (32-token) partial sums of p(i|x) for the group-balancing loss.
//
// MoGA note (papernotes.org ICLR 2026), key design 1: a linear projection
// with softmax gating gives p(i|x); the token goes to the most probable
// group; the blog (xugj520.cn) section 2.3 sketches the same bias-free layer.
//
// Design (HBM-bound: one read of x):
//   * eight threads per token; thread s of a token reads the 16-byte chunks
//     s, s+8, s+16, ... of the row, so the eight threads of a token read 128
//     contiguous bytes per step (every sector fully used); each thread
//     serves up to 4 tokens so that each shared-memory read of W_r feeds
//     several tokens;
//   * several chunks are loaded before they are used, keeping enough bytes
//     in flight per SM to cover HBM latency;
//   * W_r is staged in shared memory as fp32 transposed to [M][k], so the
//     eight threads of a token read adjacent 32-byte pieces and the 4 tokens
//     of a warp share them (broadcast);
//     d is processed in chunks that fit the shared-memory budget;
//   * logits accumulate in fp32 registers, the eight partial sums of a token
//     are combined with three shuffles.
#include "common.cuh"
#include "route_tc.cu"

namespace moga {
namespace route_detail {

constexpr int kThreads = 256;
constexpr int kSub = 8;                       // threads per token
constexpr int kTokens = kThreads / kSub;      // tokens per block
constexpr int kSmemBudget = 64 * 1024;        // fp32 W_r chunk
constexpr int kUnroll = 4;                    // 16-byte chunks loaded ahead per thread

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  // 8 elements = 16 bytes
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* f) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Vec<float> {
  static __device__ __forceinline__ void load(const float* p, float* f) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

// TT tokens per thread (strided by 4 inside the warp's 16): every W_r value
// read from shared memory feeds TT tokens, which keeps the shared-memory
// traffic per byte of x below the HBM rate.
template <int MP>
struct Tokens {
  static constexpr int value = 4;   // 128 tokens per block: 8 partial rows per 128 tokens
};

template <typename T, int MP>
__global__ void __launch_bounds__(kThreads)
route_kernel(const T* __restrict__ x, const T* __restrict__ w_r, const float* __restrict__ bias,
             int N, int d, int M, int KC,
             int32_t* __restrict__ group_id, float* __restrict__ gate_prob,
             float* __restrict__ psum_partial, float* __restrict__ probs) {
  constexpr int TT = Tokens<MP>::value;
  constexpr int U = MP <= 8 ? 2 : 1;   // 16-byte chunks of each token loaded ahead
  extern __shared__ float4 smem_f4[];
  float* ws = reinterpret_cast<float*>(smem_f4);   // [MP][KC]

  const int tid = threadIdx.x;
  const int sub = tid & (kSub - 1);
  const int lane = tid & 31, warp = tid >> 5;
  // warp w owns the 16 tokens [16w, 16w + 16) of the block's 128; thread
  // (lane / 8) of a warp's token slots takes tokens lane/8 + 4t
  const int tok0 = blockIdx.x * kTokens * TT + 16 * warp + (lane >> 3);
  const T* xrow[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const int tok = tok0 + 4 * t;
    xrow[t] = x + (size_t)(tok < N ? tok : 0) * d;
  }

  float acc[TT][MP];
#pragma unroll
  for (int t = 0; t < TT; ++t)
#pragma unroll
    for (int m = 0; m < MP; ++m) acc[t][m] = 0.f;

  for (int k0 = 0; k0 < d; k0 += KC) {
    const int kc = min(KC, d - k0);
    __syncthreads();
    // one row of W_r (M contiguous values) per thread per step; all loads of
    // a row are issued before the shared-memory stores
    for (int kk = tid; kk < kc; kk += kThreads) {
      const T* src = w_r + (size_t)(k0 + kk) * M;
      float wv[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) wv[m] = (m < M) ? to_f32(__ldg(src + m)) : 0.f;
#pragma unroll
      for (int m = 0; m < MP; ++m) ws[m * KC + kk] = wv[m];
    }
    __syncthreads();
    const int nchunk = kc / 8;   // 8-element chunks in this part of the row
    for (int c0 = sub; c0 < nchunk; c0 += kSub * U) {
      float xv[U][TT][8];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kSub;
        if (c < nchunk)
#pragma unroll
          for (int t = 0; t < TT; ++t) Vec<T>::load(xrow[t] + k0 + 8 * c, xv[u][t]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kSub;
        if (c < nchunk) {
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            const float4* wv = reinterpret_cast<const float4*>(ws + m * KC + 8 * c);
            const float4 a = wv[0], b = wv[1];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              float sacc = acc[t][m];
              sacc = fmaf(xv[u][t][0], a.x, sacc);
              sacc = fmaf(xv[u][t][1], a.y, sacc);
              sacc = fmaf(xv[u][t][2], a.z, sacc);
              sacc = fmaf(xv[u][t][3], a.w, sacc);
              sacc = fmaf(xv[u][t][4], b.x, sacc);
              sacc = fmaf(xv[u][t][5], b.y, sacc);
              sacc = fmaf(xv[u][t][6], b.z, sacc);
              sacc = fmaf(xv[u][t][7], b.w, sacc);
              acc[t][m] = sacc;
            }
          }
        }
      }
    }
  }

  float psum[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) psum[m] = 0.f;
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const int tok = tok0 + 4 * t;
    // combine the eight partial logits of the token
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      acc[t][m] += __shfl_xor_sync(0xffffffffu, acc[t][m], 1);
      acc[t][m] += __shfl_xor_sync(0xffffffffu, acc[t][m], 2);
      acc[t][m] += __shfl_xor_sync(0xffffffffu, acc[t][m], 4);
    }
    if (tok < N && sub == 0) {
      // softmax, argmax (lowest index wins a tie), gate
      float best = -INFINITY;
      int g = 0;
      float r[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        r[m] = acc[t][m] + ((bias && m < M) ? __ldg(bias + m) : 0.f);
        if (m < M && r[m] > best) { best = r[m]; g = m; }
      }
      float e[MP], z = 0.f;
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        e[m] = (m < M) ? expf(r[m] - best) : 0.f;
        z += e[m];
      }
      const float inv = 1.f / z;
#pragma unroll
      for (int m = 0; m < MP; ++m) psum[m] += e[m] * inv;
      group_id[tok] = g;
      gate_prob[tok] = inv;   // exp(r_g - max) = 1
      if (probs != nullptr)
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < M) probs[(size_t)tok * M + m] = e[m] * inv;
    }
  }

  // fixed-order sums of p(i|x) per 32-token chunk (warps 2j and 2j+1 hold
  // chunk j of the block): one partial row per chunk, the layout the loss reads
  __shared__ float red[kThreads / 32][MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    float v = psum[m];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][m] = v;
  }
  __syncthreads();
  const int chunk = blockIdx.x * 4 + (warp >> 1);
  if ((warp & 1) == 0 && lane < M && chunk * 32 < N)
    psum_partial[(size_t)chunk * M + lane] = red[warp][lane] + red[warp + 1][lane];
}

template <typename T, int MP>
moga_status launch(const void* x, const void* w_r, const float* bias, int N, int d, int M,
                   int32_t* g, float* gate, float* partial, float* probs, cudaStream_t s) {
  int KC = kSmemBudget / (MP * 4);
  KC = (KC / (8 * kSub)) * (8 * kSub);   // whole 8-element chunks for every thread of a token
  if (KC >= d) KC = d;
  const size_t smem = (size_t)KC * MP * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<T, MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_route: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  const int blocks = ceil_div(N, kTokens * Tokens<MP>::value);
  route_kernel<T, MP><<<blocks, kThreads, smem, s>>>(static_cast<const T*>(x), static_cast<const T*>(w_r),
                                                     bias, N, d, M, KC, g, gate, partial, probs);
  return check_launch("moga_route");
}

template <typename T>
moga_status dispatch(const void* x, const void* w_r, const float* bias, int N, int d, int M,
                     int32_t* g, float* gate, float* partial, float* probs, cudaStream_t s) {
  switch ((M + 3) / 4) {
    case 1: return launch<T, 4>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 2: return launch<T, 8>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 3: return launch<T, 12>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 4: return launch<T, 16>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 5: return launch<T, 20>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 6: return launch<T, 24>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    case 7: return launch<T, 28>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
    default: return launch<T, 32>(x, w_r, bias, N, d, M, g, gate, partial, probs, s);
  }
}

}  // namespace route_detail

// Rows of Σp partials in the route workspace: one per 32-token chunk (both
// the tensor-core path and the fp32 path write exactly these rows).
int route_partial_rows(int64_t N) { return ceil_div((int)N, 32); }

static size_t route_partial_bytes(int64_t N, int M) {
  return ((size_t)route_partial_rows(N) * (size_t)M * sizeof(float) + 255) / 256 * 256;
}

}  // namespace moga

extern "C" size_t moga_route_ws_bytes(int64_t N, int32_t d, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32 || d <= 0 || d % 8 != 0) return 0;
  return moga::route_partial_bytes(N, M) + moga::route_tc::wt_bytes(d);
}

namespace moga {

static moga_status route_impl(const void* x, const void* w_r, moga_dtype dt, const float* bias, int64_t N, int32_t d,
                              int32_t M, int32_t* group_id, float* gate_prob, float* probs, void* ws,
                              size_t ws_bytes, void* stream) {
  using namespace moga;
  if (!x || !w_r || !group_id || !gate_prob || !ws) return fail(MOGA_ERR_INVALID_ARG, "moga_route: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_route: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_route: M=%d not in [1, 32]", M);
  if (dt != MOGA_F32 && dt != MOGA_BF16) return fail(MOGA_ERR_INVALID_ARG, "moga_route: bad dtype %d", (int)dt);
  if (d <= 0 || d % 8 != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route: d=%d must be a positive multiple of 8", d);
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route: x not 16-byte aligned");
  const size_t need = moga_route_ws_bytes(N, d, M);
  if (ws_bytes < need) return fail(MOGA_ERR_WORKSPACE, "moga_route: workspace %zu < %zu bytes", ws_bytes, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(MOGA_ERR_INVALID_ARG, "moga_route: workspace not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* partial = static_cast<float*>(ws);
  if (dt == MOGA_BF16) {
    // tensor-core path; W_r^T scratch after the partial rows
    void* wt = static_cast<uint8_t*>(ws) + route_partial_bytes(N, M);
    return route_tc::launch(x, w_r, bias, (int)N, d, M, group_id, gate_prob, partial, probs, wt, kWaitLimitCycles, s);
  }
  return route_detail::dispatch<float>(x, w_r, bias, (int)N, d, M, group_id, gate_prob, partial, probs, s);
}

}  // namespace moga

extern "C" moga_status moga_route(const void* x, const void* w_r, moga_dtype dt, const float* bias,
                                  int64_t N, int32_t d, int32_t M, int32_t* group_id, float* gate_prob,
                                  void* ws, size_t ws_bytes, void* stream) {
  return moga::route_impl(x, w_r, dt, bias, N, d, M, group_id, gate_prob, nullptr, ws, ws_bytes, stream);
}

extern "C" moga_status moga_route_train(const void* x, const void* w_r, moga_dtype dt, const float* bias,
                                        int64_t N, int32_t d, int32_t M, int32_t* group_id, float* gate_prob,
                                        float* probs, void* ws, size_t ws_bytes, void* stream) {
  if (!probs) return moga::fail(MOGA_ERR_INVALID_ARG, "moga_route_train: null probs");
  return moga::route_impl(x, w_r, dt, bias, N, d, M, group_id, gate_prob, probs, ws, ws_bytes, stream);
}
