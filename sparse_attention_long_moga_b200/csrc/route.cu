// Router kernel: r = x . W_r (+ bias), p = softmax(r), g = argmax p, gate = p_g,
// plus per-block partial sums of p(i|x) for the group-balancing loss.
//
// MoGA note (papernotes.org ICLR 2026), key design 1: a linear projection
// with softmax gating gives p(i|x); the token goes to the most probable
// group; the blog (xugj520.cn) section 2.3 sketches the same bias-free layer.
//
// Design (HBM-bound: one read of x):
//   * four threads per token, 64 tokens per 256-thread block; thread s of a
//     token reads the 16-byte chunks s, s+4, s+8, ... of the row, so the
//     four threads of a token read 64 contiguous bytes per step and a warp
//     reads 8 such segments (every 32-byte sector fully used);
//   * several chunks are loaded before they are used, keeping enough bytes
//     in flight per SM to cover HBM latency;
//   * W_r is staged in shared memory as fp32 transposed to [M][k], so the
//     four threads of a token read adjacent 32-byte pieces (no bank
//     conflicts) and the 8 tokens of a warp share them (broadcast);
//     d is processed in chunks that fit the shared-memory budget;
//   * logits accumulate in fp32 registers, the four partial sums of a token
//     are combined with two shuffles.
#include "common.cuh"

namespace moga {
namespace route_detail {

constexpr int kThreads = 256;
constexpr int kSub = 4;                       // threads per token
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

template <typename T, int MP>
__global__ void __launch_bounds__(kThreads)
route_kernel(const T* __restrict__ x, const T* __restrict__ w_r, const float* __restrict__ bias,
             int N, int d, int M, int KC,
             int32_t* __restrict__ group_id, float* __restrict__ gate_prob,
             float* __restrict__ psum_partial) {
  extern __shared__ float4 smem_f4[];
  float* ws = reinterpret_cast<float*>(smem_f4);   // [MP][KC]
  __shared__ float red[kThreads / 32][MP];

  const int tid = threadIdx.x;
  const int sub = tid & (kSub - 1);
  const int tok = blockIdx.x * kTokens + tid / kSub;
  const bool active = tok < N;
  const T* xrow = x + (size_t)(active ? tok : 0) * d;

  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;

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
    if (active) {
      const int nchunk = kc / 8;   // 8-element chunks in this part of the row
      for (int c0 = sub; c0 < nchunk; c0 += kSub * kUnroll) {
        float xv[kUnroll][8];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * kSub;
          if (c < nchunk) Vec<T>::load(xrow + k0 + 8 * c, xv[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * kSub;
          if (c < nchunk) {
#pragma unroll
            for (int m = 0; m < MP; ++m) {
              const float4* wv = reinterpret_cast<const float4*>(ws + m * KC + 8 * c);
              const float4 a = wv[0], b = wv[1];
              float s = acc[m];
              s = fmaf(xv[u][0], a.x, s);
              s = fmaf(xv[u][1], a.y, s);
              s = fmaf(xv[u][2], a.z, s);
              s = fmaf(xv[u][3], a.w, s);
              s = fmaf(xv[u][4], b.x, s);
              s = fmaf(xv[u][5], b.y, s);
              s = fmaf(xv[u][6], b.z, s);
              s = fmaf(xv[u][7], b.w, s);
              acc[m] = s;
            }
          }
        }
      }
    }
  }
  // combine the four partial logits of each token
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 1);
    acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 2);
  }

  // softmax, argmax (lowest index wins a tie), gate
  float p[MP];
  const bool writer = active && sub == 0;
  if (active) {
    float best = -INFINITY;
    int g = 0;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      if (m < M) {
        const float r = acc[m] + (bias ? __ldg(bias + m) : 0.f);
        acc[m] = r;
        if (r > best) { best = r; g = m; }
      }
    }
    float z = 0.f;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      p[m] = (m < M) ? expf(acc[m] - best) : 0.f;
      z += p[m];
    }
    const float inv = 1.f / z;
#pragma unroll
    for (int m = 0; m < MP; ++m) p[m] = writer ? p[m] * inv : 0.f;
    if (writer) {
      group_id[tok] = g;
      gate_prob[tok] = inv;   // exp(r_g - max) = 1
    }
  } else {
#pragma unroll
    for (int m = 0; m < MP; ++m) p[m] = 0.f;
  }

  // fixed-order block reduction of p(i|x): warp butterfly, then warps in order
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    float v = p[m];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][m] = v;
  }
  __syncthreads();
  if (tid < M) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += red[w][tid];
    psum_partial[(size_t)blockIdx.x * M + tid] = s;
  }
}

template <typename T, int MP>
moga_status launch(const void* x, const void* w_r, const float* bias, int N, int d, int M,
                   int32_t* g, float* gate, float* partial, cudaStream_t s) {
  int KC = kSmemBudget / (MP * 4);
  KC = (KC / 32) * 32;            // whole 8-element chunks for all four threads
  if (KC >= d) KC = d;
  const size_t smem = (size_t)KC * MP * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<T, MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_route: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  const int blocks = ceil_div(N, kTokens);
  route_kernel<T, MP><<<blocks, kThreads, smem, s>>>(static_cast<const T*>(x), static_cast<const T*>(w_r),
                                                     bias, N, d, M, KC, g, gate, partial);
  return check_launch("moga_route");
}

template <typename T>
moga_status dispatch(const void* x, const void* w_r, const float* bias, int N, int d, int M,
                     int32_t* g, float* gate, float* partial, cudaStream_t s) {
  switch ((M + 3) / 4) {
    case 1: return launch<T, 4>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 2: return launch<T, 8>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 3: return launch<T, 12>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 4: return launch<T, 16>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 5: return launch<T, 20>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 6: return launch<T, 24>(x, w_r, bias, N, d, M, g, gate, partial, s);
    case 7: return launch<T, 28>(x, w_r, bias, N, d, M, g, gate, partial, s);
    default: return launch<T, 32>(x, w_r, bias, N, d, M, g, gate, partial, s);
  }
}

}  // namespace route_detail

int route_blocks(int64_t N) { return ceil_div((int)N, route_detail::kTokens); }

}  // namespace moga

extern "C" size_t moga_route_ws_bytes(int64_t N, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32) return 0;
  return (size_t)moga::route_blocks(N) * (size_t)M * sizeof(float);
}

extern "C" moga_status moga_route(const void* x, const void* w_r, moga_dtype dt, const float* bias,
                                  int64_t N, int32_t d, int32_t M, int32_t* group_id, float* gate_prob,
                                  void* ws, size_t ws_bytes, void* stream) {
  using namespace moga;
  if (!x || !w_r || !group_id || !gate_prob || !ws) return fail(MOGA_ERR_INVALID_ARG, "moga_route: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_route: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_route: M=%d not in [1, 32]", M);
  if (dt != MOGA_F32 && dt != MOGA_BF16) return fail(MOGA_ERR_INVALID_ARG, "moga_route: bad dtype %d", (int)dt);
  if (d <= 0 || d % 8 != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route: d=%d must be a positive multiple of 8", d);
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_route: x not 16-byte aligned");
  if (ws_bytes < moga_route_ws_bytes(N, M)) return fail(MOGA_ERR_WORKSPACE, "moga_route: workspace %zu < %zu bytes", ws_bytes, moga_route_ws_bytes(N, M));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* partial = static_cast<float*>(ws);
  if (dt == MOGA_BF16)
    return route_detail::dispatch<__nv_bfloat16>(x, w_r, bias, (int)N, d, M, group_id, gate_prob, partial, s);
  return route_detail::dispatch<float>(x, w_r, bias, (int)N, d, M, group_id, gate_prob, partial, s);
}
