// Stable counting sort of tokens by routing group: perm, cu_seqlens, counts,
// max_seqlen.  MoGA note (papernotes.org ICLR 2026), key design 2: tokens
// are permuted so each group is contiguous and the group boundaries are
// described by cu_seqlens / max_seqlen.  Inside a group the order is
// ascending token index (the unique stable order).
//
// Three launches, each a single pass over an int32 array:
//   1. tile histogram: tile of kTile tokens -> hist[tile][M]
//   2. scan (one block): counts, cu_seqlens, max_seqlen and the start
//      offset of every (group, tile) pair, group-major
//   3. stable scatter: each tile walks its tokens in order; a warp ranks its
//      32 tokens with match.any (same-group lanes below), warps are ranked by
//      a per-round prefix over warp histograms, rounds by a running offset.
#include "common.cuh"

namespace moga {
namespace permute_detail {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kTile = kThreads * kPerThread;   // 2048 tokens per tile
constexpr int kWarps = kThreads / 32;

// Sort key of token t: its group, offset by M per video for a batch of
// videos of n_per tokens each (key = (t / n_per) * M + g); K = B * M keys.
// KMAX bounds K (32 for one video, 1024 for a batch).
__device__ __forceinline__ int sort_key(int gi, int t, int M, int n_per) { return (t / n_per) * M + gi; }

template <int KMAX>
__global__ void __launch_bounds__(kThreads)
tile_hist_kernel(const int32_t* __restrict__ g, int N, int M, int n_per, int K, int32_t* __restrict__ hist) {
  __shared__ int h[KMAX];
  for (int i = threadIdx.x; i < K; i += kThreads) h[i] = 0;
  __syncthreads();
  const int base = blockIdx.x * kTile;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int t = base + i * kThreads + threadIdx.x;
    if (t < N) {
      const int gi = __ldg(g + t);
      if ((unsigned)gi < (unsigned)M)
        atomicAdd(&h[sort_key(gi, t, M, n_per)], 1);
      else
        record_device_error(MOGA_ERR_BAD_INDEX);   // skipped here and by the scatter
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += kThreads) hist[(size_t)blockIdx.x * K + i] = h[i];
}

// One block of 32 * 32 threads: warp w owns keys w, w + 32, ...; lanes stride
// over tiles.
template <int KMAX>
__global__ void __launch_bounds__(1024)
scan_kernel(const int32_t* __restrict__ hist, int n_tiles, int K, int32_t* __restrict__ tile_off,
            int32_t* __restrict__ cu, int32_t* __restrict__ counts, int32_t* __restrict__ max_seqlen) {
  __shared__ int total[KMAX];
  __shared__ int start[KMAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pass 1: per-key totals
  for (int key = warp; key < K; key += 32) {
    int s = 0;
    for (int t = lane; t < n_tiles; t += 32) s += hist[(size_t)t * K + key];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) total[key] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0, mx = 0;
    for (int i = 0; i < K; ++i) {
      start[i] = run;
      cu[i] = run;
      counts[i] = total[i];
      mx = max(mx, total[i]);
      run += total[i];
    }
    cu[K] = run;
    *max_seqlen = mx;
  }
  __syncthreads();
  // pass 2: per-(key, tile) exclusive offsets, 32 tiles per step
  for (int key = warp; key < K; key += 32) {
    int run = start[key];
    for (int t0 = 0; t0 < n_tiles; t0 += 32) {
      const int t = t0 + lane;
      const int v = t < n_tiles ? hist[(size_t)t * K + key] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (t < n_tiles) tile_off[(size_t)t * K + key] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

template <int KMAX>
__global__ void __launch_bounds__(kThreads)
scatter_kernel(const int32_t* __restrict__ g, int N, int M, int n_per, int K, const int32_t* __restrict__ tile_off,
               int32_t* __restrict__ perm) {
  __shared__ int warp_cnt[kWarps][KMAX];
  __shared__ int running[KMAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < K; i += kThreads) running[i] = tile_off[(size_t)blockIdx.x * K + i];
  const int base = blockIdx.x * kTile;
  for (int r = 0; r < kPerThread; ++r) {
    const int t = base + r * kThreads + threadIdx.x;
    const int gi = (t < N) ? __ldg(g + t) : -1;
    const bool valid = (unsigned)gi < (unsigned)M;
    const int key = valid ? sort_key(gi, t, M, n_per) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(same & ((1u << lane) - 1u));
    __syncthreads();   // previous round's readers of warp_cnt / running are done
    for (int i = lane; i < K; i += 32) warp_cnt[warp][i] = 0;
    __syncwarp();
    // the highest lane of each key run writes the warp's count for it
    if (valid && (same >> lane) == 1u) warp_cnt[warp][key] = __popc(same);
    __syncthreads();
    if (valid) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w][key];
      perm[running[key] + before + rank] = t;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < K; i += kThreads) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += warp_cnt[w][i];
      running[i] += s;
    }
  }
}

template <int KMAX>
static moga_status run_permute(const int32_t* g, int n, int M, int n_per, int K, int32_t* perm, int32_t* cu,
                               int32_t* counts, int32_t* max_seqlen, void* ws, cudaStream_t s) {
  const int tiles = ceil_div(n, kTile);
  int32_t* hist = static_cast<int32_t*>(ws);
  int32_t* tile_off = hist + (size_t)tiles * K;
  tile_hist_kernel<KMAX><<<tiles, kThreads, 0, s>>>(g, n, M, n_per, K, hist);
  moga_status st = check_launch("moga_permute/hist");
  if (st != MOGA_OK) return st;
  scan_kernel<KMAX><<<1, 1024, 0, s>>>(hist, tiles, K, tile_off, cu, counts, max_seqlen);
  st = check_launch("moga_permute/scan");
  if (st != MOGA_OK) return st;
  scatter_kernel<KMAX><<<tiles, kThreads, 0, s>>>(g, n, M, n_per, K, tile_off, perm);
  return check_launch("moga_permute/scatter");
}

constexpr int kMaxKeys = 1024;   // B * M of a batch

}  // namespace permute_detail
}  // namespace moga

extern "C" size_t moga_permute_ws_bytes(int64_t N, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32) return 0;
  const size_t tiles = (size_t)moga::ceil_div((int)N, moga::permute_detail::kTile);
  return 2 * tiles * (size_t)M * sizeof(int32_t);
}

extern "C" moga_status moga_permute(const int32_t* group_id, int64_t N, int32_t M, int32_t* perm,
                                    int32_t* cu_seqlens, int32_t* counts, int32_t* max_seqlen,
                                    void* ws, size_t ws_bytes, void* stream) {
  using namespace moga;
  using namespace moga::permute_detail;
  if (!group_id || !perm || !cu_seqlens || !counts || !max_seqlen || !ws)
    return fail(MOGA_ERR_INVALID_ARG, "moga_permute: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_permute: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_permute: M=%d not in [1, 32]", M);
  if (ws_bytes < moga_permute_ws_bytes(N, M))
    return fail(MOGA_ERR_WORKSPACE, "moga_permute: workspace %zu < %zu bytes", ws_bytes, moga_permute_ws_bytes(N, M));
  return run_permute<32>(group_id, (int)N, M, (int)N, M, perm, cu_seqlens, counts, max_seqlen, ws,
                         static_cast<cudaStream_t>(stream));
}

extern "C" size_t moga_permute_batched_ws_bytes(int64_t n_per, int32_t B, int32_t M) {
  if (n_per <= 0 || B < 1 || M < 1 || M > 32 || (int64_t)B * M > moga::permute_detail::kMaxKeys ||
      n_per * B > INT32_MAX)
    return 0;
  const size_t tiles = (size_t)moga::ceil_div((int)(n_per * B), moga::permute_detail::kTile);
  return 2 * tiles * (size_t)B * M * sizeof(int32_t);
}

extern "C" moga_status moga_permute_batched(const int32_t* group_id, int64_t n_per, int32_t B, int32_t M,
                                            int32_t* perm, int32_t* cu_seqlens, int32_t* counts,
                                            int32_t* max_seqlen, void* ws, size_t ws_bytes, void* stream) {
  using namespace moga;
  using namespace moga::permute_detail;
  if (!group_id || !perm || !cu_seqlens || !counts || !max_seqlen || !ws)
    return fail(MOGA_ERR_INVALID_ARG, "moga_permute_batched: null pointer");
  if (B < 1 || n_per <= 0 || n_per * B > INT32_MAX)
    return fail(MOGA_ERR_INVALID_ARG, "moga_permute_batched: B=%d x n_per=%lld out of range", B, (long long)n_per);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_permute_batched: M=%d not in [1, 32]", M);
  if ((int64_t)B * M > kMaxKeys)
    return fail(MOGA_ERR_UNSUPPORTED, "moga_permute_batched: B*M=%lld above %d", (long long)B * M, kMaxKeys);
  const size_t need = moga_permute_batched_ws_bytes(n_per, B, M);
  if (ws_bytes < need) return fail(MOGA_ERR_WORKSPACE, "moga_permute_batched: workspace %zu < %zu bytes", ws_bytes, need);
  const int n = (int)(n_per * B), K = B * M;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (K <= 32) return run_permute<32>(group_id, n, M, (int)n_per, K, perm, cu_seqlens, counts, max_seqlen, ws, s);
  return run_permute<kMaxKeys>(group_id, n, M, (int)n_per, K, perm, cu_seqlens, counts, max_seqlen, ws, s);
}
