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

__global__ void __launch_bounds__(kThreads)
tile_hist_kernel(const int32_t* __restrict__ g, int N, int M, int32_t* __restrict__ hist) {
  __shared__ int h[32];
  if (threadIdx.x < 32) h[threadIdx.x] = 0;
  __syncthreads();
  const int base = blockIdx.x * kTile;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int t = base + i * kThreads + threadIdx.x;
    if (t < N) {
      const int gi = __ldg(g + t);
      if ((unsigned)gi < (unsigned)M) atomicAdd(&h[gi], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < M) hist[(size_t)blockIdx.x * M + threadIdx.x] = h[threadIdx.x];
}

// One block of 32 * 32 threads: warp w owns group w; lanes stride over tiles.
__global__ void __launch_bounds__(1024)
scan_kernel(const int32_t* __restrict__ hist, int n_tiles, int M, int32_t* __restrict__ tile_off,
            int32_t* __restrict__ cu, int32_t* __restrict__ counts, int32_t* __restrict__ max_seqlen) {
  __shared__ int total[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pass 1: per-group totals
  if (warp < M) {
    int s = 0;
    for (int t = lane; t < n_tiles; t += 32) s += hist[(size_t)t * M + warp];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) total[warp] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0, mx = 0;
    for (int i = 0; i < M; ++i) {
      cu[i] = run;
      counts[i] = total[i];
      mx = max(mx, total[i]);
      run += total[i];
    }
    cu[M] = run;
    *max_seqlen = mx;
  }
  __syncthreads();
  // pass 2: per-(group, tile) exclusive offsets, 32 tiles per step
  if (warp < M) {
    int run = 0;
    for (int i = 0; i < warp; ++i) run += total[i];
    for (int t0 = 0; t0 < n_tiles; t0 += 32) {
      const int t = t0 + lane;
      const int v = t < n_tiles ? hist[(size_t)t * M + warp] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (t < n_tiles) tile_off[(size_t)t * M + warp] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

__global__ void __launch_bounds__(kThreads)
scatter_kernel(const int32_t* __restrict__ g, int N, int M, const int32_t* __restrict__ tile_off,
               int32_t* __restrict__ perm) {
  __shared__ int warp_cnt[kWarps][32];
  __shared__ int running[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < M) running[threadIdx.x] = tile_off[(size_t)blockIdx.x * M + threadIdx.x];
  const int base = blockIdx.x * kTile;
  for (int r = 0; r < kPerThread; ++r) {
    const int t = base + r * kThreads + threadIdx.x;
    const int gi = (t < N) ? __ldg(g + t) : -1;
    const bool valid = (unsigned)gi < (unsigned)M;
    const unsigned same = __match_any_sync(0xffffffffu, valid ? gi : -1);
    const int rank = __popc(same & ((1u << lane) - 1u));
    __syncthreads();   // previous round's readers of warp_cnt / running are done
    if (lane < 32 && lane < M) warp_cnt[warp][lane] = 0;
    __syncwarp();
    // the highest lane of each group run writes the warp's count for it
    if (valid && (same >> lane) == 1u) warp_cnt[warp][gi] = __popc(same);
    __syncthreads();
    if (valid) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w][gi];
      perm[running[gi] + before + rank] = t;
    }
    __syncthreads();
    if (threadIdx.x < M) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += warp_cnt[w][threadIdx.x];
      running[threadIdx.x] += s;
    }
  }
}

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
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = (int)N;
  const int tiles = ceil_div(n, kTile);
  int32_t* hist = static_cast<int32_t*>(ws);
  int32_t* tile_off = hist + (size_t)tiles * M;
  tile_hist_kernel<<<tiles, kThreads, 0, s>>>(group_id, n, M, hist);
  moga_status st = check_launch("moga_permute/hist");
  if (st != MOGA_OK) return st;
  scan_kernel<<<1, 1024, 0, s>>>(hist, tiles, M, tile_off, cu_seqlens, counts, max_seqlen);
  st = check_launch("moga_permute/scan");
  if (st != MOGA_OK) return st;
  scatter_kernel<<<tiles, kThreads, 0, s>>>(group_id, n, M, tile_off, perm);
  return check_launch("moga_permute/scatter");
}
