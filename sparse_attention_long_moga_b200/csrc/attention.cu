// Grouped full attention on sm_100a: the MoGA groups, the STGA window groups
// and the per-frame groups share one tcgen05 kernel.
//
// What it computes (MoGA note, papernotes.org ICLR 2026, key designs 1, 2, 4):
// inside every group, non-causal softmax attention
//     O = softmax(Q K^T * scale) V
// per head, with the MoGA output scaled by the token's gate p(g(x)|x) and
// written back at the token's own row (no repermute pass).  The static
// groups add their outputs into the same fp32 accumulator.
//
// Two kernels per branch:
//   gather3_kernel   HBM-bound row copy of Q, K, V into segment order (rows
//                    picked through perm for MoGA, through the window map for
//                    the static windows), so that every group is a contiguous
//                    row range.  Frames are contiguous already and skip it.
//                    (gather_both_kernel writes both orders in one pass for
//                    the call that runs all three branches.)
//   attn_kernel      one CTA per (group, head, pair of 128-row query tiles):
//     warps 0-3 / 4-7  softmax + epilogue of query tile 0 / 1
//                      (thread = query row = TMEM lane)
//     warp 8           producer: 3-D tiled TMA loads (128B swizzle) of the
//                      two Q tiles and a 2-stage ring of K and V tiles
//     warp 9           TMEM allocator; lane 0 issues tcgen05.mma
//     warps 10-11      idle (complete the third warpgroup)
//   TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
//   The softmax writes P as bf16 pairs over the first 64 columns of its S
//   and the P.V product reads it from there (A operand in tensor memory).
//   Issue order per KV tile j:  PV0_j, S0_{j+1}, PV1_j, S1_{j+1}, so the
//   softmax of one tile runs while the tensor core serves the other; the
//   same order continues across work tiles (the next tile's first S0 goes
//   between the last PV0 and PV1 when its Q and K have landed).
//   Output rows leave through a per-warp shared-memory stage as whole
//   128-byte lines.
//   The running row max only moves (and O is rescaled) when it grows by
//   more than 2^8; the final 1/l uses the same reference, so the result is
//   exact.
// Every wait is bounded; on a timeout the CTA records MOGA_ERR_TIMEOUT,
// drains what it has in flight, frees TMEM and exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "tc_common.cuh"
#include "../../include/moga_testing.h"

namespace moga {
namespace attn {

constexpr int BM = 128;        // query rows per tile (two tiles per CTA)
constexpr int BN = 128;        // key/value rows per tile
constexpr int kThreads = 384;  // 12 warps: two softmax warpgroups + producer, MMA and two idle warps
// Register split (setmaxnreg): the kernel launches at 168 registers per
// thread (384 x 168 = 64512); the producer/MMA warpgroup gives back down to
// 120 and the two softmax warpgroups take 192: 128 x 120 + 256 x 192 = 64512.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 192;
constexpr int kControlRegs = 120;
static_assert(kThreads * kLaunchRegs == 128 * kControlRegs + 256 * kSoftmaxRegs, "register split must balance");
constexpr int kMaxTG = 256;    // temporal groups per launch
constexpr uint32_t kTmemCols = 512;
constexpr int kHalfBytes = BM * 128;   // one 64-column half of a 128-row tile (16 KB)

enum Mode : int { MODE_MOGA = 0, MODE_WINDOW = 1, MODE_FRAME = 2 };

struct TGroup {
  int t0, t1, a_prev, a_next;
};

struct Params {
  int N, H, mode;
  float scale_log2;
  // MoGA
  const int32_t* perm;
  const int32_t* cu;
  int M;
  const float* gate;
  // output accumulator [N][H][hd]
  float* o_acc;
  // frame launch of stga_attn_mean: out = bf16((o_acc + o_frame) / 3)
  // instead of adding into o_acc
  __nv_bfloat16* out;
  // training forward: per-row log2-domain log-sum-exp of the scaled scores,
  // lse[t][h] = m + log2(l) so that P = 2^(s * scale * log2(e) - lse) ([N][H]
  // fp32, optional), and the static branches write their own output instead
  // of adding into a shared accumulator
  float* lse;
  int write_static;
  // STGA geometry
  int T, h, w, win_h, win_w, n_wx, n_win, whw, hw;
  int n_tg;
  int tg_tiles[kMaxTG + 1];   // prefix of CTAs over temporal groups
  TGroup tg[kMaxTG];
  long long timeout_cycles;
  int debug_flags;            // bit 0: producer skips the Q load (timeout test)
};

using namespace moga::tc;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------------ index maps

// Read-only load: through the non-coherent cache on the device; a plain load
// when the same index code runs on the host (test hooks).
__host__ __device__ __forceinline__ int load_ro(const int32_t* a) {
#ifdef __CUDA_ARCH__
  return __ldg(a);
#else
  return *a;
#endif
}

// Token at position idx of the window-major order (window, frame, position
// inside the window), in which a temporal group's keys/values -- including
// the frames borrowed from the neighbouring shots -- are one contiguous range.
__host__ __device__ __forceinline__ int window_token(const Params& p, int idx) {
  const int local = idx % p.whw;
  const int wf = idx / p.whw;
  const int frame = wf % p.T;
  const int win = wf / p.T;
  const int wy = win / p.n_wx, wx = win - wy * p.n_wx;
  const int row = wy * p.win_h + local / p.win_w;
  const int col = wx * p.win_w + local % p.win_w;
  return frame * p.hw + row * p.w + col;
}

// Token (row of q, k, v and the outputs) at segment position idx.  The
// checking build returns -1 for a row outside [0, N) (a bad perm entry) after
// recording MOGA_ERR_BAD_INDEX; callers then skip the access.
__device__ __forceinline__ int token_of(const Params& p, int idx) {
  const int t = p.mode == MODE_MOGA ? __ldg(p.perm + idx) : (p.mode == MODE_FRAME ? idx : window_token(p, idx));
  if (kCheckIndices && (unsigned)t >= (unsigned)p.N) {
    record_device_error(MOGA_ERR_BAD_INDEX);
    return -1;
  }
  return t;
}

struct Tile {
  int head, q_begin, q_end, kv_begin, kv_end;
  int valid;  // 0: past the last tile
};

// MoGA groups in processing order (largest first), built once per CTA.
struct GroupTable {
  int n;
  int start[32], size[32];
  int prefix[33];   // CTA-tile prefix over the ordered groups
};

// unit_rows: query rows per work unit (two 128-row tiles in the forward, one
// in the backward)
__host__ __device__ void build_group_table(const Params& p, GroupTable& gt, int unit_rows = 2 * BM) {
  int size[32], order[32];
  if (kCheckIndices) {
    // cu_seqlens must split a range inside [0, N] without going backwards;
    // otherwise the launch gets no tiles (every CTA builds the same table)
    bool ok = load_ro(p.cu) >= 0 && load_ro(p.cu + p.M) <= p.N;
    for (int i = 0; i < p.M; ++i) ok = ok && load_ro(p.cu + i) <= load_ro(p.cu + i + 1);
    if (!ok) {
#ifdef __CUDA_ARCH__
      record_device_error(MOGA_ERR_BAD_INDEX);
#endif
      gt.n = 0;
      gt.prefix[0] = 0;
      return;
    }
  }
  for (int i = 0; i < p.M; ++i) {
    size[i] = load_ro(p.cu + i + 1) - load_ro(p.cu + i);
    order[i] = i;
  }
  for (int i = 1; i < p.M; ++i) {   // insertion sort, descending size, stable
    const int o = order[i];
    int j = i - 1;
    while (j >= 0 && size[order[j]] < size[o]) {
      order[j + 1] = order[j];
      --j;
    }
    order[j + 1] = o;
  }
  gt.n = p.M;
  gt.prefix[0] = 0;
  for (int k = 0; k < p.M; ++k) {
    const int g = order[k];
    gt.start[k] = load_ro(p.cu + g);
    gt.size[k] = size[g];
    gt.prefix[k + 1] = gt.prefix[k] + ceil_div(size[g], unit_rows) * p.H;
  }
}

// Tile L (a pair of 128-row query tiles of one group and head).  Tiles are
// ordered so that consecutive ones share a group's K/V through L2.
__host__ __device__ __forceinline__ Tile decode_tile(const Params& p, const GroupTable& gt, int L) {
  Tile t;
  t.valid = 0;
  constexpr int kPair = 2 * BM;
  if (p.mode == MODE_MOGA) {
    if (L >= gt.prefix[gt.n]) return t;
    int k = 0;
    while (gt.prefix[k + 1] <= L) ++k;
    const int qp = ceil_div(gt.size[k], kPair);
    const int rem = L - gt.prefix[k];
    t.head = rem / qp;
    const int qi = rem - t.head * qp;
    t.q_begin = gt.start[k] + qi * kPair;
    t.q_end = min(gt.start[k] + gt.size[k], t.q_begin + kPair);
    t.kv_begin = gt.start[k];
    t.kv_end = gt.start[k] + gt.size[k];
    t.valid = 1;
    return t;
  }
  if (p.mode == MODE_FRAME) {
    const int qp = ceil_div(p.hw, kPair);
    if (L >= p.T * p.H * qp) return t;
    const int frame = L / (p.H * qp);
    const int rem = L - frame * p.H * qp;
    t.head = rem / qp;
    const int qi = rem - t.head * qp;
    t.kv_begin = frame * p.hw;
    t.kv_end = t.kv_begin + p.hw;
    t.q_begin = t.kv_begin + qi * kPair;
    t.q_end = min(t.kv_end, t.q_begin + kPair);
    t.valid = 1;
    return t;
  }
  // window groups: temporal group, window, head, query-tile pair
  if (L >= p.tg_tiles[p.n_tg]) return t;
  int g = 0;
  while (p.tg_tiles[g + 1] <= L) ++g;
  const TGroup tg = p.tg[g];
  const int qlen = (tg.t1 - tg.t0) * p.whw;
  const int qp = ceil_div(qlen, kPair);
  const int rem = L - p.tg_tiles[g];
  const int win = rem / (p.H * qp);
  const int rem2 = rem - win * p.H * qp;
  t.head = rem2 / qp;
  const int qi = rem2 - t.head * qp;
  const int base = win * p.T;
  t.q_begin = (base + tg.t0) * p.whw + qi * kPair;
  t.q_end = min((base + tg.t1) * p.whw, t.q_begin + kPair);
  t.kv_begin = (base + tg.t0 - tg.a_prev) * p.whw;
  t.kv_end = (base + tg.t1 + tg.a_next) * p.whw;
  t.valid = 1;
  return t;
}

// ------------------------------------------------------------------ gather

// dst[j] = src[map(j)] for the rows of Q, K and V ([N][H*hd] bf16, rows of
// `row_u4` 16-byte vectors); one warp per destination row.
template <int MODE>
__global__ void __launch_bounds__(256)
gather3_kernel(const __grid_constant__ Params p, const uint4* __restrict__ q, const uint4* __restrict__ k,
               const uint4* __restrict__ v, uint4* __restrict__ qd, uint4* __restrict__ kd, uint4* __restrict__ vd,
               int row_u4) {
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= p.N) return;
  const int lane = threadIdx.x & 31;
  const int src = MODE == MODE_MOGA ? __ldg(p.perm + j) : window_token(p, j);
  if (kCheckIndices && (unsigned)src >= (unsigned)p.N) {
    if (lane == 0) record_device_error(MOGA_ERR_BAD_INDEX);
    return;
  }
  const size_t so = (size_t)src * row_u4, dofs = (size_t)j * row_u4;
  for (int c = lane; c < row_u4; c += 32) {
    const uint4 a = __ldg(q + so + c);
    const uint4 b = __ldg(k + so + c);
    const uint4 e = __ldg(v + so + c);
    qd[dofs + c] = a;
    kd[dofs + c] = b;
    vd[dofs + c] = e;
  }
}

// Position of token t in the window-major order: the inverse of window_token.
__host__ __device__ __forceinline__ int window_pos(const Params& p, int t) {
  const int frame = t / p.hw;
  const int r = t - frame * p.hw;
  const int row = r / p.w, col = r - row * p.w;
  const int win = (row / p.win_h) * p.n_wx + col / p.win_w;
  const int local = (row % p.win_h) * p.win_w + col % p.win_w;
  return (win * p.T + frame) * p.whw + local;
}

// Both segment orders in one pass: for group position j, the token
// t = perm[j]'s rows of Q, K, V are read once and written to position j of
// the group-order copy and to position window_pos(t) of the window-order
// copy (one warp per position).
__global__ void __launch_bounds__(256)
gather_both_kernel(const __grid_constant__ Params p, const uint4* __restrict__ q, const uint4* __restrict__ k,
                   const uint4* __restrict__ v, uint4* __restrict__ gq, uint4* __restrict__ gk, uint4* __restrict__ gv,
                   uint4* __restrict__ wq, uint4* __restrict__ wk, uint4* __restrict__ wv, int row_u4) {
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= p.N) return;
  const int lane = threadIdx.x & 31;
  const int src = __ldg(p.perm + j);
  if (kCheckIndices && (unsigned)src >= (unsigned)p.N) {
    if (lane == 0) record_device_error(MOGA_ERR_BAD_INDEX);
    return;
  }
  const size_t so = (size_t)src * row_u4, go = (size_t)j * row_u4, wo = (size_t)window_pos(p, src) * row_u4;
  for (int c = lane; c < row_u4; c += 32) {
    const uint4 a = __ldg(q + so + c);
    const uint4 b = __ldg(k + so + c);
    const uint4 e = __ldg(v + so + c);
    gq[go + c] = a;
    gk[go + c] = b;
    gv[go + c] = e;
    wq[wo + c] = a;
    wk[wo + c] = b;
    wv[wo + c] = e;
  }
}

// ------------------------------------------------------------------ shared memory

template <int HD>
struct SmemLayout {
  static constexpr int kHalves = HD / 64;
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // one 128-row Q/K/V tile
  static constexpr int kQ = 0;                              // two Q tiles
  static constexpr int kK0 = kQ + 2 * kTileBytes;           // two K stages
  static constexpr int kV0 = kK0 + 2 * kTileBytes;          // two V stages
  static constexpr int kBar = kV0 + 2 * kTileBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTable = kMisc + 64;
  // epilogue staging: per softmax warp, its 32 rows x 32 fp32 columns (4 KB)
  static constexpr int kStage = (kTable + (int)sizeof(GroupTable) + 127) & ~127;
  static constexpr int kStageWarpBytes = 32 * 32 * 4;
  static constexpr int kEnd = kStage + 8 * kStageWarpBytes;
  // 1 KB slack to align the dynamic base to 1024 bytes; the hd = 64 layout is
  // padded so that two CTAs never share an SM (each holds all 512 TMEM columns)
  static constexpr int kBytes = (HD == 64 && kEnd < 120 * 1024 ? 120 * 1024 : kEnd) + 1024;
};

enum Bar : int {
  B_FULL_Q = 0,
  B_EMPTY_Q = 1,
  B_FULL_K = 2,   // +stage
  B_FULL_V = 4,   // +stage
  B_EMPTY_K = 6,  // +stage
  B_EMPTY_V = 8,  // +stage
  B_S_FULL = 10,  // +query tile
  B_P_FULL = 12,  // +query tile
  B_O_FULL = 14,  // +query tile
  B_O_EMPTY = 16, // +query tile
  B_MMA_END = 18,
  B_COUNT = 19
};

// ------------------------------------------------------------------ the kernel

// Persistent: CTA b processes tiles b, b + gridDim.x, ...  Barrier phases run
// on across tiles (counters below); TMEM is allocated once.  The producer
// loads the next tile's Q as soon as the last S MMA of the current tile has
// read Q, and the MMA warp starts the next tile's S products while the
// softmax warps are still writing the current tile's output.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using S = SmemLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + S::kBar + 8u * (uint32_t)i; };
  int* misc = reinterpret_cast<int*>(smem + S::kMisc);
  volatile int* abort_flag = misc + 0;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
  GroupTable* gt_sh = reinterpret_cast<GroupTable*>(smem + S::kTable);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    if (p.mode == MODE_MOGA) build_group_table(p, *gt_sh);
    mbar_init(bar(B_FULL_Q), 1);
    mbar_init(bar(B_EMPTY_Q), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_FULL_K + s), 1);
      mbar_init(bar(B_FULL_V + s), 1);
      mbar_init(bar(B_EMPTY_K + s), 1);
      mbar_init(bar(B_EMPTY_V + s), 1);
      mbar_init(bar(B_S_FULL + s), 1);
      mbar_init(bar(B_P_FULL + s), BM);
      mbar_init(bar(B_O_FULL + s), 1);
      mbar_init(bar(B_O_EMPTY + s), BM);
    }
    mbar_init(bar(B_MMA_END), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const GroupTable& gt = *gt_sh;
  if (!decode_tile(p, gt, blockIdx.x).valid) return;   // uniform: this CTA has no tile

  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long timeout = p.timeout_cycles;

  // Each warpgroup adjusts its register budget once, inside its own branch,
  // so the code of each role is compiled against its own budget.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const bool skip_q = (p.debug_flags & 1) != 0;
      int last_k[2] = {-1, -1}, last_v[2] = {-1, -1}, last_q = -1;
      int c = 0;   // K/V tiles issued so far (ring position)
      bool ok = true;
      for (int i = 0, L = blockIdx.x; ok; ++i, L += gridDim.x) {
        const Tile t = decode_tile(p, gt, L);
        if (!t.valid) break;
        const bool has_q1 = t.q_begin + BM < t.q_end;
        // Q of the previous tile has been read by its last S product
        if (!(ok = mbar_wait(bar(B_EMPTY_Q), (i & 1) ^ 1, abort_flag, timeout))) break;
        if (!skip_q) {
          mbar_arrive_expect_tx(bar(B_FULL_Q), (has_q1 ? 2 : 1) * S::kTileBytes);
          for (int qt = 0; qt < (has_q1 ? 2 : 1); ++qt)
#pragma unroll
            for (int hh = 0; hh < S::kHalves; ++hh)
              tma_load_3d(sbase + S::kQ + qt * S::kTileBytes + hh * kHalfBytes, &tm_q, hh * 64, t.head,
                          t.q_begin + qt * BM, bar(B_FULL_Q));
          last_q = i;
        }
        const int n_kv = ceil_div(t.kv_end - t.kv_begin, BN);
        for (int j = 0; j < n_kv; ++j, ++c) {
          const int st = c & 1;
          const uint32_t ph = (c >> 1) & 1;
          const int row = t.kv_begin + j * BN;
          if (!(ok = mbar_wait(bar(B_EMPTY_K + st), ph ^ 1, abort_flag, timeout))) break;
          mbar_arrive_expect_tx(bar(B_FULL_K + st), S::kTileBytes);
#pragma unroll
          for (int hh = 0; hh < S::kHalves; ++hh)
            tma_load_3d(sbase + S::kK0 + st * S::kTileBytes + hh * kHalfBytes, &tm_k, hh * 64, t.head, row,
                        bar(B_FULL_K + st));
          last_k[st] = c;
          if (!(ok = mbar_wait(bar(B_EMPTY_V + st), ph ^ 1, abort_flag, timeout))) break;
          mbar_arrive_expect_tx(bar(B_FULL_V + st), S::kTileBytes);
#pragma unroll
          for (int hh = 0; hh < S::kHalves; ++hh)
            tma_load_3d(sbase + S::kV0 + st * S::kTileBytes + hh * kHalfBytes, &tm_v, hh * 64, t.head, row,
                        bar(B_FULL_V + st));
          last_v[st] = c;
        }
      }
      // let every copy started here land before the CTA can exit
      if (last_q >= 0) mbar_drain(bar(B_FULL_Q), last_q & 1, timeout);
      for (int st = 0; st < 2; ++st) {
        if (last_k[st] >= 0) mbar_drain(bar(B_FULL_K + st), (last_k[st] >> 1) & 1, timeout);
        if (last_v[st] >= 0) mbar_drain(bar(B_FULL_V + st), (last_v[st] >> 1) & 1, timeout);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = instr_desc(BN, false);
      constexpr uint32_t idesc_pv = instr_desc(HD, true);
      const uint32_t tmem_s[2] = {tmem, tmem + 128};
      const uint32_t tmem_o[2] = {tmem + 256, tmem + 384};
      int c = 0;                   // K/V ring position
      int pc[2] = {0, 0};          // P tiles consumed per query tile
      int oc[2] = {0, 0};          // outputs produced per query tile
      auto issue_s = [&](int qt, int cc) {
        const uint32_t qa = sbase + S::kQ + qt * S::kTileBytes;
        const uint32_t ka = sbase + S::kK0 + (cc & 1) * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint64_t ad = smem_desc(qa + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(ka + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem_s[qt], ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_S_FULL + qt));
      };
      auto issue_pv = [&](int qt, int cc, bool acc) {
        const uint32_t va = sbase + S::kV0 + (cc & 1) * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t bd = smem_desc(va + ks * 16 * 128, kHalfBytes, 1024);
          tc_mma_ts(tmem_o[qt], tmem_s[qt] + ks * 8, bd, idesc_pv, (acc || ks > 0) ? 1u : 0u);
        }
      };
      // The first S product of a tile's query tile 0 is issued right after
      // the previous tile's last P.V of query tile 0 (the order inside a
      // tile), when the new Q and K are already there; otherwise, and for
      // query tile 1 (whose S columns hold the previous tile's last P until
      // its P.V), after the previous tile's last P.V products.  O_FULL of each
      // query tile is committed right after its last P.V, so its epilogue
      // overlaps the other query tile's last products.
      auto first_s0 = [&](int i, int cc) {
        if (!(mbar_wait(bar(B_FULL_Q), i & 1, abort_flag, timeout) &&
              mbar_wait(bar(B_FULL_K + (cc & 1)), (cc >> 1) & 1, abort_flag, timeout)))
          return false;
        tc_fence_after();
        issue_s(0, cc);
        return true;
      };
      auto first_s1 = [&](const Tile& t, int cc) {
        if (t.q_begin + BM < t.q_end) issue_s(1, cc);
        if (t.kv_end - t.kv_begin <= BN) tc_commit(bar(B_EMPTY_Q));   // a single K/V tile: Q is read
        tc_commit(bar(B_EMPTY_K + (cc & 1)));
      };
      int L = blockIdx.x;
      Tile t = decode_tile(p, gt, L);
      bool ok = t.valid && first_s0(0, c);
      if (ok) first_s1(t, c);
      for (int i = 0; ok && t.valid; ++i) {
        const bool has_q1 = t.q_begin + BM < t.q_end;
        const int nq = has_q1 ? 2 : 1;
        const int n_kv = ceil_div(t.kv_end - t.kv_begin, BN);
        const Tile tn = decode_tile(p, gt, L + gridDim.x);
        bool next_started = false;
        for (int j = 0; j < n_kv; ++j, ++c) {
          const int st = c & 1;
          const uint32_t ph = (c >> 1) & 1;
          const bool more = j + 1 < n_kv;
          for (int qt = 0; qt < nq; ++qt) {
            // the first P.V of a tile overwrites O: the epilogue of this query
            // tile's previous output must have read it
            if (j == 0 && !(ok = mbar_wait(bar(B_O_EMPTY + qt), (oc[qt] & 1) ^ 1, abort_flag, timeout))) break;
            if (qt == 0 && !(ok = mbar_wait(bar(B_FULL_V + st), ph, abort_flag, timeout))) break;
            if (!(ok = mbar_wait(bar(B_P_FULL + qt), pc[qt] & 1, abort_flag, timeout))) break;
            tc_fence_after();
            issue_pv(qt, c, j > 0);
            ++pc[qt];
            if (!more) {
              tc_commit(bar(B_O_FULL + qt));
              ++oc[qt];
            }
            if (qt == 0 && more) {
              if (!(ok = mbar_wait(bar(B_FULL_K + ((c + 1) & 1)), ((c + 1) >> 1) & 1, abort_flag, timeout))) break;
              tc_fence_after();
              issue_s(0, c + 1);
            } else if (qt == 0 && tn.valid && has_q1 && mbar_test(bar(B_FULL_Q), (i + 1) & 1) &&
                       mbar_test(bar(B_FULL_K + ((c + 1) & 1)), ((c + 1) >> 1) & 1)) {
              if (!(ok = first_s0(i + 1, c + 1))) break;
              next_started = true;
            }
          }
          if (!ok) break;
          tc_commit(bar(B_EMPTY_V + st));
          if (more) {
            if (has_q1) issue_s(1, c + 1);
            if (j + 2 == n_kv) tc_commit(bar(B_EMPTY_Q));   // last S products of this tile issued
            tc_commit(bar(B_EMPTY_K + ((c + 1) & 1)));
          }
        }
        if (!ok) break;
        if (tn.valid) {
          if (!next_started) ok = first_s0(i + 1, c);
          if (ok) first_s1(tn, c);
        }
        t = tn;
        L += gridDim.x;
      }
      // every MMA issued here has finished before TMEM is released
      tc_commit(bar(B_MMA_END));
      mbar_drain(bar(B_MMA_END), 0, timeout);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ---------------------------------------------------------------- softmax
    const int qt = warp >> 2;                            // query tile of this warpgroup
    const int row = (warp & 3) * 32 + lane;              // TMEM lane == query row
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr + qt * 128;
    const uint32_t o_addr = tmem + lane_addr + 256 + qt * 128;
    const float sl = p.scale_log2;
    int sc = 0, oc = 0;   // S tiles and outputs handled by this warpgroup
    bool ok = true;
    for (int L = blockIdx.x; ok; L += gridDim.x) {
      const Tile t = decode_tile(p, gt, L);
      if (!t.valid) break;
      if (qt == 1 && !(t.q_begin + BM < t.q_end)) continue;   // no second query tile here
      const int n_kv = ceil_div(t.kv_end - t.kv_begin, BN);
      if (p.out != nullptr) {
        // the fused mean reads this row of the accumulator in the epilogue:
        // start bringing it into L2 now, a whole work tile ahead
        const int q_pre = t.q_begin + qt * BM + row;
        const int tok_pre = q_pre < t.q_end ? token_of(p, q_pre) : -1;
        if (tok_pre >= 0) {
          const char* a = reinterpret_cast<const char*>(p.o_acc + ((size_t)tok_pre * p.H + t.head) * HD);
#pragma unroll
          for (int e = 0; e < HD * 4; e += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(a + e));
        }
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n_kv; ++j, ++sc) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + qt), sc & 1, abort_flag, timeout));
        if (!ok) break;
        tc_fence_after();
        // scores as pairs, so the scale-and-shift and the row sum run as
        // packed f32x2 operations (half the instructions)
        float2 s2[BN / 2];
        float* s = reinterpret_cast<float*>(s2);
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(s_addr + cc * 32, s + cc * 32);
        tmem_wait_ld();
        const int valid = t.kv_end - (t.kv_begin + j * BN);
        if (valid < BN) {
#pragma unroll
          for (int cc = 0; cc < BN; ++cc)
            if (cc >= valid) s[cc] = -INFINITY;
        }
        // row max with 8 independent chains of three-input max
        float mp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mp[e] = s[e];
#pragma unroll
        for (int cc = 8; cc < BN; cc += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) mp[e] = max3(mp[e], s[cc + e], s[cc + 8 + e]);
        const float mx = max3(max3(mp[0], mp[1], mp[2]), max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        const float m_new = fmaxf(m_run, mx * sl);
        // Move the reference max only when it grows by more than 2^8 (tile 0
        // always sets it); rows that move it rescale O and l after P is written.
        const bool need = j > 0 && m_new > m_run + 8.0f;
        const float m_old = m_run;
        if (j == 0 || need) m_run = m_new;
        const float neg_m = -m_run;
        const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(neg_m, neg_m);
        float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int cc = 0; cc < BN / 16; ++cc) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 xab = __ffma2_rn(s2[cc * 8 + e], sl2, nm2);
            const float2 pab = make_float2(fast_exp2(xab.x), fast_exp2(xab.y));
            acc2[e & 3] = __fadd2_rn(acc2[e & 3], pab);
            pk[e] = pack_bf16x2(pab.x, pab.y);
          }
          // P overwrites S columns [8cc, 8cc+8), whose scores were read above
          tmem_st8(s_addr + cc * 8, pk);
        }
        const float2 acc01 = __fadd2_rn(acc2[0], acc2[1]), acc23 = __fadd2_rn(acc2[2], acc2[3]);
        const float row_sum = (acc01.x + acc01.y) + (acc23.x + acc23.y);
        if (__any_sync(0xffffffffu, need)) {
          // P.V of tile j-1 finished before S of tile j (issue order), so O
          // may be rescaled here, before P_j is released to the MMA warp
          const float f = need ? fast_exp2(m_old - m_new) : 1.0f;
#pragma unroll 1
          for (int cc = 0; cc < HD / 32; ++cc) {
            float o[32];
            tmem_ld32(o_addr + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= f;
            tmem_st32(o_addr + cc * 32, o);
          }
          l_run *= f;
        }
        l_run += row_sum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + qt));
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL + qt), oc & 1, abort_flag, timeout));
      if (!ok) break;
      ++oc;
      tc_fence_after();
      float o[HD];
#pragma unroll
      for (int cc = 0; cc < HD / 32; ++cc) tmem_ld32(o_addr + cc * 32, o + cc * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_O_EMPTY + qt));   // O may be overwritten by the next tile now
      const int q_idx = t.q_begin + qt * BM + row;
      const int tok = q_idx < t.q_end ? token_of(p, q_idx) : -1;
      float scale = 1.0f / l_run;
      if (tok >= 0 && p.mode == MODE_MOGA) scale *= __ldg(p.gate + tok);
      if (tok >= 0 && p.lse != nullptr) p.lse[(size_t)tok * p.H + t.head] = m_run + log2f(l_run);
      if (p.out == nullptr || p.mode == MODE_MOGA || p.write_static) {
        // Rows leave through shared memory so that each warp instruction
        // writes whole 128-byte lines: per 32-column chunk, every thread puts
        // its row there (16-byte chunk k of row r at slot k ^ (r & 7), which
        // keeps the stores and the loads free of bank conflicts), then the
        // warp writes four rows per instruction, eight lanes per row.  The
        // MoGA branch stores; the static branches add into the accumulator
        // with fire-and-forget vector reductions (each element is updated by
        // exactly one thread per launch, so the result equals load-add-store
        // without the load latency).
        float4* stage = reinterpret_cast<float4*>(smem + S::kStage + warp * S::kStageWarpBytes);
        const bool plain = p.mode == MODE_MOGA || p.write_static;
        const int sub = lane & 7;
#pragma unroll
        for (int cc = 0; cc < HD / 32; ++cc) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            stage[lane * 8 + (k ^ (lane & 7))] =
                make_float4(o[cc * 32 + 4 * k] * scale, o[cc * 32 + 4 * k + 1] * scale, o[cc * 32 + 4 * k + 2] * scale,
                            o[cc * 32 + 4 * k + 3] * scale);
          __syncwarp();
#pragma unroll
          for (int r4 = 0; r4 < 8; ++r4) {
            const int rr = r4 * 4 + (lane >> 3);   // row of this warp written by this lane
            const int tr = __shfl_sync(0xffffffffu, tok, rr);
            const float4 val = stage[rr * 8 + (sub ^ (rr & 7))];
            if (tr >= 0) {
              float4* d = reinterpret_cast<float4*>(p.o_acc + ((size_t)tr * p.H + t.head) * HD + cc * 32) + sub;
              if (plain)
                *d = val;
              else
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(d), "f"(val.x), "f"(val.y),
                             "f"(val.z), "f"(val.w)
                             : "memory");
            }
          }
          __syncwarp();
        }
      } else if (tok >= 0) {
        const float4* d4 = reinterpret_cast<const float4*>(p.o_acc + ((size_t)tok * p.H + t.head) * HD);
        {
          // last branch of the layer: the three-way mean, fused (the frames
          // partition the tokens, so this thread owns the row)
          // product and sum rounded separately (no FMA contraction), as in
          // the reduction-then-mean path, so both give identical bits
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)tok * p.H + t.head) * HD);
          auto avg = [&](float acc, float v) { return __fadd_rn(acc, __fmul_rn(v, scale)) / 3.0f; };
#pragma unroll
          for (int e = 0; e < HD / 8; ++e) {
            const float4 a = d4[2 * e], b = d4[2 * e + 1];
            const float* oe = o + 8 * e;
            dst[e] = make_uint4(pack_bf16x2(avg(a.x, oe[0]), avg(a.y, oe[1])), pack_bf16x2(avg(a.z, oe[2]), avg(a.w, oe[3])),
                                pack_bf16x2(avg(b.x, oe[4]), avg(b.y, oe[5])), pack_bf16x2(avg(b.z, oe[6]), avg(b.w, oe[7])));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// [rows][H][hd] bf16 viewed as 3-D {hd, H, rows}; box {64, 1, 128}, 128B swizzle.
static moga_status make_map(CUtensorMap* m, const void* base, int64_t rows, int H, int hd) {
  auto fn = encode_fn();
  if (!fn) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gdim[3] = {(cuuint64_t)hd, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t gstride[2] = {(cuuint64_t)hd * 2, (cuuint64_t)H * hd * 2};
  cuuint32_t box[3] = {64, 1, BM};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOGA_OK;
}

static long long default_timeout_cycles() {
  return kWaitLimitCycles;
}

template <int HD>
static moga_status launch_attn(const Params& prm, int grid, const void* q, const void* k, const void* v,
                               cudaStream_t s) {
  using S = SmemLayout<HD>;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  CUtensorMap mq, mk, mv;
  moga_status st;
  if ((st = make_map(&mq, q, prm.N, prm.H, HD)) != MOGA_OK) return st;
  if ((st = make_map(&mk, k, prm.N, prm.H, HD)) != MOGA_OK) return st;
  if ((st = make_map(&mv, v, prm.N, prm.H, HD)) != MOGA_OK) return st;
  if (grid <= 0) return MOGA_OK;
  attn_kernel<HD><<<grid, kThreads, S::kBytes, s>>>(prm, mq, mk, mv);
  return check_launch("attention kernel");
}

static moga_status launch_gather(const Params& prm, int hd, const void* q, const void* k, const void* v, void* ws,
                                 cudaStream_t s) {
  const size_t bytes = (size_t)prm.N * prm.H * hd * 2;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int row_u4 = prm.H * hd / 8;
  const int grid = ceil_div(prm.N, 8);
  const uint4 *qs = static_cast<const uint4*>(q), *ks = static_cast<const uint4*>(k),
              *vs = static_cast<const uint4*>(v);
  uint4 *qd = reinterpret_cast<uint4*>(w), *kd = reinterpret_cast<uint4*>(w + bytes),
        *vd = reinterpret_cast<uint4*>(w + 2 * bytes);
  if (prm.mode == MODE_MOGA)
    gather3_kernel<MODE_MOGA><<<grid, 256, 0, s>>>(prm, qs, ks, vs, qd, kd, vd, row_u4);
  else
    gather3_kernel<MODE_WINDOW><<<grid, 256, 0, s>>>(prm, qs, ks, vs, qd, kd, vd, row_u4);
  return check_launch("gather kernel");
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

// Timing hook (declared in include/moga_testing.h): events recorded on the
// launching stream around the attention-kernel launches of the next call on
// this thread.  armed 1: `before` goes in front of the next launch; armed 2:
// `after` follows every launch until the hook is set again.
static thread_local cudaEvent_t t_ev_before = nullptr, t_ev_after = nullptr;
static thread_local int t_ev_armed = 0;
extern "C" void moga_test_set_attn_events(void* before, void* after) {
  t_ev_before = static_cast<cudaEvent_t>(before);
  t_ev_after = static_cast<cudaEvent_t>(after);
  t_ev_armed = (before && after) ? 1 : 0;
}

// `tiles` is the number of tile pairs (or an upper bound); the persistent
// grid has one CTA per SM at most.
static moga_status dispatch_attn(const Params& prm, int tiles, int hd, const void* q, const void* k, const void* v,
                                 cudaStream_t s) {
  const int grid = std::min(tiles, sm_count());
  if (t_ev_armed == 1) {
    const cudaError_t e = cudaEventRecord(t_ev_before, s);
    if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "attention timing event: %s", cudaGetErrorString(e));
    t_ev_armed = 2;
  }
  const moga_status st = hd == 128 ? launch_attn<128>(prm, grid, q, k, v, s) : launch_attn<64>(prm, grid, q, k, v, s);
  if (st == MOGA_OK && t_ev_armed == 2) {
    const cudaError_t e = cudaEventRecord(t_ev_after, s);
    if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "attention timing event: %s", cudaGetErrorString(e));
  }
  return st;
}

static size_t attn_ws_bytes(int64_t N, int H, int hd) { return 3 * (size_t)N * H * hd * 2; }

static moga_status check_common(const void* q, const void* k, const void* v, int64_t N, int H, int hd,
                                const float* o_acc, const void* ws, size_t ws_bytes, bool need_ws, const char* who) {
  if (!q || !k || !v || !o_acc) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (N <= 0 || H <= 0 || N * (int64_t)H >= INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "%s: N*H out of range", who);
  if (hd != 64 && hd != 128) return fail(MOGA_ERR_UNSUPPORTED, "%s: head_dim %d (supported: 64, 128)", who, hd);
  const uintptr_t a = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                      reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o_acc) |
                      reinterpret_cast<uintptr_t>(ws);
  if (a & 15) return fail(MOGA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  if (need_ws) {
    if (!ws) return fail(MOGA_ERR_INVALID_ARG, "%s: null workspace", who);
    if (ws_bytes < attn_ws_bytes(N, H, hd))
      return fail(MOGA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws_bytes, attn_ws_bytes(N, H, hd));
  }
  return MOGA_OK;
}

// Temporal groups of the static window branch (as-equal-as-possible runs of
// at most tg_max frames inside each shot, longer runs first; adjacent-shot
// frames on the K/V side at each cut).
static void build_temporal_groups(const moga_stga_geom& g, std::vector<TGroup>& out) {
  int start = 0;
  for (int s = 0; s < g.n_shots; ++s) {
    const int len = g.shot_len[s];
    const int n = g.tg_max == 0 ? 1 : (len + g.tg_max - 1) / g.tg_max;
    const int q = len / n, r = len % n;
    int f = start;
    for (int i = 0; i < n; ++i) {
      const int run = q + (i < r ? 1 : 0);
      TGroup tg{f, f + run, 0, 0};
      if (i == 0 && s > 0) tg.a_prev = std::min(g.aug_frames, g.shot_len[s - 1]);
      if (i == n - 1 && s + 1 < g.n_shots) tg.a_next = std::min(g.aug_frames, g.shot_len[s + 1]);
      out.push_back(tg);
      f += run;
    }
    start += len;
  }
}

}  // namespace attn
}  // namespace moga

using namespace moga;
using namespace moga::attn;

// Test hook (declared in include/moga_testing.h): bounded-wait limit in SM
// cycles and debug flags for the next attention launches on this thread.
static thread_local long long t_timeout_override = 0;
static thread_local int t_debug_flags = 0;
extern "C" void moga_test_set_attn_debug(long long timeout_cycles, int flags) {
  t_timeout_override = timeout_cycles;
  t_debug_flags = flags;
}

static void fill_debug(Params& prm) {
  prm.timeout_cycles = t_timeout_override > 0 ? t_timeout_override : default_timeout_cycles();
  prm.debug_flags = t_debug_flags;
}

extern "C" size_t moga_attn_ws_bytes(int64_t N, int32_t H, int32_t hd) {
  if (N <= 0 || H <= 0 || (hd != 64 && hd != 128) || N * (int64_t)H >= INT32_MAX) return 0;
  return attn_ws_bytes(N, H, hd);
}

// B videos of N / B tokens each (B = 1: one video): cu_seqlens holds B * M + 1
// boundaries, video b's groups are segments [b M, b M + M).  One gather into
// segment order, then one attention launch per video.
static moga_status moga_impl(const void* q, const void* k, const void* v, int64_t N, int32_t B, int32_t H,
                             int32_t hd, const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                             const float* gate_prob, float softmax_scale, float* o_acc, float* lse, void* ws,
                             size_t ws_bytes, void* stream) {
  moga_status st = check_common(q, k, v, N, H, hd, o_acc, ws, ws_bytes, true, "moga_group_attn");
  if (st != MOGA_OK) return st;
  if (!perm || !cu_seqlens || !gate_prob) return fail(MOGA_ERR_INVALID_ARG, "moga_group_attn: null pointer");
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_group_attn: M=%d not in [1, 32]", M);
  if (!(softmax_scale > 0.f)) return fail(MOGA_ERR_INVALID_ARG, "moga_group_attn: softmax_scale must be > 0");
  Params prm;
  memset(&prm, 0, sizeof(prm));
  prm.N = (int)N;
  prm.H = H;
  prm.mode = MODE_MOGA;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.perm = perm;
  prm.cu = cu_seqlens;
  prm.M = M;
  prm.gate = gate_prob;
  prm.o_acc = o_acc;
  prm.lse = lse;
  fill_debug(prm);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = launch_gather(prm, hd, q, k, v, ws, s)) != MOGA_OK) return st;
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  const size_t bytes = (size_t)N * H * hd * 2;
  // upper bound on a video's tile count: sum_i ceil(n_i / 256) <= n / 256 + M
  const int tiles = (ceil_div((int)(N / B), 2 * BM) + M) * H;
  for (int b = 0; b < B; ++b) {
    prm.cu = cu_seqlens + (size_t)b * M;
    if ((st = dispatch_attn(prm, tiles, hd, w, w + bytes, w + 2 * bytes, s)) != MOGA_OK) return st;
  }
  return MOGA_OK;
}

extern "C" moga_status moga_group_attn(const void* q, const void* k, const void* v, int64_t N, int32_t H, int32_t hd,
                                       const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                       const float* gate_prob, float softmax_scale, float* o_acc, void* ws,
                                       size_t ws_bytes, void* stream) {
  return moga_impl(q, k, v, N, 1, H, hd, perm, cu_seqlens, M, gate_prob, softmax_scale, o_acc, nullptr, ws, ws_bytes,
                   stream);
}

extern "C" moga_status moga_group_attn_batched(const void* q, const void* k, const void* v, int64_t n_per, int32_t B,
                                               int32_t H, int32_t hd, const int32_t* perm, const int32_t* cu_seqlens,
                                               int32_t M, const float* gate_prob, float softmax_scale, float* o_acc,
                                               float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (B < 1 || n_per <= 0 || n_per * B > INT32_MAX)
    return fail(MOGA_ERR_INVALID_ARG, "moga_group_attn_batched: B=%d x n_per=%lld out of range", B, (long long)n_per);
  return moga_impl(q, k, v, n_per * B, B, H, hd, perm, cu_seqlens, M, gate_prob, softmax_scale, o_acc, lse, ws,
                   ws_bytes, stream);
}

extern "C" moga_status moga_group_attn_train(const void* q, const void* k, const void* v, int64_t N, int32_t H,
                                             int32_t hd, const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                             const float* gate_prob, float softmax_scale, float* o_moga, float* lse,
                                             void* ws, size_t ws_bytes, void* stream) {
  if (!lse) return fail(MOGA_ERR_INVALID_ARG, "moga_group_attn_train: null lse");
  return moga_impl(q, k, v, N, 1, H, hd, perm, cu_seqlens, M, gate_prob, softmax_scale, o_moga, lse, ws, ws_bytes,
                   stream);
}

// Validates the STGA geometry and fills the static-branch fields of prm
// (temporal groups, window tiling, tile prefix); N = T*h*w.
static moga_status stga_params(const moga_stga_geom* geom, int32_t H, float softmax_scale, Params& prm,
                               int64_t& N, const char* who) {
  if (!geom || !geom->shot_len) return fail(MOGA_ERR_INVALID_ARG, "%s: null geometry", who);
  const moga_stga_geom& g = *geom;
  if (g.T <= 0 || g.h <= 0 || g.w <= 0 || g.win_h <= 0 || g.win_w <= 0 || g.n_shots <= 0 || g.tg_max < 0 ||
      g.aug_frames < 0)
    return fail(MOGA_ERR_INVALID_ARG, "%s: bad geometry", who);
  if (g.h % g.win_h || g.w % g.win_w) return fail(MOGA_ERR_INVALID_ARG, "%s: windows must tile the frame", who);
  long long tsum = 0;
  for (int s = 0; s < g.n_shots; ++s) {
    if (g.shot_len[s] <= 0) return fail(MOGA_ERR_INVALID_ARG, "%s: shot %d has length %d", who, s, g.shot_len[s]);
    tsum += g.shot_len[s];
  }
  if (tsum != g.T) return fail(MOGA_ERR_INVALID_ARG, "%s: shot lengths sum to %lld, T=%d", who, tsum, g.T);
  if (!(softmax_scale > 0.f)) return fail(MOGA_ERR_INVALID_ARG, "%s: softmax_scale must be > 0", who);
  N = (int64_t)g.T * g.h * g.w;
  if (N * (int64_t)H >= INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "%s: N*H out of range", who);
  std::vector<TGroup> tgs;
  build_temporal_groups(g, tgs);
  if ((int)tgs.size() > kMaxTG)
    return fail(MOGA_ERR_UNSUPPORTED, "%s: %zu temporal groups (max %d)", who, tgs.size(), kMaxTG);
  memset(&prm, 0, sizeof(prm));
  prm.N = (int)N;
  prm.H = H;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.T = g.T;
  prm.h = g.h;
  prm.w = g.w;
  prm.win_h = g.win_h;
  prm.win_w = g.win_w;
  prm.n_wx = g.w / g.win_w;
  prm.n_win = (g.h / g.win_h) * prm.n_wx;
  prm.whw = g.win_h * g.win_w;
  prm.hw = g.h * g.w;
  prm.n_tg = (int)tgs.size();
  prm.tg_tiles[0] = 0;
  for (int i = 0; i < prm.n_tg; ++i) {
    prm.tg[i] = tgs[i];
    const int qp = ceil_div((tgs[i].t1 - tgs[i].t0) * prm.whw, 2 * BM);
    prm.tg_tiles[i + 1] = prm.tg_tiles[i] + prm.n_win * H * qp;
  }
  fill_debug(prm);
  return MOGA_OK;
}

// o_win / o_frame: the same accumulator (added to) unless write is set, in
// which case each branch writes its own buffer; out: fused mean (frame pass).
static moga_status stga_impl(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                             const moga_stga_geom* geom, float softmax_scale, float* o_win, float* o_frame,
                             float* lse_win, float* lse_frame, bool write, void* out, void* ws, size_t ws_bytes,
                             void* stream, const char* who) {
  Params prm;
  int64_t N = 0;
  moga_status st = stga_params(geom, H, softmax_scale, prm, N, who);
  if (st != MOGA_OK) return st;
  if ((st = check_common(q, k, v, N, H, hd, o_win, ws, ws_bytes, true, who)) != MOGA_OK) return st;
  if (!o_frame || (reinterpret_cast<uintptr_t>(o_frame) & 15))
    return fail(MOGA_ERR_INVALID_ARG, "%s: frame output must be a 16-byte aligned pointer", who);
  if (out && (reinterpret_cast<uintptr_t>(out) & 15))
    return fail(MOGA_ERR_INVALID_ARG, "%s: out must be 16-byte aligned", who);
  prm.write_static = write ? 1 : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // window groups (gathered into window-major order), then frames (already
  // contiguous); both add into o_acc and stream order keeps them apart
  prm.mode = MODE_WINDOW;
  prm.o_acc = o_win;
  prm.lse = lse_win;
  if ((st = launch_gather(prm, hd, q, k, v, ws, s)) != MOGA_OK) return st;
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  const size_t bytes = (size_t)N * H * hd * 2;
  st = dispatch_attn(prm, prm.tg_tiles[prm.n_tg], hd, w, w + bytes, w + 2 * bytes, s);
  if (st != MOGA_OK) return st;
  prm.mode = MODE_FRAME;
  prm.o_acc = o_frame;
  prm.lse = lse_frame;
  prm.out = static_cast<__nv_bfloat16*>(out);
  return dispatch_attn(prm, prm.T * H * ceil_div(prm.hw, 2 * BM), hd, q, k, v, s);
}

extern "C" moga_status stga_attn(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                                 const moga_stga_geom* geom, float softmax_scale, float* o_acc, void* ws,
                                 size_t ws_bytes, void* stream) {
  return stga_impl(q, k, v, H, hd, geom, softmax_scale, o_acc, o_acc, nullptr, nullptr, false, nullptr, ws, ws_bytes,
                   stream, "stga_attn");
}

// B videos of the same geometry, video-major: one pair of launches per video
// on its slice of q, k, v and o_acc (the workspace is reused in stream order).
extern "C" moga_status stga_attn_batched(const void* q, const void* k, const void* v, int32_t B, int32_t H, int32_t hd,
                                         const moga_stga_geom* geom, float softmax_scale, float* o_acc, void* ws,
                                         size_t ws_bytes, void* stream) {
  if (B < 1) return fail(MOGA_ERR_INVALID_ARG, "stga_attn_batched: B=%d", B);
  if (!geom) return fail(MOGA_ERR_INVALID_ARG, "stga_attn_batched: null geometry");
  const int64_t n = (int64_t)geom->T * geom->h * geom->w;
  if (n * B * (int64_t)H >= INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "stga_attn_batched: B*N*H out of range");
  const size_t elems = (size_t)n * H * hd;
  for (int b = 0; b < B; ++b) {
    const size_t off = (size_t)b * elems * 2;
    moga_status st = stga_impl(static_cast<const uint8_t*>(q) + off, static_cast<const uint8_t*>(k) + off,
                               static_cast<const uint8_t*>(v) + off, H, hd, geom, softmax_scale, o_acc + b * elems,
                               o_acc + b * elems, nullptr, nullptr, false, nullptr, ws, ws_bytes, stream,
                               "stga_attn_batched");
    if (st != MOGA_OK) return st;
  }
  return MOGA_OK;
}

extern "C" moga_status stga_attn_mean(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                                      const moga_stga_geom* geom, float softmax_scale, float* o_acc, void* out,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (!out) return fail(MOGA_ERR_INVALID_ARG, "stga_attn_mean: null out");
  return stga_impl(q, k, v, H, hd, geom, softmax_scale, o_acc, o_acc, nullptr, nullptr, false, out, ws, ws_bytes,
                   stream, "stga_attn_mean");
}

// The three branches into one accumulator with a single gather pass:
// o_acc = MoGA (written), then windows and frames (added), as
// moga_group_attn followed by stga_attn on one stream, bit for bit.  The
// workspace holds both copies: [group order: Q, K, V][window order: Q, K, V].
extern "C" size_t visual_attn_ws_bytes(int64_t N, int32_t H, int32_t hd) {
  if (N <= 0 || H <= 0 || (hd != 64 && hd != 128) || N * (int64_t)H >= INT32_MAX) return 0;
  return 2 * attn_ws_bytes(N, H, hd);
}

extern "C" moga_status visual_attn_branches(const void* q, const void* k, const void* v, int64_t N, int32_t H,
                                            int32_t hd, const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                            const float* gate_prob, const moga_stga_geom* geom, float softmax_scale,
                                            float* o_acc, void* ws, size_t ws_bytes, void* stream) {
  const char* who = "visual_attn_branches";
  Params prm;
  int64_t n_geom = 0;
  moga_status st = stga_params(geom, H, softmax_scale, prm, n_geom, who);
  if (st != MOGA_OK) return st;
  if (n_geom != N) return fail(MOGA_ERR_INVALID_ARG, "%s: geometry has %lld tokens, N=%lld", who, (long long)n_geom,
                               (long long)N);
  if ((st = check_common(q, k, v, N, H, hd, o_acc, ws, ws_bytes, true, who)) != MOGA_OK) return st;
  if (ws_bytes < 2 * attn_ws_bytes(N, H, hd))
    return fail(MOGA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws_bytes, 2 * attn_ws_bytes(N, H, hd));
  if (!perm || !cu_seqlens || !gate_prob) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "%s: M=%d not in [1, 32]", who, M);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)N * H * hd * 2;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint8_t* wwin = w + 3 * bytes;
  prm.perm = perm;
  prm.cu = cu_seqlens;
  prm.M = M;
  prm.gate = gate_prob;
  prm.o_acc = o_acc;
  const int row_u4 = H * hd / 8;
  gather_both_kernel<<<ceil_div((int)N, 8), 256, 0, s>>>(
      prm, static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      reinterpret_cast<uint4*>(w), reinterpret_cast<uint4*>(w + bytes), reinterpret_cast<uint4*>(w + 2 * bytes),
      reinterpret_cast<uint4*>(wwin), reinterpret_cast<uint4*>(wwin + bytes),
      reinterpret_cast<uint4*>(wwin + 2 * bytes), row_u4);
  if ((st = check_launch("visual_attn_branches/gather")) != MOGA_OK) return st;
  // MoGA groups (written), as moga_group_attn
  prm.mode = MODE_MOGA;
  const int tiles = (ceil_div((int)N, 2 * BM) + M) * H;
  if ((st = dispatch_attn(prm, tiles, hd, w, w + bytes, w + 2 * bytes, s)) != MOGA_OK) return st;
  // windows and frames (added), as stga_attn
  prm.mode = MODE_WINDOW;
  if ((st = dispatch_attn(prm, prm.tg_tiles[prm.n_tg], hd, wwin, wwin + bytes, wwin + 2 * bytes, s)) != MOGA_OK)
    return st;
  prm.mode = MODE_FRAME;
  return dispatch_attn(prm, prm.T * H * ceil_div(prm.hw, 2 * BM), hd, q, k, v, s);
}

// Test hook (declared in include/moga_testing.h): the temporal groups the
// static-group launches use for a geometry, as (first frame, end frame,
// borrowed frames before, borrowed frames after) per group, in time order.
// Host code only: it validates the geometry exactly as stga_attn does and
// launches nothing.
extern "C" int32_t moga_test_stga_groups(const moga_stga_geom* geom, int32_t* out, int32_t cap) {
  Params prm;
  int64_t N = 0;
  if (stga_params(geom, 1, 1.0f, prm, N, "moga_test_stga_groups") != MOGA_OK) return -1;
  for (int i = 0; i < prm.n_tg && i < cap; ++i) {
    out[4 * i + 0] = prm.tg[i].t0;
    out[4 * i + 1] = prm.tg[i].t1;
    out[4 * i + 2] = prm.tg[i].a_prev;
    out[4 * i + 3] = prm.tg[i].a_next;
  }
  return prm.n_tg;
}

// Test hooks (include/moga_testing.h): the work tiles of one attention launch
// and the window-major token order, computed by the kernels' own index code
// (decode_tile, build_group_table, window_token) compiled for the host.
extern "C" int32_t moga_test_attn_tiles(int32_t mode, const int32_t* cu_seqlens, int32_t M, int64_t N, int32_t H,
                                        const moga_stga_geom* geom, int32_t* out, int32_t cap) {
  Params prm;
  if (mode == MODE_MOGA) {
    if (!cu_seqlens || M < 1 || M > 32 || N <= 0 || N > INT32_MAX || H <= 0) {
      fail(MOGA_ERR_INVALID_ARG, "moga_test_attn_tiles: bad MoGA arguments");
      return -1;
    }
    memset(&prm, 0, sizeof(prm));
    prm.N = (int)N;
    prm.H = H;
    prm.M = M;
    prm.cu = cu_seqlens;
  } else if (mode == MODE_WINDOW || mode == MODE_FRAME) {
    int64_t n = 0;
    if (stga_params(geom, H, 1.0f, prm, n, "moga_test_attn_tiles") != MOGA_OK) return -1;
  } else {
    fail(MOGA_ERR_INVALID_ARG, "moga_test_attn_tiles: mode %d", mode);
    return -1;
  }
  prm.mode = mode;
  GroupTable gt;
  memset(&gt, 0, sizeof(gt));
  if (mode == MODE_MOGA) build_group_table(prm, gt);
  int32_t n = 0;
  for (int L = 0;; ++L) {
    const Tile t = decode_tile(prm, gt, L);
    if (!t.valid) break;
    if (n < cap) {
      int32_t* o = out + 5 * (size_t)n;
      o[0] = t.head;
      o[1] = t.q_begin;
      o[2] = t.q_end;
      o[3] = t.kv_begin;
      o[4] = t.kv_end;
    }
    ++n;
  }
  return n;
}

extern "C" int32_t moga_test_window_tokens(const moga_stga_geom* geom, int32_t begin, int32_t end, int32_t* out) {
  Params prm;
  int64_t N = 0;
  if (stga_params(geom, 1, 1.0f, prm, N, "moga_test_window_tokens") != MOGA_OK) return -1;
  if (begin < 0 || end > N || begin > end) {
    fail(MOGA_ERR_INVALID_ARG, "moga_test_window_tokens: range [%d, %d) outside [0, %lld)", begin, end, (long long)N);
    return -1;
  }
  for (int i = begin; i < end; ++i) out[i - begin] = window_token(prm, i);
  return end - begin;
}

extern "C" moga_status stga_attn_train(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                                       const moga_stga_geom* geom, float softmax_scale, float* o_win, float* lse_win,
                                       float* o_frame, float* lse_frame, void* ws, size_t ws_bytes, void* stream) {
  if (!lse_win || !lse_frame) return fail(MOGA_ERR_INVALID_ARG, "stga_attn_train: null lse");
  return stga_impl(q, k, v, H, hd, geom, softmax_scale, o_win, o_frame, lse_win, lse_frame, true, nullptr, ws,
                   ws_bytes, stream, "stga_attn_train");
}
