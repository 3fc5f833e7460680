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
// Structure of one CTA (one 128-row query tile of one group and one head):
//   warps 0-3  softmax + epilogue: thread = query row = TMEM lane
//   warp  4    producer: TMA tile::gather4 of Q/K/V rows, rows chosen by an
//              index map (perm for MoGA, window arithmetic for STGA,
//              identity for frames); 128B-swizzled tiles
//   warp  5    TMEM allocator; lane 0 issues tcgen05.mma
// TMEM columns: S double buffer [0,128) and [128,256), O at [256, 256+hd).
// Pipeline per KV tile j: S_j = Q K_j^T (MMA) -> row max, exp2, P_j -> bf16
// into shared memory (softmax warps) -> O += P_j V_j (MMA).  The MMA of
// S_{j+1} overlaps the softmax of tile j.  The running max is only moved
// (and O rescaled) when it grows by more than 2^8, which keeps the result
// exact while skipping most rescales.
// Every wait is bounded; on a timeout the CTA records MOGA_ERR_TIMEOUT,
// drains what it has in flight, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"

namespace moga {
namespace attn {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // key/value rows per tile
constexpr int kThreads = 192;  // 6 warps
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
  // STGA geometry
  int T, h, w, win_h, win_w, n_wx, n_win, whw, hw;
  int n_tg;
  int tg_tiles[kMaxTG + 1];   // prefix of tiles over temporal groups
  TGroup tg[kMaxTG];
  long long timeout_cycles;
  int debug_flags;            // bit 0: producer skips the Q load (timeout test)
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false if the CTA is aborting or the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long timeout) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > timeout) {
      record_device_error(MOGA_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (draining in-flight copies).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, long long timeout) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > timeout) {
      record_device_error(MOGA_ERR_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, int col, int r0, int r1, int r2,
                                            int r3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread i gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, M = 128, A K-major.
__host__ __device__ constexpr uint32_t instr_desc(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// ------------------------------------------------------------------ index maps

struct Tile {
  int head, q_begin, q_end, kv_begin, kv_end;
  int valid;  // 0: this CTA has no work
};

__device__ __forceinline__ int token_of(const Params& p, int idx) {
  if (p.mode == MODE_MOGA) return __ldg(p.perm + idx);
  if (p.mode == MODE_FRAME) return idx;
  const int local = idx % p.whw;
  const int wf = idx / p.whw;
  const int frame = wf % p.T;
  const int win = wf / p.T;
  const int wy = win / p.n_wx, wx = win - wy * p.n_wx;
  const int row = wy * p.win_h + local / p.win_w;
  const int col = wx * p.win_w + local % p.win_w;
  return frame * p.hw + row * p.w + col;
}

// Decode blockIdx into a tile (thread 0 only; result shared via smem).
__device__ void decode_tile(const Params& p, int L, Tile& t) {
  t.valid = 0;
  if (p.mode == MODE_MOGA) {
    // largest groups first, then head, then query tile (K/V of one group and
    // head are reused by consecutive CTAs through L2)
    int size[32], order[32];
    for (int i = 0; i < p.M; ++i) {
      size[i] = __ldg(p.cu + i + 1) - __ldg(p.cu + i);
      order[i] = i;
    }
    for (int i = 1; i < p.M; ++i) {
      const int o = order[i];
      int j = i - 1;
      while (j >= 0 && size[order[j]] < size[o]) {
        order[j + 1] = order[j];
        --j;
      }
      order[j + 1] = o;
    }
    int rem = L;
    for (int k = 0; k < p.M; ++k) {
      const int g = order[k];
      const int qt = ceil_div(size[g], BM);
      const int n = qt * p.H;
      if (rem < n) {
        const int start = __ldg(p.cu + g);
        t.head = rem / qt;
        const int qi = rem - t.head * qt;
        t.q_begin = start + qi * BM;
        t.q_end = min(start + size[g], t.q_begin + BM);
        t.kv_begin = start;
        t.kv_end = start + size[g];
        t.valid = 1;
        return;
      }
      rem -= n;
    }
    return;
  }
  if (p.mode == MODE_FRAME) {
    const int qt = ceil_div(p.hw, BM);
    const int total = p.T * p.H * qt;
    if (L >= total) return;
    const int frame = L / (p.H * qt);
    const int rem = L - frame * p.H * qt;
    t.head = rem / qt;
    const int qi = rem - t.head * qt;
    t.kv_begin = frame * p.hw;
    t.kv_end = t.kv_begin + p.hw;
    t.q_begin = t.kv_begin + qi * BM;
    t.q_end = min(t.kv_end, t.q_begin + BM);
    t.valid = 1;
    return;
  }
  // window groups: temporal group, window, head, query tile
  if (L >= p.tg_tiles[p.n_tg]) return;
  int g = 0;
  while (p.tg_tiles[g + 1] <= L) ++g;
  const TGroup tg = p.tg[g];
  const int qlen = (tg.t1 - tg.t0) * p.whw;
  const int qt = ceil_div(qlen, BM);
  const int rem = L - p.tg_tiles[g];
  const int win = rem / (p.H * qt);
  const int rem2 = rem - win * p.H * qt;
  t.head = rem2 / qt;
  const int qi = rem2 - t.head * qt;
  const int base = win * p.T;
  t.q_begin = (base + tg.t0) * p.whw + qi * BM;
  t.q_end = min((base + tg.t1) * p.whw, t.q_begin + BM);
  t.kv_begin = (base + tg.t0 - tg.a_prev) * p.whw;
  t.kv_end = (base + tg.t1 + tg.a_next) * p.whw;
  t.valid = 1;
}

// ------------------------------------------------------------------ shared memory

template <int HD>
struct SmemLayout {
  static constexpr int kHalves = HD / 64;
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // one Q/K/V tile
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + kTileBytes;
  static constexpr int kV0 = kK0 + 2 * kTileBytes;
  static constexpr int kP = kV0 + 2 * kTileBytes;
  static constexpr int kBar = kP + 2 * kHalfBytes;
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kEnd = kMisc + 64;
  // 1 KB slack to align the dynamic base to 1024 bytes; HD = 64 is padded so
  // two CTAs never share an SM (each allocates all 512 TMEM columns)
  static constexpr int kBytes = (HD == 64 ? 120 * 1024 : kEnd) + 1024;
};

enum Bar : int {
  B_FULL_Q = 0,
  B_FULL_K = 1,   // +stage
  B_FULL_V = 3,   // +stage
  B_EMPTY_K = 5,  // +stage
  B_EMPTY_V = 7,  // +stage
  B_S_FULL = 9,   // +buffer
  B_S_FREE = 11,  // +buffer
  B_P_FULL = 13,
  B_O_DONE = 14,
  B_MMA_END = 15
};

// ------------------------------------------------------------------ the kernel

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
group_attn_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using S = SmemLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + S::kBar + 8u * (uint32_t)i; };
  int* misc = reinterpret_cast<int*>(smem + S::kMisc);
  volatile int* abort_flag = misc + 0;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
  Tile* tile_sh = reinterpret_cast<Tile*>(misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    Tile t;
    decode_tile(p, blockIdx.x, t);
    *tile_sh = t;
    *abort_flag = 0;
    mbar_init(bar(B_FULL_Q), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_FULL_K + s), 1);
      mbar_init(bar(B_FULL_V + s), 1);
      mbar_init(bar(B_EMPTY_K + s), 1);
      mbar_init(bar(B_EMPTY_V + s), 1);
      mbar_init(bar(B_S_FULL + s), 1);
      mbar_init(bar(B_S_FREE + s), BM);
    }
    mbar_init(bar(B_P_FULL), BM);
    mbar_init(bar(B_O_DONE), 1);
    mbar_init(bar(B_MMA_END), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const Tile t = *tile_sh;
  if (!t.valid) return;   // uniform across the CTA

  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 256;
  const long long timeout = p.timeout_cycles;
  const int n_kv = ceil_div(t.kv_end - t.kv_begin, BN);

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    // lane l gathers rows 4l .. 4l+3 of every tile
    auto rows_of = [&](int begin, int end, int* r) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = min(begin + 4 * lane + i, end - 1);
        r[i] = token_of(p, idx) * p.H + t.head;
      }
    };
    auto issue_tile = [&](const CUtensorMap* map, uint32_t dst, const int* r, uint32_t b) {
#pragma unroll
      for (int hh = 0; hh < S::kHalves; ++hh)
        tma_gather4(dst + hh * kHalfBytes + lane * 512, map, hh * 64, r[0], r[1], r[2], r[3], b);
    };
    bool ok = true;
    int issued_k[2] = {-1, -1}, issued_v[2] = {-1, -1};
    const bool skip_q = (p.debug_flags & 1) != 0;
    if (!skip_q) {
      int r[4];
      rows_of(t.q_begin, t.q_end, r);
      if (lane == 0) mbar_arrive_expect_tx(bar(B_FULL_Q), S::kTileBytes);
      __syncwarp();
      issue_tile(&tm_q, sbase + S::kQ, r, bar(B_FULL_Q));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      int r[4];
      rows_of(t.kv_begin + j * BN, t.kv_end, r);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_EMPTY_K + st), ph ^ 1, abort_flag, timeout));
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(bar(B_FULL_K + st), S::kTileBytes);
      __syncwarp();
      issue_tile(&tm_k, sbase + S::kK0 + st * S::kTileBytes, r, bar(B_FULL_K + st));
      issued_k[st] = j;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_EMPTY_V + st), ph ^ 1, abort_flag, timeout));
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(bar(B_FULL_V + st), S::kTileBytes);
      __syncwarp();
      issue_tile(&tm_v, sbase + S::kV0 + st * S::kTileBytes, r, bar(B_FULL_V + st));
      issued_v[st] = j;
    }
    // let every copy this warp started land before the CTA can exit
    if (!skip_q) mbar_drain(bar(B_FULL_Q), 0, timeout);
    for (int st = 0; st < 2; ++st) {
      if (issued_k[st] >= 0) mbar_drain(bar(B_FULL_K + st), (issued_k[st] >> 1) & 1, timeout);
      if (issued_v[st] >= 0) mbar_drain(bar(B_FULL_V + st), (issued_v[st] >> 1) & 1, timeout);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = instr_desc(BN, false);
      constexpr uint32_t idesc_pv = instr_desc(HD, true);
      bool ok = mbar_wait(bar(B_FULL_Q), 0, abort_flag, timeout);
      auto issue_pv = [&](int i) -> bool {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(bar(B_FULL_V + st), ph, abort_flag, timeout)) return false;
        if (!mbar_wait(bar(B_P_FULL), i & 1, abort_flag, timeout)) return false;
        tc_fence_after();
        const uint32_t pa = sbase + S::kP;
        const uint32_t va = sbase + S::kV0 + st * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t ad = smem_desc(pa + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(va + ks * 16 * 128, kHalfBytes, 1024);
          tc_mma(tmem_o, ad, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_O_DONE));
        tc_commit(bar(B_EMPTY_V + st));
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        ok = mbar_wait(bar(B_FULL_K + st), ph, abort_flag, timeout) &&
             mbar_wait(bar(B_S_FREE + st), ph ^ 1, abort_flag, timeout);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = sbase + S::kQ;
        const uint32_t ka = sbase + S::kK0 + st * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint64_t ad = smem_desc(qa + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(ka + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
          tc_mma(tmem + st * 128, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_S_FULL + st));
        tc_commit(bar(B_EMPTY_K + st));
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(n_kv - 1);
      // every MMA this thread issued has finished before TMEM is released
      tc_commit(bar(B_MMA_END));
      mbar_drain(bar(B_MMA_END), 0, timeout);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    const int row = warp * 32 + lane;                    // TMEM lane == query row
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const float sl = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    uint8_t* prow = smem + S::kP + row * 128;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + sb), ph, abort_flag, timeout));
      if (!ok) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem + lane_addr + sb * 128 + c * 32, s + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE + sb));
      const int valid = t.kv_end - (t.kv_begin + j * BN);
      if (valid < BN) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl);
      if (j > 0) {
        // PV_{j-1} has finished: P may be overwritten and O rescaled
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_DONE), (j - 1) & 1, abort_flag, timeout));
        if (!ok) break;
        tc_fence_after();
        const bool need = m_new > m_run + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            float o[32];
            tmem_ld32(tmem_o + lane_addr + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= f;
            tmem_st32(tmem_o + lane_addr + c * 32, o);
          }
          tmem_wait_st();
          if (need) {
            l_run *= f;
            m_run = m_new;
          }
        }
      } else {
        m_run = m_new;
      }
      float sum = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < BN / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = fast_exp2(fmaf(s[c8 * 8 + 2 * i], sl, -m_run));
          const float b = fast_exp2(fmaf(s[c8 * 8 + 2 * i + 1], sl, -m_run));
          sum += a + b;
          __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
          w[i] = *reinterpret_cast<uint32_t*>(&pr);
        }
        const int half = c8 >> 3, chunk = c8 & 7;
        const int off = half * kHalfBytes + ((chunk ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l_run += sum;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_DONE), (n_kv - 1) & 1, abort_flag, timeout));
    if (ok) {
      tc_fence_after();
      const int q_idx = t.q_begin + row;
      const bool live = q_idx < t.q_end;
      float scale = 0.f;
      float* dst = nullptr;
      if (live) {
        const int tok = token_of(p, q_idx);
        scale = 1.0f / l_run;
        if (p.mode == MODE_MOGA) scale *= __ldg(p.gate + tok);
        dst = p.o_acc + ((size_t)tok * p.H + t.head) * HD;
      }
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tmem_o + lane_addr + c * 32, o);
        tmem_wait_ld();
        if (live) {
          float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
          if (p.mode == MODE_MOGA) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(o[4 * i] * scale, o[4 * i + 1] * scale, o[4 * i + 2] * scale, o[4 * i + 3] * scale);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 a = d4[i];
              a.x = fmaf(o[4 * i], scale, a.x);
              a.y = fmaf(o[4 * i + 1], scale, a.y);
              a.z = fmaf(o[4 * i + 2], scale, a.z);
              a.w = fmaf(o[4 * i + 3], scale, a.w);
              d4[i] = a;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
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

// [rows = N*H][hd] bf16 view, box of 64 columns x 1 row, 128-byte swizzle.
static moga_status make_row_map(CUtensorMap* m, const void* base, int64_t rows, int hd) {
  auto fn = encode_fn();
  if (!fn) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gdim[2] = {(cuuint64_t)hd, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)hd * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOGA_OK;
}

static long long default_timeout_cycles() {
  // about two seconds at the maximum SM clock
  return 4000000000LL;
}

template <int HD>
static moga_status launch(const Params& prm, int grid, const void* q, const void* k, const void* v,
                          cudaStream_t s) {
  using S = SmemLayout<HD>;
  cudaError_t e = cudaFuncSetAttribute(group_attn_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  CUtensorMap mq, mk, mv;
  const int64_t rows = (int64_t)prm.N * prm.H;
  moga_status st;
  if ((st = make_row_map(&mq, q, rows, HD)) != MOGA_OK) return st;
  if ((st = make_row_map(&mk, k, rows, HD)) != MOGA_OK) return st;
  if ((st = make_row_map(&mv, v, rows, HD)) != MOGA_OK) return st;
  if (grid <= 0) return MOGA_OK;
  group_attn_kernel<HD><<<grid, kThreads, S::kBytes, s>>>(prm, mq, mk, mv);
  return check_launch("group attention kernel");
}

static moga_status check_common(const void* q, const void* k, const void* v, int64_t N, int H, int hd,
                                const float* o_acc, const char* who) {
  if (!q || !k || !v || !o_acc) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (N <= 0 || H <= 0 || N * (int64_t)H >= INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "%s: N*H out of range", who);
  if (hd != 64 && hd != 128) return fail(MOGA_ERR_UNSUPPORTED, "%s: head_dim %d (supported: 64, 128)", who, hd);
  const uintptr_t a = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                      reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o_acc);
  if (a & 15) return fail(MOGA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  return MOGA_OK;
}

static moga_status dispatch(const Params& prm, int grid, int hd, const void* q, const void* k, const void* v,
                            cudaStream_t s) {
  return hd == 128 ? launch<128>(prm, grid, q, k, v, s) : launch<64>(prm, grid, q, k, v, s);
}

// Temporal groups of the static window branch (as-equal-as-possible runs of
// at most tg_max frames inside each shot, longer runs first; adjacent-shot
// frames on the K/V side at each cut).
static moga_status build_temporal_groups(const moga_stga_geom& g, std::vector<TGroup>& out) {
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
  return MOGA_OK;
}

}  // namespace attn
}  // namespace moga

using namespace moga;
using namespace moga::attn;

// Test hook (not declared in the public header): bounded-wait timeout in SM
// cycles and debug flags for the next group-attention launch on this thread.
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

extern "C" moga_status moga_group_attn(const void* q, const void* k, const void* v, int64_t N, int32_t H, int32_t hd,
                                       const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                       const float* gate_prob, float softmax_scale, float* o_acc, void* stream) {
  moga_status st = check_common(q, k, v, N, H, hd, o_acc, "moga_group_attn");
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
  fill_debug(prm);
  // upper bound on the tile count: sum_i ceil(n_i / BM) <= N / BM + M
  const int grid = (ceil_div((int)N, BM) + M) * H;
  return dispatch(prm, grid, hd, q, k, v, static_cast<cudaStream_t>(stream));
}

extern "C" moga_status stga_attn(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                                 const moga_stga_geom* geom, float softmax_scale, float* o_acc, void* stream) {
  if (!geom || !geom->shot_len) return fail(MOGA_ERR_INVALID_ARG, "stga_attn: null geometry");
  const moga_stga_geom& g = *geom;
  if (g.T <= 0 || g.h <= 0 || g.w <= 0 || g.win_h <= 0 || g.win_w <= 0 || g.n_shots <= 0 || g.tg_max < 0 ||
      g.aug_frames < 0)
    return fail(MOGA_ERR_INVALID_ARG, "stga_attn: bad geometry");
  if (g.h % g.win_h || g.w % g.win_w) return fail(MOGA_ERR_INVALID_ARG, "stga_attn: windows must tile the frame");
  long long tsum = 0;
  for (int s = 0; s < g.n_shots; ++s) {
    if (g.shot_len[s] <= 0) return fail(MOGA_ERR_INVALID_ARG, "stga_attn: shot %d has length %d", s, g.shot_len[s]);
    tsum += g.shot_len[s];
  }
  if (tsum != g.T) return fail(MOGA_ERR_INVALID_ARG, "stga_attn: shot lengths sum to %lld, T=%d", tsum, g.T);
  const int64_t N = (int64_t)g.T * g.h * g.w;
  moga_status st = check_common(q, k, v, N, H, hd, o_acc, "stga_attn");
  if (st != MOGA_OK) return st;
  if (!(softmax_scale > 0.f)) return fail(MOGA_ERR_INVALID_ARG, "stga_attn: softmax_scale must be > 0");
  std::vector<TGroup> tgs;
  build_temporal_groups(g, tgs);
  if ((int)tgs.size() > kMaxTG)
    return fail(MOGA_ERR_UNSUPPORTED, "stga_attn: %zu temporal groups (max %d)", tgs.size(), kMaxTG);

  Params prm;
  memset(&prm, 0, sizeof(prm));
  prm.N = (int)N;
  prm.H = H;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.o_acc = o_acc;
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
    const int qt = ceil_div((tgs[i].t1 - tgs[i].t0) * prm.whw, BM);
    prm.tg_tiles[i + 1] = prm.tg_tiles[i] + prm.n_win * H * qt;
  }
  fill_debug(prm);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // window groups, then frames: both add into o_acc; stream order keeps them apart
  prm.mode = MODE_WINDOW;
  st = dispatch(prm, prm.tg_tiles[prm.n_tg], hd, q, k, v, s);
  if (st != MOGA_OK) return st;
  prm.mode = MODE_FRAME;
  return dispatch(prm, g.T * H * ceil_div(prm.hw, BM), hd, q, k, v, s);
}
