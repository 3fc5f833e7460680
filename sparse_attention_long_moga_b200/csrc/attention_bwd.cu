// Backward of the grouped attention on sm_100a, for the three branches of the
// layer (MoGA groups, STGA windows, frames).
//
// What it computes (MoGA note, key designs 1 and 3: the layer is trained end
// to end, the gate p(g(x)|x) multiplying the MoGA output is how the router
// gets its gradient).  Per group and head, with S = Q K^T * scale,
// P = softmax(S), O = P V and an upstream gradient dO of the attention
// output:  dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),
// dS = P * (dP - D),  dQ = dS K * scale,  dK = dS^T Q * scale.
// The layer's upstream gradient dout reaches each branch through the mean
// (1/3) and, for MoGA, the gate: dO = c * dout with c = p_g / 3 (MoGA) or
// 1/3 (static).  c is applied in fp32 inside the kernels, folded into the
// exponent (2^(S sl - lse + log2 c) = c P), so the bf16 copy of dout is
// exact; the softmax scale of dS is applied to dK and dQ in the epilogues.  D is taken as c * D' with
// D' = rowsum(dout * O_attn); for MoGA O_attn = o_moga / p_g, which also gives
// the gate's gradient  dgate[t] = sum_h D'[t, h] / 3.
//
// Kernels per branch:
//   bwd_prep_kernel   one warp per segment position: Q, K, V and dout rows
//                     into segment order (as the forward's gather), and the
//                     per-row statistics the tiles need: the forward's
//                     log-sum-exp, D' and c (and dgate for MoGA)
//   bwd_dkdv_kernel   one CTA per (segment, head, 128-key tile): loops over
//                     the segment's queries in 64-row halves of 128-row
//                     tiles; S^T = K Q^T and dP^T = V dO^T on tcgen05 (keys
//                     on the TMEM lanes, so c P^T and dS^T come out as the A
//                     operand of the next two products), then dV += (c P)^T dO
//                     and dK += dS^T Q accumulate in TMEM; two TMEM buffers,
//                     so the products of one half overlap the exponentials of
//                     the other; the epilogue adds dV, dK into dv, dk
//   bwd_dq_kernel     one CTA per (segment, head, 128-query tile): Q and dO
//                     copied once into TMEM as bf16 pairs (the A operands of
//                     S = Q K^T and dP = dO V^T), the segment's keys streamed
//                     in 64-row halves, dQ += dS K in TMEM; the epilogue adds
//                     into dq
// Both: warps 0-3 compute (thread = TMEM lane), warp 4 TMA producer, warp 5
// TMEM allocator and MMA issuer.  All waits are bounded.
//
// P is recomputed as 2^(S * scale * log2(e) - lse) with lse from the forward
// (log2 domain), so no row max is needed here.

namespace moga {
namespace attn {

struct BwdParams {
  Params f;               // branch, geometry, perm / cu / gate, N, H, scale_log2
  float scale;            // softmax scale
  const float* lse_seg;   // [N][H] forward log-sum-exp (log2 domain) less log2 c, segment order
  const float* dd_seg;    // [N][H] D' = rowsum(dout * O_attn), segment order
  float* dq;              // [N][H][hd] fp32, token order, added to
  float* dk;
  float* dv;
  int q_units[kMaxTG + 1];    // window branch: prefix of 128-query-tile units over temporal groups
  int kv_units[kMaxTG + 1];   // window branch: prefix of 128-key-tile units over temporal groups
};

// One work unit: a 128-row tile [t_begin, t_end) (queries for dQ, keys for
// dK/dV) of one segment and head; the segment's query rows are
// [q_begin, q_end) and its key rows [kv_begin, kv_end), in segment order.
struct Unit {
  int head, q_begin, q_end, kv_begin, kv_end, t_begin, t_end;
  int valid;
};

// KEYS: tile over the key range (dK/dV) instead of the query range (dQ).
template <bool KEYS>
__host__ __device__ __forceinline__ Unit decode_unit(const BwdParams& b, const GroupTable& gt, int L) {
  const Params& p = b.f;
  Unit u;
  u.valid = 0;
  if (p.mode == MODE_MOGA) {
    if (L >= gt.prefix[gt.n]) return u;
    int k = 0;
    while (gt.prefix[k + 1] <= L) ++k;
    const int nt = ceil_div(gt.size[k], BM);
    const int rem = L - gt.prefix[k];
    u.head = rem / nt;
    const int ti = rem - u.head * nt;
    u.q_begin = u.kv_begin = gt.start[k];
    u.q_end = u.kv_end = gt.start[k] + gt.size[k];
    u.t_begin = u.q_begin + ti * BM;
    u.t_end = min(u.q_end, u.t_begin + BM);
    u.valid = 1;
    return u;
  }
  if (p.mode == MODE_FRAME) {
    const int nt = ceil_div(p.hw, BM);
    if (L >= p.T * p.H * nt) return u;
    const int frame = L / (p.H * nt);
    const int rem = L - frame * p.H * nt;
    u.head = rem / nt;
    const int ti = rem - u.head * nt;
    u.q_begin = u.kv_begin = frame * p.hw;
    u.q_end = u.kv_end = u.q_begin + p.hw;
    u.t_begin = u.q_begin + ti * BM;
    u.t_end = min(u.q_end, u.t_begin + BM);
    u.valid = 1;
    return u;
  }
  // window groups: temporal group, window, head, tile
  const int* pre = KEYS ? b.kv_units : b.q_units;
  if (L >= pre[p.n_tg]) return u;
  int g = 0;
  while (pre[g + 1] <= L) ++g;
  const TGroup tg = p.tg[g];
  const int qlen = (tg.t1 - tg.t0) * p.whw;
  const int kvlen = (tg.t1 - tg.t0 + tg.a_prev + tg.a_next) * p.whw;
  const int nt = ceil_div(KEYS ? kvlen : qlen, BM);
  const int rem = L - pre[g];
  const int win = rem / (p.H * nt);
  const int rem2 = rem - win * p.H * nt;
  u.head = rem2 / nt;
  const int ti = rem2 - u.head * nt;
  const int base = win * p.T;
  u.q_begin = (base + tg.t0) * p.whw;
  u.q_end = (base + tg.t1) * p.whw;
  u.kv_begin = (base + tg.t0 - tg.a_prev) * p.whw;
  u.kv_end = (base + tg.t1 + tg.a_next) * p.whw;
  const int r0 = KEYS ? u.kv_begin : u.q_begin, r1 = KEYS ? u.kv_end : u.q_end;
  u.t_begin = r0 + ti * BM;
  u.t_end = min(r1, u.t_begin + BM);
  u.valid = 1;
  return u;
}

// ------------------------------------------------------------------ prep

// One warp per segment position j.  Copies the Q, K, V and dout rows of the
// token at position j into segment order (not for frames, already in order),
// and writes lse_seg (the forward's log-sum-exp less log2 c, so that
// 2^(S sl - lse_seg) = c P) and dd_seg (D'); MoGA also writes dgate.
template <int MODE>
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const __grid_constant__ BwdParams b, const uint4* __restrict__ q, const uint4* __restrict__ k,
                const uint4* __restrict__ v, const uint4* __restrict__ dout, const float* __restrict__ o_branch,
                const float* __restrict__ lse, uint4* __restrict__ qd, uint4* __restrict__ kd, uint4* __restrict__ vd,
                uint4* __restrict__ dod, float* __restrict__ lse_seg, float* __restrict__ dd_seg,
                float* __restrict__ dgate, int hd) {
  const Params& p = b.f;
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= p.N) return;
  const int lane = threadIdx.x & 31;
  const int src = MODE == MODE_MOGA ? __ldg(p.perm + j) : (MODE == MODE_WINDOW ? window_token(p, j) : j);
  if (kCheckIndices && (unsigned)src >= (unsigned)p.N) {
    if (lane == 0) record_device_error(MOGA_ERR_BAD_INDEX);
    return;
  }
  const int row_u4 = p.H * hd / 8;
  const size_t so = (size_t)src * row_u4, dofs = (size_t)j * row_u4;
  if (MODE != MODE_FRAME) {
    for (int c = lane; c < row_u4; c += 32) {
      const uint4 a = __ldg(q + so + c), bb = __ldg(k + so + c), e = __ldg(v + so + c), f = __ldg(dout + so + c);
      qd[dofs + c] = a;
      kd[dofs + c] = bb;
      vd[dofs + c] = e;
      dod[dofs + c] = f;
    }
  }
  // D'[h] = sum_d dout[src][h][d] * o[src][h][d] (/ gate for MoGA): each lane
  // takes 8 consecutive elements; hd / 8 lanes cover one head
  const float gsc = MODE == MODE_MOGA ? __ldg(p.gate + src) : 1.0f;
  const float log2c = log2f(gsc / 3.0f);   // c = gate / 3 (MoGA) or 1 / 3
  const int lph = hd / 8;              // lanes per head
  const float4* orow = reinterpret_cast<const float4*>(o_branch) + (size_t)src * p.H * hd / 4;
  float dsum = 0.f;
  for (int c0 = 0; c0 < row_u4; c0 += 32) {
    const int c = c0 + lane;
    float part = 0.f;
    if (c < row_u4) {
      const uint4 du = __ldg(dout + so + c);
      const float4 o0 = __ldg(orow + 2 * c), o1 = __ldg(orow + 2 * c + 1);
      const uint32_t w[4] = {du.x, du.y, du.z, du.w};
      const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        part = fmaf(__uint_as_float(w[i] << 16), ov[2 * i], part);
        part = fmaf(__uint_as_float(w[i] & 0xFFFF0000u), ov[2 * i + 1], part);
      }
    }
    // reduce over the lanes of one head (lph = 8 or 16 consecutive lanes)
    for (int off = lph / 2; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (c < row_u4 && (lane % lph) == 0) {
      const int h = c / lph;
      const float dd = part / gsc;
      dd_seg[(size_t)j * p.H + h] = dd;
      lse_seg[(size_t)j * p.H + h] = __ldg(lse + (size_t)src * p.H + h) - log2c;
      dsum += dd;
    }
  }
  if (MODE == MODE_MOGA) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (lane == 0) dgate[src] = dsum / 3.0f;
  }
}

// ------------------------------------------------------------------ shared pieces

template <int HD>
struct BwdSmem {
  static constexpr int kTile = SmemLayout<HD>::kTileBytes;   // one 128-row tile
  // dK/dV kernel: K, V resident, two stages of (Q, dO); dQ kernel: Q, dO
  // resident, two stages of (K, V).  Same footprint.
  static constexpr int kRes0 = 0, kRes1 = kTile;               // resident tiles
  static constexpr int kStageA = 2 * kTile;                    // + s * kTile (Q or K)
  static constexpr int kStageB = 4 * kTile;                    // + s * kTile (dO or V)
  static constexpr int kStats = 6 * kTile;                     // [2][3][128] fp32 (dK/dV kernel)
  static constexpr int kBar = kStats + 2 * 3 * BM * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTable = kMisc + 64;
  static constexpr int kEnd = kTable + (int)sizeof(GroupTable);
  static constexpr int kBytes = kEnd + 1024;
  static_assert(kBytes <= 227 * 1024, "backward shared memory");
};

enum BwdBar : int {
  BB_RES = 0,        // resident tiles landed
  BB_FULL = 1,       // +stage: streamed tiles landed
  BB_EMPTY = 3,      // +stage: streamed tiles consumed by the MMAs
  BB_S = 5,          // +buffer: S (and dP) products of a 64-wide half tile in TMEM
  BB_P = 7,          // +buffer: compute wrote the bf16 operands of that half (128 arrivals)
  BB_DONE = 9,       // accumulators final
  BB_END = 10,       // every MMA finished (teardown)
  BB_A = 11,         // resident operands copied into TMEM (128 arrivals)
  BB_STATS = 12,     // +stage: a query tile's statistics landed (dK/dV; 32 cp.async arrivals)
  BB_COUNT = 14
};
static_assert(BB_COUNT <= BwdSmem<128>::kNumBars, "barrier area");

// Statistics of a row past the segment: an exponent offset that makes c P
// exactly 0, and D' = 0 (source of the cp.async that fills such rows).
__device__ float g_bwd_stat_pad[2] = {3.0e38f, 0.0f};

__device__ __forceinline__ void cp_async4(uint32_t dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// arrive on bar once this thread's earlier cp.async copies have landed (the
// barrier's count includes the arrival)
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint32_t bwd_pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// fp32 gradient rows g (this lane's row; tok < 0: none) added into
// dst[token][head][:] with fire-and-forget vector reductions (keys shared by
// two window groups receive two contributions).  Called by all 32 lanes of a
// warp: per 32-column chunk each lane puts its row into the warp's 4 KB
// stage (16-byte chunk k of row r at slot k ^ (r & 7), free of bank
// conflicts), then each reduction covers four rows of 128 bytes, eight lanes
// per row, instead of 32 scattered rows.
template <int HD>
__device__ __forceinline__ void add_rows(float* dst, int tok, int H, int head, const float* g, float4* stage,
                                         int lane) {
  const int sub = lane & 7;
#pragma unroll
  for (int cc = 0; cc < HD / 32; ++cc) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      stage[lane * 8 + (k ^ (lane & 7))] =
          make_float4(g[cc * 32 + 4 * k], g[cc * 32 + 4 * k + 1], g[cc * 32 + 4 * k + 2], g[cc * 32 + 4 * k + 3]);
    __syncwarp();
#pragma unroll
    for (int r4 = 0; r4 < 8; ++r4) {
      const int rr = r4 * 4 + (lane >> 3);   // row of this warp written by this lane
      const int tr = __shfl_sync(0xffffffffu, tok, rr);
      const float4 v = stage[rr * 8 + (sub ^ (rr & 7))];
      if (tr >= 0) {
        float4* d = reinterpret_cast<float4*>(dst + ((size_t)tr * H + head) * HD + cc * 32) + sub;
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(d), "f"(v.x), "f"(v.y), "f"(v.z),
                     "f"(v.w)
                     : "memory");
      }
    }
    __syncwarp();
  }
}

// Common prologue of both kernels: barriers, group table, TMEM (512 columns).
// Returns false (uniformly) when this CTA has no unit.
template <int HD, bool KEYS>
__device__ __forceinline__ bool bwd_setup(const BwdParams& b, uint8_t* smem, uint32_t sbase, Unit& u,
                                          uint32_t& tmem) {
  using SM = BwdSmem<HD>;
  int* misc = reinterpret_cast<int*>(smem + SM::kMisc);
  GroupTable* gt = reinterpret_cast<GroupTable*>(smem + SM::kTable);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    misc[0] = 0;   // abort flag
    if (b.f.mode == MODE_MOGA) build_group_table(b.f, *gt, BM);
    const uint32_t bar0 = sbase + SM::kBar;
    mbar_init(bar0 + 8 * BB_RES, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar0 + 8 * (BB_FULL + s), 1);
      mbar_init(bar0 + 8 * (BB_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar0 + 8 * (BB_S + s), 1);
      mbar_init(bar0 + 8 * (BB_P + s), BM);
    }
    mbar_init(bar0 + 8 * BB_DONE, 1);
    mbar_init(bar0 + 8 * BB_END, 1);
    mbar_init(bar0 + 8 * BB_A, BM);
    for (int s = 0; s < 2; ++s) mbar_init(bar0 + 8 * (BB_STATS + s), 32);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  u = decode_unit<KEYS>(b, *gt, blockIdx.x);
  if (!u.valid) return false;
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(reinterpret_cast<uint32_t*>(misc + 1))),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = *reinterpret_cast<volatile uint32_t*>(misc + 1);
  return true;
}

template <int HD>
__device__ __forceinline__ void bwd_teardown(uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
}

// TMA of one 128-row tile (rows r0.., all hd columns of one head) into dst.
template <int HD>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, int head, int r0, uint32_t bar) {
#pragma unroll
  for (int hh = 0; hh < HD / 64; ++hh) tma_load_3d(dst + hh * kHalfBytes, map, hh * 64, head, r0, bar);
}

// S-type product over a 64-wide half: D[128 x 64] = A[128 x HD] . B[64 x HD]^T,
// B the rows [64 half, 64 half + 64) of a K-major 128-row tile.
template <int HD>
__device__ __forceinline__ void mma_nt_half(uint32_t d_tmem, uint32_t a, uint32_t bt, int half) {
  constexpr uint32_t idesc = instr_desc(BN / 2, false);
  const uint32_t b = bt + half * (BN / 2) * 128;
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) {
    const uint64_t ad = smem_desc(a + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
    const uint64_t bd = smem_desc(b + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
    tc_mma_ss(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
  }
}

// Accumulating product over a 64-deep half: D[128 x HD] (+)= A[128 x 64] .
// B[64 x HD], A in TMEM (bf16 pairs, 32 columns), B the rows [64 half, ...)
// of an MN-major 128-row tile.
template <int HD>
__device__ __forceinline__ void mma_tn_half(uint32_t d_tmem, uint32_t a_tmem, uint32_t b, int half, bool acc) {
  constexpr uint32_t idesc = instr_desc(HD, true);
#pragma unroll
  for (int ks = 0; ks < BN / 32; ++ks) {
    const uint64_t bd = smem_desc(b + (half * (BN / 2) + ks * 16) * 128, kHalfBytes, 1024);
    tc_mma_ts(d_tmem, a_tmem + ks * 8, bd, idesc, (acc || ks > 0) ? 1u : 0u);
  }
}

// Row `row` of a 128-row SW128 tile in shared memory (HD columns in 64-column
// halves) into TMEM as bf16 pairs: column c holds elements 2c, 2c+1, the
// layout of an A operand in tensor memory.  Called by the thread whose TMEM
// lane is `row`.
template <int HD>
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int row, uint32_t taddr) {
#pragma unroll
  for (int hh = 0; hh < HD / 64; ++hh) {
    const uint8_t* base = tile + hh * kHalfBytes + row * 128;
    float w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + ((c ^ (row & 7)) << 4));
      w[4 * c] = __uint_as_float(v.x);
      w[4 * c + 1] = __uint_as_float(v.y);
      w[4 * c + 2] = __uint_as_float(v.z);
      w[4 * c + 3] = __uint_as_float(v.w);
    }
    tmem_st32(taddr + hh * 32, w);
  }
}

// S-type product over a 64-wide half with A in TMEM: D[128 x 64] = A[128 x HD]
// (bf16 pairs) . B[64 x HD]^T, B the rows [64 half, ...) of a K-major tile.
// Only B is read from shared memory (2 KB per MMA instead of 6 KB).
template <int HD>
__device__ __forceinline__ void mma_ts_half(uint32_t d_tmem, uint32_t a_tmem, uint32_t bt, int half) {
  constexpr uint32_t idesc = instr_desc(BN / 2, false);
  const uint32_t b = bt + half * (BN / 2) * 128;
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) {
    const uint64_t bd = smem_desc(b + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
    tc_mma_ts(d_tmem, a_tmem + ks * 8, bd, idesc, ks > 0 ? 1u : 0u);
  }
}

// ------------------------------------------------------------------ dK, dV

// TMEM: two 128-column buffers for 64-query halves (S^T at +0, dP^T at +64;
// c P^T and dS^T overwrite the first 32 columns of each), dV [256, 256 + HD),
// dK [256 + HD, 256 + 2 HD).  K and V stay in shared memory: copying them into
// TMEM as A operands leaves room for one buffer only at HD = 128, and the
// exponentials then no longer overlap the products (measured slower).
template <int HD>
__global__ void __launch_bounds__(192, 1)
bwd_dkdv_kernel(const __grid_constant__ BwdParams b, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_do) {
  using SM = BwdSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + SM::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<int*>(smem + SM::kMisc);
  float* stats = reinterpret_cast<float*>(smem + SM::kStats);   // [2][2][BM]: lse - log2 c, D'
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long timeout = b.f.timeout_cycles;
  const Params& p = b.f;
  Unit u;
  uint32_t tmem;
  if (!bwd_setup<HD, true>(b, smem, sbase, u, tmem)) return;
  const int n_q = ceil_div(u.q_end - u.q_begin, BM);

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    bool ok = true;
    int last[2] = {-1, -1};
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(BB_RES), 2 * SM::kTile);
      load_tile<HD>(sbase + SM::kRes0, &tm_k, u.head, u.t_begin, bar(BB_RES));
      load_tile<HD>(sbase + SM::kRes1, &tm_v, u.head, u.t_begin, bar(BB_RES));
    }
    for (int i = 0; i < n_q && ok; ++i) {
      const int s = i & 1;
      const uint32_t ph = (i >> 1) & 1;
      ok = __shfl_sync(0xffffffffu, lane == 0 ? (int)mbar_wait(bar(BB_EMPTY + s), ph ^ 1, abort_flag, timeout) : 0, 0);
      if (!ok) break;
      const int r0 = u.q_begin + i * BM;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(BB_FULL + s), 2 * SM::kTile);
        load_tile<HD>(sbase + SM::kStageA + s * SM::kTile, &tm_q, u.head, r0, bar(BB_FULL + s));
        load_tile<HD>(sbase + SM::kStageB + s * SM::kTile, &tm_do, u.head, r0, bar(BB_FULL + s));
        last[s] = i;
      }
      // the tile's per-query statistics (lse - log2 c, D'), 4 rows per lane,
      // by asynchronous copies that complete on BB_STATS; rows past the
      // segment copy the pad values, so their c P and dS are exactly 0
      const uint32_t st = sbase + SM::kStats + (uint32_t)(s * 2 * BM * 4);
#pragma unroll
      for (int e = 0; e < BM / 32; ++e) {
        const int qi = lane + 32 * e, r = r0 + qi;
        const bool in = r < u.q_end;
        cp_async4(st + qi * 4, in ? b.lse_seg + (size_t)r * p.H + u.head : &g_bwd_stat_pad[0]);
        cp_async4(st + (BM + qi) * 4, in ? b.dd_seg + (size_t)r * p.H + u.head : &g_bwd_stat_pad[1]);
      }
      cp_async_arrive_noinc(bar(BB_STATS + s));
    }
    cp_async_wait_all();
    if (lane == 0) {
      mbar_drain(bar(BB_RES), 0, timeout);
      for (int s = 0; s < 2; ++s)
        if (last[s] >= 0) mbar_drain(bar(BB_FULL + s), (last[s] >> 1) & 1, timeout);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // 64-query half tiles hq = 2i + h; half hq uses TMEM buffer hq & 1
      // (S^T at +0, dP^T at +64).  Order: S/dP of hq + 2 right after dV/dK of
      // hq, so the compute of hq + 1 overlaps those products.
      const int nh = 2 * n_q;
      auto issue_sd = [&](int hq) -> bool {
        const int i = hq >> 1, s = i & 1, h = hq & 1;
        if (h == 0 && !mbar_wait(bar(BB_FULL + s), (i >> 1) & 1, abort_flag, timeout)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + SM::kStageA + s * SM::kTile, doa = sbase + SM::kStageB + s * SM::kTile;
        const uint32_t buf = tmem + (hq & 1) * 128;
        mma_nt_half<HD>(buf, sbase + SM::kRes0, qa, h);        // S^T = K Q^T (64 queries)
        mma_nt_half<HD>(buf + 64, sbase + SM::kRes1, doa, h);  // dP^T = V dO^T
        tc_commit(bar(BB_S + (hq & 1)));
        return true;
      };
      bool ok = mbar_wait(bar(BB_RES), 0, abort_flag, timeout);
      if (ok && nh > 0) ok = issue_sd(0);
      if (ok && nh > 1) ok = issue_sd(1);
      for (int hq = 0; hq < nh && ok; ++hq) {
        const int i = hq >> 1, s = i & 1, h = hq & 1;
        if (!(ok = mbar_wait(bar(BB_P + (hq & 1)), (hq >> 1) & 1, abort_flag, timeout))) break;
        tc_fence_after();
        const uint32_t qa = sbase + SM::kStageA + s * SM::kTile, doa = sbase + SM::kStageB + s * SM::kTile;
        const uint32_t buf = tmem + (hq & 1) * 128;
        mma_tn_half<HD>(tmem + 256, buf, doa, h, hq > 0);             // dV += (c P)^T dO
        mma_tn_half<HD>(tmem + 256 + HD, buf + 64, qa, h, hq > 0);    // dK += dS^T Q / scale
        if (h == 1) tc_commit(bar(BB_EMPTY + s));   // Q_i, dO_i read by both halves
        if (hq + 2 < nh) ok = issue_sd(hq + 2);
      }
      tc_commit(bar(BB_DONE));
      tc_commit(bar(BB_END));
      mbar_drain(bar(BB_END), 0, timeout);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute
    // thread = key row of the tile = TMEM lane
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr;
    const float sl = p.scale_log2;
    bool ok = true;
    for (int hq = 0; hq < 2 * n_q && ok; ++hq) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BB_S + (hq & 1)), (hq >> 1) & 1, abort_flag, timeout) &&
                                       ((hq & 1) || mbar_wait(bar(BB_STATS + ((hq >> 1) & 1)), (hq >> 2) & 1,
                                                              abort_flag, timeout)));
      if (!ok) break;
      tc_fence_after();
      // statistics of the 64 queries of this half (lse - log2 c at +0, D' at +BM)
      const float* st = stats + ((hq >> 1) & 1) * 2 * BM + (hq & 1) * (BM / 2);
      const uint32_t sb = s_addr + (hq & 1) * 128, db = sb + 64;
      // all 64 scores and dP values of the half with one wait
      float sv[64], dpv[64];
      tmem_ld32(sb, sv);
      tmem_ld32(sb + 32, sv + 32);
      tmem_ld32(db, dpv);
      tmem_ld32(db + 32, dpv + 32);
      tmem_wait_ld();
      const float4* st4 = reinterpret_cast<const float4*>(st);   // 4 queries per load
      float pk[32], dk[32];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 l4 = st4[e4], d4 = st4[BM / 4 + e4];
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
        float pc[4], ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qi = 4 * e4 + e;
          pc[e] = fast_exp2(sv[qi] * sl - lv[e]);   // c P
          ds[e] = pc[e] * (dpv[qi] - dv4[e]);       // dS / scale
        }
        pk[2 * e4] = __uint_as_float(bwd_pack(pc[0], pc[1]));
        pk[2 * e4 + 1] = __uint_as_float(bwd_pack(pc[2], pc[3]));
        dk[2 * e4] = __uint_as_float(bwd_pack(ds[0], ds[1]));
        dk[2 * e4 + 1] = __uint_as_float(bwd_pack(ds[2], ds[3]));
      }
      // bf16 pairs of the 64 queries into the first 32 columns of each half
      // region (all of whose fp32 values were read above)
      tmem_st32(sb, pk);
      tmem_st32(db, dk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BB_P + (hq & 1)));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(BB_DONE), 0, abort_flag, timeout));
    if (ok) {
      tc_fence_after();
      const int kr = u.t_begin + row;
      const bool in = kr < u.t_end;
      const int tok = in ? token_of(p, kr) : -1;
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        float g[HD];
#pragma unroll
        for (int cc = 0; cc < HD / 32; ++cc) tmem_ld32(tmem + lane_addr + 256 + part * HD + cc * 32, g + cc * 32);
        tmem_wait_ld();
        if (part == 1)
#pragma unroll
          for (int e = 0; e < HD; ++e) g[e] *= b.scale;   // dK = scale dS^T Q
        // the streamed stages are idle once every product has finished
        add_rows<HD>(part == 0 ? b.dv : b.dk, tok, p.H, u.head, g,
                     reinterpret_cast<float4*>(smem + SM::kStageA + warp * 4096), lane);
      }
    }
  }
  bwd_teardown<HD>(tmem);
}

// ------------------------------------------------------------------ dQ

// TMEM: dQ [0, HD), Q [HD, 1.5 HD) and dO [1.5 HD, 2 HD) as bf16 pairs (the
// A operands of S = Q K^T and dP = dO V^T, so only the streamed K and V
// halves are read from shared memory), and two 128-column buffers for the
// 64-key halves (S at +0, dP at +64; dS overwrites the first 32 columns of S).
template <int HD>
__global__ void __launch_bounds__(192, 1)
bwd_dq_kernel(const __grid_constant__ BwdParams b, const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_do) {
  using SM = BwdSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + SM::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<int*>(smem + SM::kMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long timeout = b.f.timeout_cycles;
  const Params& p = b.f;
  Unit u;
  uint32_t tmem;
  if (!bwd_setup<HD, false>(b, smem, sbase, u, tmem)) return;
  const int n_kv = ceil_div(u.kv_end - u.kv_begin, BN);

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int last[2] = {-1, -1};
      mbar_arrive_expect_tx(bar(BB_RES), 2 * SM::kTile);
      load_tile<HD>(sbase + SM::kRes0, &tm_q, u.head, u.t_begin, bar(BB_RES));
      load_tile<HD>(sbase + SM::kRes1, &tm_do, u.head, u.t_begin, bar(BB_RES));
      for (int j = 0; j < n_kv; ++j) {
        const int s = j & 1;
        if (!mbar_wait(bar(BB_EMPTY + s), ((j >> 1) & 1) ^ 1, abort_flag, timeout)) break;
        const int r0 = u.kv_begin + j * BN;
        mbar_arrive_expect_tx(bar(BB_FULL + s), 2 * SM::kTile);
        load_tile<HD>(sbase + SM::kStageA + s * SM::kTile, &tm_k, u.head, r0, bar(BB_FULL + s));
        load_tile<HD>(sbase + SM::kStageB + s * SM::kTile, &tm_v, u.head, r0, bar(BB_FULL + s));
        last[s] = j;
      }
      mbar_drain(bar(BB_RES), 0, timeout);
      for (int s = 0; s < 2; ++s)
        if (last[s] >= 0) mbar_drain(bar(BB_FULL + s), (last[s] >> 1) & 1, timeout);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // 64-key half tiles hk = 2j + h; half hk uses TMEM buffer hk & 1 (S at
      // +0, dP at +64); S/dP of hk + 2 right after dQ of hk
      const int nh = 2 * n_kv;
      auto issue_sd = [&](int hk) -> bool {
        const int j = hk >> 1, s = j & 1, h = hk & 1;
        if (h == 0 && !mbar_wait(bar(BB_FULL + s), (j >> 1) & 1, abort_flag, timeout)) return false;
        tc_fence_after();
        const uint32_t ka = sbase + SM::kStageA + s * SM::kTile, va = sbase + SM::kStageB + s * SM::kTile;
        const uint32_t buf = tmem + 2 * HD + (hk & 1) * 128;
        mma_ts_half<HD>(buf, tmem + HD, ka, h);                // S = Q K^T (64 keys)
        mma_ts_half<HD>(buf + 64, tmem + HD + HD / 2, va, h);  // dP = dO V^T
        tc_commit(bar(BB_S + (hk & 1)));
        return true;
      };
      bool ok = mbar_wait(bar(BB_A), 0, abort_flag, timeout);
      if (ok && nh > 0) ok = issue_sd(0);
      if (ok && nh > 1) ok = issue_sd(1);
      for (int hk = 0; hk < nh && ok; ++hk) {
        const int j = hk >> 1, s = j & 1, h = hk & 1;
        if (!(ok = mbar_wait(bar(BB_P + (hk & 1)), (hk >> 1) & 1, abort_flag, timeout))) break;
        tc_fence_after();
        const uint32_t ka = sbase + SM::kStageA + s * SM::kTile;
        mma_tn_half<HD>(tmem, tmem + 2 * HD + (hk & 1) * 128, ka, h, hk > 0);   // dQ += dS K / scale
        if (h == 1) tc_commit(bar(BB_EMPTY + s));
        if (hk + 2 < nh) ok = issue_sd(hk + 2);
      }
      tc_commit(bar(BB_DONE));
      tc_commit(bar(BB_END));
      mbar_drain(bar(BB_END), 0, timeout);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute
    // thread = query row of the tile = TMEM lane
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr;
    const float sl = p.scale_log2;
    const int qr = u.t_begin + row;
    const bool in = qr < u.t_end;
    // log-sum-exp less log2 c, so 2^(S sl - lse2) is c P; huge past the segment
    const float lse2 = in ? __ldg(b.lse_seg + (size_t)qr * p.H + u.head) : 3.0e38f;
    const float dd = in ? __ldg(b.dd_seg + (size_t)qr * p.H + u.head) : 0.f;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(BB_RES), 0, abort_flag, timeout));
    if (ok) {
      tile_row_to_tmem<HD>(smem + SM::kRes0, row, tmem + lane_addr + HD);            // Q
      tile_row_to_tmem<HD>(smem + SM::kRes1, row, tmem + lane_addr + HD + HD / 2);   // dO
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BB_A));
    }
    for (int hk = 0; hk < 2 * n_kv && ok; ++hk) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BB_S + (hk & 1)), (hk >> 1) & 1, abort_flag, timeout));
      if (!ok) break;
      tc_fence_after();
      // keys of this half tile that belong to the segment
      const int valid = u.kv_end - (u.kv_begin + (hk >> 1) * BN + (hk & 1) * (BN / 2));
      const uint32_t sb = s_addr + 2 * HD + (hk & 1) * 128, db = sb + 64;
      float sv[64], dpv[64];
      tmem_ld32(sb, sv);
      tmem_ld32(sb + 32, sv + 32);
      tmem_ld32(db, dpv);
      tmem_ld32(db + 32, dpv + 32);
      tmem_wait_ld();
      float dk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float ds[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int ki = 2 * e + h2;
          const float pc = fast_exp2(sv[ki] * sl - lse2);
          ds[h2] = ki < valid ? pc * (dpv[ki] - dd) : 0.f;   // dS / scale
        }
        dk[e] = __uint_as_float(bwd_pack(ds[0], ds[1]));
      }
      tmem_st32(sb, dk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BB_P + (hk & 1)));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(BB_DONE), 0, abort_flag, timeout));
    if (ok) {
      tc_fence_after();
      float g[HD];
#pragma unroll
      for (int cc = 0; cc < HD / 32; ++cc) tmem_ld32(tmem + lane_addr + cc * 32, g + cc * 32);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < HD; ++e) g[e] *= b.scale;   // dQ = scale dS K
      const int tok = in ? token_of(p, qr) : -1;
      // the streamed stages are idle once every product has finished
      add_rows<HD>(b.dq, tok, p.H, u.head, g, reinterpret_cast<float4*>(smem + SM::kStageA + warp * 4096), lane);
    }
  }
  bwd_teardown<HD>(tmem);
}

// ------------------------------------------------------------------ host side

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// q, k, v, dout in segment order, then lse_seg, dd_seg [N][H]
static size_t bwd_ws_bytes(int64_t N, int H, int hd) {
  const size_t t = align256((size_t)N * H * hd * 2);
  return 4 * t + 2 * align256((size_t)N * H * 4);
}

struct BwdWs {
  uint8_t *q, *k, *v, *dout;
  float *lse, *dd;
};

static BwdWs carve_bwd_ws(void* ws, int64_t N, int H, int hd) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t t = align256((size_t)N * H * hd * 2), st = align256((size_t)N * H * 4);
  BwdWs r;
  r.q = w;
  r.k = w + t;
  r.v = w + 2 * t;
  r.dout = w + 3 * t;
  r.lse = reinterpret_cast<float*>(w + 4 * t);
  r.dd = reinterpret_cast<float*>(w + 4 * t + st);
  return r;
}

template <int HD>
static moga_status launch_bwd_kernels(const BwdParams& b, int q_units, int kv_units, const void* q, const void* k,
                                      const void* v, const void* dout, cudaStream_t s) {
  using SM = BwdSmem<HD>;
  CUtensorMap mq, mk, mv, mdo;
  moga_status st;
  if ((st = make_map(&mq, q, b.f.N, b.f.H, HD)) != MOGA_OK) return st;
  if ((st = make_map(&mk, k, b.f.N, b.f.H, HD)) != MOGA_OK) return st;
  if ((st = make_map(&mv, v, b.f.N, b.f.H, HD)) != MOGA_OK) return st;
  if ((st = make_map(&mdo, dout, b.f.N, b.f.H, HD)) != MOGA_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dq_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "attention backward: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  if (kv_units > 0) {
    bwd_dkdv_kernel<HD><<<kv_units, 192, SM::kBytes, s>>>(b, mq, mk, mv, mdo);
    if ((st = check_launch("attention backward (dK, dV)")) != MOGA_OK) return st;
  }
  if (q_units > 0) {
    bwd_dq_kernel<HD><<<q_units, 192, SM::kBytes, s>>>(b, mq, mk, mv, mdo);
    if ((st = check_launch("attention backward (dQ)")) != MOGA_OK) return st;
  }
  return MOGA_OK;
}

// prep + both kernels for one branch; prm.mode selects it.  For frames the
// inputs are read in place; otherwise they are copied into segment order.
static moga_status run_branch_bwd(BwdParams& b, int hd, int q_units, int kv_units, const void* q, const void* k,
                                  const void* v, const void* dout, const float* o_branch, const float* lse,
                                  float* dgate, void* ws, cudaStream_t s) {
  const BwdWs w = carve_bwd_ws(ws, b.f.N, b.f.H, hd);
  b.lse_seg = w.lse;
  b.dd_seg = w.dd;
  const int grid = ceil_div(b.f.N, 8);
  const uint4 *q4 = static_cast<const uint4*>(q), *k4 = static_cast<const uint4*>(k),
              *v4 = static_cast<const uint4*>(v), *d4 = static_cast<const uint4*>(dout);
  uint4 *qd = reinterpret_cast<uint4*>(w.q), *kd = reinterpret_cast<uint4*>(w.k), *vd = reinterpret_cast<uint4*>(w.v),
        *dd = reinterpret_cast<uint4*>(w.dout);
  if (b.f.mode == MODE_MOGA)
    bwd_prep_kernel<MODE_MOGA><<<grid, 256, 0, s>>>(b, q4, k4, v4, d4, o_branch, lse, qd, kd, vd, dd, w.lse, w.dd,
                                                     dgate, hd);
  else if (b.f.mode == MODE_WINDOW)
    bwd_prep_kernel<MODE_WINDOW><<<grid, 256, 0, s>>>(b, q4, k4, v4, d4, o_branch, lse, qd, kd, vd, dd, w.lse, w.dd,
                                                       dgate, hd);
  else
    bwd_prep_kernel<MODE_FRAME><<<grid, 256, 0, s>>>(b, q4, k4, v4, d4, o_branch, lse, qd, kd, vd, dd, w.lse, w.dd,
                                                      dgate, hd);
  moga_status st = check_launch("attention backward (prep)");
  if (st != MOGA_OK) return st;
  const bool in_place = b.f.mode == MODE_FRAME;
  const void* qs = in_place ? q : w.q;
  const void* ks = in_place ? k : w.k;
  const void* vs = in_place ? v : w.v;
  const void* ds = in_place ? dout : w.dout;
  return hd == 128 ? launch_bwd_kernels<128>(b, q_units, kv_units, qs, ks, vs, ds, s)
                   : launch_bwd_kernels<64>(b, q_units, kv_units, qs, ks, vs, ds, s);
}

static moga_status check_bwd(const void* dout, const float* dq, const float* dk, const float* dv, const void* ws,
                             size_t ws_bytes, int64_t N, int H, int hd, const char* who) {
  if (!dout || !dq || !dk || !dv || !ws) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  const uintptr_t a = reinterpret_cast<uintptr_t>(dout) | reinterpret_cast<uintptr_t>(dq) |
                      reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv) |
                      reinterpret_cast<uintptr_t>(ws);
  if (a & 15) return fail(MOGA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  if (reinterpret_cast<uintptr_t>(ws) & 255)
    return fail(MOGA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  if (ws_bytes < bwd_ws_bytes(N, H, hd))
    return fail(MOGA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws_bytes, bwd_ws_bytes(N, H, hd));
  return MOGA_OK;
}

}  // namespace attn
}  // namespace moga

extern "C" size_t moga_attn_bwd_ws_bytes(int64_t N, int32_t H, int32_t hd) {
  if (N <= 0 || H <= 0 || N * (int64_t)H >= INT32_MAX || (hd != 64 && hd != 128)) return 0;
  return moga::attn::bwd_ws_bytes(N, H, hd);
}

namespace moga {
namespace attn {

// Units launched for the MoGA branch: an upper bound on the 128-row tiles of
// all groups (sum of ceil(n_i / 128) <= N / 128 + M per head); units past the
// last tile exit at once.
static int moga_bwd_units(int64_t N, int M, int H) { return (ceil_div((int)N, BM) + M) * H; }

// Window branch: prefixes of the 128-query-tile and 128-key-tile units over
// the temporal groups (windows x heads x tiles per group).
static void fill_window_units(BwdParams& b, int H) {
  const Params& p = b.f;
  b.q_units[0] = b.kv_units[0] = 0;
  for (int i = 0; i < p.n_tg; ++i) {
    const TGroup& tg = p.tg[i];
    const int qlen = (tg.t1 - tg.t0) * p.whw, kvlen = (tg.t1 - tg.t0 + tg.a_prev + tg.a_next) * p.whw;
    b.q_units[i + 1] = b.q_units[i] + p.n_win * H * ceil_div(qlen, BM);
    b.kv_units[i + 1] = b.kv_units[i] + p.n_win * H * ceil_div(kvlen, BM);
  }
}

}  // namespace attn
}  // namespace moga

extern "C" moga_status moga_group_attn_bwd(const void* q, const void* k, const void* v, int64_t N, int32_t H,
                                           int32_t hd, const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                           const float* gate_prob, float softmax_scale, const float* o_moga,
                                           const float* lse, const void* dout, float* dq, float* dk, float* dv,
                                           float* dgate, void* ws, size_t ws_bytes, void* stream) {
  using namespace moga;
  using namespace moga::attn;
  const char* who = "moga_group_attn_bwd";
  moga_status st = check_common(q, k, v, N, H, hd, o_moga, nullptr, 0, false, who);
  if (st != MOGA_OK) return st;
  if (!perm || !cu_seqlens || !gate_prob || !lse || !dgate) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "%s: M=%d not in [1, 32]", who, M);
  if (!(softmax_scale > 0.f)) return fail(MOGA_ERR_INVALID_ARG, "%s: softmax_scale must be > 0", who);
  if ((st = check_bwd(dout, dq, dk, dv, ws, ws_bytes, N, H, hd, who)) != MOGA_OK) return st;
  BwdParams b;
  memset(&b, 0, sizeof(b));
  b.f.N = (int)N;
  b.f.H = H;
  b.f.mode = MODE_MOGA;
  b.f.scale_log2 = softmax_scale * 1.4426950408889634f;
  b.f.perm = perm;
  b.f.cu = cu_seqlens;
  b.f.M = M;
  b.f.gate = gate_prob;
  fill_debug(b.f);
  b.scale = softmax_scale;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  const int units = moga_bwd_units(N, M, H);
  return run_branch_bwd(b, hd, units, units, q, k, v, dout, o_moga, lse, dgate, ws,
                        static_cast<cudaStream_t>(stream));
}

extern "C" moga_status stga_attn_bwd(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                                     const moga_stga_geom* geom, float softmax_scale, const float* o_win,
                                     const float* lse_win, const float* o_frame, const float* lse_frame,
                                     const void* dout, float* dq, float* dk, float* dv, void* ws, size_t ws_bytes,
                                     void* stream) {
  using namespace moga;
  using namespace moga::attn;
  const char* who = "stga_attn_bwd";
  BwdParams b;
  memset(&b, 0, sizeof(b));
  int64_t N = 0;
  moga_status st = stga_params(geom, H, softmax_scale, b.f, N, who);
  if (st != MOGA_OK) return st;
  if ((st = check_common(q, k, v, N, H, hd, o_win, nullptr, 0, false, who)) != MOGA_OK) return st;
  if (!o_frame || !lse_win || !lse_frame) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (reinterpret_cast<uintptr_t>(o_frame) & 15) return fail(MOGA_ERR_INVALID_ARG, "%s: o_frame not aligned", who);
  if ((st = check_bwd(dout, dq, dk, dv, ws, ws_bytes, N, H, hd, who)) != MOGA_OK) return st;
  b.scale = softmax_scale;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  const Params& p = b.f;
  fill_window_units(b, H);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  b.f.mode = MODE_WINDOW;
  if ((st = run_branch_bwd(b, hd, b.q_units[p.n_tg], b.kv_units[p.n_tg], q, k, v, dout, o_win, lse_win, nullptr, ws,
                           s)) != MOGA_OK)
    return st;
  b.f.mode = MODE_FRAME;
  const int fu = p.T * H * ceil_div(p.hw, BM);
  return run_branch_bwd(b, hd, fu, fu, q, k, v, dout, o_frame, lse_frame, nullptr, ws, s);
}

// Test hook (include/moga_testing.h): the work units of one backward launch
// (keys = 0: the dQ kernel, tiles over queries; keys = 1: the dK/dV kernel,
// tiles over keys), decoded by the kernels' own decode_unit compiled for the
// host, with the grid the launch uses.  Host code only.
extern "C" int32_t moga_test_bwd_units(int32_t mode, int32_t keys, const int32_t* cu_seqlens, int32_t M, int64_t N,
                                       int32_t H, const moga_stga_geom* geom, int32_t* grid, int32_t* out,
                                       int32_t cap) {
  using namespace moga;
  using namespace moga::attn;
  BwdParams b;
  memset(&b, 0, sizeof(b));
  int g = 0;
  if (mode == MODE_MOGA) {
    if (!cu_seqlens || M < 1 || M > 32 || N <= 0 || N > INT32_MAX || H <= 0) {
      fail(MOGA_ERR_INVALID_ARG, "moga_test_bwd_units: bad MoGA arguments");
      return -1;
    }
    b.f.N = (int)N;
    b.f.H = H;
    b.f.M = M;
    b.f.cu = cu_seqlens;
    g = moga_bwd_units(N, M, H);
  } else if (mode == MODE_WINDOW || mode == MODE_FRAME) {
    int64_t n = 0;
    if (stga_params(geom, H, 1.0f, b.f, n, "moga_test_bwd_units") != MOGA_OK) return -1;
    fill_window_units(b, H);
    g = mode == MODE_WINDOW ? (keys ? b.kv_units[b.f.n_tg] : b.q_units[b.f.n_tg])
                            : b.f.T * H * ceil_div(b.f.hw, BM);
  } else {
    fail(MOGA_ERR_INVALID_ARG, "moga_test_bwd_units: mode %d", mode);
    return -1;
  }
  b.f.mode = mode;
  GroupTable gt;
  memset(&gt, 0, sizeof(gt));
  if (mode == MODE_MOGA) build_group_table(b.f, gt, BM);
  if (grid) *grid = g;
  int32_t n = 0;
  for (int L = 0; L < g; ++L) {
    const Unit u = keys ? decode_unit<true>(b, gt, L) : decode_unit<false>(b, gt, L);
    if (!u.valid) continue;
    if (n < cap) {
      int32_t* o = out + 7 * (size_t)n;
      o[0] = u.head;
      o[1] = u.q_begin;
      o[2] = u.q_end;
      o[3] = u.kv_begin;
      o[4] = u.kv_end;
      o[5] = u.t_begin;
      o[6] = u.t_end;
    }
    ++n;
  }
  return n;
}
