// The router fused into the Q/K/V projection: one tcgen05 GEMM
//   [q | k | v] = x . W_qkv^T   (bf16 out, fp32 accumulation)
// whose x tiles also feed the router's r = x . W_r, so the router needs no
// pass of its own over x (the projection reads x anyway).  MoGA note, key
// design 1: the router is a linear projection of the token onto M group
// scores followed by a softmax and an argmax; the Q/K/V projection is the
// attention layer's own input projection, the step just before the path.
//
// The product runs on pairs of SMs (a cluster of two CTAs, tcgen05
// cta_group::2): one tile is 256 tokens x 256 columns, each CTA of the pair
// holding 128 of the tokens (its x rows) and 128 of the 256 B rows, so each
// SM streams half of the B tile through its shared memory; the leader CTA
// issues M = 256 products and each CTA's TMEM receives its 128 rows.  The
// first column tile of every token tile holds output columns [0, 192) and the
// router's 64 columns; the others hold 256 output columns each.  The
// router's columns form S slots of NP (S = 64 / NP): its weight is expanded
// once (a small kernel) into a [64][d] matrix whose slot-s rows carry W_r^T
// only on the k stages with (k / 64) % S == s and zeros elsewhere, so the
// product adds every stage into its own slot (adding the zero rows is exact).
// The epilogue adds the S slots in fp32 with round to nearest: the tensor
// core's fp32 accumulation does not round to nearest, and splitting the sum
// keeps the logits close to a plain fp32 dot product.  192 threads per CTA:
//   warp 4     producer: TMA of this CTA's x rows (128 x 64 k) and B rows
//              (128 x 64 k), completing on the leader's stage barrier
//   warp 5     TMEM allocator (both CTAs); in the leader, lane 0 issues
//              tcgen05.mma.cta_group::2 (M=256, N=256, K=16) into one of two
//              accumulator buffers (columns 0, 256) and commits to both CTAs
//   warps 0-3  epilogue, thread = token row = TMEM lane: accumulator columns
//              -> bf16 -> the token's q, k or v row (16-byte stores), and for
//              first tiles the router epilogue (bias, softmax, argmax with
//              the lowest index on a tie, gate, per-32-token sums of p(i|x)
//              for L_gb, in the layout moga_route writes); then they release
//              the buffer on the leader's barrier
// The two accumulator buffers let the epilogue of one tile overlap the
// products of the next.  All mbarrier waits are bounded.
namespace moga {
namespace qkv {

using namespace moga::tc;

constexpr int BM = 128, BN = 256, BK = 64;   // BM: token rows per CTA (256 per pair)
constexpr int kRouterCols = 64;          // router columns of a first tile
constexpr int kFirstCols = BN - kRouterCols;   // 192 output columns in a first tile
constexpr int kStages = 6;
constexpr int kThreads = 192;
constexpr int kXBytes = BM * 128;        // 16 KB
constexpr int kBBytes = (BN / 2) * 128;  // 16 KB: this CTA's half of the B rows
constexpr int kStageBytes = kXBytes + kBBytes;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kMiscOff = kBarOff + 32 * 8;
constexpr int kSmemBytes = kMiscOff + 64 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// first output column of column tile n (tile 0 is a first tile)
__host__ __device__ inline int tile_col0(int n) { return n == 0 ? 0 : kFirstCols + (n - 1) * BN; }

// wx[s * NP + m][k] = W_r[k][m] if m < M, k < d and (k / 64) % S == s, else 0;
// [64][dpad] bf16 (S = 64 / NP slots of NP columns)
__global__ void __launch_bounds__(256)
prep_router_kernel(const __nv_bfloat16* __restrict__ w_r, int d, int M, int NP, int dpad,
                   __nv_bfloat16* __restrict__ wx) {
  const int S = kRouterCols / NP;
  const int total = kRouterCols * dpad;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < total; i += gridDim.x * 256) {
    const int row = i / dpad, k = i - row * dpad;
    const int s = row / NP, m = row - s * NP;
    const bool on = m < M && k < d && (k / BK) % S == s;
    wx[i] = on ? w_r[(size_t)k * M + m] : __float2bfloat16(0.f);
  }
}

// barriers
constexpr int Q_FULL = 0;                 // [kStages]
constexpr int Q_EMPTY = kStages;          // [kStages]
constexpr int Q_ACC_FULL = 2 * kStages;   // [2]
constexpr int Q_ACC_EMPTY = Q_ACC_FULL + 2;   // [2] (128 arrivals)
constexpr int Q_END = Q_ACC_EMPTY + 2;
static_assert(Q_END < 32, "barrier area");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct Params {
  int N, d, M, n_out, hhd;     // hhd = H * hd (one of q, k, v per row)
  int n_k, m_tiles, n_tiles;
  const float* bias;
  __nv_bfloat16 *q, *k, *v;
  int32_t* group_id;
  float* gate_prob;
  float* partial;              // [ceil(N/32)][M]
  long long timeout;
};

// bf16 of 32 accumulator columns [c0, c0 + 32) of the tile into the token's
// q / k / v row (output columns past n_out skipped; 8 columns never straddle
// q, k and v since H * hd is a multiple of 64)
__device__ __forceinline__ void store_cols(const Params& p, int tok, int col0, const float* v) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int col = col0 + 8 * e;
    if (col < p.n_out) {
      const int which = col / p.hhd, rem = col - which * p.hhd;
      __nv_bfloat16* dst = (which == 0 ? p.q : which == 1 ? p.k : p.v) + (size_t)tok * p.hhd + rem;
      uint4 pk;
      pk.x = pack_bf16x2(v[8 * e], v[8 * e + 1]);
      pk.y = pack_bf16x2(v[8 * e + 2], v[8 * e + 3]);
      pk.z = pack_bf16x2(v[8 * e + 4], v[8 * e + 5]);
      pk.w = pack_bf16x2(v[8 * e + 6], v[8 * e + 7]);
      *reinterpret_cast<uint4*>(dst) = pk;
    }
  }
}

constexpr uint32_t kIdescPair = pair_desc(instr_desc(BN, false));   // M = 256, N = 256

template <int NP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
qkv_route_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_w128, const __grid_constant__ CUtensorMap tm_w64,
                 const __grid_constant__ CUtensorMap tm_r) {
  constexpr int S = kRouterCols / NP;     // router slots
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kBarOff + 8u * (uint32_t)i; };
  int* misc = reinterpret_cast<int*>(smem + kMiscOff);
  volatile int* abort_flag = misc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long timeout = p.timeout;
  const uint32_t rank = cluster_rank();          // 0: leader, 1: peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_tiles_total = p.m_tiles * p.n_tiles;   // m_tiles counts 256-token tiles

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Q_FULL + s), 1);
      mbar_init(bar(Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Q_ACC_FULL + b), 1);
      mbar_init(bar(Q_ACC_EMPTY + b), 2 * BM);
    }
    mbar_init(bar(Q_END), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w128)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w64)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_r)) : "memory");
      int c = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles_total && ok; t += n_pairs) {
        const int m = t / p.n_tiles, n = t - m * p.n_tiles;
        const int xrow = m * 2 * BM + (int)rank * BM;
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages;
          if (!(ok = mbar_wait(bar(Q_EMPTY + st), ((c / kStages) & 1) ^ 1, abort_flag, timeout))) break;
          const uint32_t full_leader = peer_addr(bar(Q_FULL + st), 0);
          // the leader's barrier expects both CTAs' bytes
          if (leader) mbar_arrive_expect_tx(bar(Q_FULL + st), 2 * kStageBytes);
          const uint32_t dst = sbase + st * kStageBytes;
          tma_load_2d_pair(dst, &tm_x, kt * BK, xrow, full_leader);
          if (n != 0) {
            tma_load_2d_pair(dst + kXBytes, &tm_w128, kt * BK, tile_col0(n) + (int)rank * (BN / 2), full_leader);
          } else if (leader) {   // W rows [0, 128)
            tma_load_2d_pair(dst + kXBytes, &tm_w128, kt * BK, 0, full_leader);
          } else {               // W rows [128, 192) and the 64 router rows
            tma_load_2d_pair(dst + kXBytes, &tm_w64, kt * BK, BN / 2, full_leader);
            tma_load_2d_pair(dst + kXBytes + 64 * 128, &tm_r, kt * BK, 0, full_leader);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int c = 0, j = 0;   // stage and local tile counters
      bool ok = true;
      for (int t = pair; t < n_tiles_total && ok; t += n_pairs, ++j) {
        const int b = j & 1;
        if (!(ok = mbar_wait(bar(Q_ACC_EMPTY + b), ((j >> 1) & 1) ^ 1, abort_flag, timeout))) break;
        const uint32_t acc = tmem + b * BN;
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages;
          if (!(ok = mbar_wait(bar(Q_FULL + st), (c / kStages) & 1, abort_flag, timeout))) break;
          tc_fence_after();
          const uint32_t xa = sbase + st * kStageBytes, ba = xa + kXBytes;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks)
            mma_pair(acc, smem_desc(xa + ks * 32, 16, 1024), smem_desc(ba + ks * 32, 16, 1024), kIdescPair,
                     (kt > 0 || ks > 0) ? 1u : 0u);
          commit_pair(bar(Q_EMPTY + st));
        }
        if (!ok) break;
        commit_pair(bar(Q_ACC_FULL + b));
      }
      commit_pair(bar(Q_END));
      mbar_drain(bar(Q_END), 0, timeout);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    float bias[NP];
#pragma unroll
    for (int mm = 0; mm < NP; ++mm) bias[mm] = (p.bias && mm < p.M) ? __ldg(p.bias + mm) : 0.f;
    int j = 0;
    bool ok = true;
    for (int t = pair; t < n_tiles_total && ok; t += n_pairs, ++j) {
      const int m = t / p.n_tiles, n = t - m * p.n_tiles;
      const int b = j & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_ACC_FULL + b), (j >> 1) & 1, abort_flag, timeout)))) break;
      tc_fence_after();
      const int tok = m * 2 * BM + (int)rank * BM + row;
      const bool in = tok < p.N;
      const uint32_t acc = tmem + lane_addr + b * BN;
      const uint32_t empty_leader = peer_addr(bar(Q_ACC_EMPTY + b), 0);
      const int ncols = n == 0 ? kFirstCols : BN;
#pragma unroll 1
      for (int c0 = 0; c0 < ncols; c0 += 32) {
        float v[32];
        tmem_ld32(acc + c0, v);
        tmem_wait_ld();
        if (in) store_cols(p, tok, tile_col0(n) + c0, v);
      }
      if (n != 0) {
        tc_fence_before();
        mbar_arrive_cluster(empty_leader);
        continue;
      }
      // router: S slots of NP logits in columns [192, 256), added in order
      float rs[kRouterCols];
      tmem_ld32(acc + kFirstCols, rs);
      tmem_ld32(acc + kFirstCols + 32, rs + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_cluster(empty_leader);
      float r[NP];
#pragma unroll
      for (int mm = 0; mm < NP; ++mm) {
        r[mm] = rs[mm];
#pragma unroll
        for (int s = 1; s < S; ++s) r[mm] += rs[s * NP + mm];
      }
      float pr[NP];
      if (in) {
        float best = -INFINITY;
        int g = 0;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) {
          r[mm] += bias[mm];
          if (mm < p.M && r[mm] > best) {
            best = r[mm];
            g = mm;
          }
        }
        float z = 0.f;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) {
          pr[mm] = (mm < p.M) ? expf(r[mm] - best) : 0.f;
          z += pr[mm];
        }
        const float inv = 1.f / z;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) pr[mm] *= inv;
        p.group_id[tok] = g;
        p.gate_prob[tok] = inv;   // exp(r_g - max) = 1
      } else {
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) pr[mm] = 0.f;
      }
      // sum of p(i|x) over the warp's 32 tokens (one chunk row), fixed order
      const int chunk = (m * 2 * BM + (int)rank * BM) / 32 + warp;
      if (chunk * 32 < p.N) {
        float* dst = p.partial + (size_t)chunk * p.M;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) {
          if (mm < p.M) {
            float sum = pr[mm];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane == 0) dst[mm] = sum;
          }
        }
      }
    }
  }

  // every product of the pair has completed (the leader drained them) and no
  // remote arrival is pending before either CTA frees its TMEM and exits
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
}

inline size_t router_bytes(int d) { return (size_t)kRouterCols * route_tc::dpad_of(d) * 2; }

template <int NP>
static moga_status launch_np(const Params& prm, const void* x, const void* w_qkv, const void* wx, int dpad,
                             cudaStream_t s) {
  CUtensorMap mx, mw128, mw64, mr;
  moga_status st;
  if ((st = route_tc::make_map(&mx, x, prm.N, prm.d, (int64_t)prm.d * 2, BM)) != MOGA_OK) return st;
  if ((st = route_tc::make_map(&mw128, w_qkv, prm.n_out, prm.d, (int64_t)prm.d * 2, BN / 2)) != MOGA_OK) return st;
  if ((st = route_tc::make_map(&mw64, w_qkv, prm.n_out, prm.d, (int64_t)prm.d * 2, 64)) != MOGA_OK) return st;
  if ((st = route_tc::make_map(&mr, wx, kRouterCols, dpad, (int64_t)dpad * 2, kRouterCols)) != MOGA_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(qkv_route_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_qkv_route: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  // one pair of CTAs per pair of SMs (persistent), at most one pair per tile
  const int pairs = std::min(prm.m_tiles * prm.n_tiles, route_tc::sm_count() / 2);
  qkv_route_kernel<NP><<<2 * pairs, kThreads, kSmemBytes, s>>>(prm, mx, mw128, mw64, mr);
  return check_launch("moga_qkv_route");
}

}  // namespace qkv
}  // namespace moga

extern "C" size_t moga_qkv_route_ws_bytes(int64_t N, int32_t d, int32_t M) {
  if (N <= 0 || N > INT32_MAX || M < 1 || M > 32 || d <= 0 || d % 8 != 0) return 0;
  return moga::route_partial_bytes(N, M) + moga::qkv::router_bytes(d);
}

extern "C" moga_status moga_qkv_route(const void* x, const void* w_qkv, const void* w_r, const float* bias,
                                      int64_t N, int32_t d, int32_t H, int32_t hd, int32_t M, void* q, void* k,
                                      void* v, int32_t* group_id, float* gate_prob, void* ws, size_t ws_bytes,
                                      void* stream) {
  using namespace moga;
  if (!x || !w_qkv || !w_r || !q || !k || !v || !group_id || !gate_prob || !ws)
    return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: null pointer");
  if (N <= 0 || N > INT32_MAX) return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: N=%lld out of range", (long long)N);
  if (M < 1 || M > 32) return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: M=%d not in [1, 32]", M);
  if (d <= 0 || d % 8 != 0) return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: d=%d must be a positive multiple of 8", d);
  if (H <= 0 || (hd != 64 && hd != 128))
    return fail(MOGA_ERR_UNSUPPORTED, "moga_qkv_route: H=%d, head_dim %d (supported: 64, 128)", H, hd);
  if (N * (int64_t)H * hd >= ((int64_t)1 << 40) || (int64_t)3 * H * hd >= INT32_MAX)
    return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: sizes out of range");
  const uintptr_t a = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_qkv) |
                      reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                      reinterpret_cast<uintptr_t>(v);
  if (a & 15) return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: x, w_qkv, q, k, v must be 16-byte aligned");
  const size_t need = moga_qkv_route_ws_bytes(N, d, M);
  if (ws_bytes < need) return fail(MOGA_ERR_WORKSPACE, "moga_qkv_route: workspace %zu < %zu bytes", ws_bytes, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255)
    return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: workspace not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dpad = route_tc::dpad_of(d);
  const int NP = M <= 16 ? 16 : 32;
  void* wx = static_cast<uint8_t*>(ws) + route_partial_bytes(N, M);
  qkv::prep_router_kernel<<<ceil_div(qkv::kRouterCols * dpad, 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(w_r), d, M, NP, dpad, static_cast<__nv_bfloat16*>(wx));
  moga_status st = check_launch("moga_qkv_route/prep");
  if (st != MOGA_OK) return st;
  qkv::Params prm;
  prm.N = (int)N;
  prm.d = d;
  prm.M = M;
  prm.hhd = H * hd;
  prm.n_out = 3 * H * hd;
  prm.n_k = dpad / qkv::BK;
  prm.m_tiles = ceil_div((int)N, 2 * qkv::BM);   // 256-token tiles (one per SM pair)
  prm.n_tiles = 1 + ceil_div(prm.n_out - qkv::kFirstCols, qkv::BN);
  prm.bias = bias;
  prm.q = static_cast<__nv_bfloat16*>(q);
  prm.k = static_cast<__nv_bfloat16*>(k);
  prm.v = static_cast<__nv_bfloat16*>(v);
  prm.group_id = group_id;
  prm.gate_prob = gate_prob;
  prm.partial = static_cast<float*>(ws);
  prm.timeout = kWaitLimitCycles;
  return NP == 16 ? qkv::launch_np<16>(prm, x, w_qkv, wx, dpad, s) : qkv::launch_np<32>(prm, x, w_qkv, wx, dpad, s);
}
