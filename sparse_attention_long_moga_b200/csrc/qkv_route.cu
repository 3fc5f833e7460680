// The router fused into the Q/K/V projection: one tcgen05 GEMM
//   [q | k | v] = x . W_qkv^T   (bf16 out, fp32 accumulation)
// whose x tiles also feed the router's r = x . W_r, so the router needs no
// pass of its own over x (the projection reads x anyway).  MoGA note, key
// design 1: the router is a linear projection of the token onto M group
// scores followed by a softmax and an argmax; the Q/K/V projection is the
// attention layer's own input projection, the step just before the path.
//
// Tiles of 128 tokens x 192 output columns; the router's NP (16 or 32)
// columns ride along with the first column tile of every token tile.  One
// persistent CTA per SM, 192 threads:
//   warp 4     producer: TMA of x (128 x 64 k) and W_qkv (192 x 64 k) per
//              stage, plus W_r^T (NP x 64 k) for router tiles; 4 stages
//   warp 5     TMEM allocator; lane 0 issues tcgen05.mma: M=128, N=192, K=16
//              into one of two accumulator buffers (columns 0 and 256), and
//              for router tiles M=128, N=NP into kSlots slots beside them,
//              k stage kt going to slot kt % kSlots (each slot sums a few
//              stages; the epilogue adds the slots in fp32 with round to
//              nearest, which keeps the logits close to a plain fp32 dot
//              product: the tensor core's accumulation does not round to
//              nearest)
//   warps 0-3  epilogue, thread = token row = TMEM lane: 192 accumulator
//              columns -> bf16 -> the token's q, k or v row (16-byte stores),
//              then for router tiles the router epilogue (bias, softmax,
//              argmax with the lowest index on a tie, gate, per-32-token
//              sums of p(i|x) for L_gb, in the layout moga_route writes)
// The two accumulator buffers let the epilogue of one tile overlap the
// products of the next.  All waits are bounded.
namespace moga {
namespace qkv {

using namespace moga::tc;

constexpr int BM = 128, BN = 192, BK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kXBytes = BM * 128;      // 16 KB
constexpr int kWBytes = BN * 128;      // 24 KB
// TMEM: accumulator buffers at columns 0 and 256 (192 columns each); the
// router slots fill the two 64-column gaps [192, 256) and [448, 512)
constexpr int kAccStride = 256;
constexpr int kRouterCols = 2 * (kAccStride - BN);   // 128 columns of router slots

template <int NP>
struct Cfg {
  static constexpr int kSlots = kRouterCols / NP;          // 8 or 4
  static constexpr int kHalf = kSlots / 2;                 // slots per gap
  __device__ static uint32_t slot_col(int s) {
    return (uint32_t)((s < kHalf ? BN : kAccStride + BN) + (s % kHalf) * NP);
  }
  static constexpr int kRBytes = NP * 128;
  static constexpr int kStageBytes = kXBytes + kWBytes + kRBytes;   // multiple of 1024
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kMiscOff = kBarOff + 32 * 8;
  static constexpr int kSmemBytes = kMiscOff + 64 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// barriers
constexpr int Q_FULL = 0;                 // [kStages]
constexpr int Q_EMPTY = kStages;          // [kStages]
constexpr int Q_ACC_FULL = 2 * kStages;   // [2]
constexpr int Q_ACC_EMPTY = Q_ACC_FULL + 2;   // [2] (128 arrivals)
constexpr int Q_R_FULL = Q_ACC_EMPTY + 2;
constexpr int Q_R_EMPTY = Q_R_FULL + 1;   // 128 arrivals
constexpr int Q_END = Q_R_EMPTY + 1;
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

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
qkv_route_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_r) {
  using C = Cfg<NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::kBarOff + 8u * (uint32_t)i; };
  int* misc = reinterpret_cast<int*>(smem + C::kMiscOff);
  volatile int* abort_flag = misc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long timeout = p.timeout;
  const int n_tiles_total = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Q_FULL + s), 1);
      mbar_init(bar(Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Q_ACC_FULL + b), 1);
      mbar_init(bar(Q_ACC_EMPTY + b), BM);
    }
    mbar_init(bar(Q_R_FULL), 1);
    mbar_init(bar(Q_R_EMPTY), BM);
    mbar_init(bar(Q_END), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_r)) : "memory");
      int c = 0;
      int last[kStages];
      for (int s = 0; s < kStages; ++s) last[s] = -1;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x) {
        const int m = t / p.n_tiles, n = t - m * p.n_tiles;
        const bool router = n == 0;
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages;
          if (!(ok = mbar_wait(bar(Q_EMPTY + st), ((c / kStages) & 1) ^ 1, abort_flag, timeout))) break;
          mbar_arrive_expect_tx(bar(Q_FULL + st), kXBytes + kWBytes + (router ? C::kRBytes : 0));
          const uint32_t dst = sbase + st * C::kStageBytes;
          tma_load_2d(dst, &tm_x, kt * BK, m * BM, bar(Q_FULL + st));
          tma_load_2d(dst + kXBytes, &tm_w, kt * BK, n * BN, bar(Q_FULL + st));
          if (router) tma_load_2d(dst + kXBytes + kWBytes, &tm_r, kt * BK, 0, bar(Q_FULL + st));
          last[st] = c;
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (last[s] >= 0) mbar_drain(bar(Q_FULL + s), (last[s] / kStages) & 1, timeout);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_w = instr_desc(BN, false);
      constexpr uint32_t idesc_r = instr_desc(NP, false);
      int c = 0, j = 0, nr = 0;   // stage, local tile and router tile counters
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x, ++j) {
        const int n = t % p.n_tiles;
        const bool router = n == 0;
        const int b = j & 1;
        if (!(ok = mbar_wait(bar(Q_ACC_EMPTY + b), ((j >> 1) & 1) ^ 1, abort_flag, timeout))) break;
        if (router && !(ok = mbar_wait(bar(Q_R_EMPTY), (nr & 1) ^ 1, abort_flag, timeout))) break;
        const uint32_t acc = tmem + b * kAccStride;
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages;
          if (!(ok = mbar_wait(bar(Q_FULL + st), (c / kStages) & 1, abort_flag, timeout))) break;
          tc_fence_after();
          const uint32_t xa = sbase + st * C::kStageBytes, wa = xa + kXBytes, ra = wa + kWBytes;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks)
            tc_mma_ss(acc, smem_desc(xa + ks * 32, 16, 1024), smem_desc(wa + ks * 32, 16, 1024), idesc_w,
                      (kt > 0 || ks > 0) ? 1u : 0u);
          if (router) {
            const uint32_t slot = tmem + C::slot_col(kt % C::kSlots);
#pragma unroll
            for (int ks = 0; ks < BK / 16; ++ks)
              tc_mma_ss(slot, smem_desc(xa + ks * 32, 16, 1024), smem_desc(ra + ks * 32, 16, 1024), idesc_r,
                        (kt >= C::kSlots || ks > 0) ? 1u : 0u);
          }
          tc_commit(bar(Q_EMPTY + st));
        }
        if (!ok) break;
        tc_commit(bar(Q_ACC_FULL + b));
        if (router) {
          tc_commit(bar(Q_R_FULL));
          ++nr;
        }
      }
      tc_commit(bar(Q_END));
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
    const int used_slots = min(C::kSlots, p.n_k);
    int j = 0, nr = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x, ++j) {
      const int m = t / p.n_tiles, n = t - m * p.n_tiles;
      const int b = j & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_ACC_FULL + b), (j >> 1) & 1, abort_flag, timeout)))) break;
      tc_fence_after();
      const int tok = m * BM + row;
      const bool in = tok < p.N;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_addr + b * kAccStride + c0, v);
        tmem_wait_ld();
        if (in) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = n * BN + c0 + 8 * e;   // 8 columns = 16 bytes, never across q|k|v
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
      }
      tc_fence_before();
      mbar_arrive(bar(Q_ACC_EMPTY + b));
      if (n != 0) continue;
      // router epilogue for the tile's 128 tokens
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_R_FULL), nr & 1, abort_flag, timeout)))) break;
      ++nr;
      tc_fence_after();
      float r[NP];
#pragma unroll
      for (int mm = 0; mm < NP; ++mm) r[mm] = 0.f;
      for (int s = 0; s < used_slots; ++s) {
        float sv[NP];
        if constexpr (NP == 16) tmem_ld16(tmem + lane_addr + C::slot_col(s), sv);
        else tmem_ld32(tmem + lane_addr + C::slot_col(s), sv);
        tmem_wait_ld();
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) r[mm] += sv[mm];
      }
      tc_fence_before();
      mbar_arrive(bar(Q_R_EMPTY));
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
      const int chunk = m * (BM / 32) + warp;
      if (chunk * 32 < p.N) {
        float* dst = p.partial + (size_t)chunk * p.M;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm) {
          if (mm < p.M) {
            float s = pr[mm];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) dst[mm] = s;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
}

template <int NP>
static moga_status launch_np(const Params& prm, const void* x, const void* w_qkv, const void* wt, int dpad,
                             cudaStream_t s) {
  using C = Cfg<NP>;
  CUtensorMap mx, mw, mr;
  moga_status st;
  if ((st = route_tc::make_map(&mx, x, prm.N, prm.d, (int64_t)prm.d * 2, BM)) != MOGA_OK) return st;
  if ((st = route_tc::make_map(&mw, w_qkv, prm.n_out, prm.d, (int64_t)prm.d * 2, BN)) != MOGA_OK) return st;
  if ((st = route_tc::make_map(&mr, wt, NP, dpad, (int64_t)dpad * 2, NP)) != MOGA_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(qkv_route_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_qkv_route: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  const int grid = std::min(prm.m_tiles * prm.n_tiles, route_tc::sm_count());
  qkv_route_kernel<NP><<<grid, kThreads, C::kSmemBytes, s>>>(prm, mx, mw, mr);
  return check_launch("moga_qkv_route");
}

}  // namespace qkv
}  // namespace moga

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
  const size_t need = moga_route_ws_bytes(N, d, M);
  if (ws_bytes < need) return fail(MOGA_ERR_WORKSPACE, "moga_qkv_route: workspace %zu < %zu bytes", ws_bytes, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255)
    return fail(MOGA_ERR_INVALID_ARG, "moga_qkv_route: workspace not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dpad = route_tc::dpad_of(d);
  void* wt = static_cast<uint8_t*>(ws) + route_partial_bytes(N, M);
  route_tc::prep_wt_kernel<<<ceil_div(route_tc::NPMAX * dpad, 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(w_r), d, M, dpad, static_cast<__nv_bfloat16*>(wt));
  moga_status st = check_launch("moga_qkv_route/prep");
  if (st != MOGA_OK) return st;
  qkv::Params prm;
  prm.N = (int)N;
  prm.d = d;
  prm.M = M;
  prm.hhd = H * hd;
  prm.n_out = 3 * H * hd;
  prm.n_k = dpad / qkv::BK;
  prm.m_tiles = ceil_div((int)N, qkv::BM);
  prm.n_tiles = ceil_div(prm.n_out, qkv::BN);
  prm.bias = bias;
  prm.q = static_cast<__nv_bfloat16*>(q);
  prm.k = static_cast<__nv_bfloat16*>(k);
  prm.v = static_cast<__nv_bfloat16*>(v);
  prm.group_id = group_id;
  prm.gate_prob = gate_prob;
  prm.partial = static_cast<float*>(ws);
  prm.timeout = 4000000000LL;
  return M <= 16 ? qkv::launch_np<16>(prm, x, w_qkv, wt, dpad, s) : qkv::launch_np<32>(prm, x, w_qkv, wt, dpad, s);
}
