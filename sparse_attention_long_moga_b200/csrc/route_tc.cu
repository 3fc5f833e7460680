// Tensor-core router for bf16 inputs: r = x . W_r on tcgen05, then the
// fused softmax / argmax / gate epilogue and per-warp sums of p(i|x).
//
// MoGA note (papernotes.org ICLR 2026), key design 1: the router is a linear
// projection of the token onto M group scores followed by a softmax; the
// token goes to the most probable group.  The projection is a skinny
// contraction [N x d] . [d x M]: it is bound by reading x once from HBM, and
// running it on the tensor core keeps the SM's other pipes (and its shared
// memory) out of the way of that stream.
//
// One persistent CTA per SM, 192 threads:
//   warps 0-3  epilogue: thread = token row = TMEM lane.  Each 128-wide k
//              slice of the contraction lands in its own TMEM slot; the thread adds
//              the slot's NP partial logits into fp32 registers (round to
//              nearest), then after the last slice adds the bias and takes
//              softmax, argmax, gate and the fixed-order per-warp sum of p(i|x)
//   warp 4     producer: TMA loads of x tiles (four chunks of 32 tokens x
//              64 k as one 128-row box, or the chunks one by one for a
//              CTA's last, partial group; 128B swizzle, the same shared-
//              memory layout either way) and of the matching W_r^T tile (NP
//              groups x 64 k) into a ring of 11-12 stages (~220 KB of
//              shared memory, enough bytes in flight per SM to cover the
//              HBM latency at the per-SM share of the bandwidth)
// Work is split in 32-token chunks: CTA b takes chunks [b*C/G, (b+1)*C/G)
// of the C = ceil(N/32) chunks and walks them four at a time, so every SM
// streams the same number of bytes to within one chunk (with whole 128-token
// tiles, 256 tiles on 148 SMs would leave 40 SMs idle for half the time).
// Rows of a tile past the CTA's last chunk hold stale data; the MMA computes
// them (rows of A are independent) and the epilogue ignores them.
//   warp 5     TMEM allocator; lane 0 issues tcgen05.mma (M=128, N=NP, K=16),
//              eight per k slice, into a ring of 8 NP-column slots
// Why one slot per k slice: the tensor core's fp32 accumulation does not
// round to nearest, and summing all d/16 products inside it drifts by about
// one unit in the last place of the running sum per step (relative 1e-5 on
// the gate at d = 5120).  Eight steps per slot plus round-to-nearest adds in
// registers keep the logits about as accurate as a plain fp32 dot product.
// W_r is first copied (transposed, zero-padded to 32 groups and to a multiple
// of 64 in k) into the route workspace by a small kernel.
#include <cudaTypedefs.h>

#include <algorithm>

#include "tc_common.cuh"

namespace moga {
namespace route_tc {

using namespace moga::tc;

constexpr int BT = 128;                 // tokens per tile
constexpr int BK = 64;                  // k per stage (one 128-byte row)
constexpr int NPMAX = 32;               // groups padded for the MMA's N (rows of the W_r^T scratch)
constexpr int kStagesMax = 12;          // TMA ring (barrier layout)
constexpr int kSlots = 8;               // TMEM ring of per-slice partial logits
constexpr int kSliceStages = 2;         // k stages (of 64) summed in one TMEM slot
constexpr int kChunk = 32;              // tokens per chunk (one epilogue warp)
constexpr int kChunkBytes = kChunk * 128;   // 4 KB: one chunk x 64 k
constexpr int kXBytes = BT * 128;       // 16 KB
constexpr int kThreads = 192;

template <int NP>
struct Cfg {
  static constexpr int kWBytes = NP * 128;
  static constexpr int kStageBytes = kXBytes + kWBytes;   // multiple of 1024
  static constexpr int kStages = NP == 16 ? 12 : 11;
  static_assert(kStages <= kStagesMax, "ring");
  static constexpr uint32_t kTmemCols = kSlots * NP;      // 128 or 256
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kMiscOff = kBarOff + 64 * 8;
  static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack
};

// barrier indices
constexpr int B_FULL = 0;                          // [kStages] TMA -> MMA
constexpr int B_EMPTY = kStagesMax;                // [kStages] MMA -> TMA
constexpr int B_SLOT_FULL = 2 * kStagesMax;        // [kSlots]  MMA -> epilogue
constexpr int B_SLOT_EMPTY = 2 * kStagesMax + kSlots;   // [kSlots] epilogue -> MMA (128 arrivals)
constexpr int B_END = 2 * kStagesMax + 2 * kSlots;
static_assert(B_END < 64, "barrier area");

struct Params {
  int N, d, M, n_k, n_chunks;
  const float* bias;
  int32_t* group_id;
  float* gate_prob;
  float* partial;      // [n_chunks][M]: sum of p(i|x) over the chunk's tokens
  float* probs;        // [N][M] p(i|x) (training forward) or null
  long long timeout;
};

// wt[n][k] = W_r[k][n] for n < M and k < d, zero elsewhere; [NPMAX][dpad] bf16.
__global__ void __launch_bounds__(256)
prep_wt_kernel(const __nv_bfloat16* __restrict__ w_r, int d, int M, int dpad, __nv_bfloat16* __restrict__ wt) {
  const int total = NPMAX * dpad;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < total; i += gridDim.x * 256) {
    const int n = i / dpad, k = i - n * dpad;
    wt[i] = (n < M && k < d) ? w_r[(size_t)k * M + n] : __float2bfloat16(0.f);
  }
}

template <int NP>
__device__ __forceinline__ void ld_slot(uint32_t taddr, float* v) {
  if constexpr (NP == 16) tmem_ld16(taddr, v);
  else tmem_ld32(taddr, v);
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
route_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_x,
                const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x4) {
  using C = Cfg<NP>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::kBarOff + 8u * (uint32_t)i; };
  int* misc = reinterpret_cast<int*>(smem + C::kMiscOff);
  volatile int* abort_flag = misc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long timeout = p.timeout;
  const int c_lo = (int)((long long)blockIdx.x * p.n_chunks / gridDim.x);
  const int c_hi = (int)((long long)(blockIdx.x + 1) * p.n_chunks / gridDim.x);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(bar(B_SLOT_FULL + s), 1);
      mbar_init(bar(B_SLOT_EMPTY + s), BT);
    }
    mbar_init(bar(B_END), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x4)) : "memory");
      int c = 0;
      int last[kStages];
      for (int s = 0; s < kStages; ++s) last[s] = -1;
      bool ok = true;
      for (int c0 = c_lo; c0 < c_hi && ok; c0 += 4) {
        const int nch = min(4, c_hi - c0);
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages;
          const uint32_t ph = (c / kStages) & 1;
          if (!(ok = mbar_wait(bar(B_EMPTY + st), ph ^ 1, abort_flag, timeout))) break;
          mbar_arrive_expect_tx(bar(B_FULL + st), nch * kChunkBytes + C::kWBytes);
          const uint32_t dst = sbase + st * C::kStageBytes;
          if (nch == 4)   // the four chunks as one 128-row box
            tma_load_2d(dst, &tm_x4, kt * BK, c0 * kChunk, bar(B_FULL + st));
          else
            for (int j = 0; j < nch; ++j)
              tma_load_2d(dst + j * kChunkBytes, &tm_x, kt * BK, (c0 + j) * kChunk, bar(B_FULL + st));
          tma_load_2d(dst + kXBytes, &tm_w, kt * BK, 0, bar(B_FULL + st));
          last[st] = c;
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (last[s] >= 0) mbar_drain(bar(B_FULL + s), (last[s] / kStages) & 1, timeout);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(NP, false);
      int c = 0, q = 0;   // stage and slot counters
      bool ok = true;
      for (int c0 = c_lo; c0 < c_hi && ok; c0 += 4) {
        for (int kt = 0; kt < p.n_k; ++kt, ++c) {
          const int st = c % kStages, sl = q % kSlots;
          const bool first = kt % kSliceStages == 0;
          const bool last = kt % kSliceStages == kSliceStages - 1 || kt == p.n_k - 1;
          if (first && !(ok = mbar_wait(bar(B_SLOT_EMPTY + sl), ((q / kSlots) & 1) ^ 1, abort_flag, timeout)))
            break;
          if (!(ok = mbar_wait(bar(B_FULL + st), (c / kStages) & 1, abort_flag, timeout))) break;
          tc_fence_after();
          const uint32_t xa = sbase + st * C::kStageBytes, wa = xa + kXBytes;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks)
            tc_mma_ss(tmem + sl * NP, smem_desc(xa + ks * 32, 16, 1024), smem_desc(wa + ks * 32, 16, 1024), idesc,
                      (first && ks == 0) ? 0u : 1u);
          tc_commit(bar(B_EMPTY + st));
          if (last) {
            tc_commit(bar(B_SLOT_FULL + sl));
            ++q;
          }
        }
      }
      tc_commit(bar(B_END));
      mbar_drain(bar(B_END), 0, timeout);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    float bias[NP];
#pragma unroll
    for (int m = 0; m < NP; ++m) bias[m] = (p.bias && m < p.M) ? __ldg(p.bias + m) : 0.f;
    const int n_slices = (p.n_k + kSliceStages - 1) / kSliceStages;
    int q = 0;
    bool ok = true;
    for (int c0 = c_lo; c0 < c_hi && ok; c0 += 4) {
      float r[NP];
#pragma unroll
      for (int m = 0; m < NP; ++m) r[m] = 0.f;
      for (int j = 0; j < n_slices; ++j, ++q) {
        const int sl = q % kSlots;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SLOT_FULL + sl), (q / kSlots) & 1, abort_flag, timeout))))
          break;
        tc_fence_after();
        float v[NP];
        ld_slot<NP>(tmem + lane_addr + sl * NP, v);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(B_SLOT_EMPTY + sl));
#pragma unroll
        for (int m = 0; m < NP; ++m) r[m] += v[m];
      }
      if (!ok) break;
      if (warp >= c_hi - c0) continue;   // rows past the CTA's last chunk
      const int chunk = c0 + warp;
      const int tok = chunk * kChunk + lane;
      float pr[NP];
      if (tok < p.N) {
        // softmax, argmax (lowest index wins a tie), gate
        float best = -INFINITY;
        int g = 0;
#pragma unroll
        for (int m = 0; m < NP; ++m) {
          r[m] += bias[m];
          if (m < p.M && r[m] > best) {
            best = r[m];
            g = m;
          }
        }
        float z = 0.f;
#pragma unroll
        for (int m = 0; m < NP; ++m) {
          pr[m] = (m < p.M) ? expf(r[m] - best) : 0.f;
          z += pr[m];
        }
        const float inv = 1.f / z;
#pragma unroll
        for (int m = 0; m < NP; ++m) pr[m] *= inv;
        p.group_id[tok] = g;
        p.gate_prob[tok] = inv;   // exp(r_g - max) = 1
        if (p.probs != nullptr)
#pragma unroll
          for (int m = 0; m < NP; ++m)
            if (m < p.M) p.probs[(size_t)tok * p.M + m] = pr[m];
      } else {
#pragma unroll
        for (int m = 0; m < NP; ++m) pr[m] = 0.f;
      }
      // sum of p(i|x) over the chunk's 32 tokens, fixed order; one row per chunk
      float* dst = p.partial + (size_t)chunk * p.M;
#pragma unroll
      for (int m = 0; m < NP; ++m) {
        if (m < p.M) {
          float v = pr[m];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
          if (lane == 0) dst[m] = v;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols) : "memory");
}

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

// [rows][cols] bf16, box {64 cols, box_rows rows}, 128B swizzle, zero fill outside.
static moga_status make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t row_bytes,
                            int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOGA_OK;
}

inline int dpad_of(int d) { return (d + BK - 1) / BK * BK; }
inline size_t wt_bytes(int d) { return (size_t)NPMAX * dpad_of(d) * 2; }

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

template <int NP>
static moga_status launch_np(const Params& prm, const void* wt, int dpad, const void* x, cudaStream_t s) {
  using C = Cfg<NP>;
  CUtensorMap mx, mw, mx4;
  moga_status st;
  if ((st = make_map(&mx, x, prm.N, prm.d, (int64_t)prm.d * 2, kChunk)) != MOGA_OK) return st;
  if ((st = make_map(&mx4, x, prm.N, prm.d, (int64_t)prm.d * 2, BT)) != MOGA_OK) return st;
  if ((st = make_map(&mw, wt, NP, dpad, (int64_t)dpad * 2, NP)) != MOGA_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return fail(MOGA_ERR_CUDA, "moga_route: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  const int grid = std::min(prm.n_chunks, sm_count());
  route_tc_kernel<NP><<<grid, kThreads, C::kSmemBytes, s>>>(prm, mx, mw, mx4);
  return check_launch("moga_route");
}

// x [N][d] bf16, w_r [d][M] bf16; partial [ceil(N/32)][M]; wt scratch of wt_bytes(d).
moga_status launch(const void* x, const void* w_r, const float* bias, int N, int d, int M, int32_t* g, float* gate,
                   float* partial, float* probs, void* wt, long long timeout, cudaStream_t s) {
  const int dpad = dpad_of(d);
  prep_wt_kernel<<<ceil_div(NPMAX * dpad, 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w_r), d, M, dpad,
                                                            static_cast<__nv_bfloat16*>(wt));
  moga_status st = check_launch("moga_route/prep");
  if (st != MOGA_OK) return st;
  Params prm;
  prm.N = N;
  prm.d = d;
  prm.M = M;
  prm.n_k = dpad / BK;
  prm.n_chunks = ceil_div(N, kChunk);
  prm.bias = bias;
  prm.group_id = g;
  prm.gate_prob = gate;
  prm.partial = partial;
  prm.probs = probs;
  prm.timeout = timeout;
  return M <= 16 ? launch_np<16>(prm, wt, dpad, x, s) : launch_np<32>(prm, wt, dpad, x, s);
}

}  // namespace route_tc
}  // namespace moga
