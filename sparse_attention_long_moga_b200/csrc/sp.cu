// Sequence parallelism of the layer over P GPUs (MoGA note, key design 2,
// and translation, 方法: each rank routes its own tokens, which carry all
// heads, and the routing results of all tokens are collected before the
// exchange that gives each rank whole sequences for a subset of heads).
// Each rank holds n = N / P consecutive tokens; an all-to-all turns the
// sequence shards of Q, K, V into head shards (H / P heads, all N tokens),
// the layer runs per head shard, and a second all-to-all returns the output
// to sequence shards.
//
// The collectives are the caller's (NCCL through torch.distributed); these
// kernels lay the buffers out for them:
//   sp_pack_heads     src [n][H][hd] -> dst [P][n][H/P][hd]: the send buffer
//                     of the first all-to-all (chunk j goes to rank j)
//   sp_unpack_heads   src [P][n][H/P][hd] -> dst [n][H][hd]: the receive
//                     buffer of the second all-to-all (chunk j came from the
//                     rank holding heads [j H/P, (j+1) H/P))
// One warp per (row, chunk), 16-byte copies; HBM-bound (2 bytes read and
// written per element).
#include "common.cuh"

namespace moga {
namespace sp_detail {

// dir 0: pack, 1: unpack.  cu4 = uint4s per chunk row (H / P * hd * 2 / 16).
template <int DIR>
__global__ void __launch_bounds__(256)
heads_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int n, int P, int cu4) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)n * P) return;
  const int lane = threadIdx.x & 31;
  const int t = (int)(w / P), j = (int)(w - (long long)t * P);
  // [t][j] in the row-major [n][P] view is the head chunk j of row t;
  // [j][t] in the [P][n] view is the same chunk in rank-major order
  const size_t a = ((size_t)t * P + j) * cu4, b = ((size_t)j * n + t) * cu4;
  const uint4* s = src + (DIR == 0 ? a : b);
  uint4* d = dst + (DIR == 0 ? b : a);
  for (int c = lane; c < cu4; c += 32) d[c] = __ldg(s + c);
}

static moga_status run(int dir, const void* src, void* dst, int64_t n, int32_t H, int32_t hd, int32_t P,
                       void* stream, const char* who) {
  if (!src || !dst) return fail(MOGA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (n <= 0 || H <= 0 || P <= 0 || hd <= 0 || H % P != 0)
    return fail(MOGA_ERR_INVALID_ARG, "%s: n=%lld H=%d hd=%d P=%d (H must be a multiple of P)", who, (long long)n, H,
                hd, P);
  if (n * P > INT32_MAX || n * (int64_t)H * hd >= ((int64_t)1 << 40))
    return fail(MOGA_ERR_INVALID_ARG, "%s: sizes out of range", who);
  const int64_t chunk_bytes = (int64_t)(H / P) * hd * 2;
  if (chunk_bytes % 16 != 0) return fail(MOGA_ERR_INVALID_ARG, "%s: (H/P)*hd*2 must be a multiple of 16", who);
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15)
    return fail(MOGA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const long long warps = n * P;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint4* s4 = static_cast<const uint4*>(src);
  uint4* d4 = static_cast<uint4*>(dst);
  if (dir == 0)
    heads_kernel<0><<<grid, 256, 0, s>>>(s4, d4, (int)n, P, (int)(chunk_bytes / 16));
  else
    heads_kernel<1><<<grid, 256, 0, s>>>(s4, d4, (int)n, P, (int)(chunk_bytes / 16));
  return check_launch(who);
}

}  // namespace sp_detail
}  // namespace moga

extern "C" moga_status moga_sp_pack_heads(const void* src, int64_t n, int32_t H, int32_t hd, int32_t P, void* dst,
                                          void* stream) {
  return moga::sp_detail::run(0, src, dst, n, H, hd, P, stream, "moga_sp_pack_heads");
}

extern "C" moga_status moga_sp_unpack_heads(const void* src, int64_t n, int32_t H, int32_t hd, int32_t P, void* dst,
                                            void* stream) {
  return moga::sp_detail::run(1, src, dst, n, H, hd, P, stream, "moga_sp_unpack_heads");
}
