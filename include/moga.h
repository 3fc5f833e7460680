/*
 * moga.h -- C ABI of the B200 (sm_100a) MoGA visual-attention layer forward.
 *
 * The layer (MoGA paper: papernotes.org ICLR 2026 note, flowchart and key
 * designs 1-4; jxzklqfsx.com translation, section 方法) is:
 *
 *   route    r = x . W_r, p = softmax(r), g = argmax p, gate = p[g]
 *   permute  tokens grouped by g (stable), cu_seqlens / counts / max_seqlen
 *   MoGA     o_moga[t] = gate[t] * SA(q_t, K_g(t), V_g(t))   (scattered back)
 *   STGA     o_win[t]  = SA over the token's spatial window x temporal group,
 *                        K/V widened by frames of the adjacent shot at a cut
 *            o_frame[t]= SA over the token's latent frame
 *   mean     out = (o_moga + o_win + o_frame) / 3
 *   loss     L_gb = alpha * M * sum_i F_i * P_i
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless marked HOST.  The caller allocates
 *     and owns every buffer, including workspaces; the library allocates and
 *     frees nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronise the host.
 *   - Tensors are dense row-major.  Q, K, V and outputs use the token-major
 *     "thd" layout [N][H][hd] (bf16 Q/K/V, fp32 accumulator).
 *   - Arguments are validated before any launch.  A bad argument returns
 *     MOGA_ERR_INVALID_ARG (or MOGA_ERR_UNSUPPORTED / MOGA_ERR_WORKSPACE) and
 *     launches nothing; moga_last_error() then describes it.  A failed launch
 *     returns MOGA_ERR_CUDA.  Kernels never trap: a device-side wait that
 *     runs out of time records MOGA_ERR_TIMEOUT in a per-device error word,
 *     which moga_device_status() reports.
 *   - Index arguments in device memory (group ids, perm, cu_seqlens) cannot
 *     be checked on the host.  The permute records MOGA_ERR_BAD_INDEX for a
 *     group id outside [0, M) in every build.  The checking build of this
 *     library (libmoga_debug.so, compiled with -DMOGA_DEBUG; same ABI) also
 *     checks, before each access, every perm entry against [0, N), that
 *     cu_seqlens is a non-decreasing split inside [0, N], and that every
 *     token row the kernels derive lies in [0, N); a failed check records
 *     MOGA_ERR_BAD_INDEX and skips the access it guards (a bad cu_seqlens
 *     skips the whole attention launch), so a bad index never reaches
 *     memory.  In the default build such inputs are unchecked and their
 *     result is undefined.
 *   - Limits: N * H < 2^31, 1 <= M <= 32, d % 8 == 0, hd in {64, 128}.
 */
#ifndef MOGA_H
#define MOGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOGA_OK = 0,
  MOGA_ERR_INVALID_ARG = 1,
  MOGA_ERR_UNSUPPORTED = 2,
  MOGA_ERR_WORKSPACE = 3,
  MOGA_ERR_CUDA = 4,
  MOGA_ERR_TIMEOUT = 5,
  MOGA_ERR_BAD_INDEX = 6
} moga_status;

typedef enum { MOGA_F32 = 0, MOGA_BF16 = 1 } moga_dtype;

/* Static-group geometry (note, key design 4; translation, 时空分组注意力).
 * Tokens are in raster order t = frame*h*w + row*w + col.  Windows tile the
 * frame without overlap (h % win_h == 0, w % win_w == 0).  Each shot is cut
 * into ceil(len / tg_max) temporal groups of as-equal-as-possible length,
 * longer first (tg_max == 0: one group per shot).  A group that starts a shot
 * after a cut adds the last min(aug_frames, len) frames of the previous shot
 * to its keys/values; a group that ends a shot before a cut adds the first
 * min(aug_frames, len) frames of the next shot.  Queries are never added. */
typedef struct {
  int32_t T, h, w;           /* latent frames, token rows and columns per frame */
  int32_t win_h, win_w;      /* spatial window */
  int32_t n_shots;           /* >= 1 */
  const int32_t* shot_len;   /* HOST [n_shots], each >= 1, summing to T */
  int32_t tg_max;            /* max frames per temporal group, 0 = whole shot */
  int32_t aug_frames;        /* frames borrowed from each adjacent shot (pages: 2) */
} moga_stga_geom;

/* ---------------------------------------------------------------- routing --
 * Linear top-1 router (note, key design 1; blog section 2.3):
 *   r = x . W_r (+ bias), p = softmax(r), g = argmax_i p_i (lowest index on
 *   a tie), gate_prob = p_g.  Logits are accumulated in fp32.
 * x:         [N][d], dtype `dt` (MOGA_F32 or MOGA_BF16)
 * w_r:       [d][M], same dtype as x
 * bias:      [M] fp32 or NULL (the pages' router has no bias)
 * group_id:  [N] int32 out;  gate_prob: [N] fp32 out
 * ws:        workspace of at least moga_route_ws_bytes(N, d, M) bytes, 256-byte
 *            aligned; on return it holds partial sums of p(i|x) (one row of
 *            M per 32 tokens) that moga_balance_loss() reads.  Keep it until the
 *            loss is taken.  bf16 inputs run on the tensor cores (x tiles
 *            staged by TMA, fp32 accumulation in tensor memory); fp32 inputs
 *            on the FMA pipe.
 * moga_route_ws_bytes returns 0 for arguments moga_route would reject.
 */
size_t moga_route_ws_bytes(int64_t N, int32_t d, int32_t M);
moga_status moga_route(const void* x, const void* w_r, moga_dtype dt, const float* bias,
                       int64_t N, int32_t d, int32_t M,
                       int32_t* group_id, float* gate_prob,
                       void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- permute --
 * Stable counting sort of tokens by group (note, key design 2: permute so
 * each group is contiguous; boundaries as cu_seqlens / max_seqlen):
 *   counts[i] = #{t : g_t = i}, cu_seqlens = exclusive prefix (cu[M] = N),
 *   perm[cu[i] + j] = the j-th smallest token index with g = i,
 *   *max_seqlen = max_i counts[i].
 * group_id: [N] int32, every value in [0, M); a value outside is skipped
 *           (perm then holds fewer than N entries and counts sum to less
 *           than N) and recorded as MOGA_ERR_BAD_INDEX in the device error
 *           word, which moga_device_status() returns
 * perm [N], cu_seqlens [M+1], counts [M], max_seqlen [1]: int32 out
 * ws:       at least moga_permute_ws_bytes(N, M) bytes of scratch.
 */
size_t moga_permute_ws_bytes(int64_t N, int32_t M);
moga_status moga_permute(const int32_t* group_id, int64_t N, int32_t M,
                         int32_t* perm, int32_t* cu_seqlens, int32_t* counts, int32_t* max_seqlen,
                         void* ws, size_t ws_bytes, void* stream);

/* The same stable permute without a caller workspace.  The paper has no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory when they run the layer: code running inside another runtime's
 * plugin or callback whose device memory that runtime owns, programs that
 * plan a fixed device-memory budget up front and forbid cudaMalloc while
 * serving (it can also stall the device), and C callers with no allocator at
 * hand.  Scratch comes from a 512 KiB array the library keeps on each GPU
 * that loads it, for the life of the process.
 *   - N must be <= 4,194,304 (larger N returns MOGA_ERR_WORKSPACE, nothing
 *     is launched); M in [1, 32].  Outputs as for moga_permute.
 *   - All calls on one GPU share that array.  Calls whose kernels overlap on
 *     the GPU (other streams or host threads) race on it: serialise them.
 *     Nothing in it needs to start at zero; each call writes what it reads.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: it does not survive
 *     cudaDeviceReset() or another teardown of the device's primary context,
 *     after which this call must not be used in the same process.
 *   - Allocates nothing and calls no allocating routine. */
moga_status moga_permute_noalloc(const int32_t* group_id, int64_t N, int32_t M,
                                 int32_t* perm, int32_t* cu_seqlens, int32_t* counts,
                                 int32_t* max_seqlen, void* stream);

/* ------------------------------------------------------ attention scratch --
 * Both attention calls first copy Q, K and V into segment order (rows of a
 * group contiguous) so that the attention kernel streams whole tiles; they
 * need a caller workspace of at least moga_attn_ws_bytes(N, H, hd) bytes
 * (3 * N * H * hd * 2).  One workspace can serve both calls on one stream.
 * Returns 0 for arguments the calls would reject. */
size_t moga_attn_ws_bytes(int64_t N, int32_t H, int32_t hd);

/* ------------------------------------------- the three branches, one gather --
 * o_acc = MoGA attention (written) + window-group and per-frame attention
 * (added): the result of moga_group_attn followed by stga_attn on one
 * stream, bit for bit (the same kernels on the same data), with one pass
 * over Q, K, V that writes both the group-order and the window-order copy
 * instead of two passes that each read Q, K, V.  Arguments as for
 * moga_group_attn and stga_attn together; N must equal geom's T*h*w.
 * ws: at least visual_attn_ws_bytes(N, H, hd) bytes (6 * N * H * hd * 2:
 * both copies), 16-byte aligned.  The layer's mean and loss follow as usual
 * (visual_attn_mean, moga_balance_loss). */
size_t visual_attn_ws_bytes(int64_t N, int32_t H, int32_t hd);
moga_status visual_attn_branches(const void* q, const void* k, const void* v, int64_t N, int32_t H, int32_t hd,
                                 const int32_t* perm, const int32_t* cu_seqlens, int32_t M, const float* gate_prob,
                                 const moga_stga_geom* geom, float softmax_scale, float* o_acc,
                                 void* ws, size_t ws_bytes, void* stream);

/* -------------------------------------------------------- group attention --
 * MoGA attention (note, key designs 1-2): for every group i and head h,
 * full non-causal softmax attention among the tokens perm[cu[i] .. cu[i+1]),
 * each output row scaled by its token's gate and written to that token's own
 * row:  o_acc[perm[j]][h][:] = gate_prob[perm[j]] * softmax(q k^T * scale) v.
 * q, k, v:  [N][H][hd] bf16;  perm, cu_seqlens: from moga_permute
 * o_acc:    [N][H][hd] fp32, OVERWRITTEN for every token (empty groups are
 *           skipped; tokens are covered because perm is a permutation)
 * softmax_scale: usually 1/sqrt(hd).
 * ws:       attention workspace (see moga_attn_ws_bytes), 16-byte aligned.
 */
moga_status moga_group_attn(const void* q, const void* k, const void* v,
                            int64_t N, int32_t H, int32_t hd,
                            const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                            const float* gate_prob, float softmax_scale,
                            float* o_acc, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------- STGA --
 * Static spatial-temporal group attention plus per-frame attention (note,
 * key design 4; translation, 时空分组注意力; blog 3.2): for every token,
 *   o_acc[t] += SA(q_t, K/V of its window group incl. adjacent-shot frames)
 *             + SA(q_t, K/V of its latent frame).
 * q, k, v: [N][H][hd] bf16 with N = T*h*w;  o_acc: [N][H][hd] fp32, ADDED TO.
 * geom: HOST pointer, read during the call only.
 * ws:   attention workspace (see moga_attn_ws_bytes), 16-byte aligned.
 */
moga_status stga_attn(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                      const moga_stga_geom* geom, float softmax_scale,
                      float* o_acc, void* ws, size_t ws_bytes, void* stream);

/* STGA with the three-way mean fused into its last pass (note, flowchart
 * "多组输出取均值"): the window branch adds into o_acc as in stga_attn, then
 * the per-frame pass writes
 *   out[t] = bf16_rn((o_acc[t] + o_frame[t]) / 3)
 * instead of adding o_frame into o_acc, so no separate mean pass runs.  With
 * o_acc = o_moga on entry this is the layer output, equal to
 * stga_attn + visual_attn_mean up to the order of the fp32 additions.
 * out: [N][H][hd] bf16, 16-byte aligned.  On return o_acc holds
 * o_moga + o_win (the frame term is not added to it). */
moga_status stga_attn_mean(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                           const moga_stga_geom* geom, float softmax_scale,
                           float* o_acc, void* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------- mean --
 * Three-way mean (note, flowchart "多组输出取均值" and key design 4):
 *   out[i] = bf16_rn(o_acc[i] / 3) for i < n_elems, where o_acc already
 *   holds o_moga + o_win + o_frame.
 * o_acc: fp32 [n_elems];  out: bf16 [n_elems] (16-byte aligned pointers).
 */
moga_status visual_attn_mean(const float* o_acc, int64_t n_elems, void* out, void* stream);

/* ------------------------------------------------------------------- loss --
 * Group-balancing loss (note, key design 3):
 *   L_gb = alpha * M * sum_i F_i * P_i,  F_i = counts[i] / N,
 *   P_i = (1/N) sum_t p(i | x_t)   (mean over all N tokens).
 * counts: [M] int32 from moga_permute;  route_ws: the workspace moga_route
 * filled for the same N and M;  loss: [1] fp64 out (device).
 */
moga_status moga_balance_loss(const int32_t* counts, const void* route_ws, int64_t N, int32_t M,
                              float alpha, double* loss, void* stream);

/* =============================================================== training
 * Forward calls that keep what the backward needs, and the backward of the
 * layer (MoGA note, key designs 1 and 3: the layer is trained end to end; the
 * gate p(g(x)|x) on the MoGA output is the router's path to a gradient, and
 * L_gb is added to the objective).  The backward differentiates
 *   J = sum(dout * out) + dloss * L_gb
 * with g(x) = argmax and the counts treated as constants (zero gradient).
 * Q, K, V are inputs of the layer: their projection from x is outside it, so
 * x receives gradient through the router only.  Conventions as above
 * (device pointers, caller-owned buffers, asynchronous on `stream`). */

/* moga_route plus probs [N][M] fp32 out: p(i|x_t), the softmax the backward
 * differentiates. */
moga_status moga_route_train(const void* x, const void* w_r, moga_dtype dt, const float* bias,
                             int64_t N, int32_t d, int32_t M, int32_t* group_id, float* gate_prob,
                             float* probs, void* ws, size_t ws_bytes, void* stream);

/* moga_group_attn plus lse [N][H] fp32 out: the log-sum-exp of each row's
 * scaled scores in log2 units (lse = log2 sum_j 2^(q.k_j * scale * log2 e)),
 * so that P = 2^(q.k * scale * log2 e - lse).  o_moga is written as in
 * moga_group_attn (gate * attention). */
moga_status moga_group_attn_train(const void* q, const void* k, const void* v,
                                  int64_t N, int32_t H, int32_t hd,
                                  const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                  const float* gate_prob, float softmax_scale,
                                  float* o_moga, float* lse, void* ws, size_t ws_bytes, void* stream);

/* STGA with the two static branches kept apart: o_win and o_frame
 * [N][H][hd] fp32 are WRITTEN (each token is a query of exactly one window
 * group and one frame), lse_win / lse_frame [N][H] fp32 as above. */
moga_status stga_attn_train(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                            const moga_stga_geom* geom, float softmax_scale,
                            float* o_win, float* lse_win, float* o_frame, float* lse_frame,
                            void* ws, size_t ws_bytes, void* stream);

/* out[i] = bf16_rn(((o_moga[i] + o_win[i]) + o_frame[i]) / 3); n_elems % 4 == 0,
 * 16-byte aligned pointers. */
moga_status visual_attn_mean3(const float* o_moga, const float* o_win, const float* o_frame,
                              int64_t n_elems, void* out, void* stream);

/* Attention backward workspace: Q, K, V and dout copied into segment order
 * plus per-row statistics; 256-byte aligned, at least this many bytes.
 * Returns 0 for arguments the calls would reject. */
size_t moga_attn_bwd_ws_bytes(int64_t N, int32_t H, int32_t hd);

/* Backward of the MoGA branch.  Per group and head, with S = Q K^T * scale,
 * P = softmax(S), O = P V and the branch's upstream gradient
 * dO = gate * dout / 3:  dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)),
 * dQ = dS K * scale, dK = dS^T Q * scale;  dgate[t] = sum_{h,d} dout/3 * O.
 * o_moga, lse: from moga_group_attn_train;  dout [N][H][hd] bf16;
 * dq, dk, dv [N][H][hd] fp32: ADDED TO (all three branches accumulate);
 * dgate [N] fp32: written. */
moga_status moga_group_attn_bwd(const void* q, const void* k, const void* v,
                                int64_t N, int32_t H, int32_t hd,
                                const int32_t* perm, const int32_t* cu_seqlens, int32_t M,
                                const float* gate_prob, float softmax_scale,
                                const float* o_moga, const float* lse, const void* dout,
                                float* dq, float* dk, float* dv, float* dgate,
                                void* ws, size_t ws_bytes, void* stream);

/* Backward of the two static branches (window groups with their
 * adjacent-shot frames, and frames), dO = dout / 3 for each; keys shared by
 * two window groups receive both contributions.  o_win, lse_win, o_frame,
 * lse_frame: from stga_attn_train;  dq, dk, dv: ADDED TO. */
moga_status stga_attn_bwd(const void* q, const void* k, const void* v, int32_t H, int32_t hd,
                          const moga_stga_geom* geom, float softmax_scale,
                          const float* o_win, const float* lse_win,
                          const float* o_frame, const float* lse_frame, const void* dout,
                          float* dq, float* dk, float* dv, void* ws, size_t ws_bytes, void* stream);

/* Router backward workspace (dr per token, per-block partial sums of dW_r
 * and dbias); 256-byte aligned.  Returns 0 for arguments moga_route_bwd
 * would reject. */
size_t moga_route_bwd_ws_bytes(int64_t N, int32_t d, int32_t M);

/* Router backward through the gate and the balancing loss:
 *   u[t][m] = dgate[t] * [m == g_t] + dloss * alpha * M * (counts[m] / N) / N,
 *   dr[t] = p_t * (u[t] - <u[t], p_t>),
 *   dx = dr W_r^T ([N][d] fp32, written), dW_r = x^T dr ([d][M] fp32, written),
 *   dbias = sum_t dr[t] ([M] fp32, written; NULL to skip).
 * x, w_r: as for moga_route (dtype dt);  group_id, probs: from
 * moga_route_train;  dgate: from moga_group_attn_bwd;  counts: from
 * moga_permute;  dloss: the objective's weight on L_gb.  d must be a
 * positive multiple of 8 and x, dx 16-byte aligned (MOGA_ERR_INVALID_ARG
 * otherwise).  Deterministic: every sum runs in a fixed order. */
moga_status moga_route_bwd(const void* x, const void* w_r, moga_dtype dt, int64_t N, int32_t d, int32_t M,
                           const int32_t* group_id, const float* probs, const float* dgate,
                           const int32_t* counts, float alpha, float dloss,
                           float* dx, float* dw_r, float* dbias, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------- batch of videos --
 * B videos of n_per tokens each, flattened video-major (token t of video b is
 * row b * n_per + t), sharing the router (MoGA note, key design 1: routing is
 * per token; training setup: the MMDiT-based model at M = 20).  Readings: a
 * token's MoGA group holds tokens of its own video only (sort key
 * b * M + g(x), so B * M segments), the STGA groups are per video with one
 * geometry, and L_gb takes F_i and P_i over all B * n_per tokens.  Route the
 * batch with moga_route(N = B * n_per) and average with visual_attn_mean.
 */

/* Permute workspace for a batch; 0 for arguments the call would reject. */
size_t moga_permute_batched_ws_bytes(int64_t n_per, int32_t B, int32_t M);

/* Stable counting sort of B * n_per tokens by b * M + group_id:
 *   perm:       [B*n_per] int32, flattened token indices, segment-major
 *   cu_seqlens: [B*M + 1] int32;  counts: [B*M] int32 (segment b*M + i holds
 *               video b's tokens of group i);  max_seqlen: [1] int32
 * Requires B * n_per < 2^31, 1 <= M <= 32 and B * M <= 1024
 * (MOGA_ERR_UNSUPPORTED above).  Bit-identical to moga_permute when B = 1. */
moga_status moga_permute_batched(const int32_t* group_id, int64_t n_per, int32_t B, int32_t M,
                                 int32_t* perm, int32_t* cu_seqlens, int32_t* counts,
                                 int32_t* max_seqlen, void* ws, size_t ws_bytes, void* stream);

/* MoGA attention of a batch: as moga_group_attn over N = B * n_per tokens
 * with perm / cu_seqlens from moga_permute_batched (video b's groups are
 * segments [b M, b M + M)); o_acc [B*n_per][H][hd] fp32 written (=);
 * lse [B*n_per][H] fp32 (log2 domain) written when not NULL.  Workspace:
 * moga_attn_ws_bytes(B * n_per, H, hd).  One gather, one launch per video. */
moga_status moga_group_attn_batched(const void* q, const void* k, const void* v, int64_t n_per, int32_t B,
                                    int32_t H, int32_t hd, const int32_t* perm, const int32_t* cu_seqlens,
                                    int32_t M, const float* gate_prob, float softmax_scale, float* o_acc,
                                    float* lse, void* ws, size_t ws_bytes, void* stream);

/* STGA of a batch: stga_attn on each video's slice (geometry per video,
 * N = T*h*w tokens each); o_acc [B*N][H][hd] accumulates (+=).  Workspace:
 * moga_attn_ws_bytes(N, H, hd) (one video's, reused in stream order). */
moga_status stga_attn_batched(const void* q, const void* k, const void* v, int32_t B, int32_t H, int32_t hd,
                              const moga_stga_geom* geom, float softmax_scale, float* o_acc, void* ws,
                              size_t ws_bytes, void* stream);

/* L_gb of a batch: counts [B*M] from moga_permute_batched (summed over the
 * videos per group), route_ws from moga_route over the N = B * n_per tokens;
 * N must be a multiple of B.  loss: [1] double, written. */
moga_status moga_balance_loss_batched(const int32_t* counts, int32_t B, const void* route_ws, int64_t N,
                                      int32_t M, float alpha, double* loss, void* stream);

/* ------------------------------------------- router fused into Q/K/V --
 * The attention layer's Q/K/V projection (the step just before the path)
 * with the router riding on the same x tiles (MoGA note, key design 1: the
 * router is a linear projection of the same tokens), so routing needs no
 * pass of its own over x:
 *   [q | k | v][t] = W_qkv . x[t]   (fp32 accumulation, bf16 out)
 *   r = x . W_r (+ bias), p = softmax(r), g = argmax p, gate = p[g]
 * x:      [N][d] bf16;  w_qkv: [3*H*hd][d] bf16 (a linear layer's weight:
 *         rows [0, H*hd) for Q, then K, then V);  w_r: [d][M] bf16;
 *         bias: [M] fp32 or NULL
 * q, k, v: [N][H][hd] bf16, written;  group_id [N] int32, gate_prob [N]
 *         fp32, written
 * ws:     moga_qkv_route_ws_bytes(N, d, M) bytes, 256-byte aligned; on
 *         return it starts with the per-32-token sums of p(i|x) that
 *         moga_balance_loss reads, in moga_route's layout.
 * Requires d % 8 == 0, 1 <= M <= 32, 16-byte aligned x, w_qkv, q, k, v
 * (else MOGA_ERR_INVALID_ARG) and hd in {64, 128} (else
 * MOGA_ERR_UNSUPPORTED); a smaller workspace returns MOGA_ERR_WORKSPACE.
 * moga_qkv_route_ws_bytes returns 0 for arguments the call rejects. */
size_t moga_qkv_route_ws_bytes(int64_t N, int32_t d, int32_t M);
moga_status moga_qkv_route(const void* x, const void* w_qkv, const void* w_r, const float* bias, int64_t N,
                           int32_t d, int32_t H, int32_t hd, int32_t M, void* q, void* k, void* v,
                           int32_t* group_id, float* gate_prob, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------- sequence parallelism --
 * P ranks (one GPU each) share one video of N tokens, rank r holding tokens
 * [r n, (r+1) n), n = N / P (MoGA note, key design 2; translation, 方法:
 * route the local tokens, which carry every head, collect the routing results
 * of all tokens, then exchange sequence shards for head shards).  The
 * collectives belong to the caller; these calls lay out their buffers and
 * give each rank its share of the loss.  H must be a multiple of P and
 * (H / P) * hd * 2 a multiple of 16; pointers 16-byte aligned.
 */

/* src [n][H][hd] bf16 -> dst [P][n][H/P][hd] bf16: chunk j is the slice of
 * heads [j H/P, (j+1) H/P) of every local token, sent to rank j by an equal-
 * split all-to-all (which then delivers [N][H/P][hd] in token order). */
moga_status moga_sp_pack_heads(const void* src, int64_t n, int32_t H, int32_t hd, int32_t P, void* dst,
                               void* stream);

/* src [P][n][H/P][hd] bf16 (the receive buffer of the return all-to-all:
 * chunk j holds this rank's n tokens for rank j's heads) -> dst [n][H][hd]. */
moga_status moga_sp_unpack_heads(const void* src, int64_t n, int32_t H, int32_t hd, int32_t P, void* dst,
                                 void* stream);

/* This rank's share of L_gb: counts [M] over all N tokens (moga_permute of the
 * gathered group ids), route_ws from moga_route over the rank's n_local
 * tokens; F_i and P_i both normalised by N.  The sum over ranks (an
 * all-reduce) is L_gb.  loss: [1] double, written. */
moga_status moga_balance_loss_part(const int32_t* counts, const void* route_ws, int64_t n_local, int64_t N,
                                   int32_t M, float alpha, double* loss, void* stream);

/* ------------------------------------------------------------- diagnostics */
/* Text of the last host-side error of the calling thread ("" if none). */
const char* moga_last_error(void);
/* Synchronises `stream`, then reads and clears the current device's error
 * word: MOGA_OK, or the first device-side error recorded since the last
 * call (e.g. MOGA_ERR_TIMEOUT from a bounded wait). */
moga_status moga_device_status(void* stream);
/* Library version string. */
const char* moga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOGA_H */
