/*
 * ds.h -- C ABI of the token-sparse decode-attention library (libds.so).
 *
 * Method: "Post-Training Sparse Attention with Double Sparsity" (arXiv
 * 2408.07092).  A static set of important feature channels per head (channel
 * sparsity, fixed offline: Method details, Core idea / Technical framework)
 * is used to score every cached token cheaply; the tokens with the highest
 * scores are kept (Method details, Key design); exact softmax attention then
 * runs over the kept tokens only (token sparsity: Abstract, Key points 2).
 *
 * Notation (one decode step, one query token per sequence):
 *   B      sequences in the batch
 *   Hq     query heads; Hkv KV heads; Hq % Hkv == 0; query head h reads
 *          KV head g(h) = h / (Hq / Hkv)
 *   d      head dimension; the library supports d == 128 only
 *   T_cap  token capacity of the K/V and label caches; T <= T_cap tokens valid
 *   r      label channels per query head (1 <= r <= d)
 *   k      tokens kept per query head (1 <= k <= T)
 *
 * Layouts (row-major, contiguous, element type in brackets):
 *   Q      [B, Hq, d]            (bf16)
 *   K, V   [B, Hkv, T_cap, d]    (bf16)   one 256-byte row per token
 *   C      [Hq, r]               (int32)  channel ids in [0, d), ascending
 *                                         by convention (any order works)
 *   label  [B, Hq, T_cap, r]     (bf16)   label[b,h,t,j] = K[b,g(h),t,C[h,j]]
 *   scores [B*Hq, T]             (fp32)
 *   idx    [B*Hq, k]             (int32)  ascending token ids
 *   O      [B, Hq, d]            (fp32)
 *   lse    [B, Hq]               (fp32)   natural log of the softmax
 *                                         denominator, including the scale
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or synchronises.  Every pointer must be 16-byte
 *     aligned.  Calls are asynchronous on `stream` (0 = legacy default).
 *   - KV offload: K and V may instead be page-locked host memory mapped into
 *     the device's address space (cudaHostAlloc, or pinned memory under
 *     unified addressing).  The kernels then read over the host link only the
 *     rows they use: the kept rows in the sparse calls, one row per step in
 *     ds_label_append (Double Sparsity page, Abstract and Experimental
 *     highlights: combined with offloading the KV cache to host memory).
 *     Other host memory is refused with DS_ERR_INVALID_ARG before launch.
 *     ds_decode_step and ds_decode_step_kv also take Q, O and lse (and
 *     ds_decode_step_kv its new K/V rows, as ds_kv_append does) in such host
 *     memory: a decode loop then hands the step its query and reads its
 *     result with no copy of their own (the kernel reads Q and writes O over
 *     the host link).
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns DS_ERR_INVALID_ARG (or DS_ERR_UNSUPPORTED for a valid
 *     but unimplemented shape) and launches nothing.
 *   - Device-side values the host cannot see cheaply (channel ids, token
 *     indices) are masked or clamped into range inside the kernels so that no
 *     access leaves its buffer; each such event sets a bit in a per-device
 *     status word read by ds_device_status().  Kernels never trap.
 *   - A launch failure returns DS_ERR_CUDA (details: ds_last_cuda_error()).
 *   - Calls on different streams may run concurrently if their outputs and
 *     workspaces do not overlap.
 */
#ifndef POST_TOKEN_SPARSE_DS_H_
#define POST_TOKEN_SPARSE_DS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same opaque handle as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st* ds_stream_t;

typedef enum {
  DS_OK = 0,
  DS_ERR_INVALID_ARG = 1, /* null/misaligned pointer, out-of-range size     */
  DS_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d != 128)      */
  DS_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required     */
  DS_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed    */
} ds_status;

typedef struct {
  int32_t B, Hq, Hkv, d, T_cap, r;
} ds_dims;

/* Operation ids for ds_workspace_size(). */
enum {
  DS_OP_LABEL_APPEND = 0,
  DS_OP_SCORE = 1,
  DS_OP_TOPK = 2,
  DS_OP_SPARSE_DECODE = 3,
  DS_OP_DECODE = 4,
  DS_OP_SCORE_TOPK = 5,
  DS_OP_DECODE_STEP = 6,
  DS_OP_CALIBRATE = 7, /* k: calibration queries per head (Nq) */
  DS_OP_GROUP_SPARSE_DECODE = 8,
  DS_OP_BLOCK_SPARSE_DECODE = 9, /* k: kept rows = kb * bs */
  DS_OP_GROUP_DECODE_STEP = 10
};

/* Device status bits (ds_device_status). */
enum {
  DS_DEV_BAD_CHANNEL = 1u, /* a channel id in C was outside [0, d); masked  */
  DS_DEV_BAD_INDEX = 2u,   /* a token index was outside [0, T); clamped     */
  DS_DEV_TIMEOUT = 4u      /* a bounded in-kernel wait ran out: that call's
                              results are invalid (the kernel returned
                              instead of hanging)                           */
};

/*
 * ds_kv_append -- write one decode step's new K and V rows into the caches.
 *
 * K[b,g,t,:] = K_new[b,g,:] and V[b,g,t,:] = V_new[b,g,:] for every b, g.
 * K_new, V_new: [B, Hkv, d] bf16, device memory or page-locked host memory
 * mapped into the device (read directly; no separate host-to-device copy).
 * K, V: the caches, as for ds_sparse_decode (device or mapped host memory).
 * Requires 0 <= t < T_cap.  Bit-exact copy; one launch.  A decode step then
 * appends the label row of token t (ds_label_append, or ds_decode_step with
 * append) and attends with T = t + 1.
 */
ds_status ds_kv_append(const void* K_new, const void* V_new, void* K, void* V, ds_dims dims,
                       int32_t t, ds_stream_t stream);

/*
 * ds_label_append -- build or extend the label cache.
 *
 * label[b,h,t,j] = K[b, g(h), t, C[h,j]] for every b, h, j and
 * t0 <= t < t0 + n.  The label cache is the contiguous copy of each query
 * head's r calibrated channels of K (channel sparsity; Double Sparsity page,
 * Method details: Core idea and Technical framework -- the channel pattern is
 * static, so it is found offline and applied at run time).  Call once over
 * the prompt (t0 = 0, n = T) and once per generated token (t0 = T-1, n = 1).
 *
 * K: [B,Hkv,T_cap,d] bf16.  C: [Hq,r] int32.  label: [B,Hq,T_cap,r] bf16,
 * written only in rows [t0, t0+n).  Requires 0 <= t0, 1 <= n,
 * t0 + n <= T_cap.  Bit-exact copy: no arithmetic.
 */
ds_status ds_label_append(const void* K, const int32_t* C, void* label, ds_dims dims,
                          int32_t t0, int32_t n, ds_stream_t stream);

/*
 * ds_score -- approximate (channel-sparse) attention scores.
 *
 * scores[b*Hq+h, t] = sum_j q[b,h,C[h,j]] * label[b,h,t,j] for t < T,
 * unscaled, products and sums in fp32.  The tokens with the higher values of
 * this score are the important ones (Double Sparsity page, Method details:
 * Key design).
 *
 * Q: [B,Hq,d] bf16.  C: [Hq,r] int32.  label: [B,Hq,T_cap,r] bf16.
 * scores: [B*Hq, T] fp32.  Requires 1 <= T <= T_cap.
 */
ds_status ds_score(const void* Q, const int32_t* C, const void* label, float* scores,
                   ds_dims dims, int32_t T, ds_stream_t stream);

/*
 * ds_topk -- per-row top-k token indices.
 *
 * For each of the BH rows of `scores` ([BH, T] fp32), writes to idx ([BH, k]
 * int32) the k indices with the largest scores, ascending.  Ties go to the
 * lower index; -0.0 and +0.0 are equal; +-inf order normally; NaN is outside
 * the contract (no fault, unspecified choice).  Token selection by the higher
 * activation (Double Sparsity page, Method details: Key design).
 *
 * Requires 1 <= k <= T <= 1048576 and BH <= 65535.  ws: NULL, or
 * ds_workspace_size(DS_OP_TOPK, dims, T, k) bytes (dims.B * dims.Hq = BH) of
 * 16-byte aligned device memory, zero-filled before first use (its counters
 * are left at zero).  When that size is nonzero (4096 < T <= 16384) and ws
 * is given, one launch turns tiles of 4096 scores into 16-bit key prefixes
 * and the last tile of each row selects from them (exact keys from the
 * scores); otherwise the selection kernel reads the scores directly.  Same
 * result either way.
 */
ds_status ds_topk(const float* scores, int32_t* idx, int32_t BH, int32_t T, int32_t k,
                  void* ws, size_t ws_bytes, ds_stream_t stream);

/*
 * ds_score_topk -- ds_score followed by ds_topk.
 *
 * Same results as the two calls (same fp32 scores, same index set).  With a
 * workspace of ds_workspace_size(DS_OP_SCORE_TOPK, dims, T, k) bytes (nonzero
 * when r is 8, 16, 32, 64 or 128 and 4096 < T <= 32768): one launch that
 * scores tiles of every head, keeps each token's 16-bit key prefix in the
 * workspace, and selects each head in the CTA that finishes its last tile.
 * Otherwise (no workspace, or other sizes): with scores == NULL one launch
 * that computes the scores while selecting; with a scores buffer the same
 * launch, except for r >= 16 and T > 4096, where the scores are written first
 * and the selection reads them (two launches).  scores ([B*Hq, T] fp32) is
 * written when given.  ws: device memory, zero-filled before its first use
 * (its first 256 KiB hold per-head counters that every call leaves at zero);
 * may be NULL.  Limits as for ds_topk.
 */
ds_status ds_score_topk(const void* Q, const int32_t* C, const void* label, float* scores,
                        int32_t* idx, ds_dims dims, int32_t T, int32_t k, void* ws,
                        size_t ws_bytes, ds_stream_t stream);

/*
 * ds_sparse_decode -- exact softmax attention over the selected tokens.
 *
 * For each (b, h) with rows i = idx[b*Hq+h, 0..k):
 *   l_i = scale * (q[b,h,:] . K[b,g(h),i,:]);  w = softmax(l);
 *   O[b,h,:] = sum_i w_i V[b,g(h),i,:];  lse[b,h] = log sum_i exp(l_i).
 * Self-attention computed with the important tokens only (Double Sparsity
 * page, Abstract; Key points 2).  The k rows of all heads, head after head,
 * are cut into equal contiguous ranges, one per warp of a grid of one
 * 16-warp CTA per SM; each range keeps a running max and sum per head it
 * touches, and a head shared by several ranges is combined by log-sum-exp
 * weights (first within a CTA, then across CTAs).  fp32 accumulation.
 *
 * Q: [B,Hq,d] bf16; K, V: [B,Hkv,T_cap,d] bf16; idx: [B*Hq,k] int32 with
 * entries in [0, T) (out-of-range entries are clamped and flagged);
 * O: [B,Hq,d] fp32; lse: [B,Hq] fp32 or NULL.  Requires 1 <= k <= T <= T_cap.
 * ws: ds_workspace_size(DS_OP_SPARSE_DECODE, dims, T, k) bytes of device
 * memory, zero-filled before its first use; may be NULL when that size is 0.
 * Its first 256 KiB hold one arrival counter per head at a fixed place, which
 * every call leaves at zero again, and the per-range partials follow; so one
 * buffer of the largest size needed serves any number of calls, of any sizes,
 * that do not overlap on the GPU.  Calls that may overlap on the GPU need
 * separate workspaces.
 */
ds_status ds_sparse_decode(const void* Q, const void* K, const void* V, const int32_t* idx,
                           float* O, float* lse, ds_dims dims, int32_t T, int32_t k, float scale,
                           void* ws, size_t ws_bytes, ds_stream_t stream);

/*
 * ds_decode_step -- one whole token-sparse decode step: the calls above in the
 * order a decoder makes them, fused into one launch where the sizes allow.
 *
 * With append != 0, first the label row of the newest token (t = T-1) is
 * written, as ds_label_append(K, C, label, dims, T-1, 1) would; then the top-k
 * selection of ds_score_topk (the same index set, written to idx) and the
 * attention of ds_sparse_decode over it.  Double Sparsity's decode: the
 * calibrated channels pick the important tokens (Method details: Core idea,
 * Key design) and self-attention runs over those tokens only (Abstract).
 *
 * One CTA per query head performs the three phases on chip when r is 8, 16,
 * 32, 64 or 128, k <= 8192, B*Hq <= 296 (one wave of two CTAs per SM) and the
 * head's selection fits one CTA; otherwise the three calls are issued on
 * `stream` (the selection through a score buffer in the workspace when
 * r >= 16 and T > 4096, or the one-launch selection, see ds_score_topk).
 * idx: [B*Hq, k] int32
 * (required).  O and lse as for ds_sparse_decode; the attention's summation
 * order may differ from ds_sparse_decode's (fp32 rounding only).  ws:
 * ds_workspace_size(DS_OP_DECODE_STEP, dims, T, k) bytes, zero-filled before
 * first use (0 bytes when fused).  Other arguments as for the calls above.
 */
ds_status ds_decode_step(const void* Q, const void* K, const void* V, const int32_t* C,
                         void* label, int32_t* idx, float* O, float* lse, ds_dims dims,
                         int32_t T, int32_t k, float scale, int32_t append, void* ws,
                         size_t ws_bytes, ds_stream_t stream);

/*
 * ds_decode_step_kv -- ds_decode_step for a decoder that hands over the newest
 * token's K and V rows with the step.
 *
 * Exactly ds_kv_append(K_new, V_new, K, V, dims, T-1) followed by
 * ds_decode_step(Q, K, V, C, label, idx, O, lse, dims, T, k, scale, 1, ...):
 * the new rows are stored at t = T-1, the label row of t = T-1 is appended,
 * then top-k selection and sparse attention over the T tokens.  Where
 * ds_decode_step runs as one launch, so does this call: the new rows are
 * stored by the step kernel itself, which also reads token T-1's rows from
 * K_new / V_new.  The online inference phase of Double Sparsity (page, Method
 * details: Technical framework) runs once per generated token; storing that
 * token's K and V first is ordinary decoder bookkeeping, which the pages do
 * not describe (the plainest reading: the new token is attended to).
 *
 * K_new, V_new: [B, Hkv, d] bf16, device memory or page-locked host memory
 * mapped into the device; they must not overlap K, V or label.  K, V: the
 * caches, written in row T-1 only.  Requires 1 <= T <= T_cap.  Q, O and lse
 * may be mapped host memory as for ds_decode_step; other arguments, results,
 * errors and the workspace (DS_OP_DECODE_STEP) as for ds_decode_step.
 */
ds_status ds_decode_step_kv(const void* Q, const void* K_new, const void* V_new, void* K,
                            void* V, const int32_t* C, void* label, int32_t* idx, float* O,
                            float* lse, ds_dims dims, int32_t T, int32_t k, float scale,
                            void* ws, size_t ws_bytes, ds_stream_t stream);

/*
 * ds_decode -- dense decode attention over all T cached tokens: the operation
 * token sparsity accelerates (Double Sparsity page, Experimental highlights:
 * attention-operation speed-up).  Same as ds_sparse_decode with
 * idx = 0..T-1 for every head.  ws: ds_workspace_size(DS_OP_DECODE, dims, T,
 * T) bytes, zero-filled before first use as for ds_sparse_decode.
 */
ds_status ds_decode(const void* Q, const void* K, const void* V, float* O, float* lse,
                    ds_dims dims, int32_t T, float scale, void* ws, size_t ws_bytes,
                    ds_stream_t stream);

/*
 * ds_sparse_decode_noalloc -- ds_sparse_decode for callers that cannot
 * allocate device memory.  (The paper has no counterpart: this is a property
 * of the library's interface, not of the method.)
 *
 * Some callers cannot hand the library a workspace: a serving loop that
 * reserved all of HBM for its KV cache at start-up and forbids further
 * allocation (so a request can never fail with out-of-memory half-way), code
 * on a latency-critical path where cudaMalloc's implicit device-wide
 * synchronisation is unacceptable, or a plug-in that is given only its input
 * and output buffers by a host framework that owns all device memory.  This
 * call computes exactly what ds_sparse_decode computes, with the same kernels
 * and the same split plan, but keeps the split partials in a fixed array
 * inside the library (DS_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU
 * that loads the library until the process exits).  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Arguments as for ds_sparse_decode, without ws / ws_bytes.  Returns
 * DS_ERR_WORKSPACE, launching nothing, when the workspace these sizes need
 * (ds_workspace_size(DS_OP_SPARSE_DECODE, dims, T, k)) exceeds
 * DS_NOALLOC_SCRATCH_BYTES.  With the work plan of ds_sparse_decode that does
 * not happen for sizes the library accepts: heads are shared by several warps
 * only when there are fewer heads than warps in the grid (148 CTAs of 16), so
 * at most 148 + 2367 partials of 528 bytes follow the 256 KiB of counters
 * (1.6 MB).  Sizes beyond the library's limits (B*Hq > 65535) return
 * DS_ERR_UNSUPPORTED.
 *
 * The first call on each device looks up the array's device address with
 * that device current (cudaGetSymbolAddress).  All calls on a device share
 * the one array and it keeps the previous call's contents.
 * Its layout is that of the ds_sparse_decode workspace: the per-head counters
 * sit at its start, are zero when the library is loaded and are left at zero
 * by every call, so no call has to clear anything first.  Calls that may
 * overlap on the GPU -- on different streams without an ordering between them
 * -- race on the array and must not be issued.
 */
#define DS_NOALLOC_SCRATCH_BYTES (4u << 20)
ds_status ds_sparse_decode_noalloc(const void* Q, const void* K, const void* V,
                                   const int32_t* idx, float* O, float* lse, ds_dims dims,
                                   int32_t T, int32_t k, float scale, ds_stream_t stream);

/*
 * ds_group_score_topk -- one token selection per KV group (grouped KV heads).
 *
 * The G = Hq/Hkv query heads of a group read the same K/V rows; selecting
 * once per group lets each kept row be read once for all of them (token
 * sparsity, Double Sparsity page, Abstract and Key points 2; the page gives
 * no group score -- reading taken: the sum of the member heads' approximate
 * scores).  group_scores[b*Hkv+g, t] = sum over h = g*G .. g*G+G-1, in that
 * order, of the fp32 score ds_score gives for head h (same operation order),
 * for t < T; idx[b*Hkv+g] = the k tokens of largest group score, ties to the
 * lower index, ascending (as ds_topk).
 *
 * Q: [B,Hq,d] bf16.  C: [Hq,r] int32.  label: [B,Hq,T_cap,r] bf16.
 * group_scores: [B*Hkv, T] fp32 (written; the caller's buffer).  idx:
 * [B*Hkv, k] int32.  Requires r in {8,16,32,64,128}, G*r <= 12288,
 * 1 <= k <= T <= min(T_cap, 1048576).  Two launches.
 */
ds_status ds_group_score_topk(const void* Q, const int32_t* C, const void* label,
                              float* group_scores, int32_t* idx, ds_dims dims, int32_t T,
                              int32_t k, ds_stream_t stream);

/*
 * ds_group_sparse_decode -- attention over the group's kept tokens.
 *
 * As ds_sparse_decode, except that idx has one row per KV group
 * ([B*Hkv, k], e.g. from ds_group_score_topk) and every query head of the
 * group attends over its group's row.  The group's heads are adjacent in
 * launch order, so a kept K/V row is fetched from HBM once and served to the
 * other heads from L2.  ws: ds_workspace_size(DS_OP_GROUP_SPARSE_DECODE, dims,
 * T, k) bytes, zero-filled before first use (left zero-filled).
 */
ds_status ds_group_sparse_decode(const void* Q, const void* K, const void* V,
                                 const int32_t* idx, float* O, float* lse, ds_dims dims,
                                 int32_t T, int32_t k, float scale, void* ws, size_t ws_bytes,
                                 ds_stream_t stream);

/*
 * ds_group_decode_step -- one decode step with group-shared selection:
 * ds_label_append(K, C, label, dims, T-1, 1) (when append != 0), then
 * ds_group_score_topk and ds_group_sparse_decode, in three launches instead
 * of four: the group-score kernel appends the newest token's label rows (the
 * CTA whose tile holds token T-1 gathers them from K) and scores that token
 * from them.  Results identical to the three calls.
 *
 * Arguments as for those calls (label written at T-1 when append != 0).  ws:
 * ds_workspace_size(DS_OP_GROUP_DECODE_STEP, dims, T, k) bytes, zero-filled
 * before first use: the attention's workspace, then, for 4096 < T <= 16384,
 * that of the one-launch top-k over the group scores (as ds_topk's).
 * Requires what ds_group_score_topk requires, with G*r*6 <= 49152.
 */
ds_status ds_group_decode_step(const void* Q, const void* K, const void* V, const int32_t* C,
                               void* label, float* group_scores, int32_t* idx, float* O,
                               float* lse, ds_dims dims, int32_t T, int32_t k, float scale,
                               int32_t append, void* ws, size_t ws_bytes, ds_stream_t stream);

/*
 * ds_block_score_topk -- block-granular token selection.
 *
 * Block informativeness (page "Jenga: Enhancing LLM Long-Context Fine-tuning
 * with Contextual Token Sparsity", Core method 1: a token's informativeness
 * counts positive scores only, a block's is the largest of its tokens';
 * Observation 2: blocks of 64 tokens).  block_scores[bh, j] = max over the
 * tokens t of block j (t in [j*bs, min((j+1)*bs, T))) of max(s[bh,t], 0), s
 * the fp32 score of ds_score; bidx[bh] = the kb blocks of largest block score,
 * ties to the lower block, ascending (a fixed count: the page keeps blocks
 * against a threshold tuned per layer on a model).
 *
 * Q, C, label as for ds_score.  block_scores: [B*Hq, ceil(T/bs)] fp32
 * (written).  bidx: [B*Hq, kb] int32.  Requires bs a power of two <= 64, r in
 * {8,16,32,64,128}, 1 <= kb <= ceil(T/bs), T <= T_cap.  Two launches.
 */
ds_status ds_block_score_topk(const void* Q, const int32_t* C, const void* label,
                              float* block_scores, int32_t* bidx, ds_dims dims, int32_t T,
                              int32_t bs, int32_t kb, ds_stream_t stream);

/*
 * ds_block_sparse_decode -- attention over the tokens of the kept blocks.
 *
 * As ds_sparse_decode over the kb*bs rows of the blocks bidx[bh] ([B*Hq, kb],
 * e.g. from ds_block_score_topk): row r is token bidx[bh, r/bs]*bs + r%bs;
 * rows at or past T (the short last block) are skipped.  A block's rows are
 * contiguous in K and V, so the gathers read whole runs of bs rows.  ws:
 * ds_workspace_size(DS_OP_BLOCK_SPARSE_DECODE, dims, T, kb*bs) bytes,
 * zero-filled before first use (left zero-filled).
 */
ds_status ds_block_sparse_decode(const void* Q, const void* K, const void* V,
                                 const int32_t* bidx, float* O, float* lse, ds_dims dims,
                                 int32_t T, int32_t bs, int32_t kb, float scale, void* ws,
                                 size_t ws_bytes, ds_stream_t stream);

/*
 * ds_hier_score_topk -- hierarchical (top-down) token selection.
 *
 * Page "A Training-free Sub-quadratic Cost Transformer Model Serving
 * Framework With Hierarchically Pruned Attention": nearby tokens score alike
 * (Core idea, attention locality), and a hierarchy of tokens is searched
 * tree-like for each query's important keys (Technical framework).  Reading:
 * k contiguous parts of [0, T) (part i = [floor(iT/k), floor((i+1)T/k))) are
 * halved level by level (the first half takes the extra token); each part is
 * scored by its first token's approximate score (as ds_score computes it); the
 * k best parts stay (score descending, start ascending); when every part is
 * one token, idx[bh] = those k tokens, ascending.  Reads about 2k*log2(T/k)
 * label rows per head instead of T; equals ds_score_topk when the scores fall
 * with position or k = T, and otherwise is an approximation that relies on
 * locality.
 *
 * Q, C, label as for ds_score.  idx: [B*Hq, k] int32.  Requires r in
 * {8,16,32,64,128}, 1 <= k <= min(T, 2048), T <= T_cap.  One launch, no
 * workspace.
 */
ds_status ds_hier_score_topk(const void* Q, const int32_t* C, const void* label, int32_t* idx,
                             ds_dims dims, int32_t T, int32_t k, ds_stream_t stream);

/*
 * ds_calibrate -- offline channel calibration: the label channels C.
 *
 * The channel pattern is static, so it is fixed offline from a calibration
 * set (Double Sparsity page, Method details: Core idea and Technical
 * framework); the page leaves the criterion open ("unknown", Key design).
 * Reading taken: the importance of channel c for query head h is the mean,
 * over every pair (calibration query n, cached token t < T) of the same
 * sequence b, of |q[b,h,n,c] * k[b,g(h),t,c]|:
 *   I[h,c] = sum_b (sum_n |q[b,h,n,c]|) * (sum_t |k[b,g(h),t,c]|) / (B*Nq*T),
 * column sums in fp32 in a fixed order (deterministic).  C[h] holds the r
 * channels of largest I[h,.] (ties to the lower channel), ascending -- the
 * input ds_label_append expects.
 *
 * Qc: [B,Hq,Nq,d] bf16 calibration queries.  K: [B,Hkv,T_cap,d] bf16, rows
 * t < T read.  C: [Hq, r] int32 out (r = dims.r).  importance: [Hq, d] fp32
 * out, or NULL.  ws: ds_workspace_size(DS_OP_CALIBRATE, dims, T, Nq) bytes of
 * device memory (scratch; no contents required).  Requires 1 <= T <= T_cap,
 * Nq >= 1, 1 <= r <= d.  Two launches, no host synchronisation.
 */
ds_status ds_calibrate(const void* Qc, int32_t Nq, const void* K, ds_dims dims, int32_t T,
                       int32_t* C, float* importance, void* ws, size_t ws_bytes,
                       ds_stream_t stream);

/*
 * Bytes of device workspace `op` needs for these sizes (0 if none).  Depends
 * only on the arguments, never on the device.  Returns 0 for invalid sizes.
 */
size_t ds_workspace_size(int32_t op, ds_dims dims, int32_t T, int32_t k);

/* Human-readable name of a status code (static storage). */
const char* ds_status_string(ds_status s);

/* Text of the last CUDA error seen by this library on the calling thread. */
const char* ds_last_cuda_error(void);

/*
 * Reads (and, if `clear` != 0, resets) the status bits that kernels set on
 * the current device (DS_DEV_*).  Synchronises `stream` first.
 */
ds_status ds_device_status(uint32_t* bits, int32_t clear, ds_stream_t stream);

/* Number of kernels this library has launched in this process (host count). */
uint64_t ds_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* POST_TOKEN_SPARSE_DS_H_ */
