/*
 * lighthouse.h - C ABI of the Lighthouse Attention layer's hot path on one
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one of "Long Context Pre-Training with Lighthouse
 * Attention" (arXiv 2605.06554): a four-stage pipeline that replaces causal
 * scaled dot-product attention (Sec. 3.2):
 *   (i)   symmetric mean pooling of per-head Q, K, V into an L-level pyramid
 *         with pooling factor p (Sec. 3.3);
 *   (ii)  parameter-free scores (per-head l2 norms at level 0, max-pooled at
 *         coarser levels) and one joint top-k over the QK and KQ streams
 *         (Sec. 3.4);
 *   (iii) a gather of the selected (Q, K, V) triples into a contiguous
 *         sub-sequence of length S = N/p^(L-1) + (L-1) p k, ordered so that a
 *         plain S x S causal mask applies, and dense causal softmax attention
 *         over it (Sec. 3.5, Eq. 8 and 9);
 *   (iv)  a scatter of each output back to the base positions it represents,
 *         shifted by p^l - 1 (Sec. 3.6);
 * plus the backward of (iv), (iii) and the gather/pooling into dQ, dK, dV
 * (Sec. 3.2: the selection itself carries no gradient).
 *
 * Conventions shared by every call
 * --------------------------------
 * - bf16 tensors are passed as lh_bf16 (the raw 16-bit pattern).  Token
 *   tensors are [B, N, H, d] row-major; gathered tensors are [B, H, S, d];
 *   per-entry arrays are [B, H, P] with P = sum_{l<L} N / p^l and the flat
 *   pyramid index f(l, i) = sum_{l'<l} N/p^l' + i.
 * - Every pointer that a kernel touches is a device pointer on the current
 *   device, 16-byte aligned, and the buffers must not overlap.  The caller
 *   owns all memory: no entry point allocates, frees or synchronises, except
 *   lh_get_device_status, which synchronises the given stream.
 * - `stream` is a cudaStream_t (passed as void*; NULL = legacy stream).  All
 *   work is enqueued on it, asynchronously.
 * - Errors: argument errors are reported synchronously, before any launch
 *   (LH_ERR_INVALID_ARGUMENT, LH_ERR_UNSUPPORTED, LH_ERR_WORKSPACE).  A
 *   failed launch returns LH_ERR_CUDA.  Errors found on the device (a wait
 *   that ran out, an index out of range) are recorded in a device status word
 *   that lh_get_device_status reads and clears.
 * - Determinism: the same inputs give the same output bits, run after run.
 * - Inputs must be finite.
 */
#ifndef LIGHTHOUSE_H
#define LIGHTHOUSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t lh_bf16; /* bit pattern of a bfloat16 value */

typedef enum {
  LH_OK = 0,
  LH_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size or config */
  LH_ERR_UNSUPPORTED = 2,      /* valid for the method, not built here (e.g. d) */
  LH_ERR_WORKSPACE = 3,        /* workspace or saved buffer too small */
  LH_ERR_CUDA = 4,             /* a CUDA launch or driver call failed */
  LH_ERR_DEVICE_TIMEOUT = 5,   /* a bounded device-side wait ran out */
  LH_ERR_DEVICE_BOUNDS = 6     /* a device-side index check failed */
} lh_status;

/* One layer call.  Sec. 3.3 requires p^(L-1) | N; the budget (L-1) p k must
 * not exceed the finer-level entry count.  scale <= 0 selects 1/sqrt(d).
 * scatter_mode: 0 = gather-side (pull) scatter; 1 = fixed-point integer
 * atomic scatter (same placement, order-independent sums).
 * select_mode: 0 = one joint top-k over all finer levels (Sec. 3.4);
 *   1 = per-level quota: each of the L-1 finer levels contributes exactly
 *   p k entries (the Eq. 8 accounting read literally), chosen within the
 *   level by the same key order; needs p k <= N / p^(L-2);
 *   2 = stratified (the chunked top-k of the implementation note in Sec. 3):
 *   the finer-level entries, in flat-index order, are cut into
 *   n = (L-1) p k / select_chunk contiguous chunks, chunk s covering
 *   [floor(s C / n), floor((s+1) C / n)) of the C candidates, and each chunk
 *   keeps its top select_chunk entries by the same key order; select_chunk
 *   must be >= 1 and divide (L-1) p k (else LH_ERR_INVALID_ARGUMENT), and
 *   B H n must be below 2^31 (else LH_ERR_UNSUPPORTED).
 *   S is the same in every mode.  Other values: LH_ERR_UNSUPPORTED.
 * select_chunk: the per-chunk quota m of select_mode 2; ignored otherwise. */
typedef struct {
  int64_t B, N, H, d, L, p, k;
  float scale;
  int32_t scatter_mode;
  int32_t select_mode;
  int64_t select_chunk;
} lh_config;

/* Returns LH_OK when the config is valid and supported: B, N, H >= 1,
 * p >= 2, 1 <= L <= 6, p^(L-1) | N, 0 <= (L-1) p k <= sum_{l<L-1} N/p^l,
 * d in {64, 128}, every index fits in int32 per (b, h), and B H (times L-1
 * in select_mode 1) <= 65535, the launch-grid limit of the per-head
 * selection kernels (else LH_ERR_UNSUPPORTED). */
lh_status lh_config_check(const lh_config* cfg);

/* S = N/p^(L-1) + (L-1) p k (Sec. 3.5, Eq. 8); -1 for an invalid config. */
int64_t lh_subseq_len(const lh_config* cfg);

/* P = sum_{l=0}^{L-1} N / p^l, entries per (b, h) (Sec. 3.3); -1 if invalid. */
int64_t lh_total_entries(const lh_config* cfg);

/* Pooled rows per batch row: sum_{l=1}^{L-1} N / p^l; -1 if invalid. */
int64_t lh_pooled_rows(const lh_config* cfg);

/* Byte sizes of the caller-owned buffers:
 *  fwd_ws  - scratch of lh_forward and lh_score_topk;
 *  bwd_ws  - scratch of lh_backward and lh_attn_bwd;
 *  saved   - what lh_forward leaves for lh_backward (see lh_saved_offsets).
 * Any output pointer may be NULL. */
lh_status lh_workspace_bytes(const lh_config* cfg, size_t* fwd_ws, size_t* bwd_ws,
                             size_t* saved);

/* Byte offsets inside the saved buffer, in this order: sel_idx (int32
 * [B,H,S]), slot_map (int32 [B,H,P]), qg, kg, vg, og, og_lo (bf16
 * [B,H,S,d]), lse (fp32 [B,H,S]).  `offsets` has room for 8 values. */
lh_status lh_saved_offsets(const lh_config* cfg, size_t* offsets);

/* Byte offsets inside the backward scratch (bwd_ws) that lh_backward leaves
 * filled when it returns, in this order: delta (fp32 [B,H,S], D of the
 * attention backward), dog (bf16 [B,H,S,d], the scatter adjoint), dqg, dkg,
 * dvg (bf16 [B,H,S,d], the gradients of the gathered sub-sequence).
 * `offsets` has room for 5 values.  Lets a caller inspect the per-stage
 * results of the layer backward without a second run. */
lh_status lh_bwd_ws_offsets(const lh_config* cfg, size_t* offsets);

/* (i) + the level-0/coarse scores of (ii), in one pass over Q, K, V.
 * Sec. 3.3: level l, entry i = mean of base rows i p^l .. (i+1) p^l - 1.
 * Sec. 3.4: qk/kq at level 0 are ||Q_t||_2 and ||K_t||_2 (squares summed in
 * fp64, fp64 square root, rounded once to fp32); at level l they are the max
 * of the level-0 scores in the window.
 *  q, k, v        in  bf16 [B, N, H, d]
 *  q_lv,k_lv,v_lv out bf16, levels 1..L-1 back to back; level l is
 *                     [B, N/p^l, H, d] and starts after the rows of levels
 *                     1..l-1 (lh_pooled_rows rows per batch row in total);
 *                     may be NULL when L == 1
 *  qk, kq         out fp32 [B, H, P]                                      */
lh_status lh_pyramid(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                     const lh_bf16* v, lh_bf16* q_lv, lh_bf16* k_lv, lh_bf16* v_lv,
                     float* qk, float* kq, void* stream);

/* (ii) joint top-k and the topological order of (iii), Sec. 3.4-3.5.
 * Exactly (L-1) p k entries of levels 0..L-2 are chosen per (b, h) by the
 * key r = max(qk, kq), descending, ties to the lower flat index; all of
 * level L-1 is added.  select_mode 1 takes p k from each finer level and
 * select_mode 2 select_chunk from each chunk (see lh_config), by the same
 * key.  Entries are ordered by their last base token e = (i+1) p^l - 1,
 * then by level.
 *  sel_idx  out int32 [B, H, S]  flat pyramid index of each slot
 *  slot_map out int32 [B, H, P]  slot of each entry, -1 if not selected
 *  ws       scratch of at least fwd_ws bytes (lh_workspace_bytes)          */
lh_status lh_score_topk(const lh_config* cfg, const float* qk, const float* kq,
                        int32_t* sel_idx, int32_t* slot_map, void* ws, size_t ws_bytes,
                        void* stream);

/* lh_score_topk for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a convenience of this library.  Some callers
 * cannot hand the library a workspace: their device memory is owned by
 * another allocator that must not be bypassed, their plugin interface has no
 * slot for a scratch pointer, or their step may not allocate at all.  This
 * entry point needs none: its scratch is a fixed 8 MiB device array inside
 * the library (lh_score_topk_noalloc_max_bytes), held by every device that
 * loads the library until the process exits.  It allocates nothing and
 * calls no allocating routine.
 *  - Same arguments and results as lh_score_topk, minus ws / ws_bytes.
 *  - Returns LH_ERR_WORKSPACE, before any launch, when the selection
 *    scratch of cfg (the part of fwd_ws that lh_score_topk uses) exceeds the
 *    array.  That scratch is, roughly: select_mode 0, B*H*48 KB of digit
 *    histograms; select_mode 1, B*H*(L-1)*48 KB; select_mode 2, B*H*n*24
 *    bytes for its n chunks; plus B*H*N/256 bytes of order counts in every
 *    mode.  So B*H <= 128 heads fit at N = 2^20 in modes 0 and 2, and
 *    B*H*(L-1) <= 128 in mode 1.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears what it needs zeroed.  Calls whose work
 *    overlaps on the GPU (different streams, no ordering between them) race
 *    on the array: order them, e.g. on one stream. */
lh_status lh_score_topk_noalloc(const lh_config* cfg, const float* qk, const float* kq,
                                int32_t* sel_idx, int32_t* slot_map, void* stream);

/* Size in bytes of the fixed scratch array of lh_score_topk_noalloc. */
size_t lh_score_topk_noalloc_max_bytes(void);

/* (iii) gather: row m of qg/kg/vg is the pyramid entry sel_idx[m]
 * (level 0 from q/k/v, coarser levels from q_lv/k_lv/v_lv).
 *  qg, kg, vg out bf16 [B, H, S, d]                                        */
lh_status lh_gather(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                    const lh_bf16* v, const lh_bf16* q_lv, const lh_bf16* k_lv,
                    const lh_bf16* v_lv, const int32_t* sel_idx, lh_bf16* qg,
                    lh_bf16* kg, lh_bf16* vg, void* stream);

/* (iii) causal softmax attention over the gathered sub-sequence (Eq. 9):
 * og[m] = sum_{m' <= m} softmax(scale qg[m].kg[m']) vg[m'], lse[m] = natural
 * log of the softmax normaliser.  tcgen05 tensor cores, fp32 accumulation.
 *  qg, kg, vg in  bf16 [B, H, S, d];  og out bf16 [B, H, S, d] (the fp32
 *  result rounded once); og_lo out bf16 [B, H, S, d] or NULL: the rounding
 *  residual, so og + og_lo carries the output to ~16 significant bits for
 *  the D = rowsum(dO * O) of the backward;  lse out fp32 [B, H, S]        */
lh_status lh_attn_fwd(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                      const lh_bf16* vg, lh_bf16* og, lh_bf16* og_lo, float* lse,
                      void* stream);

/* Backward of lh_attn_fwd (Sec. 3.2: gradients flow from the loss through
 * stages (iv) and (iii) into the gathered Q, K, V; the attention is the
 * masked softmax attention of Sec. 3.5, Eq. 9, so its backward is the
 * standard one): with P the softmax rows, D = rowsum(dog * O)
 * (O = og + og_lo; og_lo may be NULL), dS = P (dog vg^T - D):
 * dqg = scale dS kg, dkg = scale dS^T qg, dvg = P^T dog.  Deterministic (no
 * floating-point atomics).  Computes D into ws (>= bwd_ws bytes), then runs
 * lh_attn_bwd_dkdv and lh_attn_bwd_dq. */
lh_status lh_attn_bwd(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                      const lh_bf16* vg, const lh_bf16* og, const lh_bf16* og_lo,
                      const float* lse, const lh_bf16* dog, lh_bf16* dqg, lh_bf16* dkg,
                      lh_bf16* dvg, void* ws, size_t ws_bytes, void* stream);

/* The dK/dV half of lh_attn_bwd (Sec. 3.2 and 3.5, Eq. 9), given delta = D
 * (fp32 [B, H, S], e.g. from lh_scatter_bwd): one CTA per 128 key rows walks
 * the query rows at and after its diagonal.  qg, kg, vg, dog in bf16
 * [B, H, S, d]; lse in fp32 [B, H, S] from lh_attn_fwd; dkg, dvg out bf16
 * [B, H, S, d].  Deterministic: each output row is written by one thread. */
lh_status lh_attn_bwd_dkdv(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                           const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                           const float* delta, lh_bf16* dkg, lh_bf16* dvg, void* stream);

/* The dQ half of lh_attn_bwd (Sec. 3.2 and 3.5, Eq. 9), given delta: one
 * CTA per 128 query rows walks the key rows up to its diagonal.  Inputs as
 * for lh_attn_bwd_dkdv; dqg out bf16 [B, H, S, d]. */
lh_status lh_attn_bwd_dq(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                         const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                         const float* delta, lh_bf16* dqg, void* stream);

/* ---- ring attention steps (context parallelism) ----
 * The pages' multi-GPU training note (single-B200 latency paragraph of the
 * experiments, with App. D.4 cited): the sequence is cut into contiguous
 * shards, pyramid pooling, scoring and top-k run shard-locally, and the
 * gathered sub-sequences go through ring attention.  Every entry of shard
 * r' < r ends before any entry of shard r, so over the shards'
 * sub-sequences concatenated in shard order the plain causal mask applies:
 * shard r's rows see all of every earlier shard's block and their own
 * block causally.  One step is one (query shard, K/V block) pair; `cfg` is
 * the config of one shard (N = its tokens), so every block has S rows.
 *  mode   LH_BLOCK_DIAG: the shard's own block (causal);
 *         LH_BLOCK_FULL: an earlier shard's block (every key visible).
 *  first  1: this step opens the sum (accumulators written, not read).
 *  last   1: this step closes it (the bf16 results are written instead of
 *         the accumulators).  first = last = 1 is the plain single-block
 *         call, and then the accumulators may be NULL.
 * Accumulators are fp32 and owned by the caller; steps that share them must
 * run in order (e.g. on one stream).  Sums run in step order, so results
 * are bitwise reproducible.  Invalid mode, flags or a missing pointer:
 * LH_ERR_INVALID_ARGUMENT before any launch. */
#define LH_BLOCK_DIAG 0
#define LH_BLOCK_FULL 1

/* Forward step: the partial softmax attention of qg [B,H,S,d] against the
 * block kg, vg [B,H,S,d] merges into o_acc (fp32 [B,H,S,d], normalised
 * output so far) and lse2_acc (fp32 [B,H,S], base-2 log-sum-exp so far) by
 * log-sum-exp.  On the last step og, og_lo (may be NULL) and lse (natural
 * log) are written as by lh_attn_fwd. */
lh_status lh_attn_fwd_block(const lh_config* cfg, int32_t mode, int32_t first, int32_t last,
                            const lh_bf16* qg, const lh_bf16* kg, const lh_bf16* vg,
                            float* o_acc, float* lse2_acc, lh_bf16* og, lh_bf16* og_lo,
                            float* lse, void* stream);

/* Backward step, the block's side: this query shard's share of dK, dV of
 * the block (the query rows' final lse and delta = D), added to dk_acc,
 * dv_acc (fp32 [B,H,S,d]); the closing step writes dkg, dvg (bf16). */
lh_status lh_attn_bwd_dkdv_block(const lh_config* cfg, int32_t mode, int32_t first,
                                 int32_t last, const lh_bf16* qg, const lh_bf16* kg,
                                 const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                                 const float* delta, float* dk_acc, float* dv_acc, lh_bf16* dkg,
                                 lh_bf16* dvg, void* stream);

/* Backward step, the query side: the block's share of dQ of the query
 * shard, added to dq_acc (fp32 [B,H,S,d]); the closing step writes dqg. */
lh_status lh_attn_bwd_dq_block(const lh_config* cfg, int32_t mode, int32_t first, int32_t last,
                               const lh_bf16* qg, const lh_bf16* kg, const lh_bf16* vg,
                               const lh_bf16* dog, const float* lse, const float* delta,
                               float* dq_acc, lh_bf16* dqg, void* stream);

/* (iv) scatter-back, Sec. 3.6: o[t] = sum over levels l of og[slot] for the
 * selected entry (l, i) with (i+1) p^l - 1 <= t <= (i+2) p^l - 2, i.e.
 * i = floor((t+1)/p^l) - 1; levels are summed in ascending order in fp32 and
 * rounded once; a position no entry reaches gets 0.
 *  o out bf16 [B, N, H, d].  scatter_mode 1 needs ws (fwd_ws bytes).      */
lh_status lh_scatter(const lh_config* cfg, const lh_bf16* og, const int32_t* slot_map,
                     lh_bf16* o, void* ws, size_t ws_bytes, void* stream);

/* Adjoint of lh_scatter (Sec. 3.6 scatter, differentiated as Sec. 3.2
 * prescribes: the gradient reaches the gathered outputs through stage (iv)):
 * dog[m] = sum of dO[t] over the shifted range of
 * slot m (clipped to t < N), rounded once to bf16, and delta[m] =
 * rowsum(dog[m] * (og[m] + og_lo[m])) (the D of the attention backward;
 * og_lo may be NULL), both per (b, h).
 *  dout in bf16 [B, N, H, d]; dog out bf16 [B, H, S, d]; delta out fp32
 *  [B, H, S]                                                               */
lh_status lh_scatter_bwd(const lh_config* cfg, const lh_bf16* dout, const lh_bf16* og,
                         const lh_bf16* og_lo, const int32_t* sel_idx, lh_bf16* dog,
                         float* delta, void* stream);

/* Adjoint of the gather and the mean pooling (Sec. 3.3 pyramid and Sec. 3.5
 * gather, differentiated as Sec. 3.2 prescribes: gradients reach Q, K, V
 * through the gather; the selection carries none): dq[t] = sum over levels l of
 * p^-l dqg[slot(l, floor(t/p^l))] for selected entries (unshifted window),
 * likewise dk and dv.
 *  dq, dk, dv out bf16 [B, N, H, d]                                        */
lh_status lh_gather_bwd(const lh_config* cfg, const lh_bf16* dqg, const lh_bf16* dkg,
                        const lh_bf16* dvg, const int32_t* slot_map, lh_bf16* dq,
                        lh_bf16* dk, lh_bf16* dv, void* stream);

/* Whole layer forward, the four stages of Sec. 3.2 in order (Sec. 3.3-3.6):
 * lh_pyramid, lh_score_topk, lh_gather, lh_attn_fwd, lh_scatter.  o out bf16 [B, N, H, d].  `saved` (>= saved bytes) receives
 * what lh_backward needs; `ws` (>= fwd_ws bytes) is scratch.               */
lh_status lh_forward(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                     const lh_bf16* v, lh_bf16* o, void* saved, size_t saved_bytes,
                     void* ws, size_t ws_bytes, void* stream);

/* Whole layer backward from the saved buffer of the matching lh_forward
 * (Sec. 3.2: through stages (iv), (iii) and the gather, indices frozen):
 * lh_scatter_bwd (which also gives D), lh_attn_bwd_dkdv, lh_attn_bwd_dq,
 * lh_gather_bwd.  dq, dk, dv out bf16
 * [B, N, H, d]; `ws` (>= bwd_ws bytes) is scratch.                          */
lh_status lh_backward(const lh_config* cfg, const void* saved, size_t saved_bytes,
                      const lh_bf16* dout, lh_bf16* dq, lh_bf16* dk, lh_bf16* dv,
                      void* ws, size_t ws_bytes, void* stream);

/* ---- the layer in halves around its attention ----
 * lh_forward = lh_forward_gather, lh_attn_fwd on the saved qg/kg/vg (into
 * the saved og/og_lo/lse), lh_forward_scatter; lh_backward =
 * lh_backward_scatter, the attention backward from the bwd_ws dog/delta
 * into the bwd_ws dqg/dkg/dvg (lh_bwd_ws_offsets), lh_backward_gather.
 * Same buffers, sizes and errors as lh_forward / lh_backward.  Splitting the
 * layer there lets another schedule of the attention run in the middle:
 * ring attention over the shards of a sequence (lh_attn_*_block). */

/* Stages (i)-(iii) up to the gather (Sec. 3.3-3.5): pyramid, scores,
 * selection and order, gather into the saved qg, kg, vg; sel_idx and
 * slot_map into the saved buffer. */
lh_status lh_forward_gather(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                            const lh_bf16* v, void* saved, size_t saved_bytes, void* ws,
                            size_t ws_bytes, void* stream);

/* Stage (iv) (Sec. 3.6): scatter of the saved og into o [B, N, H, d]. */
lh_status lh_forward_scatter(const lh_config* cfg, const void* saved, size_t saved_bytes,
                             lh_bf16* o, void* ws, size_t ws_bytes, void* stream);

/* Adjoint of stage (iv) (Sec. 3.2, 3.6): dog and delta = D into bwd_ws. */
lh_status lh_backward_scatter(const lh_config* cfg, const void* saved, size_t saved_bytes,
                              const lh_bf16* dout, void* ws, size_t ws_bytes, void* stream);

/* Adjoint of the gather and pooling (Sec. 3.2, 3.3, 3.5): the bwd_ws dqg,
 * dkg, dvg into dq, dk, dv [B, N, H, d]. */
lh_status lh_backward_gather(const lh_config* cfg, const void* saved, size_t saved_bytes,
                             const void* ws, size_t ws_bytes, lh_bf16* dq, lh_bf16* dk,
                             lh_bf16* dv, void* stream);

/* ---- plain GEMMs for the projections around the layer (Sec. 3.1: per-head
 * Q, K, V come from the layer's own W_Q, W_K, W_V; an output projection
 * follows).  Not part of the pages' custom kernels: the pages leave these to
 * the training framework; they are here so a whole layer can be timed.
 *
 *   C[M, N] = sum_{i < npairs} A_i[M, K_i] B_i[N, K_i]^T
 *
 * bf16 in, fp32 accumulate, bf16 out (C row-major, leading dimension ldc).
 * a_mn = 0: A_i[m, k] at a + m * lda + k (K contiguous); a_mn = 1: at
 * a + k * lda + m (M contiguous).  Likewise b_mn for B_i with n.  npairs in
 * 1..3; M, N, K_i >= 1; N, K_i, lda, ldb, ldc multiples of 8; pointers
 * 16-byte aligned; lda >= K_i (a_mn = 0) or M (a_mn = 1), ldb likewise.
 * splits > 1 divides the summed K range over CTAs (for long K and few
 * output tiles) and needs `ws` of lh_gemm_ws_bytes bytes for fp32 partials,
 * summed afterwards in split order, so the result is deterministic.
 * Invalid arguments return LH_ERR_INVALID_ARGUMENT before any launch.  The
 * caller guarantees that every operand holds its full extent (M or N rows
 * by K_i, at its leading dimension): the library cannot see allocations. */
typedef struct {
  const lh_bf16* a;
  const lh_bf16* b;
  int64_t k, lda, ldb;
} lh_gemm_operand;

size_t lh_gemm_ws_bytes(int64_t M, int64_t N, int32_t splits);

lh_status lh_gemm(int64_t M, int64_t N, int32_t npairs, const lh_gemm_operand* ops, int32_t a_mn,
                  int32_t b_mn, lh_bf16* c, int64_t ldc, int32_t splits, void* ws,
                  size_t ws_bytes, void* stream);

/* Failure-detection check (no fault is involved): enqueues one warp that
 * waits on an mbarrier nothing arrives at, through the same bounded wait the
 * attention and GEMM kernels use.  After about 4e9 SM clock cycles (about
 * 2 s) the wait gives up, records LH_ERR_DEVICE_TIMEOUT with detail
 * LH_WAIT_TIMEOUT_CHECK_DETAIL in the device status word, and the kernel
 * returns; the CUDA context stays usable.  Returns LH_OK once the launch is
 * enqueued (LH_ERR_CUDA if it fails); read the outcome with
 * lh_get_device_status. */
#define LH_WAIT_TIMEOUT_CHECK_DETAIL 900
lh_status lh_check_wait_timeout(void* stream);

/* Synchronises `stream`, returns the first device-side error recorded since
 * the last call (LH_OK if none) and clears it.  *detail (may be NULL)
 * receives a kernel-specific code locating the failure. */
lh_status lh_get_device_status(void* stream, int32_t* detail);

/* Human-readable name of a status code (static string). */
const char* lh_status_string(lh_status s);

/* Number of kernel launches one lh_forward / lh_backward call makes. */
int32_t lh_forward_launches(const lh_config* cfg);
int32_t lh_backward_launches(const lh_config* cfg);

#ifdef __cplusplus
}
#endif
#endif /* LIGHTHOUSE_H */
