/*
 * moc.h - C ABI of the Mixture of Contexts (MoC) sparse-attention forward pass
 * on NVIDIA B200 (sm_100a).
 *
 * The method (pages: "Mixture of Contexts for Long Video Generation | Summary",
 * §3.1-§3.3; the jxzklqfsx.com MoC write-up, sections "內容對齊的塊劃分",
 * "固定的跨模態選擇", "固定的鏡頭內選擇", "稀疏 MoC 中的因果性", "計算效率"):
 * the flattened text+video token stream is cut into content-aligned chunks
 * (caption segments and video frames or sub-frames). Keys are mean-pooled per
 * chunk. Every video query scores its candidate chunks by the dot product with
 * the pooled keys and keeps the top-k; candidates are the video chunks that are
 * not mandatory for it, restricted to strictly earlier chunks under the causal
 * routing mask. Mandatory anchors (every caption token plus the query's own
 * shot, local frame window or own chunk) are always attended. Exact softmax
 * attention then runs over the union of anchors and selected chunks. Caption
 * queries attend densely to every token of the sample.
 *
 * Conventions shared by every call:
 *  - Tensors are head-major, contiguous: Q, K, V and O are bf16 [B][H][L][d];
 *    d is 64 or 128. Device pointers must be 16-byte aligned.
 *  - The caller owns every device buffer (inputs, outputs, workspace). The
 *    library allocates device memory only inside moc_build_layout (its tables,
 *    freed by moc_layout_destroy); no hot-path call allocates.
 *  - Compute calls are asynchronous on the given stream and return after
 *    enqueueing (except moc_forward_host, which takes host buffers and returns
 *    once its host outputs are complete). Argument errors are returned before
 *    anything is enqueued; a launch failure returns MOC_ERR_CUDA. No call
 *    throws across the ABI.
 *  - Limits: 1 <= C <= 16384 chunks, L < 2^26, B*H <= 65535, B*H*L*max(k,1) < 2^31,
 *    0 <= k <= 31, every chunk non-empty.
 */
#ifndef MOC_H
#define MOC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (the same object as cudaStream_t / CUstream). */
struct CUstream_st;
typedef struct CUstream_st* moc_stream_t;

typedef enum {
    MOC_OK = 0,
    MOC_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, bad size, bad k or d */
    MOC_ERR_LAYOUT = 2,              /* inconsistent segment description */
    MOC_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moc_attention_workspace_bytes(...) */
    MOC_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
    MOC_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up */
    MOC_ERR_UNSUPPORTED = 6,         /* valid request outside what this build handles */
    MOC_ERR_DEVICE_CHECK = 7         /* a device-side consistency check failed */
} moc_status;

/* Segment kinds and anchor modes of moc_layout_desc. */
enum { MOC_CAPTION = 0, MOC_VIDEO = 1 };
enum {
    MOC_ANCHOR_SHOT = 0,  /* every video chunk of the query's shot (multi-shot scenes) */
    MOC_ANCHOR_LOCAL = 1, /* video chunks of the query's shot within +-local_radius frames */
    MOC_ANCHOR_CHUNK = 2  /* the query's own chunk only */
};

/* Host-memory description of one scene's token stream, in stream order
 * (content-aligned chunking: "內容對齊的塊劃分" of the jxzklqfsx.com write-up;
 * the boundary tables of its "計算效率" section). Each segment is one chunk.
 *   seg_len[i]   token count (> 0) of segment i;
 *   seg_kind[i]  MOC_CAPTION or MOC_VIDEO;
 *   seg_shot[i]  shot id of a video segment (informational for captions);
 *   seg_frame[i] frame index of a video segment within its shot; sub-chunks
 *                of one frame repeat it.
 * Video segments of one shot must be contiguous in the stream with frame
 * indices non-decreasing. The arrays are read during moc_build_layout only. */
typedef struct {
    int32_t n_segments;
    const int32_t* seg_len;
    const int32_t* seg_kind;
    const int32_t* seg_shot;
    const int32_t* seg_frame;
    int32_t anchor_mode;   /* MOC_ANCHOR_* */
    int32_t local_radius;  /* frames, for MOC_ANCHOR_LOCAL (>= 0) */
} moc_layout_desc;

typedef struct moc_layout moc_layout; /* opaque */

/* Text of a status code (static storage). */
const char* moc_status_string(moc_status s);

/* Build the chunk tables of a scene: chunk offsets, chunk -> shot/frame/kind,
 * query groups (runs of chunks sharing one anchor set), per-group anchor key
 * ranges and candidate chunk lists ("計算效率": boundary tagging and prefix-sum
 * tables; the pre-routing mask that keeps mandatory chunks out of top-k).
 * device >= 0: the tables are also copied to that CUDA device (allocated here,
 * freed by moc_layout_destroy); device == -1: host-only layout, usable with the
 * query calls below but rejected by every compute call.
 * On success *out owns the layout. On error *out is set to NULL. */
moc_status moc_build_layout(const moc_layout_desc* desc, int device, moc_layout** out);

/* Free a layout and its device tables (NULL is a no-op). Not stream-ordered:
 * call it only when no launched work still uses the layout. */
void moc_layout_destroy(moc_layout* layout);

/* Sizes of a built layout: tokens L, chunks C, distinct shots (any may be NULL). */
moc_status moc_layout_info(const moc_layout* layout, int64_t* L, int32_t* C, int32_t* n_shots);

/* Host-side copy of one layout table, for inspection and tests.
 * which: 0 chunk_off[C+1], 1 group token range (q0,q1)[G][2],
 *        2 group anchor key ranges as (start,end) pairs in group order,
 *        3 anchor range offsets per group [G+1], 4 candidate chunk ids in
 *        group order, 5 candidate offsets per group [G+1],
 *        6 causal candidate count per group [G], 7 segment (shot, numbered in
 *        stream order) of every candidate in table 4, 8 segment of every
 *        group's queries [G] (-1: caption group), 9 offsets of every segment's
 *        video chunks in table 10 [S+1], 10 video chunk ids in stream order,
 *        11 / 12 prefix of the router's estimated tile costs for the full /
 *        causal candidate lists [router tiles + 1],
 *        backward key blocks (a video chunk, or a run of caption chunks the
 *        same groups attend): 13 token range (k0,k1)[NKB][2], 14 video chunk
 *        of the block or -1 [NKB], 15 offsets into table 16 [NKB+1], 16 query
 *        groups whose anchor ranges hold the block, 17 blocks by descending
 *        anchoring query rows [NKB], 18 prefix of 128-key tiles over table 17
 *        [NKB+1].
 * Writes min(count, cap) int32 values to out (may be NULL with cap 0) and
 * the full count to *count. */
moc_status moc_layout_table(const moc_layout* layout, int which, int32_t* out, int64_t cap,
                            int64_t* count);

/* (1) Segmented mean pool of keys ("計算效率": segment_reduce mean pooling;
 * Summary §3.1: the chunk descriptor is the mean of the chunk's keys):
 *   Kbar[b][h][c][e] = (1/n_c) * sum_{t in chunk c} K[b][h][t][e],
 * accumulated in fp32 from bf16. K: device bf16 [B][H][L][d]; Kbar: device
 * fp32 [B][H][C][d], 16-byte aligned. Deterministic. */
moc_status moc_pool_keys(const moc_layout* layout, int B, int H, int d, const void* K,
                         float* Kbar, moc_stream_t stream);

/* (2) Routing (Summary §3.1 top-k by dot product with the pooled key; §3.2
 * causal mask j < i before top-k; "計算效率": mandatory chunks excluded from
 * the candidates). For every video query t of chunk i, candidates are the
 * video chunks j that are not mandatory for it, and with causal != 0 only
 * those with j < i. Scores s_j = q_t . Kbar_j (unscaled, fp32 accumulation of
 * exact bf16 x (hi+lo bf16 split of Kbar) products). sel[b][h][t][0..k) gets
 * the chunk ids of the top-min(k, |candidates|) candidates ordered by
 * (score descending, chunk id ascending), padded with -1. Caption queries get
 * all -1 (they attend densely). Q: device bf16 [B][H][L][d]; Kbar from (1);
 * sel: device int32 [B][H][L][k]. k == 0 enqueues nothing. */
moc_status moc_route(const moc_layout* layout, int B, int H, int d, const void* Q,
                     const float* Kbar, int k, int causal, int32_t* sel, moc_stream_t stream);

/* (2'') Outer-loop context routing (Summary, appendix I): a coarse router
 * picks, per query block, the top-M context segments the inner router may
 * select from. Segments are the shots' video chunks, numbered 0..S-1 in stream
 * order (S <= 64); a query block is a query group of the layout (queries
 * sharing one anchor set; table 1 of moc_layout_table lists them, G of them).
 * Features are token means - the block's queries and the segment's keys -
 * formed from per-chunk means (Qbar from moc_pool_keys applied to Q, Kbar from
 * (1)) weighted by chunk length, in fp32; score = unscaled dot product.
 * Candidates are the other segments (with causal != 0 only earlier ones); top-M
 * by (score descending, segment ascending), all when fewer than M. seg_mask:
 * device uint64 [B][H][G], bit s set = segment s allowed; the block's own
 * segment is always set (mandatory context); caption blocks get 0. */
moc_status moc_outer_route(const moc_layout* layout, int B, int H, int d, const float* Qbar,
                           const float* Kbar, int M, int causal, uint64_t* seg_mask,
                           moc_stream_t stream);

/* (2) restricted by an outer-loop mask: as moc_route, with a query's
 * candidates limited to chunks of segments whose bit is set in its block's
 * seg_mask (from moc_outer_route). */
moc_status moc_route_masked(const moc_layout* layout, int B, int H, int d, const void* Q,
                            const float* Kbar, int k, int causal, const uint64_t* seg_mask,
                            int32_t* sel, moc_stream_t stream);

/* (2') Training-time routing perturbations (Summary, appendix training
 * details; [DL] slide 14): context drop-off and drop-in on a selection from
 * (2). Per (b, h, query) - caption queries get all -1 - with the random draws
 * given as data, rnd: device uint32 [B][H][L][2 + k + m_max]:
 *   drop-off: n_drop = floor((rnd[0] / 2^32) * p_max * k) (fp64 products, left
 *     to right; at most the number of selected chunks); the n_drop selected
 *     entries with the smallest (rnd[2 + j], j) are removed;
 *   drop-in: m = min(m_max, Poisson(lambda) inverted at rnd[1]) (the
 *     distribution function is accumulated in fp64 from exp(-lambda) and
 *     compared as floor(F * 2^32)); the a-th added chunk is entry
 *     floor(rnd[2 + k + a] * n_left / 2^32) of the query's routing candidates
 *     (same causal flag as (2)) that are neither in sel nor already added,
 *     in ascending chunk order.
 * sel: device int32 [B][H][L][k] from (2) (NULL when k == 0); sel_out: device
 * int32 [B][H][L][k + m_max]: survivors in their original order, then the
 * added chunks, -1 padded - a selection the attention calls take with
 * k + m_max in place of k. 0 <= p_max <= 1, lambda >= 0 finite, m_max >= 0,
 * 1 <= k + m_max <= 31. Deterministic. */
moc_status moc_route_perturb(const moc_layout* layout, int B, int H, int k, int causal,
                             const int32_t* sel, const uint32_t* rnd, float p_max, float lambda,
                             int m_max, int32_t* sel_out, moc_stream_t stream);

/* Bytes of device workspace moc_attention_fwd and the three stage calls need
 * for this problem (0 on invalid arguments). Holds the per-chunk query lists,
 * the scheduler's counters and the partial outputs (1+k fp32 rows of d plus
 * a log-sum-exp per query): the storage of the attention over Omega(q) split
 * into disjoint parts (Summary §3.1: Omega(q) is the union of the anchors and
 * the selected chunks), which replaces the packed variable-length buffers of
 * the jxzklqfsx.com write-up's "計算效率" section. */
size_t moc_attention_workspace_bytes(const moc_layout* layout, int B, int H, int d, int k);

/* (3) Query-list builder ("計算效率" of the jxzklqfsx.com write-up: the
 * selected (query, chunk) pairs are grouped so that each chunk's keys are
 * attended by all the queries that chose it, in place of its packing of
 * variable-length groups for one FlashAttention varlen call): invert sel into
 * per-(b, h, chunk) lists of (query, slot) entries by count -> exclusive
 * prefix sum -> ordered scatter; each list is sorted by query index. Fills the
 * workspace. An entry of sel that is >= C is ignored and recorded as
 * MOC_ERR_DEVICE_CHECK (detail 3) in the workspace's error word. */
moc_status moc_build_qlists(const moc_layout* layout, int B, int H, int k, const int32_t* sel,
                            void* ws, size_t ws_bytes, moc_stream_t stream);

/* (4) Chunk-major attention over the work items (Summary §3.1 attention over
 * Omega(q)): per 256 consecutive queries of a query group, attention over the
 * group's anchor key ranges (partial slot 0); per 256 entries of a chunk's
 * query list, attention of the gathered query rows over that chunk (slot 1 +
 * position in sel). Each partial is the normalised softmax output and its log-sum-exp of
 * the raw scaled scores. softmax_scale is normally 1/sqrt(d). Needs the
 * workspace filled by (3) for the same sel. */
moc_status moc_attend_partials(const moc_layout* layout, int B, int H, int d, const void* Q,
                               const void* K, const void* V, int k, float softmax_scale,
                               void* ws, size_t ws_bytes, moc_stream_t stream);

/* (4) and (5) in one kernel: the attention of (4) with the merge of (5) done in
 * place. Routed items run first and write their partials; each anchor item
 * then combines its own part (kept in TMEM, never written) with its rows'
 * routed partials by the log-sum-exp rule of (5), in the same fixed slot order,
 * and writes the bf16 output row and lse (nullable) itself - the anchor
 * partials are never stored or read back. An entry of sel outside [0, C) is
 * skipped. Needs the workspace filled by (3) for the same sel. It moves ~4 GB
 * less through HBM on the eight-shot scene than (4) + (5), but the partial
 * reads sit in the softmax warps' epilogue, and on one B200 it measured no
 * faster than (4) + (5); moc_attention_fwd uses (4) + (5). */
moc_status moc_attend_merged(const moc_layout* layout, int B, int H, int d, const void* Q,
                             const void* K, const void* V, const int32_t* sel, int k,
                             float softmax_scale, void* O, float* lse, void* ws, size_t ws_bytes,
                             moc_stream_t stream);

/* (5) Log-sum-exp merge of every query's partials (Summary §3.1: softmax
 * attention over Omega(q); Omega(q) is a disjoint union of the anchor keys and
 * the selected chunks, and softmax over a disjoint union equals the
 * log-sum-exp-weighted combination of the softmax over each part): with
 * M = max lse_j over the valid slots, w_j = exp(lse_j - M),
 * O = sum_j w_j O_j / sum_j w_j rounded to bf16 (nearest even),
 * lse = M + log sum_j w_j (fp32, nullable). Slots are visited in a fixed order,
 * so the result is deterministic. */
moc_status moc_merge(const moc_layout* layout, int B, int H, int d, int k, const int32_t* sel,
                     void* O, float* lse, void* ws, size_t ws_bytes, moc_stream_t stream);

/* Full attention stage (Summary §3.1: o = Softmax(q K_Omega^T / sqrt(d))
 * V_Omega over Omega(q) = anchors + the chunks in sel): (3), (4) and (5) in
 * order on one stream (measured faster than (3) + moc_attend_merged). sel: device int32 [B][H][L][k] from (2) or (2'),
 * -1 padded (NULL when k == 0); O: device bf16 [B][H][L][d]; lse: device fp32
 * [B][H][L] (nullable); ws: the caller's workspace, 256-byte aligned, of at
 * least moc_attention_workspace_bytes() bytes. */
moc_status moc_attention_fwd(const moc_layout* layout, int B, int H, int d, const void* Q,
                             const void* K, const void* V, const int32_t* sel, int k,
                             float softmax_scale, void* O, float* lse, void* ws,
                             size_t ws_bytes, moc_stream_t stream);

/* Bytes of device workspace moc_attention_bwd needs (0 on invalid arguments):
 * the query lists of (3), D = dO . o per row and the dQ partial rows (1+k fp32
 * rows of d per query). */
size_t moc_attention_bwd_workspace_bytes(const moc_layout* layout, int B, int H, int d, int k);

/* Backward pass of the attention stage: dQ, dK, dV for an upstream gradient dO
 * of O ("Mixture of Contexts for Long Video Generation | Summary", appendix on
 * training: the model is trained through a custom autograd function of the
 * attention over the selected keys and values; the top-k choice is discrete
 * and is not differentiated). The selection sel is a constant, so no gradient
 * reaches the pooled keys, and the loss depends on O only (no gradient on lse).
 * With p_tu = exp(scale q_t.k_u - lse_t) over u in Omega(t) and
 * D_t = dO_t . O_t:
 *   ds_tu = p_tu (dO_t . v_u - D_t),   dQ_t = scale sum_u ds_tu k_u,
 *   dK_u = scale sum_t ds_tu q_t,      dV_u = sum_t p_tu dO_t.
 * Q, K, V, O, dO: device bf16 [B][H][L][d] (O from the forward pass); lse:
 * device fp32 [B][H][L], the forward pass's log-sum-exp; sel: as for
 * moc_attention_fwd (the selection the forward pass used); dQ, dK, dV: device
 * bf16 [B][H][L][d] outputs, accumulated in fp32 and rounded to nearest even.
 * ws: 256-byte aligned, at least moc_attention_bwd_workspace_bytes() bytes.
 * Deterministic: dQ is summed per row from per-part partials in fixed order;
 * each key's dK and dV are accumulated by one CTA over a fixed query order.
 * Asynchronous on the stream; device errors as for moc_attention_fwd. */
moc_status moc_attention_bwd(const moc_layout* layout, int B, int H, int d, const void* Q,
                             const void* K, const void* V, const void* O, const float* lse,
                             const void* dO, const int32_t* sel, int k, float softmax_scale,
                             void* dQ, void* dK, void* dV, void* ws, size_t ws_bytes,
                             moc_stream_t stream);

/* moc_attention_fwd without a caller workspace, for callers that cannot
 * allocate device memory (a plugin given only its input and output buffers, a
 * real-time loop that must stay off the driver's allocation path, a library
 * inside a host application that budgets every device byte up front). The pages
 * describe no counterpart: this is a deployment variant of (3)-(5) above.
 * Scratch: a static 64 MiB device array inside the library, held on every GPU
 * that loads it until the process exits; nothing is allocated per call.
 * Returns MOC_ERR_WORKSPACE_TOO_SMALL when moc_attention_workspace_bytes()
 * for the problem exceeds 64 MiB. The first call on a device looks up the
 * array's device address (make that first call before any stream capture).
 * All calls share the array: calls that overlap on the GPU race. Arguments
 * otherwise as moc_attention_fwd. */
moc_status moc_attention_fwd_static(const moc_layout* layout, int B, int H, int d, const void* Q,
                                    const void* K, const void* V, const int32_t* sel, int k,
                                    float softmax_scale, void* O, float* lse, moc_stream_t stream);

/* Read and clear the device error word of moc_attention_fwd_static on the
 * current device (its scratch, and so its error word, is not visible to the
 * caller). The pages describe no counterpart. Synchronises the stream; returns
 * what moc_check_device_error returns for a caller workspace. Every
 * moc_attention_fwd_static call clears the word when it starts, so read it
 * after the call whose errors matter and before the next one. */
moc_status moc_check_device_error_static(int32_t* detail, moc_stream_t stream);

/* E4M3 variant of the attention stage (the pages' future-work lists: "Mixture
 * of Contexts for Long Video Generation | Summary", limitations, and the
 * jxzklqfsx.com write-up, "局限性與未來工作", name quantisation).
 *
 * moc_quantize_e4m3: per (b, h) slice of X (device bf16 [BH][L][d]) a scale
 * that is a power of two, scale = 2^ceil(log2(amax / 448)) (1 for an all-zero
 * slice), written to scale[BH] (device fp32), and X8 = E4M3(X / scale)
 * (device bytes [BH][L][d], OCP E4M3 as in NVIDIA's e4m3 type, round to
 * nearest even; X / scale is exact and never exceeds 448). X8 * scale is then
 * exactly representable in bf16. */
moc_status moc_quantize_e4m3(int BH, int64_t L, int d, const void* X, void* X8, float* scale,
                             moc_stream_t stream);

/* (4) on E4M3 inputs from moc_quantize_e4m3 (d = 128 only; other d return
 * MOC_ERR_UNSUPPORTED): S = Q8 K8^T and O += P V8 on kind::f8f6f4 tensor cores,
 * scores scaled by q_scale[bh] k_scale[bh] softmax_scale, P = exp of the scaled
 * scores minus the running max, written to TMEM as E4M3 of P * 2^6 (the running
 * max is raised once it grows by more than 2^2, so P * 2^6 <= 256 < 448), the
 * row sum taken in fp32 on the unrounded P, O scaled by v_scale[bh] at the end.
 * Writes the same partial rows and log-sum-exps as (4), for (5). Needs the
 * workspace filled by (3). */
moc_status moc_attend_partials_e4m3(const moc_layout* layout, int B, int H, int d, const void* Q8,
                                    const void* K8, const void* V8, const float* q_scale,
                                    const float* k_scale, const float* v_scale, int k,
                                    float softmax_scale, void* ws, size_t ws_bytes,
                                    moc_stream_t stream);

/* (3), moc_attend_partials_e4m3 and (5) in order on one stream: the attention
 * stage on E4M3 inputs, bf16 O and fp32 lse out as moc_attention_fwd. */
moc_status moc_attention_fwd_e4m3(const moc_layout* layout, int B, int H, int d, const void* Q8,
                                  const void* K8, const void* V8, const float* q_scale,
                                  const float* k_scale, const float* v_scale, const int32_t* sel,
                                  int k, float softmax_scale, void* O, float* lse, void* ws,
                                  size_t ws_bytes, moc_stream_t stream);

/* Whole forward pass on HOST buffers: (1) pooling, (2) routing (when k > 0)
 * and (3)-(5) for every (b, h) slice, the end-to-end call for inputs that live
 * in host memory. Q, K, V: host bf16 [B][H][L][d] (page-locked memory lets the
 * copies run concurrently with the kernels); O: host bf16 [B][H][L][d]; lse
 * (nullable): host fp32 [B][H][L]; sel (nullable): host int32 [B][H][L][k].
 * The slices are processed in chunks of heads_per_chunk consecutive (b, h)
 * slices (<= 0: B*H/12 rounded up; the first and the last chunk are half
 * that): chunk c+1's inputs are copied in while chunk c
 * is computed on `stream` and chunk c-1's outputs are copied out, each of the
 * three on its own stream. Every stage is independent per (b, h) (Summary
 * §3.1; "計算效率": head-independent operations), so results are bitwise those
 * of the device calls on the whole tensors. dev: device scratch of
 * moc_forward_host_device_bytes() bytes, 256-byte aligned (two input and two
 * output stages, pooled keys and the attention workspace of one chunk);
 * nothing is allocated on the device. Work already queued on `stream` runs
 * first; the call synchronises and returns when the host outputs are
 * complete, reporting a device error word as moc_check_device_error and
 * moc_layout_device_error do. */
moc_status moc_forward_host(const moc_layout* layout, int B, int H, int d, int k, int causal,
                            float softmax_scale, const void* Q, const void* K, const void* V,
                            void* O, float* lse, int32_t* sel, void* dev, size_t dev_bytes,
                            int heads_per_chunk, moc_stream_t stream);

/* Bytes of device scratch moc_forward_host needs (0 on invalid arguments). */
size_t moc_forward_host_device_bytes(const moc_layout* layout, int B, int H, int d, int k,
                                     int heads_per_chunk);

/* Read and clear the device error word the kernels set when a bounded wait
 * gives up or a consistency check fails. Synchronises the stream. Returns
 * MOC_OK, MOC_ERR_DEVICE_TIMEOUT or MOC_ERR_DEVICE_CHECK; *detail (nullable)
 * receives a kernel-specific code. */
moc_status moc_check_device_error(void* ws, size_t ws_bytes, int32_t* detail,
                                  moc_stream_t stream);

/* Diagnostic (the pages have no counterpart): run the bounded mbarrier wait
 * the kernels use on a barrier nothing arrives at. After its time limit (2 s)
 * it records ERR_TIMEOUT in dev_word[0] and a site code in dev_word[1] (device
 * int32[2], e.g. the first bytes of an attention workspace, so that
 * moc_check_device_error then reports MOC_ERR_DEVICE_TIMEOUT) and returns;
 * nothing hangs or faults. Asynchronous on the stream. */
moc_status moc_selftest_bounded_wait(int32_t* dev_word, moc_stream_t stream);

/* Diagnostic (the pages have no counterpart): the work schedule of the
 * attention kernel (4) for the calls that follow in this process - n_ctas
 * persistent CTAs (0: one per SM; more than the SM count means one per SM)
 * taking the work items in their natural order (item_order 0: anchor items,
 * longest first, then routed items) or reversed (1). Every item is computed
 * by one CTA from its inputs alone, so results do not depend on the schedule;
 * tests use this to show it. Not thread-safe against concurrent launches. */
moc_status moc_set_attend_schedule(int n_ctas, int item_order);

/* Diagnostic (the pages have no counterpart): which kernel computes the
 * attention stage (4) in the calls that follow in this process - 0 the default,
 * 1 the single-CTA kernel, 2 the CTA-pair kernel (clusters of two SMs sharing
 * every MMA, tcgen05 cta_group::2; bf16 with d = 128 only: other shapes then
 * return MOC_ERR_INVALID_ARG). Both compute the same partials (Summary §3.1);
 * their summation orders differ only inside the MMAs. Returns
 * MOC_ERR_INVALID_ARG for another variant. Not thread-safe against concurrent
 * launches. */
moc_status moc_set_attend_kernel(int variant);

/* Read and clear the device error word kept with a layout, where kernels that
 * run without a workspace (the router, (2)) record a bounded wait that gave up.
 * Synchronises the stream. Returns MOC_OK, MOC_ERR_DEVICE_TIMEOUT or
 * MOC_ERR_DEVICE_CHECK; *detail (nullable) receives a kernel-specific code. */
moc_status moc_layout_device_error(const moc_layout* layout, int32_t* detail, moc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOC_H */
