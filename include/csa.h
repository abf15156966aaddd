/*
 * csa.h -- C ABI of the B200 library for DeepSeek-V4's hybrid attention:
 * Compressed Sparse Attention (CSA) and Heavily Compressed Attention (HCA).
 *
 * Sources (web pages; they print no formulas, so the readings below are the
 * ones this library fixes):
 *   [RN]  "DeepSeek-V4 發佈說明：為 AI Agents 提供高效的 1M-Token 上下文",
 *         sections 壓縮稀疏注意力 (CSA), 重度壓縮注意力 (HCA), 架構實現.
 *   [WK]  "DeepSeek V4: Towards Highly Efficient Million-Token Context
 *         Intelligence" (wiki summary), sections 架构创新 and 基础设施.
 *   [AR]  "DeepSeek-V4预览版：原生支持100万token上下文的全栈重构大模型",
 *         section 二.1 混合注意力.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, dense row-major with the shapes stated.  Nothing is allocated:
 *     scratch memory is the caller's `workspace`, sized by
 *     csa_workspace_size().  Calls enqueue work on `stream` and return without
 *     synchronising; a call is not complete until the stream is.
 *   - Return value: CSA_OK (0) or a negative csa_status.  Argument errors are
 *     detected on the host before anything is launched and leave all buffers
 *     untouched.  CSA_ERR_CUDA reports a failed launch.
 *   - Kernels that meet bad data (an out-of-range selected index, a value the
 *     tensor-core path cannot represent) record it in a device status word and
 *     skip the offending item instead of faulting; read it with
 *     csa_device_status().
 *   - Positions are absolute token indices t >= 0.  Pooled block j covers
 *     tokens [m*j, m*j+m).  Block j is visible to query t iff m*j+m-1 < t-W,
 *     so n_elig(t) = max(0, floor((t-W)/m)).  The window of query t is the raw
 *     tokens i with t-W < i <= t, its own token included.
 *   - Formats (csa_format): F32 = float; BF16 = uint16 bfloat16 bits;
 *     FP8_S64 = uint8 OCP E4M3 codes [rows][d] plus float scales
 *     [rows][d/64], value = e4m3 * scale; MXFP4 = packed OCP E2M1 (element 2i
 *     in the low nibble of byte i) [rows][d/2] plus uint8 E8M0 scales
 *     [rows][d/32], value = e2m1 * 2^(e8m0-127).
 */
#ifndef CSA13_CSA_H
#define CSA13_CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum csa_format {
    CSA_F32 = 0,
    CSA_BF16 = 1,
    CSA_FP8_S64 = 2,
    CSA_MXFP4 = 3
} csa_format;

typedef enum csa_status {
    CSA_OK = 0,
    CSA_ERR_ARG = -1,         /* null pointer, non-positive size, inconsistent parameters */
    CSA_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
    CSA_ERR_UNSUPPORTED = -3, /* a shape / format combination this library does not implement */
    CSA_ERR_WORKSPACE = -4,   /* workspace smaller than csa_workspace_size() */
    CSA_ERR_CUDA = -5         /* a kernel launch failed (the CUDA error is not cleared) */
} csa_status;

/* Bits of the device status word (csa_device_status). */
#define CSA_DEV_BAD_INDEX 0x1u   /* a selected id >= the entries available; item skipped */
#define CSA_DEV_RANGE 0x2u       /* reserved: no kernel raises it (every stored value is representable) */
#define CSA_DEV_TIMEOUT 0x4u     /* a kernel's bounded wait gave up; its output is invalid */

/* Per-layer parameters.  Dimensions must be multiples of 64 (head_dim) and
 * of 32 (idx_dim).  act_fmt is the format of q, raw tokens x, gate logits z
 * and the output (F32 or BF16); kv_fmt of pooled entries (F32, BF16 or
 * FP8_S64); idx_fmt of indexer queries and keys (F32, BF16 or MXFP4). */
typedef struct csa_params {
    int32_t m;         /* tokens per pooled entry: 4 for CSA, 128 for HCA ([RN], [AR]) */
    int32_t window;    /* W, raw tokens in the sliding-window branch ([WK] 架构创新) */
    int32_t top_k;     /* k, pooled blocks kept per query (CSA only) ([AR] 512-1024) */
    int32_t n_heads;   /* H query heads sharing one KV head (MQA, [WK]) */
    int32_t head_dim;  /* d, width of q, raw tokens and pooled entries */
    int32_t idx_heads; /* HI, lightning-indexer heads ([RN] multi-head dot products) */
    int32_t idx_dim;   /* dI, width of indexer queries and keys */
    float scale;       /* softmax scale applied to q.k (not to the sink logit) */
    int32_t act_fmt;
    int32_t kv_fmt;
    int32_t idx_fmt;
    uint32_t flags;    /* CSA_FLAG_* bits; 0 for the default behaviour */
} csa_params;

/* Flags of csa_params.
 *
 * CSA_FLAG_BATCH_INVARIANT -- batch-invariant, deterministic results ([WK]
 *   基础设施: a batch-invariant, deterministic kernel library gives bitwise
 *   reproducible inference).  Every output row is computed with the same
 *   arithmetic in the same order whatever else is in the call: how a row's
 *   attention items are split over CTAs, and the order in which the partial
 *   results are combined, depend only on that row's own item count (about
 *   three 64-item tiles per split, at most 8 splits), never on the number of
 *   rows.  The indexer scores and the top-k selection are batch-invariant in
 *   both modes (each score is one fixed-order sum; the selection is exact).
 *   Without the flag the split count also depends on the number of rows, to
 *   fill the GPU, so a row's output may differ in its last bits between
 *   batch sizes (always within the matching tolerance).  Results are
 *   deterministic run to run in both modes. */
#define CSA_FLAG_BATCH_INVARIANT 0x1u

/* CSA_FLAG_QI_BF16 -- the write path of the indexer queries ([WK] 基础设施:
 *   MXFP4 on the indexer QK path; [RN] CSA: the indexer runs in FP4).  With
 *   p->idx_fmt == CSA_MXFP4, qI is given as bf16 [..][HI][dI] and qI_scales
 *   is not read: the indexer kernel quantises each query block to MXFP4 as it
 *   loads it, with the rule of csa_quantize (block exponent floor(log2(max
 *   |v|)) - 2, E2M1 codes rounded to nearest even), so the scores are those
 *   of csa_quantize followed by the MXFP4 indexer, without the separate pass
 *   or the stored quantised query.  Applies to indexer_score, csa_decode,
 *   csa_decode_noalloc and csa_prefill; CSA_ERR_ARG with another idx_fmt,
 *   CSA_ERR_UNSUPPORTED where the tensor-core indexer does not apply (HI !=
 *   64, dI != 128, max_blocks not a multiple of 4, fewer than 128 keys). */
#define CSA_FLAG_QI_BF16 0x2u

/* CSA_FLAG_INDEXER_FP8 -- the lossless FP4 -> FP8 path ([WK] 基础设施: FP4 ->
 *   FP8 dequantisation is lossless, so FP8 machinery is reused).  With
 *   p->idx_fmt == CSA_MXFP4, every stored E2M1 code of the keys and queries
 *   is expanded to the E4M3 byte of the same value (exact: E4M3 holds every
 *   E2M1 value) and the product runs as the MXFP8 block-scaled tensor-core
 *   MMA with the same E8M0 block scales.  Every product is the same exact
 *   value as on the MXFP4 path; the scores may differ from it only in the
 *   order of the fp32 additions.  Same scope and errors as CSA_FLAG_QI_BF16,
 *   with which it combines. */
#define CSA_FLAG_INDEXER_FP8 0x4u

/* ------------------------------------------------------------------------
 * csa_compress -- softmax-gated pooling with a learned positional bias
 * ([RN] CSA: KV entries are pooled 4x along the sequence by a softmax gate
 * with a learned positional bias; [RN] HCA: the same at 128x).
 *   out[j][c] = sum_{r<m} softmax_r(z[m*j+r][c] + bias[r][c]) * x[m*j+r][c]
 * computed in fp32 and stored in out_fmt (F32, BF16, FP8_S64 or MXFP4; the
 * FP8 scale is amax/448 per 64 channels, the MXFP4 exponent floor(log2
 * amax)-2 per 32, both rounding to nearest even).
 *   x, z:      [n_tokens][d] in p->act_fmt; n_tokens a multiple of p->m
 *   bias:      float [p->m][d]
 *   out:       [n_tokens/m][d] in out_fmt; out_scales as the format needs
 *              (NULL for F32 / BF16).  out_scales needs only 4-byte alignment
 *              (FP8_S64) or none (MXFP4), so that one pooled row can be
 *              written at any row index of a cache
 *   d:         channels (a multiple of 64); p->head_dim is not used, so the
 *              same call pools indexer keys (d = idx_dim)
 * ------------------------------------------------------------------------ */
int csa_compress(const csa_params* p, int32_t d, const void* x, const void* z,
                 const float* bias, int64_t n_tokens, int32_t out_fmt, void* out,
                 void* out_scales, csa_stream_t stream);

/* csa_quantize -- store fp32 rows as FP8_S64, MXFP4 or BF16 with the same
 * rounding rules as csa_compress (the write path of [RN] 架構實現: FP8 KV
 * entries, FP4 indexer).  src float [rows][d]; out / out_scales as above. */
int csa_quantize(int32_t fmt, const float* src, int64_t rows, int32_t d, void* out,
                 void* out_scales, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * indexer_score -- lightning-indexer scores ([RN] CSA: ReLU-scored
 * multi-head dot products in FP4; [WK] 基础设施: MXFP4 on the indexer QK path)
 *   scores[b][i][j] = sum_h w[b][i][h] * ReLU(qI[b][i][h] . kI[b][j])
 * for j < min(n_elig(q_pos[b][i]), max_blocks); other columns are not
 * written.  Accumulation in fp32.
 *   qI:        [batch][n_q][HI][dI] in p->idx_fmt (+ qI_scales); bf16 (and
 *              no scales) with CSA_FLAG_QI_BF16
 *   w:         float [batch][n_q][HI]
 *   kI:        [batch][max_blocks][dI] in p->idx_fmt (+ kI_scales)
 *   q_pos:     int64 [batch][n_q]
 *   scores:    float [batch][n_q][ld_scores], ld_scores >= max_blocks
 * The tensor-core kernels take MXFP4 with HI = 64, dI = 128, max_blocks a
 * multiple of 4 and batch * max_blocks >= 128, and BF16 with at least 4
 * queries per sequence; other calls run on the CUDA cores (much slower at
 * long contexts: allocate max_blocks in multiples of 4).  Formats without a
 * tensor-core path take at most 65535 query rows (batch * n_q) per call;
 * larger calls return CSA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
int indexer_score(const csa_params* p, int32_t batch, int32_t n_q, const void* qI,
                  const void* qI_scales, const float* w, const void* kI, const void* kI_scales,
                  int64_t max_blocks, const int64_t* q_pos, float* scores, int64_t ld_scores,
                  csa_stream_t stream);

/* ------------------------------------------------------------------------
 * topk_select -- per query, the min(k, n) best blocks by fp32 score, n =
 * min(n_elig(t), max_blocks) ([WK] 架构创新: top-k sparse selection).  Ties
 * go to the lower index; -0.0 equals +0.0.  idx int32 [batch][n_q][k],
 * written in ascending order and padded with -1.
 * ------------------------------------------------------------------------ */
int topk_select(const csa_params* p, int32_t batch, int32_t n_q, const float* scores,
                int64_t ld_scores, int64_t max_blocks, const int64_t* q_pos, int32_t* idx,
                csa_stream_t stream);

/* ------------------------------------------------------------------------
 * sparse_mqa_attn -- CSA attention over the selected pooled entries, the
 * raw window and a per-head sink ([WK] 架构创新: top-k + MQA, sliding window
 * branch and Attention Sink; [RN] CSA).  For query (b,i) at t = q_pos[b][i]
 * and head h, over items e = {kv[b][idx[b][i][a]] : idx >= 0} followed by the
 * raw tokens at positions t-W < pos <= t that lie in the raw buffer:
 *   l_e = scale * q.k_e,  M = max(sinks[h], max_e l_e)
 *   out = sum_e e^(l_e-M) k_e / (sum_e e^(l_e-M) + e^(sinks[h]-M))
 * (every item is its own key and value; sinks == NULL means no sink term).
 *   q:         [batch][n_q][H][d] in p->act_fmt
 *   kv:        [batch][max_entries][d] in p->kv_fmt (+ kv_scales)
 *   idx:       int32 [batch][n_q][k]
 *   raw:       [batch][n_raw][d] in p->act_fmt; row r of sequence b is the
 *              token at position raw_pos0[b] + r
 *   sinks:     float [H] or NULL
 *   out:       [batch][n_q][H][d] in p->act_fmt
 *   workspace: >= csa_workspace_size(p, CSA_OP_SPARSE_ATTN, batch, n_q, 0)
 * The tensor-core path takes BF16 activations with FP8_S64 or BF16 entries
 * at H = 64, d = 512; other shapes and formats take at most 65535 query
 * rows (batch * n_q) per call (also for hca_attn, csa_decode and
 * csa_prefill), larger calls returning CSA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
int sparse_mqa_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q,
                    const void* kv, const void* kv_scales, int64_t max_entries,
                    const int32_t* idx, const void* raw, int64_t n_raw, const int64_t* raw_pos0,
                    const int64_t* q_pos, const float* sinks, void* out, void* workspace,
                    size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * hca_attn -- HCA: dense attention over every visible pooled entry (all j <
 * min(n_elig(t), max_entries)) plus the same window and sink ([RN] HCA:
 * dense attention over the short pooled sequence plus a sliding window).
 * Arguments as sparse_mqa_attn without idx; p->top_k is ignored.
 *   workspace: >= csa_workspace_size(p, CSA_OP_HCA_ATTN, batch, n_q, max_entries)
 * ------------------------------------------------------------------------ */
int hca_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q, const void* kv,
             const void* kv_scales, int64_t max_entries, const void* raw, int64_t n_raw,
             const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks, void* out,
             void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * window_attn -- attention over the sliding window and the sink alone, with
 * no pooled entry ([RN] 架構實現: the final MTP block of V4-Pro uses only
 * sliding-window attention).  For query (b,i) at t = q_pos[b][i], over the
 * raw tokens at positions t-W < pos <= t that lie in the raw buffer, the
 * same softmax as sparse_mqa_attn with the sink in the denominator.
 * Arguments as hca_attn without kv; p->m, p->top_k and p->kv_fmt are not used.
 *   workspace: >= csa_workspace_size(p, CSA_OP_WINDOW_ATTN, batch, n_q, 0)
 * ------------------------------------------------------------------------ */
int window_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q, const void* raw,
                int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
                void* out, void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_decode -- one CSA read step for one new token per sequence:
 * indexer_score -> topk_select -> sparse_mqa_attn, launched back to back on
 * `stream` with the scores and selection in the workspace.  Shapes as above
 * with n_q = 1: q [batch][H][d], qI [batch][HI][dI], w [batch][HI],
 * q_pos [batch].  idx_out (int32 [batch][k]) receives the selection if not
 * NULL.
 *   workspace: >= csa_workspace_size(p, CSA_OP_DECODE, batch, 1, max_blocks)
 * ------------------------------------------------------------------------ */
int csa_decode(const csa_params* p, int32_t batch, const void* q, const void* qI,
               const void* qI_scales, const float* w, const void* kv, const void* kv_scales,
               const void* kI, const void* kI_scales, int64_t max_blocks, const void* raw,
               int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
               void* out, int32_t* idx_out, void* workspace, size_t ws_bytes,
               csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_prefill -- one CSA layer over a chunk of T tokens starting at position
 * t0 (a multiple of m) of every sequence: pool the chunk's complete blocks
 * into kv (entries t0/m .. (t0+T)/m - 1, stored in p->kv_fmt), score every
 * query's visible blocks, select the top-k and attend.
 *   raw:       [batch][n_raw][d] in p->act_fmt, positions raw_pos0 ..; it must
 *              hold the chunk (positions t0 .. t0+T-1, the pooled tokens) and
 *              the W-1 tokens before it when t0 > 0
 *   z:         [batch][T][d] gate logits of the chunk tokens; bias float [m][d]
 *   q:         [batch][T][H][d]; qI [batch][T][HI][dI]; w float [batch][T][HI]
 *   kv:        [batch][max_blocks][d] in p->kv_fmt, entries < t0/m already
 *              filled by the caller (written here: the chunk's entries)
 *   kI:        [batch][max_blocks][dI] in p->idx_fmt, filled by the caller
 *   out:       [batch][T][H][d] in p->act_fmt; idx_out int32 [batch][T][k] or NULL
 *   workspace: >= csa_workspace_size(p, CSA_OP_PREFILL, batch, T, max_blocks)
 * ------------------------------------------------------------------------ */
int csa_prefill(const csa_params* p, int32_t batch, int64_t T, int64_t t0, const void* raw,
                int64_t n_raw, int64_t raw_pos0, const void* z, const float* bias,
                const void* q, const void* qI, const void* qI_scales, const float* w, void* kv,
                void* kv_scales, const void* kI, const void* kI_scales, int64_t max_blocks,
                const float* sinks, void* out, int32_t* idx_out, void* workspace,
                size_t ws_bytes, csa_stream_t stream);

/* Operations for csa_workspace_size. */
#define CSA_OP_SPARSE_ATTN 0
#define CSA_OP_HCA_ATTN 1
#define CSA_OP_DECODE 2
#define CSA_OP_PREFILL 3
#define CSA_OP_WINDOW_ATTN 4
#define CSA_OP_SHARD_SELECT 5
#define CSA_OP_SHARD_ATTEND 6
#define CSA_OP_HCA_SHARD 7

/* Bytes of workspace an operation needs (0 on bad arguments; SIZE_MAX when
 * the size does not fit in size_t, which no buffer satisfies).  n_ctx is
 * max_entries (HCA) or max_blocks (decode, prefill); unused otherwise. */
size_t csa_workspace_size(const csa_params* p, int32_t op, int32_t batch, int64_t n_q,
                          int64_t n_ctx);

/* ------------------------------------------------------------------------
 * csa_decode_noalloc -- csa_decode for callers that cannot allocate device
 * memory.  The method itself has no counterpart of this call: it exists
 * only to serve such callers, because csa_decode needs a workspace.  Examples
 * are a host program with no device allocator of its own, a decode loop
 * that must not call cudaMalloc between steps (cudaMalloc synchronises the
 * device), and a server whose device memory is all committed at start-up.
 *
 * It computes exactly what csa_decode computes, with the same kernels and
 * the same arguments, minus `workspace` and `ws_bytes`.  The scores,
 * selection and split-K partials go to a fixed scratch area that the library
 * reserves statically in every CUDA context that loads it (one per device
 * in the usual case): CSA_NOALLOC_SCRATCH_BYTES, which is 32 MiB.  At m = 4, k = 512, W = 128 and 64 heads of 512, that covers any
 * batch of 1 to 252 sequences of 128K tokens, or 32 sequences of up to
 * 500,000 tokens.  Nothing is allocated, not even on the first call.
 *
 *   errors: CSA_ERR_WORKSPACE, with nothing launched, when
 *           csa_workspace_size(p, CSA_OP_DECODE, batch, 1, max_blocks) is
 *           larger than CSA_NOALLOC_SCRATCH_BYTES.  Otherwise the errors are
 *           those of csa_decode.  CSA_ERR_CUDA if the scratch address cannot
 *           be found in the current context.
 *   device: the scratch belongs to the CUDA context that is current on
 *           the calling thread (normally the device's primary context).  The
 *           stream and all pointers must belong to that context too.  Its
 *           address is looked up on every call, so a device reset or a
 *           switch to another context is followed correctly.
 *   first call: the first call in a context may load the library's device
 *           code to find the scratch.  So make the first call on each device
 *           outside any stream capture, before the calls you intend to
 *           record.
 *   initial contents: none required.  Each scratch byte a call reads was
 *           written earlier in the same call, so nothing needs to start at
 *           zero.  The device status word (csa_device_status) is separate
 *           from the scratch and behaves as for csa_decode.
 *   overlap: every call on a device shares the one scratch area.  Two calls
 *           on that device whose work can overlap race on it and corrupt
 *           each other's results: calls from different streams, or from
 *           different host threads.  Order them on one stream or with events.
 * ------------------------------------------------------------------------ */
#define CSA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

int csa_decode_noalloc(const csa_params* p, int32_t batch, const void* q, const void* qI,
                       const void* qI_scales, const float* w, const void* kv,
                       const void* kv_scales, const void* kI, const void* kI_scales,
                       int64_t max_blocks, const void* raw, int64_t n_raw,
                       const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
                       void* out, int32_t* idx_out, csa_stream_t stream);

/* ========================================================================
 * Sharded decode: one sequence's pooled entries split over ranks along the
 * entry axis, for contexts of 1M tokens and beyond ([RN] 架構實現 and the
 * paper summary: 1M-token context; a CSA layer takes the top-k of all
 * visible entries, an HCA layer attends to all of them).  Rank r holds the
 * contiguous entries [entry0, entry0 + n_entries) of every sequence of the
 * batch (local entry j is global entry entry0 + j); exactly one rank passes
 * the raw window (n_raw > 0), the others n_raw = 0.  Per CSA layer:
 *   1. csa_shard_select on every rank -> k candidates (score, global id);
 *   2. all-gather of the candidates, rank-major: [n_parts][batch][k];
 *   3. csa_shard_attend on every rank -> the exact global top-k (the union
 *      of the shards' top-k under the order score descending, id ascending
 *      contains it), attention over the selected entries this rank holds
 *      (and the window) as an unnormalised partial;
 *   4. all-gather of the partials, rank-major; attn_merge -> the output.
 * Per HCA layer: hca_shard_attend, all-gather, attn_merge.  The partial of
 * a row is O [H][D] fp32 (sum of e^(logit - M) v over this rank's items)
 * and (M, L) per head (float pairs: M in natural-log units, L the sum of
 * e^(logit - M)); a rank with no item gives M = -inf, L = 0, O = 0.  The
 * exchange itself is the caller's (an NCCL all-gather); these calls only
 * read and write device memory on `stream`.
 * ======================================================================== */

/* csa_shard_select -- the indexer over this rank's keys and their local
 * top-k.  Key j is scored for query t only if entry0 + j < n_elig(t).
 *   qI, qI_scales, w, q_pos as for csa_decode (p->flags apply); kI: this
 *   rank's keys [batch][n_entries][dI] in p->idx_fmt.
 *   cand_scores float [batch][k], cand_ids int32 [batch][k]: the local top-k
 *   (ids global, in ascending order), padded with (-inf, -1).
 *   workspace: >= csa_workspace_size(p, CSA_OP_SHARD_SELECT, batch, 1, n_entries) */
int csa_shard_select(const csa_params* p, int32_t batch, const void* qI, const void* qI_scales, const float* w,
                     const void* kI, const void* kI_scales, int64_t n_entries, int64_t entry0,
                     const int64_t* q_pos, float* cand_scores, int32_t* cand_ids, void* workspace,
                     size_t ws_bytes, csa_stream_t stream);

/* csa_shard_attend -- the global top-k of the gathered candidates and this
 * rank's partial of the sparse attention.
 *   cand_scores, cand_ids: [n_parts][batch][k] (every rank's csa_shard_select
 *   output, rank-major); n_parts <= 64, n_parts * k <= 16384 and k <= 4096,
 *   else CSA_ERR_UNSUPPORTED.  kv: this rank's entries [batch][n_entries][d] in
 *   p->kv_fmt; raw / n_raw / raw_pos0: the window as for csa_decode on the
 *   rank that attends to it, n_raw = 0 (raw may be NULL) elsewhere.
 *   part_o float [batch][H][d], part_ml float [batch][H][2]: the partial.
 *   idx_out int32 [batch][k] (may be NULL): the global selection, ascending
 *   ids, -1 padded -- the same on every rank.
 *   workspace: >= csa_workspace_size(p, CSA_OP_SHARD_ATTEND, batch, 1, n_entries) */
int csa_shard_attend(const csa_params* p, int32_t batch, const void* q, int32_t n_parts, const float* cand_scores,
                     const int32_t* cand_ids, const void* kv, const void* kv_scales, int64_t n_entries,
                     int64_t entry0, const void* raw, int64_t n_raw, const int64_t* raw_pos0,
                     const int64_t* q_pos, float* part_o, float* part_ml, int32_t* idx_out, void* workspace,
                     size_t ws_bytes, csa_stream_t stream);

/* hca_shard_attend -- this rank's partial of the dense HCA attention: local
 * entries j with entry0 + j < n_elig(t), plus the window on the rank that
 * passes it.  Arguments as csa_shard_attend without the candidates.
 *   workspace: >= csa_workspace_size(p, CSA_OP_HCA_SHARD, batch, 1, n_entries) */
int hca_shard_attend(const csa_params* p, int32_t batch, const void* q, const void* kv, const void* kv_scales,
                     int64_t n_entries, int64_t entry0, const void* raw, int64_t n_raw,
                     const int64_t* raw_pos0, const int64_t* q_pos, float* part_o, float* part_ml,
                     void* workspace, size_t ws_bytes, csa_stream_t stream);

/* attn_merge -- LSE merge of n_parts partials per row (rank-major:
 * part_o [n_parts][batch][H][d], part_ml [n_parts][batch][H][2]) with the
 * per-head sink (NULL: none):
 *   out = sum_r e^(M_r - M) O_r / (sum_r e^(M_r - M) L_r + e^(sink - M))
 * in p->act_fmt [batch][H][d].  n_parts <= 64 (else CSA_ERR_UNSUPPORTED). */
int attn_merge(const csa_params* p, int32_t batch, int32_t n_parts, const float* part_o, const float* part_ml,
               const float* sinks, void* out, csa_stream_t stream);

/* Synchronise `stream`, return the device status word (CSA_DEV_* bits) in
 * *flags, and clear it if `reset` is non-zero.  The word is shared by every
 * call on the current device. */
int csa_device_status(csa_stream_t stream, uint32_t* flags, int32_t reset);

/* Static description of a status code; never NULL. */
const char* csa_strerror(int status);

/* Library version string, e.g. "csa13 0.1.0 sm_100a". */
const char* csa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA13_CSA_H */
