// C-ABI entry points (declared in include/csa.h): argument checks on the
// host, workspace layout, and the choice of kernel for each format.
#include <stdio.h>

#include <mutex>

#include "kernels.h"

namespace csa {

__device__ unsigned int g_status = 0;

cudaError_t ensure_smem_impl(const void* kernel, size_t bytes) {
    struct Entry { const void* k; int dev; size_t bytes; };
    static Entry table[64];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].k == kernel && table[i].dev == dev && table[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e != cudaSuccess) return e;
    for (int i = 0; i < used; ++i)
        if (table[i].k == kernel && table[i].dev == dev) { table[i].bytes = bytes; return e; }
    if (used < 64) table[used++] = Entry{kernel, dev, bytes};
    return e;
}

static bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static bool act_ok(int f) { return f == CSA_F32 || f == CSA_BF16; }
static bool kv_ok(int f) { return f == CSA_F32 || f == CSA_BF16 || f == CSA_FP8_S64; }
static bool idx_ok(int f) { return f == CSA_F32 || f == CSA_BF16 || f == CSA_MXFP4; }

static int check_params(const csa_params* p, bool need_idx, bool need_attn) {
    if (!p) return CSA_ERR_ARG;
    if (p->m <= 0 || p->window < 0) return CSA_ERR_ARG;
    if (p->flags & ~(CSA_FLAG_BATCH_INVARIANT | CSA_FLAG_QI_BF16 | CSA_FLAG_INDEXER_FP8)) return CSA_ERR_ARG;
    if (need_attn) {
        if (p->n_heads <= 0 || p->head_dim <= 0 || (p->head_dim % 64) != 0) return CSA_ERR_ARG;
        if (!act_ok(p->act_fmt) || !kv_ok(p->kv_fmt)) return CSA_ERR_ARG;
        if (!(p->scale == p->scale)) return CSA_ERR_ARG;
    }
    if (need_idx) {
        if (p->idx_heads <= 0 || p->idx_dim <= 0 || (p->idx_dim % 32) != 0) return CSA_ERR_ARG;
        if (!idx_ok(p->idx_fmt) || p->top_k <= 0) return CSA_ERR_ARG;
    }
    return CSA_OK;
}

static int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return CSA_OK;
    if (e == cudaErrorInvalidValue) return CSA_ERR_UNSUPPORTED;
    return CSA_ERR_CUDA;
}

// ------------------------------------------------------------ attention
static int choose_splits(int64_t rows, int64_t items_per_row) {
    // Enough CTAs to cover every SM about twice, with at least 64 items per split.
    if (rows <= 0 || rows >= 2 * kNumSMs) return 1;
    int64_t s = ceil_div(2 * kNumSMs, rows);
    s = std::min<int64_t>(s, ceil_div(items_per_row, 64));
    return int(std::max<int64_t>(1, std::min<int64_t>(s, 64)));
}

struct AttnPlan {
    int n_splits;
    size_t part_o_bytes, part_ml_bytes;
    size_t bytes() const { return n_splits > 1 ? part_o_bytes + part_ml_bytes : 0; }
};

// The tensor-core kernel runs one ~215 KB CTA per SM, so its splits fill the
// 148 SMs in a single wave with at least one 64-item tile per split.
static int choose_splits_tc(int64_t rows, int64_t items_per_row) {
    if (rows <= 0 || rows >= kNumSMs) return 1;
    const int64_t s = std::min<int64_t>(kNumSMs / rows, ceil_div(items_per_row, 64));
    return int(std::max<int64_t>(1, std::min<int64_t>(s, 64)));
}

// Batch-invariant mode: the split count of a row depends on the row's own
// number of items only (never on how many rows share the launch), so a row's
// partial sums, their combine order and hence its output bits are the same
// in any batch.  About three 64-item tiles per split, at most 8 (one cluster).
static int choose_splits_invariant(int64_t items_per_row) {
    const int64_t tiles = ceil_div(std::max<int64_t>(items_per_row, 1), 64);
    return int(std::max<int64_t>(1, std::min<int64_t>(8, ceil_div(tiles, 3))));
}

static AttnPlan plan_attn(const csa_params* p, int64_t rows, int64_t items_per_row) {
    AttnPlan a;
    // (the tensor-core kernel is also limited to rows that fit 32 bits; with
    // larger buffers the CUDA-core kernel runs with the same split count)
    if (p->flags & CSA_FLAG_BATCH_INVARIANT)
        a.n_splits = choose_splits_invariant(items_per_row);
    else
        a.n_splits = attn_tc_supported(p->act_fmt, p->kv_fmt, p->n_heads, p->head_dim)
                         ? choose_splits_tc(rows, items_per_row)
                         : choose_splits(rows, items_per_row);
    const int64_t items = rows * a.n_splits;
    a.part_o_bytes = size_t(items) * p->n_heads * p->head_dim * sizeof(float);
    a.part_ml_bytes = size_t(items) * p->n_heads * sizeof(float2);
    a.part_o_bytes = (a.part_o_bytes + 255) & ~size_t(255);
    return a;
}

// Attention over each row's items into `out`.  With part_ml set, the result
// is instead the row's unnormalised partial (part_ml: max and sum per head,
// out: fp32 O [rows][H][D]) without the sink, for a later merge with other
// shards' partials; kv_base is the global index of kv's entry 0 (dense rows).
static int run_attn(const csa_params* p, int batch, int n_q, const void* q, const void* kv,
                    const void* kv_s, int64_t max_entries, const int32_t* idx, const void* raw,
                    int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos,
                    const float* sinks, void* out, void* ws, size_t ws_bytes, int64_t items_per_row,
                    cudaStream_t s, bool pdl = false, float2* part_ml = nullptr, int64_t kv_base = 0,
                    const int32_t* n_sel = nullptr) {
    const int64_t rows = int64_t(batch) * n_q;
    if (!attn_simt_supported(p->act_fmt, p->kv_fmt, p->n_heads, p->head_dim) &&
        !attn_tc_supported(p->act_fmt, p->kv_fmt, p->n_heads, p->head_dim))
        return CSA_ERR_UNSUPPORTED;
    const AttnPlan plan = plan_attn(p, rows, items_per_row);
    if (plan.bytes() > ws_bytes) return CSA_ERR_WORKSPACE;
    if (plan.bytes() && !ws) return CSA_ERR_ARG;
    AttnArgs a;
    a.H = p->n_heads; a.D = p->head_dim; a.m = p->m; a.W = p->window; a.k = p->top_k;
    a.scale = p->scale;
    a.q = q; a.kv = kv; a.kv_s = kv_s; a.kv_fmt = p->kv_fmt; a.max_entries = max_entries; a.idx = idx;
    a.raw = raw; a.n_raw = n_raw; a.raw_pos0 = raw_pos0; a.q_pos = q_pos; a.sinks = sinks;
    a.n_q = n_q; a.n_splits = plan.n_splits; a.out = out;
    a.part_o = (float*)ws;
    a.part_ml = (float2*)((char*)ws + plan.part_o_bytes);
    a.partial_out = part_ml != nullptr;
    a.kv_base = kv_base;
    a.n_sel = n_sel;
    if (part_ml && plan.n_splits == 1) {  // the one split's partial is the result
        a.part_o = (float*)out;
        a.part_ml = part_ml;
    }
    const bool tc = attn_tc_supported(p->act_fmt, p->kv_fmt, p->n_heads, p->head_dim) &&
                    attn_tc_rows_fit(max_entries, n_raw);
    // the CUDA-core kernel puts the query rows on the grid's y axis
    if (!tc && rows > kMaxGridY) return CSA_ERR_UNSUPPORTED;
    a.fused_combine = 0;
    a.row_base = 0;
    bool combined = false;
    int st = cuda_status(tc ? launch_attn_tc(a, rows, s, &combined, pdl)
                            : launch_attn_simt(p->act_fmt, p->kv_fmt, a, rows, s));
    if (st) return st;
    // the combine always follows this function's own attention launch
    if (plan.n_splits > 1 && !combined)
        st = cuda_status(launch_combine_strided(p->act_fmt, part_ml != nullptr, p->n_heads, p->head_dim,
                                                plan.n_splits, rows, plan.n_splits, 1, a.part_o, a.part_ml,
                                                sinks, out, part_ml, s, /*pdl=*/true));
    return st;
}

__global__ void fill_positions_kernel(int64_t* q_pos, int64_t* pos0, int batch, int64_t T,
                                      int64_t t0, int64_t raw_pos0) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < int64_t(batch) * T) q_pos[i] = t0 + i % T;
    if (i < batch) pos0[i] = raw_pos0;
}

static cudaError_t launch_fill_positions(int64_t* q_pos, int64_t* pos0, int batch, int64_t T,
                                         int64_t t0, int64_t raw_pos0, cudaStream_t s) {
    const int64_t n = std::max<int64_t>(int64_t(batch) * T, batch);
    fill_positions_kernel<<<unsigned(ceil_div(n, 256)), 256, 0, s>>>(q_pos, pos0, batch, T, t0, raw_pos0);
    return cudaGetLastError();
}

static int check_attn_ptrs(const void* q, const void* kv, const void* kv_s, int kv_fmt,
                           const void* raw, int64_t n_raw, const int64_t* raw_pos0,
                           const int64_t* q_pos, void* out, bool need_kv = true) {
    if (!q || (need_kv && !kv) || !q_pos || !out || !raw_pos0) return CSA_ERR_ARG;
    if (n_raw < 0 || (n_raw > 0 && !raw)) return CSA_ERR_ARG;
    if (need_kv && kv_fmt == CSA_FP8_S64 && !kv_s) return CSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(kv_s) || !aligned16(raw) || !aligned16(out))
        return CSA_ERR_ALIGN;
    return CSA_OK;
}

}  // namespace csa

using namespace csa;

extern "C" {

int csa_compress(const csa_params* p, int32_t d, const void* x, const void* z, const float* bias,
                 int64_t n_tokens, int32_t out_fmt, void* out, void* out_scales,
                 csa_stream_t stream) {
    if (!p || p->m <= 0 || d <= 0 || (d % 64) != 0 || n_tokens < 0 || (n_tokens % p->m) != 0)
        return CSA_ERR_ARG;
    if (!act_ok(p->act_fmt)) return CSA_ERR_ARG;
    if (out_fmt < CSA_F32 || out_fmt > CSA_MXFP4) return CSA_ERR_ARG;
    if (n_tokens == 0) return CSA_OK;
    if (!x || !z || !bias || !out) return CSA_ERR_ARG;
    if ((out_fmt == CSA_FP8_S64 || out_fmt == CSA_MXFP4) && !out_scales) return CSA_ERR_ARG;
    // scales are stored one by one (fp32 for FP8_S64, one byte for MXFP4), so
    // a single pooled row can be appended at any index
    const bool scales_ok = out_fmt != CSA_FP8_S64 || (reinterpret_cast<uintptr_t>(out_scales) & 3) == 0;
    if (!aligned16(x) || !aligned16(z) || !aligned16(bias) || !aligned16(out) || !scales_ok)
        return CSA_ERR_ALIGN;
    return cuda_status(launch_compress(p->act_fmt, out_fmt, x, z, bias, n_tokens, p->m, d, out,
                                       out_scales, (cudaStream_t)stream));
}

int csa_quantize(int32_t fmt, const float* src, int64_t rows, int32_t d, void* out,
                 void* out_scales, csa_stream_t stream) {
    if (d <= 0 || (d % 64) != 0 || rows < 0) return CSA_ERR_ARG;
    if (fmt != CSA_BF16 && fmt != CSA_FP8_S64 && fmt != CSA_MXFP4 && fmt != CSA_F32) return CSA_ERR_ARG;
    if (rows == 0) return CSA_OK;
    if (!src || !out || (fmt >= CSA_FP8_S64 && !out_scales)) return CSA_ERR_ARG;
    if (!aligned16(src) || !aligned16(out) || !aligned16(out_scales)) return CSA_ERR_ALIGN;
    return cuda_status(launch_quantize(fmt, src, rows, d, out, out_scales, (cudaStream_t)stream));
}

int indexer_score(const csa_params* p, int32_t batch, int32_t n_q, const void* qI,
                  const void* qI_scales, const float* w, const void* kI, const void* kI_scales,
                  int64_t max_blocks, const int64_t* q_pos, float* scores, int64_t ld_scores,
                  csa_stream_t stream) {
    int st = check_params(p, true, false);
    if (st) return st;
    if (batch < 0 || n_q < 0 || max_blocks < 0 || ld_scores < max_blocks) return CSA_ERR_ARG;
    if (batch == 0 || n_q == 0 || max_blocks == 0) return CSA_OK;
    if (!qI || !w || !kI || !q_pos || !scores) return CSA_ERR_ARG;
    // the write-path variants of the MXFP4 indexer (bf16 queries quantised in
    // the kernel; the exact E2M1 -> E4M3 expansion on the MXFP8 MMA)
    const bool q_bf16 = (p->flags & CSA_FLAG_QI_BF16) != 0;
    const bool fp8 = (p->flags & CSA_FLAG_INDEXER_FP8) != 0;
    if ((q_bf16 || fp8) && p->idx_fmt != CSA_MXFP4) return CSA_ERR_ARG;
    if (p->idx_fmt == CSA_MXFP4 && ((!q_bf16 && !qI_scales) || !kI_scales)) return CSA_ERR_ARG;
    if (!aligned16(qI) || !aligned16(kI) || !aligned16(scores) || !aligned16(qI_scales) ||
        !aligned16(kI_scales))
        return CSA_ERR_ALIGN;
    if (indexer_tc_supported(p->idx_fmt, p->idx_heads, p->idx_dim, max_blocks, batch,
                             int64_t(batch) * n_q))
        return cuda_status(launch_indexer_tc(qI, q_bf16 ? nullptr : qI_scales, w, kI, kI_scales, max_blocks,
                                             q_pos, batch, n_q, p->m, p->window, scores, ld_scores, q_bf16,
                                             fp8, (cudaStream_t)stream));
    if (q_bf16 || fp8) return CSA_ERR_UNSUPPORTED;  // the variants exist on the tensor-core path only
    if (indexer_bf16_tc_supported(p->idx_fmt, p->idx_heads, p->idx_dim, max_blocks, batch, n_q))
        return cuda_status(launch_indexer_bf16_tc(qI, w, kI, max_blocks, q_pos, batch, n_q, p->m,
                                                  p->window, scores, ld_scores, (cudaStream_t)stream));
    // the CUDA-core kernel puts the query rows on the grid's y axis
    if (int64_t(batch) * n_q > kMaxGridY) return CSA_ERR_UNSUPPORTED;
    return cuda_status(launch_indexer_simt(p->idx_fmt, p->idx_heads, p->idx_dim, p->m, p->window,
                                           qI, qI_scales, w, kI, kI_scales, max_blocks, q_pos,
                                           batch, n_q, max_blocks, scores, ld_scores,
                                           (cudaStream_t)stream));
}

static int topk_impl(const csa_params* p, int32_t batch, int32_t n_q, const float* scores,
                     int64_t ld_scores, int64_t max_blocks, const int64_t* q_pos, int32_t* idx,
                     csa_stream_t stream, bool pdl) {
    if (!p || p->m <= 0 || p->window < 0 || p->top_k <= 0) return CSA_ERR_ARG;
    if (batch < 0 || n_q < 0 || max_blocks < 0 || ld_scores < max_blocks) return CSA_ERR_ARG;
    if (max_blocks > INT32_MAX) return CSA_ERR_UNSUPPORTED;
    if (batch == 0 || n_q == 0) return CSA_OK;
    if (!q_pos || !idx || (max_blocks > 0 && !scores)) return CSA_ERR_ARG;
    return cuda_status(launch_topk(scores, ld_scores, max_blocks, q_pos, p->m, p->window, p->top_k,
                                   int64_t(batch) * n_q, idx, (cudaStream_t)stream, pdl));
}

int topk_select(const csa_params* p, int32_t batch, int32_t n_q, const float* scores,
                int64_t ld_scores, int64_t max_blocks, const int64_t* q_pos, int32_t* idx,
                csa_stream_t stream) {
    return topk_impl(p, batch, n_q, scores, ld_scores, max_blocks, q_pos, idx, stream, false);
}

static int sparse_attn_impl(const csa_params* p, int32_t batch, int32_t n_q, const void* q,
                            const void* kv, const void* kv_scales, int64_t max_entries,
                            const int32_t* idx, const void* raw, int64_t n_raw,
                            const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
                            void* out, void* workspace, size_t ws_bytes, csa_stream_t stream,
                            bool pdl);

int sparse_mqa_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q, const void* kv,
                    const void* kv_scales, int64_t max_entries, const int32_t* idx,
                    const void* raw, int64_t n_raw, const int64_t* raw_pos0,
                    const int64_t* q_pos, const float* sinks, void* out, void* workspace,
                    size_t ws_bytes, csa_stream_t stream) {
    return sparse_attn_impl(p, batch, n_q, q, kv, kv_scales, max_entries, idx, raw, n_raw, raw_pos0,
                            q_pos, sinks, out, workspace, ws_bytes, stream, false);
}

static int sparse_attn_impl(const csa_params* p, int32_t batch, int32_t n_q, const void* q,
                            const void* kv, const void* kv_scales, int64_t max_entries,
                            const int32_t* idx, const void* raw, int64_t n_raw,
                            const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
                            void* out, void* workspace, size_t ws_bytes, csa_stream_t stream,
                            bool pdl) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (p->top_k <= 0 || batch < 0 || n_q < 0 || max_entries < 0) return CSA_ERR_ARG;
    if (batch == 0 || n_q == 0) return CSA_OK;
    if (!idx) return CSA_ERR_ARG;
    st = check_attn_ptrs(q, kv, kv_scales, p->kv_fmt, raw, n_raw, raw_pos0, q_pos, out);
    if (st) return st;
    return run_attn(p, batch, n_q, q, kv, kv_scales, max_entries, idx, raw, n_raw, raw_pos0, q_pos,
                    sinks, out, workspace, ws_bytes, int64_t(p->top_k) + p->window,
                    (cudaStream_t)stream, pdl);
}

int hca_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q, const void* kv,
             const void* kv_scales, int64_t max_entries, const void* raw, int64_t n_raw,
             const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks, void* out,
             void* workspace, size_t ws_bytes, csa_stream_t stream) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (batch < 0 || n_q < 0 || max_entries < 0) return CSA_ERR_ARG;
    if (batch == 0 || n_q == 0) return CSA_OK;
    st = check_attn_ptrs(q, kv, kv_scales, p->kv_fmt, raw, n_raw, raw_pos0, q_pos, out);
    if (st) return st;
    return run_attn(p, batch, n_q, q, kv, kv_scales, max_entries, nullptr, raw, n_raw, raw_pos0,
                    q_pos, sinks, out, workspace, ws_bytes, max_entries + p->window,
                    (cudaStream_t)stream);
}

int window_attn(const csa_params* p, int32_t batch, int32_t n_q, const void* q, const void* raw,
                int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
                void* out, void* workspace, size_t ws_bytes, csa_stream_t stream) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (batch < 0 || n_q < 0) return CSA_ERR_ARG;
    if (batch == 0 || n_q == 0) return CSA_OK;
    st = check_attn_ptrs(q, nullptr, nullptr, p->kv_fmt, raw, n_raw, raw_pos0, q_pos, out, false);
    if (st) return st;
    // no pooled entry is visible: the dense path over zero entries attends the
    // window (and the sink) alone
    return run_attn(p, batch, n_q, q, nullptr, nullptr, 0, nullptr, raw, n_raw, raw_pos0, q_pos, sinks,
                    out, workspace, ws_bytes, p->window, (cudaStream_t)stream);
}

size_t csa_workspace_size(const csa_params* p, int32_t op, int32_t batch, int64_t n_q,
                          int64_t n_ctx) {
    if (!p || batch < 0 || n_q < 0 || n_ctx < 0 || p->n_heads <= 0 || p->head_dim <= 0) return 0;
    // Every term below is at most rows x max(n_ctx, top_k + window, 64 x H x d) x 8 bytes
    // (64 splits of fp32 partials); beyond size_t the answer saturates.
    {
        const unsigned __int128 rows_ = (unsigned __int128)batch * (uint64_t)n_q;
        const int64_t per_row = std::max<int64_t>(std::max<int64_t>(n_ctx, int64_t(p->top_k) + p->window),
                                                  int64_t(64) * p->n_heads * p->head_dim);
        const unsigned __int128 per = (unsigned __int128)(uint64_t)per_row;
        if (rows_ * per * 8 + (rows_ + 1) * 4096 > (unsigned __int128)(SIZE_MAX / 4)) return SIZE_MAX;
    }
    const int64_t rows = int64_t(batch) * n_q;
    switch (op) {
    case CSA_OP_SPARSE_ATTN:
        return plan_attn(p, rows, int64_t(p->top_k) + p->window).bytes() + 256;
    case CSA_OP_HCA_ATTN:
        return plan_attn(p, rows, n_ctx + p->window).bytes() + 256;
    case CSA_OP_WINDOW_ATTN:
        return plan_attn(p, rows, p->window).bytes() + 256;
    case CSA_OP_DECODE:
    case CSA_OP_PREFILL: {
        const size_t pos = op == CSA_OP_PREFILL ? ((size_t(rows) + batch) * 8 + 255) & ~size_t(255) : 0;
        const size_t scores = ((size_t(rows) * size_t(std::max<int64_t>(n_ctx, 1)) * 4) + 255) & ~size_t(255);
        const size_t sel = ((size_t(rows) * p->top_k * 4) + 255) & ~size_t(255);
        return pos + scores + sel + plan_attn(p, rows, int64_t(p->top_k) + p->window).bytes() + 256;
    }
    case CSA_OP_SHARD_SELECT: {
        const size_t pos = ((size_t(rows) * 8) + 255) & ~size_t(255);
        const size_t scores = ((size_t(rows) * size_t(std::max<int64_t>(n_ctx, 1)) * 4) + 255) & ~size_t(255);
        const size_t sel = ((size_t(rows) * p->top_k * 4) + 255) & ~size_t(255);
        return pos + scores + sel + 256;
    }
    case CSA_OP_SHARD_ATTEND: {
        const size_t sel = ((size_t(rows) * p->top_k * 4) + 255) & ~size_t(255);
        const size_t cnt = ((size_t(rows) * 4) + 255) & ~size_t(255);
        const size_t merge = topk_merge_workspace(rows, p->top_k);
        return 2 * sel + cnt + std::max(merge, plan_attn(p, rows, int64_t(p->top_k) + p->window).bytes()) + 256;
    }
    case CSA_OP_HCA_SHARD:
        return plan_attn(p, rows, n_ctx + p->window).bytes() + 256;
    default:
        return 0;
    }
}

int csa_decode(const csa_params* p, int32_t batch, const void* q, const void* qI,
               const void* qI_scales, const float* w, const void* kv, const void* kv_scales,
               const void* kI, const void* kI_scales, int64_t max_blocks, const void* raw,
               int64_t n_raw, const int64_t* raw_pos0, const int64_t* q_pos, const float* sinks,
               void* out, int32_t* idx_out, void* workspace, size_t ws_bytes,
               csa_stream_t stream) {
    int st = check_params(p, true, true);
    if (st) return st;
    if (batch < 0 || max_blocks < 0) return CSA_ERR_ARG;
    if (batch == 0) return CSA_OK;
    if (!workspace) return CSA_ERR_ARG;
    if (ws_bytes < csa_workspace_size(p, CSA_OP_DECODE, batch, 1, max_blocks)) return CSA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA_ERR_ALIGN;
    const int64_t ld = std::max<int64_t>(max_blocks, 1);
    float* scores = (float*)workspace;
    const size_t sc_bytes = ((size_t(batch) * ld * 4) + 255) & ~size_t(255);
    int32_t* sel = idx_out ? idx_out : (int32_t*)((char*)workspace + sc_bytes);
    const size_t sel_bytes = ((size_t(batch) * p->top_k * 4) + 255) & ~size_t(255);
    void* ws_attn = (char*)workspace + sc_bytes + sel_bytes;
    const size_t ws_attn_bytes = ws_bytes - sc_bytes - sel_bytes;
    st = indexer_score(p, batch, 1, qI, qI_scales, w, kI, kI_scales, max_blocks, q_pos, scores, ld,
                       stream);
    if (st) return st;
    // (Launching top-k and attention as programmatic dependents of the kernel
    // before them measured slower on this step: their early CTAs take SM
    // slots from the running kernel.  They are launched normally.)
    st = topk_impl(p, batch, 1, scores, ld, max_blocks, q_pos, sel, stream, false);
    if (st) return st;
    return sparse_attn_impl(p, batch, 1, q, kv, kv_scales, max_blocks, sel, raw, n_raw, raw_pos0,
                            q_pos, sinks, out, ws_attn, ws_attn_bytes, stream, false);
}

int csa_prefill(const csa_params* p, int32_t batch, int64_t T, int64_t t0, const void* raw,
                int64_t n_raw, int64_t raw_pos0, const void* z, const float* bias, const void* q,
                const void* qI, const void* qI_scales, const float* w, void* kv, void* kv_scales,
                const void* kI, const void* kI_scales, int64_t max_blocks, const float* sinks,
                void* out, int32_t* idx_out, void* workspace, size_t ws_bytes,
                csa_stream_t stream) {
    int st = check_params(p, true, true);
    if (st) return st;
    if (batch < 0 || T < 0 || t0 < 0 || (t0 % p->m) != 0 || max_blocks < 0) return CSA_ERR_ARG;
    if (batch == 0 || T == 0) return CSA_OK;
    if (!raw || !z || !bias || !kv || !workspace) return CSA_ERR_ARG;
    if (T > INT32_MAX) return CSA_ERR_UNSUPPORTED;
    // the chunk's tokens must be in the raw buffer; the window needs the W-1 before it
    if (raw_pos0 > t0 || raw_pos0 + n_raw < t0 + T) return CSA_ERR_ARG;
    if (raw_pos0 > std::max<int64_t>(0, t0 - p->window + 1)) return CSA_ERR_ARG;
    const int64_t nb_end = (t0 + T) / p->m;  // pooled entries after the chunk
    if (nb_end > max_blocks) return CSA_ERR_ARG;
    if (ws_bytes < csa_workspace_size(p, CSA_OP_PREFILL, batch, T, max_blocks)) return CSA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t rows = int64_t(batch) * T;
    const int64_t ld = std::max<int64_t>(max_blocks, 1);
    char* wp = (char*)workspace;
    int64_t* q_pos = (int64_t*)wp;
    wp += ((size_t(rows) + size_t(batch)) * 8 + 255) & ~size_t(255);
    int64_t* pos0 = q_pos + rows;
    float* scores = (float*)wp;
    wp += ((size_t(rows) * ld * 4) + 255) & ~size_t(255);
    int32_t* sel = idx_out ? idx_out : (int32_t*)wp;
    wp += ((size_t(rows) * p->top_k * 4) + 255) & ~size_t(255);
    const size_t used = size_t(wp - (char*)workspace);
    st = cuda_status(launch_fill_positions(q_pos, pos0, batch, T, t0, raw_pos0, s));
    if (st) return st;
    // 1. pool the chunk's complete blocks into kv entries [t0/m, (t0+T)/m)
    const int64_t n_pool = (T / p->m) * p->m;
    const size_t act_es = p->act_fmt == CSA_F32 ? 4 : 2;
    const size_t kv_es = p->kv_fmt == CSA_F32 ? 4 : (p->kv_fmt == CSA_BF16 ? 2 : 1);
    const int d = p->head_dim;
    for (int b = 0; b < batch && n_pool > 0; ++b) {
        const char* xb = (const char*)raw + (size_t(b) * n_raw + size_t(t0 - raw_pos0)) * d * act_es;
        const char* zb = (const char*)z + size_t(b) * T * d * act_es;
        char* ob = (char*)kv + (size_t(b) * max_blocks + size_t(t0 / p->m)) * d * kv_es;
        char* osb = nullptr;
        if (p->kv_fmt == CSA_FP8_S64) {
            if (!kv_scales) return CSA_ERR_ARG;
            osb = (char*)kv_scales + (size_t(b) * max_blocks + size_t(t0 / p->m)) * (d / 64) * 4;
        }
        st = csa_compress(p, d, xb, zb, bias, n_pool, p->kv_fmt, ob, osb, stream);
        if (st) return st;
    }
    // 2-4. score, select, attend
    st = indexer_score(p, batch, int32_t(T), qI, qI_scales, w, kI, kI_scales, max_blocks, q_pos,
                       scores, ld, stream);
    if (st) return st;
    st = topk_select(p, batch, int32_t(T), scores, ld, max_blocks, q_pos, sel, stream);
    if (st) return st;
    return sparse_mqa_attn(p, batch, int32_t(T), q, kv, kv_scales, max_blocks, sel, raw, n_raw,
                           pos0, q_pos, sinks, out, wp, ws_bytes - used, stream);
}

int csa_device_status(csa_stream_t stream, uint32_t* flags, int32_t reset) {
    if (!flags) return CSA_ERR_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return CSA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return CSA_ERR_CUDA;
    *flags = v;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return CSA_ERR_CUDA;
    }
    return CSA_OK;
}

const char* csa_strerror(int status) {
    switch (status) {
    case CSA_OK: return "ok";
    case CSA_ERR_ARG: return "invalid argument";
    case CSA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case CSA_ERR_UNSUPPORTED: return "shape or format combination not supported";
    case CSA_ERR_WORKSPACE: return "workspace too small";
    case CSA_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
    }
}

const char* csa_version(void) { return "csa13 0.1.0 sm_100a"; }


// ------------------------------------------------------------ sharded decode
int csa_shard_select(const csa_params* p, int32_t batch, const void* qI, const void* qI_scales, const float* w,
                     const void* kI, const void* kI_scales, int64_t n_entries, int64_t entry0,
                     const int64_t* q_pos, float* cand_scores, int32_t* cand_ids, void* workspace,
                     size_t ws_bytes, csa_stream_t stream) {
    int st = check_params(p, true, false);
    if (st) return st;
    if (batch < 0 || n_entries < 0 || entry0 < 0 || entry0 + n_entries > INT32_MAX) return CSA_ERR_ARG;
    if (batch == 0) return CSA_OK;
    if (!q_pos || !cand_scores || !cand_ids || !workspace) return CSA_ERR_ARG;
    if (ws_bytes < csa_workspace_size(p, CSA_OP_SHARD_SELECT, batch, 1, n_entries)) return CSA_ERR_WORKSPACE;
    if (!aligned16(workspace) || !aligned16(cand_scores) || !aligned16(cand_ids)) return CSA_ERR_ALIGN;
    const cudaStream_t s = (cudaStream_t)stream;
    const int64_t ld = std::max<int64_t>(n_entries, 1);
    int64_t* q_local = (int64_t*)workspace;
    float* scores = (float*)((char*)workspace + (((size_t(batch) * 8) + 255) & ~size_t(255)));
    int32_t* sel = (int32_t*)((char*)scores + (((size_t(batch) * ld * 4) + 255) & ~size_t(255)));
    // the shard's eligible entries are those with entry0 + j < n_elig(t):
    // the count n_elig seen at t - entry0 * m
    st = cuda_status(launch_shift_positions(q_pos, q_local, batch, entry0 * int64_t(p->m), s));
    if (st) return st;
    if (n_entries > 0) {
        st = indexer_score(p, batch, 1, qI, qI_scales, w, kI, kI_scales, n_entries, q_local, scores, ld, stream);
        if (st) return st;
    }
    if (n_entries > 0) {
        st = topk_impl(p, batch, 1, scores, ld, n_entries, q_local, sel, stream, false);
        if (st) return st;
    }
    return cuda_status(launch_shard_candidates(batch, p->top_k, scores, ld, n_entries > 0 ? sel : nullptr, entry0,
                                               cand_scores, cand_ids, s));
}

int csa_shard_attend(const csa_params* p, int32_t batch, const void* q, int32_t n_parts, const float* cand_scores,
                     const int32_t* cand_ids, const void* kv, const void* kv_scales, int64_t n_entries,
                     int64_t entry0, const void* raw, int64_t n_raw, const int64_t* raw_pos0,
                     const int64_t* q_pos, float* part_o, float* part_ml, int32_t* idx_out, void* workspace,
                     size_t ws_bytes, csa_stream_t stream) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (p->top_k <= 0 || batch < 0 || n_parts <= 0 || n_entries < 0 || entry0 < 0) return CSA_ERR_ARG;
    if (batch == 0) return CSA_OK;
    if (n_parts > 64 || !topk_merge_supported(n_parts * p->top_k, p->top_k)) return CSA_ERR_UNSUPPORTED;
    if (!cand_scores || !cand_ids || !part_ml || !workspace) return CSA_ERR_ARG;
    st = check_attn_ptrs(q, kv, kv_scales, p->kv_fmt, raw, n_raw, raw_pos0, q_pos, part_o, n_entries > 0);
    if (st) return st;
    if (!aligned16(part_ml) || !aligned16(workspace)) return CSA_ERR_ALIGN;
    if (ws_bytes < csa_workspace_size(p, CSA_OP_SHARD_ATTEND, batch, 1, n_entries)) return CSA_ERR_WORKSPACE;
    const cudaStream_t s = (cudaStream_t)stream;
    const size_t sel_bytes = ((size_t(batch) * p->top_k * 4) + 255) & ~size_t(255);
    const size_t cnt_bytes = ((size_t(batch) * 4) + 255) & ~size_t(255);
    int32_t* sel_global = idx_out ? idx_out : (int32_t*)workspace;
    int32_t* sel_local = (int32_t*)((char*)workspace + sel_bytes);
    int32_t* n_local = (int32_t*)((char*)workspace + 2 * sel_bytes);
    char* rest = (char*)workspace + 2 * sel_bytes + cnt_bytes;
    const size_t rest_bytes = ws_bytes - 2 * sel_bytes - cnt_bytes;
    // the merge's scratch and the attention's split partials share the space
    // after the selections (the merge is done before the attention starts)
    st = cuda_status(launch_topk_merge(batch, n_parts, p->top_k, cand_scores, cand_ids, entry0, n_entries,
                                       sel_global, sel_local, n_local, rest, p->m, p->window, s));
    if (st) return st;
    // the local selection is compacted: the attention visits only its n_local slots
    return run_attn(p, batch, 1, q, kv, kv_scales, n_entries, sel_local, raw, n_raw, raw_pos0, q_pos, nullptr,
                    part_o, rest, rest_bytes, int64_t(p->top_k) + p->window, s, false, (float2*)part_ml, 0,
                    n_local);
}

int hca_shard_attend(const csa_params* p, int32_t batch, const void* q, const void* kv, const void* kv_scales,
                     int64_t n_entries, int64_t entry0, const void* raw, int64_t n_raw,
                     const int64_t* raw_pos0, const int64_t* q_pos, float* part_o, float* part_ml,
                     void* workspace, size_t ws_bytes, csa_stream_t stream) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (batch < 0 || n_entries < 0 || entry0 < 0) return CSA_ERR_ARG;
    if (batch == 0) return CSA_OK;
    if (!part_ml) return CSA_ERR_ARG;
    st = check_attn_ptrs(q, kv, kv_scales, p->kv_fmt, raw, n_raw, raw_pos0, q_pos, part_o, n_entries > 0);
    if (st) return st;
    if (!aligned16(part_ml)) return CSA_ERR_ALIGN;
    if (ws_bytes < csa_workspace_size(p, CSA_OP_HCA_SHARD, batch, 1, n_entries)) return CSA_ERR_WORKSPACE;
    return run_attn(p, batch, 1, q, kv, kv_scales, n_entries, nullptr, raw, n_raw, raw_pos0, q_pos, nullptr,
                    part_o, workspace, ws_bytes, n_entries + p->window, (cudaStream_t)stream, false,
                    (float2*)part_ml, entry0);
}

int attn_merge(const csa_params* p, int32_t batch, int32_t n_parts, const float* part_o, const float* part_ml,
               const float* sinks, void* out, csa_stream_t stream) {
    int st = check_params(p, false, true);
    if (st) return st;
    if (batch < 0 || n_parts <= 0) return CSA_ERR_ARG;
    if (n_parts > 64) return CSA_ERR_UNSUPPORTED;
    if (batch == 0) return CSA_OK;
    if (!part_o || !part_ml || !out) return CSA_ERR_ARG;
    if (!aligned16(part_o) || !aligned16(part_ml) || !aligned16(out)) return CSA_ERR_ALIGN;
    if ((p->head_dim % 4) != 0) return CSA_ERR_UNSUPPORTED;
    return cuda_status(launch_combine_strided(p->act_fmt, false, p->n_heads, p->head_dim, n_parts, batch, 1, batch,
                                              part_o, (const float2*)part_ml, sinks, out, nullptr,
                                              (cudaStream_t)stream));
}

}  // extern "C"
