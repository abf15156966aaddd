// Host-side launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include "common.cuh"

namespace csa {

// Arguments of the attention kernels (sparse CSA and dense HCA).
struct AttnArgs {
    int H, D, m, W, k;
    float scale;
    const void* q;          // [rows][H][D] act format
    const void* kv;         // [batch][max_entries][D] kv format
    const void* kv_s;       // scales of kv (FP8_S64) or null
    int kv_fmt;             // stored format of kv
    int64_t max_entries;
    const int32_t* idx;     // [rows][k] selected ids, or null for dense (HCA)
    const void* raw;        // [batch][n_raw][D] act format
    int64_t n_raw;
    const int64_t* raw_pos0;  // [batch]
    const int64_t* q_pos;     // [rows]
    const float* sinks;       // [H] or null
    int n_q;                  // queries per sequence (row = b * n_q + i)
    int n_splits;
    void* out;                // final output when n_splits == 1
    float* part_o;            // [rows][n_splits][H][D]
    float2* part_ml;          // [rows][n_splits][H] (running max, running sum)
    int fused_combine;        // tensor-core kernel: the splits of a row form a cluster and
                              // combine through distributed shared memory (set by the launcher)
    int64_t row_base;         // tensor-core kernel: first row of this launch (set by the launcher)
    int partial_out;          // write (m, l, O) partials even with one split; no sink applied
    int64_t kv_base;          // global index of entry 0 of kv (a shard); dense rows attend to
                              // entries j with kv_base + j < n_elig(t)
    const int32_t* n_sel;     // [rows] or null: row r's selection is compacted, only its first
                              // n_sel[r] slots can hold ids (the slots after them are -1)
};

cudaError_t launch_compress(int in_fmt, int out_fmt, const void* x, const void* z,
                            const float* bias, int64_t n_tokens, int m, int d, void* out,
                            void* out_scales, cudaStream_t s);
cudaError_t launch_quantize(int out_fmt, const float* src, int64_t rows, int d, void* out,
                            void* out_scales, cudaStream_t s);
cudaError_t launch_indexer_simt(int fmt, int HI, int dI, int m, int W, const void* qI,
                                const void* qI_s, const float* w, const void* kI,
                                const void* kI_s, int64_t max_blocks, const int64_t* q_pos,
                                int batch, int n_q, int64_t max_elig, float* scores, int64_t ld,
                                cudaStream_t s);
bool indexer_tc_supported(int fmt, int HI, int dI, int64_t max_blocks, int64_t batch, int64_t rows);
cudaError_t launch_indexer_tc(const void* qI, const void* qI_s, const float* w, const void* kI,
                              const void* kI_s, int64_t max_blocks, const int64_t* q_pos,
                              int batch, int n_q, int m, int W, float* scores, int64_t ld,
                              bool q_bf16, bool fp8, cudaStream_t s);
bool indexer_bf16_tc_supported(int fmt, int HI, int dI, int64_t max_blocks, int64_t batch, int n_q);
cudaError_t launch_indexer_bf16_tc(const void* qI, const float* w, const void* kI, int64_t max_blocks,
                                   const int64_t* q_pos, int batch, int n_q, int m, int W,
                                   float* scores, int64_t ld, cudaStream_t s);
// pdl: launched as a programmatic dependent of the previous kernel (which
// wrote `scores`); only set when that kernel is known.
cudaError_t launch_topk(const float* scores, int64_t ld, int64_t max_blocks, const int64_t* q_pos,
                        int m, int W, int k, int64_t rows, int32_t* idx, cudaStream_t s,
                        bool pdl = false);
bool attn_tc_supported(int act, int kvf, int H, int D);
bool attn_tc_rows_fit(int64_t max_entries, int64_t n_raw);
// Sets *combined when the splits were combined inside the kernel (no
// launch_combine needed).
// pdl: launched as a programmatic dependent of the kernel that wrote a.idx
// (the query, entries and window are read before waiting for it).
cudaError_t launch_attn_tc(const AttnArgs& a, int64_t rows, cudaStream_t s, bool* combined,
                           bool pdl = false);
cudaError_t launch_attn_simt(int act, int kvf, const AttnArgs& a, int64_t rows, cudaStream_t s);
bool attn_simt_supported(int act, int kvf, int H, int D);
cudaError_t launch_combine(int act, int H, int D, int n_splits, int64_t rows, const float* part_o,
                           const float2* part_ml, const float* sinks, void* out, cudaStream_t s,
                           bool pdl = false);
// The same with explicit strides (partial s of row r is item r * row_stride +
// s * split_stride); partial = true writes the merged (M, L) and fp32 O
// without a sink instead of the normalised output.
cudaError_t launch_combine_strided(int act, bool partial, int H, int D, int n_splits, int64_t rows,
                                   int64_t row_stride, int64_t split_stride, const float* part_o,
                                   const float2* part_ml, const float* sinks, void* out, float2* out_ml,
                                   cudaStream_t s, bool pdl = false);

// Sharded decode helpers (k_shard.cu).
// q_local[i] = q_pos[i] - delta: a shard whose first entry is entry0 sees the
// eligible count n_elig(t) - entry0 at position t - entry0 * m.
cudaError_t launch_shift_positions(const int64_t* q_pos, int64_t* q_local, int64_t n, int64_t delta,
                                   cudaStream_t s);
// The shard's local top-k as candidates: (score, entry0 + local id), or
// (-inf, -1) for an empty slot.
cudaError_t launch_shard_candidates(int64_t rows, int k, const float* scores, int64_t ld, const int32_t* sel,
                                    int64_t entry0, float* cand_scores, int32_t* cand_ids, cudaStream_t s);
// Global top-k of each row's candidates (gathered rank-major: [n_parts][rows][k]),
// ranked by score and then by the smaller id; writes the selection as
// ascending global ids (-1 padded) and the part in [entry0, entry0 + n_entries)
// as ascending local ids (-1 padded).
// ws: topk_merge_workspace(rows, k) bytes (candidate rows, positions, the
// selected positions); m, W: the layer's, for the eligibility rule the top-k
// kernels apply.
bool topk_merge_supported(int n_cand, int k);
size_t topk_merge_workspace(int64_t rows, int k);
cudaError_t launch_topk_merge(int64_t rows, int n_parts, int k, const float* cand_scores, const int32_t* cand_ids,
                              int64_t entry0, int64_t n_entries, int32_t* sel_global, int32_t* sel_local,
                              int32_t* n_local, void* ws, int m, int W, cudaStream_t s);

}  // namespace csa
