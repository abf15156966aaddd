// Sharded decode of one long sequence: its pooled entries are split along the
// entry axis over ranks ("DeepSeek-V4 發佈說明", section 架構實現 and the
// paper summary's 1M-token context: a CSA layer selects the top-k of all
// visible entries; an HCA layer attends to all of them).  A rank holds the
// contiguous entries [entry0, entry0 + n).  Because the global top-k under the
// order (score descending, id ascending) is contained in the union of the
// shards' local top-k under the same order, one exchange of k candidates per
// rank gives the exact global selection; the attention over a rank's selected
// entries is then one split of the same softmax, merged with the others (and
// the sink) by the LSE combine.
#include "kernels.h"

namespace csa {

__global__ void shift_positions_kernel(const int64_t* __restrict__ q_pos, int64_t* __restrict__ q_local,
                                       int64_t n, int64_t delta) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) q_local[i] = q_pos[i] - delta;
}

cudaError_t launch_shift_positions(const int64_t* q_pos, int64_t* q_local, int64_t n, int64_t delta,
                                   cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    shift_positions_kernel<<<unsigned(ceil_div(n, 256)), 256, 0, s>>>(q_pos, q_local, n, delta);
    return cudaGetLastError();
}

__global__ void shard_candidates_kernel(int64_t rows, int k, const float* __restrict__ scores, int64_t ld,
                                        const int32_t* __restrict__ sel, int64_t entry0,
                                        float* __restrict__ cand_scores, int32_t* __restrict__ cand_ids) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= rows * k) return;
    const int64_t r = i / k;
    const int32_t j = sel ? sel[i] : -1;  // no selection: an empty shard
    cand_scores[i] = j >= 0 ? scores[r * ld + j] : -INFINITY;
    cand_ids[i] = j >= 0 ? int32_t(entry0 + j) : -1;
}

cudaError_t launch_shard_candidates(int64_t rows, int k, const float* scores, int64_t ld, const int32_t* sel,
                                    int64_t entry0, float* cand_scores, int32_t* cand_ids, cudaStream_t s) {
    const int64_t n = rows * k;
    if (n == 0) return cudaSuccess;
    shard_candidates_kernel<<<unsigned(ceil_div(n, 256)), 256, 0, s>>>(rows, k, scores, ld, sel, entry0,
                                                                       cand_scores, cand_ids);
    return cudaGetLastError();
}

namespace {

constexpr int kMergeThreads = 1024;
constexpr int kMergeCap = 16384;  // candidates per row (128 KB of 64-bit keys)

// Order-preserving map of an fp32 score to 32 bits (larger score, larger key).
__device__ __forceinline__ uint32_t mono(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// In-place bitonic sort, descending, of n (a power of two) 64-bit keys.
__device__ void bitonic_desc(uint64_t* key, int n) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));  // first of the pair
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t a = key[lo], b = key[hi];
                if ((a < b) == desc) { key[lo] = b; key[hi] = a; }
            }
        }
    }
    __syncthreads();
}

}  // namespace

// One CTA per row.  Valid candidates are keyed (mono(score) << 32) | ~id, so a
// larger key is a higher score or, for equal scores, a smaller id; empty slots
// are key 0, below every valid key (mono of any score is >= 0x007FFFFF).
__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(
    int n_parts, int k, int64_t rows, const float* __restrict__ cand_scores, const int32_t* __restrict__ cand_ids,
    int64_t entry0, int64_t n_entries, int32_t* __restrict__ sel_global, int32_t* __restrict__ sel_local) {
    extern __shared__ uint64_t key[];
    __shared__ int lo_cnt, hi_cnt;
    const int64_t r = blockIdx.x;
    const int n_cand = n_parts * k;
    int n = 1;
    while (n < n_cand) n <<= 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        uint64_t v = 0;
        if (i < n_cand) {
            const int64_t src = (int64_t(i / k) * rows + r) * k + i % k;
            const int32_t id = cand_ids[src];
            if (id >= 0) v = (uint64_t(mono(cand_scores[src])) << 32) | uint64_t(~uint32_t(id));
        }
        key[i] = v;
    }
    if (threadIdx.x == 0) { lo_cnt = 0; hi_cnt = 0; }
    bitonic_desc(key, n);
    // the first k keys are the selection; re-key them by id (ascending) and
    // sort again: a valid entry becomes ~id (descending order = ascending
    // id), an empty one 0 (last)
    const int kk = min(k, n);
    int n2 = 1;
    while (n2 < kk) n2 <<= 1;
    uint64_t* ids = key + n;  // scratch after the candidates (n2 <= n)
    for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        uint64_t v = 0;
        if (i < kk && key[i] != 0) v = uint64_t(uint32_t(key[i]));  // ~id: a larger key is a smaller id
        ids[i] = v;
    }
    bitonic_desc(ids, n2);
    // ascending ids; count those below entry0 and below entry0 + n_entries
    int below_lo = 0, below_hi = 0;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const bool valid = i < kk && ids[i] != 0;
        const int64_t id = valid ? int64_t(0xFFFFFFFFu - uint32_t(ids[i])) : -1;
        sel_global[r * k + i] = int32_t(id);
        if (valid && id < entry0) ++below_lo;
        if (valid && id < entry0 + n_entries) ++below_hi;
    }
    atomicAdd(&lo_cnt, below_lo);
    atomicAdd(&hi_cnt, below_hi);
    __syncthreads();
    const int a = lo_cnt, b = hi_cnt;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const int src = a + i;
        sel_local[r * k + i] = src < b ? int32_t((0xFFFFFFFFu - uint32_t(ids[src])) - entry0) : -1;
    }
}

bool topk_merge_supported(int n_cand) { return n_cand > 0 && n_cand <= kMergeCap; }
// (k <= 4096 keeps the candidates and the re-keyed selection within 160 KB)

cudaError_t launch_topk_merge(int64_t rows, int n_parts, int k, const float* cand_scores, const int32_t* cand_ids,
                              int64_t entry0, int64_t n_entries, int32_t* sel_global, int32_t* sel_local,
                              cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int n_cand = n_parts * k;
    if (!topk_merge_supported(n_cand)) return cudaErrorInvalidValue;
    int n = 1;
    while (n < n_cand) n <<= 1;
    int n2 = 1;
    while (n2 < std::min(k, n)) n2 <<= 1;
    const size_t sm = size_t(n + n2) * sizeof(uint64_t);
    cudaError_t e = ensure_smem(topk_merge_kernel, sm);
    if (e != cudaSuccess) return e;
    topk_merge_kernel<<<unsigned(rows), kMergeThreads, sm, s>>>(n_parts, k, rows, cand_scores, cand_ids, entry0,
                                                                n_entries, sel_global, sel_local);
    return cudaGetLastError();
}

}  // namespace csa
