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

constexpr int kMergeCap = 16384;   // candidates per row
constexpr int kMapThreads = 1024;  // one CTA per row in the id mapping

__global__ void gather_candidates_kernel(int64_t rows, int n_parts, int k, const float* __restrict__ cand_scores,
                                         float* __restrict__ row_scores, int64_t* __restrict__ pos, int m, int W) {
    const int64_t n = int64_t(n_parts) * k;
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < rows * n) {
        const int64_t r = i / n, c = i - r * n;
        row_scores[i] = cand_scores[((c / k) * rows + r) * k + c % k];
    }
    // the position whose eligible count is exactly the n candidates
    if (i < rows) pos[i] = W + int64_t(m) * n;
}

// Exclusive prefix sum over the CTA (kMapThreads threads) of one value per
// thread; returns this thread's offset and the total in *total.
__device__ __forceinline__ int block_excl_scan(int v, int* total) {
    __shared__ int warp_sum[kMapThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = lane < kMapThreads / 32 ? warp_sum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sum[lane] = w;  // inclusive prefix of the warp totals
    }
    __syncthreads();
    const int before = (wid ? warp_sum[wid - 1] : 0) + x - v;
    *total = warp_sum[kMapThreads / 32 - 1];
    __syncthreads();  // warp_sum is reused by the next call
    return before;
}

// Row r: the selected candidate positions (ascending) -> their global ids.
// Positions ascend in (rank, slot) order, ranks hold increasing entry ranges
// and each rank's candidates are in ascending id order, so the valid ids come
// out ascending; empty candidates (-1) are dropped.
__global__ void __launch_bounds__(kMapThreads) map_selection_kernel(
    int64_t rows, int n_parts, int k, const int32_t* __restrict__ sel_pos, const int32_t* __restrict__ cand_ids,
    int64_t entry0, int64_t n_entries, int32_t* __restrict__ sel_global, int32_t* __restrict__ sel_local,
    int32_t* __restrict__ n_local) {
    const int64_t r = blockIdx.x;
    const int per = (k + kMapThreads - 1) / kMapThreads;  // consecutive slots per thread (<= 4)
    const int i0 = threadIdx.x * per;
    int32_t id[4];
    int n_valid = 0, n_in = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        id[u] = -1;
        if (u < per && i0 + u < k) {
            const int32_t p = sel_pos[r * k + i0 + u];
            if (p >= 0) id[u] = cand_ids[(int64_t(p / k) * rows + r) * k + p % k];
        }
        n_valid += id[u] >= 0;
        n_in += id[u] >= entry0 && id[u] < entry0 + n_entries;
    }
    int tot_valid, tot_in;
    int og = block_excl_scan(n_valid, &tot_valid);
    int ol = block_excl_scan(n_in, &tot_in);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (id[u] < 0) continue;
        sel_global[r * k + og++] = id[u];
        if (id[u] >= entry0 && id[u] < entry0 + n_entries) sel_local[r * k + ol++] = int32_t(id[u] - entry0);
    }
    for (int i = tot_valid + threadIdx.x; i < k; i += kMapThreads) sel_global[r * k + i] = -1;
    for (int i = tot_in + threadIdx.x; i < k; i += kMapThreads) sel_local[r * k + i] = -1;
    if (threadIdx.x == 0) n_local[r] = tot_in;
}

}  // namespace

bool topk_merge_supported(int n_cand, int k) { return n_cand > 0 && n_cand <= kMergeCap && k <= 4 * kMapThreads; }

size_t topk_merge_workspace(int64_t rows, int k) {
    const size_t sc = (size_t(rows) * kMergeCap * 4 + 255) & ~size_t(255);
    const size_t ps = (size_t(rows) * 8 + 255) & ~size_t(255);
    const size_t sp = (size_t(rows) * k * 4 + 255) & ~size_t(255);
    return sc + ps + sp;
}

cudaError_t launch_topk_merge(int64_t rows, int n_parts, int k, const float* cand_scores, const int32_t* cand_ids,
                              int64_t entry0, int64_t n_entries, int32_t* sel_global, int32_t* sel_local,
                              int32_t* n_local, void* ws, int m, int W, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int n_cand = n_parts * k;
    if (!topk_merge_supported(n_cand, k)) return cudaErrorInvalidValue;
    // the candidates of a row side by side: the top-k over positions, ties
    // to the lower position, is the top-k by score then id
    float* row_scores = (float*)ws;
    int64_t* pos = (int64_t*)((char*)ws + ((size_t(rows) * kMergeCap * 4 + 255) & ~size_t(255)));
    int32_t* sel_pos = (int32_t*)((char*)pos + ((size_t(rows) * 8 + 255) & ~size_t(255)));
    const int64_t n = rows * n_cand;
    gather_candidates_kernel<<<unsigned(ceil_div(std::max<int64_t>(n, rows), 256)), 256, 0, s>>>(
        rows, n_parts, k, cand_scores, row_scores, pos, m, W);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_topk(row_scores, n_cand, n_cand, pos, m, W, k, rows, sel_pos, s);
    if (e != cudaSuccess) return e;
    map_selection_kernel<<<unsigned(rows), kMapThreads, 0, s>>>(rows, n_parts, k, sel_pos, cand_ids, entry0,
                                                                n_entries, sel_global, sel_local, n_local);
    return cudaGetLastError();
}

}  // namespace csa
