// Top-k block selection ("DeepSeek V4" wiki summary, section 架构创新: the
// lightning indexer makes a top-k sparse selection of pooled entries).
//
// Radix select on the order-preserving 32-bit image of each fp32 score: three
// histogram passes over 11, 11 and 10 bits find the exact k-th largest key
// T and how many elements equal to T are needed; a final pass writes every
// element above T and the first needed elements equal to T, in ascending
// index order, so ties resolve to the lower index.  -0.0 is folded into +0.0
// before ranking.  One 1024-thread CTA per query row; rows are read from
// global memory (an L2-resident score row in the decode path).
#include <cooperative_groups.h>

#include "kernels.h"

namespace csa {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide scan of two ints over NT threads (a multiple of 32,
// at most 1024).
template <int NT = kTopkThreads>
__device__ __forceinline__ int2 block_scan2(int2 v, int2* warp_tot) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ax = __shfl_up_sync(0xffffffffu, v.x, o);
        const int ay = __shfl_up_sync(0xffffffffu, v.y, o);
        if (lane >= o) { v.x += ax; v.y += ay; }
    }
    if (lane == 31) warp_tot[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int2 t = lane < NT / 32 ? warp_tot[lane] : make_int2(0, 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ax = __shfl_up_sync(0xffffffffu, t.x, o);
            const int ay = __shfl_up_sync(0xffffffffu, t.y, o);
            if (lane >= o) { t.x += ax; t.y += ay; }
        }
        if (lane < NT / 32) warp_tot[lane] = t;
    }
    __syncthreads();
    if (wid > 0) { v.x += warp_tot[wid - 1].x; v.y += warp_tot[wid - 1].y; }
    __syncthreads();
    return v;
}

// Output pass shared by both kernels: every key above T is taken, plus the
// first `remaining` keys equal to T in index order; ids are written in
// ascending order.  Warp w owns a contiguous segment of the row and walks it
// 32 consecutive keys at a time (coalesced / bank-conflict free), compacting
// with ballots; a block scan of the per-warp counts gives each warp its
// output offset and its number of earlier equal keys.
template <typename KeyAt>
__device__ __forceinline__ void write_selection_impl(KeyAt key_at, int64_t n, uint32_t T, int remaining,
                                                     int k, int32_t* out, int2* warp_tot) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    constexpr int kWarps = kTopkThreads / 32;
    const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int64_t lo = min(n, wid * seg), hi = min(n, lo + seg);
    int gt = 0, eq = 0;
    for (int64_t base = lo; base < hi; base += 32) {
        const int64_t i = base + lane;
        const uint32_t u = i < hi ? key_at(i) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < hi && u > T));
        eq += __popc(__ballot_sync(0xffffffffu, i < hi && u == T));
    }
    // exclusive scan over warps (lane 0 of each warp contributes)
    const int2 inc = block_scan2(make_int2(lane == 0 ? gt : 0, lane == 0 ? eq : 0), warp_tot);
    // block_scan2 is inclusive over threads; lane 0's value is the warp's inclusive total
    const int gt_incl = __shfl_sync(0xffffffffu, inc.x, 0), eq_incl = __shfl_sync(0xffffffffu, inc.y, 0);
    int eq_before = eq_incl - eq;
    int pos = (gt_incl - gt) + min(eq_before, remaining);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t base = lo; base < hi; base += 32) {
        const int64_t i = base + lane;
        const uint32_t u = i < hi ? key_at(i) : 0u;
        const bool is_eq = i < hi && u == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
        const int my_eq_rank = eq_before + __popc(eqm & lt_mask);
        const bool take = i < hi && (u > T || (is_eq && my_eq_rank < remaining));
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        if (take) {
            const int p = pos + __popc(tm & lt_mask);
            if (p < k) out[p] = int32_t(i);
        }
        pos += __popc(tm);
        eq_before += __popc(eqm);
    }
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t max_blocks,
    const int64_t* __restrict__ q_pos, int m, int W, int k, int32_t* __restrict__ idx) {
    __shared__ int hist[2048];
    __shared__ int2 warp_tot[32];
    __shared__ int found_digit, found_above;
    pdl_wait();  // the scores come from the kernel before this one
    pdl_launch_dependents();
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const float* s = scores + row * ld;
    int32_t* out = idx + row * k;
    const int64_t n = min(n_elig(q_pos[row], m, W), max_blocks);

    if (n <= k) {
        for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
        return;
    }
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nbins = pass < 2 ? 2048 : 1024;
        for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int64_t i = tid; i < n; i += kTopkThreads) {
            const uint32_t u = order_key(s[i]);
            if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & (nbins - 1)], 1);
        }
        __syncthreads();
        // thread t owns bins b0 = nbins-1-2t and b1 = b0-1 (counted from the top)
        const int b0 = nbins - 1 - 2 * tid, b1 = b0 - 1;
        const int h0 = b0 >= 0 ? hist[b0] : 0, h1 = b1 >= 0 ? hist[b1] : 0;
        const int2 inc = block_scan2(make_int2(h0 + h1, 0), warp_tot);
        const int above = inc.x - (h0 + h1);  // elements in bins > b0
        if (b0 >= 0 && above < remaining && remaining <= above + h0) {
            found_digit = b0;
            found_above = above;
        } else if (b1 >= 0 && above + h0 < remaining && remaining <= above + h0 + h1) {
            found_digit = b1;
            found_above = above + h0;
        }
        __syncthreads();
        remaining -= found_above;
        prefix |= uint32_t(found_digit) << shift;
        pmask |= uint32_t(nbins - 1) << shift;
        __syncthreads();
    }
    // prefix is now the k-th largest key; `remaining` elements equal to it are taken.
    write_selection_impl([&](int64_t i) { return order_key(s[i]); }, n, prefix, remaining, k, out, warp_tot);
}

// Rows that fit in shared memory: the row is read once into shared memory as
// order keys; four passes of 8-bit digits find the k-th largest key.  Pass 0
// sees every element: each warp counts into its own 256-bin histogram, and
// lanes holding the same digit are merged with __match_any_sync so that one
// leader adds their count (N(0, s) scores put most elements into a few
// exponent bins, which would otherwise serialise the shared atomics).
// Passes 1-3 only count the elements that still match the selected prefix.
constexpr int kTopkSmemMax = 45056;  // keys kept in shared memory (176 KB)

__global__ void __launch_bounds__(kTopkThreads) topk_smem_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t max_blocks,
    const int64_t* __restrict__ q_pos, int m, int W, int k, int32_t* __restrict__ idx) {
    extern __shared__ uint32_t keys[];                 // [n]
    __shared__ int whist[32][256];
    __shared__ int2 warp_tot[32];
    __shared__ int found_digit, found_above;
    pdl_wait();  // the scores come from the kernel before this one
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const float* s = scores + row * ld;
    int32_t* out = idx + row * k;
    const int n = int(min(n_elig(q_pos[row], m, W), max_blocks));
    if (n <= k) {
        for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
        return;
    }
    // fill: batches of 8 independent loads per thread so their latencies overlap
    for (int base = 0; base < n; base += 8 * kTopkThreads) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * kTopkThreads + tid;
            v[j] = i < n ? s[i] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * kTopkThreads + tid;
            if (i < n) keys[i] = order_key(v[j]);
        }
    }
    for (int i = tid; i < 32 * 256; i += kTopkThreads) (&whist[0][0])[i] = 0;
    __syncthreads();
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (pass == 0) {
            for (int base = 0; base < n; base += kTopkThreads) {   // whole warps iterate together
                const int i = base + tid;
                const bool in = i < n;
                const uint32_t dg = in ? (keys[i] >> 24) : 0xFFFFFFFFu;
                const unsigned same = __match_any_sync(0xffffffffu, dg);
                if (in && lane == __ffs(same) - 1) whist[wid][dg] += __popc(same);
            }
            __syncthreads();
            if (tid < 256) {
                int c = 0;
                for (int w = 0; w < 32; ++w) c += whist[w][tid];
                whist[0][tid] = c;
            }
        } else {
            for (int i = tid; i < n; i += kTopkThreads) {
                const uint32_t u = keys[i];
                if ((u & pmask) == prefix) atomicAdd(&whist[0][(u >> shift) & 255], 1);
            }
        }
        __syncthreads();
        if (wid == 0) {
            // lane l owns the 8 bins counted from the top: 255-8l .. 248-8l
            int loc[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { loc[j] = whist[0][255 - 8 * lane - j]; sum += loc[j]; }
            int inc = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            int above = inc - sum;
            if (above < remaining && remaining <= inc) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (above < remaining && remaining <= above + loc[j]) {
                        found_digit = 255 - 8 * lane - j;
                        found_above = above;
                    }
                    above += loc[j];
                }
            }
        }
        __syncthreads();
        remaining -= found_above;
        prefix |= uint32_t(found_digit) << shift;
        pmask |= 0xFFu << shift;
        if (tid < 256) whist[0][tid] = 0;
        __syncthreads();
    }
    write_selection_impl([&](int64_t i) { return keys[i]; }, int64_t(n), prefix, remaining, k, out, warp_tot);
}

// Few rows (decode): one thread-block cluster of kClu CTAs per row (rows of
// up to 8 x 512 x 72 = 294,912 scores).  CTA r holds keys
// [r * E * 512, (r + 1) * E * 512) of the row in registers
// (thread t, slot j: key r * E * 512 + j * 512 + t, so ascending index order
// is slot-major).  Four 8-bit digit passes as above, except that each CTA
// counts its own keys and every CTA then sums all kClu histograms through
// distributed shared memory, so all of them pick the same digit; histograms
// are double-buffered, so one cluster barrier per pass suffices (a buffer is
// cleared only after every CTA has passed the barrier that follows its last
// remote read).  The output offsets of each CTA (keys above T and keys equal
// to T in lower CTAs) are exchanged the same way.
namespace cg = cooperative_groups;
constexpr int kClu = 8;
constexpr int kCluThreads = 512;
constexpr int kCluWarps = kCluThreads / 32;

template <int E>
__global__ void __cluster_dims__(kClu, 1, 1) __launch_bounds__(kCluThreads)
    topk_cluster_kernel(const float* __restrict__ scores, int64_t ld, int64_t max_blocks,
                        const int64_t* __restrict__ q_pos, int m, int W, int k,
                        int32_t* __restrict__ idx) {
    __shared__ int hist[2][256];
    __shared__ int2 warp_tot[32];
    __shared__ int2 cnt[E * kCluWarps];   // per (slot, warp): (keys above T, keys equal to T)
    __shared__ int2 cta_tot;
    __shared__ int found_digit, found_above;
    cg::cluster_group cluster = cg::this_cluster();
    pdl_wait();  // the scores come from the kernel before this one
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int r = int(cluster.block_rank());
    const int64_t row = blockIdx.x / kClu;
    const float* s = scores + row * ld;
    int32_t* out = idx + row * k;
    const int n = int(min(n_elig(q_pos[row], m, W), max_blocks));
    const int base = r * E * kCluThreads;
    if (n <= k) {  // every eligible block is selected (uniform over the cluster)
        for (int i = base + tid; i < min(k, base + E * kCluThreads); i += kCluThreads)
            out[i] = i < n ? i : -1;
        return;
    }
    uint32_t key[E];
#pragma unroll
    for (int j = 0; j < E; ++j) {
        const int i = base + j * kCluThreads + tid;
        key[j] = i < n ? order_key(s[i]) : 0u;
    }
    if (tid < 256) { hist[0][tid] = 0; hist[1][tid] = 0; }
    __syncthreads();
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        int* H = hist[pass & 1];
        // lanes holding the same digit are merged so that one leader adds
        // their count (most N(0, s) scores share a few top digits)
#pragma unroll
        for (int j = 0; j < E; ++j) {
            const int i = base + j * kCluThreads + tid;
            const bool in = i < n && (key[j] & pmask) == prefix;
            const uint32_t dg = in ? ((key[j] >> shift) & 255u) : 0xFFFFFFFFu;
            const unsigned same = __match_any_sync(0xffffffffu, dg);
            if (in && lane == __ffs(same) - 1) atomicAdd(&H[dg], __popc(same));
        }
        cluster.sync();
        // thread t < 256 owns bin 255 - t (bins counted from the top)
        int c = 0;
        if (tid < 256) {
#pragma unroll
            for (int q = 0; q < kClu; ++q) c += cluster.map_shared_rank(H, q)[255 - tid];
            hist[(pass + 1) & 1][tid] = 0;  // its last remote reads were before this barrier
        }
        const int2 inc = block_scan2<kCluThreads>(make_int2(c, 0), warp_tot);
        const int above = inc.x - c;
        if (tid < 256 && above < remaining && remaining <= inc.x) {
            found_digit = 255 - tid;
            found_above = above;
        }
        __syncthreads();
        remaining -= found_above;
        prefix |= uint32_t(found_digit) << shift;
        pmask |= 0xFFu << shift;
    }
    // prefix is the k-th largest key T; the first `remaining` keys equal to T
    // (in index order) are taken with every key above T.
    const uint32_t T = prefix;
    const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < E; ++j) {
        const int i = base + j * kCluThreads + tid;
        const unsigned gm = __ballot_sync(0xffffffffu, i < n && key[j] > T);
        const unsigned em = __ballot_sync(0xffffffffu, i < n && key[j] == T);
        if (lane == 0) cnt[j * kCluWarps + wid] = make_int2(__popc(gm), __popc(em));
    }
    __syncthreads();
    // exclusive offsets of every (slot, warp) in index order, and the CTA
    // total; thread t scans the R consecutive entries [t R, t R + R)
    constexpr int kEntries = E * kCluWarps, R = (kEntries + kCluThreads - 1) / kCluThreads;
    int2 mine[R], sum = make_int2(0, 0);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int e = tid * R + i;
        mine[i] = e < kEntries ? cnt[e] : make_int2(0, 0);
        sum.x += mine[i].x;
        sum.y += mine[i].y;
    }
    const int2 vi = block_scan2<kCluThreads>(sum, warp_tot);
    int2 run = make_int2(vi.x - sum.x, vi.y - sum.y);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int e = tid * R + i;
        if (e < kEntries) cnt[e] = run;
        run.x += mine[i].x;
        run.y += mine[i].y;
    }
    if (tid == kCluThreads - 1) cta_tot = vi;
    cluster.sync();
    int gt_base = 0, eq_base = 0;
    for (int q = 0; q < r; ++q) {
        const int2 t = *cluster.map_shared_rank(&cta_tot, q);
        gt_base += t.x;
        eq_base += t.y;
    }
#pragma unroll
    for (int j = 0; j < E; ++j) {
        const int i = base + j * kCluThreads + tid;
        const bool gt = i < n && key[j] > T, eq = i < n && key[j] == T;
        const unsigned gm = __ballot_sync(0xffffffffu, gt);
        const unsigned em = __ballot_sync(0xffffffffu, eq);
        const int2 off = cnt[j * kCluWarps + wid];
        const int gt_before = gt_base + off.x + __popc(gm & lt_mask);
        const int eq_before = eq_base + off.y + __popc(em & lt_mask);
        if (gt || (eq && eq_before < remaining)) {
            const int p = gt_before + min(eq_before, remaining);
            if (p < k) out[p] = int32_t(i);
        }
    }
    cluster.sync();  // keep this CTA's shared memory alive until every remote read is done
}

template <int E>
static cudaError_t launch_topk_cluster(const float* scores, int64_t ld, int64_t max_blocks,
                                       const int64_t* q_pos, int m, int W, int k, int64_t rows,
                                       int32_t* idx, cudaStream_t s, bool pdl) {
    return launch_ex(topk_cluster_kernel<E>, dim3(unsigned(rows * kClu)), dim3(kCluThreads), 0, s, pdl,
                     scores, ld, max_blocks, q_pos, m, W, k, idx);
}

cudaError_t launch_topk(const float* scores, int64_t ld, int64_t max_blocks, const int64_t* q_pos,
                        int m, int W, int k, int64_t rows, int32_t* idx, cudaStream_t s, bool pdl) {
    if (rows == 0) return cudaSuccess;
    // Few rows cannot fill the GPU with one CTA each: give each row a cluster.
    if (rows <= 2 * kNumSMs / kClu && k <= kClu * kCluThreads && max_blocks <= kClu * kCluThreads * 72) {
        const int64_t per = ceil_div(max_blocks, kClu * kCluThreads);
        if (per <= 2) return launch_topk_cluster<2>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (per <= 4) return launch_topk_cluster<4>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (per <= 8) return launch_topk_cluster<8>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (per <= 16) return launch_topk_cluster<16>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (per <= 32) return launch_topk_cluster<32>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        return launch_topk_cluster<72>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
    }
    if (max_blocks <= kTopkSmemMax) {
        const size_t sm = size_t(std::max<int64_t>(max_blocks, 1)) * 4;
        cudaError_t e = ensure_smem(topk_smem_kernel, size_t(sm));
        if (e != cudaSuccess) return e;
        return launch_ex(topk_smem_kernel, dim3(unsigned(rows)), dim3(kTopkThreads), sm, s, pdl, scores, ld,
                         max_blocks, q_pos, m, W, k, idx);
    }
    return launch_ex(topk_kernel, dim3(unsigned(rows)), dim3(kTopkThreads), 0, s, pdl, scores, ld,
                     max_blocks, q_pos, m, W, k, idx);
}

}  // namespace csa
