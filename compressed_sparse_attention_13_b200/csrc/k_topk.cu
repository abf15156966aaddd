// Top-k block selection ("DeepSeek V4" wiki summary, section 架构创新: the
// lightning indexer makes a top-k sparse selection of pooled entries).
//
// Every kernel here ranks the order-preserving 32-bit image of each fp32 score
// (-0.0 folded into +0.0), finds the exact k-th largest key T by radix passes
// and how many keys equal to T are taken, and writes the selected ids in
// ascending order, ties going to the lower index.  Many rows of up to 2,048
// scores (prefill chunks) take one warp per row; rows of up to 32,768 scores
// (decode at 128K context) take topk_sel_kernel, which narrows the row to a
// few times k candidates with a sampled threshold first; longer rows take a
// thread-block cluster per row (few rows) or one CTA per row reading the row
// from global memory (many rows).
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

// Many short rows (prefill chunks: up to 2,048 scores per row): one warp per
// row with the row in registers (lane l holds keys l + 32 i), so the four
// radix passes and the ordered output synchronise only the warp.  Each pass
// counts the keys that match the prefix so far into the warp's 256-bin
// shared histogram, lanes holding the same digit merged by __match_any_sync
// (N(0, s) scores share a few exponent digits); the output walks the row 32
// consecutive keys at a time, compacting with ballots.
constexpr int kWarpRowMax = 2048;
constexpr int kWarpRowThreads = 128;  // 4 rows per CTA

__global__ void __launch_bounds__(kWarpRowThreads, 6) topk_warp_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t max_blocks, const int64_t* __restrict__ q_pos, int m,
    int W, int k, int64_t rows, int32_t* __restrict__ idx) {
    constexpr int kPer = kWarpRowMax / 32;
    __shared__ int hist[kWarpRowThreads / 32][256];
    pdl_wait();  // the scores come from the kernel before this one
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int64_t row = int64_t(blockIdx.x) * (kWarpRowThreads / 32) + wl;
    if (row >= rows) return;  // whole warps leave together
    const float* s = scores + row * ld;
    int32_t* out = idx + row * k;
    const int n = int(min(n_elig(q_pos[row], m, W), max_blocks));
    if (n <= k) {
        for (int i = lane; i < k; i += 32) out[i] = i < n ? i : -1;
        return;
    }
    uint32_t key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = 32 * i + lane;
        key[i] = e < n ? order_key(s[e]) : 0u;
    }
    int* h = hist[wl];
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int j = lane; j < 256; j += 32) h[j] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            if (32 * i >= n) break;  // uniform across the warp
            const int e = 32 * i + lane;
            const bool in = e < n && (key[i] & pmask) == prefix;
            const uint32_t dg = in ? ((key[i] >> shift) & 255u) : 0xFFFFFFFFu;
            const unsigned same = __match_any_sync(0xffffffffu, dg);
            if (in && lane == __ffs(same) - 1) h[dg] += __popc(same);
        }
        __syncwarp();
        // lane l owns the 8 bins counted from the top: 255-8l .. 248-8l
        int loc[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { loc[j] = h[255 - 8 * lane - j]; sum += loc[j]; }
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        int above = inc - sum, fd = -1, fa = 0;
        if (above < remaining && remaining <= inc) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (above < remaining && remaining <= above + loc[j]) { fd = 255 - 8 * lane - j; fa = above; }
                above += loc[j];
            }
        }
        const int src = __ffs(__ballot_sync(0xffffffffu, fd >= 0)) - 1;
        fd = __shfl_sync(0xffffffffu, fd, src);
        fa = __shfl_sync(0xffffffffu, fa, src);
        remaining -= fa;
        prefix |= uint32_t(fd) << shift;
        pmask |= 0xFFu << shift;
        __syncwarp();
    }
    // every key above T = prefix, then the first `remaining` keys equal to T
    const unsigned lt = (1u << lane) - 1u;
    int pos = 0, eq_before = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        if (32 * i >= n) break;
        const int e = 32 * i + lane;
        const bool valid = e < n;
        const bool is_eq = valid && key[i] == prefix;
        const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
        const bool take = valid && (key[i] > prefix || (is_eq && eq_before + __popc(eqm & lt) < remaining));
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        if (take) out[pos + __popc(tm & lt)] = e;
        pos += __popc(tm);
        eq_before += __popc(eqm);
    }
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

// Rows of any length with a sampled threshold (topk_sel_kernel): a cluster of
// CPR CTAs per row (one CTA for short rows), CTA r holding keys [r SEG,
// (r+1) SEG) of the row, SEG = 4 V kSelThreads, loaded as float4 chunks (chunk
// u of thread t: keys 4 (u kSelThreads + t) .. + 3 of the segment).
//  1. each CTA builds an 11-bit histogram (13 bits for rows beyond 32K) of a
//     sample of its keys (the first chunk, or two, of every thread in its
//     first batch) and takes a threshold bin b_r such that, by a wide margin,
//     its segment's share of the row's top k lies in bins >= b_r (rows of at
//     most 4096 keys take every key: b_r = 0);
//  2. each CTA pushes its keys in bins >= b_r, as (key, id) pairs, into the
//     candidate area of the cluster's first CTA (the leader), one remote
//     slot reservation per warp, and records b_r there;
//  3. the leader finds the exact k-th largest candidate T (four 8-bit radix
//     passes, lanes with equal digits merged before the shared atomics) and
//     how many candidates equal to T are taken; if more equal T than are
//     taken, a radix select over their complemented ids keeps the lowest ids;
//  4. the selected ids are marked in a bitmap of the row and written in
//     ascending order (a block scan of the bitmap words' population counts).
// The selection is exact when T >= every CTA's threshold (any key left out
// then lies below T) and the candidates fit; otherwise the leader runs an
// exact radix select over the whole row in global memory instead.
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelCap = 16384;          // most candidates kept in the leader's shared memory
// Threshold bins: the top 11 bits of the order key for rows of up to 32K
// scores, 13 bits (and a sample twice as large) for longer rows, whose
// skewed score tails would otherwise put too many keys into the threshold bin.
__host__ __device__ constexpr int sel_bin_bits(int CPR) { return CPR >= 8 ? 13 : 11; }
constexpr int kSelNoSampleMax = 4096;   // rows this short take every key as a candidate

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Histogram add from a whole warp: lanes holding the same bin are merged so
// that one leader adds their count (candidates share most of their top bits).
__device__ __forceinline__ void warp_hist_add(int* hist, bool in, uint32_t bin) {
    const uint32_t dg = in ? bin : 0xFFFFFFFFu;
    const unsigned same = __match_any_sync(0xffffffffu, dg);
    if (in && (threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[dg], __popc(same));
}

// The k-th largest value among v[0..C) passing `keep` (1 <= k <= their
// number): four 8-bit radix passes over the whole CTA.  Returns the value T,
// how many values equal to T are among the k largest (rem) and how many
// equal T (eq).
template <typename Keep>
__device__ __forceinline__ void sel_radix(const uint32_t* v, int C, int k, Keep keep, int* hist,
                                          int* sh, uint32_t& T, int& rem, int& eq) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < C; i0 += kSelThreads) {  // whole warps iterate together
            const int i = i0 + tid;
            const uint32_t u = i < C ? v[i] : 0u;
            warp_hist_add(hist, i < C && (u & pmask) == prefix && keep(i), (u >> shift) & 255u);
        }
        __syncthreads();
        if (wid == 0) {
            // lane l owns the 8 bins 255-8l .. 248-8l (counted from the top)
            int loc[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { loc[j] = hist[255 - 8 * lane - j]; sum += loc[j]; }
            int inc = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += x;
            }
            int above = inc - sum;
            if (above < remaining && remaining <= inc) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (above < remaining && remaining <= above + loc[j]) {
                        sh[0] = 255 - 8 * lane - j;
                        sh[1] = above;
                        sh[2] = loc[j];
                    }
                    above += loc[j];
                }
            }
        }
        __syncthreads();
        remaining -= sh[1];
        prefix |= uint32_t(sh[0]) << shift;
        pmask |= 0xFFu << shift;
        eq = sh[2];
        __syncthreads();  // sh is rewritten by the next pass
    }
    T = prefix;
    rem = remaining;
}

// The k-th largest of v[0..C) (1 <= k <= C) like sel_radix, in one histogram
// pass when the values are spread: 2048 bins over [min, max] of the values
// find the bin holding the k-th largest; when that bin holds at most 32
// values one warp sorts them, otherwise sel_radix finishes inside the bin.
__device__ __forceinline__ void sel_fine(const uint32_t* v, int C, int k, int* hist, int2* warp_tot, int* sh,
                                         uint32_t& T, int& rem, int& eq) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    __shared__ uint32_t s_lo[kSelWarps], s_hi[kSelWarps], small[33];
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = tid; i < C; i += kSelThreads) { lo = min(lo, v[i]); hi = max(hi, v[i]); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) { s_lo[wid] = lo; s_hi[wid] = hi; }
    for (int i = tid; i < 2048; i += kSelThreads) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) { lo = min(lo, s_lo[w]); hi = max(hi, s_hi[w]); }
    const uint32_t span = hi - lo;
    const int shift = span < 2048u ? 0 : 21 - __clz(int(span));  // (span >> shift) < 2048
    for (int i = tid; i < C; i += kSelThreads) atomicAdd(&hist[(v[i] - lo) >> shift], 1);
    __syncthreads();
    // thread t owns bins 2047-4t .. 2044-4t (counted from the top)
    int loc[4], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) { loc[j] = hist[2047 - 4 * tid - j]; sum += loc[j]; }
    const int2 inc = block_scan2<kSelThreads>(make_int2(sum, 0), warp_tot);
    int above = inc.x - sum;
    if (above < k && k <= inc.x) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (above < k && k <= above + loc[j]) { sh[0] = 2047 - 4 * tid - j; sh[1] = above; sh[2] = loc[j]; }
            above += loc[j];
        }
    }
    if (tid == 0) sh[3] = 0;
    __syncthreads();
    const int bin = sh[0], abv = sh[1], h = sh[2];
    const int need = k - abv;                      // values to take from the bin
    if (shift == 0) {                              // the bin is a single value
        T = lo + uint32_t(bin);
        rem = need;
        eq = h;
        return;
    }
    if (h > 32) {                                  // crowded bin: radix inside it
        sel_radix(v, C, need, [&](int i) { return int((v[i] - lo) >> shift) == bin; }, hist, sh, T, rem, eq);
        return;
    }
    // at most 32 values: gather them and let one warp sort them (descending)
    for (int i = tid; i < C; i += kSelThreads)
        if (int((v[i] - lo) >> shift) == bin) small[atomicAdd(&sh[3], 1)] = v[i];
    __syncthreads();
    if (wid == 0) {
        uint32_t x = lane < h ? small[lane] : 0u;
        // bitonic sort of 32 values, descending
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int st = size >> 1; st > 0; st >>= 1) {
                const uint32_t y = __shfl_xor_sync(0xffffffffu, x, st);
                const bool up = ((lane & size) == 0) == ((lane & st) == 0);
                x = up ? max(x, y) : min(x, y);
            }
        }
        const uint32_t t = __shfl_sync(0xffffffffu, x, need - 1);
        const int gt = __popc(__ballot_sync(0xffffffffu, lane < h && x > t));
        const int e = __popc(__ballot_sync(0xffffffffu, lane < h && x == t));
        if (lane == 0) { small[32] = t; sh[1] = gt; sh[2] = e; }
    }
    __syncthreads();
    T = small[32];
    rem = need - sh[1];
    eq = sh[2];
    __syncthreads();
}

// Exact selection over a whole row in global memory by one CTA: three
// histogram passes (11, 11 and 10 bits) and the ordered write.
__device__ __noinline__ void sel_row_global(const float* s, int64_t n, int k, int32_t* out, int* hist,
                                            int2* warp_tot, int* sh) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nbins = pass < 2 ? 2048 : 1024;
        for (int i = tid; i < nbins; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int64_t i0 = 0; i0 < n; i0 += kSelThreads) {
            const int64_t i = i0 + tid;
            const uint32_t u = i < n ? order_key(s[i]) : 0u;
            warp_hist_add(hist, i < n && (u & pmask) == prefix, (u >> shift) & uint32_t(nbins - 1));
        }
        __syncthreads();
        // thread t owns bins nbins-1-4t .. nbins-4-4t (counted from the top)
        int loc[4], sum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int b = nbins - 1 - 4 * tid - j;
            loc[j] = b >= 0 ? hist[b] : 0;
            sum += loc[j];
        }
        const int2 inc = block_scan2<kSelThreads>(make_int2(sum, 0), warp_tot);
        int above = inc.x - sum;
        if (above < remaining && remaining <= inc.x) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (above < remaining && remaining <= above + loc[j]) {
                    sh[0] = nbins - 1 - 4 * tid - j;
                    sh[1] = above;
                }
                above += loc[j];
            }
        }
        __syncthreads();
        remaining -= sh[1];
        prefix |= uint32_t(sh[0]) << shift;
        pmask |= uint32_t(nbins - 1) << shift;
        __syncthreads();
    }
    // every key above T = prefix, and the first `remaining` keys equal to it;
    // warp w walks a contiguous segment of the row
    const uint32_t T = prefix;
    const int64_t seg = ((n + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
    const int64_t lo = min(n, wid * seg), hi = min(n, lo + seg);
    int gt = 0, eq = 0;
    for (int64_t b0 = lo; b0 < hi; b0 += 32) {
        const int64_t i = b0 + lane;
        const uint32_t u = i < hi ? order_key(s[i]) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < hi && u > T));
        eq += __popc(__ballot_sync(0xffffffffu, i < hi && u == T));
    }
    const int2 incl = block_scan2<kSelThreads>(make_int2(lane == 0 ? gt : 0, lane == 0 ? eq : 0), warp_tot);
    const int gt_incl = __shfl_sync(0xffffffffu, incl.x, 0), eq_incl = __shfl_sync(0xffffffffu, incl.y, 0);
    int eq_before = eq_incl - eq;
    int pos = (gt_incl - gt) + min(eq_before, remaining);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t b0 = lo; b0 < hi; b0 += 32) {
        const int64_t i = b0 + lane;
        const uint32_t u = i < hi ? order_key(s[i]) : 0u;
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

template <int CPR, int V>
__global__ void __launch_bounds__(kSelThreads, 1)
    topk_sel_kernel(const float* __restrict__ scores, int64_t ld, int64_t max_blocks,
                    const int64_t* __restrict__ q_pos, int m, int W, int k, int32_t* __restrict__ idx,
                    int seg, int cap, int vec) {
    constexpr int kBatch = 4 * V * kSelThreads;     // keys of one batch of float4 chunks
    constexpr int kSelBinBits = sel_bin_bits(CPR);
    constexpr int kSelBins = 1 << kSelBinBits;
    constexpr int kSelBinShift = 32 - kSelBinBits;
    extern __shared__ __align__(16) uint32_t dyn[];
    uint32_t* ck = dyn;                  // leader: candidate keys [cap]
    uint32_t* ci = dyn + cap;            // leader: candidate ids [cap]
    uint32_t* bitmap = dyn + 2 * cap;    // leader: [ceil(max_blocks / 32)]
    __shared__ int hist[kSelBins > 2048 ? kSelBins : 2048];   // (sel_fine and the fallback use 2048)
    __shared__ int2 warp_tot[32];
    __shared__ int sh[4];
    __shared__ int s_count;
    __shared__ int s_bin[CPR];
    __shared__ int s_woff[kSelThreads / 32], s_base;
    pdl_wait();  // the scores come from the kernel before this one
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    int r = 0;
    if constexpr (CPR > 1) r = int(cg::this_cluster().block_rank());
    const int64_t row = blockIdx.x / CPR;
    const float* s = scores + row * ld;
    int32_t* out = idx + row * k;
    const int n = int(min(n_elig(q_pos[row], m, W), max_blocks));
    if (n <= k) {  // every eligible block is selected (uniform over the cluster)
        if (r == 0)
            for (int i = tid; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
        return;
    }
    if (r == 0 && tid == 0) s_count = 0;
    if constexpr (CPR > 1) cluster_arrive_release();  // the leader's counter is set
    int* lcount = &s_count;
    uint32_t* lck = ck;
    uint32_t* lci = ci;
    int* lbin = s_bin;
    if constexpr (CPR > 1) {
        cg::cluster_group cl = cg::this_cluster();
        lcount = cl.map_shared_rank(&s_count, 0);
        lck = cl.map_shared_rank(ck, 0);
        lci = cl.map_shared_rank(ci, 0);
        lbin = cl.map_shared_rank(s_bin, 0);
    }
    const int base = r * seg, end = min(n, base + seg);
    int b_r = 0;
#pragma unroll 1
    for (int b0 = base; b0 < end; b0 += kBatch) {
        // this batch's keys (0 = no key: every real key is nonzero)
        uint32_t key[4 * V];
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int i0 = b0 + 4 * (u * kSelThreads + tid);
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (vec && i0 + 3 < end) {
                f = *reinterpret_cast<const float4*>(s + i0);
            } else {
                if (i0 < end) f.x = s[i0];
                if (i0 + 1 < end) f.y = s[i0 + 1];
                if (i0 + 2 < end) f.z = s[i0 + 2];
                if (i0 + 3 < end) f.w = s[i0 + 3];
            }
            key[4 * u] = i0 < end ? order_key(f.x) : 0u;
            key[4 * u + 1] = i0 + 1 < end ? order_key(f.y) : 0u;
            key[4 * u + 2] = i0 + 2 < end ? order_key(f.z) : 0u;
            key[4 * u + 3] = i0 + 3 < end ? order_key(f.w) : 0u;
        }
        if (b0 == base) {
            // 1. the segment's threshold bin from its sample (the first two
            // chunks of every thread in the first batch)
            constexpr int kSampleChunks = (V < 2 || CPR < 8) ? 1 : 2;
            constexpr int kPer = kSelBins / kSelThreads;   // bins per thread in the scan
            if (n > kSelNoSampleMax) {
                for (int i = tid; i < kSelBins; i += kSelThreads) hist[i] = 0;
                __syncthreads();
#pragma unroll
                for (int c = 0; c < 4 * kSampleChunks; ++c)
                    if (key[c]) atomicAdd(&hist[key[c] >> kSelBinShift], 1);
                __syncthreads();
                const int n_s = max(0, min(4 * kSampleChunks * kSelThreads, end - base));  // sampled keys
                const float mean = float(k) * float(n_s) / float(n);
                const int target = int(ceilf(mean + 4.f * sqrtf(mean))) + 16;
                // thread t owns bins kSelBins-1-kPer t .. kSelBins-kPer-kPer t (from the top)
                int loc[kPer], sum = 0;
#pragma unroll
                for (int j = 0; j < kPer; ++j) { loc[j] = hist[kSelBins - 1 - kPer * tid - j]; sum += loc[j]; }
                const int2 inc = block_scan2<kSelThreads>(make_int2(sum, 0), warp_tot);
                if (tid == 0) sh[3] = 0;
                __syncthreads();
                int above = inc.x - sum;
                if (above < target && target <= inc.x) {
#pragma unroll
                    for (int j = 0; j < kPer; ++j) {
                        if (above < target && target <= above + loc[j]) sh[3] = kSelBins - 1 - kPer * tid - j;
                        above += loc[j];
                    }
                }
                __syncthreads();
                b_r = sh[3];  // 0 (every key) when the sample is short of the target
            }
            if constexpr (CPR > 1) cluster_wait_acquire();
            else __syncthreads();
        }
        // 2. candidates into the leader: per-warp counts, scanned in the CTA,
        // and one reservation in the leader per CTA and batch (remote atomics
        // on one counter serialise, so there are as few as possible)
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 4 * V; ++j)
            cnt += __popc(__ballot_sync(0xffffffffu, key[j] != 0u && int(key[j] >> kSelBinShift) >= b_r));
        if (lane == 0) s_woff[tid >> 5] = cnt;
        __syncthreads();
        if (tid < 32) {
            const int v = tid < kSelThreads / 32 ? s_woff[tid] : 0;
            int inc = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (tid >= o) inc += y;
            }
            const int total = __shfl_sync(0xffffffffu, inc, 31);
            if (tid < kSelThreads / 32) s_woff[tid] = inc - v;
            if (tid == 0) s_base = total ? atomicAdd(lcount, total) : 0;
        }
        __syncthreads();
        int slot = s_base + s_woff[tid >> 5];
#pragma unroll
        for (int j = 0; j < 4 * V; ++j) {
            const bool c = key[j] != 0u && int(key[j] >> kSelBinShift) >= b_r;
            const unsigned bal = __ballot_sync(0xffffffffu, c);
            if (c) {
                const int p = slot + __popc(bal & lt_mask);
                if (p < cap) {
                    lck[p] = key[j];
                    lci[p] = uint32_t(b0 + 4 * ((j >> 2) * kSelThreads + tid) + (j & 3));
                }
            }
            slot += __popc(bal);
        }
    }
    if (base >= end) {  // an empty segment still passes the barrier above
        if constexpr (CPR > 1) cluster_wait_acquire();
    }
    if (tid == 0) lbin[r] = b_r;
    if constexpr (CPR > 1) {
        cg::this_cluster().sync();  // every candidate is in the leader
        if (r != 0) return;
    } else {
        __syncthreads();
    }
    // 3. (leader) the k-th largest candidate; ties at T by the lowest ids
    const int C = s_count;
    uint32_t bmax = 0;
#pragma unroll
    for (int q = 0; q < CPR; ++q) bmax = max(bmax, uint32_t(s_bin[q]));
    bool fast = C >= k && C <= cap;
    uint32_t T = 0, T2 = 0;
    int rem = 0, eq = 0;
    if (fast) {
        sel_fine(ck, C, k, hist, warp_tot, sh, T, rem, eq);
        fast = T >= (bmax << kSelBinShift);  // every key left out lies below T
    }
    if (!fast) {
        sel_row_global(s, n, k, out, hist, warp_tot, sh);
        return;
    }
    const bool all_eq = eq == rem;
    if (!all_eq) {
        // ck becomes 1 for keys above T, 0 below, ~id (>= 2^31) equal
        for (int i = tid; i < C; i += kSelThreads) ck[i] = ck[i] == T ? ~ci[i] : (ck[i] > T ? 1u : 0u);
        __syncthreads();
        int r2, e2;
        sel_radix(ck, C, rem, [&](int i) { return ck[i] > 1u; }, hist, sh, T2, r2, e2);
    }
    // 4. bitmap of the selected ids, then the ids in ascending order
    const int words = (n + 31) >> 5;
    for (int i = tid; i < words; i += kSelThreads) bitmap[i] = 0u;
    __syncthreads();
    for (int i = tid; i < C; i += kSelThreads) {
        const bool take = all_eq ? ck[i] >= T : (ck[i] == 1u || (ck[i] > 1u && ck[i] >= T2));
        if (take) atomicOr(&bitmap[ci[i] >> 5], 1u << (ci[i] & 31u));
    }
    __syncthreads();
    // warp w owns a contiguous range of 32-word chunks; lane l reads word l of
    // a chunk (no bank conflicts), a warp scan of the words' counts places them
    constexpr int kWarps = kSelThreads / 32;
    const int wid = tid >> 5;
    const int wpw = ((words + kWarps - 1) / kWarps + 31) & ~31;  // words per warp
    const int w0 = min(words, wid * wpw), w1 = min(words, w0 + wpw);
    int c = 0;
    for (int wi = w0 + lane; wi < w1; wi += 32) c += __popc(bitmap[wi]);
    const int wc = __reduce_add_sync(0xffffffffu, c);  // every lane takes part
    const int2 incl = block_scan2<kSelThreads>(make_int2(lane == 0 ? wc : 0, 0), warp_tot);
    int pos = __shfl_sync(0xffffffffu, incl.x, 0) - wc;
    for (int cb = w0; cb < w1; cb += 32) {
        const int wi = cb + lane;
        uint32_t b = wi < w1 ? bitmap[wi] : 0u;
        const int pc = __popc(b);
        int inc = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        int p = pos + inc - pc;
        while (b) {
            const int bit = __ffs(b) - 1;
            b &= b - 1;
            if (p < k) out[p] = wi * 32 + bit;
            ++p;
        }
        pos += __shfl_sync(0xffffffffu, inc, 31);
    }
}

template <int CPR, int V>
static cudaError_t launch_topk_sel(const float* scores, int64_t ld, int64_t max_blocks, const int64_t* q_pos,
                                   int m, int W, int k, int64_t rows, int32_t* idx, cudaStream_t s, bool pdl) {
    // segment of each CTA: the row split in CPR parts, in whole float4 chunks of all threads
    const int64_t unit = 4 * kSelThreads;
    const int seg = int(ceil_div(ceil_div(max_blocks, CPR), unit) * unit);
    const int cap = int(std::min<int64_t>(kSelCap, ceil_div(max_blocks, 4) * 4));
    const size_t sm = (2 * size_t(cap) + size_t((max_blocks + 31) / 32)) * 4;
    cudaError_t e = ensure_smem(topk_sel_kernel<CPR, V>, sm);
    if (e != cudaSuccess) return e;
    if (CPR > 8) {  // clusters beyond the portable 8 CTAs
        e = cudaFuncSetAttribute(topk_sel_kernel<CPR, V>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    const int vec = ((reinterpret_cast<uintptr_t>(scores) & 15) == 0 && (ld % 4) == 0) ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(rows * CPR));
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (CPR > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = CPR;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    if (CPR > 8) {
        // a 16-CTA cluster needs 16 free SMs of one GPC; fall back when the
        // device cannot place one (queried once per device)
        static int known[64];  // 0 unknown, 1 yes, 2 no
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidValue;
        if (known[dev] == 0) {
            int n_clusters = 0;
            cudaLaunchConfig_t q = cfg;
            q.numAttrs = 1;  // the cluster dimension alone
            const bool ok = cudaOccupancyMaxActiveClusters(&n_clusters, topk_sel_kernel<CPR, V>, &q) == cudaSuccess &&
                            n_clusters > 0;
            if (!ok) (void)cudaGetLastError();
            known[dev] = ok ? 1 : 2;
        }
        if (known[dev] == 2) return cudaErrorNotSupported;
    }
    return cudaLaunchKernelEx(&cfg, topk_sel_kernel<CPR, V>, scores, ld, max_blocks, q_pos, m, W, k, idx, seg,
                              cap, vec);
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
    // Sampled-threshold selection: one CTA per row for rows of up to 8,192
    // scores (prefill chunks); for longer rows a cluster of 4 CTAs (up to 32K
    // scores) or 8 CTAs per row, so that few rows still spread over many SMs.
    // (many short rows -- a prefill chunk -- are faster with the whole row in
    // one CTA's shared memory and no sampling: topk_smem_kernel below)
    const bool many_short = rows >= 2 * kNumSMs && max_blocks <= 4096;
    if (many_short && max_blocks <= kWarpRowMax)
        return launch_ex(topk_warp_kernel, dim3(unsigned(ceil_div(rows, kWarpRowThreads / 32))),
                         dim3(kWarpRowThreads), 0, s, pdl, scores, ld, max_blocks, q_pos, m, W, k, rows, idx);
    if (k <= kSelCap / 2 && rows * 8 <= INT32_MAX && max_blocks <= INT32_MAX / 2 && !many_short) {
        if (max_blocks <= 2048) return launch_topk_sel<1, 1>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (max_blocks <= 8192) return launch_topk_sel<1, 4>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (max_blocks <= 32768) return launch_topk_sel<4, 4>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
        if (max_blocks > 65536 && rows * 16 <= kNumSMs) {
            // few long rows (a 1M-token sequence): 16 CTAs per row, one batch each
            const cudaError_t e = launch_topk_sel<16, 8>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
            if (e != cudaErrorNotSupported) return e;
        }
        return launch_topk_sel<8, 8>(scores, ld, max_blocks, q_pos, m, W, k, rows, idx, s, pdl);
    }
    // Few longer rows cannot fill the GPU with one CTA each: give each row a cluster.
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
