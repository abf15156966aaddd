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
#include "kernels.h"

namespace csa {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide scan of two ints over kTopkThreads threads.
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
        int2 t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ax = __shfl_up_sync(0xffffffffu, t.x, o);
            const int ay = __shfl_up_sync(0xffffffffu, t.y, o);
            if (lane >= o) { t.x += ax; t.y += ay; }
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    if (wid > 0) { v.x += warp_tot[wid - 1].x; v.y += warp_tot[wid - 1].y; }
    __syncthreads();
    return v;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t max_blocks,
    const int64_t* __restrict__ q_pos, int m, int W, int k, int32_t* __restrict__ idx) {
    __shared__ int hist[2048];
    __shared__ int2 warp_tot[32];
    __shared__ int found_digit, found_above;
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
    const uint32_t T = prefix;
    const int64_t seg = ceil_div(n, kTopkThreads);
    const int64_t lo = min(n, tid * seg), hi = min(n, lo + seg);
    int gt = 0, eq = 0;
    for (int64_t i = lo; i < hi; ++i) {
        const uint32_t u = order_key(s[i]);
        gt += u > T;
        eq += u == T;
    }
    const int2 inc = block_scan2(make_int2(gt, eq), warp_tot);
    int eq_before = inc.y - eq;
    int pos = (inc.x - gt) + min(eq_before, remaining);
    for (int64_t i = lo; i < hi; ++i) {
        const uint32_t u = order_key(s[i]);
        if (u > T) {
            if (pos < k) out[pos] = int32_t(i);
            ++pos;
        } else if (u == T) {
            if (eq_before < remaining) {
                if (pos < k) out[pos] = int32_t(i);
                ++pos;
            }
            ++eq_before;
        }
    }
}

cudaError_t launch_topk(const float* scores, int64_t ld, int64_t max_blocks, const int64_t* q_pos,
                        int m, int W, int k, int64_t rows, int32_t* idx, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    topk_kernel<<<unsigned(rows), kTopkThreads, 0, s>>>(scores, ld, max_blocks, q_pos, m, W, k, idx);
    return cudaGetLastError();
}

}  // namespace csa
