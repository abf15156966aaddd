// Lightning-indexer scores on CUDA cores in fp32 ("DeepSeek-V4 發佈說明",
// section 壓縮稀疏注意力 (CSA): ReLU-scored multi-head dot products):
//   s[j] = sum_h w[h] * ReLU(qI[h] . kI[j])
// One CTA scores a tile of 64 keys for one query: the query's HI x dI block
// and the key tile are decoded to fp32 in shared memory (key rows padded by
// one word so that 64 threads reading 64 different keys hit 32 different
// banks), each thread accumulates a quarter of the heads for one key, and the
// four partial sums are added at the end.  This kernel serves the fp32
// format exactly and every stored format as a plain reference-precision path.
#include "kernels.h"

namespace csa {

template <int FMT>
__global__ void __launch_bounds__(256) indexer_simt_kernel(
    int HI, int dI, int m, int W, const void* __restrict__ qI, const void* __restrict__ qI_s,
    const float* __restrict__ w, const void* __restrict__ kI, const void* __restrict__ kI_s,
    int64_t max_blocks, const int64_t* __restrict__ q_pos, int n_q, float* __restrict__ scores,
    int64_t ld) {
    extern __shared__ float smem[];
    float* q_s = smem;                    // [HI][dI]
    float* k_s = q_s + HI * dI;           // [64][dI+1]
    float* part = k_s + 64 * (dI + 1);    // [4][64]
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.y;       // b * n_q + i
    const int64_t b = row / n_q;
    const int64_t ne = min(n_elig(q_pos[row], m, W), max_blocks);
    const int64_t j0 = int64_t(blockIdx.x) * 64;
    if (j0 >= ne) return;

    for (int e = tid; e < HI * dI; e += 256)
        q_s[e] = load_elem<FMT>(qI, qI_s, row * HI + e / dI, dI, e % dI);
    for (int e = tid; e < 64 * dI; e += 256) {
        const int kk = e / dI, c = e % dI;
        const int64_t j = j0 + kk;
        k_s[kk * (dI + 1) + c] = j < ne ? load_elem<FMT>(kI, kI_s, b * max_blocks + j, dI, c) : 0.f;
    }
    __syncthreads();

    const int kk = tid & 63, hg = tid >> 6;
    const float* wr = w + row * HI;
    float acc = 0.f;
    for (int h = hg; h < HI; h += 4) {
        const float* qh = q_s + h * dI;
        const float* kr = k_s + kk * (dI + 1);
        float dot = 0.f;
        for (int c = 0; c < dI; ++c) dot = fmaf(qh[c], kr[c], dot);
        acc = fmaf(wr[h], fmaxf(dot, 0.f), acc);
    }
    part[hg * 64 + kk] = acc;
    __syncthreads();
    if (tid < 64 && j0 + tid < ne)
        scores[row * ld + j0 + tid] = (part[tid] + part[64 + tid]) + (part[128 + tid] + part[192 + tid]);
}

cudaError_t launch_indexer_simt(int fmt, int HI, int dI, int m, int W, const void* qI,
                                const void* qI_s, const float* w, const void* kI,
                                const void* kI_s, int64_t max_blocks, const int64_t* q_pos,
                                int batch, int n_q, int64_t max_elig, float* scores, int64_t ld,
                                cudaStream_t s) {
    if (max_elig <= 0 || batch * int64_t(n_q) == 0) return cudaSuccess;
    const dim3 grid(unsigned(ceil_div(max_elig, 64)), unsigned(batch * n_q));
    const size_t sm = size_t(HI * dI + 64 * (dI + 1) + 256) * sizeof(float);
    cudaError_t e;
#define CSA_LAUNCH_IDX(F)                                                                          \
    e = ensure_smem(indexer_simt_kernel<F>, sm);                                                   \
    if (e != cudaSuccess) return e;                                                                \
    indexer_simt_kernel<F><<<grid, 256, sm, s>>>(HI, dI, m, W, qI, qI_s, w, kI, kI_s, max_blocks,  \
                                                 q_pos, n_q, scores, ld);
    switch (fmt) {
    case CSA_F32: CSA_LAUNCH_IDX(CSA_F32); break;
    case CSA_BF16: CSA_LAUNCH_IDX(CSA_BF16); break;
    default: CSA_LAUNCH_IDX(CSA_MXFP4); break;
    }
#undef CSA_LAUNCH_IDX
    return cudaGetLastError();
}

}  // namespace csa
