// Softmax-gated pooling of m tokens into one entry, and the store of fp32
// rows as FP8 (E4M3 + fp32 scale per 64 channels), MXFP4 (E2M1 + E8M0 per
// 32 channels) or bf16.
//
// Pooling ("DeepSeek-V4 發佈說明", sections 壓縮稀疏注意力 (CSA) and 重度壓縮注意力
// (HCA)): per channel c, the m tokens of block j are weighted by a softmax
// over the slots of z + B[slot], then summed.  FP8 entries and an FP4
// indexer are the storage formats named in section 架構實現.
//
// One warp owns one 64-channel group of one output row: each lane holds two
// adjacent channels, so every load is a coalesced 256 B (fp32) or 128 B
// (bf16) row segment, the FP8 scale group is exactly one warp and an MXFP4
// block is one half-warp.  The pass over the m slots reads z twice (max,
// then exp-sum) so each weight is a single exp; the kernel is HBM-bound on
// the x / z reads.
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int FMT>
__device__ __forceinline__ float2 load_pair(const void* p, int64_t off) {
    if constexpr (FMT == CSA_F32) {
        return *reinterpret_cast<const float2*>((const float*)p + off);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>((const uint16_t*)p + off);
        return make_float2(__int_as_float(int(u << 16)), __int_as_float(int(u & 0xFFFF0000u)));
    }
}

// Store the pair (v0, v1) of channels (c, c+1) of row j in OUT_FMT.  All 32
// lanes of the warp must call this together (group reductions).
template <int OUT_FMT>
__device__ __forceinline__ void store_pair(float v0, float v1, int64_t j, int d, int c, int lane,
                                           void* out, void* out_scales) {
    if constexpr (OUT_FMT == CSA_F32) {
        *reinterpret_cast<float2*>((float*)out + j * d + c) = make_float2(v0, v1);
    } else if constexpr (OUT_FMT == CSA_BF16) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v0, v1);
        *reinterpret_cast<__nv_bfloat162*>((uint16_t*)out + j * d + c) = b;
    } else if constexpr (OUT_FMT == CSA_FP8_S64) {
        const float amax = warp_max(fmaxf(fabsf(v0), fabsf(v1)));
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        const uint16_t codes = cvt_e4m3x2(__fdiv_rn(v0, scale), __fdiv_rn(v1, scale));
        *reinterpret_cast<uint16_t*>((uint8_t*)out + j * d + c) = codes;
        if (lane == 0) ((float*)out_scales)[j * (d / 64) + c / 64] = scale;
    } else {  // MXFP4: a half-warp covers one 32-channel block
        float a = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        int X = a > 0.f ? ilog2_floor(a) - 2 : 0;
        X = max(-127, min(127, X));
        const float inv = pow2f(-X);
        const uint32_t byte = cvt_e2m1x2(__fmul_rn(v0, inv), __fmul_rn(v1, inv));
        ((uint8_t*)out)[j * (d / 2) + c / 2] = (uint8_t)byte;
        if ((lane & 15) == 0) ((uint8_t*)out_scales)[j * (d / 32) + c / 32] = (uint8_t)(X + 127);
    }
}

// POOL: out row j pools input rows [j*m, j*m+m) with gate z + bias.
// !POOL: out row j is input row j (a pure format conversion; m, z, bias unused).
template <int IN_FMT, int OUT_FMT, bool POOL>
__global__ void __launch_bounds__(256) pool_kernel(const void* __restrict__ x,
                                                   const void* __restrict__ z,
                                                   const float* __restrict__ bias, int64_t n_out,
                                                   int m, int d, void* out, void* out_scales) {
    const int64_t gw = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    const int groups = d / 64;
    if (gw >= n_out * groups) return;  // whole warps exit together
    const int64_t j = gw / groups;
    const int c = int(gw % groups) * 64 + 2 * lane;
    float v0, v1;
    if constexpr (POOL) {
        const int64_t r0 = j * m;
        float mx0 = -INFINITY, mx1 = -INFINITY;
        for (int r = 0; r < m; ++r) {
            const float2 zz = load_pair<IN_FMT>(z, (r0 + r) * d + c);
            const float2 bb = *reinterpret_cast<const float2*>(bias + int64_t(r) * d + c);
            mx0 = fmaxf(mx0, zz.x + bb.x);
            mx1 = fmaxf(mx1, zz.y + bb.y);
        }
        float den0 = 0.f, den1 = 0.f, acc0 = 0.f, acc1 = 0.f;
        for (int r = 0; r < m; ++r) {
            const float2 zz = load_pair<IN_FMT>(z, (r0 + r) * d + c);
            const float2 bb = *reinterpret_cast<const float2*>(bias + int64_t(r) * d + c);
            const float2 xx = load_pair<IN_FMT>(x, (r0 + r) * d + c);
            const float e0 = expf(zz.x + bb.x - mx0), e1 = expf(zz.y + bb.y - mx1);
            den0 += e0;
            den1 += e1;
            acc0 = fmaf(e0, xx.x, acc0);
            acc1 = fmaf(e1, xx.y, acc1);
        }
        v0 = acc0 / den0;
        v1 = acc1 / den1;
    } else {
        const float2 xx = load_pair<IN_FMT>(x, j * d + c);
        v0 = xx.x;
        v1 = xx.y;
    }
    store_pair<OUT_FMT>(v0, v1, j, d, c, lane, out, out_scales);
}

// ------------------------------------------------------ staged pooling (m >= 16)
// For the long blocks of HCA (m' = 128): persistent CTAs of d/2 threads (the
// channel pairs of pool_kernel, so the FP8 scale group is a warp and an MXFP4
// block a half-warp), each walking output rows j = blockIdx.x, +gridDim.x.
// One thread streams the rows of x and z through a ring of shared-memory
// stages of kPoolRows rows with 1-D bulk copies (each stage two contiguous
// copies, completion on an mbarrier), running ahead into the next output
// row; the others take each stage's slots with a running max per channel
// (rescaling the sums when a stage raises it), so x and z cross HBM once.
// The weights are 2^((z + B) log2 e - max) from the special-function unit.
constexpr int kPoolRows = 16;
constexpr float kLog2eF = 1.4426950408889634f;

// 2^x by the special-function unit (relative error about 2^-22)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int IN_FMT>
struct PoolStage {
    static constexpr int kElem = IN_FMT == CSA_F32 ? 4 : 2;
    static constexpr int kStages = IN_FMT == CSA_F32 ? 2 : 3;
};

template <int IN_FMT, int OUT_FMT>
__global__ void __launch_bounds__(544) pool_staged_kernel(const void* __restrict__ x, const void* __restrict__ z,
                                                          const float* __restrict__ bias, int64_t n_out, int m,
                                                          int d, void* out, void* out_scales) {
    using namespace sm100;
    constexpr int kSt = PoolStage<IN_FMT>::kStages, kElem = PoolStage<IN_FMT>::kElem;
    extern __shared__ __align__(128) uint8_t smem_pool[];
    __shared__ uint64_t full[kSt], empty[kSt];
    const int tid = threadIdx.x, lane = tid & 31;
    const int n_cons = d / 2;  // consumer threads (one channel pair each); then one producer warp
    const uint32_t rows_bytes = uint32_t(kPoolRows) * d * kElem;  // one tensor's rows of a stage
    uint8_t* stage_x = smem_pool;
    uint8_t* stage_z = smem_pool + kSt * rows_bytes;
    const int per_row = m / kPoolRows;  // stages per output row
    if (tid == 0) {
        for (int i = 0; i < kSt; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], n_cons / 32); }
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t my_rows = n_out > blockIdx.x ? (n_out - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t total = my_rows * per_row;  // stages this CTA streams
    if (tid >= n_cons) {
        // producer: stage s of this CTA = stage (s % per_row) of its (s / per_row)-th row
        if (tid == n_cons) {
            int64_t issued = 0;
            for (int64_t sidx = 0; sidx < total; ++sidx) {
                const int b = int(sidx % kSt);
                if (sidx >= kSt && !mbar_wait(&empty[b], uint32_t(((sidx / kSt) - 1) & 1))) break;
                const int64_t j = blockIdx.x + (sidx / per_row) * gridDim.x;
                const int64_t r = j * m + (sidx % per_row) * kPoolRows;
                mbar_arrive_expect_tx(&full[b], 2 * rows_bytes);
                bulk_g2s(stage_x + b * rows_bytes, (const uint8_t*)x + r * d * kElem, rows_bytes, &full[b]);
                bulk_g2s(stage_z + b * rows_bytes, (const uint8_t*)z + r * d * kElem, rows_bytes, &full[b]);
                issued = sidx + 1;
            }
            // every copy issued has landed before the CTA exits (already the
            // case unless a consumer gave up on a wait)
            bool drained = true;
            for (int64_t i = max(int64_t(0), issued - kSt); i < issued && drained; ++i)
                drained = mbar_wait(&full[i % kSt], uint32_t((i / kSt) & 1));
        }
    } else {
        const int c = 2 * tid;  // this thread's channel pair
        bool ok = true;
        int64_t sidx = 0;
        for (int64_t t = 0; t < my_rows; ++t) {
            const int64_t j = blockIdx.x + t * gridDim.x;
            float mx0 = -INFINITY, mx1 = -INFINITY, den0 = 0.f, den1 = 0.f, acc0 = 0.f, acc1 = 0.f;
            for (int st = 0; st < per_row; ++st, ++sidx) {
                const int b = int(sidx % kSt);
                if (ok) ok = mbar_wait(&full[b], uint32_t((sidx / kSt) & 1));
                ok = __all_sync(0xffffffffu, ok);  // whole warps go on or stop together
                if (!ok) continue;
                const uint8_t* xs = stage_x + b * rows_bytes;
                const uint8_t* zs = stage_z + b * rows_bytes;
                const float* bs = bias + int64_t(st) * kPoolRows * d + c;
                // the stage's gate logits in log2 units and their max per
                // channel, then the weights 2^(logit - running max)
                float zz[kPoolRows][2];
                float cm0 = mx0, cm1 = mx1;
#pragma unroll
                for (int i = 0; i < kPoolRows; ++i) {
                    const float2 bb = *reinterpret_cast<const float2*>(bs + int64_t(i) * d);
                    const float2 zr = load_pair<IN_FMT>(zs, int64_t(i) * d + c);
                    zz[i][0] = (zr.x + bb.x) * kLog2eF;
                    zz[i][1] = (zr.y + bb.y) * kLog2eF;
                    cm0 = fmaxf(cm0, zz[i][0]);
                    cm1 = fmaxf(cm1, zz[i][1]);
                }
                if (cm0 > mx0) {
                    const float f = mx0 == -INFINITY ? 0.f : ex2_approx(mx0 - cm0);
                    den0 *= f; acc0 *= f; mx0 = cm0;
                }
                if (cm1 > mx1) {
                    const float f = mx1 == -INFINITY ? 0.f : ex2_approx(mx1 - cm1);
                    den1 *= f; acc1 *= f; mx1 = cm1;
                }
#pragma unroll
                for (int i = 0; i < kPoolRows; ++i) {
                    const float2 xr = load_pair<IN_FMT>(xs, int64_t(i) * d + c);
                    const float e0 = ex2_approx(zz[i][0] - mx0), e1 = ex2_approx(zz[i][1] - mx1);
                    den0 += e0; den1 += e1;
                    acc0 = fmaf(e0, xr.x, acc0); acc1 = fmaf(e1, xr.y, acc1);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[b]);  // this warp is done with the stage
            }
            store_pair<OUT_FMT>(ok ? acc0 / den0 : 0.f, ok ? acc1 / den1 : 0.f, j, d, c, lane, out, out_scales);
        }
    }
    __syncthreads();
}

template <int IN_FMT>
static bool pool_staged_fits(int m, int d) {
    constexpr int kElem = PoolStage<IN_FMT>::kElem, kSt = PoolStage<IN_FMT>::kStages;
    return m >= kPoolRows && m % kPoolRows == 0 && d % 64 == 0 && d <= 1024 &&
           size_t(2) * kSt * kPoolRows * d * kElem <= size_t(200) << 10;
}

template <int IN_FMT, int OUT_FMT>
static cudaError_t launch_pool_staged(const void* x, const void* z, const float* bias, int64_t n_out, int m, int d,
                                      void* out, void* out_scales, cudaStream_t s) {
    constexpr int kElem = PoolStage<IN_FMT>::kElem, kSt = PoolStage<IN_FMT>::kStages;
    const size_t sm = size_t(2) * kSt * kPoolRows * d * kElem;
    cudaError_t e = ensure_smem(pool_staged_kernel<IN_FMT, OUT_FMT>, sm);
    if (e != cudaSuccess) return e;
    const int per_sm = int(std::max<size_t>(1, std::min<size_t>(2, (size_t(220) << 10) / sm)));
    const int grid = int(std::min<int64_t>(n_out, int64_t(per_sm) * kNumSMs));
    pool_staged_kernel<IN_FMT, OUT_FMT><<<grid, d / 2 + 32, sm, s>>>(x, z, bias, n_out, m, d, out, out_scales);
    return cudaGetLastError();
}

template <int IN_FMT, bool POOL>
static cudaError_t launch_pool_out(int out_fmt, const void* x, const void* z, const float* bias,
                                   int64_t n_out, int m, int d, void* out, void* out_scales,
                                   cudaStream_t s) {
    if (POOL && pool_staged_fits<IN_FMT>(m, d) && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
        (reinterpret_cast<uintptr_t>(z) & 15) == 0) {
        switch (out_fmt) {
        case CSA_F32: return launch_pool_staged<IN_FMT, CSA_F32>(x, z, bias, n_out, m, d, out, out_scales, s);
        case CSA_BF16: return launch_pool_staged<IN_FMT, CSA_BF16>(x, z, bias, n_out, m, d, out, out_scales, s);
        case CSA_FP8_S64:
            return launch_pool_staged<IN_FMT, CSA_FP8_S64>(x, z, bias, n_out, m, d, out, out_scales, s);
        default: return launch_pool_staged<IN_FMT, CSA_MXFP4>(x, z, bias, n_out, m, d, out, out_scales, s);
        }
    }
    const int64_t warps = n_out * (d / 64);
    const dim3 grid(unsigned(ceil_div(warps, 8)));
    switch (out_fmt) {
    case CSA_F32:
        pool_kernel<IN_FMT, CSA_F32, POOL><<<grid, 256, 0, s>>>(x, z, bias, n_out, m, d, out, out_scales);
        break;
    case CSA_BF16:
        pool_kernel<IN_FMT, CSA_BF16, POOL><<<grid, 256, 0, s>>>(x, z, bias, n_out, m, d, out, out_scales);
        break;
    case CSA_FP8_S64:
        pool_kernel<IN_FMT, CSA_FP8_S64, POOL><<<grid, 256, 0, s>>>(x, z, bias, n_out, m, d, out, out_scales);
        break;
    default:
        pool_kernel<IN_FMT, CSA_MXFP4, POOL><<<grid, 256, 0, s>>>(x, z, bias, n_out, m, d, out, out_scales);
        break;
    }
    return cudaGetLastError();
}

cudaError_t launch_compress(int in_fmt, int out_fmt, const void* x, const void* z,
                            const float* bias, int64_t n_tokens, int m, int d, void* out,
                            void* out_scales, cudaStream_t s) {
    const int64_t n_out = n_tokens / m;
    if (n_out == 0) return cudaSuccess;
    if (in_fmt == CSA_F32)
        return launch_pool_out<CSA_F32, true>(out_fmt, x, z, bias, n_out, m, d, out, out_scales, s);
    return launch_pool_out<CSA_BF16, true>(out_fmt, x, z, bias, n_out, m, d, out, out_scales, s);
}

cudaError_t launch_quantize(int out_fmt, const float* src, int64_t rows, int d, void* out,
                            void* out_scales, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    return launch_pool_out<CSA_F32, false>(out_fmt, src, nullptr, nullptr, rows, 1, d, out,
                                           out_scales, s);
}

}  // namespace csa
