// Device-side helpers shared by the library's kernels: number formats,
// warp reductions, the device status word and launch bookkeeping.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

constexpr int kNumSMs = 148;  // B200
constexpr int64_t kMaxGridY = 65535;  // largest grid extent along y (and z)

// Device status word (CSA_DEV_* bits), shared by every call on a device.
extern __device__ unsigned int g_status;

__device__ __forceinline__ void flag_status(unsigned int bits) { atomicOr(&g_status, bits); }

// Programmatic dependent launch: a kernel launched with it may start before the
// previous kernel of the stream has finished; pdl_wait() blocks until that
// kernel has completed and its memory is visible (a no-op without it), and
// pdl_launch_dependents() lets the next such kernel be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- formats
// E4M3 code -> float, exact (the hardware conversion to f16 is exact for
// every E4M3 value, and f16 -> f32 is exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

// E2M1 nibble -> float: sign, 2-bit exponent (bias 1), 1 mantissa bit.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
    const uint32_t mag = c & 7u;
    // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 for codes 0..7
    float v = (mag < 2u) ? 0.5f * float(mag)
                         : __int_as_float(int((((mag >> 1) + 126u) << 23) | ((mag & 1u) << 22)));
    return (c & 8u) ? -v : v;
}

// E8M0 byte -> 2^(c-127); c = 255 (NaN in the format) decodes as +inf.
__device__ __forceinline__ float e8m0_to_f32(uint32_t c) {
    return c == 0 ? __int_as_float(0x00400000) : __int_as_float(int(c << 23));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __int_as_float(int(uint32_t(b) << 16));
}

// fp32 -> E4M3, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float v) {
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// fp32 -> E2M1 nibble, round to nearest even, saturating to +-6.
__device__ __forceinline__ uint32_t f32_to_e2m1(float v) {
    return (uint32_t)__nv_cvt_float_to_fp4(v, __NV_E2M1, cudaRoundNearest) & 0xFu;
}

// Two fp32 values -> one byte of two E2M1 codes (lo in the low nibble), round
// to nearest even, saturating to +-6.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{ .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n mov.b16 %0, {t, 0}; }"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r & 0xFFu;
}

// 2^e as a float for e in [-127, 127] (exact).
__device__ __forceinline__ float pow2f(int e) {
    return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(0x00400000);
}

// floor(log2(a)) for a finite a > 0 (subnormals included).
__device__ __forceinline__ int ilog2_floor(float a) {
    const uint32_t u = __float_as_uint(a);
    const int e = int((u >> 23) & 0xFF);
    if (e != 0) return e - 127;
    return -127 + (31 - __clz(int(u & 0x7FFFFF))) - 22;  // subnormal: 2^-149 * mantissa
}

// One element of a stored [rows][d] tensor as float.
template <int FMT>
__device__ __forceinline__ float load_elem(const void* data, const void* scales, int64_t row,
                                           int d, int col) {
    if constexpr (FMT == CSA_F32) {
        return ((const float*)data)[row * d + col];
    } else if constexpr (FMT == CSA_BF16) {
        return bf16_bits_to_f32(((const uint16_t*)data)[row * d + col]);
    } else if constexpr (FMT == CSA_FP8_S64) {
        const uint8_t c = ((const uint8_t*)data)[row * d + col];
        return e4m3_to_f32(c) * ((const float*)scales)[row * (d / 64) + col / 64];
    } else {
        const uint8_t b = ((const uint8_t*)data)[row * (d / 2) + col / 2];
        const uint32_t c = (col & 1) ? (b >> 4) : (b & 15);
        return e2m1_to_f32(c) * e8m0_to_f32(((const uint8_t*)scales)[row * (d / 32) + col / 32]);
    }
}

// ------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Number of pooled blocks visible to a query at position t.
__host__ __device__ __forceinline__ int64_t n_elig(int64_t t, int m, int W) {
    const int64_t a = t - W;
    return a <= 0 ? 0 : a / m;
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Raise a kernel's dynamic shared-memory limit once per (kernel, device): the
// attribute call is host work that would otherwise sit between launches.
cudaError_t ensure_smem_impl(const void* kernel, size_t bytes);

// Launch with cudaLaunchKernelEx, optionally as a programmatic dependent of
// the previous kernel in the stream (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
template <typename K>
inline cudaError_t ensure_smem(K* kernel, size_t bytes) {
    return ensure_smem_impl(reinterpret_cast<const void*>(kernel), bytes);
}

}  // namespace csa
