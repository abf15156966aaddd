// MQA attention over FP8 pooled entries + the bf16 raw window + a per-head
// sink on the 5th-generation tensor cores (wiki summary "DeepSeek V4",
// section 架构创新: top-k sparse selection + MQA, sliding-window branch,
// attention sink; release note sections CSA and HCA; FP8 KV storage per
// section 架構實現).
//
// Shapes: 64 query heads x 512 dims, one KV head; every attended item is its
// own key and value.  Work item = (query row, split) over a contiguous range
// of the row's item slots (pooled slots first, then window tokens), taken in
// tiles of 128 items.  Per tile:
//
//   S^T[item][head] = K[item][:] . Q[head][:]     M=128 items, N=64, K=512
//   P^T = exp2(S^T * scale*log2e - m_head)         (softmax warps, online)
//   O^T[dim][head] += V^T[dim][item] . P^T[item][head]   4 x (M=128 dims, N=64, K=128)
//
// The dequantised tile (E4M3 x fp32 scale -> f16, or the bf16 window -> f16)
// is stored once as 8 regions of [128 items][64 dims] with 128-byte swizzled
// rows; the same bytes are the K-major A operand of the first product and
// the MN-major A operand of the second.  S^T (64 columns) and O^T (4 x 64
// columns) live in TMEM: the softmax thread of TMEM lane i owns item i's 64
// logits, and the epilogue thread of lane i owns dims i, 128+i, 256+i,
// 384+i of every head.
//
// Roles (416 threads): warps 0-3 softmax + epilogue, warps 4-11 load and
// dequantise the tile a quarter (128 dims) at a time, warp 12 issues the
// MMAs.  The per-head running max m is kept in log2 units and only raised
// when a tile's max exceeds it by more than 8 (so P <= 2^8), in which case the
// softmax warps rescale O^T in TMEM before the next P.V product.
// Bounded waits as in sm100.cuh; a role that timed out keeps iterating
// through the named barriers without waiting.
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kH = 64, kD = 512, kTileItems = 128;
constexpr int kThreads = 416;
constexpr int kProducerThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct SmemAttn {
    uint8_t kv[8][kTileItems * 128];  // 8 dim blocks x [128 items][64 f16] swizzled (128 KB)
    uint8_t q[8][kH * 128];           // 8 dim blocks x [64 heads][64 f16] swizzled (64 KB)
    uint8_t p[kTileItems * 128];      // [128 items][64 heads f16] swizzled (16 KB)
    float red_max[4][kH];
    float red_sum[4][kH];
    float m_used[kH], l_run[kH], alpha[kH], fin[kH];
    uint64_t kv_full[4], kv_empty[4], s_full, p_full, o_done, q_full;
    uint32_t tmem_base;
    int rescale;
};

// E4M3 pairs of a 32-bit word -> f16x2 (exact); low pair from bytes 0-1,
// high pair from bytes 2-3.  Only 32-bit operands cross the asm boundary.
__device__ __forceinline__ void f16x2_of_e4m3x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n"
        " cvt.rn.f16x2.e4m3x2 %0, a;\n cvt.rn.f16x2.e4m3x2 %1, b;\n}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// two bf16 (packed) -> two f16 (packed), rounding to nearest
__device__ __forceinline__ uint32_t f16x2_of_bf16x2(uint32_t v) {
    const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Slot {
    int64_t src;  // global row of the item (pooled: b*max_entries + j; raw: b*n_raw + r), -1 = empty
    int raw;
};

__device__ __forceinline__ Slot resolve_slot(const AttnArgs& a, int64_t row, int64_t b,
                                             int64_t n_kv, int64_t win_lo, int64_t slot,
                                             int64_t s_hi) {
    Slot s{-1, 0};
    if (slot >= s_hi) return s;
    if (slot < n_kv) {
        const int64_t j = a.idx ? int64_t(a.idx[row * a.k + slot]) : slot;
        if (j >= a.max_entries) flag_status(CSA_DEV_BAD_INDEX);
        else if (j >= 0) s.src = b * a.max_entries + j;
    } else {
        s.src = b * a.n_raw + (win_lo + (slot - n_kv) - a.raw_pos0[b]);
        s.raw = 1;
    }
    return s;
}

}  // namespace

// Reduce-scatter over the 32 lanes of a warp: v[0..63] per lane in, on return
// lane l holds the reduction of heads 2l, 2l+1 in r0, r1.
template <bool MAX>
__device__ __forceinline__ void warp_reduce_scatter64(float (&v)[64], float& r0, float& r1) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int half = 32 >> step;  // current live count: 64 >> step values
        const int bit = 16 >> step;   // partner distance
        const bool upper = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, bit);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    r0 = v[0];
    r1 = v[1];
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    SmemAttn& S = *reinterpret_cast<SmemAttn*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using namespace sm100;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t row = blockIdx.y;
    const int split = blockIdx.x;
    const int64_t b = row / a.n_q;
    const int64_t t = a.q_pos[row];
    const int64_t n_kv = a.idx ? a.k : min(n_elig(t, a.m, a.W), a.max_entries);
    const int64_t p0 = a.raw_pos0[b];
    const int64_t win_lo = max(max(t - a.W + 1, int64_t(0)), p0);
    const int64_t n_win = max(int64_t(0), min(t + 1, p0 + a.n_raw) - win_lo);
    const int64_t total = n_kv + n_win;
    const int64_t per = ceil_div(total, a.n_splits);
    const int64_t s_lo = min(total, split * per), s_hi = min(total, s_lo + per);
    const int n_tiles = int(ceil_div(s_hi - s_lo, kTileItems));

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) { mbar_init(&S.kv_full[i], kProducerThreads); mbar_init(&S.kv_empty[i], 1); }
        mbar_init(&S.s_full, 1);
        mbar_init(&S.p_full, 128);
        mbar_init(&S.o_done, 1);
        mbar_init(&S.q_full, kProducerThreads);
        fence_mbar_init();
    }
    if (threadIdx.x < kH) {
        S.m_used[threadIdx.x] = -INFINITY;
        S.l_run[threadIdx.x] = 0.f;
    }
    if (threadIdx.x == 0) S.rescale = 0;
    if (warp == 12) { tmem_alloc(&S.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tS = tmem, tO = tmem + 64;  // S^T: cols [0,64); O^T quarter q: cols [64+64q, 128+64q)

    if (warp >= 4 && warp < 12) {
        // ---------------------------------------------------------- producers
        const int pt = threadIdx.x - 128;  // 0..255
        const int c = pt & 15;             // 8-dim unit within a 128-dim quarter
        if (n_tiles > 0) {
            // query: 64 heads x 512 bf16 -> f16, K-major B tile (8 dim blocks)
            const uint16_t* qg = (const uint16_t*)a.q + row * int64_t(kH) * kD;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {  // 2 x 8 independent 16-byte loads per thread
                uint4 v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = pt + kProducerThreads * (8 * half + j);
                    v[j] = *reinterpret_cast<const uint4*>(qg + (u >> 6) * kD + (u & 63) * 8);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = pt + kProducerThreads * (8 * half + j);
                    const int h = u >> 6, cc = u & 63;  // 8-dim chunk cc of head h
                    const uint4 o = make_uint4(f16x2_of_bf16x2(v[j].x), f16x2_of_bf16x2(v[j].y),
                                               f16x2_of_bf16x2(v[j].z), f16x2_of_bf16x2(v[j].w));
                    *reinterpret_cast<uint4*>(S.q[cc >> 3] + sw128_offset(h, cc & 7)) = o;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&S.q_full);
        }
        // Software pipeline over (tile, quarter) steps: the loads of step g+1
        // are issued before step g waits for its buffer and converts, so two
        // quarters of loads are in flight per thread.
        const int n_steps = 4 * n_tiles;
        int64_t src[8];  // source rows of this thread's 8 items in the tile being loaded
        uint4 raw[2][8];
        float sc[2][8];
        // buffers are compile-time indices (the step loop is unrolled by two)
        auto issue = [&](auto bufc, int g) {
            constexpr int buf = decltype(bufc)::value;
            const int tile = g >> 2, qt = g & 3;
            const int64_t slot0 = s_lo + int64_t(tile) * kTileItems + (pt >> 4);
            if (qt == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    src[i] = resolve_slot(a, row, b, n_kv, win_lo, slot0 + 16 * i, s_hi).src;
            }
            const int dim0 = 128 * qt + 8 * c;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                raw[buf][i] = make_uint4(0, 0, 0, 0);
                sc[buf][i] = 0.f;
                if (src[i] >= 0) {
                    if (slot0 + 16 * i >= n_kv) {  // a window token (bf16)
                        raw[buf][i] = *reinterpret_cast<const uint4*>((const uint16_t*)a.raw + src[i] * kD + dim0);
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2*>((const uint8_t*)a.kv + src[i] * kD + dim0);
                        raw[buf][i] = make_uint4(v.x, v.y, 0, 0);
                        sc[buf][i] = ((const float*)a.kv_s)[src[i] * (kD / 64) + (dim0 >> 6)];
                    }
                }
            }
        };
        auto step = [&](auto bufc, int g) -> bool {
            constexpr int buf = decltype(bufc)::value;
            const int tile = g >> 2, qt = g & 3;
            if (g + 1 < n_steps) issue(std::integral_constant<int, buf ^ 1>{}, g + 1);
            if (tile > 0 && !mbar_wait(&S.kv_empty[qt], uint32_t((tile - 1) & 1))) return false;
            const int64_t slot0 = s_lo + int64_t(tile) * kTileItems + (pt >> 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = (pt >> 4) + 16 * i;
                uint4 o;
                if (slot0 + 16 * i >= n_kv) {  // window token (or past the end: zeros either way)
                    const uint4 r = raw[buf][i];
                    o = make_uint4(f16x2_of_bf16x2(r.x), f16x2_of_bf16x2(r.y), f16x2_of_bf16x2(r.z),
                                   f16x2_of_bf16x2(r.w));
                } else {
                    const float scl = sc[buf][i];
                    if (scl != 0.f && (scl < 6.103515625e-05f || scl > 146.0f)) flag_status(CSA_DEV_RANGE);
                    const __half2 h2 = __float2half2_rn(scl);
                    const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&h2);
                    uint32_t f0, f1, f2, f3;
                    f16x2_of_e4m3x4(raw[buf][i].x, f0, f1);
                    f16x2_of_e4m3x4(raw[buf][i].y, f2, f3);
                    o = make_uint4(hmul2(f0, s2), hmul2(f1, s2), hmul2(f2, s2), hmul2(f3, s2));
                }
                *reinterpret_cast<uint4*>(S.kv[2 * qt + (c >> 3)] + sw128_offset(e, c & 7)) = o;
            }
            fence_proxy_async_smem();
            mbar_arrive(&S.kv_full[qt]);
            return true;
        };
        bool ok = true;
        if (n_steps > 0) issue(std::integral_constant<int, 0>{}, 0);
        for (int g = 0; g < n_steps && ok; g += 2) {
            ok = step(std::integral_constant<int, 0>{}, g);
            if (ok && g + 1 < n_steps) ok = step(std::integral_constant<int, 1>{}, g + 1);
        }
    } else if (warp == 12) {
        // --------------------------------------------------------------- MMA
        if (lane == 0 && n_tiles > 0) {
            const uint32_t id_qk = instr_desc(0, 0, 0, 0, 128, 64);  // f16 x f16, both K-major
            const uint32_t id_pv = instr_desc(0, 0, 1, 1, 128, 64);  // f16 x f16, both MN-major
            const uint32_t kv0 = smem_u32(S.kv[0]), q0 = smem_u32(S.q[0]), pp = smem_u32(S.p);
            bool ok = mbar_wait(&S.q_full, 0);
            for (int tile = 0; tile < n_tiles && ok; ++tile) {
                const uint32_t ph = uint32_t(tile & 1);
                for (int qt = 0; qt < 4 && ok; ++qt) {
                    ok = mbar_wait(&S.kv_full[qt], ph);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const int blk = 2 * qt + (s >> 2);
                        mma_f16(tS, smem_desc(kv0 + blk * 16384 + (s & 3) * 32, 16, 1024),
                                smem_desc(q0 + blk * 8192 + (s & 3) * 32, 16, 1024), id_qk,
                                (qt | s) != 0);
                    }
                }
                if (!ok) break;
                mma_commit(&S.s_full);
                ok = mbar_wait(&S.p_full, ph);
                if (!ok) break;
                tc_fence_after();
                for (int qt = 0; qt < 4; ++qt) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_f16(tO + 64 * qt, smem_desc(kv0 + (2 * qt) * 16384 + ks * 2048, 16384, 1024),
                                smem_desc(pp + ks * 2048, 8192, 1024), id_pv, (tile | ks) != 0);
                    mma_commit(&S.kv_empty[qt]);
                }
                mma_commit(&S.o_done);
            }
        }
    } else {
        // ------------------------------------------------- softmax + epilogue
        const int sub = warp;                    // warps 0..3 = TMEM lane quarters
        const int e = sub * 32 + lane;           // item of the tile / dim within a quarter
        const float sl2 = a.scale * kLog2e;
        bool ok = true;
        for (int tile = 0; tile < n_tiles; ++tile) {
            const Slot me = resolve_slot(a, row, b, n_kv, win_lo, s_lo + int64_t(tile) * kTileItems + e, s_hi);
            if (ok) ok = mbar_wait(&S.s_full, uint32_t(tile & 1));
            if (ok) tc_fence_after();
            const uint32_t srow = tS + (uint32_t(sub * 32) << 16);
            float x[64];
            // pass 1: scaled logits -> per-head max over the tile
            if (ok) tmem_ld64(srow, x);
#pragma unroll
            for (int h = 0; h < 64; ++h) x[h] = (ok && me.src >= 0) ? x[h] * sl2 : -INFINITY;
            float r0, r1;
            warp_reduce_scatter64<true>(x, r0, r1);
            S.red_max[sub][2 * lane] = r0;
            S.red_max[sub][2 * lane + 1] = r1;
            named_bar(1, 128);
            if (threadIdx.x < kH) {
                const int h = threadIdx.x;
                // fold the previous tile's sums (relative to the old max) in first
                float l = S.l_run[h];
                if (tile > 0) l += S.red_sum[0][h] + S.red_sum[1][h] + S.red_sum[2][h] + S.red_sum[3][h];
                const float tmax = fmaxf(fmaxf(S.red_max[0][h], S.red_max[1][h]), fmaxf(S.red_max[2][h], S.red_max[3][h]));
                const float mold = S.m_used[h];
                float al = 1.f;
                if (tmax > mold + kRescaleThreshold || (mold == -INFINITY && tmax != -INFINITY)) {
                    al = mold == -INFINITY ? 0.f : ex2(mold - tmax);
                    S.m_used[h] = tmax;
                    if (mold != -INFINITY) S.rescale = 1;
                }
                S.alpha[h] = al;
                S.l_run[h] = l * al;
            }
            named_bar(1, 128);
            // pass 2: re-read the logits, P^T row e = exp2(x - m) as f16 into the
            // MN-major B tile
            if (ok) tmem_ld64(srow, x);
#pragma unroll
            for (int h = 0; h < 64; ++h) {
                const float mh = S.m_used[h];
                x[h] = (ok && me.src >= 0) ? ex2(x[h] * sl2 - mh) : 0.f;
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t w4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __half2 hh = __floats2half2_rn(x[8 * ch + 2 * k], x[8 * ch + 2 * k + 1]);
                    w4[k] = *reinterpret_cast<const uint32_t*>(&hh);
                }
                *reinterpret_cast<uint4*>(S.p + sw128_offset(e, ch)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            warp_reduce_scatter64<false>(x, r0, r1);
            S.red_sum[sub][2 * lane] = r0;
            S.red_sum[sub][2 * lane + 1] = r1;
            // rescale O^T (columns = heads) for heads whose max was raised; the
            // previous P.V is complete (s_full of this tile follows it) and the
            // next one waits for p_full
            const bool need = S.rescale != 0;
            if (ok && need) {
#pragma unroll 1
                for (int qc = 0; qc < 16; ++qc) {  // 16-column chunks; rolled to keep registers free
                    const int qt = qc >> 2, cc = qc & 3;
                    {
                        float o16[16];
                        const uint32_t ad = tO + 64 * qt + 16 * cc + (uint32_t(sub * 32) << 16);
                        tmem_ld16(ad, o16);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k) o16[k] *= S.alpha[16 * cc + k];
                        tmem_st16(ad, o16);
                    }
                }
                tmem_wait_st();
            }
            named_bar(1, 128);  // everyone has read S.rescale / alpha before it is reset
            if (threadIdx.x == 0) S.rescale = 0;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&S.p_full);
        }
        // ----------------------------------------------------------- epilogue
        named_bar(1, 128);
        if (threadIdx.x < kH) {
            const int h = threadIdx.x;
            float l = S.l_run[h];
            if (n_tiles > 0) l += S.red_sum[0][h] + S.red_sum[1][h] + S.red_sum[2][h] + S.red_sum[3][h];
            const float m = S.m_used[h];
            if (a.n_splits == 1) {
                float f = 1.f, den = l;
                if (a.sinks) {
                    const float sg = a.sinks[h] * kLog2e;
                    const float M = fmaxf(m, sg);
                    f = m == -INFINITY ? 0.f : ex2(m - M);
                    den = l * f + ex2(sg - M);
                }
                S.fin[h] = den > 0.f ? f / den : 0.f;
            } else {
                const int64_t item = row * a.n_splits + split;
                a.part_ml[item * kH + h] = make_float2(m == -INFINITY ? -INFINITY : m / kLog2e, l);
                S.fin[h] = 1.f;
            }
        }
        named_bar(1, 128);
        if (n_tiles > 0 && ok) ok = mbar_wait(&S.o_done, uint32_t((n_tiles - 1) & 1));
        tc_fence_after();
        for (int qt = 0; qt < 4; ++qt) {
            const int dim = 128 * qt + e;
            float o[64];
            if (n_tiles > 0 && ok) {
                float o16[4][16];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    tmem_ld16(tO + 64 * qt + 16 * cc + (uint32_t(sub * 32) << 16), o16[cc]);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 64; ++h) o[h] = o16[h >> 4][h & 15];
            } else {
#pragma unroll
                for (int h = 0; h < 64; ++h) o[h] = 0.f;
            }
            if (a.n_splits == 1) {
                __nv_bfloat16* out = (__nv_bfloat16*)a.out + row * int64_t(kH) * kD;
#pragma unroll
                for (int h = 0; h < 64; ++h) out[h * kD + dim] = __float2bfloat16_rn(o[h] * S.fin[h]);
            } else {
                float* po = a.part_o + (row * a.n_splits + split) * int64_t(kH) * kD;
#pragma unroll
                for (int h = 0; h < 64; ++h) po[h * kD + dim] = o[h];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 12) tmem_dealloc(tmem, 512);
}

bool attn_tc_supported(int act, int kvf, int H, int D) {
    return act == CSA_BF16 && kvf == CSA_FP8_S64 && H == kH && D == kD;
}

cudaError_t launch_attn_tc(const AttnArgs& a, int64_t rows, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const size_t sm = sizeof(SmemAttn) + 1024;
    cudaError_t e = ensure_smem(attn_tc_kernel, size_t(sm));
    if (e != cudaSuccess) return e;
    attn_tc_kernel<<<dim3(a.n_splits, unsigned(rows)), kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
