// MQA attention over FP8 pooled entries + the bf16 raw window + a per-head
// sink on the 5th-generation tensor cores (wiki summary "DeepSeek V4",
// section 架构创新: top-k sparse selection + MQA, sliding-window branch,
// attention sink; release note sections CSA and HCA; FP8 KV storage per
// section 架構實現).
//
// Shapes: 64 query heads x 512 dims, one KV head; every attended item is its
// own key and value.  Work item = (query row, split) over a contiguous range
// of the row's item slots (pooled slots first, then window tokens), taken in
// tiles of 64 items:
//
//   S[head][item]   = Q[head][:] . K[item][:]           M=64 heads, N=64 items, K=512
//   P[head][item]   = exp2(S * scale*log2e - m_head)     (one softmax thread per head)
//   O^T[dim][head] += V^T[dim][item] . P[head][item]^T   4 x (M=128 dims, N=64, K=64)
//
// The dequantised tile (E4M3 x fp32 scale -> f16, or the bf16 window -> f16)
// is stored once as 8 regions of [64 items][64 dims] with 128-byte swizzled
// rows: the K-major B operand of the first product and the MN-major A operand
// of the second.  Two tile buffers let the loaders fill tile t+1 while tile t
// is multiplied.  S (M=64: head h in TMEM lane 32*(h/16) + h%16) is double
// buffered in TMEM so QK of tile t+1 runs while the softmax works on tile t;
// O^T takes 4 x 64 columns, one dim per lane.
//
// Roles (416 threads): warps 0-3 softmax (lanes 0-15: one head each) and
// epilogue (all 128 lanes: one dim each per quarter), warps 4-11 load and
// dequantise with kLook quarter-steps of loads in flight per thread, warp 12
// issues the MMAs as their inputs become ready: QK of the next tile quarter
// by quarter, and P.V of the current tile as soon as its P is written, so a
// slow load of tile t+1 never holds back P.V of tile t.  The running max is kept per head in
// log2 units and raised only when a tile exceeds it by more than 8, in which
// case O^T is rescaled in TMEM before the next P.V.  Bounded waits (sm100.cuh).
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kH = 64, kD = 512, kTile = 64;
constexpr int kProducerWarps = 8;
constexpr int kProducerThreads = 32 * kProducerWarps;
constexpr int kMmaWarp = 4 + kProducerWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kUnits = kTile * 16 / kProducerThreads;  // 8-dim units per thread per quarter (4)
constexpr int kLook = 2;                               // quarter-steps of loads in flight ahead
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct SmemAttn {
    uint8_t kv[2][8][kTile * 128];  // 2 buffers x 8 dim blocks x [64 items][64 f16] (128 KB)
    uint8_t q[8][kH * 128];         // 8 dim blocks x [64 heads][64 f16] (64 KB)
    uint8_t p[2][kH * 128];         // 2 buffers x [64 heads][64 items f16] (16 KB)
    float alpha[kH], fin[kH];
    uint64_t kv_full[2][4], kv_empty[2][4], s_full[2], p_full[2], o_done, q_full;
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

// Row of slot `slot` within the sequence's own buffer (pooled entry j, or
// window row r of the raw buffer), or -1 when the slot is empty or past the
// range.  Rows fit in 32 bits (checked on the host).
__device__ __forceinline__ int32_t slot_source(const AttnArgs& a, int64_t row, int64_t n_kv,
                                               int64_t win_lo, int64_t raw_pos0, int64_t slot,
                                               int64_t s_hi) {
    if (slot >= s_hi) return -1;
    if (slot < n_kv) {
        const int64_t j = a.idx ? int64_t(a.idx[row * a.k + slot]) : slot;
        if (j >= a.max_entries) {
            flag_status(CSA_DEV_BAD_INDEX);
            return -1;
        }
        return j >= 0 ? int32_t(j) : -1;
    }
    return int32_t(win_lo + (slot - n_kv) - raw_pos0);
}

}  // namespace

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
    const int n_tiles = int(ceil_div(s_hi - s_lo, kTile));

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            for (int q = 0; q < 4; ++q) { mbar_init(&S.kv_full[i][q], kProducerThreads); mbar_init(&S.kv_empty[i][q], 1); }
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], 128);
        }
        mbar_init(&S.o_done, 1);
        mbar_init(&S.q_full, kProducerThreads);
        S.rescale = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) { tmem_alloc(&S.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tS = tmem, tO = tmem + 128;  // S[buf]: cols [64 buf, 64 buf + 64); O^T quarter q: [128+64q, 192+64q)
    const uint8_t* kv_seq = (const uint8_t*)a.kv + b * a.max_entries * int64_t(kD);
    const float* kvs_seq = (const float*)a.kv_s + b * a.max_entries * int64_t(kD / 64);
    const uint16_t* raw_seq = (const uint16_t*)a.raw + b * a.n_raw * int64_t(kD);

    if (warp >= 4 && warp < kMmaWarp) {
        // ---------------------------------------------------------- producers
        const int pt = threadIdx.x - 128;  // 0..kProducerThreads-1
        const int c = pt & 15;             // 8-dim unit within a 128-dim quarter
        const int e0 = pt >> 4;            // items e0 + 16 u, u < kUnits
        if (n_tiles > 0) {
            // query: 64 heads x 512 bf16 -> f16, K-major (A operand): 4096 16-byte
            // chunks, 8 loads in flight per thread
            const uint16_t* qg = (const uint16_t*)a.q + row * int64_t(kH) * kD;
            static_assert((kH * kD / 8) % (8 * kProducerThreads) == 0, "query chunks per batch");
#pragma unroll 1
            for (int base = 0; base < kH * kD / 8; base += 8 * kProducerThreads) {
                uint4 v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = base + pt + kProducerThreads * j;
                    v[j] = *reinterpret_cast<const uint4*>(qg + (u >> 6) * kD + (u & 63) * 8);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int u = base + pt + kProducerThreads * j;
                    const int h = u >> 6, cc = u & 63;
                    *reinterpret_cast<uint4*>(S.q[cc >> 3] + sw128_offset(h, cc & 7)) =
                        make_uint4(f16x2_of_bf16x2(v[j].x), f16x2_of_bf16x2(v[j].y),
                                   f16x2_of_bf16x2(v[j].z), f16x2_of_bf16x2(v[j].w));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&S.q_full);
        }
        // Software pipeline over (tile, quarter) steps g: the loads of steps
        // g+1 .. g+kLook are in flight while step g waits for its buffer and is
        // converted.  Register buffers are compile-time indices (the step loop
        // is unrolled by kLook+1).
        constexpr int kBufs = kLook + 1;
        const int n_steps = 4 * n_tiles;
        int32_t src[kBufs][kUnits];
        uint4 raw[kBufs][kUnits];
        float sc[kBufs][kUnits];
        auto issue = [&](auto bufc, int g) {
            constexpr int buf = decltype(bufc)::value;
            constexpr int prev = (buf + kBufs - 1) % kBufs;
            const int tile = g >> 2, qt = g & 3;
            const int64_t slot0 = s_lo + int64_t(tile) * kTile + e0;
            const int dim0 = 128 * qt + 8 * c;
#pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                // sources are resolved once per tile (quarter 0), then carried
                const int32_t sr = qt == 0 ? slot_source(a, row, n_kv, win_lo, p0, slot0 + 16 * u, s_hi)
                                           : src[prev][u];
                src[buf][u] = sr;
                raw[buf][u] = make_uint4(0, 0, 0, 0);
                sc[buf][u] = 0.f;
                if (sr >= 0) {
                    if (slot0 + 16 * u >= n_kv) {  // window token (bf16)
                        raw[buf][u] = *reinterpret_cast<const uint4*>(raw_seq + int64_t(sr) * kD + dim0);
                    } else {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(kv_seq + int64_t(sr) * kD + dim0);
                        raw[buf][u] = make_uint4(w2.x, w2.y, 0, 0);
                        sc[buf][u] = kvs_seq[int64_t(sr) * (kD / 64) + (dim0 >> 6)];
                    }
                }
            }
        };
        auto step = [&](auto bufc, int g) -> bool {
            constexpr int buf = decltype(bufc)::value;
            const int tile = g >> 2, qt = g & 3, kb = tile & 1;
            if (g + kLook < n_steps) issue(std::integral_constant<int, (buf + kLook) % kBufs>{}, g + kLook);
            if (tile >= 2 && !mbar_wait(&S.kv_empty[kb][qt], uint32_t(((tile >> 1) - 1) & 1))) return false;
            const int64_t slot0 = s_lo + int64_t(tile) * kTile + e0;
#pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                uint4 o = make_uint4(0, 0, 0, 0);
                if (src[buf][u] >= 0) {
                    if (slot0 + 16 * u >= n_kv) {
                        const uint4 r = raw[buf][u];
                        o = make_uint4(f16x2_of_bf16x2(r.x), f16x2_of_bf16x2(r.y), f16x2_of_bf16x2(r.z),
                                       f16x2_of_bf16x2(r.w));
                    } else {
                        const float scl = sc[buf][u];
                        if (scl < 6.103515625e-05f || scl > 146.0f) flag_status(CSA_DEV_RANGE);
                        const __half2 h2 = __float2half2_rn(scl);
                        const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&h2);
                        uint32_t f0, f1, f2, f3;
                        f16x2_of_e4m3x4(raw[buf][u].x, f0, f1);
                        f16x2_of_e4m3x4(raw[buf][u].y, f2, f3);
                        o = make_uint4(hmul2(f0, s2), hmul2(f1, s2), hmul2(f2, s2), hmul2(f3, s2));
                    }
                }
                *reinterpret_cast<uint4*>(S.kv[kb][2 * qt + (c >> 3)] + sw128_offset(e0 + 16 * u, c & 7)) = o;
            }
            fence_proxy_async_smem();
            mbar_arrive(&S.kv_full[kb][qt]);
            return true;
        };
        using I0 = std::integral_constant<int, 0>;
        using I1 = std::integral_constant<int, 1>;
        using I2 = std::integral_constant<int, 2>;
        static_assert(kBufs == 3, "the unrolled step loop below assumes three buffers");
        if (n_steps > 0) issue(I0{}, 0);
        if (n_steps > 1) issue(I1{}, 1);
        bool ok = true;
        for (int g = 0; g < n_steps && ok; g += kBufs) {
            ok = step(I0{}, g);
            if (ok && g + 1 < n_steps) ok = step(I1{}, g + 1);
            if (ok && g + 2 < n_steps) ok = step(I2{}, g + 2);
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------------------- MMA
        if (lane == 0 && n_tiles > 0) {
            const uint32_t id_qk = instr_desc(0, 0, 0, 0, 64, 64);   // f16: A = Q K-major, B = K K-major
            const uint32_t id_pv = instr_desc(0, 0, 1, 0, 128, 64);  // f16: A = V^T MN-major, B = P K-major
            const uint32_t q0 = smem_u32(S.q[0]);
            bool ok = mbar_wait(&S.q_full, 0);
            // QK(t) may run at most one tile ahead of P.V: it overwrites S[t&1],
            // which the softmax of tile t-2 has finished reading once P.V(t-2)
            // has been issued.  Each wait is a single poll; the loop as a whole
            // is bounded by kWaitNs without progress.
            int qk_t = 0, qk_q = 0, pv_t = 0;
            uint64_t t_last = global_ns();
            while (ok && pv_t < n_tiles) {
                bool progressed = false;
                if (qk_t < n_tiles && qk_t <= pv_t + 1) {
                    const int kb = qk_t & 1;
                    if (mbar_try_wait(&S.kv_full[kb][qk_q], uint32_t((qk_t >> 1) & 1))) {
                        tc_fence_after();
                        const uint32_t kv0 = smem_u32(S.kv[kb][0]);
#pragma unroll
                        for (int s = 0; s < 8; ++s) {
                            const int blk = 2 * qk_q + (s >> 2);
                            mma_f16(tS + 64 * kb, smem_desc(q0 + blk * 8192 + (s & 3) * 32, 16, 1024),
                                    smem_desc(kv0 + blk * 8192 + (s & 3) * 32, 16, 1024), id_qk,
                                    (qk_q | s) != 0);
                        }
                        if (++qk_q == 4) {
                            mma_commit(&S.s_full[kb]);
                            qk_q = 0;
                            ++qk_t;
                        }
                        progressed = true;
                    }
                }
                if (pv_t < qk_t) {
                    const int kb = pv_t & 1;
                    if (mbar_try_wait(&S.p_full[kb], uint32_t((pv_t >> 1) & 1))) {
                        tc_fence_after();
                        const uint32_t kv0 = smem_u32(S.kv[kb][0]), pp = smem_u32(S.p[kb]);
                        for (int qt = 0; qt < 4; ++qt) {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_f16(tO + 64 * qt, smem_desc(kv0 + (2 * qt) * 8192 + ks * 2048, 8192, 1024),
                                        smem_desc(pp + ks * 32, 16, 1024), id_pv, (pv_t | ks) != 0);
                            mma_commit(&S.kv_empty[kb][qt]);
                        }
                        mma_commit(&S.o_done);
                        ++pv_t;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_last = global_ns();
                } else if (global_ns() - t_last > kWaitNs) {
                    flag_status(CSA_DEV_TIMEOUT);
                    ok = false;
                }
            }
        }
    } else {
        // ------------------------------------------------- softmax + epilogue
        const int sub = warp;                        // warps 0..3 = TMEM lane quarters
        const bool head_lane = lane < 16;
        const int h = 16 * sub + (lane & 15);        // head of this lane (head lanes only)
        const float sl2 = a.scale * kLog2e;
        float m_run = -INFINITY, l_run = 0.f;        // per head, log2 units
        bool ok = true;
        // item validity (slot < s_hi and a pooled id in range, or a window
        // token) as a 64-bit mask built from two coalesced loads per lane and
        // ballots; the loads for tile t+1 are issued while tile t is processed
        auto load_ids = [&](int tt, int32_t& j0, int32_t& j1) {
            const int64_t s0 = s_lo + int64_t(tt) * kTile + lane, s1 = s0 + 32;
            j0 = (a.idx && s0 < min(s_hi, n_kv)) ? a.idx[row * a.k + s0] : 0;
            j1 = (a.idx && s1 < min(s_hi, n_kv)) ? a.idx[row * a.k + s1] : 0;
        };
        auto mask_of = [&](int tt, int32_t j0, int32_t j1, unsigned& vm0, unsigned& vm1) {
            const int64_t s0 = s_lo + int64_t(tt) * kTile + lane, s1 = s0 + 32;
            vm0 = __ballot_sync(0xffffffffu, s0 < s_hi && (s0 >= n_kv || (j0 >= 0 && j0 < a.max_entries)));
            vm1 = __ballot_sync(0xffffffffu, s1 < s_hi && (s1 >= n_kv || (j1 >= 0 && j1 < a.max_entries)));
        };
        // Warm L2 with every row this work item reads (pooled FP8 rows with
        // their scales, bf16 window rows) while the loaders fetch the query:
        // their gathers then hit L2 instead of waiting on HBM one by one.
        for (int64_t sl = s_lo + threadIdx.x; sl < s_hi; sl += 128) {
            const int32_t sr = slot_source(a, row, n_kv, win_lo, p0, sl, s_hi);
            if (sr < 0) continue;
            if (sl >= n_kv) {
                prefetch_l2_bulk(raw_seq + int64_t(sr) * kD, kD * 2);
            } else {
                prefetch_l2_bulk(kv_seq + int64_t(sr) * kD, kD);
                prefetch_l2_bulk(kvs_seq + int64_t(sr) * (kD / 64), (kD / 64) * 4);
            }
        }
        int32_t nj0 = 0, nj1 = 0;
        if (n_tiles > 0) load_ids(0, nj0, nj1);
        for (int tile = 0; tile < n_tiles; ++tile) {
            const int kb = tile & 1;
            unsigned vm0, vm1;
            mask_of(tile, nj0, nj1, vm0, vm1);
            if (tile + 1 < n_tiles) load_ids(tile + 1, nj0, nj1);
            if (ok) ok = mbar_wait(&S.s_full[kb], uint32_t((tile >> 1) & 1));
            if (ok) tc_fence_after();
            const uint32_t srow = tS + 64 * kb + (uint32_t(sub * 32) << 16);
            // pass 1: max of the scaled, masked logits (two 32-item halves)
            float mx = -INFINITY;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {  // rolled: one 32-column half live at a time
                float x[32];
                if (ok) tmem_ld32(srow + 32 * hf, x);
                const unsigned vm = hf ? vm1 : vm0;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (ok && ((vm >> i) & 1u)) mx = fmaxf(mx, x[i] * sl2);
            }
            float al = 1.f;
            if (mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx != -INFINITY)) {
                al = m_run == -INFINITY ? 0.f : ex2(m_run - mx);
                m_run = mx;
            }
            // P.V of the previous tile must be done before P[kb] (read by P.V
            // two tiles back) is rewritten and before O^T is rescaled
            if (ok && tile > 0) ok = mbar_wait(&S.o_done, uint32_t((tile - 1) & 1));
            // pass 2: P = exp2(x - m) as f16 rows of the K-major B tile, and the sum
            float sum = 0.f;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                float x[32];
                if (ok) tmem_ld32(srow + 32 * hf, x);
                const unsigned vm = hf ? vm1 : vm0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = (ok && ((vm >> i) & 1u)) ? ex2(x[i] * sl2 - m_run) : 0.f;
                    sum += x[i];
                }
                if (head_lane) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t w4[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const __half2 hh = __floats2half2_rn(x[8 * ch + 2 * k], x[8 * ch + 2 * k + 1]);
                            w4[k] = *reinterpret_cast<const uint32_t*>(&hh);
                        }
                        *reinterpret_cast<uint4*>(S.p[kb] + sw128_offset(h, 4 * hf + ch)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            l_run = l_run * al + sum;
            if (head_lane) {
                S.alpha[h] = al;
                if (al != 1.f && tile > 0) S.rescale = 1;
            }
            named_bar(1, 128);
            if (ok && S.rescale != 0) {
                tc_fence_after();
#pragma unroll 1
                for (int qc = 0; qc < 16; ++qc) {  // 16-column chunks of O^T; rolled to keep registers free
                    const int qt = qc >> 2, cc = qc & 3;
                    float o16[16];
                    const uint32_t ad = tO + 64 * qt + 16 * cc + (uint32_t(sub * 32) << 16);
                    tmem_ld16(ad, o16);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k) o16[k] *= S.alpha[16 * cc + k];
                    tmem_st16(ad, o16);
                }
                tmem_wait_st();
            }
            named_bar(1, 128);  // everyone has read S.rescale before it is reset
            if (threadIdx.x == 0) S.rescale = 0;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&S.p_full[kb]);
        }
        // ----------------------------------------------------------- epilogue
        if (head_lane) {
            if (a.n_splits == 1) {
                float f = 1.f, den = l_run;
                if (a.sinks) {
                    const float sg = a.sinks[h] * kLog2e;
                    const float M = fmaxf(m_run, sg);
                    f = m_run == -INFINITY ? 0.f : ex2(m_run - M);
                    den = l_run * f + ex2(sg - M);
                }
                S.fin[h] = den > 0.f ? f / den : 0.f;
            } else {
                const int64_t item = row * a.n_splits + split;
                a.part_ml[item * kH + h] = make_float2(m_run == -INFINITY ? -INFINITY : m_run / kLog2e, l_run);
                S.fin[h] = 1.f;
            }
        }
        named_bar(1, 128);
        if (n_tiles > 0 && ok) ok = mbar_wait(&S.o_done, uint32_t((n_tiles - 1) & 1));
        tc_fence_after();
        const int e = sub * 32 + lane;
        for (int qt = 0; qt < 4; ++qt) {
            const int dim = 128 * qt + e;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                float o[32];
                if (n_tiles > 0 && ok) {
                    tmem_ld32(tO + 64 * qt + 32 * hf + (uint32_t(sub * 32) << 16), o);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0.f;
                }
                if (a.n_splits == 1) {
                    __nv_bfloat16* out = (__nv_bfloat16*)a.out + row * int64_t(kH) * kD;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int hh = 32 * hf + i;
                        out[hh * kD + dim] = __float2bfloat16_rn(o[i] * S.fin[hh]);
                    }
                } else {
                    float* po = a.part_o + (row * a.n_splits + split) * int64_t(kH) * kD;
#pragma unroll
                    for (int i = 0; i < 32; ++i) po[(32 * hf + i) * kD + dim] = o[i];
                }
            }
        }
    }
    // the producer and MMA roles run on one lane: reconverge every warp so
    // that the CTA barrier (an aligned bar.sync) sees whole warps and really
    // waits for those lanes before TMEM is freed
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

bool attn_tc_supported(int act, int kvf, int H, int D) {
    return act == CSA_BF16 && kvf == CSA_FP8_S64 && H == kH && D == kD;
}

bool attn_tc_rows_fit(int64_t max_entries, int64_t n_raw) {
    return max_entries < (int64_t(1) << 31) && n_raw < (int64_t(1) << 31);
}

cudaError_t launch_attn_tc(const AttnArgs& a, int64_t rows, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const size_t sm = sizeof(SmemAttn) + 1024;
    cudaError_t e = ensure_smem(attn_tc_kernel, sm);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<<<dim3(a.n_splits, unsigned(rows)), kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
