// MQA attention over FP8 pooled entries + the bf16 raw window + a per-head
// sink on the 5th-generation tensor cores (wiki summary "DeepSeek V4",
// section 架构创新: top-k sparse selection + MQA, sliding-window branch,
// attention sink; release note sections CSA and HCA; FP8 KV storage per
// section 架構實現).
//
// Shapes: 64 query heads x 512 dims, one KV head; every attended item is its
// own key and value.  A query row's items are cut into 64-item tiles, pooled
// entries first and then the window tokens, so that no tile mixes the two;
// work item = (query row, split) over a contiguous range of those tiles:
//
//   S[head][item]   = Q[head][:] . K[item][:]           M=64 heads, N=64 items, K=512
//   P[head][item]   = exp2(S * scale*log2e - m_head)     (one softmax thread per head)
//   O^T[dim][head] += V^T[dim][item] . P[head][item]^T   4 x (M=128 dims, N=64, K=64)
//
// Operands are bf16: the query and the window tokens are used as stored,
// and each pooled E4M3 x fp32-scale value is rounded once to bf16 (the
// accumulation is fp32).  A tile is stored once as 8 regions of [64 items]
// [64 dims] with 128-byte swizzled rows: the K-major B operand of the first
// product and the MN-major A operand of the second.  Two tile buffers let
// tile t+1 be fetched and converted while tile t is multiplied.  S (M=64:
// head h in TMEM lane 32*(h/16) + h%16) is double buffered in TMEM so QK of
// tile t+1 runs while the softmax works on tile t; O^T takes 4 x 64 columns,
// one dim per lane.
//
// Data movement: the query (8 tensor copies) and window tiles (8 tensor
// copies from a [batch][n_raw][512] map; rows past the sequence read as
// zero) land directly in operand layout.  Pooled entries come in two stored
// formats (template parameter KVF):
//  * FP8: a tile's rows land by bulk copy (one per selected row, or one per
//    tile for dense HCA rows) in the upper half of the tile's own buffer and
//    are dequantised in place: dims 0..255 go to the lower half, dims
//    256..511 are read into registers before any thread overwrites the upper
//    half.
//  * bf16: selected rows are gathered by the converter warps with 16-byte
//    asynchronous copies straight to their swizzled place (unselected slots
//    are zero-filled); dense HCA tiles arrive by tensor copy like the window.
//
// Roles (448 threads): warps 0-3 softmax (lanes 0-15: one head each) and
// epilogue (all 128 lanes: one dim each per quarter), warps 4-11 convert,
// warp 12 issues the MMAs as their inputs become ready (QK of the next tile,
// and P.V of the current tile as soon as its P is written), warp 13 resolves
// the selected ids and issues the copies of each tile as soon as P.V of the
// tile two back has released its buffer.  The running max is kept per head
// in log2 units and raised only when a tile exceeds it by more than 8, in
// which case O^T is rescaled in TMEM before the next P.V.  Bounded waits
// (sm100.cuh).
#include <string.h>

#include <cooperative_groups.h>
#include <mutex>

#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kH = 64, kD = 512, kTile = 64;
constexpr int kConvWarps = 8;
constexpr int kConvThreads = 32 * kConvWarps;
constexpr int kMmaWarp = 4 + kConvWarps;
constexpr int kIssuerWarp = kMmaWarp + 1;
constexpr int kThreads = 32 * (kIssuerWarp + 1);
constexpr int kUnits = kTile * 16 / kConvThreads;  // 8-dim units per thread per quarter (4)
constexpr int kRawBlk = 4;                         // FP8 rows of a pooled tile: upper half (blocks 4..7)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct SmemAttn {
    uint8_t kv[2][8][kTile * 128];  // 2 buffers x 8 dim blocks x [64 items][64 bf16] (128 KB)
    uint8_t q[8][kH * 128];         // 8 dim blocks x [64 heads][64 bf16] (64 KB)
    uint8_t p[2][kH * 128];         // 2 buffers x [64 heads][64 items bf16] (16 KB)
    float kvs[2][kTile][kD / 64];   // per buffer: FP8 scales of the tile's items (4 KB)
    int32_t valid[2][kTile];        // per buffer: item holds data
    int32_t ids[2][kTile];          // per buffer: entry id of each item (bf16 gather), -1 if none
    float alpha[kH], fin[kH];
    float2 ml[kH];                  // cluster combine: this split's (max in log2 units, sum) per head
    float cw[8][kH], cinv[kH];      // cluster combine: weight of each split, 1 / denominator
    uint64_t raw_full[2], kv_half[2], kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done, q_full;
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

// (f16x2 x fp32 scale) -> bf16x2, the product rounded once from fp32
__device__ __forceinline__ uint32_t bf16x2_scaled(uint32_t h2, float s) {
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    const float2 f = __half22float2(h);
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(f.y * s), "f"(f.x * s));
    return r;
}

// 8 E4M3 values (two words) times their scale -> 8 bf16 (one 16-byte chunk)
__device__ __forceinline__ uint4 dequant8(uint2 w, float s) {
    uint32_t f0, f1, f2, f3;
    f16x2_of_e4m3x4(w.x, f0, f1);
    f16x2_of_e4m3x4(w.y, f2, f3);
    return make_uint4(bf16x2_scaled(f0, s), bf16x2_scaled(f1, s), bf16x2_scaled(f2, s),
                      bf16x2_scaled(f3, s));
}

// 16-byte global -> shared copy that bypasses L1; fewer than 16 source bytes
// (here 0) zero-fill the destination
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sm100::smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace

template <int KVF>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_win,
                   const __grid_constant__ CUtensorMap map_kv, const AttnArgs a) {
    static_assert(KVF == CSA_FP8_S64 || KVF == CSA_BF16, "pooled entries are FP8 or bf16");
    constexpr bool kFp8 = KVF == CSA_FP8_S64;
    extern __shared__ uint8_t smem_raw[];
    SmemAttn& S = *reinterpret_cast<SmemAttn*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using namespace sm100;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t row = a.row_base + blockIdx.y;
    const int split = blockIdx.x;
    const int64_t b = row / a.n_q;
    const int64_t t = a.q_pos[row];
    const int64_t n_kv = a.idx ? (a.n_sel ? min(int64_t(a.n_sel[row]), int64_t(a.k)) : a.k)
                               : min(max(n_elig(t, a.m, a.W) - a.kv_base, int64_t(0)), a.max_entries);
    const int64_t p0 = a.raw_pos0[b];
    const int64_t win_lo = max(max(t - a.W + 1, int64_t(0)), p0);
    const int64_t n_win = max(int64_t(0), min(t + 1, p0 + a.n_raw) - win_lo);
    const int kv_tiles = int(ceil_div(n_kv, kTile)), win_tiles = int(ceil_div(n_win, kTile));
    const int total_tiles = kv_tiles + win_tiles;
    const int per = int(ceil_div(total_tiles, a.n_splits));
    const int tile0 = min(total_tiles, split * per);
    const int n_tiles = min(total_tiles, tile0 + per) - tile0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.raw_full[i], 2);  // expect_tx arrival + arrival after the ids / scales
            mbar_init(&S.kv_half[i], kConvWarps);  // one arrival per converter warp: dims 0..255 ready
            mbar_init(&S.kv_full[i], kConvWarps);  // one arrival per converter warp
            mbar_init(&S.kv_empty[i], 1);
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], 4);            // one arrival per softmax warp
        }
        mbar_init(&S.o_done, 1);
        mbar_init(&S.q_full, 1);
        S.rescale = 0;
        fence_mbar_init();
        // the query's copy starts now, while TMEM is allocated and the CTA
        // meets (this thread initialised its barrier)
        prefetch_tmap(&map_win);
        prefetch_tmap(&map_kv);
        if (n_tiles > 0) {
            mbar_arrive_expect_tx(&S.q_full, uint32_t(kH * kD * 2));
#pragma unroll
            for (int blk = 0; blk < 8; ++blk)
                tma_load_2d(S.q[blk], &map_q, 64 * blk, int32_t(row * kH), &S.q_full);
        }
    }
    if (warp == kMmaWarp) { tmem_alloc(&S.tmem_base, 512); tmem_relinquish(); }
    // the issuer reads the first tile's selected ids before the CTA barrier
    int32_t ids0[2] = {-1, -1};
    if (warp == kIssuerWarp && n_tiles > 0) {
        pdl_wait();  // the selected ids come from the kernel before this one
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int64_t slot = int64_t(tile0) * kTile + lane + 32 * h2;
            ids0[h2] = (tile0 < kv_tiles && a.idx && slot < n_kv) ? a.idx[row * a.k + slot] : -1;
        }
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tS = tmem, tO = tmem + 128;  // S[buf]: cols [64 buf, 64 buf + 64); O^T quarter q: [128+64q, 192+64q)

    if (warp >= 4 && warp < kMmaWarp) {
        // --------------------------------------------------------- converters
        const int pt = threadIdx.x - 128;  // 0..kConvThreads-1
        const int c = pt & 15;             // 8-dim unit within a 128-dim quarter
        const int e0 = pt >> 4;            // items e0 + 16 u, u < kUnits
        bool ok = true;
#pragma unroll 1
        for (int lt = 0; lt < n_tiles && ok; ++lt) {
            const int kb = lt & 1;
            ok = mbar_wait(&S.raw_full[kb], uint32_t((lt >> 1) & 1));
            if (!ok) break;
            if (!kFp8 && a.idx && tile0 + lt < kv_tiles) {
                // bf16 gather: 64 threads per 1024-byte row (one 16-byte
                // granule each), four rows per pass
                const uint8_t* kv_seq = (const uint8_t*)a.kv + b * a.max_entries * int64_t(kD * 2);
                const int g = pt & 63;
#pragma unroll
                for (int u = 0; u < kTile / 4; ++u) {
                    const int item = (pt >> 6) + 4 * u;
                    const int32_t id = S.ids[kb][item];
                    const uint8_t* src = kv_seq + int64_t(id < 0 ? 0 : id) * (kD * 2) + 16 * g;
                    cp_async16(S.kv[kb][g >> 3] + sw128_offset(item, g & 7), src, id < 0 ? 0u : 16u);
                }
                cp_async_wait_all();
            } else if (kFp8 && tile0 + lt < kv_tiles) {
                const uint8_t* raw = S.kv[kb][kRawBlk];  // [64 items][512 E4M3] over blocks 4..7
                // every code and scale of this thread's units is read first (16
                // independent shared-memory loads in flight), then converted:
                // dims 0..255 to the lower half (the rows sit in the upper half)
                uint2 w[4][kUnits];
                float sc[4][kUnits];
#pragma unroll
                for (int qt = 0; qt < 4; ++qt)
#pragma unroll
                    for (int u = 0; u < kUnits; ++u) {
                        const int item = e0 + 16 * u;
                        const bool v = S.valid[kb][item] != 0;
                        w[qt][u] = v ? *reinterpret_cast<const uint2*>(raw + kD * item + 128 * qt + 8 * c)
                                     : make_uint2(0, 0);
                        sc[qt][u] = v ? S.kvs[kb][item][(128 * qt + 8 * c) >> 6] : 0.f;
                    }
#pragma unroll
                for (int qt = 0; qt < 2; ++qt)
#pragma unroll
                    for (int u = 0; u < kUnits; ++u) {
                        const int item = e0 + 16 * u;
                        *reinterpret_cast<uint4*>(S.kv[kb][2 * qt + (c >> 3)] + sw128_offset(item, c & 7)) =
                            dequant8(w[qt][u], sc[qt][u]);
                    }
                // the product over dims 0..255 may start while the upper half converts
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.kv_half[kb]);
                // dims 256..511 overwrite the raw rows once every converter has read them
                named_bar(2, kConvThreads);
#pragma unroll
                for (int qt = 2; qt < 4; ++qt)
#pragma unroll
                    for (int u = 0; u < kUnits; ++u) {
                        const int item = e0 + 16 * u;
                        *reinterpret_cast<uint4*>(S.kv[kb][2 * qt + (c >> 3)] + sw128_offset(item, c & 7)) =
                            dequant8(w[qt][u], sc[qt][u]);
                    }
            } else {
                // window tile (or dense bf16 tile): already in place; clear
                // rows past the window or past the eligible entries
                for (int i = pt; i < kTile * 8 * 8; i += kConvThreads) {
                    const int item = i >> 6, blk = (i >> 3) & 7, ch = i & 7;
                    if (!S.valid[kb][item])
                        *reinterpret_cast<uint4*>(S.kv[kb][blk] + sw128_offset(item, ch)) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();  // the whole warp's tile writes are done: one arrival per warp
            if (lane == 0) {
                if (!(kFp8 && tile0 + lt < kv_tiles)) mbar_arrive(&S.kv_half[kb]);
                mbar_arrive(&S.kv_full[kb]);
            }
        }
    } else if (warp == kIssuerWarp) {
        // ------------------------------------------------------------- issuer
        // lane l handles items l and l + 32 of each tile
        if (n_tiles > 0) {
            const uint8_t* kv_seq = (const uint8_t*)a.kv + b * a.max_entries * int64_t(kFp8 ? kD : 0);
            const float* kvs_seq = (const float*)a.kv_s + b * a.max_entries * int64_t(kFp8 ? kD / 64 : 0);
            bool ok = true;
            int issued = 0;
            // software pipeline: the ids of tile lt+1 are loaded during tile lt,
            // and tile lt's scales are loaded before waiting for its buffer
            auto load_ids = [&](int lt, int32_t (&j)[2]) {
                const int T = tile0 + lt;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int64_t slot = int64_t(T) * kTile + lane + 32 * h2;
                    j[h2] = (T < kv_tiles && a.idx && slot < n_kv) ? a.idx[row * a.k + slot] : -1;
                }
            };
            int32_t jn[2] = {ids0[0], ids0[1]};  // tile 0's ids, read before the CTA barrier
#pragma unroll 1
            for (int lt = 0; lt < n_tiles && ok; ++lt) {
                const int kb = lt & 1, T = tile0 + lt;
                const bool pooled = T < kv_tiles;
                int32_t sr[2];
                float4 scl[2][2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int64_t slot = int64_t(T) * kTile + lane + 32 * h2;
                    const int64_t j = a.idx ? int64_t(jn[h2]) : slot;
                    if (pooled && slot < n_kv && j >= a.max_entries) flag_status(CSA_DEV_BAD_INDEX);
                    sr[h2] = (pooled && slot < n_kv && j >= 0 && j < a.max_entries) ? int32_t(j) : -1;
                    scl[h2][0] = scl[h2][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (kFp8 && a.idx && sr[h2] >= 0) {
                        const float4* sp = reinterpret_cast<const float4*>(kvs_seq + int64_t(sr[h2]) * (kD / 64));
                        scl[h2][0] = sp[0];
                        scl[h2][1] = sp[1];
                    }
                }
                if (lt + 1 < n_tiles) load_ids(lt + 1, jn);
                if (lt >= 2) ok = mbar_wait(&S.kv_empty[kb], uint32_t(((lt >> 1) - 1) & 1));
                if (!ok) break;
                if (pooled && !kFp8) {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        S.valid[kb][lane + 32 * h2] = sr[h2] >= 0;
                        S.ids[kb][lane + 32 * h2] = sr[h2];
                    }
                    if (!a.idx) {
                        // dense: the tile's rows are consecutive; rows past the
                        // entries read as zero, rows past n_kv are cleared
                        const int64_t j0 = int64_t(T) * kTile;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&S.raw_full[kb], uint32_t(kTile * kD * 2));
#pragma unroll
                            for (int blk = 0; blk < 8; ++blk)
                                tma_load_3d(S.kv[kb][blk], &map_kv, 64 * blk, int32_t(j0), int32_t(b),
                                            &S.raw_full[kb]);
                        }
                    } else if (lane == 0) {
                        mbar_arrive(&S.raw_full[kb]);  // the converters gather the rows
                    }
                } else if (pooled) {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) S.valid[kb][lane + 32 * h2] = sr[h2] >= 0;
                    uint8_t* dst = S.kv[kb][kRawBlk];
                    if (!a.idx) {
                        // dense: the tile's rows (and scales) are consecutive
                        const int64_t j0 = int64_t(T) * kTile;
                        const uint32_t nv = uint32_t(min(int64_t(kTile), n_kv - j0));
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&S.raw_full[kb], nv * (kD + 32));
                            bulk_g2s(dst, kv_seq + j0 * kD, nv * kD, &S.raw_full[kb]);
                            bulk_g2s(&S.kvs[kb][0][0], kvs_seq + j0 * (kD / 64), nv * 32, &S.raw_full[kb]);
                        }
                    } else {
                        uint32_t bytes = (sr[0] >= 0 ? kD : 0) + (sr[1] >= 0 ? kD : 0);
                        bytes = __reduce_add_sync(0xffffffffu, bytes);
                        if (lane == 0) mbar_arrive_expect_tx(&S.raw_full[kb], bytes);
                        __syncwarp();
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2)
                            if (sr[h2] >= 0)
                                bulk_g2s(dst + kD * (lane + 32 * h2), kv_seq + int64_t(sr[h2]) * kD, kD,
                                         &S.raw_full[kb]);
                        // the scales were loaded before the wait; store them now
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float4* dp = reinterpret_cast<float4*>(&S.kvs[kb][lane + 32 * h2][0]);
                            dp[0] = scl[h2][0];
                            dp[1] = scl[h2][1];
                        }
                    }
                } else {
                    const int64_t w0 = int64_t(T - kv_tiles) * kTile;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) S.valid[kb][lane + 32 * h2] = w0 + lane + 32 * h2 < n_win;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&S.raw_full[kb], uint32_t(kTile * kD * 2));
#pragma unroll
                        for (int blk = 0; blk < 8; ++blk)
                            tma_load_3d(S.kv[kb][blk], &map_win, 64 * blk, int32_t(win_lo - p0 + w0),
                                        int32_t(b), &S.raw_full[kb]);
                    }
                }
                __syncwarp();  // every lane's ids and scales precede lane 0's releasing arrival
                if (lane == 0) mbar_arrive(&S.raw_full[kb]);
                ++issued;
            }
            // Let every copy still in flight land before the CTA exits (already
            // the case unless a consumer gave up on a wait).
            if (lane == 0) {
                bool drained = mbar_wait(&S.q_full, 0);
                for (int i = max(0, issued - 2); i < issued && drained; ++i)
                    drained = mbar_wait(&S.raw_full[i & 1], uint32_t((i >> 1) & 1));
            }
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------------------- MMA
        if (lane == 0 && n_tiles > 0) {
            const uint32_t id_qk = instr_desc(1, 1, 0, 0, 64, 64);   // bf16: A = Q K-major, B = K K-major
            const uint32_t id_pv = instr_desc(1, 1, 1, 0, 128, 64);  // bf16: A = V^T MN-major, B = P K-major
            const uint32_t q0 = smem_u32(S.q[0]);
            bool ok = mbar_wait(&S.q_full, 0);
            // QK(t) may run at most one tile ahead of P.V: it overwrites S[t&1],
            // which the softmax of tile t-2 has finished reading once P.V(t-2)
            // has been issued.  Each wait is a single non-blocking test; the
            // loop as a whole is bounded by kWaitNs without progress.
            // QK of a tile runs in two halves over the dims: 0..255 once the
            // converters have written them, 256..511 once the whole tile is in
            int qk_t = 0, pv_t = 0, qk_half = 0;
            uint64_t t_last = global_ns();
            while (ok && pv_t < n_tiles) {
                bool progressed = false;
                if (qk_t < n_tiles && qk_t <= pv_t + 1) {
                    const int kb = qk_t & 1;
                    const uint32_t par = uint32_t((qk_t >> 1) & 1);
                    if (mbar_test_wait(qk_half ? &S.kv_full[kb] : &S.kv_half[kb], par)) {
                        tc_fence_after();
                        const uint32_t kv0 = smem_u32(S.kv[kb][0]);
#pragma unroll
                        for (int s = 0; s < 16; ++s) {
                            const int blk = 4 * qk_half + (s >> 2);
                            mma_f16(tS + 64 * kb, smem_desc(q0 + blk * 8192 + (s & 3) * 32, 16, 1024),
                                    smem_desc(kv0 + blk * 8192 + (s & 3) * 32, 16, 1024), id_qk,
                                    (qk_half | s) != 0);
                        }
                        if (qk_half) {
                            mma_commit(&S.s_full[kb]);
                            ++qk_t;
                        }
                        qk_half ^= 1;
                        progressed = true;
                    }
                }
                if (pv_t < qk_t) {
                    const int kb = pv_t & 1;
                    if (mbar_test_wait(&S.p_full[kb], uint32_t((pv_t >> 1) & 1))) {
                        tc_fence_after();
                        const uint32_t kv0 = smem_u32(S.kv[kb][0]), pp = smem_u32(S.p[kb]);
#pragma unroll
                        for (int qt = 0; qt < 4; ++qt)
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_f16(tO + 64 * qt, smem_desc(kv0 + (2 * qt) * 8192 + ks * 2048, 8192, 1024),
                                        smem_desc(pp + ks * 32, 16, 1024), id_pv, (pv_t | ks) != 0);
                        mma_commit(&S.kv_empty[kb]);
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
        // item validity as a 64-bit mask: pooled slots below n_kv whose id is in
        // range, or window positions below n_win; the ids of tile t+1 are loaded
        // while tile t is processed
        auto load_ids = [&](int lt, int32_t& j0, int32_t& j1) {
            const int T = tile0 + lt;
            const int64_t s0 = int64_t(T) * kTile + lane, s1 = s0 + 32;
            const bool pooled = T < kv_tiles;
            j0 = (pooled && a.idx && s0 < n_kv) ? a.idx[row * a.k + s0] : 0;
            j1 = (pooled && a.idx && s1 < n_kv) ? a.idx[row * a.k + s1] : 0;
        };
        auto mask_of = [&](int lt, int32_t j0, int32_t j1, unsigned& vm0, unsigned& vm1) {
            const int T = tile0 + lt;
            if (T < kv_tiles) {
                const int64_t s0 = int64_t(T) * kTile + lane, s1 = s0 + 32;
                vm0 = __ballot_sync(0xffffffffu, s0 < n_kv && j0 >= 0 && j0 < a.max_entries);
                vm1 = __ballot_sync(0xffffffffu, s1 < n_kv && j1 >= 0 && j1 < a.max_entries);
            } else {
                const int64_t w0 = int64_t(T - kv_tiles) * kTile + lane;
                vm0 = __ballot_sync(0xffffffffu, w0 < n_win);
                vm1 = __ballot_sync(0xffffffffu, w0 + 32 < n_win);
            }
        };
        int32_t nj0 = 0, nj1 = 0;
        pdl_wait();  // the selected ids come from the kernel before this one
        if (n_tiles > 0) load_ids(0, nj0, nj1);
        for (int tile = 0; tile < n_tiles; ++tile) {
            const int kb = tile & 1;
            unsigned vm0, vm1;
            mask_of(tile, nj0, nj1, vm0, vm1);
            if (tile + 1 < n_tiles) load_ids(tile + 1, nj0, nj1);
            if (ok) ok = mbar_wait(&S.s_full[kb], uint32_t((tile >> 1) & 1));
            if (ok) tc_fence_after();
            const uint32_t srow = tS + 64 * kb + (uint32_t(sub * 32) << 16);
            // lanes 0-15 hold items 0..31 of head h, lanes 16-31 items 32..63
            const bool upper = lane >= 16;
            const unsigned vm = upper ? vm1 : vm0;
            float x[32];
            if (ok) tmem_ld16x2_32(srow, x);
            // the max of the scaled, masked logits over both halves
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (ok && ((vm >> i) & 1u)) mx = fmaxf(mx, x[i] * sl2);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            float al = 1.f;
            if (mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx != -INFINITY)) {
                al = m_run == -INFINITY ? 0.f : ex2(m_run - mx);
                m_run = mx;
            }
            // P[kb] was read by P.V two tiles back: that one must be done (its
            // completion also releases the tile buffer, hence kv_empty)
            if (ok && tile >= 2) ok = mbar_wait(&S.kv_empty[kb], uint32_t(((tile >> 1) - 1) & 1));
            // P = exp2(x - m) as bf16 rows of the K-major B tile (each lane its
            // 32 items: 16-byte chunks 0-3 or 4-7 of row h), and the sum
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = (ok && ((vm >> i) & 1u)) ? ex2(x[i] * sl2 - m_run) : 0.f;
                sum += x[i];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t w4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[8 * ch + 2 * k], x[8 * ch + 2 * k + 1]);
                    w4[k] = *reinterpret_cast<const uint32_t*>(&hh);
                }
                *reinterpret_cast<uint4*>(S.p[kb] + sw128_offset(h, 4 * int(upper) + ch)) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            l_run = l_run * al + sum;
            if (head_lane) {
                S.alpha[h] = al;
                if (al != 1.f && tile > 0) S.rescale = 1;
            }
            named_bar(1, 128);
            if (ok && S.rescale != 0) {
                // O^T is rescaled only once P.V of the previous tile is done
                // (P.V two tiles back is done, so the phase is unambiguous)
                ok = mbar_wait(&S.o_done, uint32_t((tile - 1) & 1));
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
            __syncwarp();  // one arrival per warp once all its P writes and O updates are done
            if (lane == 0) mbar_arrive(&S.p_full[kb]);
        }
        // ----------------------------------------------------------- epilogue
        if (head_lane) {
            if (a.n_splits == 1 && !a.partial_out) {
                float f = 1.f, den = l_run;
                if (a.sinks) {
                    const float sg = a.sinks[h] * kLog2e;
                    const float M = fmaxf(m_run, sg);
                    f = m_run == -INFINITY ? 0.f : ex2(m_run - M);
                    den = l_run * f + ex2(sg - M);
                }
                S.fin[h] = den > 0.f ? f / den : 0.f;
            } else if (a.fused_combine) {
                S.ml[h] = make_float2(m_run, l_run);
                S.fin[h] = 1.f;
            } else {
                const int64_t item = row * a.n_splits + split;
                a.part_ml[item * kH + h] = make_float2(m_run == -INFINITY ? -INFINITY : m_run / kLog2e, l_run);
                S.fin[h] = 1.f;
            }
        }
        named_bar(1, 128);
        // every P.V done: the one two tiles back first, so that the last
        // o_done phase is unambiguous
        if (n_tiles >= 2 && ok)
            ok = mbar_wait(&S.kv_empty[(n_tiles - 2) & 1], uint32_t(((n_tiles - 2) >> 1) & 1));
        if (n_tiles > 0 && ok) ok = mbar_wait(&S.o_done, uint32_t((n_tiles - 1) & 1));
        tc_fence_after();
        // Every P.V has completed, so the two tile buffers (128 KB) are free:
        // O goes there as [64 heads][512 dims] (fp32 partials, or the final
        // bf16 output) and leaves in a few bulk stores.
        const int e = sub * 32 + lane;
        const bool final_out = a.n_splits == 1 && !a.partial_out;
        float* so32 = reinterpret_cast<float*>(&S.kv[0][0][0]);
        __nv_bfloat16* so16 = reinterpret_cast<__nv_bfloat16*>(&S.kv[0][0][0]);
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
                if (final_out) {
                    // the 32 factors first: loads that followed stores into
                    // the same shared memory would each wait for the store
                    float f[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 f4 = reinterpret_cast<const float4*>(&S.fin[32 * hf])[j];
                        f[4 * j] = f4.x; f[4 * j + 1] = f4.y; f[4 * j + 2] = f4.z; f[4 * j + 3] = f4.w;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) so16[(32 * hf + i) * kD + dim] = __float2bfloat16_rn(o[i] * f[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) so32[(32 * hf + i) * kD + dim] = o[i];
                }
            }
        }
        fence_proxy_async_smem();
        named_bar(1, 128);
        if (threadIdx.x == 0 && !a.fused_combine) {
            const uint32_t bytes = final_out ? kH * kD * 2 : kH * kD * 4;
            uint8_t* dst = final_out ? (uint8_t*)a.out + row * int64_t(kH) * kD * 2
                                     : (uint8_t*)(a.part_o + (row * a.n_splits + split) * int64_t(kH) * kD);
            const uint8_t* src = &S.kv[0][0][0];
            for (uint32_t off = 0; off < bytes; off += 16384) bulk_s2g(dst + off, src + off, 16384);
            bulk_commit_wait_read();
        }
    }
    // the issuer and MMA roles run on one lane: reconverge every warp so that
    // the CTA barrier (an aligned bar.sync) sees whole warps and really waits
    // for those lanes before TMEM is freed
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
    if (a.fused_combine) {
        // The splits of this row form the cluster; each has staged its fp32 O
        // ([64 heads][512 dims] in its tile buffers) and (m, l) per head.  CTA
        // r combines an r-th of the output, reading every split's partial
        // through distributed shared memory, and writes the final bf16.
        namespace cg = cooperative_groups;
        cg::cluster_group cl = cg::this_cluster();
        const int ns = a.n_splits, r = int(cl.block_rank());
        cl.sync();
        if (threadIdx.x < kH) {
            const int hh = threadIdx.x;
            float m[8], l[8];
            float M = a.sinks ? a.sinks[hh] * kLog2e : -INFINITY;
            for (int q = 0; q < ns; ++q) {
                const float2 v = cl.map_shared_rank(&S.ml[0], q)[hh];
                m[q] = v.x;
                l[q] = v.y;
                M = fmaxf(M, v.x);
            }
            float den = 0.f;
            for (int q = 0; q < ns; ++q) {
                const float wq = m[q] == -INFINITY ? 0.f : ex2(m[q] - M);
                S.cw[q][hh] = wq;
                den += wq * l[q];
            }
            if (a.sinks) den += ex2(a.sinks[hh] * kLog2e - M);
            S.cinv[hh] = den > 0.f ? 1.f / den : 0.f;
        }
        __syncthreads();
        constexpr int n4 = kH * kD / 4;
        const int lo = r * n4 / ns, hi = (r + 1) * n4 / ns;
        const float4* part = reinterpret_cast<const float4*>(&S.kv[0][0][0]);
        __nv_bfloat16* out = (__nv_bfloat16*)a.out + row * int64_t(kH) * kD;
        // the splits' partials of a position are all requested before any is
        // used (at most 8 remote loads in flight per thread), then summed in
        // split order
        const float4* rp[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) rp[q] = q < ns ? cl.map_shared_rank(part, q) : part;
        for (int i = lo + threadIdx.x; i < hi; i += kThreads) {
            const int hh = (4 * i) / kD;
            float4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < ns) v[q] = rp[q][i];
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < ns) {
                    const float wq = S.cw[q][hh];
                    acc.x += wq * v[q].x; acc.y += wq * v[q].y; acc.z += wq * v[q].z; acc.w += wq * v[q].w;
                }
            const float inv = S.cinv[hh];
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
            const __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
            *reinterpret_cast<uint2*>(out + 4 * int64_t(i)) = pk;
        }
        cl.sync();  // keep this CTA's shared memory alive until every remote read is done
    }
}

bool attn_tc_supported(int act, int kvf, int H, int D) {
    return act == CSA_BF16 && (kvf == CSA_FP8_S64 || kvf == CSA_BF16) && H == kH && D == kD;
}

bool attn_tc_rows_fit(int64_t max_entries, int64_t n_raw) {
    return max_entries < (int64_t(1) << 31) && n_raw < (int64_t(1) << 31);
}

// Whether clusters of cfg's size can be scheduled for this kernel on the
// current device (queried once per device, entry format and size).
template <int KVF>
static bool cluster_fits(const cudaLaunchConfig_t& cfg) {
    static std::mutex mu;
    static int known[64][9];  // 0 unknown, 1 yes, 2 no
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const int n = int(cfg.gridDim.x);
    std::lock_guard<std::mutex> lock(mu);
    if (known[dev][n] == 0) {
        int n_clusters = 0;
        const bool ok = cudaOccupancyMaxActiveClusters(&n_clusters, attn_tc_kernel<KVF>, &cfg) == cudaSuccess &&
                        n_clusters > 0;
        if (!ok) (void)cudaGetLastError();
        known[dev][n] = ok ? 1 : 2;
    }
    return known[dev][n] == 1;
}

template <int KVF>
static cudaError_t launch_attn_tc_fmt(AttnArgs a, int64_t rows, cudaStream_t s, bool* combined, bool pdl) {
    if (rows * kH >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    // query [rows * 64][512] bf16 and window tokens [batch][n_raw][512] bf16,
    // both read as [64 rows][64 dims] boxes with 128-byte swizzle
    CUtensorMap map_q, map_win;
    const uint64_t qd[2] = {uint64_t(kD), uint64_t(rows * kH)};
    const uint64_t qs[1] = {uint64_t(kD) * 2};
    const uint32_t box2[2] = {64, 64};
    if (!encode_tile_map(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, qd, qs, box2,
                         CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    memset(&map_win, 0, sizeof(map_win));
    if (a.n_raw > 0) {
        const int64_t batch = rows / a.n_q;
        const uint64_t wd[3] = {uint64_t(kD), uint64_t(a.n_raw), uint64_t(batch)};
        const uint64_t ws[2] = {uint64_t(kD) * 2, uint64_t(a.n_raw) * kD * 2};
        const uint32_t box3[3] = {64, 64, 1};
        if (!encode_tile_map(&map_win, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.raw, wd, ws, box3,
                             CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // bf16 entries [batch][max_entries][512]: dense tiles read as [64 rows][64 dims] boxes
    CUtensorMap map_kv;
    memset(&map_kv, 0, sizeof(map_kv));
    if (KVF == CSA_BF16 && !a.idx && a.max_entries > 0) {
        const int64_t batch = rows / a.n_q;
        const uint64_t kd[3] = {uint64_t(kD), uint64_t(a.max_entries), uint64_t(batch)};
        const uint64_t ks[2] = {uint64_t(kD) * 2, uint64_t(a.max_entries) * kD * 2};
        const uint32_t box3[3] = {64, 64, 1};
        if (!encode_tile_map(&map_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.kv, kd, ks, box3,
                             CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    const size_t sm = sizeof(SmemAttn) + 1024;
    cudaError_t e = ensure_smem(attn_tc_kernel<KVF>, sm);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_splits, unsigned(std::min<int64_t>(rows, kMaxGridY)));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(a.n_splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    // The splits of a row combine inside the kernel when they fit one portable
    // cluster and such clusters can be scheduled; otherwise launch_combine runs.
    if (a.n_splits >= 2 && a.n_splits <= 8 && !a.partial_out) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cluster_fits<KVF>(cfg)) {
            a.fused_combine = 1;
            cfg.numAttrs = pdl ? 2 : 1;
            e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<KVF>, map_q, map_win, map_kv, a);
            if (e == cudaSuccess) *combined = true;
            return e;
        }
    }
    a.fused_combine = 0;
    cfg.attrs = pdl ? &attr[1] : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    // the grid's y extent is limited: long prefill chunks take several launches
    for (int64_t r0 = 0; r0 < rows; r0 += kMaxGridY) {
        a.row_base = r0;
        cfg.gridDim.y = unsigned(std::min(kMaxGridY, rows - r0));
        e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<KVF>, map_q, map_win, map_kv, a);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_attn_tc(const AttnArgs& a, int64_t rows, cudaStream_t s, bool* combined, bool pdl) {
    *combined = false;
    if (rows == 0) return cudaSuccess;
    if (a.kv_fmt == CSA_BF16) return launch_attn_tc_fmt<CSA_BF16>(a, rows, s, combined, pdl);
    if (a.kv_fmt == CSA_FP8_S64) return launch_attn_tc_fmt<CSA_FP8_S64>(a, rows, s, combined, pdl);
    return cudaErrorInvalidValue;
}

}  // namespace csa
