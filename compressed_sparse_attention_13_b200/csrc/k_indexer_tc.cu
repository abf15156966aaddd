// Lightning indexer on the 5th-generation tensor cores, for MXFP4 queries and
// keys ("DeepSeek-V4 發佈說明", section 壓縮稀疏注意力 (CSA): ReLU-scored
// multi-head dot products in FP4; wiki summary, section 基础设施: MXFP4 on
// the indexer QK path).
//
//   s[j] = sum_h w[h] * ReLU(qI[h] . kI[j])
//
// The contraction runs as the block-scaled tcgen05.mma.kind::mxf4: the packed
// E2M1 keys and queries are the operands as stored, and the E8M0 block
// exponents are the MMA's scale factors, so no element is converted and every
// stored value enters the fp32 accumulation exactly.
// One MMA: M = 128 keys (A), N = 64 heads (B = the query block), K = 64; a
// 128-key tile takes two (K = 128).  Both operands are K-major with 64-byte
// rows in the 64-byte-swizzled layout that the 2-D tensor copy writes.  The
// fp32 accumulator D[key][head] lives in TMEM, so the epilogue thread of TMEM
// lane j owns key j's 64 head scores and reduces them without cross-thread
// traffic.
//
// The single threads that issue copies and MMAs pay a fixed cost per pipeline
// step in barrier and tcgen05 instruction latency (about 0.5 us), which paces
// a pipeline; so each SM runs two independent pipelines (two CTAs of 320
// threads, 256 TMEM columns and ~86 KB of shared memory each).  Persistent
// CTAs take contiguous ranges of (query row, 128-key step) units and walk
// them in order, skipping steps past the row's eligible blocks; the k-th
// eligible step of a CTA is "step it = k".  Warp roles:
//   warp 0      tensor copy of the step's keys (+ a bulk copy of their scale
//               bytes) into a kStages ring, and of the query block of each
//               new row into a kQBufs ring (one elected lane); TMEM allocation
//   warp 1      MMA issue (one elected lane)
//   warps 2-5   scale writers: per step, copy the keys' E8M0 bytes from shared
//               memory into the TMEM scale-factor layout (and the query's on a
//               row change) with tcgen05.st
//   warps 6-9   epilogue: accumulator it % kAccBufs of step it from TMEM,
//               ReLU, weights, sum over heads
// Buffer reuse: the key scales of step it live in TMEM buffer it % kStages,
// rewritten only after the producer has reused the shared-memory stage, i.e.
// after the MMA of step it - kStages completed; a row's query scales use
// buffer (row count % kStages), safe by the same argument because kStages
// row changes need at least kStages steps.
// All waits are bounded (sm100::mbar_wait); after a timed-out wait a role
// keeps iterating without waiting or touching memory, so every thread still
// reaches the named and final barriers.
#include <string.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kHI = 64, kDI = 128;
constexpr int kTileKeys = 128;                         // keys per MMA (M)
constexpr int kStepKeys = 128;                         // keys per pipeline step
constexpr int kTilesPerStep = kStepKeys / kTileKeys;
constexpr int kQBufs = 4, kAccBufs = 2;
constexpr int kEpiGroups = 1;                          // epilogue groups of 4 warps
constexpr int kKeyBytes = kDI / 2;                     // 64: packed E2M1
constexpr int kAData = kStepKeys * kKeyBytes;          // 8192
constexpr int kQData = kHI * kKeyBytes;                // 4096
constexpr int kA8Data = kStepKeys * kDI;               // 16384: E4M3 keys of a step (FP8 variant)
constexpr int kQ8Data = kHI * kDI;                     // 8192: E4M3 query block (FP8 variant)
constexpr int kAccCols = kTilesPerStep * 64;           // tiles x 64 heads
constexpr int kTmemCols = 256;
constexpr int kEpiWarp0 = 6;
constexpr int kConvWarp0 = kEpiWarp0 + 4 * kEpiGroups; // FP8 variant: E2M1 -> E4M3 converters

// Per variant: the MXFP4 kernel (kind::mxf4, two E8M0 scales per row and
// MMA, K = 64) runs two pipelines per SM with an 8-stage ring; the FP8
// variant (kind::mxf8f6f4, one scale per row and MMA, K = 32) carries the
// expanded E4M3 copies as well, so it runs one CTA per SM with a 4-stage ring.
template <bool F8>
struct Cfg {
    static constexpr int kStages = F8 ? 4 : 8;
    static constexpr int kCtasPerSm = F8 ? 1 : 2;
    static constexpr int kThreads = 32 * (kConvWarp0 + (F8 ? 4 : 0));
    static constexpr int kKSteps = F8 ? 4 : 2;                    // MMAs per 128-dim tile
    static constexpr int kSfaPerStage = 4 * kKSteps * kTilesPerStep;  // 4 columns per k-step
    static constexpr int kSfbPerBuf = 2 * kKSteps;                // 2 columns (64 heads) per k-step
    static constexpr int kSfaCol = kAccBufs * kAccCols;           // 128
    static constexpr int kSfbCol = kSfaCol + kSfaPerStage * kStages;
    static_assert(kSfbCol + kSfbPerBuf * kStages <= kTmemCols, "TMEM columns");
};

struct IdxTcArgs {
    const uint8_t* kIs;   // [batch][max_blocks][4] E8M0
    const uint8_t* qIs;   // [rows][64][4] E8M0 (stored MXFP4 queries)
    const uint16_t* qraw; // [rows][64][128] bf16 (queries quantised in the kernel)
    const float* w;       // [rows][64]
    const int64_t* q_pos; // [rows]
    float* scores;        // [rows][ld]
    int64_t ld, max_blocks;
    int n_q, m, W;
    int64_t rows, tiles_per_row, units;
};

template <bool F8>
struct Smem {
    static constexpr int kSt = Cfg<F8>::kStages;
    uint8_t a[kSt][kAData];            // 1024-aligned: key steps (64-byte swizzle)
    uint8_t q[kQBufs][kQData];         // query blocks (64-byte swizzle)
    uint8_t a8[F8 ? kSt : 1][F8 ? kA8Data : 1024];   // FP8 variant: E4M3 keys (128-byte swizzle)
    uint8_t q8[F8 ? kQBufs : 1][F8 ? kQ8Data : 1024];  // FP8 variant: E4M3 query blocks
    uint32_t a_sf[kSt][kStepKeys];     // keys' four E8M0 bytes
    uint32_t q_sf[kQBufs][kHI];        // queries quantised here: their four E8M0 bytes per head
    float ew[kEpiGroups][kHI];         // per epilogue group: weights of its current row
    uint64_t a_full[kSt], a_empty[kSt], sf_full[kSt], a8_full[kSt];
    uint64_t q_full[kQBufs], q_empty[kQBufs], q8_full[kQBufs];
    uint64_t acc_full[kAccBufs], acc_empty[kAccBufs];
    uint32_t tmem_base;
};

// In-order walk over a CTA's units that visits only eligible tiles.  Rows
// change at most once per tile; q_pos is read once per row.
struct TileWalk {
    int64_t u, u1, row, tile, ne, tpr;
    bool started;
    __device__ __forceinline__ TileWalk(const IdxTcArgs& a, int64_t u0, int64_t u_end)
        : u(u0), u1(u_end), tpr(a.tiles_per_row), started(false) {
        row = u0 / tpr;
        tile = u0 - row * tpr;
        ne = u0 < u_end ? min(n_elig(a.q_pos[row], a.m, a.W), a.max_blocks) : 0;
    }
    // Advance to the next eligible tile; false when the range is exhausted.
    __device__ __forceinline__ bool next(const IdxTcArgs& a) {
        if (started) { ++u; ++tile; }
        started = true;
        while (u < u1) {
            if (tile == tpr) {
                tile = 0;
                ++row;
                ne = min(n_elig(a.q_pos[row], a.m, a.W), a.max_blocks);
            }
            if (tile * kStepKeys < ne) return true;
            u += tpr - tile;  // rest of this row is ineligible
            tile = tpr;
        }
        return false;
    }
    __device__ __forceinline__ int64_t k0() const { return tile * kStepKeys; }
};

__device__ __forceinline__ uint64_t pack_f32x2(float x, float y) {
    return uint64_t(__float_as_uint(x)) | (uint64_t(__float_as_uint(y)) << 32);
}
__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
    return make_float2(__uint_as_float(uint32_t(v)), __uint_as_float(uint32_t(v >> 32)));
}
// (a.x*b.x + c.x, a.y*b.y + c.y), each rounded once
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}


// Four E2M1 codes (the low 16 bits, element i in nibble i) -> four E4M3
// bytes.  Every E2M1 value (+-{0, 0.5, 1, 1.5, 2, 3, 4, 6}) is an E4M3
// value, so the expansion is exact: a byte-table lookup on the magnitude
// and the sign moved to bit 7.
__device__ __forceinline__ uint32_t e4m3x4_of_e2m1x4(uint32_t x) {
    uint32_t mag, sgn;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(mag) : "r"(0x3C383000u), "r"(0x4C484440u), "r"(x & 0x7777u));
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(sgn) : "r"(0x00008000u), "r"(0u), "r"((x >> 3) & 0x1111u));
    return mag | sgn;
}

// One 64-byte-swizzled row of 128 packed E2M1 codes -> the same row as 128
// E4M3 bytes in the 128-byte-swizzled K-major layout.
__device__ __forceinline__ void expand_row(const uint8_t* src, uint8_t* dst, uint32_t row) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + sm100::sw64_offset(row, c));
        const uint4 lo = make_uint4(e4m3x4_of_e2m1x4(w.x), e4m3x4_of_e2m1x4(w.x >> 16),
                                    e4m3x4_of_e2m1x4(w.y), e4m3x4_of_e2m1x4(w.y >> 16));
        const uint4 hi = make_uint4(e4m3x4_of_e2m1x4(w.z), e4m3x4_of_e2m1x4(w.z >> 16),
                                    e4m3x4_of_e2m1x4(w.w), e4m3x4_of_e2m1x4(w.w >> 16));
        *reinterpret_cast<uint4*>(dst + sm100::sw128_offset(row, 2 * c)) = lo;
        *reinterpret_cast<uint4*>(dst + sm100::sw128_offset(row, 2 * c + 1)) = hi;
    }
}

// Quantise 32 bf16 values (one MXFP4 block) as csa_quantize does: block
// exponent X = floor(log2(max |v|)) - 2 clamped to [-127, 127] (0 for an
// all-zero block), codes = E2M1(v * 2^-X) rounded to nearest even.  Returns
// the E8M0 byte X + 127; the 16 code bytes go to out.
__device__ __forceinline__ uint32_t quant_block32(const uint4 (&v)[4], uint4& out) {
    float f[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            f[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
    int X = amax > 0.f ? ilog2_floor(amax) - 2 : 0;
    X = max(-127, min(127, X));
    const float inv = pow2f(-X);
    uint32_t b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = cvt_e2m1x2(__fmul_rn(f[2 * i], inv), __fmul_rn(f[2 * i + 1], inv));
    out = make_uint4(b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24, b[4] | b[5] << 8 | b[6] << 16 | b[7] << 24,
                      b[8] | b[9] << 8 | b[10] << 16 | b[11] << 24, b[12] | b[13] << 8 | b[14] << 16 | b[15] << 24);
    return uint32_t(X + 127);
}

}  // namespace

template <bool QRAW, bool F8>
__global__ void __launch_bounds__(Cfg<F8>::kThreads, Cfg<F8>::kCtasPerSm)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_q, const IdxTcArgs a) {
    using C = Cfg<F8>;
    constexpr int kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    Smem<F8>& S = *reinterpret_cast<Smem<F8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using namespace sm100;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.a_full[i], 1); mbar_init(&S.a_empty[i], 1); mbar_init(&S.sf_full[i], 4);  // one arrival per scale-writer warp
            mbar_init(&S.a8_full[i], 4);  // one arrival per converter warp
        }
        for (int i = 0; i < kQBufs; ++i) {
            mbar_init(&S.q_full[i], QRAW ? 4 : 1);  // the tensor copy, or one arrival per quantiser warp
            mbar_init(&S.q_empty[i], 1);
            mbar_init(&S.q8_full[i], 4);
        }
        for (int i = 0; i < kAccBufs; ++i) { mbar_init(&S.acc_full[i], 1); mbar_init(&S.acc_empty[i], 4); }
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&S.tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    const int64_t u0 = a.units * blockIdx.x / gridDim.x;
    const int64_t u1 = a.units * (blockIdx.x + 1) / gridDim.x;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            TileWalk tw(a, u0, u1);
            int st = 0, issued = 0, q_issued = 0, rc = -1;
            uint32_t ph = 0;
            int64_t cur_row = -1;
            bool ok = true;
            for (int it = 0; ok && tw.next(a); ++it) {
                if (!QRAW && tw.row != cur_row) {
                    cur_row = tw.row;
                    ++rc;
                    const int qb = rc & (kQBufs - 1);
                    if (rc >= kQBufs) ok = mbar_wait(&S.q_empty[qb], uint32_t((rc / kQBufs) - 1) & 1u);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&S.q_full[qb], uint32_t(kQData));
                    tma_load_2d(S.q[qb], &map_q, 0, int32_t(cur_row * kHI), &S.q_full[qb]);
                    ++q_issued;
                }
                if (it >= kStages) ok = mbar_wait(&S.a_empty[st], ph ^ 1u);
                if (!ok) break;
                const int64_t k0 = tw.k0();
                int64_t nk = min(int64_t(kStepKeys), tw.ne - k0);
                nk = min((nk + 3) & ~int64_t(3), a.max_blocks - k0);  // max_blocks % 4 == 0
                const int64_t key0 = (tw.row / a.n_q) * a.max_blocks + k0;
                // the tensor copy always delivers the whole 256-row box (rows
                // past the tensor read as zero)
                mbar_arrive_expect_tx(&S.a_full[st], uint32_t(kAData + nk * 4));
                tma_load_2d(S.a[st], &map_k, 0, int32_t(key0), &S.a_full[st]);
                bulk_g2s(S.a_sf[st], a.kIs + key0 * 4, uint32_t(nk * 4), &S.a_full[st]);
                ++issued;
                if (++st == kStages) { st = 0; ph ^= 1u; }
            }
            // Let every copy still in flight land before the CTA exits (already
            // the case unless a consumer gave up on a wait).
            bool drained = true;
            for (int i = max(0, issued - kStages); i < issued && drained; ++i)
                drained = mbar_wait(&S.a_full[i % kStages], uint32_t(i / kStages) & 1u);
            for (int i = max(0, q_issued - kQBufs); i < q_issued && drained; ++i)
                drained = mbar_wait(&S.q_full[i % kQBufs], uint32_t(i / kQBufs) & 1u);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc = F8 ? instr_desc_mxf8_e4m3(128, 64) : instr_desc_mxf4(128, 64);
            TileWalk tw(a, u0, u1);
            int64_t cur_row = -1;
            int rc = -1, st = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int it = 0; ok && tw.next(a); ++it) {
                if (tw.row != cur_row) {
                    // every MMA of the previous row is issued: release its query block
                    if (rc >= 0) mma_commit(&S.q_empty[rc & (kQBufs - 1)]);
                    cur_row = tw.row;
                    ++rc;
                    const uint32_t qpar = uint32_t(rc / kQBufs) & 1u;
                    ok = mbar_wait(F8 ? &S.q8_full[rc & (kQBufs - 1)] : &S.q_full[rc & (kQBufs - 1)], qpar);
                }
                const int b = it % kAccBufs;
                const uint32_t par = uint32_t(it / kAccBufs) & 1u;
                if (ok) ok = mbar_wait(F8 ? &S.a8_full[st] : &S.a_full[st], ph);
                if (ok) ok = mbar_wait(&S.sf_full[st], ph);
                if (ok && it >= kAccBufs) ok = mbar_wait(&S.acc_empty[b], par ^ 1u);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sfa = tmem + C::kSfaCol + C::kSfaPerStage * st;
                const uint32_t sfb = tmem + C::kSfbCol + C::kSfbPerBuf * (rc & (kStages - 1));
                if constexpr (F8) {
                    // K = 32 E4M3 values (32 bytes of the 128-byte row) per MMA
                    const uint32_t a0 = smem_u32(S.a8[st]), b0 = smem_u32(S.q8[rc & (kQBufs - 1)]);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_mxf8(tmem + b * kAccCols, smem_desc(a0 + 32 * k, 16, 1024),
                                 smem_desc(b0 + 32 * k, 16, 1024), idesc, sfa + 4 * k, sfb + 2 * k, k > 0);
                } else {
                    const uint32_t a0 = smem_u32(S.a[st]), b0 = smem_u32(S.q[rc & (kQBufs - 1)]);
#pragma unroll
                    for (int t = 0; t < kTilesPerStep; ++t)
#pragma unroll
                        for (int k = 0; k < 2; ++k)
                            mma_mxf4(tmem + b * kAccCols + 64 * t,
                                     smem_desc(a0 + t * (kTileKeys * kKeyBytes) + 32 * k, 16, 512, 4),
                                     smem_desc(b0 + 32 * k, 16, 512, 4), idesc, sfa + 8 * t + 4 * k,
                                     sfb + 2 * k, k > 0);
                }
                mma_commit(&S.a_empty[st]);
                mma_commit(&S.acc_full[b]);
                if (++st == kStages) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------ scale writers
        // warp q writes TMEM lane quarter q.  Lane i handles keys 32 c + i
        // (SFA column group of MMA k-step s, column c) and heads i, 32 + i
        // (two SFB columns per k-step).  The MXFP4 MMA (K = 64) takes two
        // scales per row from bytes 0..1 of a column; the FP8 one (K = 32)
        // one scale from byte 0.
        const int quarter = warp & 3;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const int qt = threadIdx.x - 64;  // 0..127: quantiser thread (head qt / 2, dims 64 (qt & 1) ..)
        TileWalk tw(a, u0, u1);
        int64_t cur_row = -1;
        int rc = -1, st = 0;
        uint32_t ph = 0;
        bool ok = true;
        // after a timed-out wait the role keeps walking its steps without
        // waiting or touching memory, so that all 128 threads still meet at
        // the quantiser's named barrier; ok stays uniform within each warp
        for (int it = 0; tw.next(a); ++it) {
            const bool first_of_row = tw.row != cur_row;
            if (first_of_row) { cur_row = tw.row; ++rc; }
            const int qb = rc & (kQBufs - 1);
            if (QRAW && first_of_row) {
                // quantise the row's query block straight into the MMA layout
                if (ok && rc >= kQBufs) ok = mbar_wait(&S.q_empty[qb], uint32_t((rc / kQBufs) - 1) & 1u);
                if (ok) {
                    const int h = qt >> 1, half = qt & 1;
                    const uint4* src =
                        reinterpret_cast<const uint4*>(a.qraw + (cur_row * kHI + h) * kDI + 64 * half);
                    uint4 v[2][4];
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i >> 2][i & 3] = src[i];
                    uint32_t sb = 0;
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        uint4 codes;
                        sb |= quant_block32(v[blk], codes) << (8 * blk);
                        *reinterpret_cast<uint4*>(S.q[qb] + sw64_offset(h, 2 * half + blk)) = codes;
                    }
                    reinterpret_cast<uint16_t*>(&S.q_sf[qb][h])[half] = uint16_t(sb);
                    fence_proxy_async_smem();
                }
                ok = named_bar_and(1, 128, ok);  // every head's codes and scale bytes are written
                if (ok && lane == 0) mbar_arrive(&S.q_full[qb]);
            }
            // a_full of step it implies the MMA of step it - kStages is done,
            // so this stage's TMEM scale buffer is free
            if (ok) ok = mbar_wait(&S.a_full[st], ph);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                if constexpr (F8) {
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t wd = S.a_sf[st][32 * c + lane];
#pragma unroll
                        for (int k = 0; k < 4; ++k) v[4 * k + c] = __uint_as_float((wd >> (8 * k)) & 0xFFu);
                    }
                    tmem_st16(tmem + lane_addr + C::kSfaCol + C::kSfaPerStage * st, v);
                } else {
#pragma unroll
                    for (int t = 0; t < kTilesPerStep; ++t) {
                        uint32_t v[8];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint32_t wd = S.a_sf[st][128 * t + 32 * c + lane];
                            v[c] = wd & 0xFFFFu;
                            v[4 + c] = wd >> 16;
                        }
                        tmem_st8(tmem + lane_addr + C::kSfaCol + C::kSfaPerStage * st + 8 * t, v);
                    }
                }
                if (first_of_row) {
                    uint32_t w0, w1;
                    if (QRAW) {
                        w0 = S.q_sf[qb][lane];
                        w1 = S.q_sf[qb][32 + lane];
                    } else {
                        const uint32_t* qs = reinterpret_cast<const uint32_t*>(a.qIs) + cur_row * kHI;
                        w0 = qs[lane];
                        w1 = qs[32 + lane];
                    }
                    const uint32_t sfb = tmem + lane_addr + C::kSfbCol + C::kSfbPerBuf * (rc & (kStages - 1));
                    if constexpr (F8) {
                        uint32_t v[8];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[2 * k] = (w0 >> (8 * k)) & 0xFFu;
                            v[2 * k + 1] = (w1 >> (8 * k)) & 0xFFu;
                        }
                        tmem_st8(sfb, v);
                    } else {
                        tmem_st4(sfb, w0 & 0xFFFFu, w1 & 0xFFFFu, w0 >> 16, w1 >> 16);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();  // the whole warp's stores are done: one arrival per warp
                if (lane == 0) mbar_arrive(&S.sf_full[st]);
            }
            if (++st == kStages) { st = 0; ph ^= 1u; }
        }
    } else if (warp < kConvWarp0) {
        // ----------------------------------------------------------- epilogue
        const int g = (warp - kEpiWarp0) >> 2;        // group: steps with it % kEpiGroups == g
        const int sub = warp & 3;                     // TMEM lane quarter of this warp
        const int et = threadIdx.x - 32 * (kEpiWarp0 + 4 * g);  // 0..127
        float* ew = S.ew[g];
        TileWalk tw(a, u0, u1);
        int64_t cur_row = -1;
        bool ok = true;
        for (int it = 0; tw.next(a); ++it) {
            if (it % kEpiGroups != g) continue;
            if (tw.row != cur_row) {  // every thread of the group takes this branch together
                cur_row = tw.row;
                named_bar(2 + g, 128);
                if (et < kHI) ew[et] = a.w[cur_row * kHI + et];
                named_bar(2 + g, 128);
            }
            const int b = it % kAccBufs;
            if (ok) ok = mbar_wait(&S.acc_full[b], uint32_t(it / kAccBufs) & 1u);
            if (!ok) continue;
            tc_fence_after();
            float res[kTilesPerStep];
#pragma unroll
            for (int t = 0; t < kTilesPerStep; ++t) {
                const uint32_t base = tmem + (uint32_t(sub * 32) << 16) + b * kAccCols + 64 * t;
                // two interleaved partial sums, packed fma over (even, odd)
                // heads; the 64 head columns are read in two halves
                uint64_t acc2 = 0;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float v[2][16];
                    tmem_ld16(base + 32 * hf, v[0]);
                    tmem_ld16(base + 32 * hf + 16, v[1]);
                    tmem_wait_ld();
                    if (t == kTilesPerStep - 1 && hf == 1) {
                        tc_fence_before();
                        __syncwarp();  // one arrival per warp once all its loads are done
                        if (lane == 0) mbar_arrive(&S.acc_empty[b]);
                    }
#pragma unroll
                    for (int h = 0; h < 32; h += 4) {
                        const float4 wv = *reinterpret_cast<const float4*>(&ew[32 * hf + h]);
                        const float* vv = &v[h >> 4][h & 15];
                        acc2 = fma_f32x2(pack_f32x2(wv.x, wv.y),
                                         pack_f32x2(fmaxf(vv[0], 0.f), fmaxf(vv[1], 0.f)), acc2);
                        acc2 = fma_f32x2(pack_f32x2(wv.z, wv.w),
                                         pack_f32x2(fmaxf(vv[2], 0.f), fmaxf(vv[3], 0.f)), acc2);
                    }
                }
                const float2 accs = unpack_f32x2(acc2);
                res[t] = accs.x + accs.y;
            }
#pragma unroll
            for (int t = 0; t < kTilesPerStep; ++t) {
                const int64_t j = tw.k0() + kTileKeys * t + sub * 32 + lane;
                if (j < tw.ne) a.scores[cur_row * a.ld + j] = res[t];
            }
        }
    } else if constexpr (F8) {
        // ---------------------------------------------------------- converters
        // E2M1 -> E4M3 (exact) of each step's keys, and of each row's query
        // block; thread i expands row i (keys) / row i < 64 (heads).
        const int ct = threadIdx.x - 32 * kConvWarp0;  // 0..127
        TileWalk tw(a, u0, u1);
        int64_t cur_row = -1;
        int rc = -1, st = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int it = 0; ok && tw.next(a); ++it) {
            if (tw.row != cur_row) {
                cur_row = tw.row;
                ++rc;
                const int qb = rc & (kQBufs - 1);
                // q_full of row rc implies the MMAs of row rc - kQBufs are done
                ok = mbar_wait(&S.q_full[qb], uint32_t(rc / kQBufs) & 1u);
                if (!ok) break;
                if (ct < kHI) expand_row(S.q[qb], S.q8[qb], uint32_t(ct));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.q8_full[qb]);
            }
            // a_full of step it implies the MMA of step it - kStages is done
            ok = mbar_wait(&S.a_full[st], ph);
            if (!ok) break;
            expand_row(S.a[st], S.a8[st], uint32_t(ct));
            fence_proxy_async_smem();
            __syncwarp();  // one arrival per warp once all its rows are written
            if (lane == 0) mbar_arrive(&S.a8_full[st]);
            if (++st == kStages) { st = 0; ph ^= 1u; }
        }
    }
    // the producer and MMA roles run on one lane: reconverge every warp so
    // that the CTA barrier (an aligned bar.sync) sees whole warps and really
    // waits for those lanes before TMEM is freed
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

bool indexer_tc_supported(int fmt, int HI, int dI, int64_t max_blocks, int64_t batch, int64_t rows) {
    // the key map needs at least one whole 256-row box; row indices are int32
    return fmt == CSA_MXFP4 && HI == kHI && dI == kDI && (max_blocks % 4) == 0 &&
           batch * max_blocks >= kStepKeys && batch * max_blocks + kStepKeys <= INT32_MAX &&
           rows * kHI <= INT32_MAX;
}

// 2-D map over [n_rows][64] bytes with 64-byte swizzle and a box of box_rows.
static bool encode_rows64(CUtensorMap* map, const void* base, int64_t n_rows, int box_rows) {
    const uint64_t dims[2] = {uint64_t(kKeyBytes), uint64_t(n_rows)};
    const uint64_t strides[1] = {uint64_t(kKeyBytes)};
    const uint32_t box[2] = {uint32_t(kKeyBytes), uint32_t(box_rows)};
    return encode_tile_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_64B);
}

template <bool QRAW, bool F8>
static cudaError_t launch_variant(const CUtensorMap& map_k, const CUtensorMap& map_q, const IdxTcArgs& a,
                                  cudaStream_t s) {
    const size_t sm = sizeof(Smem<F8>) + 1024;
    cudaError_t e = ensure_smem(indexer_tc_kernel<QRAW, F8>, size_t(sm));
    if (e != cudaSuccess) return e;
    const int grid = int(std::min<int64_t>(int64_t(Cfg<F8>::kCtasPerSm) * kNumSMs, a.units));
    indexer_tc_kernel<QRAW, F8><<<grid, Cfg<F8>::kThreads, sm, s>>>(map_k, map_q, a);
    return cudaGetLastError();
}

cudaError_t launch_indexer_tc(const void* qI, const void* qI_s, const float* w, const void* kI,
                              const void* kI_s, int64_t max_blocks, const int64_t* q_pos,
                              int batch, int n_q, int m, int W, float* scores, int64_t ld,
                              bool q_bf16, bool fp8, cudaStream_t s) {
    IdxTcArgs a;
    a.kIs = (const uint8_t*)kI_s;
    a.qIs = q_bf16 ? nullptr : (const uint8_t*)qI_s;
    a.qraw = q_bf16 ? (const uint16_t*)qI : nullptr;
    a.w = w; a.q_pos = q_pos; a.scores = scores; a.ld = ld; a.max_blocks = max_blocks;
    a.n_q = n_q; a.m = m; a.W = W;
    a.rows = int64_t(batch) * n_q;
    a.tiles_per_row = ceil_div(max_blocks, kStepKeys);
    a.units = a.rows * a.tiles_per_row;
    if (a.units == 0) return cudaSuccess;
    CUtensorMap map_k, map_q;
    memset(&map_q, 0, sizeof(map_q));
    if (!encode_rows64(&map_k, kI, int64_t(batch) * max_blocks, kStepKeys) ||
        (!q_bf16 && !encode_rows64(&map_q, qI, a.rows * kHI, kHI)))
        return cudaErrorInvalidValue;
    if (q_bf16) return fp8 ? launch_variant<true, true>(map_k, map_q, a, s) : launch_variant<true, false>(map_k, map_q, a, s);
    return fp8 ? launch_variant<false, true>(map_k, map_q, a, s) : launch_variant<false, false>(map_k, map_q, a, s);
}

}  // namespace csa
