// Lightning indexer on the 5th-generation tensor cores, for MXFP4 queries and
// keys ("DeepSeek-V4 發佈說明", section 壓縮稀疏注意力 (CSA): ReLU-scored
// multi-head dot products in FP4; wiki summary, section 基础设施: MXFP4 on
// the indexer QK path, FP4 -> FP8 conversion is lossless).
//
//   s[j] = sum_h w[h] * ReLU(qI[h] . kI[j])
//
// The contraction runs as tcgen05.mma.kind::f8f6f4 with E4M3 operands: every
// E2M1 element times its block's E8M0 scale 2^X is exactly an E4M3 value as
// long as X lies in [-8, 6] (checked; outside it CSA_DEV_RANGE is flagged),
// so the products and the fp32 accumulation see the stored values exactly.
// The conversion is a byte-table lookup (prmt) per element nibble, with one
// 8-entry table per exponent X built once per CTA.
// One MMA tile: M = 128 keys (A, K-major, 128-byte swizzled rows), N = 64
// heads (B = the query block, K-major), K = 128 = 4 instructions of K = 32;
// the fp32 accumulator D[key][head] lives in TMEM, so the epilogue thread of
// TMEM lane j owns key j's 64 head scores and reduces them without any
// cross-thread traffic.
//
// Persistent CTAs take contiguous ranges of (query row, 128-key tile) units
// and walk them in order, skipping tiles past the row's eligible blocks; the
// k-th eligible tile of a CTA is "tile it = k".  Warp roles:
//   warp 0      bulk-async copies of raw key tiles (packed E2M1 + E8M0) into a
//               kRawStages ring (one elected lane), TMEM allocation
//   warp 1      MMA issue (one elected lane)
//   warps 2-9   two converter groups of four warps; group g converts the tiles
//               with it % 2 == g into A buffer it % 4, and the query block of
//               a row into query buffer (row count % 4) when its tile is the
//               first of that row
//   warps 10-17 two epilogue groups; group g reads accumulator it % 4 of its
//               tiles from TMEM, applies ReLU, weights and sums over heads
// Query buffers are safe to overwrite: the converter of tile it waits for the
// MMA of tile it - 4 (its A buffer), and MMAs complete in issue order; four
// row changes need at least four tiles.
// All waits are bounded (sm100::mbar_wait); after a timed-out wait a role
// keeps iterating without waiting or touching memory, so every thread still
// reaches the named and final barriers.
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kHI = 64, kDI = 128;
constexpr int kTileKeys = 128;
constexpr int kRawStages = 10;
constexpr int kABufs = 4, kAccBufs = 4, kQBufs = 4;
constexpr int kAccCols = 64;
constexpr int kKeyBytes = kDI / 2;                           // 64
constexpr int kRawData = kTileKeys * kKeyBytes;              // 8192
constexpr int kRawBytes = kRawData + kTileKeys * (kDI / 32); // + 512 scale bytes
constexpr int kATile = kTileKeys * kDI;                      // 16384 (E4M3)
constexpr int kQTile = kHI * kDI;                            // 8192
constexpr int kThreads = 576;
constexpr int kConvWarp0 = 2, kEpiWarp0 = 10;
constexpr int kLutMinX = -8, kLutMaxX = 6;  // exponents whose E2M1 x 2^X are all E4M3 values

struct IdxTcArgs {
    const uint8_t* kI;    // [batch][max_blocks][64]
    const uint8_t* kIs;   // [batch][max_blocks][4]
    const uint8_t* qI;    // [rows][64][64]
    const uint8_t* qIs;   // [rows][64][4]
    const float* w;       // [rows][64]
    const int64_t* q_pos; // [rows]
    float* scores;        // [rows][ld]
    int64_t ld, max_blocks;
    int n_q, m, W;
    int64_t rows, tiles_per_row, units;
};

struct Smem {
    uint8_t a[kABufs][kATile];         // 1024-aligned: E4M3 A tiles
    uint8_t q[kQBufs][kQTile];         // E4M3 B tiles (query blocks)
    uint8_t raw[kRawStages][kRawBytes];
    float ew[2][kHI];                  // per epilogue group: weights of its current row
    uint2 lut[kLutMaxX - kLutMinX + 1];  // E2M1 x 2^X -> E4M3 byte tables
    uint64_t raw_full[kRawStages], raw_empty[kRawStages];
    uint64_t a_full[kABufs], a_empty[kABufs], acc_full[kAccBufs], acc_empty[kAccBufs];
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
            if (tile * kTileKeys < ne) return true;
            u += tpr - tile;  // rest of this row is ineligible
            tile = tpr;
        }
        return false;
    }
    __device__ __forceinline__ int64_t k0() const { return tile * kTileKeys; }
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Byte lookup table of the eight E2M1 magnitudes times 2^X as E4M3 codes
// (x: codes 0..3, y: codes 4..7).  Every entry is exact for X in [-8, 6].
__device__ __forceinline__ uint2 make_e4m3_lut(int X) {
    const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
    uint32_t b[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint16_t r;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(ldexpf(mag[c], X)));
        b[c] = r & 0xFFu;
    }
    return make_uint2(b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24,
                      b[4] | b[5] << 8 | b[6] << 16 | b[7] << 24);
}

// Eight packed E2M1 elements (one word; element k in nibble k) -> eight E4M3
// bytes (two words): the magnitude nibbles index the table with prmt, and a
// second prmt in sign-replicate mode spreads each element's sign bit (bit 3
// of its nibble) over its output byte.
__device__ __forceinline__ uint2 e2m1x8_to_e4m3x8(uint32_t w, uint2 lut) {
    const uint32_t mag_lo = prmt(lut.x, lut.y, w & 0x7777u);
    const uint32_t mag_hi = prmt(lut.x, lut.y, (w >> 16) & 0x7777u);
    const uint32_t ws = w << 4;  // even elements' sign bits -> byte msbs
    const uint32_t sg_lo = prmt(ws, w, 0xD9C8u);
    const uint32_t sg_hi = prmt(ws, w, 0xFBEAu);
    return make_uint2(mag_lo | (sg_lo & 0x80808080u), mag_hi | (sg_hi & 0x80808080u));
}


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

// Table entry for an E8M0 byte; flags exponents outside the exact range.
__device__ __forceinline__ uint2 lut_for(const uint2* table, uint32_t e8m0) {
    int X = int(e8m0) - 127;
    if (X < kLutMinX || X > kLutMaxX) {
        flag_status(CSA_DEV_RANGE);
        X = max(kLutMinX, min(kLutMaxX, X));
    }
    return table[X - kLutMinX];
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) indexer_tc_kernel(const IdxTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using namespace sm100;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRawStages; ++i) { mbar_init(&S.raw_full[i], 1); mbar_init(&S.raw_empty[i], 128); }
        for (int i = 0; i < kABufs; ++i) { mbar_init(&S.a_full[i], 128); mbar_init(&S.a_empty[i], 1); }
        for (int i = 0; i < kAccBufs; ++i) { mbar_init(&S.acc_full[i], 1); mbar_init(&S.acc_empty[i], 128); }
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&S.tmem_base, kAccBufs * kAccCols); tmem_relinquish(); }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + (kLutMaxX - kLutMinX + 1))
        S.lut[threadIdx.x - 64] = make_e4m3_lut(int(threadIdx.x) - 64 + kLutMinX);
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
            int st = 0, issued = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int it = 0; ok && tw.next(a); ++it) {
                if (it >= kRawStages) ok = mbar_wait(&S.raw_empty[st], ph ^ 1u);
                if (!ok) break;
                ++issued;
                const int64_t k0 = tw.k0();
                int64_t nk = min(int64_t(kTileKeys), tw.ne - k0);
                nk = min((nk + 3) & ~int64_t(3), a.max_blocks - k0);  // max_blocks % 4 == 0
                const int64_t key0 = (tw.row / a.n_q) * a.max_blocks + k0;
                mbar_arrive_expect_tx(&S.raw_full[st], uint32_t(nk * (kKeyBytes + 4)));
                bulk_g2s(S.raw[st], a.kI + key0 * kKeyBytes, uint32_t(nk * kKeyBytes), &S.raw_full[st]);
                bulk_g2s(S.raw[st] + kRawData, a.kIs + key0 * 4, uint32_t(nk * 4), &S.raw_full[st]);
                if (++st == kRawStages) { st = 0; ph ^= 1u; }
            }
            // Let every copy still in flight land before the CTA exits (already
            // the case unless a consumer gave up on a wait).
            for (int i = max(0, issued - kRawStages); i < issued; ++i)
                if (!mbar_wait(&S.raw_full[i % kRawStages], uint32_t(i / kRawStages) & 1u)) break;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = instr_desc(0, 0, 0, 0, 128, 64);  // E4M3 x E4M3, K-major
            TileWalk tw(a, u0, u1);
            int64_t cur_row = -1;
            int rc = -1;
            bool ok = true;
            for (int it = 0; ok && tw.next(a); ++it) {
                if (tw.row != cur_row) { cur_row = tw.row; ++rc; }
                const int b = it & (kABufs - 1);
                const uint32_t par = uint32_t(it >> 2) & 1u;
                ok = mbar_wait(&S.a_full[b], par);
                if (ok && it >= kAccBufs) ok = mbar_wait(&S.acc_empty[b], par ^ 1u);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(S.a[b]), b0 = smem_u32(S.q[rc & (kQBufs - 1)]);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f8(tmem + b * kAccCols, smem_desc(a0 + k * 32, 16, 1024),
                           smem_desc(b0 + k * 32, 16, 1024), idesc, k > 0);
                mma_commit(&S.a_empty[b]);
                mma_commit(&S.acc_full[b]);
            }
        }
    } else if (warp < kEpiWarp0) {
        // --------------------------------------------------------- converters
        const int g = (warp - kConvWarp0) >> 2;         // group: tiles with it % 2 == g
        const int t = threadIdx.x - 32 * (kConvWarp0 + 4 * g);  // 0..127
        TileWalk tw(a, u0, u1);
        int64_t cur_row = -1;
        int rc = -1, rs = 0;
        uint32_t rph = 0;
        bool ok = true;
        for (int it = 0; ok && tw.next(a); ++it) {
            const bool first_of_row = tw.row != cur_row;
            if (first_of_row) { cur_row = tw.row; ++rc; }
            const int my_rs = rs;
            const uint32_t my_rph = rph;
            if (++rs == kRawStages) { rs = 0; rph ^= 1u; }
            if ((it & 1) != g) continue;
            const int b = it & (kABufs - 1);
            if (it >= kABufs) ok = mbar_wait(&S.a_empty[b], (uint32_t(it >> 2) & 1u) ^ 1u);
            if (!ok) break;
            if (first_of_row) {
                // query block of this row -> E4M3 B tile: thread t does head t/2, half t%2
                const int h = t >> 1, half = t & 1;
                const int64_t row = tw.row;
                uint8_t* qdst = S.q[rc & (kQBufs - 1)];
                const uint8_t* src = a.qI + (row * kHI + h) * kKeyBytes + half * 32;
                const uint8_t* srs = a.qIs + (row * kHI + h) * 4 + half * 2;
                const uint4 p0 = *reinterpret_cast<const uint4*>(src);
                const uint4 p1 = *reinterpret_cast<const uint4*>(src + 16);
                const uint2 s0 = lut_for(S.lut, srs[0]), s1 = lut_for(S.lut, srs[1]);
                const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // 16 elements per 16-byte chunk
                    const uint2 sc = c < 2 ? s0 : s1;
                    const uint2 lo = e2m1x8_to_e4m3x8(pw[2 * c], sc);
                    const uint2 hi = e2m1x8_to_e4m3x8(pw[2 * c + 1], sc);
                    *reinterpret_cast<uint4*>(qdst + sw128_offset(h, half * 4 + c)) =
                        make_uint4(lo.x, lo.y, hi.x, hi.y);
                }
            }
            ok = mbar_wait(&S.raw_full[my_rs], my_rph);
            if (!ok) break;
            // four consecutive threads share a key, one 32-element MX block each:
            // 16-byte reads at consecutive addresses, two swizzled 16-byte writes
            const int64_t k0 = tw.k0(), ne = tw.ne;
            const int blk = t & 3;
            const uint8_t* raw = S.raw[my_rs];
#pragma unroll
            for (int pass = 0; pass < 4; ++pass) {
                const int key = (t >> 2) + 32 * pass;
                uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
                if (k0 + key < ne) {
                    const uint4 pk = *reinterpret_cast<const uint4*>(raw + key * kKeyBytes + 16 * blk);
                    const uint2 sc = lut_for(S.lut, raw[kRawData + key * 4 + blk]);
                    const uint2 e0 = e2m1x8_to_e4m3x8(pk.x, sc), e1 = e2m1x8_to_e4m3x8(pk.y, sc);
                    const uint2 e2 = e2m1x8_to_e4m3x8(pk.z, sc), e3 = e2m1x8_to_e4m3x8(pk.w, sc);
                    o0 = make_uint4(e0.x, e0.y, e1.x, e1.y);
                    o1 = make_uint4(e2.x, e2.y, e3.x, e3.y);
                }
                *reinterpret_cast<uint4*>(S.a[b] + sw128_offset(key, 2 * blk)) = o0;
                *reinterpret_cast<uint4*>(S.a[b] + sw128_offset(key, 2 * blk + 1)) = o1;
            }
            fence_proxy_async_smem();
            mbar_arrive(&S.raw_empty[my_rs]);
            mbar_arrive(&S.a_full[b]);
        }
    } else {
        // ----------------------------------------------------------- epilogue
        const int g = (warp - kEpiWarp0) >> 2;        // group: tiles with it % 2 == g
        const int sub = warp & 3;                     // TMEM lane quarter of this warp
        const int key = sub * 32 + lane;              // key within the tile
        const int et = threadIdx.x - 32 * (kEpiWarp0 + 4 * g);  // 0..127
        float* ew = S.ew[g];
        TileWalk tw(a, u0, u1);
        int64_t cur_row = -1;
        bool ok = true;
        for (int it = 0; tw.next(a); ++it) {
            if ((it & 1) != g) continue;
            if (tw.row != cur_row) {  // every thread of the group takes this branch together
                cur_row = tw.row;
                named_bar(2 + g, 128);
                if (et < kHI) ew[et] = a.w[cur_row * kHI + et];
                named_bar(2 + g, 128);
            }
            const int b = it & (kAccBufs - 1);
            if (ok) ok = mbar_wait(&S.acc_full[b], uint32_t(it >> 2) & 1u);
            if (!ok) continue;
            tc_fence_after();
            const uint32_t base = tmem + (uint32_t(sub * 32) << 16) + b * kAccCols;
            // two interleaved partial sums, packed fma over (even, odd) heads;
            // the 64 head columns are read in two halves
            uint64_t acc2 = 0;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float v[2][16];
                tmem_ld16(base + 32 * hf, v[0]);
                tmem_ld16(base + 32 * hf + 16, v[1]);
                tmem_wait_ld();
                if (hf == 1) {
                    tc_fence_before();
                    mbar_arrive(&S.acc_empty[b]);
                }
#pragma unroll
                for (int h = 0; h < 32; h += 2) {
                    const float2 wv = *reinterpret_cast<const float2*>(&ew[32 * hf + h]);
                    const float r0 = fmaxf(v[h >> 4][h & 15], 0.f);
                    const float r1 = fmaxf(v[h >> 4][(h & 15) + 1], 0.f);
                    acc2 = fma_f32x2(pack_f32x2(wv.x, wv.y), pack_f32x2(r0, r1), acc2);
                }
            }
            const float2 accs = unpack_f32x2(acc2);
            const int64_t j = tw.k0() + key;
            if (j < tw.ne) a.scores[cur_row * a.ld + j] = accs.x + accs.y;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kAccBufs * kAccCols);
}

bool indexer_tc_supported(int fmt, int HI, int dI, int64_t max_blocks) {
    return fmt == CSA_MXFP4 && HI == kHI && dI == kDI && (max_blocks % 4) == 0;
}

cudaError_t launch_indexer_tc(const void* qI, const void* qI_s, const float* w, const void* kI,
                              const void* kI_s, int64_t max_blocks, const int64_t* q_pos,
                              int batch, int n_q, int m, int W, float* scores, int64_t ld,
                              cudaStream_t s) {
    IdxTcArgs a;
    a.kI = (const uint8_t*)kI; a.kIs = (const uint8_t*)kI_s;
    a.qI = (const uint8_t*)qI; a.qIs = (const uint8_t*)qI_s;
    a.w = w; a.q_pos = q_pos; a.scores = scores; a.ld = ld; a.max_blocks = max_blocks;
    a.n_q = n_q; a.m = m; a.W = W;
    a.rows = int64_t(batch) * n_q;
    a.tiles_per_row = ceil_div(max_blocks, kTileKeys);
    a.units = a.rows * a.tiles_per_row;
    if (a.units == 0) return cudaSuccess;
    const size_t sm = sizeof(Smem) + 1024;
    cudaError_t e = ensure_smem(indexer_tc_kernel, size_t(sm));
    if (e != cudaSuccess) return e;
    const int grid = int(std::min<int64_t>(kNumSMs, a.units));
    indexer_tc_kernel<<<grid, kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
