// Lightning indexer on the 5th-generation tensor cores for bf16 queries and
// keys, the prefill form ("DeepSeek-V4 發佈說明", section 壓縮稀疏注意力 (CSA):
// every query scores the compressed blocks with ReLU-activated multi-head dot
// products weighted per head):
//
//   s[t][j] = sum_h w[t][h] * ReLU(qI[t][h] . kI[j]),   j < n_elig(t)
//
// One unit = (a group of 4 consecutive query rows of one sequence, a tile of
// 128 keys):
//
//   D[key][4 x 64 heads] = kI_tile (M = 128, K = 128) . qI_group^T (N = 256)
//
// as eight kind::f16 MMAs of K = 16; both operands are K-major in the
// 128-byte-swizzled layout that the tensor copy writes ([2 dim halves][rows]
// [64 bf16]).  bf16 products are exact in fp32 and accumulate in fp32.  The
// accumulator (256 TMEM columns, two buffers) is reduced by the epilogue
// thread of TMEM lane j: key j's 64 head scores per row, ReLU, weights, sum.
// A group is computed only over the tiles below its largest eligible count,
// and each row writes only its own eligible keys.  Groups are dealt to
// persistent CTAs round-robin, latest (largest) first, so that the work of
// the causal triangle balances across SMs.
//
// Roles (192 threads, one CTA per SM: ~225 KB of shared memory, all 512
// TMEM columns):
//   warp 0      tensor copies (one elected lane): the group's queries into a
//               two-buffer ring, each key tile into a three-stage ring; TMEM
//               allocation
//   warp 1      MMA issue (one elected lane)
//   warps 2-5   epilogue (TMEM lane quarter = warp % 4)
// All waits are bounded (sm100::mbar_wait); after a timed-out wait a role
// keeps iterating without waiting or touching memory, so every thread still
// reaches the named and final barriers.
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kHI = 64, kDI = 128;
constexpr int kQ = 4;                      // query rows per group
constexpr int kN = kQ * kHI;               // 256: MMA N
constexpr int kKeys = 128;                 // MMA M
constexpr int kAStages = 3, kBBufs = 2, kAccBufs = 2;
constexpr int kAHalf = kKeys * 128;        // 16 KB: [128 keys][64 bf16]
constexpr int kBHalf = kN * 128;           // 32 KB: [256 rows][64 bf16]
constexpr int kAccCols = kN;               // 256
constexpr int kTmemCols = kAccBufs * kAccCols;
constexpr int kThreads = 192;

struct IdxBf16Args {
    const float* w;        // [rows][64]
    const int64_t* q_pos;  // [rows]
    float* scores;         // [rows][ld]
    int64_t ld, max_blocks;
    int n_q, m, W;
    int64_t groups_per_seq, n_groups;
};

struct Smem {
    uint8_t a[kAStages][2 * kAHalf];  // 1024-aligned: key tiles
    uint8_t b[kBBufs][2 * kBHalf];    // query groups
    float ew[kQ][kHI];                // weights of the epilogue's current group
    uint64_t a_full[kAStages], a_empty[kAStages], b_full[kBBufs], b_empty[kBBufs];
    uint64_t acc_full[kAccBufs], acc_empty[kAccBufs];
    uint32_t tmem_base;
};

struct Group {
    int64_t row0, key0;  // first query row; first key row of the sequence
    int nrows, tiles;
};

// g-th group of this walk (latest first); every role derives the same groups
__device__ __forceinline__ Group group_of(const IdxBf16Args& a, int64_t g) {
    const int64_t gg = a.n_groups - 1 - g;
    const int64_t b = gg / a.groups_per_seq;
    const int i0 = int(gg - b * a.groups_per_seq) * kQ;
    Group G;
    G.row0 = b * a.n_q + i0;
    G.key0 = b * a.max_blocks;
    G.nrows = min(kQ, a.n_q - i0);
    int64_t ne = 0;
    for (int r = 0; r < G.nrows; ++r) ne = max(ne, min(n_elig(a.q_pos[G.row0 + r], a.m, a.W), a.max_blocks));
    G.tiles = int(ceil_div(ne, kKeys));
    return G;
}

__device__ __forceinline__ uint64_t pack_f32x2(float x, float y) {
    return uint64_t(__float_as_uint(x)) | (uint64_t(__float_as_uint(y)) << 32);
}
// (a.x*b.x + c.x, a.y*b.y + c.y), each rounded once
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    indexer_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                           const __grid_constant__ CUtensorMap map_q, const IdxBf16Args a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using namespace sm100;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kAStages; ++i) { mbar_init(&S.a_full[i], 1); mbar_init(&S.a_empty[i], 1); }
        for (int i = 0; i < kBBufs; ++i) { mbar_init(&S.b_full[i], 1); mbar_init(&S.b_empty[i], 1); }
        for (int i = 0; i < kAccBufs; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], 4);  // one arrival per epilogue warp
        }
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&S.tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int gc = 0, it = 0, st = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int64_t g = blockIdx.x; ok && g < a.n_groups; g += gridDim.x) {
                const Group G = group_of(a, g);
                if (G.tiles == 0) continue;
                const int gb = gc & 1;
                if (gc >= kBBufs) ok = mbar_wait(&S.b_empty[gb], uint32_t((gc >> 1) - 1) & 1u);
                if (!ok) break;
                // rows of a partial group past the sequence are read but never used
                mbar_arrive_expect_tx(&S.b_full[gb], uint32_t(2 * kBHalf));
                tma_load_2d(S.b[gb], &map_q, 0, int32_t(G.row0 * kHI), &S.b_full[gb]);
                tma_load_2d(S.b[gb] + kBHalf, &map_q, 64, int32_t(G.row0 * kHI), &S.b_full[gb]);
                ++gc;
                for (int t = 0; ok && t < G.tiles; ++t) {
                    if (it >= kAStages) ok = mbar_wait(&S.a_empty[st], ph ^ 1u);
                    if (!ok) break;
                    // the whole box always arrives (rows past the tensor read as zero)
                    const int32_t k0 = int32_t(G.key0 + int64_t(t) * kKeys);
                    mbar_arrive_expect_tx(&S.a_full[st], uint32_t(2 * kAHalf));
                    tma_load_2d(S.a[st], &map_k, 0, k0, &S.a_full[st]);
                    tma_load_2d(S.a[st] + kAHalf, &map_k, 64, k0, &S.a_full[st]);
                    ++it;
                    if (++st == kAStages) { st = 0; ph ^= 1u; }
                }
            }
            // Let every copy still in flight land before the CTA exits (already
            // the case unless a consumer gave up on a wait).
            bool drained = true;
            for (int i = max(0, it - kAStages); i < it && drained; ++i)
                drained = mbar_wait(&S.a_full[i % kAStages], uint32_t(i / kAStages) & 1u);
            for (int i = max(0, gc - kBBufs); i < gc && drained; ++i)
                drained = mbar_wait(&S.b_full[i & 1], uint32_t(i >> 1) & 1u);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc(1, 1, 0, 0, kKeys, kN);  // bf16, both K-major
            int gc = 0, it = 0, st = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int64_t g = blockIdx.x; ok && g < a.n_groups; g += gridDim.x) {
                const Group G = group_of(a, g);
                if (G.tiles == 0) continue;
                const int gb = gc & 1;
                ok = mbar_wait(&S.b_full[gb], uint32_t(gc >> 1) & 1u);
                const uint32_t b0 = smem_u32(S.b[gb]);
                for (int t = 0; ok && t < G.tiles; ++t) {
                    const int ab = it & 1;
                    ok = mbar_wait(&S.a_full[st], ph);
                    if (ok && it >= kAccBufs) ok = mbar_wait(&S.acc_empty[ab], (uint32_t(it >> 1) & 1u) ^ 1u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.a[st]);
#pragma unroll
                    for (int k = 0; k < kDI / 16; ++k) {
                        const int half = k >> 2, ks = k & 3;
                        mma_f16(tmem + ab * kAccCols, smem_desc(a0 + half * kAHalf + 32 * ks, 16, 1024),
                                smem_desc(b0 + half * kBHalf + 32 * ks, 16, 1024), idesc, k > 0);
                    }
                    mma_commit(&S.a_empty[st]);
                    mma_commit(&S.acc_full[ab]);
                    ++it;
                    if (++st == kAStages) { st = 0; ph ^= 1u; }
                }
                if (ok) mma_commit(&S.b_empty[gb]);  // after the group's last MMA completes
                ++gc;
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue
        const int sub = warp & 3;                 // TMEM lane quarter of this warp
        const int et = threadIdx.x - 64;          // 0..127
        const uint32_t lane_addr = uint32_t(sub * 32) << 16;
        int it = 0;
        bool ok = true;
        for (int64_t g = blockIdx.x; g < a.n_groups; g += gridDim.x) {
            const Group G = group_of(a, g);
            if (G.tiles == 0) continue;
            named_bar(1, 128);  // every thread is done with the previous group's weights
            for (int i = et; i < kQ * kHI; i += 128) {
                const int q = i / kHI;
                S.ew[q][i % kHI] = q < G.nrows ? a.w[(G.row0 + q) * kHI + i % kHI] : 0.f;
            }
            int64_t ne[kQ];
#pragma unroll
            for (int q = 0; q < kQ; ++q)
                ne[q] = q < G.nrows ? min(n_elig(a.q_pos[G.row0 + q], a.m, a.W), a.max_blocks) : 0;
            named_bar(1, 128);
            for (int t = 0; t < G.tiles; ++t, ++it) {
                const int ab = it & 1;
                if (ok) ok = mbar_wait(&S.acc_full[ab], uint32_t(it >> 1) & 1u);
                if (!ok) continue;
                tc_fence_after();
                float res[kQ];
#pragma unroll
                for (int q = 0; q < kQ; ++q) {
                    // two interleaved partial sums, packed fma over (even, odd) heads
                    uint64_t acc2 = 0;
#pragma unroll 1
                    for (int hf = 0; hf < 2; ++hf) {
                        float v[2][16];
                        const uint32_t base = tmem + lane_addr + ab * kAccCols + 64 * q + 32 * hf;
                        tmem_ld16(base, v[0]);
                        tmem_ld16(base + 16, v[1]);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < 32; h += 4) {
                            const float4 wv = *reinterpret_cast<const float4*>(&S.ew[q][32 * hf + h]);
                            const float* vv = &v[h >> 4][h & 15];
                            acc2 = fma_f32x2(pack_f32x2(wv.x, wv.y),
                                             pack_f32x2(fmaxf(vv[0], 0.f), fmaxf(vv[1], 0.f)), acc2);
                            acc2 = fma_f32x2(pack_f32x2(wv.z, wv.w),
                                             pack_f32x2(fmaxf(vv[2], 0.f), fmaxf(vv[3], 0.f)), acc2);
                        }
                    }
                    res[q] = __uint_as_float(uint32_t(acc2)) + __uint_as_float(uint32_t(acc2 >> 32));
                }
                tc_fence_before();
                __syncwarp();  // one arrival per warp once all its loads are done
                if (lane == 0) mbar_arrive(&S.acc_empty[ab]);
                const int64_t j = int64_t(t) * kKeys + sub * 32 + lane;
#pragma unroll
                for (int q = 0; q < kQ; ++q)
                    if (j < ne[q]) a.scores[(G.row0 + q) * a.ld + j] = res[q];
            }
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

bool indexer_bf16_tc_supported(int fmt, int HI, int dI, int64_t max_blocks, int64_t batch, int n_q) {
    // the maps need at least one whole box each; row indices are int32
    const int64_t rows = batch * n_q;
    return fmt == CSA_BF16 && HI == kHI && dI == kDI && n_q >= kQ && batch * max_blocks >= kKeys &&
           batch * max_blocks + kKeys <= INT32_MAX && rows * kHI + kN <= INT32_MAX;
}

cudaError_t launch_indexer_bf16_tc(const void* qI, const float* w, const void* kI, int64_t max_blocks,
                                   const int64_t* q_pos, int batch, int n_q, int m, int W,
                                   float* scores, int64_t ld, cudaStream_t s) {
    IdxBf16Args a;
    a.w = w; a.q_pos = q_pos; a.scores = scores; a.ld = ld; a.max_blocks = max_blocks;
    a.n_q = n_q; a.m = m; a.W = W;
    a.groups_per_seq = ceil_div(int64_t(n_q), kQ);
    a.n_groups = int64_t(batch) * a.groups_per_seq;
    if (a.n_groups == 0 || max_blocks == 0) return cudaSuccess;
    // keys [batch * max_blocks][128] and queries [rows * 64][128], bf16, read
    // as boxes of [128 or 256 rows][64 dims] with 128-byte swizzle
    CUtensorMap map_k, map_q;
    const uint64_t kd[2] = {uint64_t(kDI), uint64_t(int64_t(batch) * max_blocks)};
    const uint64_t qd[2] = {uint64_t(kDI), uint64_t(int64_t(batch) * n_q * kHI)};
    const uint64_t rs[1] = {uint64_t(kDI) * 2};
    const uint32_t kbox[2] = {64, kKeys}, qbox[2] = {64, kN};
    if (!encode_tile_map(&map_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kI, kd, rs, kbox,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tile_map(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qI, qd, rs, qbox,
                         CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t sm = sizeof(Smem) + 1024;
    cudaError_t e = ensure_smem(indexer_bf16_tc_kernel, sm);
    if (e != cudaSuccess) return e;
    const int grid = int(std::min<int64_t>(kNumSMs, a.n_groups));
    indexer_bf16_tc_kernel<<<grid, kThreads, sm, s>>>(map_k, map_q, a);
    return cudaGetLastError();
}

}  // namespace csa
