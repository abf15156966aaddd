// MQA attention over pooled entries + the raw window + a per-head sink, on
// CUDA cores in fp32 (wiki summary "DeepSeek V4", section 架构创新: top-k
// sparse selection + MQA, sliding-window branch and attention sink; release
// note sections CSA and HCA).
//
// Work item = (query row, split).  The items a query attends are numbered
// slot 0.. : first the pooled slots (CSA: the k selected ids, -1 skipped;
// HCA: every visible block), then the window tokens.  A split takes a
// contiguous slot range and runs an online softmax over it in tiles of 32
// items: the tile is decoded to fp32 in shared memory, S = q.k for all heads,
// running max / sum per head, O += P.V.  With one split the CTA writes the
// normalised output (sink included); otherwise it writes (m, l, O) partials
// for the log-sum-exp combine kernel.
//
// This is the exact-fp32 path (the fp32 format) and the reference-precision
// path for every other format.
#include "kernels.h"

namespace csa {

constexpr int kAttnThreads = 256;
constexpr int kTile = 32;

// Slot layout of one query row (shared by the attention kernels).
struct RowSlots {
    int64_t n_kv;     // pooled slots
    int64_t win_lo;   // first window position
    int64_t n_win;    // window slots
};

__device__ __forceinline__ RowSlots row_slots(const AttnArgs& a, int64_t row) {
    RowSlots r;
    const int64_t b = row / a.n_q;
    const int64_t t = a.q_pos[row];
    r.n_kv = a.idx ? (a.n_sel ? min(int64_t(a.n_sel[row]), int64_t(a.k)) : a.k)
                   : min(max(n_elig(t, a.m, a.W) - a.kv_base, int64_t(0)), a.max_entries);
    const int64_t p0 = a.raw_pos0[b];
    const int64_t lo = max(max(t - a.W + 1, int64_t(0)), p0);
    const int64_t hi = min(t + 1, p0 + a.n_raw);
    r.win_lo = lo;
    r.n_win = max(int64_t(0), hi - lo);
    return r;
}

template <int DPT, int ACT, int KV>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_simt_kernel(AttnArgs a) {
    extern __shared__ float smem[];
    const int H = a.H, D = a.D;
    float* q_s = smem;                            // [H][D]
    float* k_s = q_s + H * D;                     // [kTile][D+1]
    float* p_s = k_s + kTile * (D + 1);           // [H][kTile+1]
    float* m_s = p_s + H * (kTile + 1);           // [H] running max (scaled logits)
    float* l_s = m_s + H;                         // [H] running sum
    float* al_s = l_s + H;                        // [H] rescale factor of this tile
    int64_t* src_s = (int64_t*)(al_s + H);           // [kTile] source row, -1 = empty (8B aligned: the float offset is even)
    int* israw_s = (int*)(src_s + kTile);         // [kTile]

    const int tid = threadIdx.x;
    const int64_t row = blockIdx.y;
    const int split = blockIdx.x;
    const int64_t b = row / a.n_q;
    const RowSlots rs = row_slots(a, row);
    const int64_t total = rs.n_kv + rs.n_win;
    const int64_t per = ceil_div(total, a.n_splits);
    const int64_t s_lo = min(total, split * per), s_hi = min(total, s_lo + per);

    for (int e = tid; e < H * D; e += kAttnThreads)
        q_s[e] = load_elem<ACT>(a.q, nullptr, row * H + e / D, D, e % D);
    for (int h = tid; h < H; h += kAttnThreads) { m_s[h] = -INFINITY; l_s[h] = 0.f; }

    const int TPH = kAttnThreads / H;             // threads per head in P.V
    const int my_h = tid / TPH, my_q = tid % TPH;
    float o[DPT];
#pragma unroll
    for (int j = 0; j < DPT; ++j) o[j] = 0.f;

    for (int64_t t0 = s_lo; t0 < s_hi; t0 += kTile) {
        __syncthreads();
        if (tid < kTile) {
            const int64_t slot = t0 + tid;
            int64_t src = -1;
            int is_raw = 0;
            if (slot < s_hi) {
                if (slot < rs.n_kv) {
                    const int64_t j = a.idx ? int64_t(a.idx[row * a.k + slot]) : slot;
                    if (j >= a.max_entries) flag_status(CSA_DEV_BAD_INDEX);
                    else if (j >= 0) src = b * a.max_entries + j;
                } else {
                    src = b * a.n_raw + (rs.win_lo + (slot - rs.n_kv) - a.raw_pos0[b]);
                    is_raw = 1;
                }
            }
            src_s[tid] = src;
            israw_s[tid] = is_raw;
        }
        __syncthreads();
        for (int e = tid; e < kTile * D; e += kAttnThreads) {
            const int r = e / D, c = e % D;
            const int64_t src = src_s[r];
            float v = 0.f;
            if (src >= 0)
                v = israw_s[r] ? load_elem<ACT>(a.raw, nullptr, src, D, c)
                               : load_elem<KV>(a.kv, a.kv_s, src, D, c);
            k_s[r * (D + 1) + c] = v;
        }
        __syncthreads();
        // logits: pair p -> head p / kTile, item p % kTile
        for (int p = tid; p < H * kTile; p += kAttnThreads) {
            const int h = p / kTile, e = p % kTile;
            float dot = 0.f;
            const float* qh = q_s + h * D;
            const float* kr = k_s + e * (D + 1);
            for (int c = 0; c < D; ++c) dot = fmaf(qh[c], kr[c], dot);
            p_s[h * (kTile + 1) + e] = src_s[e] >= 0 ? dot * a.scale : -INFINITY;
        }
        __syncthreads();
        for (int h = tid; h < H; h += kAttnThreads) {
            float* ph = p_s + h * (kTile + 1);
            float mx = -INFINITY;
            for (int e = 0; e < kTile; ++e) mx = fmaxf(mx, ph[e]);
            const float m_old = m_s[h];
            const float m_new = fmaxf(m_old, mx);
            float alpha = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                alpha = expf(m_old - m_new);  // 0 when m_old = -inf
                for (int e = 0; e < kTile; ++e) {
                    const float pe = expf(ph[e] - m_new);
                    ph[e] = pe;
                    sum += pe;
                }
            } else {
                for (int e = 0; e < kTile; ++e) ph[e] = 0.f;
            }
            m_s[h] = m_new;
            l_s[h] = l_s[h] * alpha + sum;
            al_s[h] = alpha;
        }
        __syncthreads();
        {
            const float alpha = al_s[my_h];
#pragma unroll
            for (int j = 0; j < DPT; ++j) o[j] *= alpha;
            const float* ph = p_s + my_h * (kTile + 1);
            for (int e = 0; e < kTile; ++e) {
                const float pe = ph[e];
                const float* kr = k_s + e * (D + 1) + my_q;
#pragma unroll
                for (int j = 0; j < DPT; ++j) o[j] = fmaf(pe, kr[j * TPH], o[j]);
            }
        }
    }
    __syncthreads();
    const float m_run = m_s[my_h], l_run = l_s[my_h];
    if (a.n_splits == 1 && !a.partial_out) {
        float den = l_run, f = 1.f;
        if (a.sinks) {
            const float sg = a.sinks[my_h];
            const float M = fmaxf(m_run, sg);
            f = (m_run == -INFINITY) ? 0.f : expf(m_run - M);
            den = l_run * f + expf(sg - M);
        }
        const float inv = den > 0.f ? f / den : 0.f;
        const int64_t base = (row * H + my_h) * int64_t(D);
#pragma unroll
        for (int j = 0; j < DPT; ++j) {
            const int c = my_q + j * TPH;
            if constexpr (ACT == CSA_F32) ((float*)a.out)[base + c] = o[j] * inv;
            else ((__nv_bfloat16*)a.out)[base + c] = __float2bfloat16_rn(o[j] * inv);
        }
    } else {
        const int64_t item = row * a.n_splits + split;
        float* po = a.part_o + (item * H + my_h) * int64_t(D);
#pragma unroll
        for (int j = 0; j < DPT; ++j) po[my_q + j * TPH] = o[j];
        if (my_q == 0) a.part_ml[item * H + my_h] = make_float2(m_run, l_run);
    }
}

template <int DPT, int ACT, int KV>
static cudaError_t launch_attn_t(const AttnArgs& a, int64_t rows, cudaStream_t s) {
    const size_t sm = size_t(a.H * a.D + kTile * (a.D + 1) + a.H * (kTile + 1) + 3 * a.H + 2) * 4 +
                      kTile * (8 + 4) + 16;
    cudaError_t e = ensure_smem(attn_simt_kernel<DPT, ACT, KV>, size_t(sm));
    if (e != cudaSuccess) return e;
    attn_simt_kernel<DPT, ACT, KV><<<dim3(a.n_splits, unsigned(rows)), kAttnThreads, sm, s>>>(a);
    return cudaGetLastError();
}

// Split-K LSE combine of a row's partial attention results ([RN] CSA / HCA:
// one softmax over all attended items and the sink).  Partial s of row r is
// item r * row_stride + s * split_stride of part_o ([item][H][D] fp32, the
// unnormalised sum relative to the item's running max) and part_ml ([item][H]:
// max in natural-log units, sum of exponentials).  The per-split weights are
// computed once into shared memory, then each thread accumulates float4
// slices with the split loads issued four at a time.
//   PARTIAL = false: out = sum_s w_s O_s / (sum_s w_s l_s + e^(sink - M)) in
//     the activation format (the sink, if any, takes part in the max M).
//   PARTIAL = true: the merged partial itself, with no sink: out (fp32) =
//     sum_s w_s O_s and out_ml = (M, sum_s w_s l_s), M the max over splits.
template <int ACT, bool PARTIAL>
__global__ void __launch_bounds__(128) combine_kernel(int H, int D, int n_splits, int64_t row_stride,
                                                      int64_t split_stride, const float* __restrict__ part_o,
                                                      const float2* __restrict__ part_ml,
                                                      const float* __restrict__ sinks, void* out,
                                                      float2* out_ml) {
    __shared__ float wgt[64];
    __shared__ float inv_s;
    pdl_wait();  // the partials come from the attention kernel before it
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y;
    const float* sk = PARTIAL ? nullptr : sinks;
    auto ml_of = [&](int s) { return part_ml[(row * row_stride + s * split_stride) * H + h]; };
    if (threadIdx.x < 32) {
        float M = sk ? sk[h] : -INFINITY;
        for (int s = threadIdx.x; s < n_splits; s += 32) M = fmaxf(M, ml_of(s).x);
        M = warp_max(M);
        float den = 0.f;
        for (int s = threadIdx.x; s < n_splits; s += 32) {
            const float2 v = ml_of(s);
            const float w = v.x == -INFINITY ? 0.f : expf(v.x - M);
            wgt[s] = w;
            den += w * v.y;
        }
        den = warp_sum(den);
        if (threadIdx.x == 0) {
            if (sk && M != -INFINITY) den += expf(sk[h] - M);
            if (PARTIAL) {
                out_ml[row * H + h] = make_float2(M, den);
                inv_s = 1.f;
            } else {
                inv_s = den > 0.f ? 1.f / den : 0.f;
            }
        }
    }
    __syncthreads();
    const float inv = inv_s;
    const int64_t stride = split_stride * H * D;  // between splits
    for (int c = 4 * threadIdx.x; c < D; c += 4 * blockDim.x) {
        const float* base = part_o + (row * row_stride * H + h) * int64_t(D) + c;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int s = 0;
        for (; s + 4 <= n_splits; s += 4) {
            float4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const float4*>(base + (s + j) * stride);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float w = wgt[s + j];
                if (w == 0.f) continue;  // an empty split adds nothing (its partial is not read)
                acc.x = fmaf(w, v[j].x, acc.x); acc.y = fmaf(w, v[j].y, acc.y);
                acc.z = fmaf(w, v[j].z, acc.z); acc.w = fmaf(w, v[j].w, acc.w);
            }
        }
        for (; s < n_splits; ++s) {
            const float w = wgt[s];
            if (w == 0.f) continue;
            const float4 v = *reinterpret_cast<const float4*>(base + s * stride);
            acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
        }
        const int64_t o = (row * H + h) * int64_t(D) + c;
        if constexpr (PARTIAL || ACT == CSA_F32) {
            *reinterpret_cast<float4*>((float*)out + o) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        } else {
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>((__nv_bfloat16*)out + o) = pk;
        }
    }
}

cudaError_t launch_combine_strided(int act, bool partial, int H, int D, int n_splits, int64_t rows,
                                   int64_t row_stride, int64_t split_stride, const float* part_o,
                                   const float2* part_ml, const float* sinks, void* out, float2* out_ml,
                                   cudaStream_t s, bool pdl) {
    if (rows == 0) return cudaSuccess;
    if (n_splits > 64) return cudaErrorInvalidValue;  // the weights live in a 64-entry table
    const dim3 grid{unsigned(rows), unsigned(H)};
    if (partial)
        return launch_ex(combine_kernel<CSA_F32, true>, grid, dim3(128), 0, s, pdl, H, D, n_splits, row_stride,
                         split_stride, part_o, part_ml, sinks, out, out_ml);
    if (act == CSA_F32)
        return launch_ex(combine_kernel<CSA_F32, false>, grid, dim3(128), 0, s, pdl, H, D, n_splits, row_stride,
                         split_stride, part_o, part_ml, sinks, out, out_ml);
    return launch_ex(combine_kernel<CSA_BF16, false>, grid, dim3(128), 0, s, pdl, H, D, n_splits, row_stride,
                     split_stride, part_o, part_ml, sinks, out, out_ml);
}

cudaError_t launch_combine(int act, int H, int D, int n_splits, int64_t rows, const float* part_o,
                           const float2* part_ml, const float* sinks, void* out, cudaStream_t s,
                           bool pdl) {
    return launch_combine_strided(act, false, H, D, n_splits, rows, n_splits, 1, part_o, part_ml, sinks, out,
                                  nullptr, s, pdl);
}

// Dispatch on (dims per thread, activation format, entry format).
cudaError_t launch_attn_simt(int act, int kvf, const AttnArgs& a, int64_t rows, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int dpt = a.H * a.D / kAttnThreads;
#define CSA_ATTN_CASE(DPT_)                                                                 \
    if (dpt == DPT_) {                                                                      \
        if (act == CSA_F32 && kvf == CSA_F32) return launch_attn_t<DPT_, CSA_F32, CSA_F32>(a, rows, s);       \
        if (act == CSA_BF16 && kvf == CSA_BF16) return launch_attn_t<DPT_, CSA_BF16, CSA_BF16>(a, rows, s);   \
        if (act == CSA_BF16 && kvf == CSA_FP8_S64) return launch_attn_t<DPT_, CSA_BF16, CSA_FP8_S64>(a, rows, s); \
        if (act == CSA_F32 && kvf == CSA_FP8_S64) return launch_attn_t<DPT_, CSA_F32, CSA_FP8_S64>(a, rows, s); \
    }
    CSA_ATTN_CASE(2)
    CSA_ATTN_CASE(128)
#undef CSA_ATTN_CASE
    return cudaErrorInvalidValue;
}

bool attn_simt_supported(int act, int kvf, int H, int D) {
    if (H <= 0 || H > kAttnThreads || (kAttnThreads % H) != 0) return false;
    if ((H * D) % kAttnThreads) return false;
    const int dpt = H * D / kAttnThreads;
    if (dpt != 2 && dpt != 128) return false;
    return (act == CSA_F32 && (kvf == CSA_F32 || kvf == CSA_FP8_S64)) ||
           (act == CSA_BF16 && (kvf == CSA_BF16 || kvf == CSA_FP8_S64));
}

}  // namespace csa
