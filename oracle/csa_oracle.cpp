// CPU oracle for the CSA / HCA hybrid attention of DeepSeek-V4.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
// CUDA library is checked against.  Only the tests, the smoke check and the
// benchmark's CPU-baseline leg load it; the library never does, and the two
// share no code (not even the number-format tables).
//
// What it computes, and where that comes from:
//   * CSA: every m tokens' KV are pooled into one entry by a softmax gate with
//     a learned positional bias; a "lightning indexer" scores the pooled
//     blocks with ReLU-scored multi-head dot products in FP4; each query keeps
//     its top-k blocks and attends to them plus a sliding window of recent raw
//     tokens.  ("DeepSeek-V4 發佈說明：為 AI Agents 提供高效的 1M-Token 上下文",
//     section 壓縮稀疏注意力 (CSA); "DeepSeek V4: Towards Highly Efficient
//     Million-Token Context Intelligence" wiki summary, section 架構创新, CSA
//     bullet: top-k sparse selection + MQA.)
//   * HCA: the same pooling at m' = 128 tokens per entry and dense attention
//     over all pooled entries plus the same window.  (Release note, section
//     重度壓縮注意力 (HCA); wiki summary, HCA bullet.)
//   * Sliding-window branch and an attention sink.  (Wiki summary, section
//     架构创新: the two kinds of layer alternate and are joined by a
//     sliding-window branch and an attention sink.)
//   * FP8 storage of KV entries and FP4 for the indexer QK path.  (Release
//     note, section 架構實現; wiki summary, section 基础设施, FP4 QAT bullet.)
//
// The pages print no formula.  The readings this library fixes (and which the
// oracle follows literally) are:
//   pooling   c_j[d] = sum_{r<m} softmax_r(z_{mj+r}[d] + B[r][d]) * x_{mj+r}[d]
//             (softmax over the m slots, separately per channel d)
//   indexer   s(t,j) = sum_h w[t][h] * ReLU(qI[t][h] . kI[j])
//   eligible  block j is visible to query t iff its last token m*j+m-1 < t-W,
//             so n_elig(t) = max(0, floor((t-W)/m))
//   top-k     the min(k, n_elig) highest fp32 scores, ties to the lower index
//   window    raw tokens i with t-W < i <= t (the query's own token included)
//   attention MQA: each pooled entry and each raw token is both key and value;
//             o = sum_e exp(l_e - M) v_e / (sum_e exp(l_e - M) + exp(sigma_h - M)),
//             l_e = scale * q_h . k_e, M = max(sigma_h, max_e l_e); the sink
//             logit sigma_h is not multiplied by the scale and has no value.
//   FP8       per 64 channels: scale = amax/448 (fp32, 1 if amax = 0),
//             code = RNE_E4M3(v/scale) saturated to +-448 (OCP OFP8 E4M3).
//   MXFP4     per 32 channels (OCP MX v1.0): X = floor(log2 amax) - 2,
//             E8M0 code X+127, element = RNE_E2M1(v / 2^X) saturated to +-6;
//             element 2i in the low nibble of byte i.
// Arithmetic is float64 throughout; pooled entries and indexer scores are
// rounded to fp32 once at the end, as the library stores them in fp32.
//
// Build: g++ -O2 -std=c++17 -shared -fPIC [-fopenmp] csa_oracle.cpp
// The optional OpenMP loop over independent query rows is only used to time
// the CPU baseline on all host cores; parity runs use one thread.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ------------------------------------------------------------------ formats
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8_S64 = 2, ORC_MXFP4 = 3, ORC_F64 = 4 };

// OCP OFP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
// S.1111.111 is NaN; exponent field 0 is subnormal (2^-6 * m/8).
double orc_e4m3_value(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
    if (e == 0) v = std::ldexp(m / 8.0, -6);
    else v = std::ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

// OCP MX E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent field 0
// is subnormal (m * 0.5).  Magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6.
double orc_e2m1_value(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

// OCP MX E8M0 scale: 2^(c-127); 255 is NaN.
double orc_e8m0_value(uint8_t c) {
    if (c == 255) return std::numeric_limits<double>::quiet_NaN();
    return std::ldexp(1.0, int(c) - 127);
}

// bfloat16: the upper 16 bits of an IEEE binary32.
double orc_bf16_value(uint16_t b) {
    uint32_t u = uint32_t(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// A read-only view of a stored [rows][d] tensor in one of the formats.
struct View {
    int fmt;
    const void* data;
    const void* scales;  // FP8_S64: float[rows][d/64]; MXFP4: uint8[rows][d/32]
    int d;
};

static double view_get(const View& t, int64_t row, int col) {
    switch (t.fmt) {
    case ORC_F32: return ((const float*)t.data)[row * t.d + col];
    case ORC_F64: return ((const double*)t.data)[row * t.d + col];
    case ORC_BF16: return orc_bf16_value(((const uint16_t*)t.data)[row * t.d + col]);
    case ORC_FP8_S64: {
        uint8_t c = ((const uint8_t*)t.data)[row * t.d + col];
        float s = ((const float*)t.scales)[row * (t.d / 64) + col / 64];
        return orc_e4m3_value(c) * double(s);
    }
    case ORC_MXFP4: {
        uint8_t b = ((const uint8_t*)t.data)[row * (t.d / 2) + col / 2];
        uint8_t c = (col & 1) ? (b >> 4) : (b & 15);
        uint8_t x = ((const uint8_t*)t.scales)[row * (t.d / 32) + col / 32];
        return orc_e2m1_value(c) * orc_e8m0_value(x);
    }
    }
    return std::numeric_limits<double>::quiet_NaN();
}

// Decode a whole stored tensor to float64 (used by the tests to look inside).
void orc_dequantize(int fmt, const void* data, const void* scales, int64_t rows, int d,
                    double* out) {
    View t{fmt, data, scales, d};
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < d; ++c) out[r * d + c] = view_get(t, r, c);
}

// --------------------------------------------------------------- quantisers
// Round-to-nearest-even of a real value onto the positive E4M3 grid, with
// saturation at the largest finite value 448 (code 0x7E).  Codes 0x00..0x7E
// are increasing in value, so the nearest code is found by bisection; a tie
// goes to the code whose mantissa LSB is 0.
static uint8_t e4m3_rne_positive(double a) {
    if (!(a > 0)) return 0;
    if (a >= 448.0) return 0x7E;
    int lo = 0, hi = 0x7E;  // value(lo) <= a < value(hi)
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (orc_e4m3_value(uint8_t(mid)) <= a) lo = mid; else hi = mid;
    }
    double dl = a - orc_e4m3_value(uint8_t(lo)), dh = orc_e4m3_value(uint8_t(hi)) - a;
    if (dl < dh) return uint8_t(lo);
    if (dh < dl) return uint8_t(hi);
    return (lo & 1) ? uint8_t(hi) : uint8_t(lo);
}

// Per-64-channel FP8 quantiser.  src is fp32 [rows][d]; codes uint8 [rows][d];
// scales fp32 [rows][d/64].  All decisions in fp32 as the stored scale is fp32:
// scale = fl(amax / 448), q = fl(v / scale).
void orc_quantize_fp8_s64(const float* src, int64_t rows, int d, uint8_t* codes, float* scales) {
    for (int64_t r = 0; r < rows; ++r) {
        for (int g = 0; g < d / 64; ++g) {
            const float* v = src + r * d + g * 64;
            float amax = 0.f;
            for (int i = 0; i < 64; ++i) amax = std::max(amax, std::fabs(v[i]));
            float scale = (amax > 0.f) ? amax / 448.0f : 1.0f;
            scales[r * (d / 64) + g] = scale;
            for (int i = 0; i < 64; ++i) {
                float q = v[i] / scale;
                uint8_t c = e4m3_rne_positive(std::fabs(double(q)));
                if (std::signbit(q)) c |= 0x80;
                codes[r * d + g * 64 + i] = c;
            }
        }
    }
}

// Round-to-nearest-even onto the positive E2M1 grid, saturating at 6.
static uint8_t e2m1_rne_positive(double a) {
    if (!(a > 0)) return 0;
    if (a >= 6.0) return 7;
    int lo = 0, hi = 7;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (orc_e2m1_value(uint8_t(mid)) <= a) lo = mid; else hi = mid;
    }
    double dl = a - orc_e2m1_value(uint8_t(lo)), dh = orc_e2m1_value(uint8_t(hi)) - a;
    if (dl < dh) return uint8_t(lo);
    if (dh < dl) return uint8_t(hi);
    return (lo & 1) ? uint8_t(hi) : uint8_t(lo);
}

// MXFP4 quantiser (OCP Microscaling Formats v1.0, conversion with a shared
// power-of-two scale per block of 32): X = floor(log2(amax)) - emax(E2M1=2).
// An all-zero block stores X = 0.  packed uint8 [rows][d/2]; e8m0 uint8 [rows][d/32].
void orc_quantize_mxfp4(const float* src, int64_t rows, int d, uint8_t* packed, uint8_t* e8m0) {
    for (int64_t r = 0; r < rows; ++r) {
        for (int g = 0; g < d / 32; ++g) {
            const float* v = src + r * d + g * 32;
            double amax = 0;
            for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(double(v[i])));
            int X = 0;
            if (amax > 0) {
                int e;
                std::frexp(amax, &e);  // amax = f * 2^e, f in [0.5, 1)
                X = (e - 1) - 2;       // floor(log2 amax) - 2
            }
            X = std::max(-127, std::min(127, X));
            e8m0[r * (d / 32) + g] = uint8_t(X + 127);
            for (int i = 0; i < 32; ++i) {
                double q = std::ldexp(double(v[i]), -X);
                uint8_t c = e2m1_rne_positive(std::fabs(q));
                if (std::signbit(v[i])) c |= 8;
                int col = g * 32 + i;
                uint8_t& b = packed[r * (d / 2) + col / 2];
                if (col & 1) b = uint8_t((b & 0x0F) | (c << 4));
                else b = uint8_t((b & 0xF0) | c);
            }
        }
    }
}

// ------------------------------------------------------------- a1: pooling
// Softmax-gated pooling with a learned positional bias (release note, CSA and
// HCA sections).  Blocks of m consecutive rows of x / z are pooled; n_tokens
// must be a multiple of m.  bias is [m][d] (row r = slot r in the block).
// out: fp32 [n_tokens/m][d].
void orc_compress(int x_fmt, const void* x, int z_fmt, const void* z, const float* bias,
                  int64_t n_tokens, int m, int d, float* out) {
    View X{x_fmt, x, nullptr, d}, Z{z_fmt, z, nullptr, d};
    int64_t nb = n_tokens / m;
    std::vector<double> g(m);
    for (int64_t j = 0; j < nb; ++j) {
        for (int c = 0; c < d; ++c) {
            double mx = -INFINITY;
            for (int r = 0; r < m; ++r) {
                g[r] = view_get(Z, j * m + r, c) + double(bias[r * d + c]);
                mx = std::max(mx, g[r]);
            }
            double den = 0;
            for (int r = 0; r < m; ++r) { g[r] = std::exp(g[r] - mx); den += g[r]; }
            double acc = 0;
            for (int r = 0; r < m; ++r) acc += (g[r] / den) * view_get(X, j * m + r, c);
            out[j * d + c] = float(acc);
        }
    }
}

// Round fp32 to bf16 bits, nearest-even (storage of bf16 pooled entries).
void orc_f32_to_bf16(const float* src, int64_t n, uint16_t* dst) {
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        std::memcpy(&u, &src[i], 4);
        uint32_t lsb = (u >> 16) & 1;
        dst[i] = uint16_t((u + 0x7FFF + lsb) >> 16);
    }
}

// ------------------------------------------------------ a2, a3: selection
static int64_t n_elig(int64_t t, int m, int W) {
    int64_t a = t - W;
    return a <= 0 ? 0 : a / m;
}

int64_t orc_n_elig(int64_t t, int m, int W) { return n_elig(t, m, W); }

// Lightning-indexer score of every eligible block for one query (release
// note, CSA: ReLU-scored multi-head dot products; wiki summary, 基础设施: the
// indexer's QK path is MXFP4).  qI: [HI][dI] rows of the view `qv` starting at
// row q_row; w: [HI]; keys: rows [0, n) of `kv`.  scores: fp32 [n].
static void indexer_row(const View& qv, int64_t q_row, const float* w, const View& kv,
                        int64_t n, int HI, int dI, float* scores) {
    std::vector<double> q(size_t(HI) * dI), k(dI);
    for (int h = 0; h < HI; ++h)
        for (int i = 0; i < dI; ++i) q[size_t(h) * dI + i] = view_get(qv, q_row + h, i);
    for (int64_t j = 0; j < n; ++j) {
        for (int i = 0; i < dI; ++i) k[i] = view_get(kv, j, i);
        double s = 0;
        for (int h = 0; h < HI; ++h) {
            double dot = 0;
            for (int i = 0; i < dI; ++i) dot += q[size_t(h) * dI + i] * k[i];
            s += double(w[h]) * std::max(0.0, dot);
        }
        scores[j] = float(s);
    }
}

// Scores for n_q queries of one sequence.  qI is [n_q*HI][dI] in q_fmt, w is
// [n_q][HI], kI is [n_keys][dI] in k_fmt.  Row q of `scores` (leading
// dimension ld) receives min(n_elig(q_pos[q]), n_keys) values; the rest is
// left alone.
void orc_indexer(int q_fmt, const void* qI, const void* qI_scales, const float* w,
                 int k_fmt, const void* kI, const void* kI_scales, int64_t n_keys,
                 const int64_t* q_pos,
                 int64_t n_q, int HI, int dI, int m, int W, float* scores, int64_t ld,
                 int n_threads) {
    View qv{q_fmt, qI, qI_scales, dI}, kv{k_fmt, kI, kI_scales, dI};
#pragma omp parallel for schedule(dynamic) num_threads(n_threads) if (n_threads > 1)
    for (int64_t q = 0; q < n_q; ++q)
        indexer_row(qv, q * HI, w + q * HI, kv, std::min(n_elig(q_pos[q], m, W), n_keys), HI, dI,
                    scores + q * ld);
}

// Top-k (wiki summary, CSA bullet: top-k sparse selection).  Returns the
// min(k, n) best indices by (fp32 score descending, index ascending), written
// in ascending index order, the rest of idx[0..k) set to -1.
static void topk_row(const float* s, int64_t n, int k, int32_t* idx) {
    std::vector<int64_t> order(n);
    for (int64_t j = 0; j < n; ++j) order[j] = j;
    std::stable_sort(order.begin(), order.end(),
                     [&](int64_t a, int64_t b) { return s[a] > s[b]; });
    int64_t take = std::min<int64_t>(k, n);
    std::vector<int64_t> sel(order.begin(), order.begin() + take);
    std::sort(sel.begin(), sel.end());
    for (int i = 0; i < k; ++i) idx[i] = i < take ? int32_t(sel[i]) : -1;
}

void orc_topk(const float* scores, int64_t ld, const int64_t* q_pos, int64_t rows, int k,
              int m, int W, int32_t* idx) {
    for (int64_t r = 0; r < rows; ++r)
        topk_row(scores + r * ld, std::min(n_elig(q_pos[r], m, W), ld), k, idx + r * k);
}

// --------------------------------------------------- a4, a5: attention
// One query, all heads.  q: rows [q_row, q_row+H) of `qv` ([H][d]).  The key
// and value of every attended item is the same vector (MQA, one KV head):
// pooled entries ent[0..n_ent) of `kv`, then raw rows [raw_lo, raw_hi) of
// `rv`.  sinks: [H] or null (no sink).  out: float64 [H][d].
static void attend_row(const View& qv, int64_t q_row, int H, int d, double scale,
                       const View& kv, const int64_t* ent, int64_t n_ent,
                       const View& rv, int64_t raw_lo, int64_t raw_hi,
                       const float* sinks, double* out) {
    const int64_t n = n_ent + std::max<int64_t>(0, raw_hi - raw_lo);
    // decode every attended item once: the key and the value of item e
    std::vector<double> item(size_t(n) * d);
    for (int64_t e = 0; e < n; ++e)
        for (int c = 0; c < d; ++c)
            item[size_t(e) * d + c] = e < n_ent ? view_get(kv, ent[e], c)
                                                : view_get(rv, raw_lo + (e - n_ent), c);
    std::vector<double> logit(n), qh(d);
    for (int h = 0; h < H; ++h) {
        for (int c = 0; c < d; ++c) qh[c] = view_get(qv, q_row + h, c);
        for (int64_t e = 0; e < n; ++e) {
            double dot = 0;
            for (int c = 0; c < d; ++c) dot += qh[c] * item[size_t(e) * d + c];
            logit[e] = scale * dot;
        }
        double M = sinks ? double(sinks[h]) : -INFINITY;
        for (int64_t e = 0; e < n; ++e) M = std::max(M, logit[e]);
        double den = sinks ? std::exp(double(sinks[h]) - M) : 0.0;
        double* o = out + int64_t(h) * d;
        for (int c = 0; c < d; ++c) o[c] = 0;
        if (n == 0 || M == -INFINITY) continue;  // nothing to attend: output 0
        for (int64_t e = 0; e < n; ++e) {
            double p = std::exp(logit[e] - M);
            den += p;
            for (int c = 0; c < d; ++c) o[c] += p * item[size_t(e) * d + c];
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
    }
}

// Attention for n_q queries of one sequence.
//   q:     [n_q*H][d] in q_fmt
//   kv:    pooled entries [n_kv][d] in kv_fmt (+ scales)
//   sel:   CSA: [n_q][k] selected entry ids (-1 = none); HCA: null, and every
//          eligible entry j < min(n_elig(t), n_kv) is attended
//   raw:   raw tokens [n_raw][d] in raw_fmt; raw row r holds position raw_pos0 + r
//   out:   float64 [n_q][H][d]
void orc_attention(int q_fmt, const void* q, int kv_fmt, const void* kv, const void* kv_scales,
                   int64_t n_kv, const int32_t* sel, int k, int raw_fmt, const void* raw, int64_t raw_pos0,
                   int64_t n_raw, const float* sinks, const int64_t* q_pos, int64_t n_q,
                   int H, int d, int m, int W, double scale, double* out, int n_threads) {
    View qv{q_fmt, q, nullptr, d}, kvv{kv_fmt, kv, kv_scales, d}, rv{raw_fmt, raw, nullptr, d};
#pragma omp parallel for schedule(dynamic) num_threads(n_threads) if (n_threads > 1)
    for (int64_t i = 0; i < n_q; ++i) {
        int64_t t = q_pos[i];
        std::vector<int64_t> ent;
        if (sel) {
            for (int a = 0; a < k; ++a) if (sel[i * k + a] >= 0) ent.push_back(sel[i * k + a]);
        } else {
            int64_t ne = std::min(n_elig(t, m, W), n_kv);
            for (int64_t j = 0; j < ne; ++j) ent.push_back(j);
        }
        // window: t-W < pos <= t, clipped to the raw rows supplied
        int64_t lo = std::max<int64_t>(t - W + 1, 0) - raw_pos0;
        int64_t hi = t + 1 - raw_pos0;
        lo = std::max<int64_t>(lo, 0);
        hi = std::min<int64_t>(hi, n_raw);
        attend_row(qv, i * H, H, d, scale, kvv, ent.data(), int64_t(ent.size()), rv, lo,
                   std::max(lo, hi), sinks, out + i * int64_t(H) * d);
    }
}

// ------------------------------------------------------ whole CSA step
// Indexer -> top-k -> attention for n_q queries of one sequence (the CSA
// layer's read path).  sel_out: [n_q][k]; out: float64 [n_q][H][d].
void orc_csa(int q_fmt, const void* q, int kv_fmt, const void* kv, const void* kv_scales,
             int idx_fmt, const void* qI, const void* qI_scales, const float* w,
             const void* kI, const void* kI_scales, int64_t n_blocks,
             int raw_fmt, const void* raw, int64_t raw_pos0, int64_t n_raw,
             const float* sinks, const int64_t* q_pos, int64_t n_q,
             int H, int d, int HI, int dI, int m, int W, int k, double scale,
             int32_t* sel_out, double* out, int n_threads) {
    View qv{q_fmt, q, nullptr, d}, kvv{kv_fmt, kv, kv_scales, d}, rv{raw_fmt, raw, nullptr, d};
    View qiv{idx_fmt, qI, qI_scales, dI}, kiv{idx_fmt, kI, kI_scales, dI};
#pragma omp parallel for schedule(dynamic) num_threads(n_threads) if (n_threads > 1)
    for (int64_t i = 0; i < n_q; ++i) {
        int64_t t = q_pos[i];
        int64_t ne = std::min<int64_t>(n_elig(t, m, W), n_blocks);
        std::vector<float> s(ne);
        indexer_row(qiv, i * HI, w + i * HI, kiv, ne, HI, dI, s.data());
        int32_t* sel = sel_out + i * k;
        topk_row(s.data(), ne, k, sel);
        std::vector<int64_t> ent;
        for (int a = 0; a < k; ++a) if (sel[a] >= 0) ent.push_back(sel[a]);
        int64_t lo = std::max<int64_t>(std::max<int64_t>(t - W + 1, 0) - raw_pos0, 0);
        int64_t hi = std::min<int64_t>(t + 1 - raw_pos0, n_raw);
        attend_row(qv, i * H, H, d, scale, kvv, ent.data(), int64_t(ent.size()), rv, lo,
                   std::max(lo, hi), sinks, out + i * int64_t(H) * d);
    }
}

int orc_max_threads() {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

}  // extern "C"
