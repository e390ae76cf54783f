/*
 * oracle.cpp -- fp64 CPU oracle for exact masked softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plainly written reference
 * that the CUDA library is checked against.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or helper with the CUDA library: every formula below is
 * restated here from the source pages.
 *
 * Source pages (cited by title and section):
 *   [P2] "FlashAttention 能否加速滑动窗口注意力的 prefill" (m.xxqk.cn/news/265020)
 *        §2 (the attention formula), §3.2 (online-softmax recurrence),
 *        §4 / §4.1 (sliding window, causal variant), §5.1 (block skip test),
 *        §5.2 (boundary mask before softmax), §5.3 (skip + break + mask),
 *        §5.4 (block-pair counts), §5.5 (skipped block == all -inf block),
 *        §7.1 (window_size=(left, right), causal flag)
 *   [P1] "算子与编译器：FlashAttention 与长上下文" (charles2530.github.io)
 *        §4 (flash decoding: short query, long K/V, parallel over the KV axis)
 *
 * Readings where the pages are silent or garbled:
 *   R1  a window w is inclusive: |i - j| <= w is in band.
 *   R3  when Lq != Lk, query i sits at key position i + (Lk - Lq).
 *   R4  LSE is the natural-log log-sum-exp of the scaled scores of the row.
 *   R5  split-KV partials (o_s normalised, lse_s) merge by
 *       lse = logsumexp_s(lse_s),  o = sum_s exp(lse_s - lse) * o_s.
 *   R7  the tiled recurrence uses m_safe = 0 while the running max is -inf,
 *       otherwise a fully masked first block gives (-inf) - (-inf) = NaN.
 *   R13 the FP8 forward ("FlashAttention 深度解析" §4 names FlashAttention-3's
 *       FP8 path and gives no algorithm): Q, K, V are e4m3 codes with one fp32
 *       descale per (batch, head); scores are the dequantized products; each
 *       key tile's probabilities, taken against the running row max and
 *       multiplied by 2^8, are rounded to e4m3 before they weight V; the
 *       denominator sums the unrounded values.
 *
 * Element types of the inputs: 0 = float64, 1 = float32, 2 = bfloat16 (raw
 * 16-bit patterns).  Every input is widened exactly to double before use, so
 * the oracle sees the very values handed to the GPU.  All outputs are double.
 * A row with no allowed key gets O = 0 and LSE = -inf.
 */
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#include <algorithm>
#include <omp.h>

namespace {

const double NEG_INF = -std::numeric_limits<double>::infinity();

/* Widen one stored element to double. bfloat16 is the top half of a float32. */
inline double widen(const void* base, long long idx, int dtype) {
    if (dtype == 0) return static_cast<const double*>(base)[idx];
    if (dtype == 1) return static_cast<double>(static_cast<const float*>(base)[idx]);
    uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[idx]) << 16;
    float f;
    std::memcpy(&f, &bits, sizeof f);
    return static_cast<double>(f);
}

/* Copy `count` elements starting at `first` into a double buffer. */
void widen_block(const void* base, long long first, long long count, int dtype, double* out) {
    for (long long t = 0; t < count; ++t) out[t] = widen(base, first + t, dtype);
}

/*
 * The mask of [P2] §4 / §4.1 / §7.1 (window_size=(left, right); causal means
 * right = 0), with R1 (inclusive) and R3 (bottom-right alignment).  Negative
 * wl / wr mean "unbounded on that side".  len_k is the number of valid keys of
 * this batch element (keys at or beyond it never take part).
 */
inline bool allowed(long long i, long long j, long long Lq, long long Lk, long long len_k,
                    int causal, long long wl, long long wr) {
    const long long pos = i + (Lk - Lq);
    if (j < 0 || j >= len_k) return false;
    if (causal && j > pos) return false;
    if (wr >= 0 && j > pos + wr) return false;
    if (wl >= 0 && j < pos - wl) return false;
    return true;
}

/*
 * One row of exact attention by the definition of [P2] §2:
 *   s_j = scale * q_i . k_j  (allowed j only),  M = max_j s_j,
 *   Z = sum_j exp(s_j - M),  O_i = sum_j exp(s_j - M) v_j / Z,
 *   LSE_i = M + ln Z.
 * Kd / Vd are the widened [Lk, d] key and value matrices of the head.
 */
void attend_row(const double* qi, const double* Kd, const double* Vd, long long i,
                long long Lq, long long Lk, long long len_k, int d, double scale,
                int causal, long long wl, long long wr, double* s, double* o_row,
                double* lse_out) {
    double M = NEG_INF;
    for (long long j = 0; j < Lk; ++j) {
        if (!allowed(i, j, Lq, Lk, len_k, causal, wl, wr)) { s[j] = NEG_INF; continue; }
        const double* kj = Kd + j * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[j] = scale * dot;
        if (s[j] > M) M = s[j];
    }
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    if (M == NEG_INF) { *lse_out = NEG_INF; return; }
    double Z = 0.0;
    for (long long j = 0; j < Lk; ++j) {
        if (s[j] == NEG_INF) continue;
        const double w = std::exp(s[j] - M);
        Z += w;
        const double* vj = Vd + j * d;
        for (int c = 0; c < d; ++c) o_row[c] += w * vj[c];
    }
    for (int c = 0; c < d; ++c) o_row[c] /= Z;
    *lse_out = M + std::log(Z);
}

/*
 * The e4m3 format ("fn" variant: no infinities): sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits.  Exponent field 0 holds subnormals m * 2^-9;
 * exponent 15 with mantissa 7 is NaN; the largest finite value is
 * 1.75 * 2^8 = 448.
 */
double e4m3_value(uint8_t code) {
    const int e = (code >> 3) & 0xF, m = code & 7;
    if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
    const double mag = e == 0 ? std::ldexp(static_cast<double>(m), -9) : std::ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -mag : mag;
}

/* Round to the nearest e4m3 value, ties to the even code, magnitudes above
 * 448 clamped to 448 (saturating conversion); NaN gives 0x7F.  Plain search
 * over the 127 finite non-negative codes. */
uint8_t e4m3_round(double x) {
    if (std::isnan(x)) return 0x7F;
    static const std::vector<double> table = [] {
        std::vector<double> t(0x7F);
        for (int c = 0; c <= 0x7E; ++c) t[c] = e4m3_value(static_cast<uint8_t>(c));
        return t;
    }();
    const double a = std::fabs(x);
    int best = 0;
    double best_d = std::numeric_limits<double>::infinity();
    for (int c = 0; c <= 0x7E; ++c) {
        const double d = std::fabs(table[c] - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    if (a > 448.0) best = 0x7E;
    return static_cast<uint8_t>(best | (std::signbit(x) ? 0x80 : 0));
}

}  // namespace

extern "C" {

/* e4m3 codec (pinned against a library conversion in the tests). */
void oracle_e4m3_decode(const uint8_t* codes, long long n, double* out) {
    for (long long t = 0; t < n; ++t) out[t] = e4m3_value(codes[t]);
}

void oracle_e4m3_encode(const double* x, long long n, uint8_t* out) {
    for (long long t = 0; t < n; ++t) out[t] = e4m3_round(x[t]);
}

/*
 * Per-group FP8 quantization: for each of `groups` runs of `group_len`
 * elements, amax = max |x|, descale = amax / 448 and code = e4m3(x * (448 /
 * amax)), where the reciprocal scale and the product are each one fp32
 * operation rounded to nearest (the precision the kernel decides in); a group
 * of zeros gets descale 1.  x is widened from its stored type to fp32 first.
 */
void oracle_quantize_fp8(const void* x, int dtype, long long groups, long long group_len, uint8_t* codes,
                         float* descale) {
    for (long long g = 0; g < groups; ++g) {
        float amax = 0.0f;
        for (long long t = 0; t < group_len; ++t)
            amax = std::max(amax, std::fabs(static_cast<float>(widen(x, g * group_len + t, dtype))));
        const volatile float four48 = 448.0f;
        const float inv = amax > 0.0f ? four48 / amax : 1.0f;
        descale[g] = amax > 0.0f ? amax / four48 : 1.0f;
        for (long long t = 0; t < group_len; ++t) {
            const volatile float y = static_cast<float>(widen(x, g * group_len + t, dtype)) * inv;
            codes[g * group_len + t] = e4m3_round(static_cast<double>(y));
        }
    }
}

/*
 * FP8 forward by the steps of reading R13 on the tiled online softmax of
 * [P2] §3.2, one query row at a time over key tiles of block_k keys, with a
 * reference max m that moves only when a tile's max exceeds it by more than
 * `slack` (log2 units; 0 = the exact running max):
 *   x_j   = scale * qd * kd * (q8_i . k8_j) * log2(e)      (allowed keys)
 *   if max_j x_j > m + slack:  m' = max_j x_j;  alpha = 2^(m - m');  l, acc *= alpha
 *   p_j   = 2^(x_j - m' + 8 - slack) <= 2^8;   l += p_j
 *   acc  += e4m3(p_j) * v8_j    (p_j itself when quantize_p == 0)
 * and at the end O = vd * acc / l, LSE = ln2 * (m + log2 l - 8 + slack).
 * Numerator and denominator share the reference, so without the rounding of
 * p the result is exact attention for any slack.  q8, k8, v8 are e4m3 codes
 * [B,H,L,d]; qd, kd, vd the per-(b,h) descales.  A row with no allowed key
 * gets O = 0 and LSE = -inf.
 */
void oracle_attn_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* qd, const float* kd,
                     const float* vd, double* o, double* lse, int B, int H, int Lq, int Lk, int d, double scale,
                     int causal, int wl, int wr, int block_k, int quantize_p, double slack) {
    const double LOG2E = 1.4426950408889634074;
    for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
        std::vector<double> Kd(static_cast<size_t>(Lk) * d), Vd(static_cast<size_t>(Lk) * d);
        for (long long t = 0; t < static_cast<long long>(Lk) * d; ++t) {
            Kd[t] = e4m3_value(k8[bh * Lk * d + t]);
            Vd[t] = e4m3_value(v8[bh * Lk * d + t]);
        }
        const double c = scale * static_cast<double>(qd[bh]) * static_cast<double>(kd[bh]) * LOG2E;
#pragma omp parallel for schedule(dynamic, 16)
        for (int i = 0; i < Lq; ++i) {
            std::vector<double> qi(d), acc(d, 0.0), x(block_k);
            std::vector<char> ok(block_k);
            for (int e = 0; e < d; ++e) qi[e] = e4m3_value(q8[(bh * Lq + i) * d + e]);
            double m = NEG_INF, l = 0.0;
            for (long long k0 = 0; k0 < Lk; k0 += block_k) {
                const int n = static_cast<int>(std::min<long long>(block_k, Lk - k0));
                double mx = NEG_INF;
                for (int t = 0; t < n; ++t) {
                    ok[t] = allowed(i, k0 + t, Lq, Lk, Lk, causal, wl, wr);
                    if (!ok[t]) continue;
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qi[e] * Kd[(k0 + t) * d + e];
                    x[t] = c * dot;
                    mx = std::max(mx, x[t]);
                }
                if (mx == NEG_INF) continue;  /* no allowed key of this row in the tile */
                if (m == NEG_INF || mx > m + slack) {
                    const double alpha = m == NEG_INF ? 0.0 : std::exp2(m - mx);
                    l *= alpha;
                    for (int e = 0; e < d; ++e) acc[e] *= alpha;
                    m = mx;
                }
                for (int t = 0; t < n; ++t) {
                    if (!ok[t]) continue;
                    const double p = std::exp2(x[t] - m + 8.0 - slack);
                    l += p;
                    const double pq = quantize_p ? e4m3_value(e4m3_round(p)) : p;
                    for (int e = 0; e < d; ++e) acc[e] += pq * Vd[(k0 + t) * d + e];
                }
            }
            const long long row = bh * Lq + i;
            if (l == 0.0) {
                for (int e = 0; e < d; ++e) o[row * d + e] = 0.0;
                lse[row] = NEG_INF;
                continue;
            }
            for (int e = 0; e < d; ++e) o[row * d + e] = static_cast<double>(vd[bh]) * acc[e] / l;
            lse[row] = std::log(2.0) * (m + std::log2(l) - 8.0 + slack);
        }
    }
}

int oracle_num_threads(void) { return omp_get_max_threads(); }

void oracle_set_num_threads(int n) { if (n > 0) omp_set_num_threads(n); }

/*
 * Exact attention for every row.  q: [B,H,Lq,d], k/v: [B,H,Lk,d], o: [B,H,Lq,d]
 * (double), lse: [B,H,Lq] (double).  seqlens_k (nullable) gives the valid key
 * count of each batch element.
 */
void oracle_attn_naive(const void* q, const void* k, const void* v, int dtype,
                       double* o, double* lse, int B, int H, int Lq, int Lk, int d,
                       double scale, int causal, int wl, int wr, const int* seqlens_k) {
    std::vector<double> Kd(static_cast<size_t>(Lk) * d), Vd(static_cast<size_t>(Lk) * d);
    for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
        const long long b = bh / H;
        const long long len_k = seqlens_k ? std::min<long long>(seqlens_k[b], Lk) : Lk;
        widen_block(k, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Kd.data());
        widen_block(v, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Vd.data());
#pragma omp parallel
        {
            std::vector<double> s(Lk), qi(d);
#pragma omp for schedule(dynamic, 8)
            for (long long i = 0; i < Lq; ++i) {
                const long long row = bh * Lq + i;
                widen_block(q, row * d, d, dtype, qi.data());
                attend_row(qi.data(), Kd.data(), Vd.data(), i, Lq, Lk, len_k, d, scale,
                           causal, wl, wr, s.data(), o + row * d, lse + row);
            }
        }
    }
}

/*
 * Exact attention for a list of rows (used at sizes where every row would take
 * too long).  rows: nrows triples (b, h, i), sorted or not.  o: [nrows, d],
 * lse: [nrows].
 */
void oracle_attn_rows(const void* q, const void* k, const void* v, int dtype,
                      const int* rows, int nrows, double* o, double* lse,
                      int B, int H, int Lq, int Lk, int d, double scale,
                      int causal, int wl, int wr, const int* seqlens_k) {
    (void)B;
    std::vector<int> order(nrows);
    for (int r = 0; r < nrows; ++r) order[r] = r;
    auto head_of = [&](int r) { return static_cast<long long>(rows[3 * r]) * H + rows[3 * r + 1]; };
    std::stable_sort(order.begin(), order.end(), [&](int a, int b2) { return head_of(a) < head_of(b2); });
    std::vector<double> Kd(static_cast<size_t>(Lk) * d), Vd(static_cast<size_t>(Lk) * d);
    int start = 0;
    while (start < nrows) {
        const long long bh = head_of(order[start]);
        int stop = start;
        while (stop < nrows && head_of(order[stop]) == bh) ++stop;
        const long long b = bh / H;
        const long long len_k = seqlens_k ? std::min<long long>(seqlens_k[b], Lk) : Lk;
        widen_block(k, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Kd.data());
        widen_block(v, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Vd.data());
#pragma omp parallel
        {
            std::vector<double> s(Lk), qi(d);
#pragma omp for schedule(dynamic, 4)
            for (int t = start; t < stop; ++t) {
                const int r = order[t];
                const long long i = rows[3 * r + 2];
                widen_block(q, (bh * Lq + i) * d, d, dtype, qi.data());
                attend_row(qi.data(), Kd.data(), Vd.data(), i, Lq, Lk, len_k, d, scale,
                           causal, wl, wr, s.data(), o + static_cast<long long>(r) * d, lse + r);
            }
        }
        start = stop;
    }
}

/*
 * Softmax probabilities of one head, P: [Lq, Lk] (double), by the definition
 * (masked entries are 0; a row with no allowed key is all 0).  Used for the
 * row-sum check and for an independent P.V contraction in the tests.
 */
void oracle_attn_probs(const void* q, const void* k, int dtype, double* P,
                       int Lq, int Lk, int d, double scale, int causal, int wl, int wr) {
    std::vector<double> Kd(static_cast<size_t>(Lk) * d), qi(d), s(Lk);
    widen_block(k, 0, static_cast<long long>(Lk) * d, dtype, Kd.data());
    for (long long i = 0; i < Lq; ++i) {
        widen_block(q, i * d, d, dtype, qi.data());
        double M = NEG_INF;
        for (long long j = 0; j < Lk; ++j) {
            if (!allowed(i, j, Lq, Lk, Lk, causal, wl, wr)) { s[j] = NEG_INF; continue; }
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qi[c] * Kd[j * d + c];
            s[j] = scale * dot;
            if (s[j] > M) M = s[j];
        }
        double* Pi = P + i * Lk;
        if (M == NEG_INF) { for (long long j = 0; j < Lk; ++j) Pi[j] = 0.0; continue; }
        double Z = 0.0;
        for (long long j = 0; j < Lk; ++j) { Pi[j] = (s[j] == NEG_INF) ? 0.0 : std::exp(s[j] - M); Z += Pi[j]; }
        for (long long j = 0; j < Lk; ++j) Pi[j] /= Z;
    }
}

/*
 * The tiled online-softmax recurrence of [P2] §3.2 with the block skip,
 * early break and boundary mask of §5.1-§5.3, in fp64, for every head.
 *
 * For each Q block (block_q rows) the running state is m_i (row max, starts at
 * -inf), l_i (row sum, starts at 0) and acc (starts at 0).  For each KV block
 * (block_k keys) that is not skipped:
 *   s_ij  = scale * q_block . k_block^T, with -inf where the mask forbids
 *   m_new = max(m_i, rowmax(s_ij))
 *   p_ij  = exp(s_ij - m_new),  alpha = exp(m_i - m_new)
 *   l_i   = alpha * l_i + rowsum(p_ij)
 *   acc   = alpha * acc + p_ij . v_block
 *   m_i   = m_new
 * and finally O = acc / l_i.  With nan_guard != 0 the two exponentials use
 * m_safe = (m_new == -inf ? 0 : m_new) (reading R7); with nan_guard == 0 they
 * use m_new literally, as the page prints it.
 *
 * skip != 0 enables the block skip test of §5.1 (a KV block whose keys all lie
 * left of the band of every row of the Q block is skipped) and the early break
 * of §5.3 (once a KV block starts right of the band of every row, no later
 * block can intersect it).  With skip == 0 every block is visited and masked.
 *
 * lse = m_i + ln(l_i) (R4).  *visited receives the number of (Q block, KV
 * block) pairs that were processed.
 */
void oracle_attn_tiled(const void* q, const void* k, const void* v, int dtype,
                       double* o, double* lse, int B, int H, int Lq, int Lk, int d,
                       double scale, int causal, int wl, int wr, int block_q, int block_k,
                       int skip, int nan_guard, long long* visited) {
    const long long right = causal ? 0 : wr;          /* -1: unbounded */
    const long long shift = static_cast<long long>(Lk) - Lq;  /* R3 */
    long long total_visited = 0;
    std::vector<double> Kd(static_cast<size_t>(Lk) * d), Vd(static_cast<size_t>(Lk) * d);
    for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
        widen_block(k, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Kd.data());
        widen_block(v, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Vd.data());
        const int nqb = (Lq + block_q - 1) / block_q;
#pragma omp parallel reduction(+ : total_visited)
        {
            std::vector<double> q_block(static_cast<size_t>(block_q) * d), acc(static_cast<size_t>(block_q) * d);
            std::vector<double> m_i(block_q), l_i(block_q), s_ij(static_cast<size_t>(block_q) * block_k);
#pragma omp for schedule(dynamic, 1)
            for (int qb = 0; qb < nqb; ++qb) {
                const long long q_start = static_cast<long long>(qb) * block_q;
                const long long q_end = std::min<long long>(q_start + block_q, Lq);  /* exclusive */
                const int n_q = static_cast<int>(q_end - q_start);
                widen_block(q, (bh * Lq + q_start) * d, static_cast<long long>(n_q) * d, dtype, q_block.data());
                for (int r = 0; r < n_q; ++r) { m_i[r] = NEG_INF; l_i[r] = 0.0; }
                std::fill(acc.begin(), acc.end(), 0.0);
                for (long long k_start = 0; k_start < Lk; k_start += block_k) {
                    const long long k_end = std::min<long long>(k_start + block_k, Lk);  /* exclusive */
                    if (skip) {
                        /* §5.3 early break: first key right of the band of the last row. */
                        if (right >= 0 && k_start > (q_end - 1) + shift + right) break;
                        /* §5.1 skip: last key left of the band of the first row. */
                        if (wl >= 0 && (k_end - 1) < q_start + shift - wl) continue;
                    }
                    ++total_visited;
                    const int n_k = static_cast<int>(k_end - k_start);
                    /* s_ij with the boundary mask applied before the softmax (§5.2). */
                    for (int r = 0; r < n_q; ++r) {
                        for (int c = 0; c < n_k; ++c) {
                            const long long i = q_start + r, j = k_start + c;
                            double sv = NEG_INF;
                            if (allowed(i, j, Lq, Lk, Lk, causal, wl, wr)) {
                                double dot = 0.0;
                                for (int e = 0; e < d; ++e) dot += q_block[r * d + e] * Kd[j * d + e];
                                sv = scale * dot;
                            }
                            s_ij[static_cast<size_t>(r) * block_k + c] = sv;
                        }
                    }
                    for (int r = 0; r < n_q; ++r) {
                        double rowmax = NEG_INF;
                        for (int c = 0; c < n_k; ++c) rowmax = std::max(rowmax, s_ij[static_cast<size_t>(r) * block_k + c]);
                        const double m_new = std::max(m_i[r], rowmax);
                        const double m_ref = (nan_guard && m_new == NEG_INF) ? 0.0 : m_new;
                        const double alpha = std::exp(m_i[r] - m_ref);
                        double rowsum = 0.0;
                        double* acc_r = acc.data() + static_cast<size_t>(r) * d;
                        for (int e = 0; e < d; ++e) acc_r[e] *= alpha;
                        for (int c = 0; c < n_k; ++c) {
                            const double p = std::exp(s_ij[static_cast<size_t>(r) * block_k + c] - m_ref);
                            rowsum += p;
                            const double* vj = Vd.data() + (k_start + c) * d;
                            for (int e = 0; e < d; ++e) acc_r[e] += p * vj[e];
                        }
                        l_i[r] = alpha * l_i[r] + rowsum;
                        m_i[r] = m_new;
                    }
                }
                for (int r = 0; r < n_q; ++r) {
                    const long long row = bh * Lq + q_start + r;
                    double* o_row = o + row * d;
                    if (l_i[r] == 0.0 && nan_guard) {
                        for (int e = 0; e < d; ++e) o_row[e] = 0.0;
                        lse[row] = NEG_INF;
                        continue;
                    }
                    for (int e = 0; e < d; ++e) o_row[e] = acc[static_cast<size_t>(r) * d + e] / l_i[r];
                    lse[row] = m_i[r] + std::log(l_i[r]);
                }
            }
        }
    }
    if (visited) *visited = total_visited;
}

/*
 * Split-KV decode ([P1] §4 flash decoding) by partials and merge (reading R5).
 * q: [B,H,1,d], k/v: [B,H,Lk,d].  Split s covers keys
 * [s*chunk, min((s+1)*chunk, len_b)) with chunk = ceil(Lk / num_splits).
 * Each split computes the exact partial (o_s normalised, lse_s) by the
 * definition; the merge takes
 *   L = max_s lse_s,  w_s = exp(lse_s - L),  lse = L + ln sum_s w_s,
 *   o = sum_s w_s o_s / sum_s w_s,
 * where a split with no key has lse_s = -inf and weight 0.
 */
void oracle_decode_splitmerge(const void* q, const void* k, const void* v, int dtype,
                              double* o, double* lse, int B, int H, int Lk, int d,
                              double scale, const int* seqlens_k, int num_splits) {
    const long long chunk = (static_cast<long long>(Lk) + num_splits - 1) / num_splits;
#pragma omp parallel
    {
        std::vector<double> Kd(static_cast<size_t>(chunk) * d), Vd(static_cast<size_t>(chunk) * d);
        std::vector<double> qi(d), s(chunk), o_s(static_cast<size_t>(num_splits) * d), lse_s(num_splits);
#pragma omp for schedule(dynamic, 1)
        for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
            const long long b = bh / H;
            const long long len_k = seqlens_k ? std::min<long long>(seqlens_k[b], Lk) : Lk;
            widen_block(q, bh * d, d, dtype, qi.data());
            for (int sp = 0; sp < num_splits; ++sp) {
                const long long lo = sp * chunk;
                const long long hi = std::min<long long>(lo + chunk, len_k);
                const long long n = hi > lo ? hi - lo : 0;
                if (n > 0) {
                    widen_block(k, (bh * Lk + lo) * d, n * d, dtype, Kd.data());
                    widen_block(v, (bh * Lk + lo) * d, n * d, dtype, Vd.data());
                }
                /* the split's keys are a sequence of length n with no mask */
                attend_row(qi.data(), Kd.data(), Vd.data(), 0, 1, n, n, d, scale, 0, -1, -1,
                           s.data(), o_s.data() + static_cast<size_t>(sp) * d, &lse_s[sp]);
            }
            double L = NEG_INF;
            for (int sp = 0; sp < num_splits; ++sp) L = std::max(L, lse_s[sp]);
            double* o_row = o + bh * d;
            for (int e = 0; e < d; ++e) o_row[e] = 0.0;
            if (L == NEG_INF) { lse[bh] = NEG_INF; continue; }
            double W = 0.0;
            for (int sp = 0; sp < num_splits; ++sp) {
                if (lse_s[sp] == NEG_INF) continue;
                const double w = std::exp(lse_s[sp] - L);
                W += w;
                for (int e = 0; e < d; ++e) o_row[e] += w * o_s[static_cast<size_t>(sp) * d + e];
            }
            for (int e = 0; e < d; ++e) o_row[e] /= W;
            lse[bh] = L + std::log(W);
        }
    }
}

/*
 * Gradients of exact attention ([P2] §3.3: the backward pass recomputes the
 * scores instead of storing them).  With the loss L = sum_i dO_i . O_i, by the
 * chain rule through O_i = sum_j P_ij v_j and the row softmax P_ij:
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij  (= dO_i . O_i)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
 * All in fp64 from the widened inputs; P by the definition (masked entries 0,
 * rows without an allowed key contribute nothing).  do_ has q's layout.
 */
void oracle_attn_bwd(const void* q, const void* k, const void* v, const void* do_, int dtype,
                     double* dq, double* dk, double* dv, int B, int H, int Lq, int Lk, int d,
                     double scale, int causal, int wl, int wr) {
    std::vector<double> Qd(static_cast<size_t>(Lq) * d), Kd(static_cast<size_t>(Lk) * d),
        Vd(static_cast<size_t>(Lk) * d), Od(static_cast<size_t>(Lq) * d);
    std::vector<double> P(static_cast<size_t>(Lq) * Lk);
    for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
        widen_block(q, bh * Lq * d, static_cast<long long>(Lq) * d, dtype, Qd.data());
        widen_block(do_, bh * Lq * d, static_cast<long long>(Lq) * d, dtype, Od.data());
        widen_block(k, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Kd.data());
        widen_block(v, bh * Lk * d, static_cast<long long>(Lk) * d, dtype, Vd.data());
        double* dq_h = dq + bh * Lq * d;
        double* dk_h = dk + bh * Lk * d;
        double* dv_h = dv + bh * Lk * d;
        /* probabilities and the row gradients, row by row */
#pragma omp parallel for schedule(dynamic, 4)
        for (long long i = 0; i < Lq; ++i) {
            double* Pi = P.data() + i * Lk;
            double M = NEG_INF;
            for (long long j = 0; j < Lk; ++j) {
                if (!allowed(i, j, Lq, Lk, Lk, causal, wl, wr)) { Pi[j] = NEG_INF; continue; }
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += Qd[i * d + c] * Kd[j * d + c];
                Pi[j] = scale * dot;
                if (Pi[j] > M) M = Pi[j];
            }
            double Z = 0.0;
            for (long long j = 0; j < Lk; ++j) {
                Pi[j] = (M == NEG_INF || Pi[j] == NEG_INF) ? 0.0 : std::exp(Pi[j] - M);
                Z += Pi[j];
            }
            for (long long j = 0; j < Lk; ++j) Pi[j] = Z > 0.0 ? Pi[j] / Z : 0.0;
            /* D_i = sum_j P_ij dP_ij, then dQ_i = scale sum_j dS_ij k_j */
            double Di = 0.0;
            for (long long j = 0; j < Lk; ++j) {
                if (Pi[j] == 0.0) continue;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += Od[i * d + c] * Vd[j * d + c];
                Di += Pi[j] * dp;
            }
            for (int c = 0; c < d; ++c) dq_h[i * d + c] = 0.0;
            for (long long j = 0; j < Lk; ++j) {
                if (Pi[j] == 0.0) continue;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += Od[i * d + c] * Vd[j * d + c];
                const double ds = Pi[j] * (dp - Di);
                for (int c = 0; c < d; ++c) dq_h[i * d + c] += scale * ds * Kd[j * d + c];
            }
        }
        /* column gradients dK_j, dV_j need every row's D_i: recompute per column */
        std::vector<double> D(Lq);
#pragma omp parallel for schedule(dynamic, 4)
        for (long long i = 0; i < Lq; ++i) {
            const double* Pi = P.data() + i * Lk;
            double Di = 0.0;
            for (long long j = 0; j < Lk; ++j) {
                if (Pi[j] == 0.0) continue;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += Od[i * d + c] * Vd[j * d + c];
                Di += Pi[j] * dp;
            }
            D[i] = Di;
        }
#pragma omp parallel for schedule(dynamic, 4)
        for (long long j = 0; j < Lk; ++j) {
            for (int c = 0; c < d; ++c) { dk_h[j * d + c] = 0.0; dv_h[j * d + c] = 0.0; }
            for (long long i = 0; i < Lq; ++i) {
                const double Pij = P[i * Lk + j];
                if (Pij == 0.0) continue;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += Od[i * d + c] * Vd[j * d + c];
                const double ds = Pij * (dp - D[i]);
                for (int c = 0; c < d; ++c) {
                    dv_h[j * d + c] += Pij * Od[i * d + c];
                    dk_h[j * d + c] += scale * ds * Qd[i * d + c];
                }
            }
        }
    }
}

/*
 * Brute-force enumeration of the mask ([P2] §5.4 block-pair accounting): for
 * block_q x block_k tiles of the Lq x Lk score matrix (rows i < Lq only),
 *   pairs   = number of allowed (i, j),
 *   visited = tiles holding at least one allowed pair,
 *   total   = ceil(Lq/block_q) * ceil(Lk/block_k),
 *   partial = visited tiles that also hold a forbidden position (a column
 *             j >= Lk of a ragged last tile counts as forbidden).
 */
void oracle_count_blocks(int Lq, int Lk, int causal, int wl, int wr, int block_q, int block_k,
                         long long* pairs, long long* visited, long long* total, long long* partial) {
    const int nqb = (Lq + block_q - 1) / block_q;
    const int nkb = (Lk + block_k - 1) / block_k;
    long long n_pairs = 0, n_visited = 0, n_partial = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : n_pairs, n_visited, n_partial)
    for (int qb = 0; qb < nqb; ++qb) {
        const long long i0 = static_cast<long long>(qb) * block_q;
        const long long i1 = std::min<long long>(i0 + block_q, Lq);
        for (int kb = 0; kb < nkb; ++kb) {
            const long long j0 = static_cast<long long>(kb) * block_k;
            long long in_tile = 0;
            bool forbidden = false;
            for (long long i = i0; i < i1; ++i) {
                for (long long j = j0; j < j0 + block_k; ++j) {
                    if (allowed(i, j, Lq, Lk, Lk, causal, wl, wr)) ++in_tile;
                    else forbidden = true;
                }
            }
            n_pairs += in_tile;
            if (in_tile > 0) {
                ++n_visited;
                if (forbidden) ++n_partial;
            }
        }
    }
    if (pairs) *pairs = n_pairs;
    if (visited) *visited = n_visited;
    if (total) *total = static_cast<long long>(nqb) * nkb;
    if (partial) *partial = n_partial;
}

}  // extern "C"
