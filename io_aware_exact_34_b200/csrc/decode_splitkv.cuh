// decode_splitkv.cuh -- split-KV decode (flash decoding) and the LSE merge.
//
// "算子与编译器：FlashAttention 与长上下文" §4 describes decode as one short
// query against a long K/V history, bound by reading that history, and flash
// decoding as parallelising along the KV axis.  Each CTA here takes one
// (split, head, batch) triple and streams its slice of K and V exactly once
// with 16-byte loads; the partial results combine by the same associativity
// that lets the online softmax of the sliding-window FlashAttention prefill
// page (m.xxqk.cn/news/265020) §3.2 fold tiles one after another: a partial
// (m_s, l_s, acc_s) is carried as its normalised output o_s = acc_s / l_s and
// its log-sum-exp lse_s, and
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s.
//
// Work layout (d = 128): a key row is 256 B = 16 lanes x 16 B, so a warp
// reads two keys per load instruction; 8 warps = 16 key groups per CTA; every
// lane keeps its 8-element slice of the running accumulator.  Scores and the
// running max are in log2 units (q is pre-multiplied by scale * log2(e)).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "dev_prims.cuh"

namespace fattn {

template <int D>
struct DecodeTraits {
    static constexpr int THREADS = 256;
    static constexpr int WARPS = THREADS / 32;
    static constexpr int LPK = D / 8;        // lanes per key row (16 B each)
    static constexpr int KPW = 32 / LPK;     // key rows per warp load step
    static constexpr int G = WARPS * KPW;    // key groups per CTA
    static constexpr int U = 4;              // key rows per group in flight
};

__device__ __forceinline__ void bf16x8_to_float(const uint4& r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// Where the key/value rows of one head live.  Contiguous caches: row
// (b*H + h)*Lk + key of [B, H, Lk, d].  Paged caches ("算子与编译器：
// FlashAttention 与长上下文" §5, paged KV): logical page key >> page_shift of
// sequence b is physical page block_table[b][...] of [num_pages, page_size,
// H, d], and the row is (page * page_size + key % page_size) * H + h.  A page
// index outside [0, num_pages) is clamped, so a bad table cannot address
// memory outside the cache.
struct KvLayout {
    const int* block_table;  // [B, max_pages] (paged only)
    int max_pages, page_shift, num_pages;
};

template <bool kPaged>
__device__ __forceinline__ long long kv_row(const KvLayout& lay, int b, int h, int H, int Lk, long long key) {
    if constexpr (kPaged) {
        int page = __ldg(lay.block_table + static_cast<long long>(b) * lay.max_pages + (key >> lay.page_shift));
        page = page < 0 ? 0 : (page >= lay.num_pages ? lay.num_pages - 1 : page);
        const long long tok = (static_cast<long long>(page) << lay.page_shift) | (key & ((1LL << lay.page_shift) - 1));
        return tok * H + h;
    } else {
        return (static_cast<long long>(b) * H + h) * Lk + key;
    }
}

// One (split s, head h, batch b) per CTA: partial output and LSE (log2 units).
template <int D, bool kPaged>
__global__ void __launch_bounds__(256)
    decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                        const __nv_bfloat16* __restrict__ v, const int* __restrict__ seqlens_k,
                        float* __restrict__ ws_o, float* __restrict__ ws_lse, int H, int Lk, int S,
                        int chunk, float c_log2, const KvLayout lay) {
    using T = DecodeTraits<D>;
    __shared__ float sm_m[T::G], sm_l[T::G];
    __shared__ float sm_acc[T::G][D];
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const long long bh = static_cast<long long>(b) * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = warp * T::KPW + lane / T::LPK;
    const int sub = lane % T::LPK;

    int len = Lk;
    if (seqlens_k != nullptr) {
        len = seqlens_k[b];
        len = len < 0 ? 0 : (len > Lk ? Lk : len);
    }
    const long long k_lo = static_cast<long long>(s) * chunk;
    long long k_hi = k_lo + chunk;
    if (k_hi > len) k_hi = len;

    float qf[8];
    bf16x8_to_float(*reinterpret_cast<const uint4*>(q + bh * D + sub * 8), qf);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[e] *= c_log2;

    float m = -CUDART_INF_F, l = 0.f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    const __nv_bfloat16* kb = k + sub * 8;
    const __nv_bfloat16* vb = v + sub * 8;
    // Rows of one step: keys base + g + u*G, u < U (zeros past the split's end).
    auto load_step = [&](long long base, uint4 (&kr)[T::U], uint4 (&vr)[T::U]) {
#pragma unroll
        for (int u = 0; u < T::U; ++u) {
            const long long key = base + g + u * T::G;
            if (key < k_hi) {
                const long long row = kv_row<kPaged>(lay, b, h, H, Lk, key);
                kr[u] = __ldcs(reinterpret_cast<const uint4*>(kb + row * D));
                vr[u] = __ldcs(reinterpret_cast<const uint4*>(vb + row * D));
            } else {
                kr[u] = make_uint4(0u, 0u, 0u, 0u);
                vr[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // Online-softmax update of this group's (m, l, acc) with one step of rows.
    auto consume_step = [&](long long base, const uint4 (&kr)[T::U], const uint4 (&vr)[T::U]) {
        float x[T::U];
#pragma unroll
        for (int u = 0; u < T::U; ++u) {
            float kf[8];
            bf16x8_to_float(kr[u], kf);
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) part = fmaf(qf[e], kf[e], part);
#pragma unroll
            for (int off = T::LPK / 2; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
            x[u] = (base + g + u * T::G < k_hi) ? part : -CUDART_INF_F;
        }
        float mloc = x[0];
#pragma unroll
        for (int u = 1; u < T::U; ++u) mloc = fmaxf(mloc, x[u]);
        const float m_new = fmaxf(m, mloc);
        const float m_safe = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        const float alpha = fast_exp2(m - m_safe);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
        for (int u = 0; u < T::U; ++u) {
            const float pu = fast_exp2(x[u] - m_safe);
            l += pu;
            float vf[8];
            bf16x8_to_float(vr[u], vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(pu, vf[e], acc[e]);
        }
        m = m_new;
    };
    constexpr long long STEP = T::G * T::U;
    if constexpr (kPaged) {
        // Paged rows: each row address waits on a block-table load; measured
        // on B200 this variant streams faster without the explicit pipeline.
        uint4 kA[T::U], vA[T::U];
        for (long long base = k_lo; base < k_hi; base += STEP) {
            load_step(base, kA, vA);
            consume_step(base, kA, vA);
        }
    } else {
        // Software pipeline: the next step's rows are in flight while this
        // step's are reduced (steps past the split's end load nothing, weigh 0).
        uint4 kA[T::U], vA[T::U], kB[T::U], vB[T::U];
        load_step(k_lo, kA, vA);
        for (long long base = k_lo; base < k_hi; base += 2 * STEP) {
            load_step(base + STEP, kB, vB);
            consume_step(base, kA, vA);
            load_step(base + 2 * STEP, kA, vA);
            consume_step(base + STEP, kB, vB);
        }
    }

    if (sub == 0) {
        sm_m[g] = m;
        sm_l[g] = l;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_acc[g][sub * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float M = -CUDART_INF_F;
#pragma unroll 4
        for (int gg = 0; gg < T::G; ++gg) M = fmaxf(M, sm_m[gg]);
        float* wo = ws_o + (bh * S + s) * D;
        if (M == -CUDART_INF_F) {
            wo[tid] = 0.f;
            if (tid == 0) ws_lse[bh * S + s] = -CUDART_INF_F;
        } else {
            float L = 0.f, od = 0.f;
#pragma unroll 4
            for (int gg = 0; gg < T::G; ++gg) {
                const float w = fast_exp2(sm_m[gg] - M);  // 0 for an empty group
                L = fmaf(w, sm_l[gg], L);
                od = fmaf(w, sm_acc[gg][tid], od);
            }
            wo[tid] = od / L;
            if (tid == 0) ws_lse[bh * S + s] = M + __log2f(L);
        }
    }
}

// One (batch, head) per CTA, D threads: merge the S partials.
template <int D>
__global__ void __launch_bounds__(D)
    decode_merge_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                        __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int S) {
    const long long bh = blockIdx.x;
    const int tid = threadIdx.x;
    const float* ls = ws_lse + bh * S;
    float M = -CUDART_INF_F;
    for (int s = 0; s < S; ++s) M = fmaxf(M, ls[s]);
    if (M == -CUDART_INF_F) {
        o[bh * D + tid] = __float2bfloat16_rn(0.f);
        if (tid == 0 && lse != nullptr) lse[bh] = -CUDART_INF_F;
        return;
    }
    float W = 0.f, acc = 0.f;
    for (int s = 0; s < S; ++s) {
        const float w = fast_exp2(ls[s] - M);
        W += w;
        acc = fmaf(w, ws_o[(bh * S + s) * D + tid], acc);
    }
    o[bh * D + tid] = __float2bfloat16_rn(acc / W);
    if (tid == 0 && lse != nullptr) lse[bh] = (M + __log2f(W)) * 0.6931471805599453f;
}

}  // namespace fattn
