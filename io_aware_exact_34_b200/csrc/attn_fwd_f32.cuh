// attn_fwd_f32.cuh -- fp32 prefill forward on the CUDA cores.
//
// Same operation and the same block skipping as the bf16 kernel, in fp32
// end to end: tensor-core rounding (bf16 / tf32 inputs) cannot meet a 1e-5
// absolute bound, FMA arithmetic can.  The online-softmax update of the
// sliding-window FlashAttention prefill page (m.xxqk.cn/news/265020) §3.2 runs
// per query row, with the row max and row sum of each KV tile reduced by warp
// shuffles: each warp owns 8 query rows, lane l scores keys l and l + 32 of
// the 64-key tile and owns output columns l, l + 32, ...
#pragma once

#include <math_constants.h>

#include "sched.cuh"

namespace fattn {

template <int D>
struct F32Traits {
    static constexpr int BQ = 32;          // query rows per CTA
    static constexpr int BK = 64;          // keys per KV tile
    static constexpr int THREADS = 128;    // 4 warps x 8 rows
    static constexpr int KPAD = D + 1;     // padded K rows: conflict-free column reads
    static constexpr int NU = D / 32;      // output columns per lane
    static constexpr int SMEM_BYTES = (BQ * D + BK * KPAD + BK * D) * 4;
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int D>
__global__ void __launch_bounds__(128)
    attn_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                        float* __restrict__ o, float* __restrict__ lse, int Lq, int Lk, float scale, int causal,
                        int window_left, int window_right) {
    using T = F32Traits<D>;
    extern __shared__ float f32_smem[];
    float* sQ = f32_smem;
    float* sK = sQ + T::BQ * D;
    float* sV = sK + T::BK * T::KPAD;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long bh = blockIdx.y;
    const long long q0 = static_cast<long long>(blockIdx.x) * T::BQ;
    const long long q_last = (q0 + T::BQ - 1 < Lq - 1) ? q0 + T::BQ - 1 : Lq - 1;
    const Band band = make_band(Lq, Lk, causal, window_left, window_right);

    for (int idx = tid; idx < T::BQ * D; idx += T::THREADS) {
        const int r = idx / D, c = idx % D;
        sQ[idx] = (q0 + r < Lq) ? q[(bh * Lq + q0 + r) * D + c] : 0.f;
    }
    int lo, hi;
    kv_tile_range(band, q0, q_last, T::BK, &lo, &hi);

    float m_i[8], l_i[8], acc[8][T::NU];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        m_i[rr] = -CUDART_INF_F;
        l_i[rr] = 0.f;
#pragma unroll
        for (int u = 0; u < T::NU; ++u) acc[rr][u] = 0.f;
    }

    for (int j = lo; j < hi; ++j) {
        const long long k0 = static_cast<long long>(j) * T::BK;
        __syncthreads();
        for (int idx = tid; idx < T::BK * D; idx += T::THREADS) {
            const int r = idx / D, c = idx % D;
            const bool in = k0 + r < Lk;
            sK[r * T::KPAD + c] = in ? k[(bh * Lk + k0 + r) * D + c] : 0.f;
            sV[idx] = in ? v[(bh * Lk + k0 + r) * D + c] : 0.f;
        }
        __syncthreads();
#pragma unroll 1
        for (int rr = 0; rr < 8; ++rr) {
            const int r = warp * 8 + rr;
            const long long i = q0 + r;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) {
                const float qc = sQ[r * D + c];
                s0 = fmaf(qc, sK[lane * T::KPAD + c], s0);
                s1 = fmaf(qc, sK[(lane + 32) * T::KPAD + c], s1);
            }
            s0 *= scale;
            s1 *= scale;
            int lo_col, hi_col;
            row_col_bounds(band, i, k0, &lo_col, &hi_col);
            if (lane < lo_col || lane > hi_col) s0 = -CUDART_INF_F;
            if (lane + 32 < lo_col || lane + 32 > hi_col) s1 = -CUDART_INF_F;
            const float m_new = fmaxf(m_i[rr], warp_max(fmaxf(s0, s1)));
            const float m_safe = (m_new == -CUDART_INF_F) ? 0.f : m_new;
            const float alpha = expf(m_i[rr] - m_safe);
            const float p0 = expf(s0 - m_safe), p1 = expf(s1 - m_safe);
            l_i[rr] = alpha * l_i[rr] + warp_sum(p0 + p1);
#pragma unroll
            for (int u = 0; u < T::NU; ++u) acc[rr][u] *= alpha;
#pragma unroll
            for (int key = 0; key < T::BK; ++key) {
                const float pk = __shfl_sync(0xffffffffu, key < 32 ? p0 : p1, key & 31);
#pragma unroll
                for (int u = 0; u < T::NU; ++u) acc[rr][u] = fmaf(pk, sV[key * D + lane + 32 * u], acc[rr][u]);
            }
            m_i[rr] = m_new;
        }
    }

#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        const long long i = q0 + warp * 8 + rr;
        if (i >= Lq) continue;
        const float l = l_i[rr];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int u = 0; u < T::NU; ++u) o[(bh * Lq + i) * D + lane + 32 * u] = acc[rr][u] * inv;
        if (lse != nullptr && lane == 0) lse[bh * Lq + i] = l > 0.f ? m_i[rr] + logf(l) : -CUDART_INF_F;
    }
}

}  // namespace fattn
