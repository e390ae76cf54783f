// attn_bwd_sm100.cuh -- bf16 attention backward with recomputation on the
// 5th-generation tensor cores.
//
// The forward keeps only O and the row log-sum-exp LSE; the backward rebuilds
// every score tile from Q and K instead of reading a stored S (the
// recomputation of the sliding-window FlashAttention prefill page
// (m.xxqk.cn/news/265020) §3.3 and of the bomianfm.com FlashAttention answer,
// "recomputation" bullet).  With s_ij = q_i . k_j and the saved LSE_i,
//
//   P_ij  = exp(scale s_ij - LSE_i)            (the forward's probabilities)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j
//   D_i   = sum_j P_ij dP_ij = dO_i . O_i
//   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
//
// which is the chain rule through O = softmax(scale Q K^T) V; the oracle's
// gradient is that definition written out in fp64.  Masked pairs have
// P_ij = 0 and contribute nothing; tile pairs with no allowed element are
// skipped exactly as in the forward (§5.1, §5.3).
//
// Three launches:
//   bwd_prep_kernel     D_i = dO_i . O_i, LSE in log2 units, dQ accumulator = 0
//   attn_bwd_sm100      one CTA per (batch*head, 128-key tile): dK_j, dV_j in
//                       tensor memory across the Q tiles of the band, dQ
//                       partials added to an fp32 accumulator in device memory
//   bwd_dq_kernel       dQ = scale * accumulator, rounded to bf16
//
// Main kernel, 512 threads:
//   warp 0       TMA producer: K_j and V_j once, then a 2-stage ring of
//                (Q_i, LSE_i, D_i) and dO_i, each half with its own barriers
//   warp 1       MMA issuer (one thread)
//   warps 4-11   two warpgroups, thread = key row; warpgroup h owns the query
//                columns [64h, 64h+64) of every score tile: P, dS
//   warps 12-15  dQ drain, thread = query row: the dQ tile leaves tensor
//                memory in two halves of D/2 columns, each staged in the dO
//                buffer of its stage (free once dV has read dO; 128 x D/2
//                fp32 is exactly its size) and TMA reduce-added into the fp32
//                accumulator in whole lines; the Q buffer is never used for
//                it, so the next Q tile loads as soon as dK has read the last
//
// Tensor memory (512 columns), lane = key row unless noted:
//   [0,128)        S^T = K_j Q_i^T (fp32), then P^T (bf16 pairs) over it
//   [128,256)      dP^T = V_j dO_i^T (fp32), then dS^T (bf16 pairs) over it,
//                  then dQ_i = dS K_j (fp32, lane = query row)
//   [256,256+D)    dV_j accumulator
//   [256+D,256+2D) dK_j accumulator
// Each warpgroup writes its bf16 P / dS into the first 32 columns of its own
// 64-column half, so no column is overwritten before its owner has read it.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "dev_prims.cuh"
#include "sched.cuh"

namespace fattn {

// Bytes of per-head working set (Q and dO in bf16, the fp32 dQ accumulator)
// that the CTAs running at one time should share: heads are scheduled in
// groups that fit it, so their re-read tiles and accumulator lines stay in L2.
#ifndef FATTN_BWD_GROUP_BYTES
#define FATTN_BWD_GROUP_BYTES (16ull << 20)
#endif

// TMA reduce-add of a 2-D fp32 box from this CTA's shared memory into global
// memory (whole-line reductions at L2), tracked in the issuing thread's bulk group.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Until every committed bulk operation of this thread has read its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Until every committed bulk operation of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int D>
struct BwdTraits {
    static constexpr int BQ = 128;                 // queries per Q tile
    static constexpr int BK = 128;                 // keys per CTA
    static constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle column)
    static constexpr int NCHUNK = D / 64;
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int NSTAGE = 2;
    static constexpr int SMEM_K_OFF = 0;
    static constexpr int SMEM_V_OFF = TILE_BYTES;
    static constexpr int SMEM_STAGE_OFF = 2 * TILE_BYTES;  // stage s: Q at +0, dO at +TILE_BYTES
    static constexpr int SMEM_DS_OFF = SMEM_STAGE_OFF + NSTAGE * 2 * TILE_BYTES;
    static constexpr int DS_BYTES = 128 * 128 * 2;  // dS as [key][query], two 64-query swizzle columns
    static constexpr int SMEM_VEC_OFF = SMEM_DS_OFF + DS_BYTES;  // stage s: LSE2 at +0, D at +512
    static constexpr int VEC_STAGE_BYTES = 1024;
    static constexpr int SMEM_BAR_OFF = SMEM_VEC_OFF + NSTAGE * VEC_STAGE_BYTES;
    static constexpr int NBAR = 1 + 4 * NSTAGE + 10;
    static constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NBAR * 8;
    static constexpr int SMEM_USED = SMEM_MISC_OFF + 16;
    // Alignment slack for the 1024-byte aligned base; the kernel checks at run
    // time that the slack it needs fits and otherwise reports an error.
    static constexpr int SMEM_BYTES = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 512;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(SMEM_USED <= 232448, "shared memory");
    // half a dQ tile (128 x D/2 fp32) is staged in a dO buffer (128 x D bf16)
    static_assert(128 * (D / 2) * 4 == TILE_BYTES, "dQ staging");
};

struct BwdParams {
    const float* lse2;   // [BH, Lq_pad]: LSE * log2(e), +inf for rows without keys or past Lq
    const float* dsum;   // [BH, Lq_pad]: D_i = dO_i . O_i, 0 past Lq
    float* dq_acc;       // [BH, Lq_pad, D] fp32, zeroed by bwd_prep_kernel
    void* dk;            // [BH, Lk, D] bf16
    void* dv;            // [BH, Lk, D] bf16
    unsigned long long* visited;  // optional: Q tiles visited, summed over CTAs
    int BH, Lq, Lk, Lq_pad, n_kv;
    float scale, scale_log2;
    int causal, window_left, window_right;
    int reverse;         // 1: launch order takes the last KV tile first
    int group;           // heads per scheduling group
};

// ---------------------------------------------------------------- prep
// One group of D/8 threads per (bh, query row) of the padded range: D_i from
// 16-byte loads of dO and O, LSE in log2 units, and the row of the dQ
// accumulator set to zero.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ dsum, float* __restrict__ dq_acc, int BH,
                                                       int Lq, int Lq_pad) {
    constexpr int G = D / 8;  // threads per row
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = gid / G;  // over BH * Lq_pad
    const int part = static_cast<int>(gid % G);
    if (row >= static_cast<long long>(BH) * Lq_pad) return;
    const long long bh = row / Lq_pad;
    const int i = static_cast<int>(row % Lq_pad);
    float acc = 0.f;
    if (i < Lq) {
        const long long off = (bh * Lq + i) * D + part * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(o + off);
        const uint4 b = *reinterpret_cast<const uint4*>(dout + off);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc += __uint_as_float(aw[e] << 16) * __uint_as_float(bw[e] << 16);
            acc += __uint_as_float(aw[e] & 0xFFFF0000u) * __uint_as_float(bw[e] & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int w = G / 2; w > 0; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w, G);
    if (part == 0) {
        float l2 = CUDART_INF_F;
        if (i < Lq) {
            const float l = lse[bh * Lq + i];
            if (l > -CUDART_INF_F) l2 = l * 1.4426950408889634f;
        }
        lse2[row] = l2;
        dsum[row] = i < Lq ? acc : 0.f;
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D) + part * 2;
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------- dQ
// dQ = scale * accumulator -> bf16, eight elements per thread.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq,
                                                     int BH, int Lq, int Lq_pad, float scale) {
    constexpr int G = D / 8;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = gid / G;  // over BH * Lq
    const int part = static_cast<int>(gid % G);
    if (row >= static_cast<long long>(BH) * Lq) return;
    const long long bh = row / Lq;
    const int i = static_cast<int>(row % Lq);
    const float4* src = reinterpret_cast<const float4*>(dq_acc + (bh * Lq_pad + i) * D) + part * 2;
    const float4 a = src[0], b = src[1];
    uint4 r;
    r.x = pack_bf16x2(a.x * scale, a.y * scale);
    r.y = pack_bf16x2(a.z * scale, a.w * scale);
    r.z = pack_bf16x2(b.x * scale, b.y * scale);
    r.w = pack_bf16x2(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4*>(dq + row * D + part * 8) = r;
}

// ---------------------------------------------------------------- main kernel
// Which (bh, KV tile) this CTA owns.  KV tile j runs over the Q tiles
// [q_lo, q_hi) of the band.  Heads go in groups of p.group; inside a group the
// launch takes KV tiles in the order that puts the longest Q ranges first
// (reverse = 1 walks j downwards), all heads of the group for each j.
struct BwdTile {
    int bh, j, q_lo, q_hi;
    long long k0, k_last;
};

__device__ __forceinline__ BwdTile bwd_tile(const BwdParams& p, const Band& band) {
    BwdTile t;
    const int per_group = p.group * p.n_kv;
    const int g = blockIdx.x / per_group;
    const int r = blockIdx.x - g * per_group;
    const int gsize = p.BH - g * p.group < p.group ? p.BH - g * p.group : p.group;
    const int jj = r / gsize;
    t.bh = g * p.group + (r - jj * gsize);
    t.j = p.reverse ? p.n_kv - 1 - jj : jj;
    t.k0 = static_cast<long long>(t.j) * 128;
    t.k_last = t.k0 + 127 < p.Lk - 1 ? t.k0 + 127 : p.Lk - 1;
    q_tile_range(band, t.k0, t.k_last, 128, &t.q_lo, &t.q_hi);
    return t;
}

template <int D>
__global__ void __launch_bounds__(512, 1)
    attn_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using T = BwdTraits<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    int* status = &g_fattn_status;
    if (base - raw + T::SMEM_USED > T::SMEM_BYTES) {
        // the dynamic shared memory window is not aligned well enough for the
        // layout: report it instead of touching memory past the window
        if (threadIdx.x == 0) atomicExch(status, -2);
        return;
    }
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sK = base + T::SMEM_K_OFF;
    const uint32_t sV = base + T::SMEM_V_OFF;
    const uint32_t sStage = base + T::SMEM_STAGE_OFF;
    const uint32_t sDS = base + T::SMEM_DS_OFF;
    const uint32_t sVec = base + T::SMEM_VEC_OFF;
    const uint32_t bar0 = base + T::SMEM_BAR_OFF;
    const uint32_t kv_full = bar0;
    const uint32_t q_full0 = bar0 + 8;                   // Q + LSE2 + D of a stage landed
    const uint32_t do_full0 = q_full0 + 8 * T::NSTAGE;   // dO of a stage landed
    const uint32_t q_empty0 = do_full0 + 8 * T::NSTAGE;  // Q half of a stage free
    const uint32_t do_empty0 = q_empty0 + 8 * T::NSTAGE; // dO half of a stage free
    const uint32_t s_full = do_empty0 + 8 * T::NSTAGE;
    const uint32_t dp_full = s_full + 8;
    const uint32_t p_ready = dp_full + 8;
    const uint32_t ds_ready = p_ready + 8;
    const uint32_t dq_full = ds_ready + 8;
    const uint32_t dq_empty = dq_full + 8;
    const uint32_t dkdv_full = dq_empty + 8;
    const uint32_t drain_bar = dkdv_full + 8;
    const uint32_t dq_staged = drain_bar + 8;
    const uint32_t stage_reuse = dq_staged + 8;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + T::SMEM_MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + T::SMEM_MISC_OFF + 4);

    const Band band = make_band(p.Lq, p.Lk, p.causal, p.window_left, p.window_right);
    const BwdTile tile = bwd_tile(p, band);
    const int n_tiles = tile.q_hi - tile.q_lo;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < T::NSTAGE; ++s) {
            mbar_init(q_full0 + 8 * s, 1);
            mbar_init(do_full0 + 8 * s, 1);
            mbar_init(q_empty0 + 8 * s, 1);   // the MMA warp's commit after dK
            mbar_init(do_empty0 + 8 * s, 2);  // the MMA warp's commit after dV and the dQ drain's release
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 256);
        mbar_init(ds_ready, 256);
        mbar_init(dq_full, 1);
        mbar_init(dq_empty, 128);
        mbar_init(dkdv_full, 1);
        mbar_init(drain_bar, 1);
        mbar_init(dq_staged, 128);
        mbar_init(stage_reuse, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_do);
        tma_prefetch_map(&tm_dq);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), T::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_tiles > 0) {
            mbar_arrive_expect_tx(kv_full, 2 * T::TILE_BYTES);
            for (int c = 0; c < T::NCHUNK; ++c) {
                tma_load_3d(sK + c * T::CHUNK_BYTES, &tm_k, kv_full, c * 64, static_cast<int>(tile.k0), tile.bh);
                tma_load_3d(sV + c * T::CHUNK_BYTES, &tm_v, kv_full, c * 64, static_cast<int>(tile.k0), tile.bh);
            }
            bool ok = true;
            int issued = 0, issued_do = 0;
            for (int n = 0; n < n_tiles && ok; ++n) {
                const int s = n & 1;
                const uint32_t use = static_cast<uint32_t>(n >> 1);
                const int q0 = (tile.q_lo + n) * 128;
                const uint32_t st = sStage + s * 2 * T::TILE_BYTES;
                if (use > 0) {
                    ok = mbar_wait(q_empty0 + 8 * s, (use - 1) & 1u, abort_flag, status, -6);
                    if (!ok) break;
                }
                const uint32_t qfb = q_full0 + 8 * s;
                mbar_arrive_expect_tx(qfb, T::TILE_BYTES + T::VEC_STAGE_BYTES);
                for (int c = 0; c < T::NCHUNK; ++c)
                    tma_load_3d(st + c * T::CHUNK_BYTES, &tm_q, qfb, c * 64, q0, tile.bh);
                const long long voff = static_cast<long long>(tile.bh) * p.Lq_pad + q0;
                bulk_load(sVec + s * T::VEC_STAGE_BYTES, p.lse2 + voff, 512, qfb);
                bulk_load(sVec + s * T::VEC_STAGE_BYTES + 512, p.dsum + voff, 512, qfb);
                ++issued;
                if (use > 0) {
                    ok = mbar_wait(do_empty0 + 8 * s, (use - 1) & 1u, abort_flag, status, -6);
                    if (!ok) break;
                }
                const uint32_t dfb = do_full0 + 8 * s;
                mbar_arrive_expect_tx(dfb, T::TILE_BYTES);
                for (int c = 0; c < T::NCHUNK; ++c)
                    tma_load_3d(st + T::TILE_BYTES + c * T::CHUNK_BYTES, &tm_do, dfb, c * 64, q0, tile.bh);
                ++issued_do;
            }
            // No copy may still be landing in shared memory when the CTA exits.
            mbar_wait(kv_full, 0, nullptr, status, -6);
            for (int s = 0; s < T::NSTAGE; ++s) {
                if (issued > s) {
                    const uint32_t uses = static_cast<uint32_t>((issued - 1 - s) / T::NSTAGE + 1);
                    mbar_wait(q_full0 + 8 * s, (uses - 1) & 1u, nullptr, status, -6);
                }
                if (issued_do > s) {
                    const uint32_t uses = static_cast<uint32_t>((issued_do - 1 - s) / T::NSTAGE + 1);
                    mbar_wait(do_full0 + 8 * s, (uses - 1) & 1u, nullptr, status, -6);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);  // K-major A and B
            constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, 0, 1);    // A in TMEM, B MN-major
            constexpr uint32_t idesc_q = idesc_bf16_f32(128, D, 1, 1);    // A and B MN-major
            bool ok = mbar_wait(kv_full, 0, abort_flag, status, -6);
            // S^T = K Q^T into [0,128): A = K (key rows), B = Q (query rows), both K-major over d
            auto issue_s = [&](int n) {
                const int s = n & 1;
                const uint32_t q_lo = sdesc_lo(sStage + s * 2 * T::TILE_BYTES, 16);
                const uint32_t k_lo = sdesc_lo(sK, 16);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = ((ks / 4) * T::CHUNK_BYTES + (ks % 4) * 32) >> 4;
                    mma_bf16_ss(tmem + T::TM_S, sdesc_from_lo(k_lo + off), sdesc_from_lo(q_lo + off), idesc_s,
                                ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
            };
            if (ok) ok = mbar_wait(q_full0, 0, abort_flag, status, -6);
            if (ok) {
                tc_fence_after_sync();
                issue_s(0);
            }
            for (int n = 0; n < n_tiles && ok; ++n) {
                const int s = n & 1;
                const uint32_t q_st = sStage + s * 2 * T::TILE_BYTES;
                const uint32_t do_st = q_st + T::TILE_BYTES;
                // dP^T = V dO^T into [128,256), once the previous dQ has left it
                if (n > 0) {
                    ok = mbar_wait(dq_empty, (n - 1) & 1u, abort_flag, status, -6);
                    if (!ok) break;
                    tc_fence_after_sync();
                }
                ok = mbar_wait(do_full0 + 8 * s, static_cast<uint32_t>(n >> 1) & 1u, abort_flag, status, -6);
                if (!ok) break;
                tc_fence_after_sync();
                {
                    const uint32_t d_lo = sdesc_lo(do_st, 16);
                    const uint32_t v_lo = sdesc_lo(sV, 16);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = ((ks / 4) * T::CHUNK_BYTES + (ks % 4) * 32) >> 4;
                        mma_bf16_ss(tmem + T::TM_DP, sdesc_from_lo(v_lo + off), sdesc_from_lo(d_lo + off), idesc_s,
                                    ks > 0 ? 1u : 0u);
                    }
                    mma_commit(dp_full);
                }
                // dV += P^T dO: A = P^T from TMEM (bf16 pairs of each half), B = dO MN-major
                ok = mbar_wait(p_ready, n & 1u, abort_flag, status, -6);
                if (!ok) break;
                tc_fence_after_sync();
                {
                    const uint32_t b_lo = sdesc_lo(do_st, T::CHUNK_BYTES);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t a_col = (ks < 4 ? 0u : 64u) + (ks & 3) * 8u;
                        mma_bf16_ts(tmem + T::TM_DV, tmem + T::TM_S + a_col, sdesc_from_lo(b_lo + ks * (2048 >> 4)),
                                    idesc_g, (n > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(do_empty0 + 8 * s);  // dV(n) was the last product to read dO(n)
                // the next tile's scores go in now that P^T has been issued to its consumer
                if (n + 1 < n_tiles) {
                    const int s1 = (n + 1) & 1;
                    ok = mbar_wait(q_full0 + 8 * s1, static_cast<uint32_t>((n + 1) >> 1) & 1u, abort_flag, status, -6);
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_s(n + 1);
                }
                ok = mbar_wait(ds_ready, n & 1u, abort_flag, status, -6);
                if (!ok) break;
                tc_fence_after_sync();
                // dK += dS^T Q: A = dS^T from TMEM, B = Q MN-major
                {
                    const uint32_t b_lo = sdesc_lo(q_st, T::CHUNK_BYTES);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t a_col = (ks < 4 ? 0u : 64u) + (ks & 3) * 8u;
                        mma_bf16_ts(tmem + T::TM_DK, tmem + T::TM_DP + a_col, sdesc_from_lo(b_lo + ks * (2048 >> 4)),
                                    idesc_g, (n > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(q_empty0 + 8 * s);  // dK(n) was the last product to read Q(n)
                // dQ = dS K into [128,256): A = dS (shared memory, query-contiguous rows
                // per key), B = K (key rows, MN-major over d); 16 keys per step
                {
                    const uint32_t a_lo = sdesc_lo(sDS, 16384);
                    const uint32_t b_lo = sdesc_lo(sK, T::CHUNK_BYTES);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ss(tmem + T::TM_DP, sdesc_from_lo(a_lo + ks * (2048 >> 4)),
                                    sdesc_from_lo(b_lo + ks * (2048 >> 4)), idesc_q, ks > 0 ? 1u : 0u);
                }
                mma_commit(dq_full);
            }
            if (ok) mma_commit(dkdv_full);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ P / dS warpgroups
        const int h = (warp - 4) >> 2;  // query half of each score tile
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // key row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const long long k = tile.k0 + row;
        // allowed queries of this key: [i_lo, i_hi] (empty past Lk)
        long long i_lo = 0, i_hi = p.Lq - 1;
        if (band.right >= 0) i_lo = k - band.shift - band.right > 0 ? k - band.shift - band.right : 0;
        if (band.left >= 0 && k - band.shift + band.left < i_hi) i_hi = k - band.shift + band.left;
        if (k >= p.Lk) {
            i_lo = 1;
            i_hi = 0;
        }
        const float c_log2 = p.scale_log2;
        bool ok = true;
        for (int n = 0; n < n_tiles && ok; ++n) {
            const int s = n & 1;
            const long long q0 = static_cast<long long>(tile.q_lo + n) * 128;
            const bool full = q0 + 127 <= p.Lq - 1 && tile_is_full(band, q0, q0 + 127, tile.k0, 128);
            const int c_lo = clamp_int(i_lo - q0) - 64 * h;  // relative to this half's first column
            const int c_hi = clamp_int(i_hi - q0) - 64 * h;
            // LSE2 of this half's 64 query columns at vec, D at vec + 512 (shared addresses)
            const uint32_t vec = sVec + s * T::VEC_STAGE_BYTES + 64 * h * 4;
            // P = exp2(s * scale * log2(e) - LSE2), zero where masked
            ok = mbar_wait(s_full, n & 1u, abort_flag, status, -6);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t pk[32];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t sr[32];
                tmem_ld32(tmem + lane_off + T::TM_S + 64 * h + 32 * cc, sr);
                tmem_wait_ld();
                reg_fence(sr);

#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 l = lds128(vec + (32 * cc + 4 * e4) * 4);
                    const float ls[4] = {l.x, l.y, l.z, l.w};
                    float pv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = 32 * cc + 4 * e4 + u;
                        const float x = __uint_as_float(sr[4 * e4 + u]) * c_log2 - ls[u];
                        const bool allowed = full || (c >= c_lo && c <= c_hi);
                        // masked: 2^-inf = 0; the exponential itself is never conditional
                        pv[u] = fast_exp2(allowed ? x : -CUDART_INF_F);
                    }
                    pk[16 * cc + 2 * e4] = pack_bf16x2(pv[0], pv[1]);
                    pk[16 * cc + 2 * e4 + 1] = pack_bf16x2(pv[2], pv[3]);
                }
            }
            tmem_st32(tmem + lane_off + T::TM_S + 64 * h, pk);
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(p_ready);
            // dS = P (dP - D), from the bf16 P just written (dS is rounded to bf16 next)
            ok = mbar_wait(dp_full, n & 1u, abort_flag, status, -6);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t dk[32];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t dr[32];
                tmem_ld32(tmem + lane_off + T::TM_DP + 64 * h + 32 * cc, dr);
                tmem_wait_ld();
                reg_fence(dr);

#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 dd = lds128(vec + 512 + (32 * cc + 4 * e4) * 4);
                    const float ds[4] = {dd.x, dd.y, dd.z, dd.w};
                    float g[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t w = pk[16 * cc + 2 * e4 + (u >> 1)];
                        const float pval = __uint_as_float((u & 1) ? (w & 0xFFFF0000u) : (w << 16));
                        g[u] = pval * (__uint_as_float(dr[4 * e4 + u]) - ds[u]);
                    }
                    dk[16 * cc + 2 * e4] = pack_bf16x2(g[0], g[1]);
                    dk[16 * cc + 2 * e4 + 1] = pack_bf16x2(g[2], g[3]);
                }
            }
            tmem_st32(tmem + lane_off + T::TM_DP + 64 * h, dk);
            // dS into shared memory as row `row` (key) of the [key][query] operand:
            // 64 queries = one 128-byte row of swizzle column h, 16-byte unit u at u ^ (row & 7)
            {
                const uint32_t drow = sDS + h * 16384 + row * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    sts128(drow + ((u ^ (row & 7)) << 4), dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
            }
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(ds_ready);
        }
        // dK_j = scale * sum_i dS^T Q, dV_j = sum_i P^T dO: warpgroup 0 writes dV, 1 writes dK
        if (ok) {
            const bool have = n_tiles > 0;
            if (have) {
                ok = mbar_wait(dkdv_full, 0, abort_flag, status, -6);
                ok = __all_sync(0xffffffffu, ok);
            }
            if (ok) {
                tc_fence_after_sync();
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(h == 0 ? p.dv : p.dk) +
                                     (static_cast<long long>(tile.bh) * p.Lk + k) * D;
                const float mult = h == 0 ? 1.f : p.scale;
                const uint32_t src = tmem + lane_off + (h == 0 ? T::TM_DV : T::TM_DK);
#pragma unroll 1
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t r[32];
                    if (have) {
                        tmem_ld32(src + ch * 32, r);
                        tmem_wait_ld();
                        reg_fence(r);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = 0u;
                    }
                    if (k < p.Lk) {
                        uint32_t pk16[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk16[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mult, __uint_as_float(r[2 * e + 1]) * mult);
                        uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            d4[v] = make_uint4(pk16[4 * v], pk16[4 * v + 1], pk16[4 * v + 2], pk16[4 * v + 3]);
                    }
                }
            }
        }
        if (p.visited && h == 0 && row == 0)
            atomicAdd(p.visited, static_cast<unsigned long long>(n_tiles));
    } else if (warp >= 12) {
        // ------------------------------------------------------------ dQ drain
        constexpr int NB = D / 64;  // 32-column boxes per half tile
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // query row of the dQ tile
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + T::TM_DP;
        const bool leader = warp == 12 && lane == 0;
        // one half tile (NB boxes of 32 columns, 128-byte rows, 128-byte swizzle) into buf
        auto stage_half = [&](uint32_t buf, uint32_t (&r)[NB][32]) {
#pragma unroll
            for (int c = 0; c < NB; ++c)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    sts128(buf + c * 16384 + row * 128 + ((u ^ (row & 7)) << 4), r[c][4 * u], r[c][4 * u + 1],
                           r[c][4 * u + 2], r[c][4 * u + 3]);
            fence_proxy_async_smem();
            mbar_arrive(dq_staged);
        };
        // leader: reduce-add the staged half once all 128 rows are in, wait until it is read
        auto reduce_half = [&](uint32_t buf, int col0, int y, uint32_t parity, uint32_t release) -> bool {
            if (!mbar_wait(dq_staged, parity, abort_flag, status, -6)) return false;
            for (int c = 0; c < NB; ++c) tma_reduce_add_2d(&tm_dq, buf + c * 16384, col0 + 32 * c, y);
            bulk_commit_group();
            bulk_wait_read_all();
            mbar_arrive(release);
            return true;
        };
        bool ok = true;
        for (int n = 0; n < n_tiles && ok; ++n) {
            const int s = n & 1;
            ok = mbar_wait(dq_full, n & 1u, abort_flag, status, -6);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            // dQ(n) has completed, so dV(n) has read dO(n): its buffer takes the halves
            const uint32_t buf = sStage + s * 2 * T::TILE_BYTES + T::TILE_BYTES;
            const int y = tile.bh * p.Lq_pad + (tile.q_lo + n) * 128;
            uint32_t r[NB][32];
#pragma unroll
            for (int c = 0; c < NB; ++c) tmem_ld32(taddr + 32 * c, r[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < NB; ++c) reg_fence(r[c]);
            stage_half(buf, r);
            // the second half goes to registers and tensor memory is released
#pragma unroll
            for (int c = 0; c < NB; ++c) tmem_ld32(taddr + D / 2 + 32 * c, r[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < NB; ++c) reg_fence(r[c]);
            tc_fence_before_sync();
            mbar_arrive(dq_empty);
            if (leader) ok = reduce_half(buf, 0, y, 0u, stage_reuse);
            __syncwarp();
            ok = __all_sync(0xffffffffu, ok) && mbar_wait(stage_reuse, n & 1u, abort_flag, status, -6);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            stage_half(buf, r);
            if (leader) ok = reduce_half(buf, D / 2, y, 1u, do_empty0 + 8 * s);
            __syncwarp();
            ok = __all_sync(0xffffffffu, ok);
        }
        // the reduce-adds land in the accumulator before the CTA exits
        if (leader) bulk_wait_all();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        if (lane == 0) {
            // every MMA this CTA issued has finished before TMEM is released
            mma_commit(drain_bar);
            mbar_wait(drain_bar, 0, nullptr, status, -6);
        }
        __syncwarp();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

}  // namespace fattn
