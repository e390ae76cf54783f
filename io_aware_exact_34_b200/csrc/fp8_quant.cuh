// fp8_quant.cuh -- bf16 -> e4m3 quantization for the FP8 forward.
//
// One fp32 scale per (batch, head) group: amax = max |x| over the group,
// code = e4m3(x * (448 / amax)) (nearest, ties to even, saturating), and the
// descale amax / 448 that the attention kernel multiplies back in.  The
// reciprocal scale and the product are single fp32 operations rounded to
// nearest, so the rounding decision is reproducible on the host.  V is written
// transposed ([d][ld] per head) so the P V product reads it K-major.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "dev_prims.cuh"

namespace fattn {

// amax of each group into amax_bits[g] (float bits; non-negative floats order
// like their bit patterns, so atomicMax on the bits is a float max).  The
// array must start at zero.  grid = (blocks per group, groups), 256 threads,
// eight elements per thread per pass.
__global__ void __launch_bounds__(256) fp8_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                       unsigned int* __restrict__ amax_bits, long long group_len) {
    const long long g = blockIdx.y;
    const __nv_bfloat16* xg = x + g * group_len;
    float m = 0.f;
    for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < group_len;
         i += static_cast<long long>(gridDim.x) * blockDim.x * 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(xg + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            m = fmaxf(m, fabsf(__uint_as_float(w[e] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int w = 1; w < 8; ++w) b = fmaxf(b, red[w]);
        atomicMax(amax_bits + g, __float_as_uint(b));
    }
}

__device__ __forceinline__ float fp8_inv_scale(unsigned int amax_bits) {
    const float amax = __uint_as_float(amax_bits);
    return amax > 0.f ? 448.f / amax : 1.f;
}

// Row-major codes: eight elements per thread.  grid = (blocks per group, groups).
__global__ void __launch_bounds__(256) fp8_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                        const unsigned int* __restrict__ amax_bits,
                                                        uint8_t* __restrict__ codes, long long group_len) {
    const long long g = blockIdx.y;
    const float inv = fp8_inv_scale(amax_bits[g]);
    for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < group_len;
         i += static_cast<long long>(gridDim.x) * blockDim.x * 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(x + g * group_len + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        float f[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            f[2 * e] = __fmul_rn(__uint_as_float(w[e] << 16), inv);
            f[2 * e + 1] = __fmul_rn(__uint_as_float(w[e] & 0xFFFF0000u), inv);
        }
        uint2 out;
        out.x = pack_e4m3x4(f[0], f[1], f[2], f[3]);
        out.y = pack_e4m3x4(f[4], f[5], f[6], f[7]);
        *reinterpret_cast<uint2*>(codes + g * group_len + i) = out;
    }
}

// Transposed codes: x is [groups][L][D], codes are [groups][D][ld] (ld >= L,
// a multiple of 16); columns [L, ld) are written as 0.  One block per
// (64-token tile, group), 256 threads.  The tile (64 x D bf16) is read with
// coalesced 16-byte loads into shared memory as it is laid out in x; then
// each thread takes a pair of d rows and 64 / (512 / D) consecutive tokens,
// reads its values as 4-byte (d, d+1) pairs (a warp reads contiguous bytes of
// one token row), quantizes them and writes one 16-byte piece of each of its
// two d rows of the codes.
template <int D>
__global__ void __launch_bounds__(256) fp8_quant_t_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const unsigned int* __restrict__ amax_bits,
                                                          uint8_t* __restrict__ codes, int L, int ld) {
    constexpr int TT = 64;                 // tokens per tile
    constexpr int PAIRS = D / 2;           // d pairs
    constexpr int SEGS = 256 / PAIRS;      // token segments per tile: 4 (D = 128) or 8 (D = 64)
    constexpr int SEG = TT / SEGS;         // tokens per thread: 16 or 8
    static_assert(SEG == 8 || SEG == 16, "one 8- or 16-byte piece per d row");
    __shared__ __align__(16) uint32_t tile[TT][D / 2];  // bf16 pairs, as in x
    const long long g = blockIdx.y;
    const int t0 = blockIdx.x * TT;
    const float inv = fp8_inv_scale(amax_bits[g]);
    for (int c = threadIdx.x; c < TT * (D / 8); c += blockDim.x) {
        const int r = c / (D / 8), c8 = c % (D / 8);
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (t0 + r < L) u = *reinterpret_cast<const uint4*>(x + (g * L + t0 + r) * D + c8 * 8);
        *reinterpret_cast<uint4*>(&tile[r][c8 * 4]) = u;
    }
    __syncthreads();
    const int dp = threadIdx.x % PAIRS, seg = threadIdx.x / PAIRS;
    const int tok0 = seg * SEG;
    const int col = t0 + tok0;
    if (col >= ld) return;
    uint32_t lo[SEG / 4], hi[SEG / 4];  // codes of d = 2 dp and 2 dp + 1, four tokens per word
#pragma unroll
    for (int w = 0; w < SEG / 4; ++w) {
        float a[4], b[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t v = tile[tok0 + 4 * w + e][dp];
            a[e] = __fmul_rn(__uint_as_float(v << 16), inv);
            b[e] = __fmul_rn(__uint_as_float(v & 0xFFFF0000u), inv);
        }
        lo[w] = pack_e4m3x4(a[0], a[1], a[2], a[3]);
        hi[w] = pack_e4m3x4(b[0], b[1], b[2], b[3]);
    }
    uint8_t* r0 = codes + (g * D + 2 * dp) * static_cast<long long>(ld) + col;
    uint8_t* r1 = r0 + ld;
    if constexpr (SEG == 16) {  // 16-byte aligned: col is a multiple of 16, ld too
        *reinterpret_cast<uint4*>(r0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(r1) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    } else {
        *reinterpret_cast<uint2*>(r0) = make_uint2(lo[0], lo[1]);
        *reinterpret_cast<uint2*>(r1) = make_uint2(hi[0], hi[1]);
    }
}

// amax bits -> descale amax / 448 (1 for an all-zero group), in place.
__global__ void fp8_descale_kernel(unsigned int* __restrict__ amax_bits_to_descale, int groups) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= groups) return;
    const float amax = __uint_as_float(amax_bits_to_descale[g]);
    reinterpret_cast<float*>(amax_bits_to_descale)[g] = amax > 0.f ? amax / 448.f : 1.f;
}

}  // namespace fattn
