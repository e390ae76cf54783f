// fattn_api.cu -- the C ABI of libfattn (declared in include/fattn.h).
//
// One translation unit: argument checks (before any CUDA call), TMA tensor
// map encoding, per-device launch attributes, kernel launches, host-side block
// accounting and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fattn.h"

#include "attn_bwd_sm100.cuh"
#include "attn_fwd_f32.cuh"
#include "attn_fwd_sm100.cuh"
#include "decode_splitkv.cuh"
#include "fp8_quant.cuh"
#include "sched.cuh"

namespace {

using namespace fattn;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool sm100 = false;
    bool fwd_regs_ok = false;  // the prefill kernels' register pool covers their split
    int num_sms = 0;
};

// The prefill kernel's warpgroups change their register budgets with
// setmaxnreg; the sum must fit the pool the block is launched with, or the
// raising warpgroups would wait forever.  Checked against the compiled kernel.
template <int D>
bool fwd_register_pool_ok() {
    cudaFuncAttributes a, b, c;
    if (cudaFuncGetAttributes(&a, attn_fwd_sm100_kernel<D, false>) != cudaSuccess ||
        cudaFuncGetAttributes(&b, attn_fwd_sm100_kernel<D, true>) != cudaSuccess ||
        cudaFuncGetAttributes(&c, attn_fwd_sm100_kernel<128, false, true>) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    using T = FwdTraits<D>;
    const long long need = 128LL * T::REGS_LOW + 256LL * T::REGS_HIGH;
    return static_cast<long long>(a.numRegs) * T::THREADS >= need && static_cast<long long>(b.numRegs) * T::THREADS >= need &&
           static_cast<long long>(c.numRegs) * T::THREADS >= need;
}

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_inject_stall{0};

// Library-owned decode scratch for attn_decode_splitkv_noalloc.  Host code
// must not pass the array's name to a kernel (on the host it names a
// stand-in, not device memory): its device address is looked up per device.
__device__ __align__(256) float g_decode_noalloc_scratch[FATTN_DECODE_NOALLOC_SCRATCH_BYTES / sizeof(float)];
void* g_noalloc_scratch_addr[kMaxDevices] = {};

// Work counters of the prefill kernels' dynamic deal: each launch takes the
// next of kSchedSlots counters (a host ticket) and zeroes it on its stream, so
// launches in flight at the same time use different counters as long as
// fewer than kSchedSlots of them overlap.
constexpr unsigned kSchedSlots = 64;
__device__ unsigned int g_sched_ctr[kSchedSlots];
unsigned int* g_sched_addr[kMaxDevices] = {};
std::atomic<unsigned> g_sched_ticket{0};

int sched_counter(unsigned int** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FATTN_ERR_NO_DEVICE;
    }
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_sched_addr[dev] == nullptr) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_sched_ctr) != cudaSuccess || addr == nullptr) {
                cudaGetLastError();
                return FATTN_ERR_CUDA;
            }
            g_sched_addr[dev] = static_cast<unsigned int*>(addr);
        }
    }
    *out = g_sched_addr[dev] + (g_sched_ticket.fetch_add(1) % kSchedSlots);
    return FATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device, checked to be sm_100 with the kernels' launch attributes set.
int device_ready(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices) return FATTN_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return FATTN_ERR_NO_DEVICE;
        }
        di.sm100 = (major == 10 && minor == 0);
        di.num_sms = sms;
        if (di.sm100) {
            cudaError_t e = cudaSuccess;
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_sm100_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdTraits<128>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_sm100_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdTraits<64>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_sm100_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdTraits<128, false, true>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_sm100_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdTraits<64, false, true>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_sm100_kernel<128, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdTraits<128, true>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_bwd_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdTraits<128>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_bwd_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdTraits<64>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, F32Traits<128>::SMEM_BYTES);
            e = e != cudaSuccess ? e : cudaFuncSetAttribute(attn_fwd_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, F32Traits<64>::SMEM_BYTES);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return FATTN_ERR_CUDA;
            }
            di.fwd_regs_ok = fwd_register_pool_ok<128>() && fwd_register_pool_ok<64>();
            if (g_encode == nullptr) {
                void* fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || fn == nullptr) {
                    cudaGetLastError();
                    return FATTN_ERR_CUDA;
                }
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
        }
        di.ready = true;
    }
    if (!di.sm100) return FATTN_ERR_NO_DEVICE;
    *out = di;
    return FATTN_OK;
}

// Common checks of the prefill entry points (host only, no CUDA call).
int check_prefill(const void* q, const void* k, const void* v, const void* o, const void* lse, int B, int H,
                  int Lq, int Lk, int d, float scale) {
    if (!q || !k || !v || !o) return FATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return FATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
    const long long bh = static_cast<long long>(B) * H;
    if (bh > 0x7fffffffLL || Lq > 0x7fffff00 || Lk > 0x7fffff00) return FATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FATTN_ERR_MISALIGNED;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FATTN_ERR_MISALIGNED;
    return FATTN_OK;
}

// [B*H, L, d] bf16 tensor, 64-element x 128-row boxes, 128-byte swizzle.
int encode_map(CUtensorMap* map, const void* base, int d, long long L, long long BH) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FATTN_OK : FATTN_ERR_CUDA;
}

// Packed [total, H, d] bf16 tensor viewed as (d, H, total): 64-element x
// 1-head x 128-token boxes land as the same 128-row, 128-byte-swizzled tile.
int encode_map_packed(CUtensorMap* map, const void* base, int d, int H, long long total) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(total)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FATTN_OK : FATTN_ERR_CUDA;
}

// An 8-bit [outer, rows, inner] tensor (row pitch `pitch` bytes) in
// 128-byte x 128-row boxes with 128-byte swizzle: the FP8 Q, K (inner = d)
// and transposed V (inner = keys) tiles.
int encode_map_u8(CUtensorMap* map, const void* base, long long inner, long long rows, long long outer, long long pitch) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch), static_cast<cuuint64_t>(pitch) * rows};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FATTN_OK : FATTN_ERR_CUDA;
}

// The fp32 dQ accumulator as a 2-D [rows, d] tensor: 32-float x 128-row boxes
// (128-byte rows, 128-byte swizzle) for the backward's TMA reduce-adds.
int encode_map_acc(CUtensorMap* map, float* base, int d, long long rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 4};
    cuuint32_t box[2] = {32, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FATTN_OK : FATTN_ERR_CUDA;
}

// Dense prefill work order: heads in groups whose K and V together take at
// most kL2GroupBytes (a part of the 126 MB L2, so the K/V tiles of the items in
// flight are read from DRAM about once), dealt dynamically from a per-launch
// counter zeroed on the stream.
#ifndef FATTN_L2_GROUP_MB
#define FATTN_L2_GROUP_MB 48
#endif
constexpr long long kL2GroupBytes = static_cast<long long>(FATTN_L2_GROUP_MB) << 20;

int setup_dense_deal(FwdParams* p, long long BH, long long kv_bytes_per_head, void* stream) {
    long long G = kv_bytes_per_head > 0 ? kL2GroupBytes / kv_bytes_per_head : BH;
    G = G < 1 ? 1 : (G > BH ? BH : G);
    p->dyn_deal = 1;
    p->group_heads = static_cast<int>(G);
    const int st = sched_counter(&p->sched_ctr);
    if (st != FATTN_OK) return st;
    if (cudaMemsetAsync(p->sched_ctr, 0, sizeof(unsigned int), static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_CUDA;
    }
    return FATTN_OK;
}

template <int D, bool kVarlen>
constexpr int fwd_smem_bytes() {
    return FwdTraits<D, false, kVarlen>::SMEM_BYTES;
}

template <bool kVarlen>
int launch_prefill_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p,
                          int d, int grid, cudaStream_t s) {
    if (d == 128)
        attn_fwd_sm100_kernel<128, kVarlen><<<grid, FwdTraits<128>::THREADS, fwd_smem_bytes<128, kVarlen>(), s>>>(mq, mk, mv, p);
    else
        attn_fwd_sm100_kernel<64, kVarlen><<<grid, FwdTraits<64>::THREADS, fwd_smem_bytes<64, kVarlen>(), s>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk, int d,
               float scale, int causal, int wl, int wr, unsigned long long* visited, void* stream) {
    int st = check_prefill(q, k, v, o, lse, B, H, Lq, Lk, d, scale);
    if (st != FATTN_OK) return st;
    DeviceInfo di;
    st = device_ready(&di);
    if (st != FATTN_OK) return st;
    if (!di.fwd_regs_ok) return FATTN_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    const long long n_qtiles = (Lq + 127) / 128;
    const long long n_pairs = (n_qtiles + 1) / 2;
    const long long n_items = BH * n_pairs;
    if (n_items > 0x7fffffffLL) return FATTN_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mv;
    if (encode_map(&mq, q, d, Lq, BH) != FATTN_OK || encode_map(&mk, k, d, Lk, BH) != FATTN_OK ||
        encode_map(&mv, v, d, Lk, BH) != FATTN_OK)
        return FATTN_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.o_vec32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
    p.lse = lse;
    p.visited = visited;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = wl < 0 ? -1 : wl;
    p.window_right = wr < 0 ? -1 : wr;
    p.n_pairs = static_cast<int>(n_pairs);
    p.n_items = static_cast<int>(n_items);
    p.cu_q = p.cu_k = nullptr;
    p.total_q = p.total_k = 0;
    st = setup_dense_deal(&p, BH, 2LL * Lk * d * 2, stream);
    if (st != FATTN_OK) return st;
    p.inject_stall = g_inject_stall.exchange(0);
    const int grid = static_cast<int>(n_items < di.num_sms ? n_items : di.num_sms);
    return launch_prefill_kernel<false>(mq, mk, mv, p, d, grid, static_cast<cudaStream_t>(stream));
}

int launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q, const int* cu_k,
                      int nseq, int H, int total_q, int total_k, int max_seqlen_q, int d, float scale, int causal,
                      int wl, int wr, unsigned long long* visited, void* stream) {
    if (!cu_q || !cu_k) return FATTN_ERR_INVALID_ARG;
    if (nseq < 1 || max_seqlen_q < 1) return FATTN_ERR_INVALID_ARG;
    int st = check_prefill(q, k, v, o, lse, nseq, H, total_q, total_k, d, scale);
    if (st != FATTN_OK) return st;
    if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u)) return FATTN_ERR_MISALIGNED;
    if (max_seqlen_q > 0x7fffff00) return FATTN_ERR_UNSUPPORTED;
    DeviceInfo di;
    st = device_ready(&di);
    if (st != FATTN_OK) return st;
    if (!di.fwd_regs_ok) return FATTN_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(nseq) * H;
    const long long n_qtiles = (max_seqlen_q + 127) / 128;
    const long long n_pairs = (n_qtiles + 1) / 2;
    const long long n_items = BH * n_pairs;
    if (n_items > 0x7fffffffLL) return FATTN_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mv;
    if (encode_map_packed(&mq, q, d, H, total_q) != FATTN_OK || encode_map_packed(&mk, k, d, H, total_k) != FATTN_OK ||
        encode_map_packed(&mv, v, d, H, total_k) != FATTN_OK)
        return FATTN_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.o_vec32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
    p.lse = lse;
    p.visited = visited;
    p.B = nseq;
    p.H = H;
    p.Lq = max_seqlen_q;
    p.Lk = 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = wl < 0 ? -1 : wl;
    p.window_right = wr < 0 ? -1 : wr;
    p.n_pairs = static_cast<int>(n_pairs);
    p.n_items = static_cast<int>(n_items);
    p.inject_stall = g_inject_stall.exchange(0);
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.total_q = total_q;
    p.total_k = total_k;
    p.vl_order = (nseq <= VL_MAX_SEQ && n_pairs <= VL_MAX_PAIRS) ? 1 : 0;
    if (p.vl_order) {
        st = sched_counter(&p.sched_ctr);
        if (st != FATTN_OK) return st;
        if (cudaMemsetAsync(p.sched_ctr, 0, sizeof(unsigned int), static_cast<cudaStream_t>(stream)) != cudaSuccess) {
            cudaGetLastError();
            return FATTN_ERR_CUDA;
        }
    }
    const int grid = static_cast<int>(n_items < di.num_sms ? n_items : di.num_sms);
    return launch_prefill_kernel<true>(mq, mk, mv, p, d, grid, static_cast<cudaStream_t>(stream));
}

long long bwd_lq_pad(int Lq) { return (static_cast<long long>(Lq) + 127) / 128 * 128; }

// Q tiles visited by all KV tiles of one head: the backward's work count.
long long bwd_visited_tiles(const Band& band, int Lk, int bq, int bk) {
    long long n = 0;
    for (long long k0 = 0; k0 < Lk; k0 += bk) {
        const long long k_last = k0 + bk - 1 < Lk - 1 ? k0 + bk - 1 : Lk - 1;
        int lo = 0, hi = 0;
        q_tile_range(band, k0, k_last, bq, &lo, &hi);
        n += hi - lo;
    }
    return n;
}

int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
               void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal, int wl, int wr,
               void* workspace, size_t workspace_bytes, unsigned long long* visited, void* stream) {
    if (!dout || !lse || !dq || !dk || !dv) return FATTN_ERR_INVALID_ARG;
    int st = check_prefill(q, k, v, o, lse, B, H, Lq, Lk, d, scale);
    if (st != FATTN_OK) return st;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FATTN_ERR_MISALIGNED;
    const long long BH = static_cast<long long>(B) * H;
    const long long n_kv = (Lk + 127) / 128;
    if (BH * n_kv > 0x7fffffffLL) return FATTN_ERR_UNSUPPORTED;
    const size_t need = attn_bwd_workspace_bytes(B, H, Lq, d);
    if (!workspace || workspace_bytes < need) return FATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FATTN_ERR_MISALIGNED;
    DeviceInfo di;
    st = device_ready(&di);
    if (st != FATTN_OK) return st;
    const long long Lq_pad = bwd_lq_pad(Lq);
    CUtensorMap mq, mk, mv, mdo;
    if (encode_map(&mq, q, d, Lq, BH) != FATTN_OK || encode_map(&mk, k, d, Lk, BH) != FATTN_OK ||
        encode_map(&mv, v, d, Lk, BH) != FATTN_OK || encode_map(&mdo, dout, d, Lq, BH) != FATTN_OK)
        return FATTN_ERR_CUDA;
    float* lse2 = static_cast<float*>(workspace);
    float* dsum = lse2 + BH * Lq_pad;
    float* dq_acc = dsum + BH * Lq_pad;
    CUtensorMap mdq;
    if (encode_map_acc(&mdq, dq_acc, d, BH * Lq_pad) != FATTN_OK) return FATTN_ERR_CUDA;
    const Band band = make_band(Lq, Lk, causal, wl, wr);
    BwdParams p;
    p.lse2 = lse2;
    p.dsum = dsum;
    p.dq_acc = dq_acc;
    p.dk = dk;
    p.dv = dv;
    p.visited = visited;
    p.BH = static_cast<int>(BH);
    p.Lq = Lq;
    p.Lk = Lk;
    p.Lq_pad = static_cast<int>(Lq_pad);
    p.n_kv = static_cast<int>(n_kv);
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = wl < 0 ? -1 : wl;
    p.window_right = wr < 0 ? -1 : wr;
    {
        // longest KV tiles first: compare the Q ranges of the first and last KV tile
        int lo0 = 0, hi0 = 0, lo1 = 0, hi1 = 0;
        const long long last0 = (n_kv - 1) * 128;
        q_tile_range(band, 0, 127 < Lk - 1 ? 127 : Lk - 1, 128, &lo0, &hi0);
        q_tile_range(band, last0, Lk - 1, 128, &lo1, &hi1);
        p.reverse = (hi1 - lo1) > (hi0 - lo0) ? 1 : 0;
    }
    {
        const unsigned long long per_head = static_cast<unsigned long long>(Lq_pad) * d * (2 + 2 + 4);
        const unsigned long long g = FATTN_BWD_GROUP_BYTES / (per_head > 0 ? per_head : 1);
        p.group = static_cast<int>(g < 1 ? 1 : (g > static_cast<unsigned long long>(BH) ? BH : g));
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* ob = static_cast<const __nv_bfloat16*>(o);
    const auto* dob = static_cast<const __nv_bfloat16*>(dout);
    auto* dqb = static_cast<__nv_bfloat16*>(dq);
    const long long prep_threads = BH * Lq_pad * (d / 8);
    const long long fin_threads = BH * Lq * (d / 8);
    if ((prep_threads + 255) / 256 > 0x7fffffffLL) return FATTN_ERR_UNSUPPORTED;
    const unsigned prep_grid = static_cast<unsigned>((prep_threads + 255) / 256);
    const unsigned fin_grid = static_cast<unsigned>((fin_threads + 255) / 256);
    const unsigned grid = static_cast<unsigned>(BH * n_kv);
    if (d == 128) {
        bwd_prep_kernel<128><<<prep_grid, 256, 0, s>>>(ob, dob, lse, lse2, dsum, dq_acc, p.BH, Lq, p.Lq_pad);
        attn_bwd_sm100_kernel<128><<<grid, BwdTraits<128>::THREADS, BwdTraits<128>::SMEM_BYTES, s>>>(mq, mk, mv, mdo, mdq, p);
        bwd_dq_kernel<128><<<fin_grid, 256, 0, s>>>(dq_acc, dqb, p.BH, Lq, p.Lq_pad, scale);
    } else {
        bwd_prep_kernel<64><<<prep_grid, 256, 0, s>>>(ob, dob, lse, lse2, dsum, dq_acc, p.BH, Lq, p.Lq_pad);
        attn_bwd_sm100_kernel<64><<<grid, BwdTraits<64>::THREADS, BwdTraits<64>::SMEM_BYTES, s>>>(mq, mk, mv, mdo, mdq, p);
        bwd_dq_kernel<64><<<fin_grid, 256, 0, s>>>(dq_acc, dqb, p.BH, Lq, p.Lq_pad, scale);
    }
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int fp8_ld(int Lk) { return (Lk + 15) / 16 * 16; }

int launch_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* qd, const float* kd, const float* vd,
                   void* o, float* lse, int B, int H, int Lq, int Lk, int d, float scale, int causal, int wl, int wr,
                   unsigned long long* visited, void* stream) {
    int st = check_prefill(q8, k8, vt8, o, lse, B, H, Lq, Lk, d, scale);
    if (st != FATTN_OK) return st;
    if (!qd || !kd || !vd) return FATTN_ERR_INVALID_ARG;
    if (d != 128) return FATTN_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(qd) | reinterpret_cast<uintptr_t>(kd) | reinterpret_cast<uintptr_t>(vd)) & 3u)
        return FATTN_ERR_MISALIGNED;
    DeviceInfo di;
    st = device_ready(&di);
    if (st != FATTN_OK) return st;
    if (!di.fwd_regs_ok) return FATTN_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    const long long n_qtiles = (Lq + 127) / 128;
    const long long n_pairs = (n_qtiles + 1) / 2;
    const long long n_items = BH * n_pairs;
    if (n_items > 0x7fffffffLL) return FATTN_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mv;
    if (encode_map_u8(&mq, q8, d, Lq, BH, d) != FATTN_OK || encode_map_u8(&mk, k8, d, Lk, BH, d) != FATTN_OK ||
        encode_map_u8(&mv, vt8, Lk, d, BH, fp8_ld(Lk)) != FATTN_OK)
        return FATTN_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.o_vec32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
    p.lse = lse;
    p.visited = visited;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = wl < 0 ? -1 : wl;
    p.window_right = wr < 0 ? -1 : wr;
    p.n_pairs = static_cast<int>(n_pairs);
    p.n_items = static_cast<int>(n_items);
    p.inject_stall = 0;
    p.cu_q = p.cu_k = nullptr;
    p.total_q = p.total_k = 0;
    p.q_descale = qd;
    p.k_descale = kd;
    p.v_descale = vd;
    st = setup_dense_deal(&p, BH, 2LL * Lk * d, stream);
    if (st != FATTN_OK) return st;
    const int grid = static_cast<int>(n_items < di.num_sms ? n_items : di.num_sms);
    attn_fwd_sm100_kernel<128, false, true><<<grid, FwdTraits<128, true>::THREADS, FwdTraits<128, true>::SMEM_BYTES,
                                               static_cast<cudaStream_t>(stream)>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int auto_splits(int B, int H, int Lk) {
    (void)B;
    (void)H;
    // largest power of two <= 64 that still leaves at least 1024 keys per split
    int S = 1;
    while (S < 64 && static_cast<long long>(Lk) / (S * 2) >= 1024) S *= 2;
    return S;
}

}  // namespace

// ---------------------------------------------------------------- host-buffer prefill
// Chunks of G heads: per head Q, K, V, O (bf16) and LSE (fp32), each array of
// a chunk buffer starting on a 256-byte boundary; two chunk buffers.
struct HostChunkPlan {
    long long heads_per_chunk = 0;
    size_t q_off = 0, k_off = 0, v_off = 0, o_off = 0, l_off = 0, chunk_bytes = 0;
};

size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

bool host_chunk_plan(int B, int H, int Lq, int Lk, int d, HostChunkPlan* plan) {
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1 || (d != 64 && d != 128)) return false;
    const long long BH = static_cast<long long>(B) * H;
    const size_t qb = static_cast<size_t>(Lq) * d * 2, kb = static_cast<size_t>(Lk) * d * 2;
    const size_t in_per_head = qb + 2 * kb;
    long long g = static_cast<long long>((size_t{32} << 20) / in_per_head);
    g = g < 1 ? 1 : (g > BH ? BH : g);
    plan->heads_per_chunk = g;
    const size_t G = static_cast<size_t>(g);
    plan->q_off = 0;
    plan->k_off = round_up256(G * qb);
    plan->v_off = plan->k_off + round_up256(G * kb);
    plan->o_off = plan->v_off + round_up256(G * kb);
    plan->l_off = plan->o_off + round_up256(G * qb);
    plan->chunk_bytes = plan->l_off + round_up256(G * static_cast<size_t>(Lq) * 4);
    return true;
}

// Library-owned streams and events of one device for attn_fwd_host, created
// on first use; g_host_mutex serialises the calls that enqueue on them.
struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, cmp = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in[2] = {}, done[2] = {}, freed[2] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_host_mutex;

int host_pipe_ready(int dev, HostPipe** out) {
    HostPipe& hp = g_pipe[dev];
    if (!hp.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
        e = e != cudaSuccess ? e : cudaStreamCreateWithFlags(&hp.cmp, cudaStreamNonBlocking);
        e = e != cudaSuccess ? e : cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
        cudaEvent_t* evs[] = {&hp.start, &hp.end, &hp.in[0], &hp.in[1], &hp.done[0], &hp.done[1], &hp.freed[0], &hp.freed[1]};
        for (cudaEvent_t* ev : evs) e = e != cudaSuccess ? e : cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return FATTN_ERR_CUDA;
        }
        hp.ready = true;
    }
    *out = &hp;
    return FATTN_OK;
}

int fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk, int d,
             float scale, int causal, int wl, int wr, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o) return FATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
    HostChunkPlan plan;
    if (!host_chunk_plan(B, H, Lq, Lk, d, &plan)) return FATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(B) * H > 0x7fffffffLL || Lq > 0x7fffff00 || Lk > 0x7fffff00) return FATTN_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < 2 * plan.chunk_bytes)
        return FATTN_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FATTN_ERR_NO_DEVICE;
    }
    DeviceInfo di;
    int st = device_ready(&di);
    if (st != FATTN_OK) return st;
    if (!di.fwd_regs_ok) return FATTN_ERR_UNSUPPORTED;

    std::lock_guard<std::mutex> lock(g_host_mutex);
    HostPipe* hp = nullptr;
    st = host_pipe_ready(dev, &hp);
    if (st != FATTN_OK) return st;
    const cudaStream_t caller = static_cast<cudaStream_t>(stream);
    const long long BH = static_cast<long long>(B) * H;
    const size_t qb = static_cast<size_t>(Lq) * d * 2, kb = static_cast<size_t>(Lk) * d * 2, lb = static_cast<size_t>(Lq) * 4;
    const long long G = plan.heads_per_chunk;
    const long long n_chunks = (BH + G - 1) / G;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* qh = static_cast<const uint8_t*>(q);
    const uint8_t* kh = static_cast<const uint8_t*>(k);
    const uint8_t* vh = static_cast<const uint8_t*>(v);
    uint8_t* oh = static_cast<uint8_t*>(o);
    uint8_t* lh = reinterpret_cast<uint8_t*>(lse);

    cudaError_t e = cudaEventRecord(hp->start, caller);
    e = e != cudaSuccess ? e : cudaStreamWaitEvent(hp->h2d, hp->start, 0);
    for (long long c = 0; c < n_chunks && e == cudaSuccess && st == FATTN_OK; ++c) {
        const int b = static_cast<int>(c & 1);
        const long long h0 = c * G;
        const long long g = BH - h0 < G ? BH - h0 : G;
        uint8_t* buf = ws + b * plan.chunk_bytes;
        // chunk c reuses the buffer of chunk c - 2 once its copy back has finished
        if (c >= 2) e = cudaStreamWaitEvent(hp->h2d, hp->freed[b], 0);
        e = e != cudaSuccess ? e : cudaMemcpyAsync(buf + plan.q_off, qh + h0 * qb, g * qb, cudaMemcpyHostToDevice, hp->h2d);
        e = e != cudaSuccess ? e : cudaMemcpyAsync(buf + plan.k_off, kh + h0 * kb, g * kb, cudaMemcpyHostToDevice, hp->h2d);
        e = e != cudaSuccess ? e : cudaMemcpyAsync(buf + plan.v_off, vh + h0 * kb, g * kb, cudaMemcpyHostToDevice, hp->h2d);
        e = e != cudaSuccess ? e : cudaEventRecord(hp->in[b], hp->h2d);
        e = e != cudaSuccess ? e : cudaStreamWaitEvent(hp->cmp, hp->in[b], 0);
        if (e != cudaSuccess) break;
        float* lbuf = lse ? reinterpret_cast<float*>(buf + plan.l_off) : nullptr;
        st = launch_fwd(buf + plan.q_off, buf + plan.k_off, buf + plan.v_off, buf + plan.o_off, lbuf, 1,
                        static_cast<int>(g), Lq, Lk, d, scale, causal, wl, wr, nullptr, hp->cmp);
        e = e != cudaSuccess ? e : cudaEventRecord(hp->done[b], hp->cmp);
        e = e != cudaSuccess ? e : cudaStreamWaitEvent(hp->d2h, hp->done[b], 0);
        e = e != cudaSuccess ? e : cudaMemcpyAsync(oh + h0 * qb, buf + plan.o_off, g * qb, cudaMemcpyDeviceToHost, hp->d2h);
        if (lse) e = e != cudaSuccess ? e : cudaMemcpyAsync(lh + h0 * lb, lbuf, g * lb, cudaMemcpyDeviceToHost, hp->d2h);
        e = e != cudaSuccess ? e : cudaEventRecord(hp->freed[b], hp->d2h);
    }
    // Whatever was queued (all of it, or a prefix after an error), the
    // caller's stream waits for it: compute -> copy-back -> copy-in -> caller.
    cudaError_t j = cudaEventRecord(hp->end, hp->cmp);
    j = j != cudaSuccess ? j : cudaStreamWaitEvent(hp->d2h, hp->end, 0);
    j = j != cudaSuccess ? j : cudaEventRecord(hp->end, hp->d2h);
    j = j != cudaSuccess ? j : cudaStreamWaitEvent(hp->h2d, hp->end, 0);
    j = j != cudaSuccess ? j : cudaEventRecord(hp->end, hp->h2d);
    j = j != cudaSuccess ? j : cudaStreamWaitEvent(caller, hp->end, 0);
    if (e != cudaSuccess || j != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_CUDA;
    }
    return st;
}

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk, int d,
             float scale, int causal, int window_left, int window_right, void* stream) {
    return launch_fwd(q, k, v, o, lse, B, H, Lq, Lk, d, scale, causal, window_left, window_right, nullptr, stream);
}

int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk, int d,
                  float scale, int causal, int window_left, int window_right, void* workspace, size_t workspace_bytes,
                  void* stream) {
    return fwd_host(q, k, v, o, lse, B, H, Lq, Lk, d, scale, causal, window_left, window_right, workspace,
                    workspace_bytes, stream);
}

size_t attn_fwd_host_workspace_bytes(int B, int H, int Lq, int Lk, int d) {
    HostChunkPlan plan;
    return host_chunk_plan(B, H, Lq, Lk, d, &plan) ? 2 * plan.chunk_bytes : 0;
}

int attn_fwd_counted(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk,
                     int d, float scale, int causal, int window_left, int window_right,
                     unsigned long long* kv_tiles_visited, void* stream) {
    if (!kv_tiles_visited) return FATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(kv_tiles_visited) & 7u) return FATTN_ERR_MISALIGNED;
    return launch_fwd(q, k, v, o, lse, B, H, Lq, Lk, d, scale, causal, window_left, window_right, kv_tiles_visited,
                      stream);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                    const int* cu_seqlens_k, int num_seqs, int H, int total_q, int total_k, int max_seqlen_q, int d,
                    float scale, int causal, int window_left, int window_right, void* stream) {
    return launch_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, H, total_q, total_k, max_seqlen_q, d,
                             scale, causal, window_left, window_right, nullptr, stream);
}

int attn_fwd_varlen_counted(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                            const int* cu_seqlens_k, int num_seqs, int H, int total_q, int total_k, int max_seqlen_q,
                            int d, float scale, int causal, int window_left, int window_right,
                            unsigned long long* kv_tiles_visited, void* stream) {
    if (!kv_tiles_visited) return FATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(kv_tiles_visited) & 7u) return FATTN_ERR_MISALIGNED;
    return launch_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, H, total_q, total_k, max_seqlen_q, d,
                             scale, causal, window_left, window_right, kv_tiles_visited, stream);
}

int attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int Lq, int Lk,
                 int d, float scale, int causal, int window_left, int window_right, void* stream) {
    int st = check_prefill(q, k, v, o, lse, B, H, Lq, Lk, d, scale);
    if (st != FATTN_OK) return st;
    if (static_cast<long long>(B) * H > 65535) return FATTN_ERR_UNSUPPORTED;  // grid.y
    DeviceInfo di;
    st = device_ready(&di);
    if (st != FATTN_OK) return st;
    const int wl = window_left < 0 ? -1 : window_left;
    const int wr = window_right < 0 ? -1 : window_right;
    dim3 grid((Lq + 31) / 32, B * H);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 128)
        attn_fwd_f32_kernel<128><<<grid, 128, F32Traits<128>::SMEM_BYTES, s>>>(q, k, v, o, lse, Lq, Lk, scale,
                                                                              causal ? 1 : 0, wl, wr);
    else
        attn_fwd_f32_kernel<64><<<grid, 128, F32Traits<64>::SMEM_BYTES, s>>>(q, k, v, o, lse, Lq, Lk, scale,
                                                                            causal ? 1 : 0, wl, wr);
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int attn_decode_auto_splits(int B, int H, int Lk, int d) {
    if (B < 1 || H < 1 || Lk < 1 || (d != 64 && d != 128)) return FATTN_ERR_INVALID_ARG;
    return auto_splits(B, H, Lk);
}

size_t attn_decode_workspace_bytes(int B, int H, int Lk, int d, int num_splits) {
    if (B < 1 || H < 1 || Lk < 1 || d < 1 || num_splits < 0) return 0;
    const long long S = num_splits == 0 ? auto_splits(B, H, Lk) : num_splits;
    return static_cast<size_t>(B) * H * S * (static_cast<size_t>(d) + 1) * sizeof(float);
}

int attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                        const int* seqlens_k, int B, int H, int Lk, int d, float scale, int num_splits,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k_cache || !v_cache || !o) return FATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Lk < 1 || num_splits < 0) return FATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || Lk > 0x7fffff00) return FATTN_ERR_UNSUPPORTED;
    const int S = num_splits == 0 ? auto_splits(B, H, Lk) : num_splits;
    if (S > Lk) return FATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return FATTN_ERR_MISALIGNED;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FATTN_ERR_MISALIGNED;
    if (seqlens_k && (reinterpret_cast<uintptr_t>(seqlens_k) & 3u)) return FATTN_ERR_MISALIGNED;
    const size_t need = attn_decode_workspace_bytes(B, H, Lk, d, S);
    if (!workspace || workspace_bytes < need) return FATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FATTN_ERR_MISALIGNED;
    DeviceInfo di;
    int st = device_ready(&di);
    if (st != FATTN_OK) return st;
    float* ws_o = static_cast<float*>(workspace);
    float* ws_lse = ws_o + static_cast<size_t>(B) * H * S * d;
    const int chunk = static_cast<int>((static_cast<long long>(Lk) + S - 1) / S);
    const float c_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dim3 grid(S, H, B);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k_cache);
    const auto* vb = static_cast<const __nv_bfloat16*>(v_cache);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    const KvLayout lay{nullptr, 0, 0, 0};
    if (d == 128) {
        decode_split_kernel<128, false><<<grid, 256, 0, s>>>(qb, kb, vb, seqlens_k, ws_o, ws_lse, H, Lk, S, chunk, c_log2, lay);
        decode_merge_kernel<128><<<B * H, 128, 0, s>>>(ws_o, ws_lse, ob, lse, S);
    } else {
        decode_split_kernel<64, false><<<grid, 256, 0, s>>>(qb, kb, vb, seqlens_k, ws_o, ws_lse, H, Lk, S, chunk, c_log2, lay);
        decode_merge_kernel<64><<<B * H, 64, 0, s>>>(ws_o, ws_lse, ob, lse, S);
    }
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table, int max_pages,
                      int page_size, int num_pages, void* o, float* lse, const int* seqlens_k, int B, int H, int d,
                      float scale, int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k_pages || !v_pages || !block_table || !seqlens_k || !o) return FATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || max_pages < 1 || num_pages < 1 || num_splits < 0) return FATTN_ERR_INVALID_ARG;
    if (page_size < 16 || (page_size & (page_size - 1)) != 0) return FATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
    const long long max_len = static_cast<long long>(max_pages) * page_size;
    if (B > 65535 || H > 65535 || max_len > 0x7fffff00 || static_cast<long long>(num_pages) * page_size > (1LL << 40))
        return FATTN_ERR_UNSUPPORTED;
    const int Lk = static_cast<int>(max_len);
    const int S = num_splits == 0 ? auto_splits(B, H, Lk) : num_splits;
    if (S > Lk) return FATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o)) return FATTN_ERR_MISALIGNED;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FATTN_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(seqlens_k) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u))
        return FATTN_ERR_MISALIGNED;
    const size_t need = attn_decode_workspace_bytes(B, H, Lk, d, S);
    if (!workspace || workspace_bytes < need) return FATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FATTN_ERR_MISALIGNED;
    DeviceInfo di;
    int st = device_ready(&di);
    if (st != FATTN_OK) return st;
    float* ws_o = static_cast<float*>(workspace);
    float* ws_lse = ws_o + static_cast<size_t>(B) * H * S * d;
    const int chunk = static_cast<int>((static_cast<long long>(Lk) + S - 1) / S);
    const float c_log2 = scale * 1.4426950408889634f;
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    const KvLayout lay{block_table, max_pages, shift, num_pages};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dim3 grid(S, H, B);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k_pages);
    const auto* vb = static_cast<const __nv_bfloat16*>(v_pages);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    if (d == 128) {
        decode_split_kernel<128, true><<<grid, 256, 0, s>>>(qb, kb, vb, seqlens_k, ws_o, ws_lse, H, Lk, S, chunk, c_log2, lay);
        decode_merge_kernel<128><<<B * H, 128, 0, s>>>(ws_o, ws_lse, ob, lse, S);
    } else {
        decode_split_kernel<64, true><<<grid, 256, 0, s>>>(qb, kb, vb, seqlens_k, ws_o, ws_lse, H, Lk, S, chunk, c_log2, lay);
        decode_merge_kernel<64><<<B * H, 64, 0, s>>>(ws_o, ws_lse, ob, lse, S);
    }
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

int attn_count_blocks(int Lq, int Lk, int causal, int window_left, int window_right, int block_q, int block_k,
                      long long* visited, long long* total, long long* partial, long long* pairs) {
    if (Lq < 1 || Lk < 1 || block_q < 1 || block_k < 1) return FATTN_ERR_INVALID_ARG;
    const Band band = make_band(Lq, Lk, causal, window_left, window_right);
    const long long nq = (Lq + block_q - 1) / block_q, nk = (Lk + block_k - 1) / block_k;
    long long n_visited = 0, n_partial = 0, n_pairs = 0;
    for (long long t = 0; t < nq; ++t) {
        const long long q_first = t * block_q;
        const long long q_last = q_first + block_q - 1 < Lq - 1 ? q_first + block_q - 1 : Lq - 1;
        int lo = 0, hi = 0;
        kv_tile_range(band, q_first, q_last, block_k, &lo, &hi);
        n_visited += hi - lo;
        for (int j = lo; j < hi; ++j)
            if (!tile_is_full(band, q_first, q_last, static_cast<long long>(j) * block_k, block_k)) ++n_partial;
    }
    for (long long i = 0; i < Lq; ++i) {
        int lo_col = 0, hi_col = 0;
        row_col_bounds(band, i, 0, &lo_col, &hi_col);
        if (hi_col >= lo_col) n_pairs += static_cast<long long>(hi_col) - lo_col + 1;
    }
    if (visited) *visited = n_visited;
    if (total) *total = nq * nk;
    if (partial) *partial = n_partial;
    if (pairs) *pairs = n_pairs;
    return FATTN_OK;
}

int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_descale, const float* k_descale,
                 const float* v_descale, void* o, float* lse, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                 int window_left, int window_right, void* stream) {
    return launch_fwd_fp8(q8, k8, vt8, q_descale, k_descale, v_descale, o, lse, B, H, Lq, Lk, d, scale, causal,
                          window_left, window_right, nullptr, stream);
}

int attn_fwd_fp8_counted(const void* q8, const void* k8, const void* vt8, const float* q_descale,
                         const float* k_descale, const float* v_descale, void* o, float* lse, int B, int H, int Lq,
                         int Lk, int d, float scale, int causal, int window_left, int window_right,
                         unsigned long long* kv_tiles_visited, void* stream) {
    if (!kv_tiles_visited) return FATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(kv_tiles_visited) & 7u) return FATTN_ERR_MISALIGNED;
    return launch_fwd_fp8(q8, k8, vt8, q_descale, k_descale, v_descale, o, lse, B, H, Lq, Lk, d, scale, causal,
                          window_left, window_right, kv_tiles_visited, stream);
}

int attn_fp8_ld(int Lk) { return Lk < 1 ? 0 : fp8_ld(Lk); }

int attn_quantize_fp8(const void* x, void* codes, float* descale, int B, int H, int L, int d, int transpose,
                      void* stream) {
    if (!x || !codes || !descale) return FATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1) return FATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
    const long long groups = static_cast<long long>(B) * H;
    if (groups > 65535 || L > 0x7fffff00) return FATTN_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(descale) & 3u)) return FATTN_ERR_MISALIGNED;
    DeviceInfo di;
    int st = device_ready(&di);
    if (st != FATTN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* bits = reinterpret_cast<unsigned int*>(descale);
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    auto* cb = static_cast<uint8_t*>(codes);
    const long long group_len = static_cast<long long>(L) * d;
    if (cudaMemsetAsync(descale, 0, static_cast<size_t>(groups) * sizeof(float), s) != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_CUDA;
    }
    long long per_group = (group_len / 8 + 255) / 256;
    const unsigned bx = static_cast<unsigned>(per_group < 64 ? per_group : 64);
    fp8_amax_kernel<<<dim3(bx, static_cast<unsigned>(groups)), 256, 0, s>>>(xb, bits, group_len);
    if (transpose) {
        const int ld = fp8_ld(L);
        const dim3 grid(static_cast<unsigned>((ld + 63) / 64), static_cast<unsigned>(groups));
        if (d == 128)
            fp8_quant_t_kernel<128><<<grid, 256, 0, s>>>(xb, bits, cb, L, ld);
        else
            fp8_quant_t_kernel<64><<<grid, 256, 0, s>>>(xb, bits, cb, L, ld);
    } else {
        fp8_quant_kernel<<<dim3(bx, static_cast<unsigned>(groups)), 256, 0, s>>>(xb, bits, cb, group_len);
    }
    fp8_descale_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, s>>>(bits, static_cast<int>(groups));
    return cudaGetLastError() == cudaSuccess ? FATTN_OK : FATTN_ERR_CUDA;
}

size_t attn_bwd_workspace_bytes(int B, int H, int Lq, int d) {
    if (B < 1 || H < 1 || Lq < 1 || (d != 64 && d != 128)) return 0;
    return static_cast<size_t>(B) * H * static_cast<size_t>(bwd_lq_pad(Lq)) * (static_cast<size_t>(d) + 2) * sizeof(float);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
             void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal, int window_left,
             int window_right, void* workspace, size_t workspace_bytes, void* stream) {
    return launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, window_left, window_right,
                      workspace, workspace_bytes, nullptr, stream);
}

int attn_bwd_counted(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                     int window_left, int window_right, void* workspace, size_t workspace_bytes,
                     unsigned long long* q_tiles_visited, void* stream) {
    if (!q_tiles_visited) return FATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(q_tiles_visited) & 7u) return FATTN_ERR_MISALIGNED;
    return launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, window_left, window_right,
                      workspace, workspace_bytes, q_tiles_visited, stream);
}

int attn_bwd_count_blocks(int Lq, int Lk, int causal, int window_left, int window_right, int block_q, int block_k,
                          long long* visited) {
    if (Lq < 1 || Lk < 1 || block_q < 1 || block_k < 1 || !visited) return FATTN_ERR_INVALID_ARG;
    const Band band = make_band(Lq, Lk, causal, window_left, window_right);
    *visited = bwd_visited_tiles(band, Lk, block_q, block_k);
    return FATTN_OK;
}

const char* fattn_status_string(int status) {
    switch (status) {
        case FATTN_OK: return "FATTN_OK";
        case FATTN_ERR_INVALID_ARG: return "FATTN_ERR_INVALID_ARG: invalid argument";
        case FATTN_ERR_UNSUPPORTED: return "FATTN_ERR_UNSUPPORTED: unsupported head dim or size";
        case FATTN_ERR_MISALIGNED: return "FATTN_ERR_MISALIGNED: pointer not 16-byte aligned";
        case FATTN_ERR_WORKSPACE: return "FATTN_ERR_WORKSPACE: workspace missing or too small";
        case FATTN_ERR_CUDA: return "FATTN_ERR_CUDA: CUDA call or launch failed";
        case FATTN_ERR_TIMEOUT: return "FATTN_ERR_TIMEOUT: a bounded in-kernel wait expired";
        case FATTN_ERR_NO_DEVICE: return "FATTN_ERR_NO_DEVICE: no usable sm_100 device";
        default: return "unknown fattn status";
    }
}

int fattn_debug_inject_stall(int on) {
    g_inject_stall.store(on ? 1 : 0);
    return FATTN_OK;
}

int fattn_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_CUDA;
    }
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, fattn::g_fattn_status, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(fattn::g_fattn_status, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return FATTN_ERR_CUDA;
    }
    return v;
}

int attn_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                                const int* seqlens_k, int B, int H, int Lk, int d, float scale, int num_splits,
                                void* stream) {
    // host-only checks first: nothing is enqueued for a call the scratch cannot hold
    if (B < 1 || H < 1 || Lk < 1 || num_splits < 0 || (d != 64 && d != 128)) {
        return attn_decode_splitkv(q, k_cache, v_cache, o, lse, seqlens_k, B, H, Lk, d, scale, num_splits,
                                   nullptr, 0, stream);
    }
    const size_t need = attn_decode_workspace_bytes(B, H, Lk, d, num_splits);
    if (need == 0 || need > FATTN_DECODE_NOALLOC_SCRATCH_BYTES) return FATTN_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FATTN_ERR_NO_DEVICE;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_noalloc_scratch_addr[dev] == nullptr) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_decode_noalloc_scratch) != cudaSuccess || addr == nullptr) {
                cudaGetLastError();
                return FATTN_ERR_CUDA;
            }
            g_noalloc_scratch_addr[dev] = addr;
        }
        scratch = g_noalloc_scratch_addr[dev];
    }
    return attn_decode_splitkv(q, k_cache, v_cache, o, lse, seqlens_k, B, H, Lk, d, scale, num_splits, scratch,
                               FATTN_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
