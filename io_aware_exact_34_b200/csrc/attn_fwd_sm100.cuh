// attn_fwd_sm100.cuh -- bf16 prefill forward on the 5th-generation tensor cores.
//
// The operation is the tiled online-softmax attention of the sliding-window
// FlashAttention prefill page (m.xxqk.cn/news/265020) §3.1-§3.2: Q, K and V
// are cut into 128-row tiles, each Q tile keeps its running row max m_i,
// running sum l_i and accumulator acc on chip, every visited KV tile updates
// them (m_new = max(m_i, rowmax s_ij), p_ij = exp(s_ij - m_new),
// alpha = exp(m_i - m_new), l_i = alpha l_i + rowsum p_ij,
// acc = alpha acc + p_ij v_j), and only O = acc / l_i reaches device memory.
// KV tiles outside the band are never loaded (§5.1, §5.3, §7.3); tiles the
// band crosses get the element mask before the softmax (§5.2).
//
// B200 mapping (one persistent CTA per SM, 384 threads):
//   warp 0        TMA producer: Q tile pair, then a ring of K / V tiles
//   warp 1        MMA issuer (one thread): S = Q K^T and O += P V with
//                 tcgen05.mma, accumulators in tensor memory (TMEM)
//   warps 4-7     softmax for Q tile 0 of the pair (one thread per row)
//   warps 8-11    softmax for Q tile 1 of the pair
// The two Q tiles share every K / V tile; while one softmax warpgroup turns
// its S into P, the tensor core works on the other tile.  A work item is one
// (batch, head, Q-tile pair); the producer deals items to the CTAs from a
// per-launch counter, in head groups whose K and V fit a part of L2 (dense
// batches) or in a compacted longest-first order (packed batches), and hands
// each item to the MMA thread and the softmax warps through shared memory.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// P (bf16, two per 32-bit column) overwrites the first 64 columns of its S
// tile and feeds the P.V MMA straight from TMEM, so a tile's next S waits for
// its P.V product.  At d = 64 in bf16 the O tiles leave 128 columns free: P0
// and P1 take [256,384), O0 and O1 move to [384,512), and a tile's next S is
// issued as soon as its softmax warps have read the current S (s_free), so
// the exponentials of one KV tile overlap the S product of the next; the
// softmax waits for the previous P.V product (p_free) before it writes P or
// rescales O.
//
// Exact rescale skipping: the running max used for the exponentials is only
// raised when a new row max exceeds it by more than kRescaleSlack (log2
// units); otherwise p = 2^(x - m) <= 2^kRescaleSlack.  Numerator and
// denominator use the same reference, so O = acc / l is unchanged (the page's
// "skipped block == all -inf block" argument of §5.5 generalises to any
// common reference), and O in TMEM is rescaled only when the reference moves.
//
// FP8 instantiation (kFp8): Q, K are e4m3 [B,H,L,128] and V is e4m3 stored
// transposed, [B,H,128,ldv], so both products read K-major operands; one fp32
// descale per (b,h) for each of Q, K, V.  S = Q K^T and O += P V run as
// kind::f8f6f4 MMAs (32 elements of K per instruction).  The reference max
// moves only when a tile's max passes it by more than kFp8Slack, and
// p = 2^(x - m + 8 - kFp8Slack) <= 2^8 is rounded to e4m3 before the P V
// product, so typical probabilities sit in e4m3's normal range; l sums the
// unrounded p; O = vd * acc / l and LSE = ln2 (m + log2 l - 8 + kFp8Slack).  This is the
// FP8 path FlashAttention-3 is named for in "FlashAttention 深度解析" §4,
// taken on the tiled recurrence above.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>
#include <stddef.h>

#include "dev_prims.cuh"
#include "sched.cuh"

namespace fattn {

constexpr float kRescaleSlack = 8.0f;
// FP8: the reference moves once a tile's max passes it by more than 4 (log2
// units), and p = 2^(x - m + 8 - 4) <= 2^8 stays inside e4m3's range, with
// typical probabilities in its normal range (reading R13).
constexpr float kFp8Slack = 4.0f;

// Work order of packed variable-length batches.  The dense item space (pair
// index descending, then sequence, then head) holds an item for every pair
// index below max_seqlen_q / 256 in every sequence; a batch of mixed lengths
// makes most of them empty and the items' costs uneven.  Each CTA therefore
// builds, in shared memory, a compacted order of the non-empty items:
// sequences longest first (ties by sequence index), within a sequence its
// pair indices descending (under causal masking a pair's cost grows with its
// index), then the heads.  With np_b = ceil(ceil(len_b / 128) / 2) pairs in
// sequence b, perm lists the sequences with np_b > 0 in that order and
// seqoff[i] = H * sum_{i' < i} np_{perm[i']} is the first slot of perm[i].
// The table is a function of the offsets alone, so every CTA builds the same
// one.  The slots are dealt dynamically: the producer thread of a CTA takes
// the next one from a per-launch counter when it starts an item, so CTAs that
// drew short items take more of them, and the items in flight at any time
// belong to few sequences, whose K and V stay in L2.
constexpr int VL_MAX_SEQ = 2048;    // larger batches keep the dense order
constexpr int VL_MAX_PAIRS = 1024;  // max_seqlen_q <= 262144
struct VarlenOrder {
    int np[VL_MAX_SEQ];           // pairs of sequence b
    int perm[VL_MAX_SEQ];         // sequences by np descending
    int seqoff[VL_MAX_SEQ + 1];   // first slot of perm[i]; seqoff[nne] = number of items
    int cursor[VL_MAX_PAIRS + 1]; // histogram of np, then the bucket positions of the scatter
    int nne;                      // sequences with at least one pair
    int item_slot[2];             // the dealt items, handed from the producer to the other roles
};
constexpr int VL_TABLE_BYTES = static_cast<int>(sizeof(VarlenOrder));

template <int D, bool kFp8 = false, bool kVarlen = false>
struct FwdTraits {
    static constexpr int ELEM = kFp8 ? 1 : 2;      // bytes per element
    static constexpr int BQ = 128;                 // rows per Q tile (one per TMEM lane)
    static constexpr int BK = 128;                 // keys per KV tile
    static constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 128 B: one 128-B swizzle column
    static constexpr int NCHUNK = D * ELEM / 128;
    static constexpr int TILE_BYTES = 128 * D * ELEM;
    static constexpr int KSTEPS_S = D * ELEM / 32;  // 32-byte K steps of S = Q K^T
    // K/V ring slots: as many as fit beside the Q pair, the barriers (at most
    // 512 bytes with the misc words), the packed-batch order table and the
    // alignment slack.  K/V tiles come from DRAM whenever the batch's K and V
    // outgrow L2, and the slots in flight hide that latency.
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int NSTAGE =
        (SMEM_LIMIT - 2 * TILE_BYTES - 512 - (kVarlen ? VL_TABLE_BYTES : 0) - 1024) / TILE_BYTES;
    static constexpr int SMEM_Q_OFF = 0;
    static constexpr int SMEM_RING_OFF = 2 * TILE_BYTES;
    static constexpr int SMEM_BAR_OFF = SMEM_RING_OFF + NSTAGE * TILE_BYTES;
    // Decoupled P (bf16, d = 64): the two O tiles take 128 TMEM columns, so P
    // gets columns of its own and a tile's next S = Q K^T is issued as soon as
    // its softmax warps have read the current S into registers, while the
    // exponentials of that S run.  At d = 128 S0, S1, O0, O1 fill TMEM and P
    // overwrites its S tile, so the next S waits for the P V product.
    static constexpr bool DEC = (D == 64) && !kFp8;
    // q_full/empty, kv_full/empty[NSTAGE], s_full/p_ready/o_full[2], drain,
    // item_full/empty[2]; decoupled: s_free[2], p_free[2]
    static constexpr int NBAR = 2 + 2 * NSTAGE + 6 + 1 + 4 + (DEC ? 4 : 0);
    static constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NBAR * 8;
    // packed batches: the VarlenOrder table after the misc words
    static constexpr int SMEM_VL_OFF = SMEM_MISC_OFF + 16;
    static constexpr int SMEM_BYTES = SMEM_VL_OFF + (kVarlen ? VL_TABLE_BYTES : 0) + 1024;  // + alignment slack
    static_assert(NBAR * 8 + 16 <= 512, "barrier space");
    static_assert(NSTAGE >= 4, "K/V ring");
    static constexpr int THREADS = 384;
    // Register split: warpgroup 0 (producer, MMA issuer) lowers to REGS_LOW,
    // the two softmax warpgroups raise to REGS_HIGH.  128*80 + 256*208 = 63488
    // (decoupled: 128*64 + 256*216 = 63488, the waits for the previous P.V
    // product need the extra softmax registers) <= 384 threads * 168
    // registers = 64512, the pool the block is launched with; the host
    // refuses to launch unless the compiled register count provides that pool.
    static constexpr uint32_t REGS_LAUNCH = 168;
    static constexpr uint32_t REGS_LOW = DEC ? 64 : 80;
    static constexpr uint32_t REGS_HIGH = DEC ? 216 : 208;
    static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= THREADS * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;
    // S0, S1 [0, 256); decoupled: P0, P1 [256, 384) (bf16, two per column),
    // O0, O1 [384, 512); otherwise O0, O1 [256, 256 + 2D) and P in its S tile
    __host__ __device__ static constexpr uint32_t tm_s(int t) { return static_cast<uint32_t>(t) * 128u; }
    __host__ __device__ static constexpr uint32_t tm_p(int t) {
        return DEC ? 256u + static_cast<uint32_t>(t) * 64u : tm_s(t);
    }
    __host__ __device__ static constexpr uint32_t tm_o(int t) {
        return (DEC ? 384u : 256u) + static_cast<uint32_t>(t) * D;
    }
    static_assert(!DEC || 384 + 2 * D <= 512, "decoupled TMEM layout");
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(!kFp8 || D == 128, "the FP8 path is built for d = 128");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
};

struct FwdParams {
    void* o;
    float* lse;
    unsigned long long* visited;
    int B, H, Lq, Lk;
    float scale_log2;  // scale * log2(e)
    int causal, window_left, window_right;
    int n_pairs, n_items;
    int vl_order;  // packed batches: 1 = work items in the compacted VarlenOrder, dealt by sched_ctr
    int dyn_deal;  // dense batches: 1 = work items in head groups, dealt by sched_ctr
    int group_heads;  // dense batches: heads per group of the dealt order (their K and V fit L2)
    unsigned int* sched_ctr;  // zeroed before the launch; the next slot to deal
    int o_vec32;   // O's base is 32-byte aligned: the epilogue writes 32-byte pieces of each row
    int inject_stall;  // test hook: CTA 0 never delivers its first K tile
    // packed variable-length batches (B = number of sequences): sequence b
    // owns tokens [cu_q[b], cu_q[b+1]) of Q/O and [cu_k[b], cu_k[b+1]) of K/V
    const int* cu_q;
    const int* cu_k;
    int total_q, total_k;
    // FP8 path: per-(b,h) descales of Q, K, V
    const float* q_descale;
    const float* k_descale;
    const float* v_descale;
};

// The sequence and head of one work item: its pair index, token offsets and
// lengths.  Dense batches: offsets 0, lengths Lq / Lk, tensors indexed by bh.
struct ItemSeq {
    int pair, bh, h;
    int q_start, k_start;  // first token of the sequence (packed batches)
    int len_q, len_k;
};

template <bool kVarlen>
__device__ __forceinline__ ItemSeq item_seq(const FwdParams& p, int item) {
    ItemSeq sq;
    const int BH = p.B * p.H;
    sq.pair = p.n_pairs - 1 - item / BH;
    sq.bh = item % BH;
    sq.h = sq.bh % p.H;
    if constexpr (kVarlen) {
        // clamp the caller's offsets into the packed tensors: every access stays in bounds
        const int b = sq.bh / p.H;
        auto clampi = [](int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); };
        sq.q_start = clampi(__ldg(p.cu_q + b), 0, p.total_q);
        sq.len_q = clampi(__ldg(p.cu_q + b + 1), sq.q_start, p.total_q) - sq.q_start;
        sq.k_start = clampi(__ldg(p.cu_k + b), 0, p.total_k);
        sq.len_k = clampi(__ldg(p.cu_k + b + 1), sq.k_start, p.total_k) - sq.k_start;
    } else {
        sq.q_start = sq.k_start = 0;
        sq.len_q = p.Lq;
        sq.len_k = p.Lk;
    }
    return sq;
}

// The two Q tiles of one work item and the KV tiles they visit.
struct PairTiles {
    int bh, h, q_start, k_start;
    int q_first[2];
    int lo_t[2], hi_t[2];
    int lo, hi;  // union range
};

// Slot of the dealt dense order -> item index (pair-major: item =
// (n_pairs - 1 - pair) * B*H + bh), or -1 past the last slot.  The dealt
// order takes the heads in groups of group_heads (the last group may be
// smaller) and, inside a group, pair indices descending, then heads: the
// items in flight at any time read the K and V of few heads, which stay in
// L2, and a CTA that drew short items takes more of them.
__device__ __forceinline__ int dense_slot_item(const FwdParams& p, int slot) {
    if (slot < 0 || slot >= p.n_items) return -1;
    const int BH = p.B * p.H;
    const int G = p.group_heads;
    const int per_group = p.n_pairs * G;
    const int g = slot / per_group;
    const int r = slot - g * per_group;
    const int gs = BH - g * G < G ? BH - g * G : G;
    const int pair = p.n_pairs - 1 - r / gs;
    const int bh = g * G + r % gs;
    return (p.n_pairs - 1 - pair) * BH + bh;
}

__device__ __forceinline__ int snake_item(int round, int cta, int grid) {
    // Work items are ordered longest first; alternating the direction of
    // each round evens out the per-CTA total.
    return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// Builds the VarlenOrder table.  Called by every thread of the CTA; on return
// the table is visible to all of them.  Needs p.B <= VL_MAX_SEQ and
// p.n_pairs <= VL_MAX_PAIRS (the host checks both).
__device__ void varlen_order_build(const FwdParams& p, VarlenOrder* vo) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int NP = p.n_pairs;
    for (int v = tid; v <= NP; v += nthr) vo->cursor[v] = 0;
    __syncthreads();
    // pairs per sequence, from the offsets clamped exactly as item_seq clamps them
    auto clampi = [](int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); };
    for (int b = tid; b < p.B; b += nthr) {
        const int c0 = clampi(__ldg(p.cu_q + b), 0, p.total_q);
        const int c1 = clampi(__ldg(p.cu_q + b + 1), c0, p.total_q);
        const int nq = (c1 - c0 + 127) / 128;
        const int np = (nq + 1) / 2 < NP ? (nq + 1) / 2 : NP;
        vo->np[b] = np;
        atomicAdd(&vo->cursor[np], 1);  // histogram of np
    }
    __syncthreads();
    if (tid < 32) {
        const int lane = tid;
        const int n = NP + 1;
        const int chunk = (n + 31) / 32;
        const int a = lane * chunk < n ? lane * chunk : n;
        const int e = a + chunk < n ? a + chunk : n;
        // first perm position of the sequences with np == v: the number with
        // np > v, a suffix sum over the histogram, one contiguous chunk of v per lane
        int part = 0;
        for (int v = a; v < e; ++v) part += vo->cursor[v];
        int suf = part;
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += x;
        }
        int run = suf - part;
        for (int v = e - 1; v >= a; --v) {
            const int h = vo->cursor[v];
            vo->cursor[v] = run;
            if (v == 0) vo->nne = run;  // sequences with np > 0
            run += h;
        }
        __syncwarp();
        // stable scatter of the sequences into perm by np descending
        for (int b0 = 0; b0 < p.B; b0 += 32) {
            const int b = b0 + lane;
            const int v = b < p.B ? vo->np[b] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, v);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            if (v > 0) vo->perm[vo->cursor[v] + rank] = b;
            __syncwarp();
            if (v > 0 && lane == 31 - __clz(peers)) vo->cursor[v] += __popc(peers);
            __syncwarp();
        }
        // seqoff: exclusive prefix sums of H * np over perm, 32 sequences per step
        const int nne = vo->nne;
        int carry = 0;
        for (int i0 = 0; i0 < nne; i0 += 32) {
            const int i = i0 + lane;
            const int x = i < nne ? vo->np[vo->perm[i]] : 0;
            int inc = x;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            if (i < nne) vo->seqoff[i] = p.H * (carry + inc - x);
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) vo->seqoff[nne] = p.H * carry;
    }
    __syncthreads();
}

// Slot of the compacted order -> item index of the dense order, or -1 past
// the last slot.  vo_s is the shared-window address of the table.
__device__ __forceinline__ int varlen_slot_item(const FwdParams& p, uint32_t vo_s, int slot) {
    const int nne = lds_s32(vo_s + static_cast<uint32_t>(offsetof(VarlenOrder, nne)));
    const uint32_t so = vo_s + static_cast<uint32_t>(offsetof(VarlenOrder, seqoff));
    if (slot < 0 || slot >= lds_s32(so + 4u * nne)) return -1;
    int lo = 0, hi = nne - 1;  // the last i with seqoff[i] <= slot (seqoff rises strictly)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (lds_s32(so + 4u * mid) <= slot) lo = mid;
        else hi = mid - 1;
    }
    const int s0 = lds_s32(so + 4u * lo);
    const int npb = (lds_s32(so + 4u * (lo + 1)) - s0) / p.H;
    const int local = slot - s0;
    const int b = lds_s32(vo_s + static_cast<uint32_t>(offsetof(VarlenOrder, perm)) + 4u * lo);
    const int pair = npb - 1 - local / p.H;
    return (p.n_pairs - 1 - pair) * (p.B * p.H) + b * p.H + local % p.H;
}

template <bool kVarlen>
__device__ __forceinline__ PairTiles pair_tiles(const FwdParams& p, int item) {
    PairTiles ts;
    const ItemSeq sq = item_seq<kVarlen>(p, item);
    const Band band = make_band(sq.len_q, sq.len_k, p.causal, p.window_left, p.window_right);
    ts.bh = sq.bh;
    ts.h = sq.h;
    ts.q_start = sq.q_start;
    ts.k_start = sq.k_start;
    ts.lo = 0x7fffffff;
    ts.hi = 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int q_first = (2 * sq.pair + t) * 128;
        const int q_last = q_first + 127 < sq.len_q - 1 ? q_first + 127 : sq.len_q - 1;
        ts.q_first[t] = q_first;
        int lo = 0, hi = 0;
        if (q_first < sq.len_q) kv_tile_range(band, q_first, q_last, 128, &lo, &hi);
        ts.lo_t[t] = lo;
        ts.hi_t[t] = hi;
        if (lo < hi) {
            ts.lo = lo < ts.lo ? lo : ts.lo;
            ts.hi = hi > ts.hi ? hi : ts.hi;
        }
    }
    if (ts.lo >= ts.hi) ts.lo = ts.hi = 0;
    return ts;
}

// What one softmax thread needs for its query row in one work item: the KV
// tile range of its Q tile, the key bounds of its row and the key window in
// which a tile needs no mask at all (absolute key indices, clamped to int).
struct RowPlan {
    long long o_off;    // element offset of this row in O
    long long lse_off;  // element offset of this row in LSE
    int lo, hi;       // KV tile range of the Q tile
    int key_lo, key_hi;   // allowed keys of this row: [key_lo, key_hi]
    int full_lo, full_hi; // a tile [k0, k0+127] is unmasked iff k0 >= full_lo && k0+127 <= full_hi
    bool tile_exists, valid;
};

template <int D, bool kVarlen>
__device__ __forceinline__ RowPlan row_plan(const FwdParams& p, int item, int t, int row) {
    RowPlan rp;
    const ItemSeq sq = item_seq<kVarlen>(p, item);
    const Band band = make_band(sq.len_q, sq.len_k, p.causal, p.window_left, p.window_right);
    const long long q_first = static_cast<long long>(2 * sq.pair + t) * 128;
    const long long q_last = q_first + 127 < sq.len_q - 1 ? q_first + 127 : sq.len_q - 1;
    const long long i = q_first + row;
    rp.tile_exists = q_first < sq.len_q;
    rp.valid = i < sq.len_q;
    if constexpr (kVarlen) {
        // packed layout: O [total_q, H, D], LSE [H, total_q]
        const long long tok = sq.q_start + i;
        rp.o_off = (tok * p.H + sq.h) * D;
        rp.lse_off = static_cast<long long>(sq.h) * p.total_q + tok;
    } else {
        rp.o_off = (static_cast<long long>(sq.bh) * p.Lq + i) * D;
        rp.lse_off = static_cast<long long>(sq.bh) * p.Lq + i;
    }
    rp.lo = rp.hi = 0;
    if (rp.tile_exists) kv_tile_range(band, q_first, q_last, 128, &rp.lo, &rp.hi);
    int lo_col, hi_col;
    row_col_bounds(band, i, 0, &lo_col, &hi_col);
    rp.key_lo = lo_col;
    rp.key_hi = hi_col;
    long long fhi = band.Lk - 1;
    if (band.right >= 0 && q_first + band.shift + band.right < fhi) fhi = q_first + band.shift + band.right;
    const long long flo = band.left >= 0 ? q_last + band.shift - band.left : 0;
    rp.full_lo = clamp_int(flo);
    rp.full_hi = clamp_int(fhi);
    return rp;
}

// Exponentials of one 128-score row: p_c = 2^(s_c * c_log2 - m_safe), packed
// to bf16 pairs in pk (key 2i in the low half of pk[i / 32][i % 32]); returns
// the fp32 row sum of the p_c.  Scores are scaled and shifted in packed f32x2
// FMAs, exponentials on the MUFU (ex2.approx); masked scores (-inf) give
// exactly 0.
__device__ __forceinline__ float softmax_tile_probs(const uint32_t (&sr)[4][32], uint32_t (&pk)[2][32], float c_log2,
                                                    float m_safe) {
    const uint64_t scale2 = f2_pack(c_log2, c_log2);
    const uint64_t shift2 = f2_pack(-m_safe, -m_safe);
    uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};  // independent partial sums: no long add chain
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const int c = 2 * i;
        const uint64_t s2 = f2_pack(__uint_as_float(sr[c >> 5][c & 31]), __uint_as_float(sr[c >> 5][(c & 31) + 1]));
        const uint64_t x2 = f2_fma(s2, scale2, shift2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        const uint64_t p2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
        sum2[i & 3] = f2_add(sum2[i & 3], p2);
        float p0, p1;
        f2_unpack(p2, p0, p1);
        pk[i >> 5][i & 31] = pack_bf16x2(p0, p1);
    }
    const uint64_t s01 = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
    float lo, hi;
    f2_unpack(s01, lo, hi);
    return lo + hi;
}

// FP8 variant: p_c = 2^(s_c * c_log2 - m_shift) (m_shift = m_safe - 8 +
// kFp8Slack, so p_c <= 2^8), rounded to e4m3 four to a word (key 4i in the low byte of
// pk[i]); returns the fp32 sum of the unrounded p_c.  Masked scores (-inf)
// give exactly 0.
__device__ __forceinline__ float softmax_tile_probs_fp8(const uint32_t (&sr)[4][32], uint32_t (&pk)[32], float c_log2,
                                                        float m_shift) {
    const uint64_t scale2 = f2_pack(c_log2, c_log2);
    const uint64_t shift2 = f2_pack(-m_shift, -m_shift);
    uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int c = 4 * i;
        const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(sr[c >> 5][c & 31]), __uint_as_float(sr[c >> 5][(c & 31) + 1])),
                                    scale2, shift2);
        const uint64_t x23 = f2_fma(f2_pack(__uint_as_float(sr[c >> 5][(c & 31) + 2]), __uint_as_float(sr[c >> 5][(c & 31) + 3])),
                                    scale2, shift2);
        float x0, x1, x2, x3;
        f2_unpack(x01, x0, x1);
        f2_unpack(x23, x2, x3);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1), p2 = fast_exp2(x2), p3 = fast_exp2(x3);
        sum2[i & 3] = f2_add(sum2[i & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
        pk[i] = pack_e4m3x4(p0, p1, p2, p3);
    }
    const uint64_t s01 = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
    float lo, hi;
    f2_unpack(s01, lo, hi);
    return lo + hi;
}

// Row max of 128 scores with four independent 3-input max chains.
__device__ __forceinline__ float row_max128(const uint32_t (&sr)[4][32]) {
    float m[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const int c = 2 * i;
        m[i & 3] = fmax3(m[i & 3], __uint_as_float(sr[c >> 5][c & 31]), __uint_as_float(sr[c >> 5][(c & 31) + 1]));
    }
    return fmax3(m[0], m[1], fmaxf(m[2], m[3]));
}

template <int D, bool kVarlen, bool kFp8 = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using T = FwdTraits<D, kFp8, kVarlen>;
    static_assert(!(kFp8 && kVarlen), "the FP8 path takes dense batches");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sQ = base + T::SMEM_Q_OFF;
    const uint32_t sRing = base + T::SMEM_RING_OFF;
    const uint32_t bar0 = base + T::SMEM_BAR_OFF;
    const uint32_t q_full = bar0;
    const uint32_t q_empty = bar0 + 8;
    const uint32_t kv_full0 = bar0 + 16;
    const uint32_t kv_empty0 = kv_full0 + 8 * T::NSTAGE;
    const uint32_t s_full0 = kv_empty0 + 8 * T::NSTAGE;
    const uint32_t p_ready0 = s_full0 + 16;
    const uint32_t o_full0 = p_ready0 + 16;
    const uint32_t drain_bar = o_full0 + 16;
    const uint32_t item_full0 = drain_bar + 8;    // [2]: the producer dealt an item (dynamic deal)
    const uint32_t item_empty0 = item_full0 + 16;  // [2]: the MMA thread and the 8 softmax warps read it
    const uint32_t s_free0 = item_empty0 + 16;     // [2] decoupled: the softmax warps have read S out of TMEM
    const uint32_t p_free0 = s_free0 + 16;         // [2] decoupled: the P V product that read P is done
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + T::SMEM_MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + T::SMEM_MISC_OFF + 4);
    int* status = &g_fattn_status;
    const uint32_t vo_s = base + T::SMEM_VL_OFF;
    const bool vl = kVarlen && p.vl_order;
    if (vl) varlen_order_build(p, reinterpret_cast<VarlenOrder*>(gbase + T::SMEM_VL_OFF));
    // dynamic deal: the producer takes slots from sched_ctr and hands the items
    // to the MMA thread and the softmax warps through a two-entry ring here
    const bool dyn = kVarlen ? vl : p.dyn_deal != 0;
    const uint32_t item_ring_s =
        kVarlen ? vo_s + static_cast<uint32_t>(offsetof(VarlenOrder, item_slot)) : base + T::SMEM_MISC_OFF + 8;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < T::NSTAGE; ++s) {
            mbar_init(kv_full0 + 8 * s, 1);
            mbar_init(kv_empty0 + 8 * s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full0 + 8 * t, 1);
            mbar_init(p_ready0 + 8 * t, 128);
            mbar_init(o_full0 + 8 * t, 1);
        }
        mbar_init(drain_bar, 1);
        for (int e = 0; e < 2; ++e) {
            mbar_init(item_full0 + 8 * e, 1);
            mbar_init(item_empty0 + 8 * e, 9);
        }
        if constexpr (T::DEC) {
            for (int t = 0; t < 2; ++t) {
                mbar_init(s_free0 + 8 * t, 4);  // lane 0 of each of the tile's four softmax warps
                mbar_init(p_free0 + 8 * t, 1);
            }
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), T::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
    
    if (warp < 4) {
      warpgroup_reg_lower<T::REGS_LOW>();
      if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t ring = 0, q_round = 0;
            bool ok = true;
            for (int round = 0; ok; ++round) {
                int item;
                if (dyn) {
                    // deal: the next slot of the launch's counter, handed to the other roles
                    const int slot = static_cast<int>(atomicAdd(p.sched_ctr, 1u));
                    item = kVarlen ? varlen_slot_item(p, vo_s, slot) : dense_slot_item(p, slot);
                    const int e = round & 1;
                    if (round >= 2) {
                        ok = mbar_wait(item_empty0 + 8 * e, ((round >> 1) - 1) & 1, abort_flag, status, -6);
                        if (!ok) break;
                    }
                    sts_s32(item_ring_s + 4u * e, item);
                    mbar_arrive(item_full0 + 8 * e);
                } else {
                    const int slot = snake_item(round, blockIdx.x, gridDim.x);
                    item = slot < p.n_items ? slot : -1;
                }
                if (item < 0) break;
                const PairTiles ts = pair_tiles<kVarlen>(p, item);
                if (ts.lo >= ts.hi) continue;
                if (q_round > 0) {
                    ok = mbar_wait(q_empty, (q_round - 1) & 1u, abort_flag, status, -6);
                    if (!ok) break;
                }
                mbar_arrive_expect_tx(q_full, 2 * T::TILE_BYTES);
                for (int t = 0; t < 2; ++t)
                    for (int c = 0; c < T::NCHUNK; ++c)
                        tma_load_3d(sQ + t * T::TILE_BYTES + c * T::CHUNK_BYTES, &tm_q, q_full, c * (128 / T::ELEM),
                                    kVarlen ? ts.h : ts.q_first[t], kVarlen ? ts.q_start + ts.q_first[t] : ts.bh);
                ++q_round;
                for (int j = ts.lo; j < ts.hi && ok; ++j) {
                    for (int kv = 0; kv < 2; ++kv) {
                        const uint32_t slot = ring % T::NSTAGE, use = ring / T::NSTAGE;
                        if (use > 0) {
                            ok = mbar_wait(kv_empty0 + 8 * slot, (use - 1) & 1u, abort_flag, status, -6);
                            if (!ok) break;
                        }
                        if (p.inject_stall && blockIdx.x == 0 && ring == 0) {
                            // Test hook: this tile is never loaded, so every wait
                            // that depends on it runs out its time limit.
                            ++ring;
                            continue;
                        }
                        const uint32_t fb = kv_full0 + 8 * slot;
                        mbar_arrive_expect_tx(fb, T::TILE_BYTES);
                        if (kFp8 && kv) {
                            // V^T tile: 128 keys (x, contiguous) of all 128 d rows
                            tma_load_3d(sRing + slot * T::TILE_BYTES, &tm_v, fb, j * 128, 0, ts.bh);
                        } else {
                            for (int c = 0; c < T::NCHUNK; ++c)
                                tma_load_3d(sRing + slot * T::TILE_BYTES + c * T::CHUNK_BYTES, kv ? &tm_v : &tm_k, fb,
                                            c * (128 / T::ELEM), kVarlen ? ts.h : j * 128,
                                            kVarlen ? ts.k_start + j * 128 : ts.bh);
                        }
                        ++ring;
                    }
                }
            }
            // No TMA write may still be landing in shared memory when the CTA exits.
            if (q_round > 0) mbar_wait(q_full, (q_round - 1) & 1u, nullptr, status, -6);
            for (uint32_t s = 0; s < T::NSTAGE; ++s) {
                if (ring > s) {
                    const uint32_t uses = (ring - 1 - s) / T::NSTAGE + 1;
                    mbar_wait(kv_full0 + 8 * s, (uses - 1) & 1u, nullptr, status, -6);
                }
            }
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = kFp8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
            // FP8: V^T is K-major; bf16: V is MN-major (d contiguous)
            constexpr uint32_t idesc_pv = kFp8 ? idesc_e4m3_f32(128, D, 0, 0) : idesc_bf16_f32(128, D, 0, 1);
            uint32_t ring = 0, q_round = 0, p_cnt[2] = {0u, 0u};
            [[maybe_unused]] uint32_t s_cnt[2] = {0u, 0u};  // decoupled: S products issued per tile
            bool ok = true;
            for (int round = 0; ok; ++round) {
                int item;
                if (dyn) {
                    const int e = round & 1;
                    ok = mbar_wait(item_full0 + 8 * e, (round >> 1) & 1, abort_flag, status, -6);
                    if (!ok) break;
                    item = lds_s32(item_ring_s + 4u * e);
                    mbar_arrive(item_empty0 + 8 * e);
                } else {
                    const int slot = snake_item(round, blockIdx.x, gridDim.x);
                    item = slot < p.n_items ? slot : -1;
                }
                if (item < 0) break;
                const PairTiles ts = pair_tiles<kVarlen>(p, item);
                if (ts.lo >= ts.hi) continue;
                ok = mbar_wait(q_full, q_round & 1u, abort_flag, status, -6);
                if (!ok) break;
                ++q_round;
                tc_fence_after_sync();
                const uint32_t ring0 = ring;
                for (int j = ts.lo; j <= ts.hi && ok; ++j) {
                    const bool haveK = j < ts.hi;
                    const bool haveV = j > ts.lo;
                    const uint32_t rK = ring0 + 2u * static_cast<uint32_t>(j - ts.lo);
                    const uint32_t rV = rK - 1u;  // V tile of KV tile j-1
                    bool doS[2], doPV[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        doS[t] = haveK && j >= ts.lo_t[t] && j < ts.hi_t[t];
                        doPV[t] = haveV && j - 1 >= ts.lo_t[t] && j - 1 < ts.hi_t[t];
                    }
                    // S_t = Q_t K_j^T
                    auto issue_s = [&](int t) {
                        const uint32_t k_lo = sdesc_lo(sRing + (rK % T::NSTAGE) * T::TILE_BYTES, 16);
                        const uint32_t q_lo = sdesc_lo(sQ + t * T::TILE_BYTES, 16);
#pragma unroll
                        for (int ks = 0; ks < T::KSTEPS_S; ++ks) {
                            // 32 B along the swizzled row per step; every 128 B the next 16 KB column
                            const uint32_t off = ((ks / 4) * T::CHUNK_BYTES + (ks % 4) * 32) >> 4;
                            if constexpr (kFp8)
                                mma_fp8_ss(tmem + T::tm_s(t), sdesc_from_lo(q_lo + off), sdesc_from_lo(k_lo + off),
                                           idesc_s, ks > 0 ? 1u : 0u);
                            else
                                mma_bf16_ss(tmem + T::tm_s(t), sdesc_from_lo(q_lo + off), sdesc_from_lo(k_lo + off),
                                            idesc_s, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(s_full0 + 8 * t);
                    };
                    // O_t += P_t V_{j-1}
                    auto issue_pv = [&](int t) {
                        const uint32_t first = (j - 1 == ts.lo_t[t]) ? 1u : 0u;
                        if constexpr (kFp8) {
                            const uint32_t v_lo = sdesc_lo(sRing + (rV % T::NSTAGE) * T::TILE_BYTES, 16);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                // 32 keys = 8 TMEM columns of packed P, 32 B along the V^T rows
                                mma_fp8_ts(tmem + T::tm_o(t), tmem + T::tm_p(t) + ks * 8,
                                           sdesc_from_lo(v_lo + ks * (32 >> 4)), idesc_pv, (first && ks == 0) ? 0u : 1u);
                            }
                        } else {
                            const uint32_t v_lo = sdesc_lo(sRing + (rV % T::NSTAGE) * T::TILE_BYTES, T::CHUNK_BYTES);
#pragma unroll
                            for (int ks = 0; ks < 8; ++ks) {
                                // 16 keys = 8 TMEM columns of packed P, 16 rows of 128 B further into the V tile
                                mma_bf16_ts(tmem + T::tm_o(t), tmem + T::tm_p(t) + ks * 8,
                                            sdesc_from_lo(v_lo + ks * (2048 >> 4)), idesc_pv,
                                            (first && ks == 0) ? 0u : 1u);
                            }
                        }
                        if (j - 1 == ts.hi_t[t] - 1) mma_commit(o_full0 + 8 * t);
                    };
                    if constexpr (T::DEC) {
                        // S of both tiles first, each as soon as its softmax warps have read
                        // the previous S; then the P V products of the previous KV tile
                        if (haveK) ok = mbar_wait(kv_full0 + 8 * (rK % T::NSTAGE), (rK / T::NSTAGE) & 1u, abort_flag, status, -6);
                        for (int t = 0; t < 2 && ok; ++t) {
                            if (!doS[t]) continue;
                            if (s_cnt[t] > 0) ok = mbar_wait(s_free0 + 8 * t, (s_cnt[t] - 1u) & 1u, abort_flag, status, -6);
                            if (!ok) break;
                            ++s_cnt[t];
                            tc_fence_after_sync();
                            issue_s(t);
                        }
                        if (!ok) break;
                        if (haveK) {
                            mma_commit(kv_empty0 + 8 * (rK % T::NSTAGE));
                            if (j == ts.hi - 1) mma_commit(q_empty);
                        }
                        if (haveV) ok = mbar_wait(kv_full0 + 8 * (rV % T::NSTAGE), (rV / T::NSTAGE) & 1u, abort_flag, status, -6);
                        for (int t = 0; t < 2 && ok; ++t) {
                            if (!doPV[t]) continue;
                            ok = mbar_wait(p_ready0 + 8 * t, p_cnt[t] & 1u, abort_flag, status, -6);
                            ++p_cnt[t];
                            if (!ok) break;
                            tc_fence_after_sync();
                            issue_pv(t);
                            mma_commit(p_free0 + 8 * t);
                        }
                        if (!ok) break;
                        if (haveV) mma_commit(kv_empty0 + 8 * (rV % T::NSTAGE));
                    } else {
                        if (haveK) ok = mbar_wait(kv_full0 + 8 * (rK % T::NSTAGE), (rK / T::NSTAGE) & 1u, abort_flag, status, -6);
                        if (ok && haveV) ok = mbar_wait(kv_full0 + 8 * (rV % T::NSTAGE), (rV / T::NSTAGE) & 1u, abort_flag, status, -6);
                        if (!ok) break;
                        tc_fence_after_sync();
                        for (int t = 0; t < 2 && ok; ++t) {
                            if (doPV[t]) {
                                ok = mbar_wait(p_ready0 + 8 * t, p_cnt[t] & 1u, abort_flag, status, -6);
                                ++p_cnt[t];
                                if (!ok) break;
                                tc_fence_after_sync();
                                issue_pv(t);
                            }
                            if (doS[t]) issue_s(t);
                        }
                        if (!ok) break;
                        if (haveV) mma_commit(kv_empty0 + 8 * (rV % T::NSTAGE));
                        if (haveK) {
                            mma_commit(kv_empty0 + 8 * (rK % T::NSTAGE));
                            if (j == ts.hi - 1) mma_commit(q_empty);
                        }
                    }
                }
                ring = ring0 + 2u * static_cast<uint32_t>(ts.hi - ts.lo);
            }
        }
      }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        warpgroup_reg_raise<T::REGS_HIGH>();
        const int t = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t taddr_s = tmem + lane_off + T::tm_s(t);
        const uint32_t taddr_o = tmem + lane_off + T::tm_o(t);
        const uint32_t taddr_p = tmem + lane_off + T::tm_p(t);
        const uint32_t s_full = s_full0 + 8 * t, p_ready = p_ready0 + 8 * t, o_full = o_full0 + 8 * t;
        constexpr float slack = kFp8 ? kFp8Slack : kRescaleSlack;
        uint32_t s_phase = 0, o_phase = 0;
        [[maybe_unused]] uint32_t p_cnt = 0;  // decoupled: P tiles this warpgroup has written
        bool ok = true;
        for (int round = 0; ok; ++round) {
            int item;
            if (dyn) {
                const int e = round & 1;
                ok = mbar_wait(item_full0 + 8 * e, (round >> 1) & 1, abort_flag, status, -6);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                item = lds_s32(item_ring_s + 4u * e);
                __syncwarp();
                if (lane == 0) mbar_arrive(item_empty0 + 8 * e);
            } else {
                const int slot = snake_item(round, blockIdx.x, gridDim.x);
                item = slot < p.n_items ? slot : -1;
            }
            if (item < 0) break;
            const RowPlan rp = row_plan<D, kVarlen>(p, item, t, row);
            if (!rp.tile_exists) continue;
            float c_log2 = p.scale_log2, o_scale = 1.f;
            if constexpr (kFp8) {
                const int bh = item_seq<kVarlen>(p, item).bh;
                c_log2 *= __ldg(p.q_descale + bh) * __ldg(p.k_descale + bh);
                o_scale = __ldg(p.v_descale + bh);
            }
            if (rp.lo >= rp.hi) {
                // no allowed key for any row of this tile
                if (rp.valid) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + rp.o_off);
#pragma unroll
                    for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                    if (p.lse) p.lse[rp.lse_off] = -CUDART_INF_F;
                }
                continue;
            }
            float m_used = -CUDART_INF_F, l = 0.f;
            for (int j = rp.lo; j < rp.hi; ++j) {
                ok = mbar_wait(s_full, s_phase & 1u, abort_flag, status, -6);
                ++s_phase;
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after_sync();
                uint32_t sr[4][32];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(taddr_s + q4 * 32, sr[q4]);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) reg_fence(sr[q4]);
                if constexpr (T::DEC) {
                    // S is in registers: the next S of this tile may overwrite its columns
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_free0 + 8 * t);
                }
                const int k0 = j * 128;
                const bool full_tile = k0 >= rp.full_lo && k0 + 127 <= rp.full_hi;
                if (!full_tile) {
                    // §5.2: the boundary mask goes on before the softmax
                    const int lo_col = rp.key_lo - k0, hi_col = rp.key_hi - k0;
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c < lo_col || c > hi_col) sr[c >> 5][c & 31] = __float_as_uint(-CUDART_INF_F);
                }
                const float mx_s = row_max128(sr) * c_log2;
                float alpha = 1.f;
                bool resc = false;
                if (mx_s > m_used + slack) {
                    alpha = fast_exp2(m_used - mx_s);  // 0 when m_used is -inf
                    resc = (j > rp.lo) && (m_used != -CUDART_INF_F);
                    m_used = mx_s;
                    l *= alpha;
                }
                const float m_safe = (m_used == -CUDART_INF_F) ? 0.f : m_used;
                if constexpr (kFp8) {
                    uint32_t pk8[32];
                    l += softmax_tile_probs_fp8(sr, pk8, c_log2, m_safe - (8.f - kFp8Slack));
                    tmem_st32(taddr_s, pk8);
                } else {
                    uint32_t pk[2][32];
                    l += softmax_tile_probs(sr, pk, c_log2, m_safe);
                    if constexpr (T::DEC) {
                        // the P V product that read the previous P of this tile, and
                        // accumulated into O, is done: P and O may be written
                        if (p_cnt > 0) {
                            ok = mbar_wait(p_free0 + 8 * t, (p_cnt - 1u) & 1u, abort_flag, status, -6);
                            ok = __all_sync(0xffffffffu, ok);
                            if (!ok) break;
                            tc_fence_after_sync();
                        }
                        ++p_cnt;
                    }
                    tmem_st32(taddr_p, pk[0]);
                    tmem_st32(taddr_p + 32, pk[1]);
                }
                if (__any_sync(0xffffffffu, resc)) {
                    const float a = resc ? alpha : 1.f;
#pragma unroll 1
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t orr[32];
                        tmem_ld32(taddr_o + ch * 32, orr);
                        tmem_wait_ld();
                        reg_fence(orr);
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * a);
                        tmem_st32(taddr_o + ch * 32, orr);
                    }
                }
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(p_ready);
            }
            if (!ok) break;
            // epilogue: O = acc / l, LSE = (m + log2 l) ln 2
            ok = mbar_wait(o_full, o_phase & 1u, abort_flag, status, -6);
            ++o_phase;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const float inv_l = l > 0.f ? o_scale / l : 0.f;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + rp.o_off;
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t orr[32];
                tmem_ld32(taddr_o + ch * 32, orr);
                tmem_wait_ld();
                reg_fence(orr);
                if (rp.valid) {
                    uint32_t pk16[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk16[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
                    if (p.o_vec32) {
                        stg256(orow + ch * 32, pk16[0], pk16[1], pk16[2], pk16[3], pk16[4], pk16[5], pk16[6], pk16[7]);
                        stg256(orow + ch * 32 + 16, pk16[8], pk16[9], pk16[10], pk16[11], pk16[12], pk16[13], pk16[14],
                               pk16[15]);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk16[4 * v], pk16[4 * v + 1], pk16[4 * v + 2], pk16[4 * v + 3]);
                    }
                }
            }
            if (rp.valid && p.lse)
                p.lse[rp.lse_off] =
                    l > 0.f ? (m_used + __log2f(l) - (kFp8 ? 8.f - kFp8Slack : 0.f)) * 0.6931471805599453f : -CUDART_INF_F;
            if (p.visited && quarter == 0 && lane == 0)
                atomicAdd(p.visited, static_cast<unsigned long long>(rp.hi - rp.lo));
        }
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
