/*
 * fattn.h -- C ABI of libfattn: exact, IO-aware tiled attention on B200 (sm_100a).
 *
 * What is computed.  For every batch element b, head h and query row i:
 *
 *     O[b,h,i,:] = sum_j softmax_j(scale * q_i . k_j) v_j        over allowed j
 *     LSE[b,h,i] = ln sum_j exp(scale * q_i . k_j)               over allowed j
 *
 * the attention formula of the sliding-window FlashAttention prefill page
 * (m.xxqk.cn/news/265020) §2, evaluated with the tiled online softmax of §3.2
 * (running row max m, running sum l, rescale alpha = exp(m_old - m_new) of the
 * accumulator) so the n x n score matrix never reaches device memory, and with
 * the band mask of §4 / §4.1 evaluated by block skipping (§5.1, §5.3, §7.3):
 * KV tiles that hold no allowed pair are never loaded or multiplied.
 *
 * The mask.  window_size = (window_left, window_right) as in §7.1:
 *   key j is allowed for query i iff, with pos = i + (Lk - Lq),
 *     j < Lk                                   (and j < seqlens_k[b] in decode)
 *     causal == 0 || j <= pos
 *     window_right < 0 || j <= pos + window_right
 *     window_left  < 0 || j >= pos - window_left
 *   A negative window means "unbounded on that side"; causal = 1 clamps the
 *   right window to 0.  Bounds are inclusive: window_left = window_right = w
 *   is the bidirectional band |i - j| <= w of §4.  When Lq != Lk, query i sits
 *   at key position i + Lk - Lq (bottom-right alignment; the pages only treat
 *   Lq == Lk).  A query row with no allowed key gets O = 0 and LSE = -inf.
 *
 * Layout.  Q is [B, H, Lq, d], K and V are [B, H, Lk, d], O is [B, H, Lq, d],
 * LSE is [B, H, Lq]: dense, row-major, d innermost, no padding.  LSE is the
 * natural-log log-sum-exp including `scale`, in fp32.
 *
 * Ownership and execution.  Every pointer argument named as a device pointer
 * is device memory owned by the caller, valid until the enqueued work is done.
 * Calls enqueue asynchronously on `stream` (a cudaStream_t, NULL = the legacy
 * default stream) and return once enqueued; the library allocates no device
 * memory.  Calls are thread-safe, with one exception: attn_decode_splitkv_noalloc
 * calls that overlap on one device share its scratch and race (see there).
 * Library-owned state: a static decode
 * scratch (attn_decode_splitkv_noalloc), 64 static work counters from which
 * the prefill kernels (attn_fwd*, attn_fwd_varlen*, attn_fwd_fp8*) deal their
 * work items (each launch zeroes one with a 4-byte cudaMemsetAsync on its
 * stream; more than 64 prefill launches in flight at once on one device
 * would share counters), and, from the first attn_fwd_host call on a device,
 * three streams and eight events of that device.
 *
 * Errors.  Every entry point returns a fattn_status; nothing aborts or throws.
 * Argument checks run before any CUDA call, so a rejected call enqueues
 * nothing.  A failed launch returns FATTN_ERR_CUDA.  The prefill kernel bounds
 * every wait; if a wait runs out it records FATTN_ERR_TIMEOUT in a device
 * status word that fattn_device_status() reads back.
 */
#ifndef FATTN_H
#define FATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FATTN_OK = 0,
    FATTN_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad window, scale <= 0 */
    FATTN_ERR_UNSUPPORTED = -2,   /* head dim other than 64 / 128, or sizes beyond int32 indexing */
    FATTN_ERR_MISALIGNED = -3,    /* a tensor base address not 16-byte aligned */
    FATTN_ERR_WORKSPACE = -4,     /* decode workspace null or smaller than attn_decode_workspace_bytes */
    FATTN_ERR_CUDA = -5,          /* a CUDA runtime call or launch failed */
    FATTN_ERR_TIMEOUT = -6,       /* a bounded in-kernel wait expired (see fattn_device_status) */
    FATTN_ERR_NO_DEVICE = -7      /* no usable sm_100 device for the current context */
} fattn_status;

/*
 * attn_fwd -- bf16 prefill forward (tensor cores: tcgen05 MMAs into tensor
 * memory, TMA-staged K/V tiles, warp-specialised pipeline).
 *
 *   q, k, v   device, bf16 [B,H,Lq,d] / [B,H,Lk,d] / [B,H,Lk,d], 16-byte aligned
 *   o         device, bf16 [B,H,Lq,d], 16-byte aligned (written)
 *   lse       device, fp32 [B,H,Lq] (written), or NULL to skip it
 *   B, H, Lq, Lk >= 1;  d in {64, 128};  scale > 0 (finite), usually 1/sqrt(d)
 *   causal, window_left, window_right: the mask above
 *   stream    cudaStream_t
 *
 * Precision: products in bf16 with fp32 accumulation; the probabilities P are
 * rounded to bf16 before the P.V product; O is rounded to bf16 (round to
 * nearest even) after the final division by l.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int Lq, int Lk, int d, float scale,
             int causal, int window_left, int window_right, void* stream);

/*
 * attn_fwd_counted -- attn_fwd that also adds, to *kv_tiles_visited (device,
 * unsigned 64-bit, caller-zeroed), the number of (128-row Q tile, 128-key KV
 * tile) pairs the kernel actually loaded and multiplied.  It is the evidence
 * that out-of-band tiles are skipped (§5.1, §9.1 "blocks computed and KV
 * blocks visited"); the count equals attn_count_blocks(..., 128, 128) visited.
 */
int attn_fwd_counted(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Lq, int Lk, int d, float scale,
                     int causal, int window_left, int window_right,
                     unsigned long long* kv_tiles_visited, void* stream);

/*
 * attn_fwd_varlen -- attn_fwd over a packed batch of sequences of different
 * lengths (the sliding-window FlashAttention prefill page §8.1: requests of
 * different lengths share one launch, each sequence with its own clipped KV
 * range, instead of padding every request to a common length).
 *
 *   q, o          device, bf16 [total_q, H, d]: the tokens of all sequences
 *                 back to back, token-major; 16-byte aligned
 *   k, v          device, bf16 [total_k, H, d]
 *   lse           device, fp32 [H, total_q], or NULL
 *   cu_seqlens_q  device, int32 [num_seqs + 1], non-decreasing: sequence b
 *                 owns query tokens [cu_seqlens_q[b], cu_seqlens_q[b+1])
 *   cu_seqlens_k  device, int32 [num_seqs + 1]: likewise for the keys/values
 *   max_seqlen_q  at least every sequence's query length (query rows beyond
 *                 it are not computed)
 * The mask applies per sequence exactly as in attn_fwd, with Lq and Lk the
 * sequence's own lengths (bottom-right alignment when they differ).  Offsets
 * read from cu_seqlens are clamped into [0, total], so no access leaves the
 * tensors; a sequence with no query token writes nothing.
 *
 * Work order: batches of up to 2048 sequences (and max_seqlen_q <= 262144)
 * are dealt item by item from a counter, longest sequences first, so that the
 * CTAs stay busy to the end and the items in flight share few sequences' K/V
 * in L2.  The counter is one of 64 library-owned counters, taken in turn and
 * zeroed on `stream` before the kernel: up to 64 such launches may run at
 * the same time on different streams (a captured graph keeps the counter of
 * its capture, so one graph must not run concurrently with itself).  Larger
 * batches use a static order.  Results do not depend on the order.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int H,
                    int total_q, int total_k, int max_seqlen_q, int d, float scale,
                    int causal, int window_left, int window_right, void* stream);

/* attn_fwd_varlen that also counts the KV tiles visited (see attn_fwd_counted). */
int attn_fwd_varlen_counted(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs, int H,
                            int total_q, int total_k, int max_seqlen_q, int d, float scale,
                            int causal, int window_left, int window_right,
                            unsigned long long* kv_tiles_visited, void* stream);

/*
 * attn_fwd_host -- attn_fwd on HOST buffers, with the host <-> device copies
 * overlapped with the computation.  The B*H heads are independent problems
 * (§5.3 parallelises over them), so the library takes them in chunks of G
 * heads (about 32 MB of Q, K, V each, G chosen here): the copy of chunk c+1
 * to the device, the kernel on chunk c and the copy of chunk c-1 back to the
 * host run at the same time on three library-owned streams, through two
 * chunk buffers in the caller's workspace.  Results are bit-identical to
 * attn_fwd on the same data.
 *
 *   q, k, v   host, bf16 [B,H,Lq,d] / [B,H,Lk,d] / [B,H,Lk,d]; page-locked
 *             (cudaHostAlloc / pinned) for the copies to overlap -- pageable
 *             memory gives the same results with the copies serialised
 *   o         host, bf16 [B,H,Lq,d] (written)
 *   lse       host, fp32 [B,H,Lq] (written), or NULL to skip it
 *   workspace device, 256-byte aligned, >= attn_fwd_host_workspace_bytes
 *             bytes; caller-owned; not read or written after the call's work
 *             on `stream` has completed
 *   stream    the caller's stream: the work starts after what is already
 *             queued on it, and work queued on it afterwards (for example a
 *             cudaStreamSynchronize) sees o and lse complete
 *   other arguments as attn_fwd
 *
 * Errors: as attn_fwd, plus FATTN_ERR_WORKSPACE for a null, misaligned or
 * short workspace.  Calls from several host threads are serialised inside the
 * library while they enqueue.
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                  int B, int H, int Lq, int Lk, int d, float scale,
                  int causal, int window_left, int window_right,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Device workspace attn_fwd_host needs for these sizes (host only; 0 if the
 * sizes are invalid). */
size_t attn_fwd_host_workspace_bytes(int B, int H, int Lq, int Lk, int d);

/*
 * attn_fwd_f32 -- the same operation on fp32 Q/K/V/O with fp32 arithmetic on
 * the CUDA cores (no tensor-core rounding), for exactness checks.  Arguments
 * as attn_fwd with fp32 tensors; d in {64, 128}; lse nullable.
 */
int attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                 int B, int H, int Lq, int Lk, int d, float scale,
                 int causal, int window_left, int window_right, void* stream);

/*
 * attn_fwd_fp8 -- the prefill forward with 8-bit (e4m3) Q, K and V on the
 * tensor cores' kind::f8f6f4 path ("FlashAttention 深度解析" §4 names
 * FlashAttention-3's FP8 path; this is the plain reading of it on the tiled
 * online softmax): S = Q K^T from the e4m3 codes with fp32 accumulation,
 * x = S * scale * q_descale * k_descale; against a reference row max m that
 * moves only when a tile's max passes it by more than 4 (log2 units; O and l
 * are rescaled when it moves), p = 2^(x*log2e - m + 4) <= 2^8 is rounded to
 * e4m3 (nearest, ties to even) before the P V product; l sums the unrounded
 * p; O = v_descale * acc / l (bf16) and LSE = ln2 (m + log2 l - 4) (fp32,
 * natural log).  Mask as attn_fwd.
 *
 *   q8         device, e4m3 codes [B,H,Lq,128]
 *   k8         device, e4m3 codes [B,H,Lk,128]
 *   vt8        device, e4m3 codes of V transposed, [B,H,128,ld] with
 *              ld = attn_fp8_ld(Lk) (Lk rounded up to 16); columns >= Lk ignored
 *   q_descale, k_descale, v_descale
 *              device, fp32 [B*H]: the value of code c of head (b,h) is
 *              e4m3(c) * descale[b*H + h] (attn_quantize_fp8 writes them)
 *   o, lse     device, bf16 [B,H,Lq,128] / fp32 [B,H,Lq] (lse nullable)
 *   d          must be 128 (FATTN_ERR_UNSUPPORTED otherwise)
 * Tensors 16-byte aligned, descales 4-byte aligned.
 *
 * Accuracy against exact attention on the dequantized inputs: rounding p to
 * e4m3 changes each weight by at most 2^-4 of itself (2^-10 absolute below
 * e4m3's normal range, against l >= 2^4), so a row's O moves by at most
 * about 2^-4 * max|v| plus n * 2^-14 * max|v| for n keys, and, for rows
 * spread over many keys, far less.
 */
int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8,
                 const float* q_descale, const float* k_descale, const float* v_descale,
                 void* o, float* lse, int B, int H, int Lq, int Lk, int d, float scale,
                 int causal, int window_left, int window_right, void* stream);

/* attn_fwd_fp8 that also counts the KV tiles visited (see attn_fwd_counted). */
int attn_fwd_fp8_counted(const void* q8, const void* k8, const void* vt8,
                         const float* q_descale, const float* k_descale, const float* v_descale,
                         void* o, float* lse, int B, int H, int Lq, int Lk, int d, float scale,
                         int causal, int window_left, int window_right,
                         unsigned long long* kv_tiles_visited, void* stream);

/* Row length of attn_fwd_fp8's transposed V: Lk rounded up to a multiple of
 * 16 (0 for Lk < 1).  Host only. */
int attn_fp8_ld(int Lk);

/*
 * attn_quantize_fp8 -- bf16 -> e4m3 with one scale per (batch, head):
 * amax = max |x| over the head, code = e4m3(x * (448 / amax)) with the
 * reciprocal and the product each one fp32 operation rounded to nearest
 * (nearest-even, saturating conversion), descale = amax / 448 (1 for a head
 * of zeros).
 *
 *   x          device, bf16 [B,H,L,d], d in {64, 128}
 *   codes      device, e4m3 [B,H,L,d] (transpose = 0) or [B,H,d,ld] with
 *              ld = attn_fp8_ld(L), columns >= L written as 0 (transpose = 1)
 *   descale    device, fp32 [B*H] (written)
 * B*H <= 65535.  Four kernels (and a memset of descale) are enqueued.
 * x must be finite: a NaN or an infinity in a head leaves that head's codes
 * and descale undefined (no status is recorded), and so the FP8 forward's
 * output for that head.
 */
int attn_quantize_fp8(const void* x, void* codes, float* descale, int B, int H, int L, int d,
                      int transpose, void* stream);

/*
 * attn_decode_splitkv -- split-KV decode for one new query per sequence (flash
 * decoding: "算子与编译器：FlashAttention 与长上下文" §4, short query and long
 * K/V, parallel along the KV axis).  Split s of num_splits covers keys
 * [s*c, min((s+1)*c, seqlens_k[b])) with c = ceil(Lk / num_splits); each
 * split writes a normalised partial output and its LSE, and a merge kernel
 * combines them: lse = logsumexp_s(lse_s), o = sum_s exp(lse_s - lse) o_s.
 *
 *   q          device, bf16 [B,H,1,d]
 *   k_cache    device, bf16 [B,H,Lk,d]
 *   v_cache    device, bf16 [B,H,Lk,d]
 *   o          device, bf16 [B,H,1,d] (written)
 *   lse        device, fp32 [B,H] (written), or NULL
 *   seqlens_k  device, int32 [B] with 0 <= seqlens_k[b] <= Lk, or NULL (all Lk).
 *              A sequence of length 0 gets O = 0 and LSE = -inf.
 *   num_splits 1 .. Lk, or 0 to let the library choose
 *   workspace  device scratch of at least attn_decode_workspace_bytes(B,H,Lk,d,S)
 *              bytes (S = the split count used), 16-byte aligned; its contents
 *              on entry are ignored and on return are unspecified
 */
int attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                        void* o, float* lse, const int* seqlens_k,
                        int B, int H, int Lk, int d, float scale, int num_splits,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged -- attn_decode_splitkv over a paged KV cache ("算子与编译器：
 * FlashAttention 与长上下文" §5, paged KV cache; the sliding-window prefill
 * page §7.2 / §8.2): each sequence's keys sit in fixed-size pages of a shared
 * pool, found through a block table, instead of one contiguous buffer.
 *
 *   q            device, bf16 [B,H,1,d]
 *   k_pages      device, bf16 [num_pages, page_size, H, d] (token-major pages)
 *   v_pages      device, bf16 [num_pages, page_size, H, d]
 *   block_table  device, int32 [B, max_pages]: logical page p of sequence b is
 *                physical page block_table[b*max_pages + p]; indices are
 *                clamped into [0, num_pages), so no access leaves the pool
 *   page_size    a power of two >= 16
 *   seqlens_k    device, int32 [B], required: keys [0, seqlens_k[b]) of
 *                sequence b are attended (clamped to max_pages*page_size)
 *   num_splits, workspace, workspace_bytes, o, lse: as attn_decode_splitkv
 *                with Lk = max_pages * page_size (for the split size and
 *                attn_decode_workspace_bytes)
 */
int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                      const int* block_table, int max_pages, int page_size, int num_pages,
                      void* o, float* lse, const int* seqlens_k, int B, int H, int d,
                      float scale, int num_splits, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Split count attn_decode_splitkv uses for num_splits = 0 (host only). */
int attn_decode_auto_splits(int B, int H, int Lk, int d);

/* Bytes of workspace attn_decode_splitkv needs: B*H*S*(d+1)*4 for S splits
 * (num_splits = 0: the automatic choice for this Lk).  0 on invalid input.
 * Host only. */
size_t attn_decode_workspace_bytes(int B, int H, int Lk, int d, int num_splits);

/*
 * attn_count_blocks -- host-only block accounting of the scheduler (§5.4):
 * for block_q x block_k tiles of one head's Lq x Lk score matrix,
 *   visited = tiles holding at least one allowed pair (exactly the tiles the
 *             kernel loads: the closed-form per-Q-tile KV range of §7.3),
 *   total   = ceil(Lq/block_q) * ceil(Lk/block_k),
 *   partial = visited tiles that need the element mask of §5.2,
 *   pairs   = allowed (query, key) pairs (4*d in-mask FLOPs each).
 * Any output pointer may be NULL.
 */
int attn_count_blocks(int Lq, int Lk, int causal, int window_left, int window_right,
                      int block_q, int block_k, long long* visited, long long* total,
                      long long* partial, long long* pairs);

/*
 * attn_bwd -- bf16 backward of attn_fwd with recomputation: the score tiles
 * are rebuilt from Q, K and the forward's LSE instead of being stored (the
 * sliding-window FlashAttention prefill page §3.3; the bomianfm.com
 * FlashAttention answer, "recomputation" bullet).  The gradients of
 * L = sum(dO * O) through the forward above, with P = exp(scale Q K^T - LSE)
 * on allowed pairs and 0 elsewhere:
 *
 *     dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
 *     dQ = scale dS K,  dK = scale dS^T Q
 *
 *   q, k, v   device, bf16, as passed to attn_fwd
 *   o         device, bf16 [B,H,Lq,d]: attn_fwd's output for these inputs
 *   dout      device, bf16 [B,H,Lq,d]: dL/dO
 *   lse       device, fp32 [B,H,Lq]: attn_fwd's LSE for these inputs (rows
 *             without keys hold -inf and get zero gradient)
 *   dq        device, bf16 [B,H,Lq,d] (written)
 *   dk, dv    device, bf16 [B,H,Lk,d] (written; keys no query sees get 0)
 *   B, H, Lq, Lk, d, scale, causal, window_left, window_right: as attn_fwd
 *   workspace device scratch of at least attn_bwd_workspace_bytes(B,H,Lq,d)
 *             bytes, 16-byte aligned; contents on entry are ignored and on
 *             return unspecified (it holds the fp32 dQ accumulator)
 * Every tensor is 16-byte aligned (lse 4-byte).  Three kernels are enqueued
 * on `stream`: the D_i / LSE pre-pass, the main kernel (one CTA per 128-key
 * tile per head, tensor cores) and the dQ conversion.
 *
 * Precision: products in bf16 with fp32 accumulation; P and dS are rounded to
 * bf16 before they enter a product, dS is formed from the bf16 P; dQ is
 * accumulated in fp32 across KV tiles (atomic adds, so its summation order
 * varies between runs); outputs are rounded to bf16 once.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv,
             int B, int H, int Lq, int Lk, int d, float scale,
             int causal, int window_left, int window_right,
             void* workspace, size_t workspace_bytes, void* stream);

/* attn_bwd that also adds, to *q_tiles_visited (device, unsigned 64-bit,
 * caller-zeroed), the number of (128-key tile, 128-query tile) pairs the main
 * kernel computed; it equals attn_bwd_count_blocks(..., 128, 128) times B*H. */
int attn_bwd_counted(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv,
                     int B, int H, int Lq, int Lk, int d, float scale,
                     int causal, int window_left, int window_right,
                     void* workspace, size_t workspace_bytes,
                     unsigned long long* q_tiles_visited, void* stream);

/* Bytes of workspace attn_bwd needs: B*H*Lq_pad*(d+2)*4 with Lq_pad = Lq
 * rounded up to 128.  0 on invalid input.  Host only. */
size_t attn_bwd_workspace_bytes(int B, int H, int Lq, int d);

/* Host-only: the number of (block_q query tile, block_k key tile) pairs the
 * backward's schedule visits for one head, summed over the key tiles (each
 * key tile walks the query tiles of the band in closed form).  It equals
 * attn_count_blocks's `visited`: both are the tiles with an allowed pair. */
int attn_bwd_count_blocks(int Lq, int Lk, int causal, int window_left, int window_right,
                          int block_q, int block_k, long long* visited);

/* Human-readable name of a fattn_status value. */
const char* fattn_status_string(int status);

/*
 * fattn_device_status -- synchronises `stream`, then returns and clears the
 * device status word of the current device (FATTN_OK, or FATTN_ERR_TIMEOUT if
 * a bounded wait in a prefill or backward kernel expired since the last call).  A debugging
 * aid; it blocks the calling thread.
 */
int fattn_device_status(void* stream);

/*
 * fattn_debug_inject_stall -- test hook for the failure path.  With on != 0
 * the next bf16 prefill kernel launch of any kind, from any thread (attn_fwd,
 * attn_fwd_counted, attn_fwd_varlen*, or one chunk of attn_fwd_host; only that
 * one launch; the flag is process-wide; the FP8 forward ignores it) leaves the
 * first K tile of CTA 0 undelivered: nothing is loaded and nothing faults,
 * the waits that depend on it run out their time limit (about 2 s), and the
 * kernel records FATTN_ERR_TIMEOUT in the device status word, drains its
 * in-flight copies and MMAs, frees its tensor memory and exits.  That launch's
 * O and LSE are garbage; later launches are unaffected.
 */
int fattn_debug_inject_stall(int on);

/*
 * attn_decode_splitkv_noalloc -- attn_decode_splitkv for callers that cannot
 * allocate device memory.  The pages have no counterpart to this entry point;
 * it exists for the library's users, not for the method.
 *
 * Who needs it: code that is handed only its input and output buffers, such
 * as a plugin inside a host application or runtime that owns every device
 * allocation, or a service that runs under a fixed memory budget and must not
 * let a request fail on a workspace allocation; cudaMalloc / cudaFree can also
 * block or synchronise the device, which such callers must avoid.  Those
 * callers still pass q, the caches, o and lse; the split partials go to a
 * scratch array compiled into this library instead of a caller workspace.
 *
 * Arguments as attn_decode_splitkv, without the workspace.  The scratch holds
 * FATTN_DECODE_NOALLOC_SCRATCH_BYTES per device; a call that needs more
 * (B*H*S*(d+1)*4 bytes for S splits, see attn_decode_workspace_bytes) returns
 * FATTN_ERR_WORKSPACE and enqueues nothing.
 *
 * - The scratch is a static device array: every GPU on which the library is
 *   used holds it until the process exits.  This function allocates nothing
 *   and calls no allocating routine.
 * - The first call on a device (with that device current) looks up the
 *   array's device address once and keeps it; make that first call before
 *   any stream capture begins.
 * - All calls share the one array, and each leaves its partials there.  No
 *   part of it needs to start at zero: a call writes every slot it reads.
 *   Calls whose executions overlap on the GPU (different streams, or several
 *   host threads) race on the scratch and give wrong results; order them.
 */
#define FATTN_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
int attn_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                void* o, float* lse, const int* seqlens_k,
                                int B, int H, int Lk, int d, float scale, int num_splits,
                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FATTN_H */
