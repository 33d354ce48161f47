/*
 * attn_b200.h — exact scaled-dot-product attention on one NVIDIA B200 (sm_100a).
 *
 * What is computed
 *   O = softmax(scale * Q K^T + mask) V, row by row, exactly up to floating-point
 *   rounding.  The formula is the one of the polydesk.ai glossary page
 *   "FlashAttention" (section "Le goulot d'étranglement de l'attention standard")
 *   and of ranksignal.fr, "FlashAttention et PagedAttention : à quoi servent-elles ?"
 *   (section "FlashAttention : calculer sur le plan de travail").  The computation is
 *   tiled with an online softmax (running row maximum and sum of exponentials,
 *   rescaled per tile; same glossary page, section "L'idée clé : IO-awareness"), so the
 *   N x N score matrix never reaches device memory.
 *
 * Conventions shared by every entry point
 *   - Pointers marked "device" must point to device memory of the current CUDA device;
 *     the library reads and writes them only from kernels on `stream`.
 *   - Every tensor is dense and row-major (the last dimension is contiguous).
 *   - bf16 tensors are IEEE bfloat16 stored as 16-bit words.
 *   - Device pointers passed to the tensor-memory-accelerator (TMA) loads (q, k, v,
 *     k_pool, v_pool) must be 16-byte aligned; every other device pointer must be
 *     aligned to its element size, and o to 16 bytes.
 *   - The caller owns every buffer.  attn_fwd and attn_fwd_ex allocate nothing;
 *     attn_decode_paged takes all its scratch from the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and never synchronise.  Entry points are thread-safe.
 *   - Errors are returned as attn_status codes; no exception crosses this interface.
 *     Argument checks run on the host before any launch; a call that fails them has
 *     launched nothing and touched no buffer.  Faults found by a kernel (a page id
 *     outside the pool, a pipeline wait that ran past its time limit) are latched in
 *     a per-device status word and reported by attn_get_device_status.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,     /* null pointer, negative size, Hq % Hkv != 0, bad scale ... */
  ATTN_ERR_UNSUPPORTED = 2,     /* a head dimension or page size this build has no kernel for */
  ATTN_ERR_ALIGNMENT = 3,       /* a device pointer breaks the alignment rule above */
  ATTN_ERR_CUDA = 4,            /* a CUDA runtime or driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded pipeline wait gave up */
  ATTN_ERR_BAD_PAGE = 6,        /* a block-table entry in use lies outside [0, num_pages) */
  ATTN_ERR_WORKSPACE = 7,       /* workspace null or smaller than attn_decode_paged_workspace_size */
  ATTN_ERR_TOO_LARGE = 8        /* attn_decode_paged_noalloc: the call needs more scratch than the
                                   library's static scratch holds; attn_fwd_masked: Nk is past
                                   the bound its block-sparse map allows */
} attn_status;

typedef enum attn_dtype {
  ATTN_DTYPE_BF16 = 0,
  ATTN_DTYPE_F32 = 1
} attn_dtype;

/* Version of this interface; bumped whenever a signature changes. */
int attn_abi_version(void);

/*
 * attn_fwd — prefill attention forward.
 *
 * Source: the formula above; causal masking is the triangular mask the
 * patricehuetz.fr page "Flash Attention : pourquoi ton GPU utilise 85% de VRAM"
 * (section "Cas 2 : masques d'attention custom") names as the supported case, and
 * grouped-query heads are those of analyticslegends.ai, "Variantes d'attention"
 * (glossary entry GQA: H_q query heads share H_kv < H_q K/V groups).
 *
 *   q    device, bf16 [B, Hq,  Nq, d]
 *   k    device, bf16 [B, Hkv, Nk, d]
 *   v    device, bf16 [B, Hkv, Nk, d]
 *   o    device, bf16 [B, Hq,  Nq, d]            (written)
 *   lse  device, fp32 [B, Hq,  Nq] or NULL       (written when not NULL)
 *        lse = ln sum_j exp(scale * q.k_j) over the visible keys j.
 *   B, Hq, Hkv, Nq, Nk >= 0 (B, Hq, Hkv >= 1 when Nq > 0);  Hq % Hkv == 0;
 *   query head h reads K/V head h / (Hq / Hkv).
 *   d    head dimension: 64, 128 or 256.
 *   scale > 0 and finite (1/sqrt(d) for the usual softmax temperature).
 *   causal  0: every key visible.  1: key j visible to query i iff
 *           j <= i + (Nk - Nq) (mask aligned to the bottom-right corner).
 *   A query row with no visible key gets O = 0 and lse = -inf.
 *   Nq == 0 is a no-op.  Limits: B*Hq and B*Hkv < 2^31, Nq and Nk < 2^31.
 * Returns ATTN_OK once the kernel is enqueued.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                     int causal, void* stream);

/*
 * attn_fwd_ex — attn_fwd with a choice of output type: the same kernel, whose
 * epilogue writes O as bf16 (o_dtype = ATTN_DTYPE_BF16) or as fp32
 * (ATTN_DTYPE_F32, o is then fp32 [B, Hq, Nq, d]).  The fp32 form exposes the
 * kernel's accumulator before the final bf16 rounding.
 */
attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, int o_dtype,
                        float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                        int causal, void* stream);

/*
 * attn_fwd_masked — attn_fwd_ex with two more masks, applied on top of the causal
 * one.  A CTA skips the key blocks its rows cannot see, so both masks also save work.
 *
 * Sources: ranksignal.fr, "Trois idées reçues à écarter" (a sliding window: each token
 * attends only to the most recent keys); polydesk.ai glossary "FlashAttention", section
 * "FlashAttention et attention block-sparse" (a mask over blocks of tokens says which
 * blocks attend to each other; sliding windows are one such pattern).
 *
 *   causal      0 or 1, as in attn_fwd.
 *   window      0 = no window.  window >= 1 requires causal = 1: query i then sees key
 *               j iff i' - window < j <= i' with i' = i + (Nk - Nq), i.e. the `window`
 *               most recent keys up to its own position, same bottom-right alignment
 *               as the causal mask.  window = 1 keeps the diagonal only.
 *   block_mask  NULL = no block mask, else device, uint8 [ceil(Nq/128), ceil(Nk/128)]
 *               row-major, read-only: entry [bq][bk] nonzero lets queries
 *               128*bq .. 128*bq+127 see keys 128*bk .. 128*bk+127.  One map serves
 *               every batch and head.  It is intersected with the causal mask and
 *               the window.  Bound: ceil(Nk/128) <= 2048 for d <= 128 and <= 1024
 *               for d = 256 (else ATTN_ERR_TOO_LARGE).
 *
 * A row with no visible key gets O = 0 and lse = -inf.  Other arguments, layouts and
 * errors are those of attn_fwd_ex; window < 0, or window > 0 with causal = 0, gives
 * ATTN_ERR_INVALID_ARG.
 */
attn_status attn_fwd_masked(const void* q, const void* k, const void* v, void* o, int o_dtype,
                            float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                            float scale, int causal, int window, const uint8_t* block_mask,
                            void* stream);

/*
 * attn_quantize_fp8 — block quantization of a bf16 tensor to e4m3 (FP8), for attn_fwd_fp8.
 *
 * Source: polydesk.ai glossary "FlashAttention", section on FlashAttention-3 (FP8 inputs
 * with one scale per block).  Format: e4m3 of the OCP 8-bit floating-point format
 * (largest finite value 448).  For each block of `block_rows` consecutive rows of a
 * plane: scale = amax / 448 (1 for an all-zero block), code = x / scale rounded to the
 * nearest e4m3 value (ties to even, saturating at 448, the sign kept when a value rounds
 * to zero); both divisions are fp32 with round-to-nearest.
 *
 *   x        device, bf16 [planes, N, d] (d even), read-only, 4-byte aligned
 *   out      device, e4m3 bytes [planes, N, d] (written), 2-byte aligned
 *   scales   device, fp32 [planes, ceil(N / block_rows)] (written)
 * attn_fwd_fp8 takes Q and K with block_rows = 128 and V with block_rows = N.
 */
attn_status attn_quantize_fp8(const void* x, void* out, float* scales, int planes, int N, int d,
                              int block_rows, void* stream);

/*
 * attn_fwd_fp8 — attn_fwd_ex with FP8 (e4m3) Q, K and V and block scales (d = 128).
 *
 * Computes the attention of the dequantized inputs (code x scale of its block):
 *   q8, k8, v8  device, e4m3 [B, Hq, Nq, 128] / [B, Hkv, Nk, 128], 16-byte aligned
 *   q_scale     device, fp32 [B, Hq, ceil(Nq/128)]: one scale per 128 query rows
 *   k_scale     device, fp32 [B, Hkv, ceil(Nk/128)]: one scale per 128 keys
 *   v_scale     device, fp32 [B, Hkv]: one scale per head
 *   o, lse, causal, scale and the other sizes as in attn_fwd_ex.
 * The probabilities are rounded to e4m3 (after a factor 256, exact in the format, so a
 * row's largest probability is exact) before P V; the log-sum-exp uses their fp32 sum.
 * d other than 128: ATTN_ERR_UNSUPPORTED.
 */
attn_status attn_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                         const void* v8, const float* v_scale, void* o, int o_dtype, float* lse,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         void* stream);

/*
 * attn_bwd_workspace_size — bytes of scratch attn_bwd needs (one fp32 per query row for
 * Delta = rowsum(dO o O)), rounded up to 256.  0 for negative sizes.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Nq);

/*
 * attn_bwd — gradients of attn_fwd with respect to Q, K and V (the backward pass).
 *
 * Source: patricehuetz.fr, "Flash Attention : pourquoi ton GPU utilise 85% de VRAM",
 * section "Ce que fait Flash Attention" (second idea: the forward pass keeps no score
 * matrix; the backward pass recomputes it block by block).  The gradients are those of
 * O = softmax(scale Q K^T + mask) V for the upstream gradient dO, recomputed from Q, K
 * and the forward's log-sum-exp:  dV = P^T dO, dS = P o (dO V^T - Delta),
 * dQ = scale dS K, dK = scale dS^T Q, Delta_i = dO_i . O_i.
 *
 *   q, dout     device, bf16 [B, Hq, Nq, d]
 *   k, v        device, bf16 [B, Hkv, Nk, d]
 *   o, lse      device, the forward's outputs: bf16 O [B, Hq, Nq, d] and fp32 natural
 *               log-sum-exp [B, Hq, Nq] (as written by attn_fwd on the same inputs)
 *   dq          device, fp32 [B, Hq, Nq, d]   (written: cleared by the call, then
 *               accumulated over the key tiles by additions in L2, so nothing else may
 *               write it while the call runs)
 *   dk, dv      device, fp32 [B, Hkv, Nk, d]  (written; for grouped heads the sums over
 *               the Hq/Hkv query heads that share the K/V head)
 *   d           64 or 128 (256: ATTN_ERR_UNSUPPORTED);  causal as in attn_fwd.
 *   workspace   device scratch of at least attn_bwd_workspace_size(B, Hq, Nq) bytes,
 *               16-byte aligned, owned by the caller (ATTN_ERR_WORKSPACE if too small).
 * Alignment: q, k, v, o, dout, dq, dk, dv 16-byte aligned.  A row with no visible key
 * (lse = -inf) gets zero gradient.  Nq = 0 writes dk = dv = 0; Nk = 0 writes dq = 0.
 * Streams: both kernels of the call (Delta, then the gradients) run on `stream`.
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, float* dq, float* dk, float* dv, int B, int Hq, int Hkv,
                     int Nq, int Nk, int d, float scale, int causal, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_workspace_size — bytes of scratch attn_decode_paged needs for
 * these sizes (fp32 partial outputs and partial log-sum-exps of the split-K pass).
 * Returns 0 for sizes attn_decode_paged would reject.
 */
size_t attn_decode_paged_workspace_size(int num_seqs, int Hq, int Hkv, int d,
                                        int max_pages_per_seq, int page_size);

/*
 * attn_decode_paged — one decode step over a paged KV cache.
 *
 * Source: ranksignal.fr, "FlashAttention et PagedAttention : à quoi servent-elles ?",
 * sections "Le cache KV, ce locataire qui grossit" (the new token attends to the kept
 * keys and values of all earlier tokens) and "PagedAttention : ranger par pages plutôt
 * que d'un seul tenant" (the cache lives in fixed-size pages reached through a table;
 * paging changes where data lives, not what is computed).
 *
 *   q            device, bf16 [num_seqs, Hq, d]: one query token per sequence
 *   k_pool       device, bf16 [num_pages, Hkv, page_size, d]
 *   v_pool       device, bf16 [num_pages, Hkv, page_size, d]
 *   block_table  device, int32 [num_seqs, max_pages_per_seq]: entry i of row s is the
 *                pool page holding tokens [i*page_size, (i+1)*page_size) of sequence s;
 *                entries past ceil(seq_lens[s]/page_size) are never read.
 *   seq_lens     device, int32 [num_seqs]: cached tokens per sequence, each in
 *                [0, max_pages_per_seq*page_size]; the query attends to all of them.
 *   o            device, bf16 [num_seqs, Hq, d]   (written)
 *   lse          device, fp32 [num_seqs, Hq] or NULL (written when not NULL)
 *   page_size    16, 32 or 64;  d: 64, 128 or 256;  Hq % Hkv == 0 (query heads of
 *                a KV head are handled 16 at a time).
 *   workspace    device scratch of at least attn_decode_paged_workspace_size(...) bytes,
 *                owned by the caller; its contents need no initialisation and are
 *                overwritten.  Two calls in flight at once need two workspaces.
 *   A sequence of length 0 gets O = 0 and lse = -inf.  A block-table entry in use that
 *   lies outside [0, num_pages) is not read: the kernel skips that page and latches
 *   ATTN_ERR_BAD_PAGE (see attn_get_device_status).
 * Launches two kernels on `stream`: the split-K pass over pages, then the merge of the
 * partial results by their log-sum-exp.
 */
attn_status attn_decode_paged(const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int page_size, void* o, float* lse, int num_seqs, int Hq,
                              int Hkv, int d, int num_pages, int max_pages_per_seq,
                              float scale, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * attn_decode_paged_noalloc — attn_decode_paged for callers that cannot allocate device
 * memory.  (The pages have no counterpart of this entry point: it is a deployment aid.)
 *
 * Some callers may not call cudaMalloc at all: a plugin loaded into a host application
 * that owns every byte of device memory through its own pool, or a serving loop that
 * must never allocate on the request path (cudaMalloc can synchronise the device and
 * its latency is unbounded).  This entry point takes no workspace and allocates
 * nothing: its scratch is a static array of ATTN_DECODE_NOALLOC_MAX_SCRATCH bytes
 * (32 MiB) inside the library, which every GPU that loads the library holds until the
 * process exits.  The caller still passes all inputs and outputs, with the meaning,
 * layout and alignment of attn_decode_paged, and gets the same results.
 *
 *   Returns ATTN_ERR_TOO_LARGE, having launched nothing, when
 *   attn_decode_paged_workspace_size(num_seqs, Hq, Hkv, d, max_pages_per_seq,
 *   page_size) exceeds that size; other argument errors are those of attn_decode_paged.
 *   The first call on a device looks up the device address of the static array (a
 *   cudaGetSymbolAddress on the current device); make that first call before any
 *   stream capture.  The address is kept for the life of the process: after a
 *   cudaDeviceReset, or anything else that destroys the device's primary context, this
 *   entry point must not be called again in the same process (it would pass the old
 *   address to the kernels).  All argument checks run before that lookup, so a call
 *   rejected for its arguments touches no device.
 *   Every call shares the one array and leaves its contents behind; nothing in it has
 *   to start at zero (each call rewrites what it later reads).  Calls that overlap on
 *   the GPU (on different streams, or from different threads) race on the array and
 *   must be serialised by the caller.
 */
#define ATTN_DECODE_NOALLOC_MAX_SCRATCH (32u << 20)
attn_status attn_decode_paged_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* block_table, const int32_t* seq_lens,
                                      int page_size, void* o, float* lse, int num_seqs, int Hq,
                                      int Hkv, int d, int num_pages, int max_pages_per_seq,
                                      float scale, void* stream);

/* Size in bytes of the static scratch of attn_decode_paged_noalloc. */
size_t attn_decode_paged_noalloc_max_scratch(void);

/*
 * attn_get_device_status — synchronises `stream`, then returns and clears the first
 * fault a kernel of this library latched on the current device since the last call
 * (ATTN_OK if none).  ATTN_ERR_CUDA if the synchronisation itself fails.
 */
attn_status attn_get_device_status(void* stream);

/*
 * attn_debug_watchdog — failure-path check, computes nothing.  Launches one CTA on
 * `stream` whose single thread waits on a pipeline barrier that nothing completes;
 * the bounded wait every kernel of this library uses gives up after timeout_ns
 * (1 ns .. 10 s) and latches ATTN_ERR_DEVICE_TIMEOUT, which attn_get_device_status
 * then reports.  The kernel exits normally; the device stays usable.
 */
attn_status attn_debug_watchdog(uint64_t timeout_ns, void* stream);

/*
 * attn_debug_fwd_stall — failure-path check of the prefill kernel (d = 64 or 128).  The
 * same call as attn_fwd_ex, except that CTA `stall_cta` leaves out its K/V ring fill
 * number `stall_fill` (0-based, in the order its producer fills the ring) and every
 * pipeline wait gives up after `timeout_ns` (1 ns .. 10 s) instead of 1 s.  The consumer
 * of the missing tile waits until its limit runs out, latches ATTN_ERR_DEVICE_TIMEOUT
 * and raises its CTA's abort flag; every role then winds down (producers wait, bounded,
 * for their copies in flight, the MMA warp for its MMAs), tensor memory is freed and
 * the kernel exits.  Other CTAs see the latched status at their next wait and wind down
 * the same way.  O and lse are then undefined; attn_get_device_status reports the
 * timeout and the device stays usable.  A stall_fill past the CTA's last fill changes
 * nothing.  ATTN_ERR_UNSUPPORTED for d = 256.  For testing only.
 */
attn_status attn_debug_fwd_stall(const void* q, const void* k, const void* v, void* o,
                                 int o_dtype, float* lse, int B, int Hq, int Hkv, int Nq,
                                 int Nk, int d, float scale, int causal, int stall_cta,
                                 int stall_fill, uint64_t timeout_ns, void* stream);

/*
 * attn_debug_bwd_stall — the same check for the backward pass: attn_bwd, with CTA
 * `stall_cta` of the gradient kernel (one CTA per batch x KV head x 128-key tile)
 * leaving out the Q tile of its step number `stall_step` (a step is one 128-query tile
 * of one head of the group, in the order the CTA walks them) and pipeline waits limited
 * to `timeout_ns` (1 ns .. 10 s).  dq, dk and dv are then undefined;
 * attn_get_device_status reports ATTN_ERR_DEVICE_TIMEOUT.  A stall_step past the CTA's
 * last step changes nothing.  For testing only.
 */
attn_status attn_debug_bwd_stall(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, const float* lse, float* dq, float* dk,
                                 float* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                 float scale, int causal, void* workspace,
                                 size_t workspace_bytes, int stall_cta, int stall_step,
                                 uint64_t timeout_ns, void* stream);

/*
 * attn_debug_decode_stall — the same check for the paged decode: attn_decode_paged, with
 * CTA `stall_cta` of the split kernel leaving out its K/V piece number `stall_piece`
 * (16 tokens of K and V, in the order its producer gathers them) and pipeline waits
 * limited to `timeout_ns` (1 ns .. 10 s).  O and lse are then undefined;
 * attn_get_device_status reports ATTN_ERR_DEVICE_TIMEOUT.  For testing only.
 */
attn_status attn_debug_decode_stall(const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* block_table, const int32_t* seq_lens,
                                    int page_size, void* o, float* lse, int num_seqs, int Hq,
                                    int Hkv, int d, int num_pages, int max_pages_per_seq,
                                    float scale, void* workspace, size_t workspace_bytes,
                                    int stall_cta, int stall_piece, uint64_t timeout_ns,
                                    void* stream);

/*
 * attn_debug_exp2 — evaluates, for i < n, y[i] = 2^x[i] with the polynomial exponential
 * the prefill kernel runs on the FMA pipe for part of its probabilities (range
 * reduction x = n + f, degree-3 minimax polynomial for 2^f).  x and y are device fp32
 * arrays of n elements; inputs below -125 are clamped to -125.  For testing.
 */
attn_status attn_debug_exp2(const float* x, float* y, int n, void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char* attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
