/*
 * exattn.h -- C ABI of the exact, IO-aware attention library (libexattn.so).
 *
 * The library computes exact scaled-dot-product attention on one NVIDIA B200
 * (sm_100a):
 *
 *   O = softmax(scale * Q K^T [+ causal mask]) V,   L = logsumexp of each row
 *
 * tile by tile with an online softmax, never writing the N x N score matrix to
 * memory ("Phase 08 -- Inference Optimization at Depth", Concepts: standard
 * attention memory, FlashAttention tiling, online softmax, logsumexp L for the
 * backward pass; Lab 01 steps 2 and 4), for grouped-/multi-query heads
 * (screna.ai interview page, MHA/MQA/GQA answer) and as a single-token decode
 * over a paged KV cache (Phase 08 page, Concepts: KV cache and paged attention;
 * Lab 03 step 4: pages reached through an indirection table).
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers to dense, row-major (C order)
 *    arrays owned by the caller.  The library never allocates or frees device
 *    memory; work is enqueued on `stream` (0 = legacy default stream) and the
 *    call returns before it finishes.  `stream` must belong to the current
 *    device, and the tensors must live on it.  Only the two status reads below
 *    wait for anything: attn_decode_read_status for its own 4-byte copy,
 *    attn_device_status for the stream it is given.
 *  - Tensor data (q, k, v, o, the page pools, dO and the gradients) and
 *    workspaces must be 16-byte aligned; int32 and float32 vectors (lse,
 *    block_table, seq_lens, cu_q, the 8-bit scales, ALiBi slopes) 4-byte
 *    aligned.  A null or misaligned pointer gives ATTN_ERR_INVALID_ARG.
 *  - Errors are reported only through the return value.  A call that returns
 *    ATTN_ERR_INVALID_ARG or ATTN_ERR_UNSUPPORTED has written none of its
 *    outputs; after ATTN_ERR_CUDA (a failed launch or runtime call) the
 *    outputs are undefined.  No call aborts or traps.
 *  - Device-side conditions that the host cannot see in advance (a block-table
 *    entry outside the page pool, a bounded wait that ran out) set ATTN_DEV_*
 *    bits in a status word.  A decode that takes a workspace (attn_decode_paged,
 *    attn_decode_paged_q8) owns the word at the start of that workspace: each
 *    such call clears it and reports only its own conditions there, read with
 *    attn_decode_read_status().  Every other call ORs its bits into one word
 *    per device, read (and cleared) with attn_device_status().
 *  - The library looks up a few device addresses once per device and keeps
 *    them; it does not support cudaDeviceReset (or a reset of the primary
 *    context) while it is loaded.
 *  - Every compute call may be captured into a CUDA graph once the same
 *    entry point has run eagerly on the device (its one-time setup happens
 *    then); the two status reads may not.
 *  - `causal` means key j is visible to query i iff j <= i (queries and keys
 *    share positions 0..N-1).
 *  - L is the natural logarithm of sum_j exp(scale * q_i . k_j) over the
 *    visible keys, stored as float32.
 *  - Query head h reads key/value head h / (Hq / Hkv): consecutive groups of
 *    Hq/Hkv query heads share one K/V head (Hkv == Hq is multi-head,
 *    Hkv == 1 is multi-query attention).
 */
#ifndef EXATTN_H_
#define EXATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EXATTN_API __attribute__((visibility("default")))
#else
#define EXATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Stream handle: the CUDA runtime's cudaStream_t (a CUstream_st pointer). */
typedef struct CUstream_st *attn_stream_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, Hq % Hkv != 0, bad scale */
    ATTN_ERR_UNSUPPORTED = 2,   /* head dim / page size not built, or no sm_100 device */
    ATTN_ERR_CUDA = 3           /* a CUDA runtime or driver call failed */
} attn_status_t;

/* Status bits (attn_decode_read_status, attn_device_status). */
#define ATTN_DEV_BAD_PAGE 0x1u  /* a decode sequence referenced a page outside the pool or
                                   had a length outside [0, max_blocks*page_size]; its
                                   outputs are NaN */
#define ATTN_DEV_TIMEOUT 0x2u   /* a bounded wait inside a kernel expired; the kernel
                                   returned early and the outputs it owed are undefined
                                   (a decode writes NaN for the sequences concerned) */
#define ATTN_DEV_LAYOUT 0x4u    /* a backward kernel found its dynamic shared memory not
                                   1024-byte aligned and returned at once; the gradients
                                   are undefined */

/*
 * attn_fwd -- bf16 prefill, forward only.  Lab 01 steps 2 and 4 of the Phase 08
 * page: Q is split into row tiles; for each, the kernel walks the K/V column
 * tiles with a running max and sum, rescales the accumulator, and writes O and
 * L once.  With causal != 0, tiles wholly above the diagonal are skipped and
 * only diagonal tiles are masked (Concepts: causal masking in FlashAttention).
 *
 *   q    [B, Hq,  N, d] bf16        k, v [B, Hkv, N, d] bf16
 *   o    [B, Hq,  N, d] bf16 (out)  lse  [B, Hq, N] float32 (out)
 *   d in {64, 128}; N >= 1; B, Hq, Hkv >= 1; Hq % Hkv == 0;
 *   scale finite and > 0 (the workloads use 1/sqrt(d)).
 * Accumulation is float32; O is rounded to nearest-even bf16.
 * Returns ATTN_ERR_UNSUPPORTED if the current device is not sm_100.
 */
EXATTN_API attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                       attn_stream_t stream);

/*
 * attn_fwd_f32 -- the same operation on float32 tensors (o is float32), with
 * float32 arithmetic throughout; the correctness path for the fp32 workload
 * (Lab 01 step 3: match standard attention within 1e-4).  d in {64, 128}.
 */
EXATTN_API attn_status_t attn_fwd_f32(const float *q, const float *k, const float *v, float *o,
                           float *lse, int B, int Hq, int Hkv, int N, int d, float scale,
                           int causal, attn_stream_t stream);

/*
 * attn_fwd_ext / attn_fwd_f32_ext -- attn_fwd / attn_fwd_f32 with the two
 * variants the Phase 08 page lists among the Lab 01 extensions: sliding-window
 * attention (as in Mistral) and ALiBi bias.  The page only names them; this
 * library reads them plainly:
 *   window > 0      key j is visible to query i only if i - j < window, on top
 *                   of causal masking (window > 0 requires causal != 0);
 *                   window == 0 means no window.
 *   alibi_slopes    NULL, or a DEVICE array of Hq floats a_h: the bias
 *                   a_h * (j - i) is added to scale * q_i . k_j before the
 *                   softmax (a_h >= 0 makes older keys weigh less); L includes it.
 * Other arguments, layouts and errors as for attn_fwd / attn_fwd_f32;
 * window < 0, a window without causal, or a misaligned slopes pointer give
 * ATTN_ERR_INVALID_ARG.
 */
EXATTN_API attn_status_t attn_fwd_ext(const void *q, const void *k, const void *v, void *o,
                                      float *lse, int B, int Hq, int Hkv, int N, int d,
                                      float scale, int causal, int window,
                                      const float *alibi_slopes, attn_stream_t stream);
EXATTN_API attn_status_t attn_fwd_f32_ext(const float *q, const float *k, const float *v,
                                          float *o, float *lse, int B, int Hq, int Hkv, int N,
                                          int d, float scale, int causal, int window,
                                          const float *alibi_slopes, attn_stream_t stream);

/*
 * attn_prefill_paged -- chunked prefill over the paged KV cache (Phase 08
 * page, Concepts: chunked prefill splits a long prompt over several steps so
 * it does not block decoding; Lab 03 Extensions: add chunked prefill; paged
 * attention as for attn_decode_paged).  Sequence s holds seq_lens[s] tokens in
 * its pages; the current chunk is its last qlen_s = cu_q[s+1] - cu_q[s] tokens,
 * whose K/V the caller has already written to the cache.  Chunk query t sits
 * at position ctx_s + t (ctx_s = seq_lens[s] - qlen_s) and attends causally to
 * keys 0 .. ctx_s + t (the causal diagonal aligned to the end of the keys);
 * window > 0 additionally keeps only keys with ctx_s + t - j < window, and
 * alibi_slopes add a_h * (j - (ctx_s + t)) to the scores, as for attn_fwd_ext.
 *
 *   q            [T, Hq, d] bf16, token-major: rows cu_q[s] .. cu_q[s+1]-1 are
 *                sequence s's chunk (T = cu_q[S])
 *   k_pages, v_pages, block_table, seq_lens   as for attn_decode_paged
 *   cu_q         [S+1] int32, non-decreasing, cu_q[0] = 0, cu_q[S] = T
 *   max_q        an upper bound of every qlen_s (sizes the grid)
 *   o            [T, Hq, d] bf16 (out)      lse [T, Hq] float32 (out)
 * d in {64, 128}; page_size == 16.  A sequence whose lengths are inconsistent
 * (qlen_s < 0, qlen_s > seq_lens[s], qlen_s > max_q, cu_q[s+1] > T, or
 * seq_lens[s] > max_blocks * 16) is skipped and sets ATTN_DEV_BAD_PAGE; one
 * whose block table names a page outside [0, num_pages) gets NaN rows and sets
 * it; no out-of-range address is dereferenced.  T == 0 is a no-op.
 */
EXATTN_API attn_status_t attn_prefill_paged(const void *q, const void *k_pages,
                                            const void *v_pages, const int32_t *block_table,
                                            const int32_t *seq_lens, const int32_t *cu_q,
                                            void *o, float *lse, int S, int Hq, int Hkv, int T,
                                            int max_q, int d, int page_size, int max_blocks,
                                            int num_pages, float scale, int window,
                                            const float *alibi_slopes, attn_stream_t stream);

/*
 * attn_bwd -- gradients of the bf16 attention above (Phase 08 page, Concepts:
 * the FlashAttention backward needs only the output O and the logsumexp L;
 * Lab 01 step 6 and Extensions: the backward pass).  For the scalar
 * sum(dO * O), with P = softmax(scale * Q K^T [mask] [+ALiBi]) recomputed tile by
 * tile from L (never stored):
 *   D = rowsum(dO * O), dP = dO V^T, dS = P * (dP - D),
 *   dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K.
 * With grouped heads, dK and dV of a K/V head sum over its query heads.
 *
 *   q, o, dout   [B, Hq, N, d] bf16 (o and lse as attn_fwd / attn_fwd_ext
 *                wrote them for the same q, k, v and options)
 *   k, v         [B, Hkv, N, d] bf16
 *   lse          [B, Hq, N] float32
 *   dq           [B, Hq, N, d] bf16 (out)     dk, dv  [B, Hkv, N, d] bf16 (out)
 *   causal, window, alibi_slopes   as for attn_fwd_ext
 *   workspace    device scratch of at least attn_bwd_workspace_bytes(B, Hq, N)
 *                bytes, owned by the caller; no initialisation needed.
 * The result is deterministic: no atomics, every output element is written by
 * one thread.  Errors as for attn_fwd_ext, plus ATTN_ERR_INVALID_ARG for a
 * workspace that is too small.
 */
EXATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int N);
EXATTN_API attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *o,
                                  const float *lse, const void *dout, void *dq, void *dk,
                                  void *dv, int B, int Hq, int Hkv, int N, int d, float scale,
                                  int causal, int window, const float *alibi_slopes,
                                  void *workspace, size_t workspace_bytes,
                                  attn_stream_t stream);

/*
 * attn_decode_workspace_bytes -- bytes of device workspace attn_decode_paged
 * (and attn_decode_paged_q8) needs for S sequences, Hq query heads, head dim d
 * and at most max_blocks pages per sequence.  The workspace starts with a
 * 256-byte block whose first 32-bit word is the call's status word (see
 * attn_decode_read_status); the chunk partials follow.  Returns 0 for invalid
 * sizes.  The pages do not say how a decode is parallelised, so this workspace
 * has no counterpart there: the split over key chunks is this library's choice.
 */
EXATTN_API size_t attn_decode_workspace_bytes(int S, int Hq, int d, int max_blocks, int page_size);

/*
 * attn_decode_paged -- one query token per sequence against its paged KV cache
 * (Phase 08 page, Concepts: KV cache, paged attention; Lab 03 step 4).  Token t
 * of sequence s lives in page block_table[s, t / page_size] at slot
 * t % page_size; each sequence sees all of its seq_lens[s] tokens (the query is
 * the newest token, so no mask applies).  The key range of a sequence is split
 * into fixed-size chunks processed in parallel; a second kernel merges the
 * chunks' partial outputs with their logsumexp weights.
 *
 *   q            [S, Hq, d] bf16
 *   k_pages      [num_pages, Hkv, page_size, d] bf16   v_pages likewise
 *   block_table  [S, max_blocks] int32 (entries past a sequence's last page are not read)
 *   seq_lens     [S] int32, each in [0, max_blocks * page_size]
 *   o            [S, Hq, d] bf16 (out)      lse [S, Hq] float32 (out)
 *   workspace    device scratch of at least attn_decode_workspace_bytes(...) bytes,
 *                owned by the caller; its contents need no initialisation.  It
 *                holds the call's status word until the next call that uses it.
 * d in {64, 128}; page_size == 16; Hq / Hkv in {1, 2, 4, 8, 16, 32, ...} (any divisor).
 * A sequence of length 0 gets O = 0 and L = -inf.  A sequence with a page id
 * outside [0, num_pages) or an out-of-range length gets NaN outputs and sets
 * ATTN_DEV_BAD_PAGE in the workspace's status word; no out-of-range address is
 * ever dereferenced.  Calls on different workspaces never share a status word,
 * so concurrent decodes on several streams each report only their own faults.
 */
EXATTN_API attn_status_t attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                const int32_t *block_table, const int32_t *seq_lens,
                                void *o, float *lse,
                                int S, int Hq, int Hkv, int d, int page_size,
                                int max_blocks, int num_pages, float scale,
                                void *workspace, size_t workspace_bytes,
                                attn_stream_t stream);

/*
 * attn_decode_paged_q8 -- attn_decode_paged over an 8-bit KV cache.  The
 * KV-cache quantisation answer of the screna.ai interview page: 8-bit storage
 * halves the cache against 16 bits, INT8 is the safe default and NVIDIA's FP8
 * the hardware format, and group-wise scales keep accuracy.  Here the group is
 * one (page, K/V head) slice: the element the attention uses is
 *   k = k_scales[p * Hkv + g] * code(k_pages[p, g, slot, c])     (v likewise)
 * with code() the E4M3 value (kv_format ATTN_KV_E4M3: sign, 4 exponent bits of
 * bias 7, 3 mantissa bits, S.1111.111 = NaN, no infinities) or the two's-
 * complement integer (ATTN_KV_INT8).  Everything else -- block table, lengths,
 * outputs, workspace (attn_decode_workspace_bytes), bad-page handling -- is as
 * for attn_decode_paged.
 *
 *   q                  [S, Hq, d] bf16
 *   k_pages, v_pages   [num_pages, Hkv, page_size, d] one byte per element,
 *                      16-byte aligned
 *   k_scales, v_scales [num_pages, Hkv] float32 (device); only the entries of
 *                      pages a sequence reaches are read
 * num_pages * Hkv < 2^31.  The query is rounded to f16 inside the kernel after
 * a per-head power-of-two normalisation and P is rounded to f16 before the P.V
 * product; scores, sums and outputs accumulate in float32.
 */
#define ATTN_KV_E4M3 0
#define ATTN_KV_INT8 1
EXATTN_API attn_status_t attn_decode_paged_q8(const void *q, const void *k_pages,
                                              const void *v_pages, const float *k_scales,
                                              const float *v_scales, int kv_format,
                                              const int32_t *block_table,
                                              const int32_t *seq_lens, void *o, float *lse,
                                              int S, int Hq, int Hkv, int d, int page_size,
                                              int max_blocks, int num_pages, float scale,
                                              void *workspace, size_t workspace_bytes,
                                              attn_stream_t stream);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged for callers that cannot
 * allocate device memory.  The pages have no counterpart to this entry point; it
 * exists for how the library is used, not for the method.
 *
 * Some callers may not call cudaMalloc at all: a plugin inside a host program
 * that owns every byte of device memory through its own pool, or a decode loop
 * that must never wait on the allocator (cudaMalloc and cudaFree can block until
 * the device is idle).  They still pass q, the page pools, block_table,
 * seq_lens, o and lse exactly as for attn_decode_paged, but no workspace: the
 * chunk partials go to a fixed scratch array of ATTN_DECODE_NOALLOC_SCRATCH_BYTES
 * that lives in the library's device memory.  This call allocates nothing and
 * frees nothing.
 *
 * - The scratch exists once per GPU that loads the library and stays allocated
 *   until the process exits.
 * - The first call on a device looks up the scratch's device address (with that
 *   device current) and caches it; make that first call before any stream
 *   capture.  `stream` must belong to the current device.
 * - The scratch's status word is shared too, so this call reports a bad page id
 *   or length (ATTN_DEV_BAD_PAGE) in the per-device word of attn_device_status,
 *   not through attn_decode_read_status.
 * - All calls on a device share the one array and leave their partials in it.
 *   Calls whose kernels overlap on the GPU (different streams, no ordering
 *   between them) race on it; order them on one stream or use attn_decode_paged
 *   with separate workspaces.  Nothing in the scratch needs to start at zero:
 *   each call writes every partial it later reads.
 * - A request whose workspace, as attn_decode_workspace_bytes(S, Hq, d,
 *   max_blocks, page_size) reports it, exceeds ATTN_DECODE_NOALLOC_SCRATCH_BYTES
 *   returns ATTN_ERR_INVALID_ARG without launching anything.  (64 sequences x
 *   32 heads x d=128 with up to 512 pages of 16 tokens need 16.9 MB.)
 * Results are identical to attn_decode_paged's for the same arguments.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
EXATTN_API attn_status_t attn_decode_paged_noalloc(const void *q, const void *k_pages,
                                                   const void *v_pages,
                                                   const int32_t *block_table,
                                                   const int32_t *seq_lens, void *o, float *lse,
                                                   int S, int Hq, int Hkv, int d, int page_size,
                                                   int max_blocks, int num_pages, float scale,
                                                   attn_stream_t stream);

/*
 * attn_decode_read_status -- the ATTN_DEV_* bits of the last attn_decode_paged
 * or attn_decode_paged_q8 call that used `workspace` (0: no sequence failed).
 * The paged decode's only device-side failure is the Lab 03 step 4 one: a
 * block-table entry (the indirection table) naming a page outside the pool, or
 * a length the table cannot hold (ATTN_DEV_BAD_PAGE); a wait that ran out gives
 * ATTN_DEV_TIMEOUT.  Synchronises nothing: the caller first synchronises the
 * stream the decode ran on (or waits on an event recorded after it); the call
 * then copies the one word to the host through a stream of its own, waiting only
 * for that copy.  `workspace` is the device pointer given to the decode.
 * ATTN_ERR_INVALID_ARG for a null or misaligned workspace or a null dev_status.
 */
EXATTN_API attn_status_t attn_decode_read_status(const void *workspace, unsigned *dev_status);

/*
 * attn_device_status -- read (and, if clear != 0, reset) the status word of the
 * current device, which every call other than the workspace decodes reports
 * into.  Waits for the work enqueued on `stream` so far, and only for that:
 * pass the stream the calls of interest ran on (kernels still running on other
 * streams may set bits later).  Library plumbing with no counterpart on the
 * pages; the conditions it reports are those listed with the ATTN_DEV_* bits.
 * The read and the clear are two steps, so a bit that a kernel on another
 * stream sets between them is lost: clear only while no other stream runs
 * library work on the device.  Not for use inside stream capture.
 */
EXATTN_API attn_status_t attn_device_status(unsigned *status, int clear, attn_stream_t stream);

/* attn_status_string -- a static, human-readable name for a status code
 * (library plumbing; no counterpart on the pages). */
EXATTN_API const char *attn_status_string(attn_status_t status);

/* attn_version -- library version string (no counterpart on the pages). */
EXATTN_API const char *attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXATTN_H_ */
