// internal.h -- launchers shared between the kernel files and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/exattn.h"

namespace exattn {

// window > 0: sliding window; slopes (device, one per query head) or nullptr: ALiBi.
attn_status_t launch_prefill_bf16(const void *q, const void *k, const void *v, void *o, float *lse,
                                  int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                                  int window, const float *slopes, cudaStream_t stream,
                                  unsigned *status);

// Chunked prefill over a paged cache (causal from the end of each sequence).
attn_status_t launch_prefill_paged(const void *q, const void *k_pages, const void *v_pages,
                                   const int *block_table, const int *seq_lens, const int *cu_q,
                                   void *o, float *lse, int S, int Hq, int Hkv, int T, int max_q,
                                   int d, int max_blocks, int num_pages, float scale, int window,
                                   const float *slopes, cudaStream_t stream, unsigned *status);

attn_status_t launch_prefill_f32(const float *q, const float *k, const float *v, float *o,
                                 float *lse, int B, int Hq, int Hkv, int N, int d, float scale,
                                 int causal, int window, const float *slopes,
                                 cudaStream_t stream);

// Number of key chunks (pages per chunk fixed) a sequence of max_blocks pages
// can be split into, and the workspace layout that follows from it.  The
// workspace starts with a 256-byte block whose first word is the call's
// ATTN_DEV_* status (read by attn_decode_read_status), then the chunk partials.
constexpr size_t kDecodeStatusBytes = 256;
struct DecodeWs {
  unsigned *status;  // the call's status word (cleared by the split kernel)
  float *o_part;     // [S][Hq][nsplit][d] normalised chunk outputs
  float *l2_part;    // [S][Hq][nsplit] chunk log2-sum-exps (tagged NaN: failed chunk)
};
int decode_max_splits(int max_blocks);
size_t decode_workspace_bytes(int S, int Hq, int d, int max_blocks);
DecodeWs decode_ws_layout(void *workspace, int S, int Hq, int d, int max_blocks);

// dev_status: nullptr, or a second word (the per-device one) that also gets
// the call's bits.
attn_status_t launch_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                  const int *block_table, const int *seq_lens, void *o, float *lse,
                                  int S, int Hq, int Hkv, int d, int max_blocks, int num_pages,
                                  float scale, void *workspace, cudaStream_t stream,
                                  unsigned *dev_status);

// Merge the chunk partials of a split decode into O (bf16) and L; chunks hold
// pages_per_split pages.  Failed chunks' bits go to ws.status (and dev_status).
attn_status_t launch_decode_combine(const DecodeWs &ws, const int *seq_lens, void *o, float *lse,
                                    int S, int Hq, int d, int max_blocks, int nsplit,
                                    int pages_per_split, cudaStream_t stream,
                                    unsigned *dev_status);

// The same decode over 8-bit pages (kv_format ATTN_KV_E4M3 or ATTN_KV_INT8) with
// per-(page, K/V head) fp32 scales; same workspace.
attn_status_t launch_decode_paged_q8(const void *q, const void *k_pages, const void *v_pages,
                                     const float *k_scales, const float *v_scales, int kv_format,
                                     const int *block_table, const int *seq_lens, void *o,
                                     float *lse, int S, int Hq, int Hkv, int d, int max_blocks,
                                     int num_pages, float scale, void *workspace,
                                     cudaStream_t stream);

// Backward: workspace (L*log2e and rowsum(dO*O) per query row, padded to whole
// 128-row tiles) and the three-kernel launch.
size_t bwd_workspace_bytes(int B, int Hq, int N);
attn_status_t launch_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dout, void *dq, void *dk, void *dv,
                              int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                              int window, const float *slopes, void *workspace,
                              cudaStream_t stream, unsigned *status);

// cuTensorMapEncodeTiled, or nullptr if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// Device address of the fixed scratch array used by attn_decode_paged_noalloc
// (ATTN_DECODE_NOALLOC_SCRATCH_BYTES bytes) on the current device.
attn_status_t noalloc_scratch_address(void **addr);

}  // namespace exattn
