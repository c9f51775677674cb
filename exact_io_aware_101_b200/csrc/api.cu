// api.cu -- the C ABI declared in include/exattn.h: argument checks, device
// checks and the status words, then a launch of the right kernel.  Nothing here
// allocates or frees; only the two status reads wait, each for the one copy (or
// the one stream) it reads through.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace exattn {
namespace {

// Status bits raised by the prefill, chunked-prefill and backward kernels (and
// the workspace-free decode) on this device (ATTN_DEV_*).  The decodes that take
// a workspace report into a word of that workspace instead.
__device__ unsigned g_status = 0;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned *g_status_ptr[kMaxDevices] = {};
int g_is_sm100[kMaxDevices] = {};  // 0 unknown, 1 yes, -1 no

// Device address of this device's status word, looked up once per device
// (a __device__ variable's address is only meaningful on the device side).
// The cache assumes the device is not reset while the library is loaded.
bool device_state(unsigned **status, bool *sm100) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return false;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return false;
    g_is_sm100[dev] = (major == 10 && minor == 0) ? 1 : -1;
    g_status_ptr[dev] = static_cast<unsigned *>(p);
  }
  *status = g_status_ptr[dev];
  *sm100 = g_is_sm100[dev] == 1;
  return true;
}

bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool good_scale(float s) { return isfinite(s) && s > 0.f; }

attn_status_t check_prefill(const void *q, const void *k, const void *v, const void *o,
                            const void *lse, int B, int Hq, int Hkv, int N, int d, float scale) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse))
    return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || Hq % Hkv != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!good_scale(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq * N * d >= (1LL << 40)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

}  // namespace
}  // namespace exattn

using namespace exattn;

extern "C" {

attn_status_t attn_fwd_ext(const void *q, const void *k, const void *v, void *o, float *lse,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           int window, const float *alibi_slopes, attn_stream_t stream) {
  attn_status_t st = check_prefill(q, k, v, o, lse, B, Hq, Hkv, N, d, scale);
  if (st != ATTN_OK) return st;
  if (window < 0 || (window > 0 && !causal) || (alibi_slopes && !aligned4(alibi_slopes)))
    return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  return launch_prefill_bf16(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window,
                             alibi_slopes, reinterpret_cast<cudaStream_t>(stream), status);
}

attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                       int Hq, int Hkv, int N, int d, float scale, int causal,
                       attn_stream_t stream) {
  return attn_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, 0, nullptr, stream);
}

attn_status_t attn_fwd_f32_ext(const float *q, const float *k, const float *v, float *o,
                               float *lse, int B, int Hq, int Hkv, int N, int d, float scale,
                               int causal, int window, const float *alibi_slopes,
                               attn_stream_t stream) {
  attn_status_t st = check_prefill(q, k, v, o, lse, B, Hq, Hkv, N, d, scale);
  if (st != ATTN_OK) return st;
  if (window < 0 || (window > 0 && !causal) || (alibi_slopes && !aligned4(alibi_slopes)))
    return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  return launch_prefill_f32(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window,
                            alibi_slopes, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           attn_stream_t stream) {
  return attn_fwd_f32_ext(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, 0, nullptr, stream);
}

attn_status_t attn_prefill_paged(const void *q, const void *k_pages, const void *v_pages,
                                 const int32_t *block_table, const int32_t *seq_lens,
                                 const int32_t *cu_q, void *o, float *lse, int S, int Hq, int Hkv,
                                 int T, int max_q, int d, int page_size, int max_blocks,
                                 int num_pages, float scale, int window,
                                 const float *alibi_slopes, attn_stream_t stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned4(block_table) ||
      !aligned4(seq_lens) || !aligned4(cu_q) || !aligned16(o) || !aligned4(lse) ||
      (alibi_slopes && !aligned4(alibi_slopes)))
    return ATTN_ERR_INVALID_ARG;
  if (S <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || T < 0 || max_q < 0 || d <= 0 ||
      page_size <= 0 || max_blocks <= 0 || num_pages <= 0 || window < 0 || !good_scale(scale))
    return ATTN_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * page_size > (1LL << 30) ||
      static_cast<long long>(num_pages) * Hkv >= (1LL << 31) ||
      static_cast<long long>(T) * Hq * d >= (1LL << 40))
    return ATTN_ERR_INVALID_ARG;
  if (T == 0 || max_q == 0) return ATTN_OK;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  return launch_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, cu_q, o, lse, S, Hq, Hkv,
                              T, max_q, d, max_blocks, num_pages, scale, window, alibi_slopes,
                              reinterpret_cast<cudaStream_t>(stream), status);
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int N) {
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  return bwd_workspace_bytes(B, Hq, N);
}

attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *o,
                       const float *lse, const void *dout, void *dq, void *dk, void *dv, int B,
                       int Hq, int Hkv, int N, int d, float scale, int causal, int window,
                       const float *alibi_slopes, void *workspace, size_t workspace_bytes,
                       attn_stream_t stream) {
  attn_status_t st = check_prefill(q, k, v, o, lse, B, Hq, Hkv, N, d, scale);
  if (st != ATTN_OK) return st;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal) || (alibi_slopes && !aligned4(alibi_slopes)))
    return ATTN_ERR_INVALID_ARG;
  if (N <= 0) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < bwd_workspace_bytes(B, Hq, N)) return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  return launch_attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal,
                         window, alibi_slopes, workspace, reinterpret_cast<cudaStream_t>(stream),
                         status);
}

size_t attn_decode_workspace_bytes(int S, int Hq, int d, int max_blocks, int page_size) {
  if (S <= 0 || Hq <= 0 || max_blocks <= 0 || page_size != 16 || (d != 64 && d != 128)) return 0;
  return decode_workspace_bytes(S, Hq, d, max_blocks);
}

attn_status_t attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                const int32_t *block_table, const int32_t *seq_lens, void *o,
                                float *lse, int S, int Hq, int Hkv, int d, int page_size,
                                int max_blocks, int num_pages, float scale, void *workspace,
                                size_t workspace_bytes, attn_stream_t stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned4(block_table) ||
      !aligned4(seq_lens) || !aligned16(o) || !aligned4(lse) || !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  if (S <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || page_size <= 0 ||
      max_blocks <= 0 || num_pages <= 0 || !good_scale(scale))
    return ATTN_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * page_size > (1LL << 30)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < decode_workspace_bytes(S, Hq, d, max_blocks)) return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  // The call's status goes to its own workspace word only.
  return launch_decode_paged(q, k_pages, v_pages, block_table, seq_lens, o, lse, S, Hq, Hkv, d,
                             max_blocks, num_pages, scale, workspace,
                             reinterpret_cast<cudaStream_t>(stream), nullptr);
}

attn_status_t attn_decode_paged_q8(const void *q, const void *k_pages, const void *v_pages,
                                   const float *k_scales, const float *v_scales, int kv_format,
                                   const int32_t *block_table, const int32_t *seq_lens, void *o,
                                   float *lse, int S, int Hq, int Hkv, int d, int page_size,
                                   int max_blocks, int num_pages, float scale, void *workspace,
                                   size_t workspace_bytes, attn_stream_t stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned4(k_scales) ||
      !aligned4(v_scales) || !aligned4(block_table) || !aligned4(seq_lens) || !aligned16(o) ||
      !aligned4(lse) || !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  if (S <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || page_size <= 0 ||
      max_blocks <= 0 || num_pages <= 0 || !good_scale(scale) ||
      (kv_format != ATTN_KV_E4M3 && kv_format != ATTN_KV_INT8))
    return ATTN_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * page_size > (1LL << 30)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(num_pages) * Hkv >= (1LL << 31)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < decode_workspace_bytes(S, Hq, d, max_blocks)) return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  return launch_decode_paged_q8(q, k_pages, v_pages, k_scales, v_scales, kv_format, block_table,
                                seq_lens, o, lse, S, Hq, Hkv, d, max_blocks, num_pages, scale,
                                workspace, reinterpret_cast<cudaStream_t>(stream));
}

// The workspace-free decode: same checks and kernels as attn_decode_paged, with
// the library's fixed per-device scratch array standing in for the workspace.
attn_status_t attn_decode_paged_noalloc(const void *q, const void *k_pages, const void *v_pages,
                                        const int32_t *block_table, const int32_t *seq_lens,
                                        void *o, float *lse, int S, int Hq, int Hkv, int d,
                                        int page_size, int max_blocks, int num_pages, float scale,
                                        attn_stream_t stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned4(block_table) ||
      !aligned4(seq_lens) || !aligned16(o) || !aligned4(lse))
    return ATTN_ERR_INVALID_ARG;
  if (S <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || page_size <= 0 ||
      max_blocks <= 0 || num_pages <= 0 || !good_scale(scale))
    return ATTN_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * page_size > (1LL << 30)) return ATTN_ERR_INVALID_ARG;
  if (decode_workspace_bytes(S, Hq, d, max_blocks) > ATTN_DECODE_NOALLOC_SCRATCH_BYTES)
    return ATTN_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  bool sm100 = false;
  if (!device_state(&status, &sm100)) return ATTN_ERR_CUDA;
  if (!sm100) return ATTN_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  attn_status_t st = noalloc_scratch_address(&scratch);
  if (st != ATTN_OK) return st;
  // The scratch is shared, so its status word belongs to no caller: the bits
  // also go to the per-device word that attn_device_status reads.
  return launch_decode_paged(q, k_pages, v_pages, block_table, seq_lens, o, lse, S, Hq, Hkv, d,
                             max_blocks, num_pages, scale, scratch,
                             reinterpret_cast<cudaStream_t>(stream), status);
}

attn_status_t attn_decode_read_status(const void *workspace, unsigned *dev_status) {
  if (!aligned16(workspace) || !dev_status) return ATTN_ERR_INVALID_ARG;
  // One 4-byte copy through this thread's own default stream: it waits for
  // nothing the caller enqueued on other streams (the caller has synchronised
  // the decode's stream already).  cudaMemcpyDefault lets the workspace live
  // on any device.
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(unsigned), cudaMemcpyDefault,
                      cudaStreamPerThread) != cudaSuccess ||
      cudaStreamSynchronize(cudaStreamPerThread) != cudaSuccess)
    return ATTN_ERR_CUDA;
  *dev_status = word;
  return ATTN_OK;
}

attn_status_t attn_device_status(unsigned *status, int clear, attn_stream_t stream) {
  if (!status) return ATTN_ERR_INVALID_ARG;
  unsigned *dev_ptr = nullptr;
  bool sm100 = false;
  if (!device_state(&dev_ptr, &sm100)) return ATTN_ERR_CUDA;
  // Everything enqueued on `stream` before this call finishes first (the copy is
  // ordered behind it); other streams are not waited for.
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, dev_ptr, sizeof(unsigned), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (clear && (cudaMemsetAsync(dev_ptr, 0, sizeof(unsigned), st) != cudaSuccess ||
                cudaStreamSynchronize(st) != cudaSuccess))
    return ATTN_ERR_CUDA;
  *status = word;
  return ATTN_OK;
}

const char *attn_status_string(attn_status_t status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
  }
  return "ATTN_UNKNOWN_STATUS";
}

const char *attn_version(void) { return "exattn 0.1.0 (sm_100a)"; }

}  // extern "C"
