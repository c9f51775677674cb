// decode_paged.cu -- single-token attention over a paged KV cache (split-KV).
//
// What it computes: for each sequence s and query head h, the exact attention
// of its one query vector over all seq_lens[s] cached keys/values, which live
// in fixed-size pages reached through a block table ("Phase 08" page, Concepts:
// KV cache and paged attention; Lab 03 step 4: attention over non-contiguous
// pages via an indirection table).  Query heads that share a K/V head
// (grouped-query attention) are served from one read of that head's pages.
//
// Decode is bound by HBM bandwidth (quiz page, question 1: few FLOPs per byte),
// so the design is about moving each K/V byte exactly once at full rate:
//  * split kernel: one CTA per (key chunk of kPagesPerSplit pages, K/V head,
//    sequence).  Each warp takes every 4th page of the chunk and reads it with
//    16-byte vector loads (a 16 x d page slice is one contiguous 4 KiB run for
//    d = 128), scores it for the group's query heads (warp-shuffle reductions),
//    and folds it into a running max / sum / accumulator (online softmax, Lab 01
//    talking points).  The CTA merges its warps and writes one normalised
//    partial output and its log2-sum-exp per head to the workspace.
//  * combine kernel: per (sequence, head), merges the chunks' partials with
//    weights 2^(L_r - L) -- the same rescaling rule applied across chunks --
//    and writes O (bf16) and L (natural log, float32).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "internal.h"

namespace exattn {
namespace {

constexpr int kPageSize = 16;
constexpr int kPagesPerSplit = 32;  // 512 tokens per chunk
constexpr int kWarps = 4;

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Workspace: o_part [S][Hq][nsplit][D] f32 (normalised), l2_part [S][Hq][nsplit]
// f32 (log2-sum-exp of scale*log2(e)*scores over the chunk; NaN marks a bad sequence).
template <int D, int GB>
__global__ void __launch_bounds__(kWarps * 32)
    decode_split_kernel(const __nv_bfloat16 *__restrict__ q,
                        const __nv_bfloat16 *__restrict__ k_pages,
                        const __nv_bfloat16 *__restrict__ v_pages,
                        const int *__restrict__ block_table, const int *__restrict__ seq_lens,
                        float *__restrict__ o_part, float *__restrict__ l2_part, int Hq, int Hkv,
                        int max_blocks, int num_pages, float scale_log2, int nsplit,
                        int head_chunks, unsigned *status) {
  constexpr int LPT = D / 8;          // lanes per token row (8 bf16 = 16 B each)
  constexpr int TPI = 32 / LPT;       // token rows per warp-wide load
  constexpr int IT = kPageSize / TPI; // loads per page per lane
  const int split = blockIdx.x;
  const int g = blockIdx.y / head_chunks;
  const int h0 = g * (Hq / Hkv) + (blockIdx.y % head_chunks) * GB;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPT;         // which token row of a load this lane holds
  const int dc = lane % LPT;          // which 8-column slice

  const int len = seq_lens[s];
  const int cap = max_blocks * kPageSize;
  const bool bad_len = len < 0 || len > cap;
  const int page_begin = split * kPagesPerSplit;
  const int n_pages = bad_len ? 0 : (len + kPageSize - 1) / kPageSize;
  if (!bad_len && page_begin >= n_pages) return;  // chunk past the end: nothing to do
  const int page_end = min(n_pages, page_begin + kPagesPerSplit);

  __shared__ float sm_m[kWarps][GB], sm_l[kWarps][GB];
  __shared__ float sm_acc[kWarps][GB][D];
  __shared__ int sm_bad;
  if (threadIdx.x == 0) sm_bad = bad_len ? 1 : 0;
  __syncthreads();

  // Query slice of this lane, pre-multiplied by scale*log2(e).
  float qf[GB][8];
#pragma unroll
  for (int hh = 0; hh < GB; ++hh) {
    const uint4 u = *reinterpret_cast<const uint4 *>(q + (static_cast<size_t>(s) * Hq + h0 + hh) * D + dc * 8);
    bf16x8_to_f32(u, qf[hh]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[hh][e] *= scale_log2;
  }

  float m[GB], l[GB], acc[GB][8];
#pragma unroll
  for (int hh = 0; hh < GB; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
  }

  for (int pg = page_begin + warp; !bad_len && pg < page_end; pg += kWarps) {
    const int pid = block_table[static_cast<size_t>(s) * max_blocks + pg];
    if (pid < 0 || pid >= num_pages) {  // never dereference a bad page id
      if (lane == 0) sm_bad = 1;
      continue;
    }
    const size_t base = (static_cast<size_t>(pid) * Hkv + g) * kPageSize * D;
    uint4 kr[IT], vr[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int tok = pg * kPageSize + it * TPI + sub;
      const size_t off = base + static_cast<size_t>(it * TPI + sub) * D + dc * 8;
      if (tok < len) {
        kr[it] = ld_stream(k_pages + off);
        vr[it] = ld_stream(v_pages + off);
      } else {
        kr[it] = make_uint4(0, 0, 0, 0);
        vr[it] = make_uint4(0, 0, 0, 0);
      }
    }
    // Scores (log2 units) of this lane's token rows for every head of the group.
    float sc[GB][IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      float kf[8];
      bf16x8_to_f32(kr[it], kf);
      const bool vis = pg * kPageSize + it * TPI + sub < len;
#pragma unroll
      for (int hh = 0; hh < GB; ++hh) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) part = fmaf(qf[hh][e], kf[e], part);
#pragma unroll
        for (int o = LPT / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        sc[hh][it] = vis ? part : -INFINITY;
      }
    }
#pragma unroll
    for (int hh = 0; hh < GB; ++hh) {
      float mx = sc[hh][0];
#pragma unroll
      for (int it = 1; it < IT; ++it) mx = fmaxf(mx, sc[hh][it]);
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m[hh], mx);  // finite: every page holds a visible token
      const float alpha = ex2f(m[hh] - m_new);
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[hh][e] *= alpha;
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const float pw = ex2f(sc[hh][it] - m_new);  // 0 for masked rows
        psum += pw;
        float vf[8];
        bf16x8_to_f32(vr[it], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] = fmaf(pw, vf[e], acc[hh][e]);
      }
      l[hh] = l[hh] * alpha + psum;
      m[hh] = m_new;
    }
  }

  // Merge the token-row groups of the warp (lanes that share a column slice).
#pragma unroll
  for (int hh = 0; hh < GB; ++hh) {
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], o);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[hh][e] += __shfl_xor_sync(0xffffffffu, acc[hh][e], o);
    }
  }
  if (lane < LPT) {
#pragma unroll
    for (int hh = 0; hh < GB; ++hh) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_acc[warp][hh][dc * 8 + e] = acc[hh][e];
      if (lane == 0) {
        sm_m[warp][hh] = m[hh];
        sm_l[warp][hh] = l[hh];
      }
    }
  }
  __syncthreads();

  // Merge the warps and write this chunk's normalised partial per head.
  const bool bad = sm_bad != 0;
  if (bad && threadIdx.x == 0) atomicOr(status, ATTN_DEV_BAD_PAGE);
  for (int idx = threadIdx.x; idx < GB * D; idx += blockDim.x) {
    const int hh = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][hh]);
    float wsum = 0.f, num = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float wt = (sm_m[w][hh] == -INFINITY) ? 0.f : ex2f(sm_m[w][hh] - M);
      wsum += wt * sm_l[w][hh];
      num += wt * sm_acc[w][hh][c];
    }
    const size_t slot = (static_cast<size_t>(s) * Hq + h0 + hh) * nsplit + split;
    o_part[slot * D + c] = bad ? NAN : num / wsum;
    if (c == 0) l2_part[slot] = bad ? NAN : M + log2f(wsum);
  }
}

// One warp per (sequence, head): merge the chunk partials.
template <int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float *__restrict__ o_part, const float *__restrict__ l2_part,
                          const int *__restrict__ seq_lens, __nv_bfloat16 *__restrict__ o,
                          float *__restrict__ lse, int S, int Hq, int max_blocks, int nsplit) {
  constexpr int DPL = D / 32;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= S * Hq) return;
  const int s = gw / Hq;
  const int len = seq_lens[s];
  const size_t head = static_cast<size_t>(gw);
  __nv_bfloat16 *orow = o + head * D;
  const bool bad_len = len < 0 || len > max_blocks * kPageSize;
  if (!bad_len && len == 0) {
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(0.f);
    if (lane == 0) lse[head] = -INFINITY;
    return;
  }
  const int nparts =
      bad_len ? 0 : ((len + kPageSize - 1) / kPageSize + kPagesPerSplit - 1) / kPagesPerSplit;
  const float *lp = l2_part + head * nsplit;
  bool bad = bad_len;
  float M = -INFINITY;
  for (int r = 0; r < nparts; ++r) {
    const float x = lp[r];
    bad |= isnan(x);
    M = fmaxf(M, x);
  }
  if (bad) {
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(NAN);
    if (lane == 0) lse[head] = NAN;
    return;
  }
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int r = 0; r < nparts; ++r) {
    const float wt = ex2f(lp[r] - M);
    wsum += wt;
    const float *op = o_part + (head * nsplit + r) * D;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wt, op[lane + 32 * e], acc[e]);
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) lse[head] = (M + log2f(wsum)) * 0.6931471805599453f;
}

template <int D, int GB>
void launch_split(dim3 grid, cudaStream_t st, const void *q, const void *kp, const void *vp,
                  const int *bt, const int *sl, float *op, float *lp, int Hq, int Hkv, int maxb,
                  int npages, float sl2, int nsplit, int hc, unsigned *status) {
  decode_split_kernel<D, GB><<<grid, kWarps * 32, 0, st>>>(
      static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(kp),
      static_cast<const __nv_bfloat16 *>(vp), bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit,
      hc, status);
}

template <int D>
bool dispatch_split(int GB, dim3 grid, cudaStream_t st, const void *q, const void *kp,
                    const void *vp, const int *bt, const int *sl, float *op, float *lp, int Hq,
                    int Hkv, int maxb, int npages, float sl2, int nsplit, int hc,
                    unsigned *status) {
  switch (GB) {
    case 8: launch_split<D, 8>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 4: launch_split<D, 4>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 2: launch_split<D, 2>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 1: launch_split<D, 1>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
  }
  return false;
}

}  // namespace

// Scratch of attn_decode_paged_noalloc.  A fixed array in the module's device
// memory: every GPU that loads this library holds it until the process exits,
// and all no-allocation calls on a device share it.  Host code must not pass
// the symbol itself to a kernel -- on the host it names a stand-in, not a
// device address -- so its device address is looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mutex;
void *g_scratch_addr[64] = {};
}  // namespace

// Device address of g_noalloc_scratch on the current device; looked up once
// per device (with that device current) on its first no-allocation call.
attn_status_t noalloc_scratch_address(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return ATTN_OK;
}

int decode_max_splits(int max_blocks) { return (max_blocks + kPagesPerSplit - 1) / kPagesPerSplit; }

size_t decode_workspace_bytes(int S, int Hq, int d, int max_blocks) {
  const size_t parts = static_cast<size_t>(S) * Hq * decode_max_splits(max_blocks);
  const size_t o_bytes = (parts * d * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return o_bytes + ((parts * sizeof(float) + 255) & ~static_cast<size_t>(255));
}

attn_status_t launch_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                  const int *block_table, const int *seq_lens, void *o, float *lse,
                                  int S, int Hq, int Hkv, int d, int max_blocks, int num_pages,
                                  float scale, void *workspace, cudaStream_t stream,
                                  unsigned *status) {
  const int G = Hq / Hkv;
  const int GB = (G % 8 == 0) ? 8 : (G % 4 == 0) ? 4 : (G % 2 == 0) ? 2 : 1;
  const int head_chunks = G / GB;
  const int nsplit = decode_max_splits(max_blocks);
  const size_t parts = static_cast<size_t>(S) * Hq * nsplit;
  float *o_part = static_cast<float *>(workspace);
  float *l2_part = reinterpret_cast<float *>(
      static_cast<uint8_t *>(workspace) +
      ((parts * d * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  if (static_cast<long long>(Hkv) * head_chunks > 65535 || S > 65535) return ATTN_ERR_UNSUPPORTED;
  dim3 grid(nsplit, Hkv * head_chunks, S);
  const float sl2 = scale * 1.4426950408889634f;
  bool ok;
  if (d == 128)
    ok = dispatch_split<128>(GB, grid, stream, q, k_pages, v_pages, block_table, seq_lens, o_part,
                             l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else if (d == 64)
    ok = dispatch_split<64>(GB, grid, stream, q, k_pages, v_pages, block_table, seq_lens, o_part,
                            l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else
    return ATTN_ERR_UNSUPPORTED;
  if (!ok) return ATTN_ERR_UNSUPPORTED;
  const int heads = S * Hq;
  const int blocks = (heads + 3) / 4;
  if (d == 128)
    decode_combine_kernel<128><<<blocks, 128, 0, stream>>>(o_part, l2_part, seq_lens,
                                                           static_cast<__nv_bfloat16 *>(o), lse, S,
                                                           Hq, max_blocks, nsplit);
  else
    decode_combine_kernel<64><<<blocks, 128, 0, stream>>>(o_part, l2_part, seq_lens,
                                                          static_cast<__nv_bfloat16 *>(o), lse, S,
                                                          Hq, max_blocks, nsplit);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace exattn
