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

#include "common.cuh"
#include "internal.h"

namespace exattn {
namespace {

constexpr int kPageSize = 16;
constexpr int kPagesPerSplit = 32;  // 512 tokens per chunk
constexpr int kWarps = 4;

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

constexpr int kStages = 8;  // shared-memory ring of (K page, V page) slices

template <int D>
constexpr int stage_bytes() { return 2 * kPageSize * D * 2; }

// Workspace: o_part [S][Hq][nsplit][D] f32 (normalised), l2_part [S][Hq][nsplit]
// f32 (log2-sum-exp of scale*log2(e)*scores over the chunk; NaN marks a bad sequence).
//
// Warps 0..kWarps-1 compute; warp kWarps is the producer: its lane 0 copies the
// visible rows of each page's K and V slices into a kStages-deep shared-memory
// ring with bulk async copies, so the bytes in flight do not depend on how many
// registers the compute warps hold.  Page i of the chunk goes to stage
// i % kStages and is consumed by warp i % kWarps.
template <int D, int GB>
__global__ void __launch_bounds__((kWarps + 1) * 32, GB >= 8 ? 2 : 3)
    decode_split_kernel(const __nv_bfloat16 *__restrict__ q,
                        const __nv_bfloat16 *__restrict__ k_pages,
                        const __nv_bfloat16 *__restrict__ v_pages,
                        const int *__restrict__ block_table, const int *__restrict__ seq_lens,
                        float *__restrict__ o_part, float *__restrict__ l2_part, int Hq, int Hkv,
                        int max_blocks, int num_pages, float scale_log2, int nsplit,
                        int head_chunks, unsigned *status) {
  constexpr int LPT = D / 8;           // lanes per token row (8 bf16 = 16 B each)
  constexpr int TPI = 32 / LPT;        // token rows per warp-wide access
  constexpr int IT = kPageSize / TPI;  // accesses per page per lane
  constexpr int SLICE = kPageSize * D; // elements of one page's K (or V) slice
  static_assert(kPagesPerSplit <= 32, "one block-table entry per producer lane");
  const int split = blockIdx.x;
  const int g = blockIdx.y / head_chunks;
  const int h0 = g * (Hq / Hkv) + (blockIdx.y % head_chunks) * GB;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPT;          // token row of an access held by this lane
  const int dc = lane % LPT;           // 8-column slice held by this lane

  const int len = seq_lens[s];
  const bool bad_len = len < 0 || len > max_blocks * kPageSize;
  const int page_begin = split * kPagesPerSplit;
  const int n_pages = bad_len ? 0 : (len + kPageSize - 1) / kPageSize;
  if (!bad_len && page_begin >= n_pages) return;  // chunk past the end: nothing to do
  const int npg = bad_len ? 0 : min(n_pages, page_begin + kPagesPerSplit) - page_begin;

  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ int stage_ntok[kStages];
  __shared__ int sm_pid[kPagesPerSplit];
  __shared__ float sm_m[kWarps][GB], sm_l[kWarps][GB];
  __shared__ float sm_acc[kWarps][GB][D];
  __shared__ int sm_bad, sm_abort;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    sm_bad = bad_len ? 1 : 0;
    sm_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ------------------------------------------------------------ producer
    if (lane < npg) sm_pid[lane] = block_table[static_cast<size_t>(s) * max_blocks + page_begin + lane];
    __syncwarp();
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < npg; ++i) {
        const int st = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[st], ((i / kStages) - 1) & 1, &sm_abort, status)) break;
        const int pid = sm_pid[i];
        const int ntok = min(kPageSize, len - (page_begin + i) * kPageSize);
        if (pid < 0 || pid >= num_pages) {  // never dereference a bad page id
          sm_bad = 1;
          stage_ntok[st] = 0;
          mbar_arrive(&full[st]);
        } else {
          stage_ntok[st] = ntok;
          const uint32_t bytes = static_cast<uint32_t>(ntok * D * 2);
          const size_t base = (static_cast<size_t>(pid) * Hkv + g) * SLICE;
          uint8_t *dst = ring + st * stage_bytes<D>();
          mbar_arrive_expect_tx(&full[st], 2 * bytes);
          bulk_load(dst, k_pages + base, bytes, &full[st]);
          bulk_load(dst + SLICE * 2, v_pages + base, bytes, &full[st]);
        }
        issued = i + 1;
      }
      // Let every copy land before the CTA (and its shared memory) goes away.
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait_drain(&full[i % kStages], (i / kStages) & 1, status);
    }
  } else {
    // ------------------------------------------------------------ compute
    // Query slice of this lane (8 columns, every head of the group) as float2
    // pairs, pre-multiplied by scale*log2(e).
    float2 q2[GB][4];
#pragma unroll
    for (int hh = 0; hh < GB; ++hh) {
      const uint4 u = *reinterpret_cast<const uint4 *>(
          q + (static_cast<size_t>(s) * Hq + h0 + hh) * D + dc * 8);
      float f[8];
      bf16x8_to_f32(u, f);
#pragma unroll
      for (int e = 0; e < 4; ++e) q2[hh][e] = make_float2(f[2 * e] * scale_log2, f[2 * e + 1] * scale_log2);
    }
    // After the transposed reduction below, this lane holds the score of one head
    // of the group: my_head; the lane holding head hh in a row group is
    // hh * (LPT / GB) within it.
    int my_head = 0;
    {
      int n = GB;
#pragma unroll
      for (int o = LPT / 2; o > 0; o >>= 1) {
        if (n > 1) {
          if (lane & o) my_head += n / 2;
          n /= 2;
        }
      }
    }
    float m = -INFINITY, l = 0.f;  // running max / sum of my_head, over this lane's rows
    float2 acc[GB][4];             // every head, this lane's 8 columns, this lane's rows
#pragma unroll
    for (int hh = 0; hh < GB; ++hh)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[hh][e] = make_float2(0.f, 0.f);

    for (int i = warp; i < npg; i += kWarps) {
      const int st = i % kStages;
      bool ok = mbar_wait(&full[st], (i / kStages) & 1, &sm_abort, status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int ntok = stage_ntok[st];
      if (ntok > 0) {
        const uint8_t *ks = ring + st * stage_bytes<D>();
        const uint8_t *vs = ks + SLICE * 2;
        // q . k for this lane's rows: partial dot over 8 columns per head, then a
        // butterfly over the LPT lanes of the row that also transposes, so each
        // lane ends with one head's full score (log2 units).
        float sc[IT];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int row = it * TPI + sub;
          float kf[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4 *>(ks + (row * D + dc * 8) * 2), kf);
          float v[GB];
#pragma unroll
          for (int hh = 0; hh < GB; ++hh) {
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 4; ++e) a = fma2(q2[hh][e], make_float2(kf[2 * e], kf[2 * e + 1]), a);
            v[hh] = a.x + a.y;
          }
          int n = GB;
#pragma unroll
          for (int o = LPT / 2; o > 0; o >>= 1) {
            if (n > 1) {
              const bool up = (lane & o) != 0;
#pragma unroll
              for (int x = 0; x < n / 2; ++x) {
                const float send = up ? v[x] : v[x + n / 2];
                const float keep = up ? v[x + n / 2] : v[x];
                v[x] = keep + __shfl_xor_sync(0xffffffffu, send, o);
              }
              n /= 2;
            } else {
              v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
            }
          }
          sc[it] = row < ntok ? v[0] : -INFINITY;
        }
        // Online softmax for my_head over this page (all rows: reduce over the
        // row groups of the warp).
        float mx = sc[0];
#pragma unroll
        for (int it = 1; it < IT; ++it) mx = fmaxf(mx, sc[it]);
#pragma unroll
        for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m, mx);  // finite: row 0 of a page is always visible
        const float alpha = ex2f(m - m_new);
        m = m_new;
        l *= alpha;
#pragma unroll
        for (int hh = 0; hh < GB; ++hh) {
          const float a = __shfl_sync(0xffffffffu, alpha, hh * (LPT / GB));
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[hh][e] = make_float2(acc[hh][e].x * a, acc[hh][e].y * a);
        }
        // P V: each lane needs every head's weight for its rows.
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int row = it * TPI + sub;
          const float pw = ex2f(sc[it] - m);  // 0 for rows past the sequence end
          l += pw;
          float vf[8];
          // Rows past ntok were not copied this time: read zeros, never stale data.
          const uint4 vraw = row < ntok ? *reinterpret_cast<const uint4 *>(vs + (row * D + dc * 8) * 2)
                                        : make_uint4(0, 0, 0, 0);
          bf16x8_to_f32(vraw, vf);
#pragma unroll
          for (int hh = 0; hh < GB; ++hh) {
            const float ph = __shfl_sync(0xffffffffu, pw, sub * LPT + hh * (LPT / GB));
            const float2 p2 = make_float2(ph, ph);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[hh][e] = fma2(p2, make_float2(vf[2 * e], vf[2 * e + 1]), acc[hh][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
    }

    // Merge the row groups of the warp: acc over lanes sharing a column slice,
    // l over lanes sharing a head.
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
      for (int hh = 0; hh < GB; ++hh)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[hh][e].x += __shfl_xor_sync(0xffffffffu, acc[hh][e].x, o);
          acc[hh][e].y += __shfl_xor_sync(0xffffffffu, acc[hh][e].y, o);
        }
    }
    if (lane < LPT) {
#pragma unroll
      for (int hh = 0; hh < GB; ++hh)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sm_acc[warp][hh][dc * 8 + 2 * e] = acc[hh][e].x;
          sm_acc[warp][hh][dc * 8 + 2 * e + 1] = acc[hh][e].y;
        }
      if (lane % (LPT / GB) == 0) {
        sm_m[warp][my_head] = m;
        sm_l[warp][my_head] = l;
      }
    }
  }
  __syncthreads();

  // Merge the warps and write this chunk's normalised partial per head.
  const bool bad = sm_bad != 0 || sm_abort != 0;
  if (bad && threadIdx.x == 0 && sm_bad) atomicOr(status, ATTN_DEV_BAD_PAGE);
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
                          float *__restrict__ lse, int S, int Hq, int max_blocks, int nsplit,
                          int pages_per_split) {
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
      bad_len ? 0 : ((len + kPageSize - 1) / kPageSize + pages_per_split - 1) / pages_per_split;
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
  constexpr int kSmem = kStages * stage_bytes<D>();
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(decode_split_kernel<D, GB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSmem);
  });
  decode_split_kernel<D, GB><<<grid, (kWarps + 1) * 32, kSmem, st>>>(
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
  return launch_decode_combine(o_part, l2_part, seq_lens, o, lse, S, Hq, d, max_blocks, nsplit,
                               kPagesPerSplit, stream);
}

attn_status_t launch_decode_combine(const float *o_part, const float *l2_part, const int *seq_lens,
                                    void *o, float *lse, int S, int Hq, int d, int max_blocks,
                                    int nsplit, int pages_per_split, cudaStream_t stream) {
  const int heads = S * Hq;
  const int blocks = (heads + 3) / 4;
  if (d == 128)
    decode_combine_kernel<128><<<blocks, 128, 0, stream>>>(o_part, l2_part, seq_lens,
                                                           static_cast<__nv_bfloat16 *>(o), lse, S,
                                                           Hq, max_blocks, nsplit, pages_per_split);
  else if (d == 64)
    decode_combine_kernel<64><<<blocks, 128, 0, stream>>>(o_part, l2_part, seq_lens,
                                                          static_cast<__nv_bfloat16 *>(o), lse, S,
                                                          Hq, max_blocks, nsplit, pages_per_split);
  else
    return ATTN_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace exattn
