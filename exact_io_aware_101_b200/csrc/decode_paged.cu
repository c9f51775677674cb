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
//  * split kernel: one CTA per (key chunk of kPagesPerSplit pages, sequence,
//    group of up to 8 K/V heads).  A producer warp brings each page of the
//    chunk into shared memory with one bulk copy per tensor covering all the
//    group's heads (they are contiguous in the pool); each compute warp owns
//    one K/V head, scores every page for the head's query heads (warp-shuffle
//    reductions), folds it into a running max / sum / accumulator (online
//    softmax, Lab 01 talking points), and writes one normalised partial
//    output and its log2-sum-exp per head to the workspace.
//  * combine kernel: per (sequence, head), merges the chunks' partials with
//    weights 2^(L_r - L) -- the same rescaling rule applied across chunks --
//    and writes O (bf16) and L (natural log, float32).
//  * status: each call owns the status word at the start of its workspace.
//    The split grid's first CTA clears it; a chunk that fails records its
//    ATTN_DEV_* bits in its partial (failed_partial); the combine kernel, which
//    starts only once the whole split grid is done, ORs them into the word.
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
constexpr float kRescaleLog2 = 8.f;  // lazy rescale: move the max only when it grows by > 2^8

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

// Page-major: one CTA per (chunk of kPagesPerSplit pages, sequence, group of
// HC K/V heads, chunk of GB query heads per K/V head).  The K slices of the HC
// heads of one page are contiguous in the pool ([page][head][16][d]), so warp
// HC (the producer) brings each page in with one bulk copy per tensor -- 32 KiB
// of K and 32 KiB of V for 8 heads at d = 128 -- instead of one small copy per
// (page, head): a stream of small copies stops well short of the HBM rate.
// Warp w < HC owns K/V head g0 + w and walks every page of the chunk.
template <int HC, int D>
struct DecCfg {
  static constexpr int SLICE = kPageSize * D * 2;  // bytes of one (page, head) K or V slice
  static constexpr int STAGE = 2 * HC * SLICE;
  static constexpr int NST = (196608 / STAGE) < 2 ? 2 : ((196608 / STAGE) > 8 ? 8 : 196608 / STAGE);
  static constexpr int SMEM = NST * STAGE;
};

// Workspace (decode_ws_layout): the call's status word, then o_part
// [S][Hq][nsplit][D] f32 (normalised) and l2_part [S][Hq][nsplit] f32
// (log2-sum-exp of scale*log2(e)*scores over the chunk; a tagged NaN marks a
// failed chunk).
template <int D, int GB, int HC>
__global__ void __launch_bounds__((HC + 1) * 32)
    decode_split_kernel(const __nv_bfloat16 *__restrict__ q,
                        const __nv_bfloat16 *__restrict__ k_pages,
                        const __nv_bfloat16 *__restrict__ v_pages,
                        const int *__restrict__ block_table, const int *__restrict__ seq_lens,
                        float *__restrict__ o_part, float *__restrict__ l2_part, int Hq, int Hkv,
                        int max_blocks, int num_pages, float scale_log2, int nsplit,
                        int head_chunks, unsigned *call_status) {
  // The call's status word starts clear; only the combine kernel, which waits
  // for this whole grid, sets bits in it.
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *call_status = 0;
  grid_dependents_launch();  // the combine kernel may be scheduled behind this grid
  using C = DecCfg<HC, D>;
  constexpr int LPT = D / 8;           // lanes per token row (8 bf16 = 16 B each)
  constexpr int TPI = 32 / LPT;        // token rows per warp-wide access
  constexpr int IT = kPageSize / TPI;  // accesses per page per lane
  static_assert(kPagesPerSplit <= 32, "one block-table entry per producer lane");
  const int split = blockIdx.x;
  const int s = blockIdx.y;
  const int kvgrp = blockIdx.z / head_chunks;
  const int hchunk = blockIdx.z % head_chunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = kvgrp * HC + min(warp, HC - 1);      // this consumer warp's K/V head
  const int h0 = g * (Hq / Hkv) + hchunk * GB;       // its first query head
  const int sub = lane / LPT;          // token row of an access held by this lane
  const int dc = lane % LPT;           // 8-column slice held by this lane

  const int len = seq_lens[s];
  const bool bad_len = len < 0 || len > max_blocks * kPageSize;
  const int page_begin = split * kPagesPerSplit;
  const int n_pages = bad_len ? 0 : (len + kPageSize - 1) / kPageSize;
  if (!bad_len && page_begin >= n_pages) return;  // chunk past the end: nothing to do
  const int npg = bad_len ? 0 : min(n_pages, page_begin + kPagesPerSplit) - page_begin;

  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[C::NST], empty[C::NST];
  __shared__ int stage_ntok[C::NST];
  __shared__ int sm_pid[kPagesPerSplit];
  __shared__ int sm_bad, sm_abort;
  __shared__ unsigned sm_status;  // ATTN_DEV_* bits of this CTA's bounded waits
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], HC);
    }
    sm_bad = bad_len ? 1 : 0;
    sm_abort = 0;
    sm_status = 0;
    fence_mbar_init();
  }
  if (warp == HC && lane < npg)
    sm_pid[lane] = block_table[static_cast<size_t>(s) * max_blocks + page_begin + lane];
  __syncthreads();

  if (warp == HC) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < npg; ++i) {
        const int st = i % C::NST;
        if (i >= C::NST && !mbar_wait(&empty[st], ((i / C::NST) - 1) & 1, &sm_abort, &sm_status))
          break;
#ifdef EXATTN_TEST_WITHHOLD
        // Test build only: stop before page EXATTN_TEST_WITHHOLD, arriving on
        // nothing and copying nothing, so the compute warps' wait runs out.
        if (i == EXATTN_TEST_WITHHOLD) break;
#endif
        const int pid = sm_pid[i];
        if (pid < 0 || pid >= num_pages) {  // never dereference a bad page id
          sm_bad = 1;
          stage_ntok[st] = 0;
          mbar_arrive(&full[st]);
        } else {
          // The whole page (16 rows of every head); rows past the sequence end
          // are never read by the compute warps.
          stage_ntok[st] = min(kPageSize, len - (page_begin + i) * kPageSize);
          const size_t base = (static_cast<size_t>(pid) * Hkv + kvgrp * HC) * (C::SLICE / 2);
          uint8_t *dst = ring + st * C::STAGE;
          mbar_arrive_expect_tx(&full[st], C::STAGE);
          bulk_load(dst, k_pages + base, HC * C::SLICE, &full[st]);
          bulk_load(dst + HC * C::SLICE, v_pages + base, HC * C::SLICE, &full[st]);
        }
        issued = i + 1;
      }
      // Let every copy land before the CTA (and its shared memory) goes away.
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        mbar_wait_drain(&full[i % C::NST], (i / C::NST) & 1, &sm_status);
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

    for (int i = 0; i < npg; ++i) {
      const int st = i % C::NST;
      bool ok = mbar_wait(&full[st], (i / C::NST) & 1, &sm_abort, &sm_status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int ntok = stage_ntok[st];
      if (ntok > 0) {
        const uint8_t *ks = ring + st * C::STAGE + warp * C::SLICE;
        const uint8_t *vs = ring + st * C::STAGE + (HC + warp) * C::SLICE;
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
        // Lazy rescale: the reference m moves (and l, acc are rescaled) only
        // when a score exceeds it by more than 2^8, so P <= 2^8 in fp32 and
        // most pages skip the rescale.  mx is finite: row 0 of a page is
        // always visible.
        if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
          const float m_new = fmaxf(m, mx);
          const float alpha = ex2f(m - m_new);  // 0 on the first page (m = -inf)
          m = m_new;
          l *= alpha;
#pragma unroll
          for (int hh = 0; hh < GB; ++hh) {
            const float a = __shfl_sync(0xffffffffu, alpha, hh * (LPT / GB));
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[hh][e] = make_float2(acc[hh][e].x * a, acc[hh][e].y * a);
          }
        }
        // P V: each lane needs every head's weight for its rows.
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int row = it * TPI + sub;
          const float pw = ex2f(sc[it] - m);  // 0 for rows past the sequence end
          l += pw;
          float vf[8];
          // Rows past the sequence end hold whatever the cache slots hold:
          // read zeros instead (a NaN there would survive a zero weight).
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
    // The warp's partial is the chunk's for its heads: normalise and write.
    // sm_bad / sm_abort are final once every page has been consumed (or the
    // warp gave up); a failed chunk's partial carries its status bits.
    const bool bad = *reinterpret_cast<volatile int *>(&sm_bad) != 0 ||
                     *reinterpret_cast<volatile int *>(&sm_abort) != 0;
    unsigned bits = *reinterpret_cast<volatile unsigned *>(&sm_status) |
                    (*reinterpret_cast<volatile int *>(&sm_bad) ? ATTN_DEV_BAD_PAGE : 0u);
    if (bad && bits == 0) bits = ATTN_DEV_TIMEOUT;  // aborted by a wait that timed out
#pragma unroll
    for (int hh = 0; hh < GB; ++hh) {
      const float mh = __shfl_sync(0xffffffffu, m, hh * (LPT / GB));
      const float lh = __shfl_sync(0xffffffffu, l, hh * (LPT / GB));
      const size_t slot = (static_cast<size_t>(s) * Hq + h0 + hh) * nsplit + split;
      if (lane < LPT) {
        const float inv = 1.f / lh;
        float4 *dst = reinterpret_cast<float4 *>(o_part + slot * D + dc * 8);
        dst[0] = bad ? make_float4(NAN, NAN, NAN, NAN)
                     : make_float4(acc[hh][0].x * inv, acc[hh][0].y * inv, acc[hh][1].x * inv,
                                   acc[hh][1].y * inv);
        dst[1] = bad ? make_float4(NAN, NAN, NAN, NAN)
                     : make_float4(acc[hh][2].x * inv, acc[hh][2].y * inv, acc[hh][3].x * inv,
                                   acc[hh][3].y * inv);
      }
      if (lane == 0) l2_part[slot] = bad ? failed_partial(bits) : mh + log2f(lh);
    }
  }
}

// One warp per (sequence, head): merge the chunk partials.  The lanes read the
// chunks' log-sum-exps side by side (lane r holds chunks r, r + 32, ...), so
// the weights cost one load round and two shuffle reductions; the weighted
// rows are then summed eight chunks at a time with their loads issued
// together.  Launched as a programmatic dependent of the split kernel: it may
// start while the split kernel's last CTAs run, and waits for that grid to
// finish (and its writes to be visible) before it reads a partial.  A failed
// sequence (a bad length, or a chunk whose partial is a tagged NaN) gets NaN
// outputs and its bits are ORed into the call's status word (and into
// dev_status when that is given).
template <int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float *__restrict__ o_part, const float *__restrict__ l2_part,
                          const int *__restrict__ seq_lens, __nv_bfloat16 *__restrict__ o,
                          float *__restrict__ lse, int S, int Hq, int max_blocks, int nsplit,
                          int pages_per_split, unsigned *call_status, unsigned *dev_status) {
  constexpr int DPL = D / 32;
  constexpr int kBatch = 8;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  grid_dependency_wait();
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
  unsigned bits = bad_len ? ATTN_DEV_BAD_PAGE : 0u;
  float M = -INFINITY;
  for (int r = lane; r < nparts; r += 32) {
    const float x = lp[r];
    if (isnan(x)) {
      bad = true;
      bits |= failed_partial_bits(x);
    }
    M = fmaxf(M, x);
  }
  bad = __any_sync(0xffffffffu, bad);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (bad) {
    bits = __reduce_or_sync(0xffffffffu, bits);
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(NAN);
    if (lane == 0) {
      lse[head] = NAN;
      if (bits) {
        atomicOr(call_status, bits);
        if (dev_status) atomicOr(dev_status, bits);
      }
    }
    return;
  }
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int r0 = 0; r0 < nparts; r0 += 32) {
    // This lane's chunk weight; lanes past the end hold 0.
    const float wl = r0 + lane < nparts ? ex2f(lp[r0 + lane] - M) : 0.f;
    wsum += wl;
    const int n = min(32, nparts - r0);
    for (int rb = 0; rb < n; rb += kBatch) {
      float v[kBatch][DPL];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float *op = o_part + (head * nsplit + r0 + min(rb + u, n - 1)) * D;
#pragma unroll
        for (int e = 0; e < DPL; ++e) v[u][e] = op[lane + 32 * e];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        // Chunks past the end re-read the last one with weight 0.
        const float wt = __shfl_sync(0xffffffffu, wl, min(rb + u, 31));
        const float w = rb + u < n ? wt : 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, v[u][e], acc[e]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.f / wsum;
#pragma unroll
  for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) lse[head] = (M + log2f(wsum)) * 0.6931471805599453f;
}

template <int D, int GB, int HC>
void launch_split(dim3 grid, cudaStream_t st, const void *q, const void *kp, const void *vp,
                  const int *bt, const int *sl, float *op, float *lp, int Hq, int Hkv, int maxb,
                  int npages, float sl2, int nsplit, int hc, unsigned *status) {
  constexpr int kSmem = DecCfg<HC, D>::SMEM;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(decode_split_kernel<D, GB, HC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSmem);
  });
  decode_split_kernel<D, GB, HC><<<grid, (HC + 1) * 32, kSmem, st>>>(
      static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(kp),
      static_cast<const __nv_bfloat16 *>(vp), bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit,
      hc, status);
}

template <int D, int HC>
bool dispatch_gb(int GB, dim3 grid, cudaStream_t st, const void *q, const void *kp,
                 const void *vp, const int *bt, const int *sl, float *op, float *lp, int Hq,
                 int Hkv, int maxb, int npages, float sl2, int nsplit, int hc, unsigned *status) {
  switch (GB) {
    case 8: launch_split<D, 8, HC>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 4: launch_split<D, 4, HC>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 2: launch_split<D, 2, HC>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
    case 1: launch_split<D, 1, HC>(grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status); return true;
  }
  return false;
}

template <int D>
bool dispatch_split(int HC, int GB, dim3 grid, cudaStream_t st, const void *q, const void *kp,
                    const void *vp, const int *bt, const int *sl, float *op, float *lp, int Hq,
                    int Hkv, int maxb, int npages, float sl2, int nsplit, int hc,
                    unsigned *status) {
  switch (HC) {
    case 8: return dispatch_gb<D, 8>(GB, grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 4: return dispatch_gb<D, 4>(GB, grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 2: return dispatch_gb<D, 2>(GB, grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 1: return dispatch_gb<D, 1>(GB, grid, st, q, kp, vp, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
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

// [status block | o_part (256-byte padded) | l2_part (256-byte padded)].
size_t decode_workspace_bytes(int S, int Hq, int d, int max_blocks) {
  const size_t parts = static_cast<size_t>(S) * Hq * decode_max_splits(max_blocks);
  const size_t o_bytes = (parts * d * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return kDecodeStatusBytes + o_bytes + ((parts * sizeof(float) + 255) & ~static_cast<size_t>(255));
}

DecodeWs decode_ws_layout(void *workspace, int S, int Hq, int d, int max_blocks) {
  const size_t parts = static_cast<size_t>(S) * Hq * decode_max_splits(max_blocks);
  uint8_t *base = static_cast<uint8_t *>(workspace);
  DecodeWs ws;
  ws.status = reinterpret_cast<unsigned *>(base);
  ws.o_part = reinterpret_cast<float *>(base + kDecodeStatusBytes);
  ws.l2_part = reinterpret_cast<float *>(
      base + kDecodeStatusBytes + ((parts * d * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  return ws;
}

attn_status_t launch_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                  const int *block_table, const int *seq_lens, void *o, float *lse,
                                  int S, int Hq, int Hkv, int d, int max_blocks, int num_pages,
                                  float scale, void *workspace, cudaStream_t stream,
                                  unsigned *dev_status) {
  const int G = Hq / Hkv;
  const int GB = (G % 8 == 0) ? 8 : (G % 4 == 0) ? 4 : (G % 2 == 0) ? 2 : 1;
  const int head_chunks = G / GB;
  const int HC = (Hkv % 8 == 0) ? 8 : (Hkv % 4 == 0) ? 4 : (Hkv % 2 == 0) ? 2 : 1;
  const int nsplit = decode_max_splits(max_blocks);
  const DecodeWs ws = decode_ws_layout(workspace, S, Hq, d, max_blocks);
  if (static_cast<long long>(Hkv / HC) * head_chunks > 65535 || S > 65535)
    return ATTN_ERR_UNSUPPORTED;
  dim3 grid(nsplit, S, (Hkv / HC) * head_chunks);
  const float sl2 = scale * 1.4426950408889634f;
  bool ok;
  if (d == 128)
    ok = dispatch_split<128>(HC, GB, grid, stream, q, k_pages, v_pages, block_table, seq_lens,
                             ws.o_part, ws.l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit,
                             head_chunks, ws.status);
  else if (d == 64)
    ok = dispatch_split<64>(HC, GB, grid, stream, q, k_pages, v_pages, block_table, seq_lens,
                            ws.o_part, ws.l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit,
                            head_chunks, ws.status);
  else
    return ATTN_ERR_UNSUPPORTED;
  if (!ok) return ATTN_ERR_UNSUPPORTED;
  return launch_decode_combine(ws, seq_lens, o, lse, S, Hq, d, max_blocks, nsplit,
                               kPagesPerSplit, stream, dev_status);
}

attn_status_t launch_decode_combine(const DecodeWs &ws, const int *seq_lens, void *o, float *lse,
                                    int S, int Hq, int d, int max_blocks, int nsplit,
                                    int pages_per_split, cudaStream_t stream,
                                    unsigned *dev_status) {
  const int heads = S * Hq;
  const int blocks = (heads + 3) / 4;
  // Programmatic dependent launch: the grid may be scheduled while the split
  // kernel before it in the stream finishes; the kernel waits for that grid.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
  cudaError_t err;
  if (d == 128)
    err = cudaLaunchKernelEx(&cfg, decode_combine_kernel<128>, ws.o_part, ws.l2_part, seq_lens,
                             ob, lse, S, Hq, max_blocks, nsplit, pages_per_split, ws.status,
                             dev_status);
  else if (d == 64)
    err = cudaLaunchKernelEx(&cfg, decode_combine_kernel<64>, ws.o_part, ws.l2_part, seq_lens,
                             ob, lse, S, Hq, max_blocks, nsplit, pages_per_split, ws.status,
                             dev_status);
  else
    return ATTN_ERR_UNSUPPORTED;
  if (err != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace exattn
