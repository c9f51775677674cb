// decode_q8.cu -- single-token attention over an 8-bit paged KV cache.
//
// What it computes: the paged decode of decode_paged.cu ("Phase 08" page,
// Concepts: KV cache and paged attention; Lab 03 step 4) over a cache whose K
// and V pages hold 8-bit codes -- FP8 E4M3 or INT8 -- with one fp32 scale per
// (page, K/V head) for K and one for V: the KV-cache quantisation answer of the
// screna.ai interview page (8-bit storage halves the cache against 16 bits;
// group-wise scales; INT8 the safe default, FP8 the hardware format).  The
// element a kernel works with is scale * code, exactly as the fp64 oracle
// dequantises it.
//
// Why it is shaped this way.  The decode reads every cached byte once, so it is
// bound by HBM bandwidth; at one byte per element the bytes halve, and the
// CUDA-core work of the 16-bit kernel (per element: decode, and one FMA per
// query head of the group for q.k and again for p.v) would no longer hide under
// the copy.  So the two contractions of a page run as warp-level m16n8k16 MMAs
// on f16 operands with f32 accumulation, with a page's 16 tokens as the M (or
// K) extent of one tile:
//   S^T[16 tok x 8 heads] = K_page[16 x d] . Q^T[d x 8]          (d/16 MMAs)
//   O^T[d x 8 heads]     += V_page^T[d x 16 tok] . P^T[16 x 8]   (d/16 MMAs)
// E4M3 and INT8 codes convert to f16 exactly (cvt.rn.f16x2.e4m3x2; for INT8
// the byte goes into the mantissa of 1024 and 1152 is subtracted), so the only
// roundings are Q's (bf16 -> f16 after a per-head power-of-two normalisation,
// exact for every element within 2^28 of the head's largest), the p.v
// operand's (f16) and the f32 accumulations.  The page scales are applied in
// f32: the K scale to the scores; the V scale multiplies P before it is
// rounded to f16, relative to the running largest contribution, so the f16
// operand is each token's actual contribution.
//
// Data movement.  At one byte per element a (page, K/V head) slice is only
// 2 KiB, and a stream of such copies was measured to stop near 4 TB/s however
// it was placed or staged.  So the kernel is page-major: one CTA serves up to
// 8 K/V heads of a chunk of a sequence's pages, and each page arrives as one
// TMA box holding all those heads' slices (16 KiB of K, 16 KiB of V at d =
// 128, contiguous in the pool).  The box is 128-byte swizzled (64-byte for d =
// 64), which makes both fragment patterns conflict-free: K rows read along d,
// and V read across token rows at one column.  Each consumer warp owns one
// K/V head and walks the chunk's pages two at a time with a running max / sum
// (online softmax, lazily rescaled): the two pages' loads, conversions and
// MMAs are independent and branch-free, so they interleave, and the softmax
// bookkeeping runs once per 32 tokens.  It writes its heads' normalised
// partials; the combine kernel of decode_paged.cu merges the chunks exactly as
// for the 16-bit cache.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace exattn {
namespace {

constexpr int kPage = 16;
// 32 pages (512 tokens) per chunk, as the 16-bit kernel (same workspace); a
// chunk of 8 K/V heads is 1 MiB of codes.
constexpr int kPagesPerSplitQ8 = 32;
constexpr float kRescaleLog2 = 8.f;  // lazy rescale: move the max only when it grows by > 2^8

template <int D>
constexpr int tile_bytes() { return kPage * D; }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two E4M3 codes in the low 16 bits (element 0 in bits 0-7) -> f16x2 (element 0
// in the low half).  Exact: every E4M3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t w) {
  uint32_t r;
  const uint16_t h = static_cast<uint16_t>(w & 0xffffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}

// INT8 codes enter the MMAs as f16 values 1024 + u with u = code + 128 (the
// code's sign bit flipped, the byte placed in the mantissa of 1024 by one byte
// permute): that is code + kInt8Bias, exactly.  A sum over d of (code + bias)
// * q is the wanted sum plus bias * (sum of q), and a sum over tokens of
// P * (code + bias) the wanted one plus bias * (sum of P); both extra terms are
// formed exactly as the MMAs see their operands and subtracted in f32.
constexpr float kInt8Bias = 1152.f;

__device__ __forceinline__ float f16_lo(uint32_t w) {
  float f;
  asm("{ .reg .f16 h, l; mov.b32 {l, h}, %1; cvt.f32.f16 %0, l; }" : "=f"(f) : "r"(w));
  return f;
}
__device__ __forceinline__ float f16_hi(uint32_t w) {
  float f;
  asm("{ .reg .f16 h, l; mov.b32 {l, h}, %1; cvt.f32.f16 %0, h; }" : "=f"(f) : "r"(w));
  return f;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of logical offset o inside a TMA-swizzled tile (tile base aligned
// to the swizzle span): 128-byte swizzle for 128-byte rows, 64-byte for 64.
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t o) {
  if constexpr (D == 128) return o ^ (((o >> 7) & 7u) << 4);
  else return o ^ (((o >> 7) & 3u) << 4);
}

// The pair of codes (lo = element 0) at bits [16h, 16h+16) of a word -> f16x2.
// INT8 codes come out biased, as code + 1152 (exact in f16): the MMAs take
// them so, and the bias is taken back out of their sums (see kInt8Bias).
template <int FMT>
__device__ __forceinline__ uint32_t codes_f16x2(uint32_t w, int h) {
  if constexpr (FMT == ATTN_KV_E4M3) {
    return e4m3x2_f16x2(h ? (w >> 16) : w);
  } else {
    return prmt(w ^ 0x80808080u, 0x64646464u, h ? 0x4342u : 0x4140u);
  }
}

// V^T fragment pair from two token rows' words A (token t) and B (token t+1):
// element e of each (e = 0..3) gives the pair (A_e, B_e).
template <int FMT>
__device__ __forceinline__ void vpairs(uint32_t A, uint32_t B, uint32_t (&p)[4]) {
  if constexpr (FMT == ATTN_KV_E4M3) {
    const uint32_t lo = prmt(A, B, 0x5140u), hi = prmt(A, B, 0x7362u);
    p[0] = e4m3x2_f16x2(lo);
    p[1] = e4m3x2_f16x2(lo >> 16);
    p[2] = e4m3x2_f16x2(hi);
    p[3] = e4m3x2_f16x2(hi >> 16);
  } else {
    const uint32_t a = A ^ 0x80808080u, b = B ^ 0x80808080u;
    const uint32_t lo = prmt(a, b, 0x5140u), hi = prmt(a, b, 0x7362u);
    p[0] = prmt(lo, 0x64646464u, 0x4140u);  // biased, as in codes_f16x2
    p[1] = prmt(lo, 0x64646464u, 0x4342u);
    p[2] = prmt(hi, 0x64646464u, 0x4140u);
    p[3] = prmt(hi, 0x64646464u, 0x4342u);
  }
}

template <int D>
struct VRow;  // one thread's slice of a V row: D/8 bytes
template <>
struct VRow<128> {
  uint32_t w[4];
};
template <>
struct VRow<64> {
  uint32_t w[2];
};

template <int D>
__device__ __forceinline__ VRow<D> load_vrow(const uint8_t *tile, int row, int g, bool live) {
  VRow<D> r;
  const uint8_t *p = tile + swz<D>(static_cast<uint32_t>(row * D + (D / 8) * g));
  if constexpr (D == 128) {
    const uint4 u = live ? *reinterpret_cast<const uint4 *>(p) : make_uint4(0, 0, 0, 0);
    r.w[0] = u.x; r.w[1] = u.y; r.w[2] = u.z; r.w[3] = u.w;
  } else {
    const uint2 u = live ? *reinterpret_cast<const uint2 *>(p) : make_uint2(0, 0);
    r.w[0] = u.x; r.w[1] = u.y;
  }
  return r;
}

// Workspace and partial layout as in decode_paged.cu (decode_ws_layout): the
// call's status word, o_part [S][Hq][nsplit][D] f32 (normalised), l2_part
// [S][Hq][nsplit] f32 (log2-sum-exp; a tagged NaN marks a failed chunk and
// carries its status bits, which the combine kernel reports).
//
// One CTA per (chunk of kPagesPerSplitQ8 pages, sequence, group of HC K/V
// heads, chunk of GB query heads per K/V head).  Warp HC is the producer: its
// lane 0 TMA-loads, per page, the page's K slices of all HC heads as one box
// (HC x 16 rows x d bytes, contiguous in the pool) and likewise V, into a
// ring of NST stages.  Warp w < HC owns K/V head g0 + w: it walks every page
// of the chunk, keeps its own running max / sum / accumulator, and writes its
// heads' normalised partials; no cross-warp merge.
template <int HC, int D>
struct Q8Cfg {
  static constexpr int SLICE = kPage * D;       // one (page, head) slice of K (or V)
  static constexpr int STAGE = 2 * HC * SLICE;  // K and V of all HC heads of one page
  // Bytes in flight: 6 x 32 KiB for 8 heads (one CTA per SM); more stages
  // for fewer heads, whose CTAs share an SM.
  static constexpr int NST = (HC >= 4) ? 6 : 12;
  static constexpr int SMEM = NST * STAGE + 1024;
};

template <int D, int GB, int FMT, int HC>
__global__ void __launch_bounds__((HC + 1) * 32)
    decode_q8_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __nv_bfloat16 *__restrict__ q, const float *__restrict__ k_scales,
                           const float *__restrict__ v_scales,
                           const int *__restrict__ block_table, const int *__restrict__ seq_lens,
                           float *__restrict__ o_part, float *__restrict__ l2_part, int Hq,
                           int Hkv, int max_blocks, int num_pages, float scale_log2, int nsplit,
                           int head_chunks, unsigned *call_status) {
  // The call's status word starts clear; only the combine kernel, which waits
  // for this whole grid, sets bits in it.
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *call_status = 0;
  grid_dependents_launch();  // the combine kernel may be scheduled behind this grid
  using C = Q8Cfg<HC, D>;
  constexpr int KS = D / 16;   // k-steps of the q.k MMA = M-tiles of the p.v MMA
  constexpr int KCH = D / 64;  // 16-byte chunks of a K row held by one thread
  static_assert(GB >= 1 && GB <= 8, "one n8 tile of heads per warp");
  static_assert(kPagesPerSplitQ8 <= 32, "one block-table entry and one page's scales per lane");
  const int split = blockIdx.x;
  const int s = blockIdx.y;
  const int kvgrp = blockIdx.z / head_chunks;
  const int hchunk = blockIdx.z % head_chunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;  // MMA fragment coordinates
  const int kvh = kvgrp * HC + min(warp, HC - 1);  // this consumer warp's K/V head
  const int h0 = kvh * (Hq / Hkv) + hchunk * GB;   // its first query head

  const int len = seq_lens[s];
  const bool bad_len = len < 0 || len > max_blocks * kPage;
  const int page_begin = split * kPagesPerSplitQ8;
  const int n_pages = bad_len ? 0 : (len + kPage - 1) / kPage;
  if (!bad_len && page_begin >= n_pages) return;  // chunk past the end: nothing to do
  const int npg = bad_len ? 0 : min(n_pages, page_begin + kPagesPerSplitQ8) - page_begin;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[C::NST], empty[C::NST];
  __shared__ int stage_ntok[C::NST];
  __shared__ int sm_pid[kPagesPerSplitQ8];
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
          stage_ntok[st] = min(kPage, len - (page_begin + i) * kPage);
          uint8_t *dst = ring + st * C::STAGE;
          const int z = pid * Hkv + kvgrp * HC;
          mbar_arrive_expect_tx(&full[st], C::STAGE);
          tma_load_3d(dst, &tm_k, &full[st], 0, 0, z);
          tma_load_3d(dst + HC * C::SLICE, &tm_v, &full[st], 0, 0, z);
        }
        issued = i + 1;
      }
      // Let every copy land before the CTA (and its shared memory) goes away.
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        mbar_wait_drain(&full[i % C::NST], (i / C::NST) & 1, &sm_status);
    }
  } else {
    // ------------------------------------------------------------ compute
    // Q^T fragments (the B operand of the q.k MMA) for head n = g: k-step t
    // takes d = (D/4)c + 4t + {0,1} and {2,3}, the same permutation of d the
    // K fragments use.  Each head is scaled by a power of two 2^e (its largest
    // |q| lands in [2^14, 2^15)) before rounding to f16; the scores get
    // scale*log2(e)*2^-e back in f32.
    uint32_t qb[KS][2];
    float sq_own;
    float qsum_own = 0.f;
    {
      float qv[D / 4];
      const bool live = g < GB;
      const __nv_bfloat16 *qp = q + (static_cast<size_t>(s) * Hq + h0 + (live ? g : 0)) * D +
                                (D / 4) * c;
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const uint4 w = live ? *reinterpret_cast<const uint4 *>(qp + 8 * u) : make_uint4(0, 0, 0, 0);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qv[8 * u + 2 * e] = __uint_as_float(ww[e] << 16);
          qv[8 * u + 2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u);
        }
      }
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < D / 4; ++e) amax = fmaxf(amax, fabsf(qv[e]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // ex = 15 - (exponent of amax + 1), so amax * 2^ex lies in [2^14, 2^15);
      // clamped so that 2^ex and 2^-ex are normal floats (exact multipliers).
      int ex = 0;
      if (amax > 0.f && amax <= 3.4028235e38f) {
        const int e_amax = static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127;
        ex = min(100, max(-113, 14 - e_amax));  // subnormal amax: e_amax = -127, clamped
      }
      const float up = __uint_as_float(static_cast<uint32_t>(127 + ex) << 23);
      const float down = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
#pragma unroll
      for (int t = 0; t < KS; ++t) {
        qb[t][0] = pack_f16x2(qv[4 * t] * up, qv[4 * t + 1] * up);
        qb[t][1] = pack_f16x2(qv[4 * t + 2] * up, qv[4 * t + 3] * up);
      }
      sq_own = scale_log2 * down;
      if constexpr (FMT != ATTN_KV_E4M3) {
        // This head's sum of q over d, from the f16 operands themselves.
        float qs = 0.f;
#pragma unroll
        for (int t = 0; t < KS; ++t)
          qs += (f16_lo(qb[t][0]) + f16_hi(qb[t][0])) + (f16_lo(qb[t][1]) + f16_hi(qb[t][1]));
        qs += __shfl_xor_sync(0xffffffffu, qs, 1);
        qs += __shfl_xor_sync(0xffffffffu, qs, 2);
        qsum_own = qs * kInt8Bias;
      }
    }
    // Score multipliers of this thread's two accumulator columns (heads 2c, 2c+1).
    const float sq0 = __shfl_sync(0xffffffffu, sq_own, 8 * c);
    const float sq1 = __shfl_sync(0xffffffffu, sq_own, 8 * c + 4);
    // (INT8) the bias's share of those columns' scores, before the multipliers.
    float qb0 = 0.f, qb1 = 0.f;
    if constexpr (FMT != ATTN_KV_E4M3) {
      qb0 = __shfl_sync(0xffffffffu, qsum_own, 8 * c);
      qb1 = __shfl_sync(0xffffffffu, qsum_own, 8 * c + 4);
    }

    // Page scales: lane i holds those of page i of the chunk.
    float ks_r = 0.f, vs_r = 0.f;
    if (lane < npg) {
      const int pid = sm_pid[lane];
      if (pid >= 0 && pid < num_pages) {
        ks_r = k_scales[static_cast<size_t>(pid) * Hkv + kvh];
        vs_r = v_scales[static_cast<size_t>(pid) * Hkv + kvh];
      }
    }

    // Two running references per head (columns 2c, 2c+1), both lazily moved
    // (only when exceeded by more than 2^8): m for the scores, which normalise
    // the sum l (fp32), and mv for the log2 contribution scale score + log2(V
    // scale), which normalises the f16 operand of the p.v MMA.  The operand is
    // then each token's contribution relative to the largest one, so it stays
    // below 2^9 and underflows only for contributions below 2^-24 of the
    // largest -- not when a page with a large V scale is barely attended.
    // The accumulator holds sum_t 2^(s_t - mv) * vscale_t * code_t, so
    // O = acc * 2^(mv - m) / l.
    float m0 = -INFINITY, m1 = -INFINITY;
    float mv0 = -INFINITY, mv1 = -INFINITY;
    float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
    float acc[KS][4];                      // rows d = (D/8)g + 2i (+1), cols 2c, 2c+1
#pragma unroll
    for (int i = 0; i < KS; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
    // (INT8) sum over tokens of the p.v operand, in the accumulator's columns:
    // the product of an all-ones tile with P^T, so it holds exactly the f16
    // values the p.v MMAs take.
    float psum[4] = {0.f, 0.f, 0.f, 0.f};
    constexpr uint32_t kOnes = 0x3c003c00u;  // f16x2 (1, 1)
    // Source lanes of the P^T fragment: tokens 2c and 2c+1 of head g.
    const int src0 = 8 * c + (g >> 1), src1 = src0 + 4;
    const uint32_t psel = (g & 1) ? 0x7632u : 0x5410u;

    // S^T = K . Q^T of one page for tokens g and g+8, scaled to log2 units and
    // masked past the page's live tokens.  Branch-free, so that two pages'
    // loads, conversions and MMAs interleave: a page with no live token (a bad
    // page id, or the missing partner of an odd last page) reads a stage whose
    // last copy has completed and been consumed, and every score is masked.
    auto page_scores = [&](const uint8_t *kt, int ntok, float ks, float (&sv)[4]) {
      uint4 ka[KCH], kb[KCH];
#pragma unroll
      for (int h = 0; h < KCH; ++h) {
        const uint32_t col = static_cast<uint32_t>((D / 4) * c + 16 * h);
        ka[h] = *reinterpret_cast<const uint4 *>(kt + swz<D>(g * D + col));
        kb[h] = *reinterpret_cast<const uint4 *>(kt + swz<D>((g + 8) * D + col));
      }
      float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < KS; ++t) {
        const uint4 &A = ka[t / 4], &B = kb[t / 4];
        const uint32_t wa = (t % 4 == 0) ? A.x : (t % 4 == 1) ? A.y : (t % 4 == 2) ? A.z : A.w;
        const uint32_t wb = (t % 4 == 0) ? B.x : (t % 4 == 1) ? B.y : (t % 4 == 2) ? B.z : B.w;
        mma_f16((t & 1) ? sd : sc, codes_f16x2<FMT>(wa, 0), codes_f16x2<FMT>(wb, 0),
                codes_f16x2<FMT>(wa, 1), codes_f16x2<FMT>(wb, 1), qb[t][0], qb[t][1]);
      }
      const float kq0 = ks * sq0, kq1 = ks * sq1;
      if constexpr (FMT != ATTN_KV_E4M3) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[e] -= (e & 1) ? qb1 : qb0;
      }
      sv[0] = g < ntok ? (sc[0] + sd[0]) * kq0 : -INFINITY;
      sv[1] = g < ntok ? (sc[1] + sd[1]) * kq1 : -INFINITY;
      sv[2] = g + 8 < ntok ? (sc[2] + sd[2]) * kq0 : -INFINITY;
      sv[3] = g + 8 < ntok ? (sc[3] + sd[3]) * kq1 : -INFINITY;
    };
    auto p_frag = [&](const float (&pv)[4], float f0, float f1, uint32_t &pb0, uint32_t &pb1) {
      const uint32_t P01 = pack_f16x2(pv[0] * f0, pv[1] * f1);
      const uint32_t P23 = pack_f16x2(pv[2] * f0, pv[3] * f1);
      const uint32_t x0 = __shfl_sync(0xffffffffu, P01, src0);
      const uint32_t x1 = __shfl_sync(0xffffffffu, P01, src1);
      const uint32_t y0 = __shfl_sync(0xffffffffu, P23, src0);
      const uint32_t y1 = __shfl_sync(0xffffffffu, P23, src1);
      pb0 = prmt(x0, x1, psel);
      pb1 = prmt(y0, y1, psel);
    };

    for (int i = 0; i < npg; i += 2) {
      const bool two = i + 1 < npg;
      const int sta = i % C::NST, stb = (i + 1) % C::NST;
      bool ok = mbar_wait(&full[sta], (i / C::NST) & 1, &sm_abort, &sm_status);
      if (two) ok = ok && mbar_wait(&full[stb], ((i + 1) / C::NST) & 1, &sm_abort, &sm_status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int na = stage_ntok[sta];
      const int nb = two ? stage_ntok[stb] : 0;
      const float ksa = __shfl_sync(0xffffffffu, ks_r, i);
      const float vsa = __shfl_sync(0xffffffffu, vs_r, i);
      const float ksb = __shfl_sync(0xffffffffu, ks_r, (i + 1) & 31);
      const float vsb_r = __shfl_sync(0xffffffffu, vs_r, (i + 1) & 31);
      const float vsb = two ? vsb_r : 0.f;
      const uint8_t *sga = ring + sta * C::STAGE, *sgb = ring + stb * C::STAGE;
      float sa[4], sb[4];
      page_scores(sga + warp * C::SLICE, na, ksa, sa);
      page_scores(sgb + warp * C::SLICE, nb, ksb, sb);
      const float lva = vsa > 0.f ? __log2f(vsa) : -INFINITY;
      const float lvb = vsb > 0.f ? __log2f(vsb) : -INFINITY;
      const float ma0 = fmaxf(sa[0], sa[2]), ma1 = fmaxf(sa[1], sa[3]);
      const float mb0 = fmaxf(sb[0], sb[2]), mb1 = fmaxf(sb[1], sb[3]);
      float mx0 = fmaxf(ma0, mb0), mx1 = fmaxf(ma1, mb1);
      float cv0 = fmaxf(ma0 + lva, mb0 + lvb), cv1 = fmaxf(ma1 + lva, mb1 + lvb);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        cv0 = fmaxf(cv0, __shfl_xor_sync(0xffffffffu, cv0, o));
        cv1 = fmaxf(cv1, __shfl_xor_sync(0xffffffffu, cv1, o));
      }
      if (__any_sync(0xffffffffu, (mx0 > m0 + kRescaleLog2) || (mx1 > m1 + kRescaleLog2))) {
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        l0 *= ex2(m0 - n0);
        l1 *= ex2(m1 - n1);
        m0 = n0;
        m1 = n1;
      }
      float pa[4], pb[4];
      pa[0] = ex2(sa[0] - m0), pa[1] = ex2(sa[1] - m1), pa[2] = ex2(sa[2] - m0), pa[3] = ex2(sa[3] - m1);
      pb[0] = ex2(sb[0] - m0), pb[1] = ex2(sb[1] - m1), pb[2] = ex2(sb[2] - m0), pb[3] = ex2(sb[3] - m1);
      l0 += (pa[0] + pa[2]) + (pb[0] + pb[2]);
      l1 += (pa[1] + pa[3]) + (pb[1] + pb[3]);
      if (__any_sync(0xffffffffu, (cv0 > mv0 + kRescaleLog2) || (cv1 > mv1 + kRescaleLog2))) {
        const float n0 = fmaxf(mv0, cv0), n1 = fmaxf(mv1, cv1);
        const float a0 = ex2(mv0 - n0), a1 = ex2(mv1 - n1);
#pragma unroll
        for (int i2 = 0; i2 < KS; ++i2) {
          acc[i2][0] *= a0;
          acc[i2][1] *= a1;
          acc[i2][2] *= a0;
          acc[i2][3] *= a1;
        }
        if constexpr (FMT != ATTN_KV_E4M3) {
          psum[0] *= a0;
          psum[1] *= a1;
          psum[2] *= a0;
          psum[3] *= a1;
        }
        mv0 = n0;
        mv1 = n1;
      }
      const float e0 = mv0 == -INFINITY ? 0.f : ex2(m0 - mv0);
      const float e1 = mv1 == -INFINITY ? 0.f : ex2(m1 - mv1);
      uint32_t pa0, pa1, pb0, pb1;
      p_frag(pa, vsa * e0, vsa * e1, pa0, pa1);
      p_frag(pb, vsb * e0, vsb * e1, pb0, pb1);
      if constexpr (FMT != ATTN_KV_E4M3) {
        mma_f16(psum, kOnes, kOnes, kOnes, kOnes, pa0, pa1);
        mma_f16(psum, kOnes, kOnes, kOnes, kOnes, pb0, pb1);
      }
      const uint8_t *vta = sga + (HC + warp) * C::SLICE, *vtb = sgb + (HC + warp) * C::SLICE;
      const VRow<D> va = load_vrow<D>(vta, 2 * c, g, 2 * c < na);
      const VRow<D> vb = load_vrow<D>(vta, 2 * c + 1, g, 2 * c + 1 < na);
      const VRow<D> vc = load_vrow<D>(vta, 2 * c + 8, g, 2 * c + 8 < na);
      const VRow<D> vd = load_vrow<D>(vta, 2 * c + 9, g, 2 * c + 9 < na);
      const VRow<D> wa = load_vrow<D>(vtb, 2 * c, g, 2 * c < nb);
      const VRow<D> wb = load_vrow<D>(vtb, 2 * c + 1, g, 2 * c + 1 < nb);
      const VRow<D> wc = load_vrow<D>(vtb, 2 * c + 8, g, 2 * c + 8 < nb);
      const VRow<D> wd = load_vrow<D>(vtb, 2 * c + 9, g, 2 * c + 9 < nb);
#pragma unroll
      for (int w = 0; w < D / 32; ++w) {
        uint32_t lo[4], hi[4], lo2[4], hi2[4];
        vpairs<FMT>(va.w[w], vb.w[w], lo);
        vpairs<FMT>(vc.w[w], vd.w[w], hi);
        vpairs<FMT>(wa.w[w], wb.w[w], lo2);
        vpairs<FMT>(wc.w[w], wd.w[w], hi2);
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          float t4[4] = {0.f, 0.f, 0.f, 0.f};
          mma_f16(t4, lo[2 * e2], lo[2 * e2 + 1], hi[2 * e2], hi[2 * e2 + 1], pa0, pa1);
          mma_f16(t4, lo2[2 * e2], lo2[2 * e2 + 1], hi2[2 * e2], hi2[2 * e2 + 1], pb0, pb1);
          float(&a)[4] = acc[2 * w + e2];
          a[0] += t4[0];
          a[1] += t4[1];
          a[2] += t4[2];
          a[3] += t4[3];
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[sta]);
        if (two) mbar_arrive(&empty[stb]);
      }
    }

    // Sums over the page tokens (lanes sharing c hold the same heads).
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    // sm_bad / sm_abort are final once every page has been consumed.
    __syncwarp();
    const bool bad = *reinterpret_cast<volatile int *>(&sm_bad) != 0 ||
                     *reinterpret_cast<volatile int *>(&sm_abort) != 0;
    unsigned bits = *reinterpret_cast<volatile unsigned *>(&sm_status) |
                    (*reinterpret_cast<volatile int *>(&sm_bad) ? ATTN_DEV_BAD_PAGE : 0u);
    if (bad && bits == 0) bits = ATTN_DEV_TIMEOUT;  // aborted by a wait that timed out
    if constexpr (FMT != ATTN_KV_E4M3) {
#pragma unroll
      for (int i = 0; i < KS; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = fmaf(-kInt8Bias, psum[e], acc[i][e]);
    }
    // O = acc * 2^(mv - m) / l.
    const float inv0 = (mv0 == -INFINITY ? 0.f : ex2(mv0 - m0)) / l0;
    const float inv1 = (mv1 == -INFINITY ? 0.f : ex2(mv1 - m1)) / l1;
    const int hA = 2 * c, hB = 2 * c + 1;
    const size_t slotA = (static_cast<size_t>(s) * Hq + h0 + hA) * nsplit + split;
    const size_t slotB = (static_cast<size_t>(s) * Hq + h0 + hB) * nsplit + split;
#pragma unroll
    for (int i = 0; i < KS; ++i) {
      const int d0 = (D / 8) * g + 2 * i;
      if (hA < GB)
        *reinterpret_cast<float2 *>(o_part + slotA * D + d0) =
            bad ? make_float2(NAN, NAN) : make_float2(acc[i][0] * inv0, acc[i][2] * inv0);
      if (hB < GB)
        *reinterpret_cast<float2 *>(o_part + slotB * D + d0) =
            bad ? make_float2(NAN, NAN) : make_float2(acc[i][1] * inv1, acc[i][3] * inv1);
    }
    if (g == 0) {
      if (hA < GB) l2_part[slotA] = bad ? failed_partial(bits) : m0 + log2f(l0);
      if (hB < GB) l2_part[slotB] = bad ? failed_partial(bits) : m1 + log2f(l1);
    }
  }
}

// Page pool [num_pages][Hkv][16][D] bytes as a 3-D tensor (D, 16, num_pages*Hkv);
// one box is the page slices of `hc` consecutive K/V heads.
bool make_page_map(CUtensorMap *map, const void *base, int D, long long slices, int hc) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(kPage),
                        static_cast<cuuint64_t>(slices)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(kPage) * D};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(kPage),
                       static_cast<cuuint32_t>(hc)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int GB, int FMT, int HC>
attn_status_t launch_split_q8(dim3 grid, cudaStream_t st, const CUtensorMap &mk,
                              const CUtensorMap &mv, const void *q, const float *ks,
                              const float *vs, const int *bt, const int *sl, float *op, float *lp,
                              int Hq, int Hkv, int maxb, int npages, float sl2, int nsplit, int hc,
                              unsigned *status) {
  using C = Q8Cfg<HC, D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(decode_q8_split_kernel<D, GB, FMT, HC>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  });
  if (attr_err != cudaSuccess) return ATTN_ERR_CUDA;
  decode_q8_split_kernel<D, GB, FMT, HC><<<grid, (HC + 1) * 32, C::SMEM, st>>>(
      mk, mv, static_cast<const __nv_bfloat16 *>(q), ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages,
      sl2, nsplit, hc, status);
  return ATTN_OK;
}

template <int D, int FMT, int HC>
attn_status_t dispatch_gb(int GB, dim3 grid, cudaStream_t st, const CUtensorMap &mk,
                          const CUtensorMap &mv, const void *q, const float *ks, const float *vs,
                          const int *bt, const int *sl, float *op, float *lp, int Hq, int Hkv,
                          int maxb, int npages, float sl2, int nsplit, int hc, unsigned *status) {
  switch (GB) {
    case 8: return launch_split_q8<D, 8, FMT, HC>(grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 4: return launch_split_q8<D, 4, FMT, HC>(grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 2: return launch_split_q8<D, 2, FMT, HC>(grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 1: return launch_split_q8<D, 1, FMT, HC>(grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
  }
  return ATTN_ERR_UNSUPPORTED;
}

template <int D, int FMT>
attn_status_t dispatch_q8(int HC, int GB, dim3 grid, cudaStream_t st, const CUtensorMap &mk,
                          const CUtensorMap &mv, const void *q, const float *ks, const float *vs,
                          const int *bt, const int *sl, float *op, float *lp, int Hq, int Hkv,
                          int maxb, int npages, float sl2, int nsplit, int hc, unsigned *status) {
  switch (HC) {
    case 8: return dispatch_gb<D, FMT, 8>(GB, grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 4: return dispatch_gb<D, FMT, 4>(GB, grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 2: return dispatch_gb<D, FMT, 2>(GB, grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
    case 1: return dispatch_gb<D, FMT, 1>(GB, grid, st, mk, mv, q, ks, vs, bt, sl, op, lp, Hq, Hkv, maxb, npages, sl2, nsplit, hc, status);
  }
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace

attn_status_t launch_decode_paged_q8(const void *q, const void *k_pages, const void *v_pages,
                                     const float *k_scales, const float *v_scales, int kv_format,
                                     const int *block_table, const int *seq_lens, void *o,
                                     float *lse, int S, int Hq, int Hkv, int d, int max_blocks,
                                     int num_pages, float scale, void *workspace,
                                     cudaStream_t stream) {
  const int G = Hq / Hkv;
  const int GB = (G % 8 == 0) ? 8 : (G % 4 == 0) ? 4 : (G % 2 == 0) ? 2 : 1;
  const int head_chunks = G / GB;
  const int HC = (Hkv % 8 == 0) ? 8 : (Hkv % 4 == 0) ? 4 : (Hkv % 2 == 0) ? 2 : 1;
  static_assert(kPagesPerSplitQ8 == 32, "chunks of the shared decode workspace layout");
  const int nsplit = decode_max_splits(max_blocks);
  const DecodeWs ws = decode_ws_layout(workspace, S, Hq, d, max_blocks);
  float *o_part = ws.o_part;
  float *l2_part = ws.l2_part;
  unsigned *status = ws.status;
  if (static_cast<long long>(Hkv / HC) * head_chunks > 65535 || S > 65535)
    return ATTN_ERR_UNSUPPORTED;
  CUtensorMap mk, mv;
  const long long slices = static_cast<long long>(num_pages) * Hkv;
  if (!make_page_map(&mk, k_pages, d, slices, HC) || !make_page_map(&mv, v_pages, d, slices, HC))
    return ATTN_ERR_CUDA;
  dim3 grid(nsplit, S, (Hkv / HC) * head_chunks);
  const float sl2 = scale * 1.4426950408889634f;
  attn_status_t st;
  if (d == 128 && kv_format == ATTN_KV_E4M3)
    st = dispatch_q8<128, ATTN_KV_E4M3>(HC, GB, grid, stream, mk, mv, q, k_scales, v_scales, block_table, seq_lens, o_part, l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else if (d == 128 && kv_format == ATTN_KV_INT8)
    st = dispatch_q8<128, ATTN_KV_INT8>(HC, GB, grid, stream, mk, mv, q, k_scales, v_scales, block_table, seq_lens, o_part, l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else if (d == 64 && kv_format == ATTN_KV_E4M3)
    st = dispatch_q8<64, ATTN_KV_E4M3>(HC, GB, grid, stream, mk, mv, q, k_scales, v_scales, block_table, seq_lens, o_part, l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else if (d == 64 && kv_format == ATTN_KV_INT8)
    st = dispatch_q8<64, ATTN_KV_INT8>(HC, GB, grid, stream, mk, mv, q, k_scales, v_scales, block_table, seq_lens, o_part, l2_part, Hq, Hkv, max_blocks, num_pages, sl2, nsplit, head_chunks, status);
  else
    return ATTN_ERR_UNSUPPORTED;
  if (st != ATTN_OK) return st;
  return launch_decode_combine(ws, seq_lens, o, lse, S, Hq, d, max_blocks, nsplit,
                               kPagesPerSplitQ8, stream, nullptr);
}

}  // namespace exattn
