// prefill_sm100.cu -- bf16 exact attention forward on B200 tensor cores.
//
// What it computes: O = softmax(scale * Q K^T [causal]) V and the logsumexp L
// for every query row, exactly up to float32 rounding ("Phase 08 -- Inference
// Optimization at Depth", Concepts: FlashAttention tiling and online softmax;
// Lab 01 steps 2 and 4).  Q is split into 128-row tiles; each tile walks the
// 128-key K/V tiles keeping a running max m and sum l per row, rescaling the
// accumulator when m grows, and writes O / l and L = m + ln l once.  The N x N
// score matrix exists only one 128 x 128 tile at a time, in tensor memory.
//
// How it maps to sm_100a:
//  * one CTA = 2 Q tiles (256 rows) of one (batch, head); 12 warps:
//      warp 0      TMA producer: Q once, then the K/V tiles, K then V of each,
//                  into a ring of NST shared-memory slots (128B-swizzled, no
//                  multicast); an ALiBi whole pair walks them from the last
//                  down, every other CTA from the first up;
//      warp 1      allocates the 512 TMEM columns and issues every tcgen05.mma
//                  from one thread;
//      warps 4-7   softmax/correction/epilogue for Q tile 0 (TMEM lanes 0-127);
//      warps 8-11  the same for Q tile 1.
//  * TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [384,384+d).
//    P (bf16) overwrites the first 64 columns of its S tile and feeds the
//    second GEMM straight from TMEM, so P never touches shared memory.
//  * S_t = Q_t K^T: 128x128x16 kind::f16 MMAs, both operands K-major.
//    O_t += P_t V: A = P from TMEM, B = V as an MN-major operand.
//  * The two Q tiles ping-pong: while softmax works on S0(j) the tensor pipe
//    runs S1(j) and PV of the other tile, and vice versa.
//  * exp2-based online softmax with scale*log2(e) folded into one FMA and a
//    lazy rescale: the reference max m only moves (and O is rescaled in TMEM)
//    when a row's max grows by more than 8 in log2 units; O/l stays exact.
//    Once m is set, an unmasked tile first takes P against m as it stands and
//    keeps it when the row sums stay at most 255, so most tiles never search
//    for their own max.  ALiBi tiles do so in the downward walk, along which
//    the bias falls.
//  * Causal: KV tiles above the diagonal are never loaded or multiplied; only
//    diagonal tiles are masked (Concepts: causal masking; Lab 01 step 4).
//  * Grid: one CTA per (Q-tile pair, batch*head).  Consecutive CTAs share K/V
//    (same head, or the query heads of one K/V group), so re-reads hit L2;
//    causal grids go heaviest pair first within groups of 8 heads.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace exattn {

namespace {

constexpr int BM = 128;       // query rows per Q tile
constexpr int BN = 128;       // keys per K/V tile
constexpr int NUM_THREADS = 384;
// Registers per thread.  With 72 for the producer/MMA warpgroup the compiler
// spilled there (and the kernel ran 3-4 % slower); 80 leaves the whole-pair
// kernel spill-free, and the softmax rows still fit in 208.
constexpr int kRegsLow = 80;    // per thread, producer/MMA warpgroup
constexpr int kRegsHigh = 208;  // per thread, softmax warpgroups
static_assert(128 * kRegsLow + 256 * kRegsHigh <= NUM_THREADS * 168 && kRegsLow % 8 == 0 &&
                  kRegsHigh % 8 == 0,
              "setmaxnreg split must fit the block's launch registers");
constexpr int kHeadGroup = 8;  // causal schedule: heads whose K/V share L2 at a time
constexpr int kRankMax = NUM_THREADS;  // chunked prefill: sequences ranked by length
constexpr int CHUNK_BYTES = 128 * 128;  // one 128-row x 128-byte swizzle column block

template <int D>
struct Cfg {
  static constexpr int CH = D / 64;                  // 64-element (128 B) column blocks
  static constexpr int TILE_BYTES = BM * D * 2;      // a Q, K or V tile
  static constexpr int NST = (D == 64) ? 8 : 4;      // ring slots
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = RING_OFF + NST * TILE_BYTES;
  static constexpr int XFER_OFF = BAR_OFF + 1024;  // split items: warpgroup 1's m and l per row
  static constexpr int SMEM_BYTES = XFER_OFF + 1024 + 1024;  // + 1 KB align slack
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
};

struct Bars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t q_full;
  uint64_t q_full1;  // whole-pair self-attention: Q tile 1, loaded behind K(jlo)
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mrg_full;     // split item: warpgroup 1's O, m, l are final (128 arrivals)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  void *o;
  float *lse;
  unsigned *status;
  int B, Hq, Hkv, N;
  int pairs;  // ceil(N / 256)
  int whole_pairs;  // split kernel: pair items [whole_pairs, ...) run as two split CTAs each
  float scale_log2;
  int causal;
  int window;            // > 0: key j visible to query i only if i - j < window
  const float *slopes;   // ALiBi slope per query head (kernel variant with the bias)
  // Chunked prefill over a paged cache (kernel variant kPaged): B = sequences;
  // queries token-major [T][Hq][D], sequence s owning rows cu_q[s]..cu_q[s+1]-1
  // at positions seq_lens[s] - qlen_s ...; keys through the block table.
  const int *block_table, *seq_lens, *cu_q;
  int max_blocks, num_pages, T;
};

// Columns cc*32 .. cc*32+31 of one thread's score row -> 16 bf16 pairs of P
// and their part of the row sum: x = s*c - m is one packed FMA per pair, 2^x
// one special-function op per column.  That 2^x is +inf from x = 128 up and
// NaN for a NaN x, so a sum stays finite only when every term is right.
__device__ __forceinline__ void exp_chunk(const uint32_t (&sv)[128], int cc, float2 c2, float2 nm2,
                                          uint32_t *pk, float2 &sum_a, float2 &sum_b) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const int col = cc * 32 + i;
    const float2 x0 = fma2(make_float2(__uint_as_float(sv[col]), __uint_as_float(sv[col + 1])), c2, nm2);
    const float2 x1 = fma2(make_float2(__uint_as_float(sv[col + 2]), __uint_as_float(sv[col + 3])), c2, nm2);
    const float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
    const float2 p1 = make_float2(ex2(x1.x), ex2(x1.y));
    sum_a = add2(sum_a, p0);
    sum_b = add2(sum_b, p1);
    pk[i >> 1] = pack_bf16x2(p0.x, p0.y);
    pk[(i >> 1) + 1] = pack_bf16x2(p1.x, p1.y);
  }
}

// One thread's 128-column score row -> P (bf16 pairs in TMEM at s_addr, over
// the first 64 of the row's S columns) and the row sum of P.
__device__ __forceinline__ float exp_row(const uint32_t (&sv)[128], float c, float m,
                                         uint32_t s_addr) {
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
  float2 sum_a = make_float2(0.f, 0.f), sum_b = make_float2(0.f, 0.f);
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t pk[16];
    exp_chunk(sv, cc, c2, nm2, pk, sum_a, sum_b);
    tmem_st16(s_addr + cc * 16, pk);
  }
  return (sum_a.x + sum_a.y) + (sum_b.x + sum_b.y);
}

// ALiBi: each score s of the row becomes s*c + slope2*col + rb, the scaled
// score plus the bias slope * (key - query) in log2 units (rb: column 0's).
__device__ __forceinline__ void add_alibi(uint32_t (&sv)[128], float c, float slope2, float rb) {
  const float2 c2 = make_float2(c, c), sl2 = make_float2(slope2, slope2), rb2 = make_float2(rb, rb);
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float2 bias = fma2(sl2, make_float2(static_cast<float>(i), static_cast<float>(i + 1)), rb2);
    const float2 x = fma2(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2, bias);
    sv[i] = __float_as_uint(x.x);
    sv[i + 1] = __float_as_uint(x.y);
  }
}

// The same P and row sum kept in registers: TMEM, and with it the S row, is
// left untouched.  (Its ALiBi form below.)
__device__ __forceinline__ float exp_row_held(const uint32_t (&sv)[128], float c, float m,
                                              uint32_t (&pk)[64]) {
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
  float2 sum_a = make_float2(0.f, 0.f), sum_b = make_float2(0.f, 0.f);
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) exp_chunk(sv, cc, c2, nm2, pk + cc * 16, sum_a, sum_b);
  return (sum_a.x + sum_a.y) + (sum_b.x + sum_b.y);
}

// exp_row_held for an ALiBi tile: x = s*c + (slope2*col + rb - m), the bias
// taken into each exponent, so that sv keeps the raw scores.
__device__ __forceinline__ float exp_row_held_alibi(const uint32_t (&sv)[128], float c, float m,
                                                    float slope2, float rb, uint32_t (&pk)[64]) {
  const float2 c2 = make_float2(c, c), sl2 = make_float2(slope2, slope2);
  const float2 b2 = make_float2(rb - m, rb - m);
  float2 sum_a = make_float2(0.f, 0.f), sum_b = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 128; i += 4) {
    const float2 o0 = fma2(sl2, make_float2(static_cast<float>(i), static_cast<float>(i + 1)), b2);
    const float2 o1 = fma2(sl2, make_float2(static_cast<float>(i + 2), static_cast<float>(i + 3)), b2);
    const float2 x0 = fma2(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2, o0);
    const float2 x1 = fma2(make_float2(__uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3])), c2, o1);
    const float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
    const float2 p1 = make_float2(ex2(x1.x), ex2(x1.y));
    sum_a = add2(sum_a, p0);
    sum_b = add2(sum_b, p1);
    pk[i >> 1] = pack_bf16x2(p0.x, p0.y);
    pk[(i >> 1) + 1] = pack_bf16x2(p1.x, p1.y);
  }
  return (sum_a.x + sum_a.y) + (sum_b.x + sum_b.y);
}

template <int D, bool kAlibi, bool kPaged, bool kSplit>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_k1,
                        const __grid_constant__ CUtensorMap tm_v1, const Params p) {
  using C = Cfg<D>;
  // An ALiBi whole-pair self-attention CTA walks its KV tiles from the last
  // to the first: the bias then falls along the walk, so that later tiles can
  // keep P against the running max.  (The other CTAs walk up from the first:
  // walking down made the causal and GQA launches about 3 % slower.)
  constexpr bool kRev = kAlibi && !kPaged && !kSplit;
  // The split CTAs of a launch come as a second grid, programmatically
  // dependent on this one: it may be scheduled on the SMs this grid frees.
  if constexpr (!kPaged && !kSplit) grid_dependents_launch();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + C::Q_OFF;
  uint8_t *sRing = smem + C::RING_OFF;
  Bars *bars = reinterpret_cast<Bars *>(smem + C::BAR_OFF);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: Q-tile pair and (batch, head).  Non-causal: head-major, so
  // the CTAs resident at one time share a few heads' K/V in L2.  Causal: groups
  // of kHeadGroup heads, heaviest pairs first inside each group (load balance)
  // while a group's K/V stays in L2.
  const int BH = p.B * p.Hq;
  int pair, bh;
  // The split variant (kSplit) runs split CTAs only: one Q tile (split_tile
  // of its pair) whose KV tiles are halved over the two softmax warpgroups --
  // both hold the same rows -- and merged at the end.  It is launched behind
  // the whole pairs for the pairs that did not fill a last wave (see launch).
  int split_tile = -1;
  if constexpr (kPaged) {
    // Chunked prefill: a CTA's work grows with its sequence's key count, which
    // varies by up to the longest context over the shortest.  The grid takes
    // the sequences longest first (ranked here by key count, ties by index),
    // each one's heaviest pair first, all heads of a pair together, so that
    // the last wave holds the short ones.  Past kRankMax sequences the order
    // stays as given (the grid is then large enough to balance by itself).
    const int lin = static_cast<int>(blockIdx.x);
    const int per_seq = p.pairs * p.Hq;
    const int r = lin / per_seq;
    const int rem = lin - r * per_seq;
    pair = p.pairs - 1 - rem / p.Hq;
    int seq = r;
    if (p.B <= kRankMax) {
      __shared__ int s_len[kRankMax];
      __shared__ int s_seq;
      const int t = static_cast<int>(threadIdx.x);
      if (t < p.B) s_len[t] = p.seq_lens[t];
      __syncthreads();
      if (t < p.B) {
        const int nt = s_len[t];
        int rank = 0;
        for (int u = 0; u < p.B; ++u) rank += (s_len[u] > nt) || (s_len[u] == nt && u < t);
        if (rank == r) s_seq = t;
      }
      __syncthreads();
      seq = s_seq;
    }
    bh = seq * p.Hq + rem % p.Hq;
  } else {
    int lin = static_cast<int>(blockIdx.x);
    if constexpr (kSplit) {
      split_tile = lin & 1;
      lin = p.whole_pairs + (lin >> 1);
    }
    if (!p.causal) {
      bh = lin / p.pairs;
      pair = lin % p.pairs;
    } else {
      const int grp = lin / (kHeadGroup * p.pairs);
      const int first = grp * kHeadGroup;
      const int hg = min(kHeadGroup, BH - first);
      const int rr = lin - grp * kHeadGroup * p.pairs;
      pair = p.pairs - 1 - rr / hg;
      bh = first + rr % hg;
    }
  }
  const int b = bh / p.Hq;
  const int hq = bh % p.Hq;
  const int hkv = hq / (p.Hq / p.Hkv);
  const int row0 = pair * 2 * BM + (split_tile > 0 ? BM : 0);
  // Rows of this (batch, head) or sequence chunk (nq), keys (nk), and the
  // position of row 0 among the keys (ctx: 0 for self-attention; for a chunk,
  // its queries are the last nq of the sequence's nk positions).
  int nq = p.N, nk = p.N, ctx = 0, qrow0 = 0;
  if constexpr (kPaged) {
    const int q0 = p.cu_q[b], q1 = p.cu_q[b + 1];
    nk = p.seq_lens[b];
    nq = q1 - q0;
    qrow0 = q0;
    // (For a chunk, p.N is the caller's bound max_q on every chunk length; the
    // grid covers it.)
    const bool bad_len = q0 < 0 || nq < 0 || q1 > p.T || nk < nq || nk > p.max_blocks * 16 ||
                         nq > p.N;
    if (bad_len) {
      if (threadIdx.x == 0 && pair == 0 && hq == 0) atomicOr(p.status, ATTN_DEV_BAD_PAGE);
      return;
    }
    if (row0 >= nq) return;  // pair past the chunk: nothing to do
    ctx = nk - nq;
  }
  if (split_tile >= 0 && row0 >= nq) return;  // split CTA of a Q tile past the rows
  const int nkv = (nk + BN - 1) / BN;
  // KV tiles [js_t, je_t) of each Q tile: the causal diagonal caps the end,
  // a sliding window moves the start; a Q tile past the rows has none.
  // (Scalars, not arrays: the issuing thread reads them every iteration.)
  const bool rows1 = split_tile < 0 && row0 + BM < nq;
  int je0, je1, js0, js1;
  if constexpr (kPaged) {  // the diagonal sits ctx keys to the right
    const int last0 = min(row0 + BM, nq) - 1, last1 = min(row0 + 2 * BM, nq) - 1;
    je0 = p.causal ? min((ctx + last0) / BN + 1, nkv) : nkv;
    je1 = !rows1 ? 0 : (p.causal ? min((ctx + last1) / BN + 1, nkv) : nkv);
    js0 = p.window > 0 ? max(0, ctx + row0 - p.window + 1) / BN : 0;
    js1 = (!rows1 || p.window <= 0) ? 0 : max(0, ctx + row0 + BM - p.window + 1) / BN;
  } else {
    je0 = p.causal ? min(row0 / BN + 1, nkv) : nkv;
    je1 = !rows1 ? 0 : (p.causal ? min((row0 + BM) / BN + 1, nkv) : nkv);
    js0 = p.window > 0 ? max(0, row0 - p.window + 1) / BN : 0;
    js1 = (!rows1 || p.window <= 0) ? 0 : max(0, row0 + BM - p.window + 1) / BN;
  }
  // A split CTA's one Q tile: its KV range halved (the first half the larger);
  // a single KV tile stays on warpgroup 0.
  bool split = false;  // (always false in the whole-pair kernel)
  int mid = 0;
  if (kSplit && je0 - js0 >= 2) {
    split = true;
    mid = js0 + (je0 - js0 + 1) / 2;
    js1 = mid;
    je1 = je0;
    je0 = mid;
  }
  const int jlo = js0;
  const int jhi = max(je0, je1);
  if constexpr (kPaged) {
    // Every page the tiles [jlo, jhi) read must be in the pool; a sequence
    // with a bad entry gets NaN rows and the status bit, and no copy is issued.
    const int pg_end = min(jhi * (BN / 16), (nk + 15) / 16);
    bool bad = false;
    for (int i = jlo * (BN / 16) + static_cast<int>(threadIdx.x); i < pg_end; i += NUM_THREADS) {
      const int pid = p.block_table[static_cast<size_t>(b) * p.max_blocks + i];
      bad |= pid < 0 || pid >= p.num_pages;
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(p.status, ATTN_DEV_BAD_PAGE);
      for (int idx = threadIdx.x; idx < 2 * BM * (D + 1); idx += NUM_THREADS) {
        const int r = idx / (D + 1), c = idx % (D + 1);
        const int row = row0 + r;
        if (row >= nq) continue;
        const size_t tok = static_cast<size_t>(qrow0 + row) * p.Hq + hq;
        if (c < D)
          reinterpret_cast<__nv_bfloat16 *>(p.o)[tok * D + c] = __float2bfloat16_rn(NAN);
        else
          p.lse[tok] = NAN;
      }
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_full1, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], BM);
      mbar_init(&bars->o_full[t], 1);
    }
    mbar_init(&bars->mrg_full, BM);
    mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // Registers (set inside each role's branch): the producer/MMA warpgroup needs
  // few, the softmax warpgroups hold a 128-column score row each.
  // 128*kRegsLow + 256*kRegsHigh fits the block's launch budget of 384*168.

  if (warp == 0) {
    // ================================================================ producer
    regs_dec<kRegsLow>();
    if constexpr (kPaged) {
      // The whole warp gathers: lane 0 runs the barrier protocol and the Q
      // copies, lanes 0-7 each bring one page of every K/V tile, so the eight
      // block-table reads and sixteen or more box copies per tile proceed in
      // parallel.
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_k1);
        tma_prefetch_desc(&tm_v1);
        mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE_BYTES);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(sQ + t * C::TILE_BYTES + c * CHUNK_BYTES, &tm_q, &bars->q_full, 64 * c,
                        hq, qrow0 + row0 + t * BM);
      }
      int issued = 0;
      for (int i = 0; i < 2 * (jhi - jlo); ++i) {
        const int slot = i % C::NST;
        const int round = i / C::NST;
        bool go = true;
        if (lane == 0 && round > 0)
          go = mbar_wait(&bars->empty[slot], (round - 1) & 1, abort_flag, p.status);
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
#ifdef EXATTN_TEST_WITHHOLD
        // Test build only: stop before ring index EXATTN_TEST_WITHHOLD, arriving
        // on nothing and copying nothing, so the consumers' waits run out.
        if (i == EXATTN_TEST_WITHHOLD) break;
#endif
        if (lane == 0) mbar_arrive_expect_tx(&bars->full[slot], C::TILE_BYTES);
        __syncwarp();
        if (lane < BN / 16) {
          // Page `lane` of the tile: a whole page as one 16-row box per 64
          // columns; the last, partly filled page row by row; rows past the
          // keys from an out-of-range coordinate, i.e. zeros (never stale
          // shared memory, which a zero P could not cancel if it held a NaN).
          const CUtensorMap *map = (i & 1) ? &tm_v : &tm_k;
          const CUtensorMap *map1 = (i & 1) ? &tm_v1 : &tm_k1;
          const int key0 = (jlo + (i >> 1)) * BN + lane * 16;
          const int ntok = min(16, nk - key0);
          const int z = ntok > 0
              ? p.block_table[static_cast<size_t>(b) * p.max_blocks + key0 / 16] * p.Hkv + hkv
              : -1;
          uint8_t *dst = sRing + slot * C::TILE_BYTES + lane * 16 * 128;
          for (int c = 0; c < C::CH; ++c) {
            if (ntok >= 16 || ntok <= 0) {
              tma_load_3d(dst + c * CHUNK_BYTES, map, &bars->full[slot], 64 * c, 0, z);
            } else {
              for (int r = 0; r < 16; ++r)
                tma_load_3d(dst + c * CHUNK_BYTES + r * 128, map1, &bars->full[slot], 64 * c, r,
                            r < ntok ? z : -1);
            }
          }
        }
        issued = i + 1;
      }
      // Drain: no copy may still be writing shared memory when the CTA exits.
      if (lane == 0) {
        mbar_wait_drain(&bars->q_full, 0, p.status);
        for (int i = max(0, issued - C::NST); i < issued; ++i)
          mbar_wait_drain(&bars->full[i % C::NST], (i / C::NST) & 1, p.status);
      }
    } else if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int zq = b * p.Hq + hq;
      const int zkv = b * p.Hkv + hkv;
      // A whole pair loads Q tile 0 here and Q tile 1 behind K(jlo), on a
      // barrier of its own, so the first score MMA waits for two tiles, not
      // three.  A split CTA's two warpgroups share its one Q tile (both slots).
      constexpr bool kQ2 = !kSplit;
      mbar_arrive_expect_tx(&bars->q_full, (kQ2 ? 1 : 2) * C::TILE_BYTES);
      for (int t = 0; t < (kQ2 ? 1 : 2); ++t)
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sQ + t * C::TILE_BYTES + c * CHUNK_BYTES, &tm_q, &bars->q_full, 64 * c,
                      row0 + (kSplit && split ? 0 : t * BM), zq);
      // Ring entries in the order the MMA issuer consumes them.  Whole pair:
      // K(jlo), then V(j) K(j+1) per KV tile j (both Q tiles use each).  Split:
      // K0(0) K1(0), then per step s V0(s) K0(s+1) V1(s) K1(s+1), where tile 0
      // walks the KV tiles from jlo and tile 1 from mid (one fewer, at most).
      int sst = 0, sph = 0;  // split walk: step, and position within the step
      auto entry = [&](int i, bool &v, int &kv) {
        if (!split) {
          v = (i & 1) != 0;
          kv = kRev ? jhi - 1 - (i >> 1) : jlo + (i >> 1);
          return;
        }
        if (i < 2) {
          v = false;
          kv = i == 0 ? jlo : mid;
          return;
        }
        const int n0 = mid - jlo, n1 = jhi - mid;
        while (true) {
          const int st = sst, ph = sph;
          if (++sph == 4) {
            sph = 0;
            ++sst;
          }
          if (ph == 0) { v = true; kv = jlo + st; return; }
          if (ph == 1 && st + 1 < n0) { v = false; kv = jlo + st + 1; return; }
          if (ph == 2 && st < n1) { v = true; kv = mid + st; return; }
          if (ph == 3 && st + 1 < n1) { v = false; kv = mid + st + 1; return; }
        }
      };
      int issued = 0;
      if constexpr (kQ2) {
        // Ring entry 0, K(jlo), then Q tile 1: S0's operands arrive first.
        mbar_arrive_expect_tx(&bars->full[0], C::TILE_BYTES);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sRing + c * CHUNK_BYTES, &tm_k, &bars->full[0], 64 * c,
                      (kRev ? jhi - 1 : jlo) * BN, zkv);
        mbar_arrive_expect_tx(&bars->q_full1, C::TILE_BYTES);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sQ + C::TILE_BYTES + c * CHUNK_BYTES, &tm_q, &bars->q_full1, 64 * c,
                      row0 + BM, zq);
        issued = 1;
      }
      for (int i = issued; i < 2 * (jhi - jlo); ++i) {
        const int slot = i % C::NST;
        const int round = i / C::NST;
        if (round > 0 && !mbar_wait(&bars->empty[slot], (round - 1) & 1, abort_flag, p.status))
          break;
#ifdef EXATTN_TEST_WITHHOLD
        // Test build only: stop before ring index EXATTN_TEST_WITHHOLD, arriving
        // on nothing and copying nothing, so the consumers' waits run out.
        if (i == EXATTN_TEST_WITHHOLD) break;
#endif
        mbar_arrive_expect_tx(&bars->full[slot], C::TILE_BYTES);
        bool ev;
        int kv;
        entry(i, ev, kv);
        const CUtensorMap *map = ev ? &tm_v : &tm_k;
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sRing + slot * C::TILE_BYTES + c * CHUNK_BYTES, map, &bars->full[slot],
                      64 * c, kv * BN, zkv);
        issued = i + 1;
      }
      // Drain: no copy may still be writing shared memory when the CTA exits.
      // Normally these phases completed long ago and each wait returns at once.
      mbar_wait_drain(&bars->q_full, 0, p.status);
      if (kQ2) mbar_wait_drain(&bars->q_full1, 0, p.status);
      for (int i = max(0, issued - C::NST); i < issued; ++i)
        mbar_wait_drain(&bars->full[i % C::NST], (i / C::NST) & 1, p.status);
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    regs_dec<kRegsLow>();
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t ring_base = smem_u32(sRing);
      auto slot_of = [](int i) { return i % C::NST; };
      auto wait_full = [&](int i) {
        return mbar_wait(&bars->full[i % C::NST], (i / C::NST) & 1, abort_flag, p.status);
      };
      // Descriptors are built once; per MMA only the start-address field moves
      // (smem addresses stay below 256 KB, so adding addr>>4 never carries out
      // of the 14-bit field).  This keeps the issuing thread's instruction
      // stream short enough to feed one MMA per 64 cycles.
      const uint64_t qdesc0 = sdesc_sw128(q_base, 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(ring_base, 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(ring_base, CHUNK_BYTES, 1024);
      const uint32_t idesc_qk = C::IDESC_QK, idesc_pv = C::IDESC_PV;
      auto issue_s = [&](int t, int kidx) {  // S_t = Q_t K^T
        const uint64_t qd = qdesc0 + ((t * C::TILE_BYTES) >> 4);
        const uint64_t kd = kdesc0 + ((slot_of(kidx) * C::TILE_BYTES) >> 4);
        const uint32_t d_tmem = tmem + t * 128;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * CHUNK_BYTES + (ks & 3) * 32) >> 4;
          mma_ss(d_tmem, qd + off, kd + off, idesc_qk, ks > 0);
        }
      };
      auto issue_pv = [&](int t, int vidx, bool acc) {  // O_t (+)= P_t V
        const uint64_t vd = vdesc0 + ((slot_of(vidx) * C::TILE_BYTES) >> 4);
        const uint32_t d_tmem = tmem + 256 + t * 128, a_tmem = tmem + t * 128;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_ts(d_tmem, a_tmem + ks * 8, vd + ((ks * 16 * 128) >> 4), idesc_pv,
                 (acc || ks > 0) ? 1u : 0u);
      };

      // K/V tile j of this CTA sits at ring index 2*(j - jlo) (K) and +1 (V).
      auto has = [&](int t, int j) {
        return t == 0 ? (j >= js0 && j < je0) : (j >= js1 && j < je1);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, p.status);
      ok = ok && wait_full(0);
      if (kSplit && split) {
        // Split CTA: tile t walks its own half of the KV tiles, so each ring
        // entry feeds one MMA group and is released right after it, in the
        // producer's order: K0(0) K1(0), then V0(s) K0(s+1) V1(s) K1(s+1).
        const int n0 = mid - jlo, n1 = jhi - mid;
        int e = 0;
        if (ok) {
          tc_fence_after();
          issue_s(0, e);
          tc_commit(&bars->s_full[0]);
          tc_commit(&bars->empty[slot_of(e++)]);
          ok = wait_full(e);
        }
        if (ok) {
          tc_fence_after();
          issue_s(1, e);
          tc_commit(&bars->s_full[1]);
          tc_commit(&bars->empty[slot_of(e++)]);
        }
        for (int st = 0; ok && st < n0; ++st) {
          if (!(ok = mbar_wait(&bars->p_full[0], st & 1, abort_flag, p.status) && wait_full(e)))
            break;
          tc_fence_after();
          issue_pv(0, e, st > 0);
          tc_commit(&bars->o_full[0]);
          tc_commit(&bars->empty[slot_of(e++)]);
          if (st + 1 < n0) {
            if (!(ok = wait_full(e))) break;
            tc_fence_after();
            issue_s(0, e);  // in order after PV0(st), which read P0 there
            tc_commit(&bars->s_full[0]);
            tc_commit(&bars->empty[slot_of(e++)]);
          }
          if (st < n1) {
            if (!(ok = mbar_wait(&bars->p_full[1], st & 1, abort_flag, p.status) && wait_full(e)))
              break;
            tc_fence_after();
            issue_pv(1, e, st > 0);
            tc_commit(&bars->o_full[1]);
            tc_commit(&bars->empty[slot_of(e++)]);
          }
          if (st + 1 < n1) {
            if (!(ok = wait_full(e))) break;
            tc_fence_after();
            issue_s(1, e);
            tc_commit(&bars->s_full[1]);
            tc_commit(&bars->empty[slot_of(e++)]);
          }
        }
      } else {
        // KV tile of walk step rj (upward from jlo, or downward from jhi - 1),
        // and a tile's step count within its own range.
        auto walk_j = [&](int rj) { return kRev ? jhi - 1 - rj : jlo + rj; };
        auto step0 = [&](int j) { return kRev ? je0 - 1 - j : j - js0; };
        auto step1 = [&](int j) { return kRev ? je1 - 1 - j : j - js1; };
        const int nwalk = jhi - jlo;
        if (ok) {
          tc_fence_after();
          if (has(0, walk_j(0))) {
            issue_s(0, 0);
            tc_commit(&bars->s_full[0]);
          }
          if constexpr (!kPaged && !kSplit) {
            // Q tile 1 arrives behind the first K tile on its own barrier.
            ok = mbar_wait(&bars->q_full1, 0, abort_flag, p.status);
            tc_fence_after();
          }
          if (ok && has(1, walk_j(0))) {
            issue_s(1, 0);
            tc_commit(&bars->s_full[1]);
          }
          if (ok) tc_commit(&bars->empty[slot_of(0)]);
        }
        for (int rj = 0; ok && rj < nwalk; ++rj) {
          const int j = walk_j(rj);
          const bool more = rj + 1 < nwalk;
          const int jn = more ? walk_j(rj + 1) : -1;  // the next tile of the walk
          // The ring entries this iteration reads, V(j) and K(jn), are checked
          // before the waits for P: their barrier latency then falls in time
          // the issuing thread spends waiting anyway, not between a P and the
          // MMAs that consume it.
          if (!(ok = wait_full(2 * rj + 1))) break;
          if (more && !(ok = wait_full(2 * rj + 2))) break;
          if (has(0, j)) {
            const int st = step0(j);
            if (!(ok = mbar_wait(&bars->p_full[0], st & 1, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(0, 2 * rj + 1, st > 0);
            tc_commit(&bars->o_full[0]);
          }
          if (more && has(0, jn)) {
            // P0(j) aliases S0.  tcgen05.mma ops issued by one thread execute in
            // order, so S0(jn) overwrites the P0(j) columns only after PV0(j),
            // issued just before, has consumed them: no completion wait needed.
            issue_s(0, 2 * rj + 2);
            tc_commit(&bars->s_full[0]);
          }
          if (has(1, j)) {
            const int st = step1(j);
            if (!(ok = mbar_wait(&bars->p_full[1], st & 1, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(1, 2 * rj + 1, st > 0);
            tc_commit(&bars->o_full[1]);
          }
          tc_commit(&bars->empty[slot_of(2 * rj + 1)]);  // V(j) no longer needed
          if (more && has(1, jn)) {
            issue_s(1, 2 * rj + 2);  // in order after PV1(j), as for tile 0
            tc_commit(&bars->s_full[1]);
          }
          if (more) tc_commit(&bars->empty[slot_of(2 * rj + 2)]);  // K(jn) done
        }
      }
      // Every MMA issued above must finish before TMEM is released.
      tc_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, p.status);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle members of the first warpgroup
  } else {
    // ====================================================== softmax / epilogue
    regs_inc<kRegsHigh>();
    const int t = (warp - 4) >> 2;        // Q tile of this warpgroup
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;    // row within the Q tile
    // (In a split CTA both warpgroups hold the rows of its one Q tile.)
    const int row = row0 + (kSplit && split ? 0 : t * BM) + r;
    const int jst = t == 0 ? js0 : js1, jen = t == 0 ? je0 : je1;
    const int nt = jen - jst;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + t * 128;
    const uint32_t o_addr = tmem + lane_off + 256 + t * 128;
    const float c = p.scale_log2;
    // ALiBi slope in log2 units; the bias slope * (key - query) joins the score
    // before the row max.
    const float slope2 = kAlibi ? p.slopes[hq] * 1.4426950408889634f : 0.f;
    float m = -INFINITY;  // reference max, in log2 units of scaled scores
    float l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < nt; ++jj) {
      const int j = kRev ? jen - 1 - jj : jst + jj;  // the walk order of the MMAs
      // Visible columns [lo, hi) of this row in KV tile j: the end of the keys,
      // the causal diagonal and the sliding window.  (Worked out, with the
      // path the tile takes, before the scores arrive.)
      int hi = min(BN, nk - j * BN);
      if (p.causal) hi = min(hi, ctx + row - j * BN + 1);
      // (Rows past the last take the last real row's window so that they never
      // force the masked path on a warp whose real rows need none.)
      const int lo = p.window > 0 ? ctx + min(row, nq - 1) - p.window + 1 - j * BN : 0;
      // Only diagonal, window-edge and last tiles carry masked columns;
      // elsewhere the warp takes the branch-free path.
      const bool masked = !__all_sync(0xffffffffu, lo <= 0 && hi >= BN);
      const bool attempt = (!kAlibi || kRev) && !masked && jj > 0 &&
                           __all_sync(0xffffffffu, m != -INFINITY);
      ok = mbar_wait(&bars->s_full[t], jj & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // The whole 128-column score row of this thread, in one TMEM load.
      uint32_t sv[128];
      tmem_ld128(s_addr, sv);
      tmem_ld_wait128(sv);
      // ALiBi: the bias of key column 0 (the slope per column is slope2).
      const float rb = kAlibi ? slope2 * static_cast<float>(j * BN - (ctx + row)) : 0.f;
      const float cx = kAlibi ? 1.0f : c;  // factor still to apply to sv in the exponent
      if (masked) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < lo || i >= hi) sv[i] = 0xff800000u;  // -inf
      }
      // Once every row of the warp has a finite reference max, an unmasked tile
      // first computes P against that max without looking for the tile's own
      // max.  If every row's P sums to at most 255, every x = s*c - m is below
      // 8 and no term overflowed: m stays the reference (the max-first step
      // below would keep it too, as it moves m only past m + 8), and P and
      // its sum are written to TMEM and l as they stand.  Otherwise the S row
      // is read back from TMEM, which the attempt left untouched, and the tile
      // takes the max-first step, which then also moves a row that missed up
      // to its running max, so that a max left low by a window's first tile
      // does not miss again.  Masked tiles take the max-first step at once:
      // their scores in registers are no longer those in TMEM.  An ALiBi
      // tile's attempt adds the bias inside each exponent, leaving the scores
      // raw, and the max-first step adds it to the row; in an upward walk,
      // where the bias rises from tile to tile and the attempt would miss
      // most, ALiBi tiles go max first at once.
      bool fast = false, missed = false;
      if (attempt) {
        uint32_t pk[64];
        const float l_tile = kAlibi ? exp_row_held_alibi(sv, c, m, slope2, rb, pk)
                                    : exp_row_held(sv, c, m, pk);
        missed = !(l_tile <= 255.0f);
        fast = !__any_sync(0xffffffffu, missed);
        if (fast) {
          l += l_tile;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            tmem_st16(s_addr + cc * 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + cc * 16));
          // The step below is skipped on this path: tell the compiler that the
          // scores are dead here, so that it keeps no copy of them alive across
          // the exponentials above.
#pragma unroll
          for (int i = 0; i < 128; ++i) asm("" : "=r"(sv[i]));
        } else {
          tmem_ld128(s_addr, sv);
          tmem_ld_wait128(sv);
        }
      }
      if (!fast) {
        if (kAlibi) add_alibi(sv, c, slope2, rb);  // (a masked -inf stays -inf)
        float mx;
        {
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 128; i += 8) {
            m0 = fmax3(m0, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
            m1 = fmax3(m1, __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]));
            m2 = fmax3(m2, __uint_as_float(sv[i + 4]), __uint_as_float(sv[i + 5]));
            m3 = fmax3(m3, __uint_as_float(sv[i + 6]), __uint_as_float(sv[i + 7]));
          }
          mx = fmax3(m0, m1, fmaxf(m2, m3));
        }
        const float m_new = fmaxf(m, mx * cx);
        const bool resc = m_new > m + 8.0f || (missed && m_new > m);
        const float alpha = resc ? ex2(m - m_new) : 1.0f;
        if (resc) m = m_new;
        l *= alpha;
        // A row that has seen no visible key yet (a window edge) keeps m = -inf;
        // its masked scores must still give P = 0, not -inf - (-inf).
        const float m_use = (m == -INFINITY) ? 0.f : m;
        // P = 2^(s*c - m), rounded to bf16 and written over the (already read) S
        // columns; the row sum stays in fp32.
        l += exp_row(sv, cx, m_use, s_addr);
        if (jj > 0 && __any_sync(0xffffffffu, resc)) {
          // Lazy rescale of O (rare once the max settles).  O is stable here:
          // this tile's S completing implies the previous PV completed, and
          // this tile's PV waits for p_full.
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            tmem_ld32(o_addr + cc * 32, ov);
            tmem_ld_wait(ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(o_addr + cc * 32, ov);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[t]);
    }
    if (ok && nt > 0) {
      ok = mbar_wait(&bars->o_full[t], (nt - 1) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (kSplit && ok && split && t == 1) {
        // Warpgroup 0 merges: it reads this O tile from TMEM itself (a warp may
        // address every column of its lane quarter), and m, l from here.
        reinterpret_cast<float2 *>(smem + C::XFER_OFF)[r] = make_float2(m, l);
        tc_fence_before();
        mbar_arrive(&bars->mrg_full);
        ok = false;  // nothing more for this warpgroup
      }
      float a0 = 1.f, a1 = 0.f;  // weights of this O tile and (split) of the other
      if (kSplit && ok && split) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->mrg_full, 0, abort_flag, p.status));
        if (ok) {
          tc_fence_after();
          // Two partial results of one row over disjoint keys: the joint max
          // and sum, each accumulator weighted by 2^(its reference - the joint).
          const float2 ml1 = reinterpret_cast<const float2 *>(smem + C::XFER_OFF)[r];
          const float mm = fmaxf(m, ml1.x);
          a0 = ex2(m - mm);
          a1 = ex2(ml1.x - mm);
          l = a0 * l + a1 * ml1.y;
          m = mm;
        }
      }
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        a0 *= inv_l;
        a1 *= inv_l;
        const uint32_t o1_addr = tmem + lane_off + 256 + 128;
        const bool valid = row < nq;
        // Row of O and L: [B][Hq][N] for self-attention, [T][Hq] for a chunk.
        const size_t orow_idx =
            kPaged ? static_cast<size_t>(qrow0 + (valid ? row : 0)) * p.Hq + hq
                   : (static_cast<size_t>(b) * p.Hq + hq) * p.N + (valid ? row : 0);
        __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + orow_idx * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(o_addr + cc * 32, ov);
          tmem_ld_wait(ov);
          uint32_t pk[16];
          if (kSplit && split) {
            uint32_t ov1[32];
            tmem_ld32(o1_addr + cc * 32, ov1);
            tmem_ld_wait(ov1);
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              pk[i >> 1] = pack_bf16x2(
                  fmaf(__uint_as_float(ov[i]), a0, __uint_as_float(ov1[i]) * a1),
                  fmaf(__uint_as_float(ov[i + 1]), a0, __uint_as_float(ov1[i + 1]) * a1));
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              pk[i >> 1] = pack_bf16x2(__uint_as_float(ov[i]) * a0, __uint_as_float(ov[i + 1]) * a0);
          }
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
        if (valid) p.lse[orow_idx] = (m + log2f(l)) * 0.6931471805599453f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // A split grid may run beside the whole-pair grid ahead of it; it does not
  // finish before that grid has, so work behind it in the stream sees both.
  if constexpr (kSplit) grid_dependency_wait();
}

// --------------------------------------------------------------- host side
}  // namespace

// cuTensorMapEncodeTiled from the driver, looked up once (no link-time libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

namespace {

// [BH][N][D] bf16 viewed as a 3-D tensor; boxes of 64 x 128 x 1, 128B swizzle.
bool make_map(CUtensorMap *map, const void *base, int D, int N, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Page pool [P][Hkv][16][D] bf16 as a 3-D tensor (D, 16, P*Hkv); boxes of 64
// columns x `rows` rows of one (page, K/V head) slice, 128B swizzle.
bool make_page_map(CUtensorMap *map, const void *base, int D, long long slices, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), 16, static_cast<cuuint64_t>(slices)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(16) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Token-major queries [T][Hq][D] bf16 as (D, Hq, T); boxes of 64 x 1 x 128.
bool make_tok_map(CUtensorMap *map, const void *base, int D, int Hq, int T) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kAlibi, bool kPaged, bool kSplit>
attn_status_t launch_kernel(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                            const CUtensorMap &mk1, const CUtensorMap &mv1, const Params &prm,
                            long long ctas, cudaStream_t stream, bool dependent = false) {
  using C = Cfg<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(prefill_bf16_kernel<D, kAlibi, kPaged, kSplit>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return ATTN_ERR_CUDA;
  if (ctas > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (ctas == 0) return ATTN_OK;
  if (!dependent) {
    prefill_bf16_kernel<D, kAlibi, kPaged, kSplit>
        <<<static_cast<unsigned>(ctas), NUM_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mk1,
                                                                               mv1, prm);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  // Programmatic dependent launch behind the grid before it in the stream.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, prefill_bf16_kernel<D, kAlibi, kPaged, kSplit>, mq, mk, mv, mk1,
                         mv1, prm) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

Params base_params(void *o, float *lse, unsigned *status, int B, int Hq, int Hkv, int N,
                   float scale, int causal, int window, const float *slopes) {
  Params prm{};
  prm.o = o;
  prm.lse = lse;
  prm.status = status;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.N = N;
  prm.pairs = (N + 2 * BM - 1) / (2 * BM);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.causal = causal ? 1 : 0;
  prm.window = window;
  prm.slopes = slopes;
  return prm;
}

template <int D, bool kAlibi>
attn_status_t launch(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                     int Hq, int Hkv, int N, float scale, int causal, int window,
                     const float *slopes, cudaStream_t stream, unsigned *status) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, N, B * Hq) || !make_map(&mk, k, D, N, B * Hkv) ||
      !make_map(&mv, v, D, N, B * Hkv))
    return ATTN_ERR_CUDA;
  if (window >= N) window = 0;  // a window of N or more keys is plain causal attention
  Params prm = base_params(o, lse, status, B, Hq, Hkv, N, scale, causal, window, slopes);
  const long long pairs = static_cast<long long>(prm.pairs) * B * Hq;
  if (pairs > 0x3fffffffLL) return ATTN_ERR_INVALID_ARG;
  // The pairs of the last, partial wave (all of them when there are fewer
  // pairs than SMs) run as two split CTAs each -- one Q tile, its KV range
  // halved over the two softmax warpgroups -- when the split CTAs fit in one
  // wave: that wave then takes about half as long.  They are a second grid of
  // the split variant, launched as a programmatic dependent of the whole
  // pairs' grid, so the whole-pair kernel carries none of the split code.
  // Not with a sliding window, whose halves could leave a row without a
  // visible key.
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return ATTN_ERR_CUDA;
  const long long rem = pairs % sms;
  const long long split_pairs = (window == 0 && rem > 0 && 2 * rem <= sms) ? rem : 0;
  prm.whole_pairs = static_cast<int>(pairs - split_pairs);
  attn_status_t st = launch_kernel<D, kAlibi, false, false>(mq, mk, mv, mk, mv, prm,
                                                            prm.whole_pairs, stream);
  if (st != ATTN_OK || split_pairs == 0) return st;
  return launch_kernel<D, kAlibi, false, true>(mq, mk, mv, mk, mv, prm, 2 * split_pairs, stream,
                                               prm.whole_pairs > 0);
}

template <int D, bool kAlibi>
attn_status_t launch_paged(const void *q, const void *k_pages, const void *v_pages,
                           const int *block_table, const int *seq_lens, const int *cu_q, void *o,
                           float *lse, int S, int Hq, int Hkv, int T, int max_q, int max_blocks,
                           int num_pages, float scale, int window, const float *slopes,
                           cudaStream_t stream, unsigned *status) {
  CUtensorMap mq, mk, mv, mk1, mv1;
  const long long slices = static_cast<long long>(num_pages) * Hkv;
  if (!make_tok_map(&mq, q, D, Hq, T) || !make_page_map(&mk, k_pages, D, slices, 16) ||
      !make_page_map(&mv, v_pages, D, slices, 16) || !make_page_map(&mk1, k_pages, D, slices, 1) ||
      !make_page_map(&mv1, v_pages, D, slices, 1))
    return ATTN_ERR_CUDA;
  Params prm = base_params(o, lse, status, S, Hq, Hkv, max_q, scale, 1, window, slopes);
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.cu_q = cu_q;
  prm.max_blocks = max_blocks;
  prm.num_pages = num_pages;
  prm.T = T;
  const long long ctas = static_cast<long long>(prm.pairs) * S * Hq;
  return launch_kernel<D, kAlibi, true, false>(mq, mk, mv, mk1, mv1, prm, ctas, stream);
}

}  // namespace

attn_status_t launch_prefill_bf16(const void *q, const void *k, const void *v, void *o, float *lse,
                                  int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                                  int window, const float *slopes, cudaStream_t stream,
                                  unsigned *status) {
  const bool alibi = slopes != nullptr;
  if (d == 128)
    return alibi ? launch<128, true>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, window, slopes,
                                     stream, status)
                 : launch<128, false>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, window,
                                      nullptr, stream, status);
  if (d == 64)
    return alibi ? launch<64, true>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, window, slopes,
                                    stream, status)
                 : launch<64, false>(q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, window,
                                     nullptr, stream, status);
  return ATTN_ERR_UNSUPPORTED;
}

attn_status_t launch_prefill_paged(const void *q, const void *k_pages, const void *v_pages,
                                   const int *block_table, const int *seq_lens, const int *cu_q,
                                   void *o, float *lse, int S, int Hq, int Hkv, int T, int max_q,
                                   int d, int max_blocks, int num_pages, float scale, int window,
                                   const float *slopes, cudaStream_t stream, unsigned *status) {
  const bool alibi = slopes != nullptr;
  if (d == 128)
    return alibi ? launch_paged<128, true>(q, k_pages, v_pages, block_table, seq_lens, cu_q, o, lse,
                                           S, Hq, Hkv, T, max_q, max_blocks, num_pages, scale,
                                           window, slopes, stream, status)
                 : launch_paged<128, false>(q, k_pages, v_pages, block_table, seq_lens, cu_q, o,
                                            lse, S, Hq, Hkv, T, max_q, max_blocks, num_pages, scale,
                                            window, nullptr, stream, status);
  if (d == 64)
    return alibi ? launch_paged<64, true>(q, k_pages, v_pages, block_table, seq_lens, cu_q, o, lse,
                                          S, Hq, Hkv, T, max_q, max_blocks, num_pages, scale,
                                          window, slopes, stream, status)
                 : launch_paged<64, false>(q, k_pages, v_pages, block_table, seq_lens, cu_q, o,
                                           lse, S, Hq, Hkv, T, max_q, max_blocks, num_pages, scale,
                                           window, nullptr, stream, status);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace exattn
