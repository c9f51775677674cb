// bwd_sm100.cu -- bf16 exact attention backward on B200 tensor cores.
//
// What it computes: dQ, dK, dV of sum(dO * O) for O = softmax(scale*Q K^T
// [+ mask, + ALiBi]) V, from Q, K, V, the forward's O and logsumexp L, and dO
// ("Phase 08" page, Concepts: the FlashAttention backward needs only O and L;
// Lab 01 step 6; quiz page: the backward recomputes the attention matrix tile
// by tile instead of storing it).  With P = exp(S - L) recomputed per tile:
//   D_i = rowsum(dO_i * O_i),  dP = dO V^T,  dS = P * (dP - D),
//   dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K.
// The N x N matrices exist one 128 x 128 tile at a time, in tensor memory.
//
// Three kernels, no atomics (the result does not depend on scheduling):
//  * bwd_prep: per query row, D = rowsum(dO * O) and L*log2(e), written to a
//    workspace padded to whole 128-row tiles (+inf / 0 past N, so padded rows
//    get P = 0 without a mask).
//  * bwd_dkdv: one CTA per 128-key tile of one (batch, K/V head).  K and V stay
//    in shared memory; 128-row tiles of Q and of dO (with their L, D) stream
//    through two rings, for every query head of the group.  Per tile:
//      S^T = K Q^T, dP^T = V dO^T        (128x128x16 MMAs, both K-major)
//      P^T = 2^(S^T c - L2), dS^T = P^T (dP^T - D)   (CUDA cores, TMEM ld/st)
//      dV += P^T dO, dK += dS^T Q          (A = P^T / dS^T from TMEM, B MN-major)
//  * bwd_dq: one CTA per 128-row Q tile of one (batch, query head); 128-key
//    tiles of K and of V stream through two rings.  S = Q K^T, dP = dO V^T,
//    dS as above, dQ += dS K (A = dS from TMEM, B = K MN-major).
// The recomputation costs two more tile products than a single kernel that
// scatters dQ with atomic adds (7 instead of 5); the FLOP rate reported counts
// the 5 of the algorithm.
//
// Scheduling.  All MMAs are 128 wide, and the two elementwise warpgroups take
// alternate tiles.  dK/dV kernel: each tile uses one 128-column TMEM buffer
// twice: the score tile S^T is written there, the tile's warpgroup loads it
// into registers and says so, and the tensor pipe then writes dP^T over it;
// the warps finally store their bf16 P^T and dS^T into the same columns.  Two
// such buffers next to dV and dK keep two tiles in flight; per tile the MMA
// issuer runs dP(i), then the gradient products of tile i-1 and the scores of
// tile i+1, so the exponentials of one tile overlap the other's products.
// dQ kernel: with one accumulator, TMEM has room for a dP buffer of its own
// beside the two score buffers, so no product waits for a score tile to be
// read: per tile j it runs dP(j+1) (once warpgroup j has read dP(j)), dQ(j)
// (once dS(j) is in the score buffer), then S(j+2) into that buffer.  The
// streamed tile whose product comes last (Q for dK, K for dQ) is live for
// three iterations and gets a three-slot ring; the other (dO, V) two slots.
//
// Warp roles (both GEMM kernels, 384 threads, as in the forward): warp 0 TMA
// producer (lane 0 for one ring, lane 1 for the other), warp 1 TMEM owner and
// MMA issuer, warps 4-7 and 8-11 the two elementwise warpgroups.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace exattn {
namespace {

constexpr int BT = 128;  // tile rows and columns: keys and queries
constexpr int NUM_THREADS = 384;
constexpr int kRegsLow = 72;
constexpr int kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= NUM_THREADS * 168 && kRegsLow % 8 == 0 &&
                  kRegsHigh % 8 == 0,
              "setmaxnreg split must fit the block's launch registers");
constexpr int kHeadGroup = 8;
constexpr int CHUNK = BT * 128;  // 128 rows x 128 bytes: one 64-column block of a tile
constexpr int NA = 3;            // slots of the three-iteration ring (Q or K)
constexpr int NB = 2;            // slots of the two-iteration ring (dO + vectors, or V)

// TMEM: two 128-column tile buffers, then the accumulators (dK/dV kernel) or
// the dP buffer and the accumulator (dQ kernel).  In a tile buffer the bf16
// results sit at columns [0, 64) (P^T, or dS) and [64, 128) (dS^T): the 128
// values of a row, two per column.
__device__ __forceinline__ uint32_t col_x(int buf) { return static_cast<uint32_t>(buf) * 128; }
constexpr uint32_t kColAcc0 = 256;  // dV (dK/dV kernel)
constexpr uint32_t kColAcc1 = 384;  // dK (dK/dV kernel)
constexpr uint32_t kColDP = 256;    // dP (dQ kernel): a buffer of its own
constexpr uint32_t kColDQ = 384;    // dQ (dQ kernel)

template <int D>
struct BCfg {
  static constexpr int CH = D / 64;
  static constexpr int TILE = BT * D * 2;
  static constexpr int VEC = 2 * BT * 4;  // L2 and D of a 128-row Q tile
  static constexpr int BSLOT_KV = TILE + VEC;  // dO tile + vectors (a multiple of 1024)
  // dK/dV kernel: K, V resident; Q ring (NA); dO + vector ring (NB).  At d =
  // 128 this is 226 KiB, so the kernel relies on the dynamic shared memory
  // starting 1024-aligned (it checks) instead of reserving slack.
  static constexpr int KV_A_OFF = 2 * TILE;
  static constexpr int KV_B_OFF = KV_A_OFF + NA * TILE;
  static constexpr int KV_BAR_OFF = KV_B_OFF + NB * BSLOT_KV;
  static constexpr int KV_SMEM = KV_BAR_OFF + 512;
  // dQ kernel: Q, dO resident; K ring (NA); V ring (NB).
  static constexpr int Q_A_OFF = 2 * TILE;
  static constexpr int Q_B_OFF = Q_A_OFF + NA * TILE;
  static constexpr int Q_BAR_OFF = Q_B_OFF + NB * TILE;
  static constexpr int Q_SMEM = Q_BAR_OFF + 512;
  // Each CTA allocates all 512 TMEM columns, so one CTA per SM: at d = 64
  // the launch asks for at least this much shared memory to make sure of it.
  static constexpr int MIN_SMEM = 116 * 1024;
  static constexpr int KV_LAUNCH = KV_SMEM > MIN_SMEM ? KV_SMEM : MIN_SMEM;
  static constexpr int Q_LAUNCH = Q_SMEM > MIN_SMEM ? Q_SMEM : MIN_SMEM;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT, false, false);
  static constexpr uint32_t IDESC_G = idesc_bf16_f32(BT, D, false, true);
};
static_assert(BCfg<128>::KV_SMEM <= 232448 && BCfg<128>::Q_SMEM <= 232448,
              "shared memory of one CTA");

struct BBars {
  uint64_t a_full[NA], a_empty[NA];  // Q (dK/dV kernel) or K (dQ kernel) ring
  uint64_t b_full[NB], b_empty[NB];  // dO + vectors, or V ring
  uint64_t res_full;                 // the resident tiles
  uint64_t s_full[2];    // buffer w holds S (S^T) of its tile
  uint64_t s_read[2];    // warpgroup w has loaded its tile into registers (count 128):
                         // S^T (dK/dV kernel) or dP (dQ kernel)
  uint64_t dp_full[2];   // buffer w holds dP (dP^T)
  uint64_t p_full[2];    // warpgroup w's bf16 results are in buffer w (count 128)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdParams {
  void *dq, *dk, *dv;
  const float *l2;    // [B*Hq][Npad]: L * log2(e), +inf past N
  const float *dvec;  // [B*Hq][Npad]: rowsum(dO * O), 0 past N
  unsigned *status;
  int B, Hq, Hkv, N, Npad;
  float scale, scale_log2;
  int causal, window;
  const float *slopes;  // per query head (ALiBi variant)
};

// Per row: D = rowsum(dO * O) (fp32 from the bf16 values) and L * log2(e); one
// warp per row, rows past N padded.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout,
                    const float *__restrict__ lse, float *__restrict__ l2,
                    float *__restrict__ dvec, int BH, int N, int Npad) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(BH) * Npad) return;
  const int bh = static_cast<int>(row / Npad), i = static_cast<int>(row % Npad);
  if (i >= N) {
    if (lane == 0) {
      l2[row] = INFINITY;
      dvec[row] = 0.f;
    }
    return;
  }
  const size_t src = (static_cast<size_t>(bh) * N + i) * D;
  float acc = 0.f;
  constexpr int EPL = D / 32;  // elements per lane: 4 (d=128) or 2 (d=64)
  if constexpr (EPL == 4) {
    const uint2 a = *reinterpret_cast<const uint2 *>(o + src + lane * 4);
    const uint2 b = *reinterpret_cast<const uint2 *>(dout + src + lane * 4);
    const uint32_t aw[2] = {a.x, a.y}, bw[2] = {b.x, b.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc);
      acc = fmaf(__uint_as_float(aw[e] & 0xffff0000u), __uint_as_float(bw[e] & 0xffff0000u), acc);
    }
  } else {
    const uint32_t a = *reinterpret_cast<const uint32_t *>(o + src + lane * 2);
    const uint32_t b = *reinterpret_cast<const uint32_t *>(dout + src + lane * 2);
    acc = fmaf(__uint_as_float(a << 16), __uint_as_float(b << 16), acc);
    acc = fmaf(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dvec[row] = acc;
    l2[row] = lse[static_cast<size_t>(bh) * N + i] * 1.4426950408889634f;
  }
}

// P = 2^(s*c + bias - l2) for 32 columns (0 where vis(i) is false), packed to
// bf16 pairs; bias = bias0 + bias_step * i (ALiBi); l2 per column (per_col) or
// one value.
template <bool kAlibi, bool kMasked, typename Vis>
__device__ __forceinline__ void p_cols(const uint32_t *sv, const float *l2c, float l2s,
                                       bool per_col, float c, float bias0, float bias_step,
                                       Vis vis, uint32_t *pk) {
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 lv = per_col ? *reinterpret_cast<const float2 *>(l2c + i) : make_float2(l2s, l2s);
    float2 x = fma2(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2,
                    make_float2(-lv.x, -lv.y));
    if (kAlibi)
      x = fma2(make_float2(bias_step, bias_step),
               make_float2(static_cast<float>(i), static_cast<float>(i + 1)),
               make_float2(x.x + bias0, x.y + bias0));
    float2 e = make_float2(ex2(x.x), ex2(x.y));
    if (kMasked) {
      if (!vis(i)) e.x = 0.f;
      if (!vis(i + 1)) e.y = 0.f;
    }
    pk[i >> 1] = pack_bf16x2(e.x, e.y);
  }
}

// dS = P * (dp - D) for 32 columns from bf16-packed P; packed bf16 out.
__device__ __forceinline__ void ds_cols(const uint32_t *pk, const uint32_t *dpv, const float *ddc,
                                        float dds, bool per_col, uint32_t *dk) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 dv = per_col ? *reinterpret_cast<const float2 *>(ddc + i) : make_float2(dds, dds);
    const uint32_t w = pk[i >> 1];
    const float2 pv = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    const float2 t = add2(make_float2(__uint_as_float(dpv[i]), __uint_as_float(dpv[i + 1])),
                          make_float2(-dv.x, -dv.y));
    dk[i >> 1] = pack_bf16x2(pv.x * t.x, pv.y * t.y);
  }
}

// ------------------------------------------------------------------ dK / dV
template <int D, bool kAlibi>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the layout needs a 1024-aligned base (see BCfg)
    if (threadIdx.x == 0) atomicOr(p.status, ATTN_DEV_LAYOUT);
    return;
  }
  uint8_t *sK = smem;
  uint8_t *sV = smem + C::TILE;
  uint8_t *sA = smem + C::KV_A_OFF;  // Q ring
  uint8_t *sB = smem + C::KV_B_OFF;  // dO + vector ring
  BBars *bars = reinterpret_cast<BBars *>(smem + C::KV_BAR_OFF);
  volatile int *abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: 128-key tile kt of (batch, K/V head).  Causal: heaviest
  // tiles (smallest kt: most query tiles) first within groups of heads.
  const int nkt = (p.N + BT - 1) / BT;
  const int BHk = p.B * p.Hkv;
  int kt, bhk;
  {
    const int lin = static_cast<int>(blockIdx.x);
    if (!p.causal) {
      bhk = lin / nkt;
      kt = lin % nkt;
    } else {
      const int grp = lin / (kHeadGroup * nkt);
      const int first = grp * kHeadGroup;
      const int hg = min(kHeadGroup, BHk - first);
      const int rr = lin - grp * kHeadGroup * nkt;
      kt = rr / hg;
      bhk = first + rr % hg;
    }
  }
  const int b = bhk / p.Hkv, g = bhk % p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int k0 = kt * BT;
  const int nqt = nkt;
  // Query tiles [qs, qe) that can see a key of this tile.
  const int qs = p.causal ? kt : 0;
  const int qe = p.window > 0 ? min(nqt, (k0 + BT - 1 + p.window - 1) / BT + 1) : nqt;
  const int nq = max(0, qe - qs);
  const int n_items = G * nq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(&bars->a_full[i], 1);
      mbar_init(&bars->a_empty[i], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&bars->b_full[i], 1);
      mbar_init(&bars->b_empty[i], 1);
    }
    mbar_init(&bars->res_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_read[t], 128);
      mbar_init(&bars->dp_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
    }
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

  if (warp == 0) {
    // ================================================================ producer
    regs_dec<kRegsLow>();
    if (lane == 0) {
      // K, V once; then the Q ring.
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sK + c * CHUNK, &tm_k, &bars->res_full, 64 * c, k0, bhk);
        tma_load_3d(sV + c * CHUNK, &tm_v, &bars->res_full, 64 * c, k0, bhk);
      }
      int issued = 0;
      for (int it = 0; it < n_items; ++it) {
        const int slot = it % NA, round = it / NA;
        if (round > 0 && !mbar_wait(&bars->a_empty[slot], (round - 1) & 1, abort_flag, p.status))
          break;
        const int zq = b * p.Hq + g * G + it / nq;
        const int q0 = (qs + it % nq) * BT;
        mbar_arrive_expect_tx(&bars->a_full[slot], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sA + slot * C::TILE + c * CHUNK, &tm_q, &bars->a_full[slot], 64 * c, q0, zq);
        issued = it + 1;
      }
      mbar_wait_drain(&bars->res_full, 0, p.status);
      for (int i = max(0, issued - NA); i < issued; ++i)
        mbar_wait_drain(&bars->a_full[i % NA], (i / NA) & 1, p.status);
    } else if (lane == 1) {
      // The dO ring, with each tile's L2 and D vectors.
      tma_prefetch_desc(&tm_do);
      int issued = 0;
      for (int it = 0; it < n_items; ++it) {
        const int slot = it % NB, round = it / NB;
        if (round > 0 && !mbar_wait(&bars->b_empty[slot], (round - 1) & 1, abort_flag, p.status))
          break;
        const int zq = b * p.Hq + g * G + it / nq;
        const int q0 = (qs + it % nq) * BT;
        uint8_t *st = sB + slot * C::BSLOT_KV;
        mbar_arrive_expect_tx(&bars->b_full[slot], C::BSLOT_KV);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(st + c * CHUNK, &tm_do, &bars->b_full[slot], 64 * c, q0, zq);
        const size_t vo = static_cast<size_t>(zq) * p.Npad + q0;
        bulk_load(st + C::TILE, p.l2 + vo, BT * 4, &bars->b_full[slot]);
        bulk_load(st + C::TILE + BT * 4, p.dvec + vo, BT * 4, &bars->b_full[slot]);
        issued = it + 1;
      }
      for (int i = max(0, issued - NB); i < issued; ++i)
        mbar_wait_drain(&bars->b_full[i % NB], (i / NB) & 1, p.status);
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    regs_dec<kRegsLow>();
    if (lane == 0) {
      const uint64_t kdesc = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t vdesc = kdesc + (C::TILE >> 4);
      const uint64_t qk0 = sdesc_sw128(smem_u32(sA), 16, 1024);        // Q, K-major
      const uint64_t qmn0 = sdesc_sw128(smem_u32(sA), CHUNK, 1024);    // Q, MN-major
      const uint64_t dok0 = sdesc_sw128(smem_u32(sB), 16, 1024);       // dO, K-major
      const uint64_t domn0 = sdesc_sw128(smem_u32(sB), CHUNK, 1024);   // dO, MN-major
      auto a_off = [](int it) { return static_cast<uint64_t>((it % NA) * C::TILE) >> 4; };
      auto b_off = [](int it) { return static_cast<uint64_t>((it % NB) * C::BSLOT_KV) >> 4; };
      auto wait_a = [&](int it) {
        return mbar_wait(&bars->a_full[it % NA], (it / NA) & 1, abort_flag, p.status);
      };
      auto wait_b = [&](int it) {
        return mbar_wait(&bars->b_full[it % NB], (it / NB) & 1, abort_flag, p.status);
      };
      auto issue_s = [&](int it) {  // S^T = K Q^T into buffer it & 1
        const uint32_t d = tmem + col_x(it & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(d, kdesc + off, qk0 + a_off(it) + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->s_full[it & 1]);
      };
      auto issue_dp = [&](int it) {  // dP^T = V dO^T over S^T (already read)
        const uint32_t d = tmem + col_x(it & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(d, vdesc + off, dok0 + b_off(it) + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->dp_full[it & 1]);
      };
      auto issue_grads = [&](int it) {  // dV += P^T dO, dK += dS^T Q
        const uint32_t x = tmem + col_x(it & 1);
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_ts(tmem + kColAcc0, x + ks * 8, domn0 + b_off(it) + ((ks * 2048) >> 4), C::IDESC_G,
                 (it > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->b_empty[it % NB]);  // dO(it) consumed: the next dO lands sooner
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_ts(tmem + kColAcc1, x + 64 + ks * 8, qmn0 + a_off(it) + ((ks * 2048) >> 4),
                 C::IDESC_G, (it > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->a_empty[it % NA]);
      };
      bool ok = mbar_wait(&bars->res_full, 0, abort_flag, p.status);
      for (int it = 0; ok && it < 2 && it < n_items; ++it) {
        if (!(ok = wait_a(it))) break;
        tc_fence_after();
        issue_s(it);
      }
      for (int it = 0; ok && it < n_items; ++it) {
        const int bb = it & 1;
        // dO(it) is checked first: its barrier latency then overlaps the wait
        // for the elementwise warpgroup instead of following it.
        if (!(ok = wait_b(it) && mbar_wait(&bars->s_read[bb], (it >> 1) & 1, abort_flag, p.status)))
          break;
        tc_fence_after();
        issue_dp(it);
        if (it >= 1) {
          if (!(ok = mbar_wait(&bars->p_full[bb ^ 1], ((it - 1) >> 1) & 1, abort_flag, p.status)))
            break;
          tc_fence_after();
          issue_grads(it - 1);
          if (it + 1 < n_items) {
            if (!(ok = wait_a(it + 1))) break;
            tc_fence_after();
            issue_s(it + 1);  // in order after grads(it-1), which read this buffer
          }
        }
      }
      if (ok && n_items > 0 &&
          (ok = mbar_wait(&bars->p_full[(n_items - 1) & 1], ((n_items - 1) >> 1) & 1, abort_flag,
                          p.status))) {
        tc_fence_after();
        issue_grads(n_items - 1);
      }
      tc_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, p.status);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();
  } else {
    // ============================================================ elementwise
    regs_inc<kRegsHigh>();
    const int wg = (warp - 4) >> 2;      // this warpgroup takes tiles wg, wg + 2, ...
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // key row in the tile
    const int key = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tX = tmem + lane_off + col_x(wg);
    const float c = p.scale_log2;
    bool ok = true;
    for (int it = wg; it < n_items; it += 2) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[wg], (it >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[128];
      tmem_ld128(tX, sv);
      tmem_ld_wait128(sv);
      tc_fence_before();
      mbar_arrive(&bars->s_read[wg]);  // the tensor pipe may now write dP^T here
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars->b_full[it % NB], (it / NB) & 1, abort_flag, p.status));
      if (!ok) break;
      const int hq = g * G + it / nq;
      const int qb0 = (qs + it % nq) * BT;  // first query of the tile
      const uint8_t *st = sB + (it % NB) * C::BSLOT_KV;
      const float *l2v = reinterpret_cast<const float *>(st + C::TILE);
      const float *ddv = l2v + BT;
      const float slope2 = kAlibi ? p.slopes[hq] * 1.4426950408889634f : 0.f;
      // ---- P^T (bf16 pairs) for the tile's 128 queries, while dP^T runs.
      uint32_t pk[64];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int qb = qb0 + 32 * h;
        auto vis = [&](int i) {
          const int qq = qb + i;
          return (!p.causal || key <= qq) && (p.window <= 0 || qq - key < p.window);
        };
        const bool full = (!p.causal || key <= qb) && (p.window <= 0 || qb + 31 - key < p.window);
        // ALiBi bias slope*(key - query) in log2 units; column i has query qb + i.
        const float bias0 = slope2 * static_cast<float>(key - qb);
        if (__all_sync(0xffffffffu, full))
          p_cols<kAlibi, false>(sv + 32 * h, l2v + 32 * h, 0.f, true, c, bias0, -slope2, vis,
                                pk + 16 * h);
        else
          p_cols<kAlibi, true>(sv + 32 * h, l2v + 32 * h, 0.f, true, c, bias0, -slope2, vis,
                               pk + 16 * h);
      }
      // ---- dS^T from P^T and dP^T; results over the buffer.
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full[wg], (it >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t ds[64];
      {
        uint32_t dp[64];
        tmem_ld64(tX, dp);  // queries 0..63
        tmem_ld_wait64(dp);
        ds_cols(pk, dp, ddv, 0.f, true, ds);
        ds_cols(pk + 16, dp + 32, ddv + 32, 0.f, true, ds + 16);
      }
      {
        // Columns [0, 64) are read: P^T goes there.
        uint32_t (&pk0)[32] = *reinterpret_cast<uint32_t (*)[32]>(pk);
        uint32_t (&pk1)[32] = *reinterpret_cast<uint32_t (*)[32]>(pk + 32);
        tmem_st32(tX, pk0);
        tmem_st32(tX + 32, pk1);
      }
      {
        uint32_t dp[64];
        tmem_ld64(tX + 64, dp);  // queries 64..127
        tmem_ld_wait64(dp);
        ds_cols(pk + 32, dp, ddv + 64, 0.f, true, ds + 32);
        ds_cols(pk + 48, dp + 32, ddv + 96, 0.f, true, ds + 48);
      }
      {
        uint32_t (&ds0)[32] = *reinterpret_cast<uint32_t (*)[32]>(ds);
        uint32_t (&ds1)[32] = *reinterpret_cast<uint32_t (*)[32]>(ds + 32);
        tmem_st32(tX + 64, ds0);
        tmem_st32(tX + 96, ds1);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[wg]);
    }
    if (ok && n_items > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->mma_done, 0, abort_flag, p.status));
      if (ok) {
        tc_fence_after();
        // Warpgroup 0 writes dV, warpgroup 1 writes dK (times scale).
        const uint32_t acc = tmem + lane_off + (wg == 0 ? kColAcc0 : kColAcc1);
        const float mul = wg == 0 ? 1.f : p.scale;
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(wg == 0 ? p.dv : p.dk) +
                             (static_cast<size_t>(bhk) * p.N + (key < p.N ? key : 0)) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(acc + cc * 32, v);
          tmem_ld_wait(v);
          uint32_t pkd[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            pkd[i >> 1] = pack_bf16x2(__uint_as_float(v[i]) * mul, __uint_as_float(v[i + 1]) * mul);
          if (key < p.N) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              d4[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
          }
        }
      }
    } else if (ok && n_items == 0) {
      // No query sees this tile (cannot happen for keys < N): zero gradients.
      __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(wg == 0 ? p.dv : p.dk) +
                           (static_cast<size_t>(bhk) * p.N + (key < p.N ? key : 0)) * D;
      if (key < p.N)
        for (int cc = 0; cc < D; cc += 8) *reinterpret_cast<uint4 *>(dst + cc) = make_uint4(0, 0, 0, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------- dQ
template <int D, bool kAlibi>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the layout needs a 1024-aligned base (see BCfg)
    if (threadIdx.x == 0) atomicOr(p.status, ATTN_DEV_LAYOUT);
    return;
  }
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + C::TILE;
  uint8_t *sA = smem + C::Q_A_OFF;  // K ring
  uint8_t *sB = smem + C::Q_B_OFF;  // V ring
  BBars *bars = reinterpret_cast<BBars *>(smem + C::Q_BAR_OFF);
  volatile int *abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: 128-row Q tile of (batch, query head); causal: heaviest first.
  const int nqt = (p.N + BT - 1) / BT;
  const int BH = p.B * p.Hq;
  int qt, bh;
  {
    const int lin = static_cast<int>(blockIdx.x);
    if (!p.causal) {
      bh = lin / nqt;
      qt = lin % nqt;
    } else {
      const int grp = lin / (kHeadGroup * nqt);
      const int first = grp * kHeadGroup;
      const int hg = min(kHeadGroup, BH - first);
      const int rr = lin - grp * kHeadGroup * nqt;
      qt = nqt - 1 - rr / hg;
      bh = first + rr % hg;
    }
  }
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int row0 = qt * BT;
  const int nkt = nqt;
  const int je = p.causal ? min(qt + 1, nkt) : nkt;
  const int js = p.window > 0 ? max(0, row0 - p.window + 1) / BT : 0;
  const int n_items = max(0, je - js);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(&bars->a_full[i], 1);
      mbar_init(&bars->a_empty[i], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&bars->b_full[i], 1);
      mbar_init(&bars->b_empty[i], 1);
    }
    mbar_init(&bars->res_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_read[t], 128);
      mbar_init(&bars->dp_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
    }
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

  if (warp == 0) {
    // ================================================================ producer
    regs_dec<kRegsLow>();
    if (lane == 0) {
      // Q, dO once; then the K ring.
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sQ + c * CHUNK, &tm_q, &bars->res_full, 64 * c, row0, bh);
        tma_load_3d(sdO + c * CHUNK, &tm_do, &bars->res_full, 64 * c, row0, bh);
      }
      int issued = 0;
      for (int j = 0; j < n_items; ++j) {
        const int slot = j % NA, round = j / NA;
        if (round > 0 && !mbar_wait(&bars->a_empty[slot], (round - 1) & 1, abort_flag, p.status))
          break;
        mbar_arrive_expect_tx(&bars->a_full[slot], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sA + slot * C::TILE + c * CHUNK, &tm_k, &bars->a_full[slot], 64 * c,
                      (js + j) * BT, bhk);
        issued = j + 1;
      }
      mbar_wait_drain(&bars->res_full, 0, p.status);
      for (int i = max(0, issued - NA); i < issued; ++i)
        mbar_wait_drain(&bars->a_full[i % NA], (i / NA) & 1, p.status);
    } else if (lane == 1) {
      // The V ring.
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int j = 0; j < n_items; ++j) {
        const int slot = j % NB, round = j / NB;
        if (round > 0 && !mbar_wait(&bars->b_empty[slot], (round - 1) & 1, abort_flag, p.status))
          break;
        mbar_arrive_expect_tx(&bars->b_full[slot], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sB + slot * C::TILE + c * CHUNK, &tm_v, &bars->b_full[slot], 64 * c,
                      (js + j) * BT, bhk);
        issued = j + 1;
      }
      for (int i = max(0, issued - NB); i < issued; ++i)
        mbar_wait_drain(&bars->b_full[i % NB], (i / NB) & 1, p.status);
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    regs_dec<kRegsLow>();
    if (lane == 0) {
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dodesc = qdesc + (C::TILE >> 4);
      const uint64_t kk0 = sdesc_sw128(smem_u32(sA), 16, 1024);       // K, K-major
      const uint64_t kmn0 = sdesc_sw128(smem_u32(sA), CHUNK, 1024);   // K, MN-major
      const uint64_t vk0 = sdesc_sw128(smem_u32(sB), 16, 1024);       // V, K-major
      auto a_off = [](int j) { return static_cast<uint64_t>((j % NA) * C::TILE) >> 4; };
      auto b_off = [](int j) { return static_cast<uint64_t>((j % NB) * C::TILE) >> 4; };
      auto wait_a = [&](int j) {
        return mbar_wait(&bars->a_full[j % NA], (j / NA) & 1, abort_flag, p.status);
      };
      auto wait_b = [&](int j) {
        return mbar_wait(&bars->b_full[j % NB], (j / NB) & 1, abort_flag, p.status);
      };
      auto issue_s = [&](int j) {  // S = Q K^T into buffer j & 1
        const uint32_t d = tmem + col_x(j & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(d, qdesc + off, kk0 + a_off(j) + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->s_full[j & 1]);
      };
      auto issue_dp = [&](int j) {  // dP = dO V^T into the dP buffer
        const uint32_t d = tmem + kColDP;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(d, dodesc + off, vk0 + b_off(j) + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->dp_full[j & 1]);
        tc_commit(&bars->b_empty[j % NB]);  // V(j) consumed
      };
      auto issue_dq = [&](int j) {  // dQ += dS K
        const uint32_t x = tmem + col_x(j & 1);
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_ts(tmem + kColDQ, x + ks * 8, kmn0 + a_off(j) + ((ks * 2048) >> 4), C::IDESC_G,
                 (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->a_empty[j % NA]);  // K(j) consumed
      };
      // dP has its own buffer, so no product waits for a score tile to be
      // read: per tile j, dP(j+1) once warpgroup j has read dP(j), then dQ(j)
      // once dS(j) is in, then S(j+2) into the buffer dQ(j) just read.
      bool ok = mbar_wait(&bars->res_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j < 2 && j < n_items; ++j) {
        if (!(ok = wait_a(j))) break;
        tc_fence_after();
        issue_s(j);
      }
      if (ok && n_items > 0 && (ok = wait_b(0))) {
        tc_fence_after();
        issue_dp(0);
      }
      for (int j = 0; ok && j < n_items; ++j) {
        const int bb = j & 1;
        if (j + 1 < n_items) {
          if (!(ok = mbar_wait(&bars->s_read[bb], (j >> 1) & 1, abort_flag, p.status) &&
                     wait_b(j + 1)))
            break;
          tc_fence_after();
          issue_dp(j + 1);  // warpgroup j has read dP(j)
        }
        if (!(ok = mbar_wait(&bars->p_full[bb], (j >> 1) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        issue_dq(j);
        if (j + 2 < n_items) {
          if (!(ok = wait_a(j + 2))) break;
          tc_fence_after();
          issue_s(j + 2);  // in order after dQ(j), which read this buffer
        }
      }
      tc_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, p.status);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();
  } else {
    // ============================================================ elementwise
    regs_inc<kRegsHigh>();
    const int wg = (warp - 4) >> 2;  // this warpgroup takes tiles wg, wg + 2, ...
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int row = row0 + r;  // query row; rows >= N have l2 = +inf, so P = 0
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tX = tmem + lane_off + col_x(wg);
    const uint32_t tDP = tmem + lane_off + kColDP;
    const float c = p.scale_log2;
    const float l2s = p.l2[static_cast<size_t>(bh) * p.Npad + row];
    const float dds = p.dvec[static_cast<size_t>(bh) * p.Npad + row];
    const float slope2 = kAlibi ? p.slopes[hq] * 1.4426950408889634f : 0.f;
    bool ok = true;
    for (int j = wg; j < n_items; j += 2) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[wg], (j >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[128];
      tmem_ld128(tX, sv);
      tmem_ld_wait128(sv);
      const int kb0 = (js + j) * BT;     // first key of the tile
      uint32_t pk[64];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int kb = kb0 + 32 * h;
        auto vis = [&](int i) {
          const int kk = kb + i;
          return kk < p.N && (!p.causal || kk <= row) && (p.window <= 0 || row - kk < p.window);
        };
        const bool full = kb + 31 < p.N && (!p.causal || kb + 31 <= row) &&
                          (p.window <= 0 || row - kb < p.window);
        const float bias0 = slope2 * static_cast<float>(kb - row);
        if (__all_sync(0xffffffffu, full))
          p_cols<kAlibi, false>(sv + 32 * h, nullptr, l2s, false, c, bias0, slope2, vis, pk + 16 * h);
        else
          p_cols<kAlibi, true>(sv + 32 * h, nullptr, l2s, false, c, bias0, slope2, vis, pk + 16 * h);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full[wg], (j >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t ds[64];
      {
        uint32_t dp[64];
        tmem_ld64(tDP, dp);  // keys 0..63
        tmem_ld_wait64(dp);
        ds_cols(pk, dp, nullptr, dds, false, ds);
        ds_cols(pk + 16, dp + 32, nullptr, dds, false, ds + 16);
      }
      {
        uint32_t dp[64];
        tmem_ld64(tDP + 64, dp);  // keys 64..127
        tmem_ld_wait64(dp);
        tc_fence_before();
        mbar_arrive(&bars->s_read[wg]);  // dP(j) is read: the buffer may take dP(j+1)
        ds_cols(pk + 32, dp, nullptr, dds, false, ds + 32);
        ds_cols(pk + 48, dp + 32, nullptr, dds, false, ds + 48);
      }
      {
        uint32_t (&ds0)[32] = *reinterpret_cast<uint32_t (*)[32]>(ds);
        uint32_t (&ds1)[32] = *reinterpret_cast<uint32_t (*)[32]>(ds + 32);
        tmem_st32(tX, ds0);
        tmem_st32(tX + 32, ds1);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[wg]);
    }
    if (ok && n_items > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->mma_done, 0, abort_flag, p.status));
      if (ok) {
        tc_fence_after();
        // Each warpgroup writes half of the row's D columns.
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.dq) +
                             (static_cast<size_t>(bh) * p.N + (row < p.N ? row : 0)) * D;
#pragma unroll
        for (int cc = wg * (D / 64); cc < (wg + 1) * (D / 64); ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + kColDQ + cc * 32, v);
          tmem_ld_wait(v);
          uint32_t pkd[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            pkd[i >> 1] = pack_bf16x2(__uint_as_float(v[i]) * p.scale, __uint_as_float(v[i + 1]) * p.scale);
          if (row < p.N) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              d4[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
          }
        }
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
}

// [BH][N][D] bf16 as a 3-D tensor (D, N, BH); boxes of 64 columns x rows x 1, 128B swizzle.
bool make_map_rows(CUtensorMap *map, const void *base, int D, int N, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kAlibi>
attn_status_t launch_bwd(const void *q, const void *k, const void *v, const void *dout,
                         const BwdParams &prm, cudaStream_t stream) {
  using C = BCfg<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(bwd_dkdv_kernel<D, kAlibi>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::KV_LAUNCH);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(bwd_dq_kernel<D, kAlibi>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::Q_LAUNCH);
  });
  if (attr_err != cudaSuccess) return ATTN_ERR_CUDA;
  const int BHq = prm.B * prm.Hq, BHk = prm.B * prm.Hkv;
  CUtensorMap mk, mv, mq, mdo;
  if (!make_map_rows(&mk, k, D, prm.N, BHk, BT) || !make_map_rows(&mv, v, D, prm.N, BHk, BT) ||
      !make_map_rows(&mq, q, D, prm.N, BHq, BT) || !make_map_rows(&mdo, dout, D, prm.N, BHq, BT))
    return ATTN_ERR_CUDA;
  const long long kv_ctas = static_cast<long long>((prm.N + BT - 1) / BT) * BHk;
  const long long q_ctas = static_cast<long long>((prm.N + BT - 1) / BT) * BHq;
  if (kv_ctas > 0x7fffffffLL || q_ctas > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  bwd_dkdv_kernel<D, kAlibi><<<static_cast<unsigned>(kv_ctas), NUM_THREADS, C::KV_LAUNCH, stream>>>(
      mk, mv, mq, mdo, prm);
  bwd_dq_kernel<D, kAlibi><<<static_cast<unsigned>(q_ctas), NUM_THREADS, C::Q_LAUNCH, stream>>>(
      mq, mdo, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int bwd_padded_rows(int N) { return (N + BT - 1) / BT * BT; }

size_t bwd_workspace_bytes(int B, int Hq, int N) {
  const size_t n = static_cast<size_t>(B) * Hq * bwd_padded_rows(N) * sizeof(float);
  return 2 * ((n + 255) & ~static_cast<size_t>(255));
}

attn_status_t launch_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dout, void *dq, void *dk, void *dv,
                              int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                              int window, const float *slopes, void *workspace,
                              cudaStream_t stream, unsigned *status) {
  BwdParams prm;
  prm.dq = dq;
  prm.dk = dk;
  prm.dv = dv;
  prm.Npad = bwd_padded_rows(N);
  const size_t n = static_cast<size_t>(B) * Hq * prm.Npad;
  float *l2 = static_cast<float *>(workspace);
  float *dvec = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                          ((n * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  prm.l2 = l2;
  prm.dvec = dvec;
  prm.status = status;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.N = N;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.causal = causal ? 1 : 0;
  prm.window = window;
  prm.slopes = slopes;
  const long long rows = static_cast<long long>(n);
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  if (d == 128)
    bwd_prep_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse, l2,
        dvec, B * Hq, N, prm.Npad);
  else if (d == 64)
    bwd_prep_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse, l2,
        dvec, B * Hq, N, prm.Npad);
  else
    return ATTN_ERR_UNSUPPORTED;
  const bool alibi = slopes != nullptr;
  if (d == 128)
    return alibi ? launch_bwd<128, true>(q, k, v, dout, prm, stream)
                 : launch_bwd<128, false>(q, k, v, dout, prm, stream);
  return alibi ? launch_bwd<64, true>(q, k, v, dout, prm, stream)
               : launch_bwd<64, false>(q, k, v, dout, prm, stream);
}

}  // namespace exattn
