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
//    in shared memory; 128-row tiles of Q and dO (and their L, D) stream
//    through a ring, for every query head of the group.  Per tile:
//      S^T = K Q^T, dP^T = V dO^T        (128x128x16 MMAs, both K-major)
//      P^T = 2^(S^T c - L2), dS^T = P^T (dP^T - D)   (CUDA cores, TMEM ld/st)
//      dV += P^T dO, dK += dS^T Q          (A = P^T / dS^T from TMEM, B MN-major)
//  * bwd_dq: one CTA per 128-row Q tile of one (batch, query head); 128-key
//    tiles of K and V stream through a ring.  S = Q K^T, dP = dO V^T,
//    dS as above, dQ += dS K (A = dS from TMEM, B = K MN-major).
// The recomputation costs two more tile products than a single kernel that
// scatters dQ with atomic adds (7 instead of 5); the FLOP rate reported counts
// the 5 of the algorithm.
//
// Scheduling.  All MMAs are 128 wide.  TMEM holds S (or S^T) and dP (or dP^T),
// 128 columns each, and the 128-column accumulators (dV and dK, or dQ): 512
// columns, so the score tiles are single-buffered.  The overlap comes from
// splitting every tile's columns between the two elementwise warpgroups: a
// warpgroup computes P from S while the tensor pipe still computes dP, and
// hands over its half of P / dS as soon as it is written, so the gradient MMAs
// of one half run while the other half is still being computed.  The next
// tile's S is issued right after the gradient MMAs that read the current one
// (tcgen05 ops from one thread execute in order).
//
// Warp roles (both GEMM kernels, 384 threads, as in the forward): warp 0 TMA
// producer, warp 1 TMEM owner and MMA issuer, warps 4-7 and 8-11 two
// elementwise warpgroups, each owning 64 of a tile's 128 columns.
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

// TMEM columns: S / S^T, dP / dP^T, and the accumulators.  Warpgroup w writes
// its 64 bf16 results (P^T and dS^T, or dS) over columns [64w, 64w+32) of the
// tile it read them from.
constexpr uint32_t kColS = 0;
constexpr uint32_t kColDP = 128;
constexpr uint32_t kColAcc0 = 256;  // dV (dK/dV kernel) or dQ (dQ kernel)
constexpr uint32_t kColAcc1 = 384;  // dK (dK/dV kernel)
__device__ __forceinline__ uint32_t packed_col(int ks) {  // k-step of 16 -> its 8 bf16 columns
  return 64 * (ks >> 2) + (ks & 3) * 8;
}

template <int D>
struct BCfg {
  static constexpr int CH = D / 64;
  static constexpr int TILE = BT * D * 2;
  // dK/dV kernel: K, V resident; stages of {Q, dO, L2[128], D[128]}.
  static constexpr int KV_NST = (D == 64) ? 4 : 2;
  static constexpr int KV_STAGE = ((2 * TILE + 2 * BT * 4) + 1023) / 1024 * 1024;
  static constexpr int KV_RING_OFF = 2 * TILE;
  static constexpr int KV_BAR_OFF = KV_RING_OFF + KV_NST * KV_STAGE;
  // dQ kernel: Q, dO resident; slots of one K or V tile.
  static constexpr int Q_NST = (D == 64) ? 8 : 4;
  static constexpr int Q_RING_OFF = 2 * TILE;
  static constexpr int Q_BAR_OFF = Q_RING_OFF + Q_NST * TILE;
  // At least 116 KiB so that one CTA fills an SM: each CTA allocates all 512
  // TMEM columns.
  static constexpr int MIN_SMEM = 116 * 1024;
  static constexpr int KV_SMEM = (KV_BAR_OFF + 2048 > MIN_SMEM) ? KV_BAR_OFF + 2048 : MIN_SMEM;
  static constexpr int Q_SMEM = (Q_BAR_OFF + 2048 > MIN_SMEM) ? Q_BAR_OFF + 2048 : MIN_SMEM;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT, false, false);
  static constexpr uint32_t IDESC_G = idesc_bf16_f32(BT, D, false, true);
};

struct BBars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t res_full;  // the resident tiles (K,V or Q,dO)
  uint64_t s_full;    // S (or S^T) of the current tile is in TMEM
  uint64_t dp_full;   // dP (or dP^T) likewise
  uint64_t p_full[2]; // warpgroup w's half of P / dS is in TMEM
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

// P = 2^(s*c + bias - l2) for 32 columns (0 where vis(i) is false); bias =
// bias0 + bias_step * i (ALiBi); l2 per column (per_col) or one value.  On
// unmasked columns one pair in four takes 2^x from the FMA-pipe cubic
// (relative error < 2^-13, below the bf16 rounding that follows), which
// shortens the special-function unit's share of the tile.
template <bool kAlibi, bool kMasked, typename Vis>
__device__ __forceinline__ void p_cols(const uint32_t (&sv)[32], const float *l2c, float l2s,
                                       bool per_col, float c, float bias0, float bias_step,
                                       Vis vis, float (&pv)[32]) {
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
    if (!kMasked && (i & 6) == 6) {  // one pair in four on the FMA pipe
      const float2 e = exp2_poly2(x);
      pv[i] = e.x;
      pv[i + 1] = e.y;
    } else {
      pv[i] = ex2(x.x);
      pv[i + 1] = ex2(x.y);
    }
    if (kMasked) {
      if (!vis(i)) pv[i] = 0.f;
      if (!vis(i + 1)) pv[i + 1] = 0.f;
    }
  }
}

__device__ __forceinline__ void pack_cols(const float (&pv)[32], uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) pk[i >> 1] = pack_bf16x2(pv[i], pv[i + 1]);
}

// dS = P * (dp - D) for 32 columns, packed bf16; D per column or one value.
__device__ __forceinline__ void ds_cols(const float (&pv)[32], const uint32_t (&dpv)[32],
                                        const float *ddc, float dds, bool per_col,
                                        uint32_t (&dk)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 dv = per_col ? *reinterpret_cast<const float2 *>(ddc + i) : make_float2(dds, dds);
    const float2 t = add2(make_float2(__uint_as_float(dpv[i]), __uint_as_float(dpv[i + 1])),
                          make_float2(-dv.x, -dv.y));
    dk[i >> 1] = pack_bf16x2(pv[i] * t.x, pv[i + 1] * t.y);
  }
}

// ------------------------------------------------------------------ dK / dV
template <int D, bool kAlibi>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sK = smem;
  uint8_t *sV = smem + C::TILE;
  uint8_t *sRing = smem + C::KV_RING_OFF;
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
    for (int i = 0; i < C::KV_NST; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    mbar_init(&bars->res_full, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full[0], 128);
    mbar_init(&bars->p_full[1], 128);
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
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sK + c * CHUNK, &tm_k, &bars->res_full, 64 * c, k0, bhk);
        tma_load_3d(sV + c * CHUNK, &tm_v, &bars->res_full, 64 * c, k0, bhk);
      }
      int issued = 0;
      for (int it = 0; it < n_items; ++it) {
        const int slot = it % C::KV_NST, round = it / C::KV_NST;
        if (round > 0 && !mbar_wait(&bars->empty[slot], (round - 1) & 1, abort_flag, p.status)) break;
        const int hq = g * G + it / nq;
        const int q0 = (qs + it % nq) * BT;
        const int zq = b * p.Hq + hq;
        uint8_t *st = sRing + slot * C::KV_STAGE;
        mbar_arrive_expect_tx(&bars->full[slot], 2 * C::TILE + 2 * BT * 4);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_3d(st + c * CHUNK, &tm_q, &bars->full[slot], 64 * c, q0, zq);
          tma_load_3d(st + C::TILE + c * CHUNK, &tm_do, &bars->full[slot], 64 * c, q0, zq);
        }
        const size_t vo = static_cast<size_t>(zq) * p.Npad + q0;
        bulk_load(st + 2 * C::TILE, p.l2 + vo, BT * 4, &bars->full[slot]);
        bulk_load(st + 2 * C::TILE + BT * 4, p.dvec + vo, BT * 4, &bars->full[slot]);
        issued = it + 1;
      }
      mbar_wait_drain(&bars->res_full, 0, p.status);
      for (int i = max(0, issued - C::KV_NST); i < issued; ++i)
        mbar_wait_drain(&bars->full[i % C::KV_NST], (i / C::KV_NST) & 1, p.status);
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    regs_dec<kRegsLow>();
    if (lane == 0) {
      const uint32_t ring = smem_u32(sRing);
      const uint64_t kdesc = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t vdesc = kdesc + (C::TILE >> 4);
      const uint64_t qk0 = sdesc_sw128(ring, 16, 1024);               // Q, K-major
      const uint64_t dok0 = qk0 + (C::TILE >> 4);                     // dO, K-major
      const uint64_t qmn0 = sdesc_sw128(ring, CHUNK, 1024);           // Q, MN-major
      const uint64_t domn0 = qmn0 + (C::TILE >> 4);                   // dO, MN-major
      auto wait_full = [&](int it) {
        return mbar_wait(&bars->full[it % C::KV_NST], (it / C::KV_NST) & 1, abort_flag, p.status);
      };
      auto stage_off = [](int it) {
        return static_cast<uint64_t>((it % C::KV_NST) * C::KV_STAGE) >> 4;
      };
      auto issue_scores = [&](int it) {  // S^T = K Q^T, commit; dP^T = V dO^T, commit
        const uint64_t so = stage_off(it);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(tmem + kColS, kdesc + off, qk0 + so + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->s_full);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(tmem + kColDP, vdesc + off, dok0 + so + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->dp_full);
      };
      auto issue_grad_half = [&](int it, int h) {  // queries [64h, 64h+64)
        const uint64_t so = stage_off(it);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int ks = 4 * h + kk;
          mma_ts(tmem + kColAcc0, tmem + kColS + packed_col(ks), domn0 + so + ((ks * 2048) >> 4),
                 C::IDESC_G, (it > 0 || ks > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int ks = 4 * h + kk;
          mma_ts(tmem + kColAcc1, tmem + kColDP + packed_col(ks), qmn0 + so + ((ks * 2048) >> 4),
                 C::IDESC_G, (it > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&bars->res_full, 0, abort_flag, p.status);
      if (ok && n_items > 0 && (ok = wait_full(0))) {
        tc_fence_after();
        issue_scores(0);
      }
      for (int it = 0; ok && it < n_items; ++it) {
        for (int h = 0; h < 2; ++h) {
          if (!(ok = mbar_wait(&bars->p_full[h], it & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_grad_half(it, h);
        }
        if (!ok) break;
        tc_commit(&bars->empty[it % C::KV_NST]);  // Q/dO stage consumed
        if (it + 1 < n_items) {
          if (!(ok = wait_full(it + 1))) break;
          tc_fence_after();
          // In order after the gradient MMAs above, which read P^T / dS^T from
          // these columns: no completion wait needed.
          issue_scores(it + 1);
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
    const int wg = (warp - 4) >> 2;      // this warpgroup's 64 columns: [64wg, 64wg+64)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // key row in the tile
    const int key = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + 64 * wg;
    const uint32_t tDP = tmem + lane_off + kColDP + 64 * wg;
    const float c = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_items; ++it) {
      ok = mbar_wait(&bars->s_full, it & 1, abort_flag, p.status) &&
           mbar_wait(&bars->full[it % C::KV_NST], (it / C::KV_NST) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int hq = g * G + it / nq;
      const int qb = (qs + it % nq) * BT + 64 * wg;  // first query of this warpgroup's columns
      const uint8_t *st = sRing + (it % C::KV_NST) * C::KV_STAGE;
      const float *l2v = reinterpret_cast<const float *>(st + 2 * C::TILE) + 64 * wg;
      const float *ddv = l2v + BT;
      const float slope2 = kAlibi ? p.slopes[hq] * 1.4426950408889634f : 0.f;
      // ---- P^T from S^T (while the tensor pipe computes dP^T)
      float pv0[32], pv1[32];
      {
        uint32_t s0[32], s1[32];
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_ld_wait(s0);
        tmem_ld_wait(s1);
        auto vis0 = [&](int i) {
          const int qq = qb + i;
          return (!p.causal || key <= qq) && (p.window <= 0 || qq - key < p.window);
        };
        auto vis1 = [&](int i) { return vis0(i + 32); };
        const bool full0 = (!p.causal || key <= qb) && (p.window <= 0 || qb + 31 - key < p.window);
        const bool full1 =
            (!p.causal || key <= qb + 32) && (p.window <= 0 || qb + 63 - key < p.window);
        // ALiBi bias slope*(key - query) in log2 units; column i has query qb + i.
        const float bias0 = slope2 * static_cast<float>(key - qb);
        if (__all_sync(0xffffffffu, full0))
          p_cols<kAlibi, false>(s0, l2v, 0.f, true, c, bias0, -slope2, vis0, pv0);
        else
          p_cols<kAlibi, true>(s0, l2v, 0.f, true, c, bias0, -slope2, vis0, pv0);
        if (__all_sync(0xffffffffu, full1))
          p_cols<kAlibi, false>(s1, l2v + 32, 0.f, true, c, bias0 - 32.f * slope2, -slope2, vis1, pv1);
        else
          p_cols<kAlibi, true>(s1, l2v + 32, 0.f, true, c, bias0 - 32.f * slope2, -slope2, vis1, pv1);
        uint32_t pk[16];
        pack_cols(pv0, pk);
        tmem_st16(tS, pk);
        pack_cols(pv1, pk);
        tmem_st16(tS + 16, pk);
      }
      // ---- dS^T from P^T and dP^T
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t d0[32], d1[32];
        tmem_ld32(tDP, d0);
        tmem_ld32(tDP + 32, d1);
        tmem_ld_wait(d0);
        tmem_ld_wait(d1);
        uint32_t dk[16];
        ds_cols(pv0, d0, ddv, 0.f, true, dk);
        tmem_st16(tDP, dk);
        ds_cols(pv1, d1, ddv + 32, 0.f, true, dk);
        tmem_st16(tDP + 16, dk);
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
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + C::TILE;
  uint8_t *sRing = smem + C::Q_RING_OFF;
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
    for (int i = 0; i < C::Q_NST; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    mbar_init(&bars->res_full, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full[0], 128);
    mbar_init(&bars->p_full[1], 128);
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
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sQ + c * CHUNK, &tm_q, &bars->res_full, 64 * c, row0, bh);
        tma_load_3d(sdO + c * CHUNK, &tm_do, &bars->res_full, 64 * c, row0, bh);
      }
      int issued = 0;
      for (int i = 0; i < 2 * n_items; ++i) {
        const int slot = i % C::Q_NST, round = i / C::Q_NST;
        if (round > 0 && !mbar_wait(&bars->empty[slot], (round - 1) & 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&bars->full[slot], C::TILE);
        const CUtensorMap *map = (i & 1) ? &tm_v : &tm_k;
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(sRing + slot * C::TILE + c * CHUNK, map, &bars->full[slot], 64 * c,
                      (js + (i >> 1)) * BT, bhk);
        issued = i + 1;
      }
      mbar_wait_drain(&bars->res_full, 0, p.status);
      for (int i = max(0, issued - C::Q_NST); i < issued; ++i)
        mbar_wait_drain(&bars->full[i % C::Q_NST], (i / C::Q_NST) & 1, p.status);
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    regs_dec<kRegsLow>();
    if (lane == 0) {
      const uint32_t ring = smem_u32(sRing);
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dodesc = qdesc + (C::TILE >> 4);
      const uint64_t rk0 = sdesc_sw128(ring, 16, 1024);        // K or V, K-major
      const uint64_t rmn0 = sdesc_sw128(ring, CHUNK, 1024);    // K, MN-major
      auto slot_off = [](int i) { return static_cast<uint64_t>((i % C::Q_NST) * C::TILE) >> 4; };
      auto wait_full = [&](int i) {
        return mbar_wait(&bars->full[i % C::Q_NST], (i / C::Q_NST) & 1, abort_flag, p.status);
      };
      auto issue_scores = [&](int jj) {  // S = Q K^T, commit; dP = dO V^T, commit
        const uint64_t sk = slot_off(2 * jj), sv = slot_off(2 * jj + 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(tmem + kColS, qdesc + off, rk0 + sk + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->s_full);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = ((ks >> 2) * CHUNK + (ks & 3) * 32) >> 4;
          mma_ss(tmem + kColDP, dodesc + off, rk0 + sv + off, C::IDESC_S, ks > 0);
        }
        tc_commit(&bars->dp_full);
        tc_commit(&bars->empty[(2 * jj + 1) % C::Q_NST]);  // V(jj) consumed by dP
      };
      auto issue_dq_half = [&](int jj, int h) {  // dQ += dS K over keys [64h, 64h+64)
        const uint64_t sk = slot_off(2 * jj);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int ks = 4 * h + kk;
          mma_ts(tmem + kColAcc0, tmem + kColS + packed_col(ks), rmn0 + sk + ((ks * 2048) >> 4),
                 C::IDESC_G, (jj > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&bars->res_full, 0, abort_flag, p.status);
      if (ok && n_items > 0 && (ok = wait_full(0) && wait_full(1))) {
        tc_fence_after();
        issue_scores(0);
      }
      for (int jj = 0; ok && jj < n_items; ++jj) {
        for (int h = 0; h < 2; ++h) {
          if (!(ok = mbar_wait(&bars->p_full[h], jj & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_dq_half(jj, h);
        }
        if (!ok) break;
        tc_commit(&bars->empty[(2 * jj) % C::Q_NST]);  // K(jj) consumed
        if (jj + 1 < n_items) {
          if (!(ok = wait_full(2 * jj + 2) && wait_full(2 * jj + 3))) break;
          tc_fence_after();
          issue_scores(jj + 1);  // in order after dQ(jj), which reads dS from these columns
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
    const int wg = (warp - 4) >> 2;  // this warpgroup's 64 key columns
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int row = row0 + r;  // query row; rows >= N have l2 = +inf, so P = 0
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + 64 * wg;
    const uint32_t tDP = tmem + lane_off + kColDP + 64 * wg;
    const float c = p.scale_log2;
    const float l2s = p.l2[static_cast<size_t>(bh) * p.Npad + row];
    const float dds = p.dvec[static_cast<size_t>(bh) * p.Npad + row];
    const float slope2 = kAlibi ? p.slopes[hq] * 1.4426950408889634f : 0.f;
    bool ok = true;
    for (int jj = 0; jj < n_items; ++jj) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, jj & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      const int kb = (js + jj) * BT + 64 * wg;  // first key of this warpgroup's columns
      float pv0[32], pv1[32];
      {
        uint32_t s0[32], s1[32];
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_ld_wait(s0);
        tmem_ld_wait(s1);
        auto vis0 = [&](int i) {
          const int kk = kb + i;
          return kk < p.N && (!p.causal || kk <= row) && (p.window <= 0 || row - kk < p.window);
        };
        auto vis1 = [&](int i) { return vis0(i + 32); };
        const bool full0 = kb + 31 < p.N && (!p.causal || kb + 31 <= row) &&
                           (p.window <= 0 || row - kb < p.window);
        const bool full1 = kb + 63 < p.N && (!p.causal || kb + 63 <= row) &&
                           (p.window <= 0 || row - kb - 32 < p.window);
        const float bias0 = slope2 * static_cast<float>(kb - row);
        if (__all_sync(0xffffffffu, full0))
          p_cols<kAlibi, false>(s0, nullptr, l2s, false, c, bias0, slope2, vis0, pv0);
        else
          p_cols<kAlibi, true>(s0, nullptr, l2s, false, c, bias0, slope2, vis0, pv0);
        if (__all_sync(0xffffffffu, full1))
          p_cols<kAlibi, false>(s1, nullptr, l2s, false, c, bias0 + 32.f * slope2, slope2, vis1, pv1);
        else
          p_cols<kAlibi, true>(s1, nullptr, l2s, false, c, bias0 + 32.f * slope2, slope2, vis1, pv1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, jj & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t d0[32], d1[32];
        tmem_ld32(tDP, d0);
        tmem_ld32(tDP + 32, d1);
        tmem_ld_wait(d0);
        tmem_ld_wait(d1);
        uint32_t dk[16];
        ds_cols(pv0, d0, nullptr, dds, false, dk);
        tmem_st16(tS, dk);
        ds_cols(pv1, d1, nullptr, dds, false, dk);
        tmem_st16(tS + 16, dk);
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
          tmem_ld32(tmem + lane_off + kColAcc0 + cc * 32, v);
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
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::KV_SMEM);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(bwd_dq_kernel<D, kAlibi>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::Q_SMEM);
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
  bwd_dkdv_kernel<D, kAlibi><<<static_cast<unsigned>(kv_ctas), NUM_THREADS, C::KV_SMEM, stream>>>(
      mk, mv, mq, mdo, prm);
  bwd_dq_kernel<D, kAlibi><<<static_cast<unsigned>(q_ctas), NUM_THREADS, C::Q_SMEM, stream>>>(
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
