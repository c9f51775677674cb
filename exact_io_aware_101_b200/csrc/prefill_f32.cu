// prefill_f32.cu -- float32 exact attention forward (CUDA cores).
//
// The correctness path for float32 inputs: the same tiled online softmax as the
// bf16 tensor-core kernel ("Phase 08" page, Lab 01 steps 2-4 and the online
// softmax recurrence of its talking points), in float32 arithmetic with the
// accurate expf/logf, so that it meets the Lab 01 bar of 1e-4 against standard
// attention.  It also takes the Lab 01 extensions: a sliding window (key j
// visible only if i - j < window) and per-head ALiBi slopes (bias
// slope * (j - i) added to the scaled score).
//
// A CTA owns 16 query rows of one (batch, head); each of its 4 warps keeps 4
// rows' running max m, sum l and output accumulator (d/32 columns per lane).
// K/V tiles of 32 keys are staged in shared memory; lane j scores key j of the
// tile, the warp reduces the tile max and sum with shuffles, then every lane
// accumulates sum_j p_j v_j for its columns.  Causal CTAs stop at the diagonal.
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"

namespace exattn {
namespace {

constexpr int kRows = 16;      // query rows per CTA
constexpr int kKeys = 32;      // keys per K/V tile
constexpr int kRowsPerWarp = 4;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(128)
    prefill_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
                       const float *__restrict__ v, float *__restrict__ o,
                       float *__restrict__ lse, int Hq, int Hkv, int N, float scale, int causal,
                       int window, const float *__restrict__ slopes) {
  constexpr int DPL = D / 32;  // output columns per lane
  __shared__ float sQ[kRows][D];
  __shared__ float sK[kKeys][D + 1];  // +1: lane j reads row j without bank conflicts
  __shared__ float sV[kKeys][D];

  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq;
  const int g = h / (Hq / Hkv);
  const int row0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float *qh = q + (static_cast<size_t>(b) * Hq + h) * N * D;
  const float *kh = k + (static_cast<size_t>(b) * Hkv + g) * N * D;
  const float *vh = v + (static_cast<size_t>(b) * Hkv + g) * N * D;

  for (int idx = threadIdx.x; idx < kRows * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    sQ[r][c] = (row0 + r < N) ? qh[static_cast<size_t>(row0 + r) * D + c] : 0.f;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][DPL];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[rr][e] = 0.f;
  }

  const int kv_end = causal ? min(N, row0 + kRows) : N;
  const int kv_begin = window > 0 ? (max(0, row0 - window + 1) / kKeys) * kKeys : 0;
  const float slope = slopes ? slopes[h] : 0.f;
  for (int kt = kv_begin; kt < kv_end; kt += kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeys * D; idx += blockDim.x) {
      const int j = idx / D, c = idx % D;
      const bool in = kt + j < N;
      sK[j][c] = in ? kh[static_cast<size_t>(kt + j) * D + c] : 0.f;
      sV[j][c] = in ? vh[static_cast<size_t>(kt + j) * D + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int lr = warp * kRowsPerWarp + rr;
      const int i = row0 + lr;
      const int j = kt + lane;
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) s = fmaf(sQ[lr][c], sK[lane][c], s);
      s = s * scale + slope * static_cast<float>(j - i);
      const bool vis = (j < N) && (!causal || j <= i) && (window <= 0 || i - j < window);
      s = vis ? s : -INFINITY;
      const float tmax = warp_max(s);
      const float m_new = fmaxf(m[rr], tmax);
      if (m_new == -INFINITY) continue;  // nothing visible yet for this row
      const float alpha = expf(m[rr] - m_new);
      const float pj = vis ? expf(s - m_new) : 0.f;
      l[rr] = l[rr] * alpha + warp_sum(pj);
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[rr][e] *= alpha;
      for (int jj = 0; jj < kKeys; ++jj) {
        const float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[rr][e] = fmaf(pb, sV[jj][lane + 32 * e], acc[rr][e]);
      }
      m[rr] = m_new;
    }
  }

#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int i = row0 + warp * kRowsPerWarp + rr;
    if (i >= N) continue;
    const float inv = 1.f / l[rr];
    float *orow = o + ((static_cast<size_t>(b) * Hq + h) * N + i) * D;
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[lane + 32 * e] = acc[rr][e] * inv;
    if (lane == 0) lse[(static_cast<size_t>(b) * Hq + h) * N + i] = m[rr] + logf(l[rr]);
  }
}

}  // namespace

attn_status_t launch_prefill_f32(const float *q, const float *k, const float *v, float *o,
                                 float *lse, int B, int Hq, int Hkv, int N, int d, float scale,
                                 int causal, int window, const float *slopes,
                                 cudaStream_t stream) {
  const long long bh = static_cast<long long>(B) * Hq;
  if (bh > 65535) return ATTN_ERR_UNSUPPORTED;
  dim3 grid((N + kRows - 1) / kRows, static_cast<unsigned>(bh));
  if (d == 128)
    prefill_f32_kernel<128><<<grid, 128, 0, stream>>>(q, k, v, o, lse, Hq, Hkv, N, scale, causal,
                                                      window, slopes);
  else if (d == 64)
    prefill_f32_kernel<64><<<grid, 128, 0, stream>>>(q, k, v, o, lse, Hq, Hkv, N, scale, causal,
                                                     window, slopes);
  else
    return ATTN_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace exattn
