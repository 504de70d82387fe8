// Per-chunk statistics of the SR-TTT surprisal gate ("SR-TTT: Surprisal-Aware Residual
// Test-Time Training", §2.1 Surprisal Filter), shared by the standalone gate kernel and the
// gate fused into the TTT-Linear scan. A chunk is 64 fp32 losses in shared memory, read by
// one warp; lane j owns tokens j and 32 + j.
#pragma once

#include <math.h>
#include <stdint.h>

namespace ttt {

// Order-preserving map of fp32 bits to uint32, with every NaN mapped to the largest key (an
// ascending sort puts NaNs last). No float maps to key 0.
__device__ __forceinline__ uint32_t f32_order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  if (isnan(v)) return 0xffffffffu;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float f32_from_order_key(uint32_t k) {
  if (k == 0xffffffffu) return __uint_as_float(0x7fc00000u);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// The n-th largest (1 ≤ n ≤ K, counted with multiplicity) of the 64 keys two per lane, the same
// in every lane: each lane keeps a descending list of its K largest keys and five butterfly
// rounds merge it with the partner lane's list (the elementwise maximum of one list and the
// other reversed holds the K largest of both as a bitonic sequence, which a bitonic sorter
// orders again). Key 0, below every float's key, pads the lists.
template <int K>
__device__ __forceinline__ uint32_t warp_top_k(uint32_t k0, uint32_t k1, int n) {
  uint32_t L[K];
  L[0] = max(k0, k1);
  L[1] = min(k0, k1);
#pragma unroll
  for (int i = 2; i < K; ++i) L[i] = 0u;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t P[K];
#pragma unroll
    for (int i = 0; i < K; ++i) P[i] = __shfl_xor_sync(0xffffffffu, L[i], o);
#pragma unroll
    for (int i = 0; i < K; ++i) L[i] = max(L[i], P[K - 1 - i]);
#pragma unroll
    for (int d = K / 2; d >= 1; d >>= 1)
#pragma unroll
      for (int i = 0; i < K; ++i)
        if ((i & d) == 0) {
          const uint32_t hi = max(L[i], L[i + d]), lo = min(L[i], L[i + d]);
          L[i] = hi;
          L[i + d] = lo;
        }
  }
  uint32_t r = L[0];
#pragma unroll
  for (int i = 1; i < K; ++i)
    if (i == n - 1) r = L[i];
  return r;
}

// p = the rank-th smallest of the 64 values (1-based nearest rank, NaNs last as in an
// ascending sort) and S = their double sum in index order, both the same in every lane.
//
// Selection, for ranks within 8 of the top (the 95th percentile of 64 is the 61st smallest,
// i.e. the 4th largest counted with multiplicity): a butterfly merge of per-lane top-K lists
// (warp_top_k). Other ranks count, for each lane's two values, how many of the 64 are
// strictly smaller (every lane reads all 64 by shared-memory broadcasts); p is the largest
// value with at most rank − 1 smaller ones.
//
// Sum: if all values are finite and non-negative and their exponent fields span at most 23
// (smallest field counted as at least 1), every partial sum is an integer multiple of the
// smallest ulp among them and below 2^53 of it, so every order of double additions is exact
// and a tree sum equals the index-order sum bit for bit. Otherwise the index-order sum is
// taken literally.
__device__ __forceinline__ void chunk_stats(const float* x, int lane, int rank, float& p, double& S) {
  const float v0 = x[lane], v1 = x[lane + 32];

  const uint32_t b0 = __float_as_uint(v0), b1 = __float_as_uint(v1);
  const uint32_t e0 = (b0 >> 23) & 0xffu, e1 = (b1 >> 23) & 0xffu;
  const bool ok = (b0 >> 31) == 0u && (b1 >> 31) == 0u && e0 != 0xffu && e1 != 0xffu;
  const uint32_t emax = __reduce_max_sync(0xffffffffu, max(e0, e1));
  const uint32_t emin =
      __reduce_min_sync(0xffffffffu, min(b0 != 0u ? max(e0, 1u) : 0xffu, b1 != 0u ? max(e1, 1u) : 0xffu));
  const bool exact = __all_sync(0xffffffffu, ok) && (int)emax - (int)emin <= 23;
  if (exact) {
    double s = (double)v0 + (double)v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    S = s;
  } else {
    double s = 0.0;
    for (int j = 0; j < 64; ++j) s += (double)x[j];
    S = s;
  }

  if (65 - rank <= 4) {
    p = f32_from_order_key(warp_top_k<4>(f32_order_key(v0), f32_order_key(v1), 65 - rank));
  } else if (65 - rank <= 8) {
    p = f32_from_order_key(warp_top_k<8>(f32_order_key(v0), f32_order_key(v1), 65 - rank));
  } else {
    float c0[8], c1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) c0[k] = c1[k] = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 q = *reinterpret_cast<const float4*>(x + 4 * i);
      const float a[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        c0[(4 * i + u) & 7] += a[u] < v0 ? 1.f : 0.f;
        c1[(4 * i + u) & 7] += a[u] < v1 ? 1.f : 0.f;
      }
    }
    const float n0 = ((c0[0] + c0[1]) + (c0[2] + c0[3])) + ((c0[4] + c0[5]) + (c0[6] + c0[7]));
    const float n1 = ((c1[0] + c1[1]) + (c1[2] + c1[3])) + ((c1[4] + c1[5]) + (c1[6] + c1[7]));
    uint32_t best = 0u;
    if (n0 <= (float)(rank - 1) && !isnan(v0)) best = f32_order_key(v0);
    if (n1 <= (float)(rank - 1) && !isnan(v1)) best = max(best, f32_order_key(v1));
    best = __reduce_max_sync(0xffffffffu, best);
    // The rank-th smallest is a NaN exactly when fewer than rank values are numbers.
    const int nans = __popc(__ballot_sync(0xffffffffu, isnan(v0))) + __popc(__ballot_sync(0xffffffffu, isnan(v1)));
    p = nans > 64 - rank ? __uint_as_float(0x7fc00000u) : f32_from_order_key(best);
  }
}

// τ after a chunk with percentile p: p for the first chunk, else fl32(fl32(a·τ) + fl32(c·p)).
__device__ __forceinline__ float tau_next(float tau, bool set, float p, float ema_old, float ema_new) {
  return set ? __fadd_rn(__fmul_rn(ema_old, tau), __fmul_rn(ema_new, p)) : p;
}

}  // namespace ttt
