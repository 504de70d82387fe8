// Richer TTT inner models ("テスト時学習（Test-Time Training）とは", the TTT layers page: the
// hidden state is itself a model trained by one self-supervised step per mini-batch; its two
// instances are TTT-Linear and TTT-MLP, and by its DeltaNet remark the full TTT-Linear carries a
// LayerNorm and a residual connection). Per (sequence, head) and inner mini-batch i of 16 tokens,
// with f(x) = x + LN(g(x)), LN over the head's 64 values with per-head gain γ and bias β:
//   O_i = f(Q_i; θ_i),   E_i = f(K_i; θ_i) − V_i,   L_t = ‖E_i[t]‖²,   θ_{i+1} = θ_i − η·∇ℓ_i(θ_i)
// with ℓ_i = 1/(2b)·‖E_i‖²; g(x) = x·W (TTT-Linear with LayerNorm and residual) or
// g(x) = GELU(x·W1)·W2 (TTT-MLP, hidden width 256).
//
// Design (B200), shared with the plain TTT-Linear scan: one CTA per (sequence, head), the weights
// in mma accumulator registers for the whole scan, every product computed transposed so each
// accumulator layout is directly the next mma's A operand, K/V/Q streamed by a TMA producer warp
// through a ring of 64-token tiles (128-byte swizzle), outputs staged in shared memory and written
// by TMA stores. The per-head chain of dependent steps bounds both kernels, as it bounds the plain
// scan; what is new is LayerNorm, whose statistics span the 64 columns that the compute warps
// split between them:
//  * inside a warp, the eight lanes that share a token reduce by a butterfly reduce-scatter
//    (seven shuffles for eight sums) and an all-gather, two-pass (mean, then the squared
//    deviations from it);
//  * across warps, the per-warp (sum, M2) pairs meet in shared memory behind one named barrier
//    and are merged by the parallel-variance formula, so each step has one barrier for the
//    forward statistics and one for the backward ones (Σg and Σg·ẑ, g = γ·E).
// The weights and the update operand S = −(η/b)·∂ℓ/∂Z reach the tensor cores as bf16 hi + lo
// pairs (x ≈ hi + lo to ~2^-17 relative, two mma per product): LayerNorm's 1/σ and the
// recurrence amplify operand rounding, and with single bf16 operands the outputs drift to
// ~1e-2 of their scale over 128 steps, against ~1e-5 with the pairs (measured on the CPU
// against float64). The weights and every accumulation stay fp32.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int kStagesI = 4;                   // 64-token tiles in flight
constexpr int kTileTokI = 64;
constexpr int kTileBytesI = kTileTokI * 128;  // 64 tokens x 64 bf16
constexpr int kMB = 16;                       // inner mini-batch

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
}

// Two fp32 values as packed bf16 hi and lo words (x ≈ hi + lo).
__device__ __forceinline__ void hilo2(float x, float y, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = pack_bf16(x - hf.x, y - hf.y);
}

// A fragment (hi and lo) of a 16x16 slice of an accumulator-layout matrix from its two
// 16x8 accumulator tiles c0 (k 0..7) and c1 (k 8..15).
__device__ __forceinline__ void afrag_hilo(const float (&c0)[4], const float (&c1)[4], uint32_t (&hi)[4],
                                           uint32_t (&lo)[4]) {
  hilo2(c0[0], c0[1], hi[0], lo[0]);
  hilo2(c0[2], c0[3], hi[1], lo[1]);
  hilo2(c1[0], c1[1], hi[2], lo[2]);
  hilo2(c1[2], c1[3], hi[3], lo[3]);
}

template <int kWarps>
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32));
}

// Butterfly reduce-scatter over the eight lanes that share lane & 3 (lane bits 2..4 = g): each
// lane brings eight values, and lane g leaves with the sum of value g over the eight lanes.
__device__ __forceinline__ float reduce_scatter8(const float (&v)[8], int g) {
  const bool b2 = g & 4, b1 = g & 2, b0 = g & 1;
  float a[4], c[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = (b2 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, b2 ? v[i] : v[i + 4], 16);
#pragma unroll
  for (int i = 0; i < 2; ++i) c[i] = (b1 ? a[i + 2] : a[i]) + __shfl_xor_sync(0xffffffffu, b1 ? a[i] : a[i + 2], 8);
  return (b0 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, b0 ? c[0] : c[1], 4);
}

// The inverse: lane g holds value g; every lane of the eight leaves with all eight values.
__device__ __forceinline__ void all_gather8(float x, float (&v)[8], int g) {
  const bool b2 = g & 4, b1 = g & 2, b0 = g & 1;
  const float y = __shfl_xor_sync(0xffffffffu, x, 4);
  const float c0 = b0 ? y : x, c1 = b0 ? x : y;  // values (g & 6) + 0, 1
  const float p0 = __shfl_xor_sync(0xffffffffu, c0, 8), p1 = __shfl_xor_sync(0xffffffffu, c1, 8);
  float a[4];  // values (g & 4) + 0..3
  a[0] = b1 ? p0 : c0;
  a[1] = b1 ? p1 : c1;
  a[2] = b1 ? c0 : p0;
  a[3] = b1 ? c1 : p1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float p = __shfl_xor_sync(0xffffffffu, a[i], 16);
    v[i] = b2 ? p : a[i];
    v[i + 4] = b2 ? a[i] : p;
  }
}

// Arguments of one scan launch (both kernels).
struct InnerArgs {
  float* W;            // [B·H] per-head weights, fp32, updated in place
  const float* W0;     // the pretrained weights (packed sequences reset to them)
  const float* gamma;  // LayerNorm gain and bias [H, 64]
  const float* beta;
  float* loss;         // [B·H, T] or null
  const int2* steps;   // packed sequences: per (sequence, mini-batch) {reset to W0 first, real tokens}; or null
  int T, heads, nsteps;  // nsteps: entries of steps a sequence
  float eta, eps;
  DevStatus status;
  int stall_tile;      // fault injection (tests): this 64-token tile is never loaded (-1: none)
};

// ============================ TTT-Linear with LayerNorm and residual ============================

constexpr int kLnWarps = 4;                       // compute warps: sixteen columns of W each
constexpr int kLnThreads = (kLnWarps + 1) * 32;   // + the TMA producer warp

struct __align__(1024) LnSmem {
  uint8_t K[kStagesI][kTileBytesI];
  uint8_t V[kStagesI][kTileBytesI];
  uint8_t Q[kStagesI][kTileBytesI];
  uint8_t O[2][kTileBytesI];
  float fwd[2][kMB][8];   // [k·W or q·W][token]: per-warp sums (warps 0..3), then per-warp M2
  float bwd[kMB][8];      // [token]: per-warp Σg, then per-warp Σg·ẑ
  float lossp[kMB][4];    // [token]: per-warp Σe²
  uint64_t full[kStagesI];
  uint64_t empty[kStagesI];
  int abort;              // set by the producer when one of its waits ran out
  int cabort[2];          // set by a compute warp whose wait for tile s ran out (index s & 1)
};

// Per-warp LayerNorm statistics of the keys' (z) and, with QUERIES, the queries' (o) products
// of a step (Zᵀ layout: this thread holds columns g, g+8 of tokens 8nt + 2q + jj): two-pass over
// the warp's sixteen columns, published as (sum, M2) in fwd[kind][token][warp] and [4 + warp].
// KEYS = false publishes the queries' statistics alone (the keys' slots are left untouched).
template <bool QUERIES, bool KEYS = true>
__device__ __forceinline__ void publish_stats(const float (&z)[2][4], const float (&o)[2][4],
                                              float (*fwd)[kMB][8], int pub_tok, int warp, int g) {
  float v8[8], all[8];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      v8[2 * nt + jj] = KEYS ? z[nt][jj] + z[nt][jj + 2] : 0.f;
      v8[4 + 2 * nt + jj] = QUERIES ? o[nt][jj] + o[nt][jj + 2] : 0.f;
    }
  const float sw = reduce_scatter8(v8, g);
  all_gather8(sw, all, g);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const float mz = all[2 * nt + jj] * (1.f / 16.f), mo = all[4 + 2 * nt + jj] * (1.f / 16.f);
      const float a = z[nt][jj] - mz, b = z[nt][jj + 2] - mz, c = o[nt][jj] - mo, d = o[nt][jj + 2] - mo;
      v8[2 * nt + jj] = KEYS ? a * a + b * b : 0.f;
      v8[4 + 2 * nt + jj] = QUERIES ? c * c + d * d : 0.f;
    }
  const float m2w = reduce_scatter8(v8, g);
  const int kind = g >> 2;
  if ((kind == 0 && KEYS) || (kind == 1 && QUERIES)) {
    fwd[kind][pub_tok][warp] = sw;
    fwd[kind][pub_tok][4 + warp] = m2w;
  }
}

// Per-token mean and 1/sqrt(var + ε) from four warps' (sum, M2) over sixteen columns each.
__device__ __forceinline__ void merge_stats(const float* p, float eps, float& mu, float& rstd) {
  const float4 S = *reinterpret_cast<const float4*>(p);
  const float4 M = *reinterpret_cast<const float4*>(p + 4);
  mu = ((S.x + S.y) + (S.z + S.w)) * (1.f / 64.f);
  const float d0 = S.x * (1.f / 16.f) - mu, d1 = S.y * (1.f / 16.f) - mu;
  const float d2 = S.z * (1.f / 16.f) - mu, d3 = S.w * (1.f / 16.f) - mu;
  const float m2 = ((M.x + M.y) + (M.z + M.w)) + 16.f * ((d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3));
  rstd = rsqrtf(m2 * (1.f / 64.f) + eps);
}

// Each lane merges the statistics it published (value g: kind g >> 2, token pub_tok) and the
// eight lanes of a token group share them: mu[i], rs[i] for value i = 4·kind + 2·nt + jj.
__device__ __forceinline__ void gather_stats(float (*fwd)[kMB][8], int pub_tok, int g, float eps, float (&mu)[8],
                                             float (&rs)[8]) {
  float m, r;
  merge_stats(fwd[g >> 2][pub_tok], eps, m, r);
  all_gather8(m, mu, g);
  all_gather8(r, rs, g);
}

__device__ __forceinline__ void stsm4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}

// Outputs q + γ·LN(o) + β of the step's sixteen tokens at this warp's sixteen columns, from the
// queries' statistics (values 4..7 of mu, rs), into the swizzled staging tile by one transposing
// stmatrix: matrix (nt, hc) holds tokens 8nt.. and columns col0 + 8hc.., its rows addressed by
// lanes 8·(2nt + hc) + row (ofs_o = that lane's row and column offset).
__device__ __forceinline__ void emit_outputs(const float (&o)[2][4], const float (&qv)[2][4], const float (&mu)[8],
                                             const float (&rs)[8], const float (&gam)[2], const float (&bet)[2],
                                             uint32_t obase, uint32_t ofs_o, int r0) {
  uint32_t r[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      float y[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int e = jj + 2 * hc, i = 4 + 2 * nt + jj;
        y[jj] = qv[nt][e] + fmaf(gam[hc], (o[nt][e] - mu[i]) * rs[i], bet[hc]);
      }
      r[2 * nt + hc] = pack_bf16(y[0], y[1]);
    }
  stsm4_t(obase + ofs_o + (uint32_t)r0 * 128u, r[0], r[1], r[2], r[3]);
}

// Plain outputs (no LayerNorm, no residual) into the staging tile, as in emit_outputs.
__device__ __forceinline__ void emit_plain(const float (&o)[2][4], uint32_t obase, uint32_t ofs_o, int r0) {
  stsm4_t(obase + ofs_o + (uint32_t)r0 * 128u, pack_bf16(o[0][0], o[0][1]), pack_bf16(o[0][2], o[0][3]),
          pack_bf16(o[1][0], o[1][1]), pack_bf16(o[1][2], o[1][3]));
}

// LN = true: TTT-Linear with LayerNorm and residual; LN = false: the plain TTT-Linear rule
// (f(x) = x·W), run by this kernel for per-token weights and packed sequences.
//
// TW: per-token weights within the mini-batch. Token t's output uses
// W_t = W_i + Σ_{s ≤ t} k_sᵀ·S_s (S = −(η/n)·∂ℓ/∂Z, every gradient at W_i), so
// q_t·W_t = q_t·W_i + Σ_{s ≤ t} (q_t·k_s)·S_s: the query products of the forward pass plus
// Sᵀ·Mᵀ with M = Q·Kᵀ masked to s ≤ t, added once S is known; with LayerNorm the outputs'
// statistics then take a third exchange.
//
// Packed sequences (a.steps set): each (sequence, mini-batch) entry says whether the weight
// goes back to W0 before it (a document's first mini-batch) and how many of its 16 tokens are
// real (a document's last mini-batch may be shorter; the rest are zero padding): padded
// tokens contribute no gradient and the step is η/n for n real tokens.
template <bool HAS_Q, bool LOSS, bool TW, bool LN>
__global__ void __launch_bounds__(kLnThreads, 1)
    k_inner_ln(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO, const InnerArgs a) {
  extern __shared__ uint8_t smem_raw[];
  LnSmem& sm = *reinterpret_cast<LnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int T = a.T;
  const int ntiles = (T + kTileTokI - 1) / kTileTokI;
  const uint32_t stage_bytes = (HAS_Q ? 3u : 2u) * kTileBytesI;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesI; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kLnWarps);
    }
    sm.abort = 0;
    sm.cabort[0] = sm.cabort[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kLnWarps) {
    // ---------------- producer: TMA loads of K, V, Q tiles ----------------
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < ntiles; ++s) {
        const int slot = s % kStagesI;
        if (s >= kStagesI && !mbar_wait(&sm.empty[slot], ((s / kStagesI) - 1) & 1, a.status, &sm.abort)) break;
        if (s != a.stall_tile) {
          mbar_arrive_expect_tx(&sm.full[slot], stage_bytes);
          tma_load_3d(sm.K[slot], &tmK, &sm.full[slot], 0, s * kTileTokI, bh);
          tma_load_3d(sm.V[slot], &tmV, &sm.full[slot], 0, s * kTileTokI, bh);
          if (HAS_Q) tma_load_3d(sm.Q[slot], &tmQ, &sm.full[slot], 0, s * kTileTokI, bh);
        }
        issued = s + 1;
      }
      // Nothing may still be landing in shared memory when the CTA exits.
      for (int s = issued - kStagesI; s < issued; ++s) {
        if (s < 0 || s == a.stall_tile) continue;
        mbar_wait(&sm.full[s % kStagesI], (s / kStagesI) & 1, a.status, nullptr);
      }
    }
    __syncthreads();
    return;
  }

  // ---------------- compute warps ----------------
  const int g = lane >> 2, q = lane & 3, mi = lane >> 3, ri = lane & 7;
  const int col0 = 16 * warp;
  float* Wg = a.W + (size_t)bh * 64 * 64;
  const float* W0g = a.W0 + (size_t)bh * 64 * 64;
  // Wᵀ slice in accumulator layout: acc[nt][e] = W[8nt + 2q + (e&1)][col0 + g + 8(e>>1)].
  float acc[8][4];
  auto load_w = [&](const float* src) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = src[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)];
  };
  load_w(Wg);
  const int h = bh % a.heads;
  float gam[2] = {1.f, 1.f}, bet[2] = {0.f, 0.f};
  if (LN) {
    gam[0] = a.gamma[h * 64 + col0 + g];
    gam[1] = a.gamma[h * 64 + col0 + g + 8];
    bet[0] = a.beta[h * 64 + col0 + g];
    bet[1] = a.beta[h * 64 + col0 + g + 8];
  }
  const int2* steps = a.steps == nullptr ? nullptr : a.steps + (size_t)(bh / a.heads) * a.nsteps;
  // Token (within the mini-batch) whose per-warp partial this lane publishes after a
  // reduce-scatter of values indexed 4·kind + 2·nt + jj.
  const int pub_tok = 8 * ((g >> 1) & 1) + 2 * q + (g & 1);
  const uint32_t ofs_o = swz128_bf16(8 * (mi >> 1) + ri, col0 + 8 * (mi & 1));

  for (int s = 0; s < ntiles; ++s) {
    const int slot = s % kStagesI;
    // Every compute warp takes the same exit decision: the flag for tile s is only written
    // before this barrier and only read after it.
    if (!mbar_wait(&sm.full[slot], (s / kStagesI) & 1, a.status, nullptr)) sm.cabort[s & 1] = 1;
    compute_sync<kLnWarps>();
    if (*reinterpret_cast<volatile int*>(&sm.cabort[s & 1])) break;
    const int ntok = min(kTileTokI, T - s * kTileTokI);
    const uint32_t kbase = smem_u32(sm.K[slot]), vbase = smem_u32(sm.V[slot]), qbase = smem_u32(sm.Q[slot]);
    const uint32_t obase = smem_u32(sm.O[s & 1]);

    for (int r0 = 0; r0 < ntok; r0 += kMB) {
      int nval = kMB;  // real tokens of this mini-batch
      if (steps != nullptr) {
        const int2 e = steps[s * (kTileTokI / kMB) + r0 / kMB];
        if (e.x) load_w(W0g);  // a document starts: the pretrained weight
        nval = e.y;
      }
      const float lr = a.eta / (float)max(nval, 1);
      // ---- forward: Zᵀ = Wᵀ·Kᵀ and (queries) Pᵀ = Wᵀ·Qᵀ, all with the weight at the step's start
      uint32_t whi[4][4], wlo[4][4];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) afrag_hilo(acc[2 * ks], acc[2 * ks + 1], whi[ks], wlo[ks]);
      float z[2][4], o[2][4];
      // TW: M = Q·Kᵀ (tokens x tokens), mm[nt][e] = M[g + 8(e>>1)][8nt + 2q + (e&1)]; Q as the A
      // operand, the K fragments of the forward product as B.
      uint32_t qa[4][4];
      float mm[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      if (TW) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) ldsm4(qbase + swz128_bf16(r0 + 8 * (mi & 1) + ri, 16 * ks + 8 * (mi >> 1)), qa[ks]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float z2[4] = {0.f, 0.f, 0.f, 0.f}, o2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 4; ++e) z[nt][e] = o[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ks += 2) {
          const uint32_t off = swz128_bf16(r0 + 8 * nt + ri, 16 * ks + 8 * mi);
          uint32_t kb[4];
          ldsm4(kbase + off, kb);
          mma_bf16(z[nt], whi[ks], kb[0], kb[1]);
          mma_bf16(z2, wlo[ks], kb[0], kb[1]);
          mma_bf16(z[nt], whi[ks + 1], kb[2], kb[3]);
          mma_bf16(z2, wlo[ks + 1], kb[2], kb[3]);
          if (TW) {
            mma_bf16(mm[nt], qa[ks], kb[0], kb[1]);
            mma_bf16(mm[nt], qa[ks + 1], kb[2], kb[3]);
          }
          if (HAS_Q) {
            uint32_t qb[4];
            ldsm4(qbase + off, qb);
            mma_bf16(o[nt], whi[ks], qb[0], qb[1]);
            mma_bf16(o2, wlo[ks], qb[0], qb[1]);
            mma_bf16(o[nt], whi[ks + 1], qb[2], qb[3]);
            mma_bf16(o2, wlo[ks + 1], qb[2], qb[3]);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          z[nt][e] += z2[e];
          o[nt][e] += o2[e];
        }
      }
      // k − v with LayerNorm's residual, −v without (and q for the residual of the outputs) at
      // this thread's (column, token) positions of the Zᵀ layout.
      float kv[2][4], qv[2][4];
      {
        const uint32_t off = swz128_bf16(r0 + 8 * (mi >> 1) + ri, col0 + 8 * (mi & 1));
        uint32_t kr[4] = {0u, 0u, 0u, 0u}, vr[4];
        if (LN) ldsm4_t(kbase + off, kr);
        ldsm4_t(vbase + off, vr);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float2 k0 = bf2_to_f2(kr[2 * nt]), k1 = bf2_to_f2(kr[2 * nt + 1]);
          const float2 v0 = bf2_to_f2(vr[2 * nt]), v1 = bf2_to_f2(vr[2 * nt + 1]);
          kv[nt][0] = k0.x - v0.x;
          kv[nt][1] = k0.y - v0.y;
          kv[nt][2] = k1.x - v1.x;
          kv[nt][3] = k1.y - v1.y;
        }
        if (HAS_Q && LN) {
          uint32_t qr[4];
          ldsm4_t(qbase + off, qr);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const float2 p = bf2_to_f2(qr[2 * nt]), r = bf2_to_f2(qr[2 * nt + 1]);
            qv[nt][0] = p.x;
            qv[nt][1] = p.y;
            qv[nt][2] = r.x;
            qv[nt][3] = r.y;
          }
        }
      }

      // The queries' outputs now, unless TW (their products are not complete before the backward).
      constexpr bool kOutNow = HAS_Q && !TW;
      float zh[2][4], ev[2][4], gg[2][4], mu[8], rs[8];
      if (LN) {
        // ---- LayerNorm statistics: per warp two-pass over its sixteen columns, then merged
        publish_stats<kOutNow>(z, o, sm.fwd, pub_tok, warp, g);
        compute_sync<kLnWarps>();
        gather_stats(sm.fwd, pub_tok, g, a.eps, mu, rs);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int i = 2 * nt + jj;
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const int e = jj + 2 * hc;
              zh[nt][e] = (z[nt][e] - mu[i]) * rs[i];
              ev[nt][e] = fmaf(gam[hc], zh[nt][e], bet[hc]) + kv[nt][e];  // f(k) − v
              gg[nt][e] = gam[hc] * ev[nt][e];
            }
          }
        if (kOutNow) emit_outputs(o, qv, mu, rs, gam, bet, obase, ofs_o, r0);
      } else {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) gg[nt][e] = ev[nt][e] = z[nt][e] + kv[nt][e];  // k·W − v
        if (kOutNow) emit_plain(o, obase, ofs_o, r0);
      }

      // ---- backward statistics: Σg and Σg·ẑ per token (LayerNorm), Σe² for the loss
      float v8[8];
      if (LN) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            v8[2 * nt + jj] = gg[nt][jj] + gg[nt][jj + 2];
            v8[4 + 2 * nt + jj] = gg[nt][jj] * zh[nt][jj] + gg[nt][jj + 2] * zh[nt][jj + 2];
          }
        const float bw = reduce_scatter8(v8, g);
        sm.bwd[pub_tok][4 * (g >> 2) + warp] = bw;
      }
      if (LOSS) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            v8[2 * nt + jj] = ev[nt][jj] * ev[nt][jj] + ev[nt][jj + 2] * ev[nt][jj + 2];
            v8[4 + 2 * nt + jj] = 0.f;
          }
        const float lw = reduce_scatter8(v8, g);
        if (g < 4) sm.lossp[pub_tok][warp] = lw;
      }
      if (LN || LOSS) compute_sync<kLnWarps>();

      // ---- dZ (LayerNorm: rstd·(g − mean g − ẑ·mean(g·ẑ)); plain: the residual), zero for
      // padding tokens; W ← W − (η/n)·Kᵀ·dZ. Each lane sums the four warps' partials of the
      // value it published; the token group shares the means.
      float dz[2][4], bm[8];
      if (LN) {
        const float4 A = *reinterpret_cast<const float4*>(&sm.bwd[pub_tok][4 * (g >> 2)]);
        all_gather8(((A.x + A.y) + (A.z + A.w)) * (1.f / 64.f), bm, g);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int i = 2 * nt + jj;
          const bool real = 8 * nt + 2 * q + jj < nval;
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            const int e = jj + 2 * hc;
            const float d = LN ? rs[i] * (gg[nt][e] - bm[i] - zh[nt][e] * bm[4 + i]) : gg[nt][e];
            dz[nt][e] = real ? -lr * d : 0.f;
          }
        }
      if (LOSS && warp == 0) {
        const float4 L = *reinterpret_cast<const float4*>(&sm.lossp[pub_tok][0]);
        if (g < 4) a.loss[(size_t)bh * T + (size_t)s * kTileTokI + r0 + pub_tok] = (L.x + L.y) + (L.z + L.w);
      }
      uint32_t shi[4], slo[4];
      afrag_hilo(dz[0], dz[1], shi, slo);
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t kb[4];
        ldsm4_t(kbase + swz128_bf16(r0 + 8 * (mi & 1) + ri, 8 * nt + 8 * (mi >> 1)), kb);
        mma_bf16(acc[nt], shi, kb[0], kb[1]);
        mma_bf16(acc[nt], slo, kb[0], kb[1]);
        mma_bf16(acc[nt + 1], shi, kb[2], kb[3]);
        mma_bf16(acc[nt + 1], slo, kb[2], kb[3]);
      }
      if (HAS_Q && TW) {
        // Pᵀ += Sᵀ·Mᵀ, M masked to s ≤ t. The Mᵀ B fragment of token n-tile nt (t = 8nt + g)
        // holds M[t][2q, 2q+1] and M[t][8 + 2q, 9 + 2q]: the accumulator values of row t.
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 8 * nt + g;
          const float m00 = 2 * q <= t ? mm[0][2 * nt] : 0.f, m01 = 2 * q + 1 <= t ? mm[0][2 * nt + 1] : 0.f;
          const float m10 = 2 * q + 8 <= t ? mm[1][2 * nt] : 0.f, m11 = 2 * q + 9 <= t ? mm[1][2 * nt + 1] : 0.f;
          uint32_t bh0, bl0, bh1, bl1;
          hilo2(m00, m01, bh0, bl0);
          hilo2(m10, m11, bh1, bl1);
          float o2[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16(o[nt], shi, bh0, bh1);
          mma_bf16(o2, shi, bl0, bl1);
          mma_bf16(o2, slo, bh0, bh1);
#pragma unroll
          for (int e = 0; e < 4; ++e) o[nt][e] += o2[e];
        }
        if (LN) {
          publish_stats<true, false>(z, o, sm.fwd, pub_tok, warp, g);
          compute_sync<kLnWarps>();
          gather_stats(sm.fwd, pub_tok, g, a.eps, mu, rs);
          emit_outputs(o, qv, mu, rs, gam, bet, obase, ofs_o, r0);
        } else {
          emit_plain(o, obase, ofs_o, r0);
        }
      }
    }
    // End of the tile: its outputs are complete in shared memory.
    if (HAS_Q) fence_proxy_async_smem();
    compute_sync<kLnWarps>();
    if (threadIdx.x == 0 && HAS_Q) {
      tma_store_3d(&tmO, sm.O[s & 1], 0, s * kTileTokI, bh);
      bulk_commit();
      bulk_wait_read<1>();  // the other staging tile is free again
    }
    compute_sync<kLnWarps>();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
  }

  if (threadIdx.x == 0 && HAS_Q) bulk_wait<0>();
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)] = acc[nt][e];
  __syncthreads();
}

// ======================================== TTT-MLP ========================================
//
// Warp w of eight owns hidden units [32w, 32w+32): its slices of W1ᵀ (32 x 64) and W2ᵀ (64 x 32)
// stay in accumulator registers (128 fp32 a thread). The second layer contracts over the hidden
// units, so each warp's Zᵀ is a partial sum: the eight partials meet in shared memory (fp32), and
// warp w finishes LayerNorm, the loss and the output rows of tokens 2w and 2w+1 with sixteen lanes
// a token (four columns a lane), then publishes S = −(η/b)·∂ℓ/∂Z as bf16 hi and lo tiles that
// every warp reads for its gradients. W2 takes part in both orientations (Z = A·W2 forward, S·W2ᵀ backward):
// the backward's operand comes from the accumulators by movmatrix. No producer warp: the loads of
// tile s + kStagesM go out from thread 0 as soon as every warp has finished tile s, which leaves
// the register file to the eight compute warps.

constexpr int kMlpWarps = 8;
constexpr int kMlpThreads = kMlpWarps * 32;
constexpr int kStagesM = 3;
constexpr int kHid = 256;
constexpr int kRedStride = 68;  // floats per token row of a partial Zᵀ (64 + 4: stores without bank conflicts)

struct __align__(1024) MlpSmem {
  uint8_t K[kStagesM][kTileBytesI];
  uint8_t V[kStagesM][kTileBytesI];
  uint8_t Q[kStagesM][kTileBytesI];
  uint8_t O[2][kTileBytesI];
  uint8_t S[2][kMB * 128];                 // −(η/b)·∂ℓ/∂Z [token][column] as bf16 hi and lo, 128-byte swizzle
  float red[2][kMlpWarps][kMB][kRedStride];  // [keys or queries][warp][token][column]: partial Z
  uint64_t full[kStagesM];
  int cabort[2];
};

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// GELU(x) = x·Φ(x) and its derivative Φ(x) + x·φ(x), through CUDA's erff and expf.
__device__ __forceinline__ void gelu_and_grad(float x, float& y, float& dy) {
  const float cdf = 0.5f * (1.f + erff(x * 0.70710678118654752f));
  y = x * cdf;
  dy = fmaf(x * 0.39894228040143268f, expf(-0.5f * x * x), cdf);
}

// Sum over the sixteen lanes that share lane >> 4.
__device__ __forceinline__ float sum16(float x) {
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// LayerNorm of one token's four columns held by this lane (sixteen lanes hold the 64 columns).
__device__ __forceinline__ void ln16(const float (&x)[4], float eps, float (&xh)[4], float& rstd) {
  const float mu = sum16((x[0] + x[1]) + (x[2] + x[3])) * (1.f / 64.f);
  float m2 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float d = x[i] - mu;
    m2 = fmaf(d, d, m2);
  }
  rstd = rsqrtf(sum16(m2) * (1.f / 64.f) + eps);
#pragma unroll
  for (int i = 0; i < 4; ++i) xh[i] = (x[i] - mu) * rstd;
}

__device__ __forceinline__ void load4_bf16(const uint8_t* tile, int row, int col, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(tile + swz128_bf16(row, col));
  const float2 a = bf2_to_f2(u.x), b = bf2_to_f2(u.y);
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}

__device__ __forceinline__ void store4_bf16(uint8_t* tile, int row, int col, const float (&x)[4]) {
  *reinterpret_cast<uint2*>(tile + swz128_bf16(row, col)) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
}

// TW: per-token weights within the mini-batch. With every gradient at the step's starting
// weights, W1_t = W1_i + Σ_{s ≤ t} k_sᵀ·dH_s and W2_t = W2_i + Σ_{s ≤ t} a_sᵀ·S_s (dH and S carry
// −η/b), so the queries' first layer is Q·W1_i + tril(Q·Kᵀ)·dH and their second layer
// A_q·W2_i + tril(A_q·Aᵀ)·S. The second Gram matrix splits over the hidden slices like the
// product itself, so each warp adds its slice's term to its partial Zᵀ; the queries' path runs
// after the backward, and their LayerNorm behind a third barrier.
template <bool HAS_Q, bool LOSS, bool TW>
__global__ void __launch_bounds__(kMlpThreads, 1)
    k_inner_mlp(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                const InnerArgs a) {
  extern __shared__ uint8_t smem_raw[];
  MlpSmem& sm = *reinterpret_cast<MlpSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3, mi = lane >> 3, ri = lane & 7;
  const int bh = blockIdx.x;
  const int T = a.T;
  const float eps = a.eps;
  const int ntiles = (T + kTileTokI - 1) / kTileTokI;
  const uint32_t stage_bytes = (HAS_Q ? 3u : 2u) * kTileBytesI;

  auto issue = [&](int s) {
    if (s == a.stall_tile) return;
    const int slot = s % kStagesM;
    mbar_arrive_expect_tx(&sm.full[slot], stage_bytes);
    tma_load_3d(sm.K[slot], &tmK, &sm.full[slot], 0, s * kTileTokI, bh);
    tma_load_3d(sm.V[slot], &tmV, &sm.full[slot], 0, s * kTileTokI, bh);
    if (HAS_Q) tma_load_3d(sm.Q[slot], &tmQ, &sm.full[slot], 0, s * kTileTokI, bh);
  };
  int issued = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesM; ++i) mbar_init(&sm.full[i], 1);
    sm.cabort[0] = sm.cabort[1] = 0;
    fence_barrier_init();
    for (; issued < kStagesM && issued < ntiles; ++issued) issue(issued);
  }
  __syncthreads();

  // Per head: W1 [64][256] then W2 [256][64], row-major fp32.
  float* W1g = a.W + (size_t)bh * 2 * 64 * kHid;
  float* W2g = W1g + 64 * kHid;
  const float* W10 = a.W0 + (size_t)bh * 2 * 64 * kHid;
  const int hid0 = 32 * warp;
  // a1[mt][nt][e] = W1ᵀ[hid0 + 16mt + g + 8(e>>1)][8nt + 2q + (e&1)]
  // a2[mt][nt][e] = W2ᵀ[16mt + g + 8(e>>1)][hid0 + 8nt + 2q + (e&1)]
  float a1[2][8][4], a2[4][4][4];
  auto load_w = [&](const float* w1, const float* w2) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          a1[mt][nt][e] = w1[(8 * nt + 2 * q + (e & 1)) * kHid + hid0 + 16 * mt + g + 8 * (e >> 1)];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          a2[mt][nt][e] = w2[(hid0 + 8 * nt + 2 * q + (e & 1)) * 64 + 16 * mt + g + 8 * (e >> 1)];
  };
  load_w(W1g, W2g);
  const int2* steps = a.steps == nullptr ? nullptr : a.steps + (size_t)(bh / a.heads) * a.nsteps;

  // LayerNorm stage: token 2·warp + (lane >> 4), columns c0 .. c0+3.
  const int ltok = 2 * warp + (lane >> 4), c0 = 4 * (lane & 15);
  const int h = bh % a.heads;
  float gam[4], bet[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    gam[i] = a.gamma[h * 64 + c0 + i];
    bet[i] = a.beta[h * 64 + c0 + i];
  }
  const uint32_t sbase[2] = {smem_u32(sm.S[0]), smem_u32(sm.S[1])};

  int s = 0;
  for (; s < ntiles; ++s) {
    const int slot = s % kStagesM;
    if (!mbar_wait(&sm.full[slot], (s / kStagesM) & 1, a.status, nullptr)) sm.cabort[s & 1] = 1;
    compute_sync<kMlpWarps>();
    if (*reinterpret_cast<volatile int*>(&sm.cabort[s & 1])) break;
    const int ntok = min(kTileTokI, T - s * kTileTokI);
    const uint8_t* Kt = sm.K[slot];
    const uint8_t* Vt = sm.V[slot];
    const uint8_t* Qt = sm.Q[slot];
    const uint32_t kbase = smem_u32(Kt), qbase = smem_u32(Qt);
    uint8_t* obuf = sm.O[s & 1];

    for (int r0 = 0; r0 < ntok; r0 += kMB) {
      int nval = kMB;  // real tokens of this mini-batch (packed sequences: see k_inner_ln)
      if (steps != nullptr) {
        const int2 e = steps[s * (kTileTokI / kMB) + r0 / kMB];
        if (e.x) load_w(W10, W10 + 64 * kHid);  // a document starts: the pretrained weights
        nval = e.y;
      }
      const float lr = a.eta / (float)max(nval, 1);
      constexpr bool kQNow = HAS_Q && !TW;  // the queries' path alongside the keys'
      // ---- first layer: Hᵀ = W1ᵀ·Kᵀ (and for the queries), hidden x tokens
      float hk[2][2][4], hq[2][2][4];
      // TW: M = Q·Kᵀ, mm[nt][e] = M[g + 8(e>>1)][8nt + 2q + (e&1)] (Q as the A operand, the K
      // fragments of the first layer as B).
      float mm[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) hk[mt][nt][e] = hq[mt][nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 4; ks += 2) {
        uint32_t kb[2][4], qb[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t off = swz128_bf16(r0 + 8 * nt + ri, 16 * ks + 8 * mi);
          ldsm4(kbase + off, kb[nt]);
          if (HAS_Q) ldsm4(qbase + off, qb[nt]);
        }
        if (TW) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            uint32_t qa[4];
            ldsm4(qbase + swz128_bf16(r0 + 8 * (mi & 1) + ri, 16 * (ks + kk) + 8 * (mi >> 1)), qa);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma_bf16(mm[nt], qa, kb[nt][2 * kk], kb[nt][2 * kk + 1]);
          }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t whi[2][4], wlo[2][4];  // k-steps ks, ks + 1
          afrag_hilo(a1[mt][2 * ks], a1[mt][2 * ks + 1], whi[0], wlo[0]);
          afrag_hilo(a1[mt][2 * ks + 2], a1[mt][2 * ks + 3], whi[1], wlo[1]);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              mma_bf16(hk[mt][nt], whi[kk], kb[nt][2 * kk], kb[nt][2 * kk + 1]);
              mma_bf16(hk[mt][nt], wlo[kk], kb[nt][2 * kk], kb[nt][2 * kk + 1]);
              if (HAS_Q) {
                // The queries' products feed only the outputs (no recurrence amplifies their
                // rounding): the bf16 weights alone, except with TW, whose corrections follow.
                mma_bf16(hq[mt][nt], whi[kk], qb[nt][2 * kk], qb[nt][2 * kk + 1]);
                if (TW) mma_bf16(hq[mt][nt], wlo[kk], qb[nt][2 * kk], qb[nt][2 * kk + 1]);
              }
            }
        }
      }
      // ---- activation; A is kept as packed bf16 pairs in the accumulator layout (the B operand
      // of the second layer's update) and GELU'(H) for the backward.
      uint32_t ak[2][2][2], aq[2][2][2];
      float dact[2][2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          float y[4], yq[4], dq;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            gelu_and_grad(hk[mt][nt][e], y[e], dact[mt][nt][e]);
            if (kQNow) gelu_and_grad(hq[mt][nt][e], yq[e], dq);
          }
          ak[mt][nt][0] = pack_bf16(y[0], y[1]);
          ak[mt][nt][1] = pack_bf16(y[2], y[3]);
          if (kQNow) {
            aq[mt][nt][0] = pack_bf16(yq[0], yq[1]);
            aq[mt][nt][1] = pack_bf16(yq[2], yq[3]);
          }
        }
      // ---- second layer, this warp's share: Zᵀ_w = W2ᵀ[:, slice]·Aᵀ[slice, :], columns x tokens.
      // Aᵀ B fragments (hidden x tokens) by transposing the 8x8 blocks of the accumulator-layout A.
      {
        uint32_t bk[2][2][2], bq[2][2][2];  // [token n-tile][hidden k-step][half]
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              bk[nt][ks][hh] = movm_t(ak[ks][nt][hh]);
              if (kQNow) bq[nt][ks][hh] = movm_t(aq[ks][nt][hh]);
            }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t whi[2][4], wlo[2][4];  // hidden k-steps 0, 1
          afrag_hilo(a2[mt][0], a2[mt][1], whi[0], wlo[0]);
          afrag_hilo(a2[mt][2], a2[mt][3], whi[1], wlo[1]);
#pragma unroll
          for (int kind = 0; kind < (kQNow ? 2 : 1); ++kind) {
            float* red = &sm.red[kind][warp][0][0];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const uint32_t(&b)[2][2] = kind == 0 ? bk[nt] : bq[nt];
              float zp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                mma_bf16(zp, whi[ks], b[ks][0], b[ks][1]);
                if (kind == 0) mma_bf16(zp, wlo[ks], b[ks][0], b[ks][1]);  // queries: bf16 weights alone
              }
#pragma unroll
              for (int e = 0; e < 4; ++e)
                red[(8 * nt + 2 * q + (e & 1)) * kRedStride + 16 * mt + g + 8 * (e >> 1)] = zp[e];
            }
          }
        }
      }
      compute_sync<kMlpWarps>();

      // ---- LayerNorm, loss, outputs and S for tokens 2w, 2w+1
      {
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < kMlpWarps; ++p) {
          const float4 v = *reinterpret_cast<const float4*>(&sm.red[0][p][ltok][c0]);
          z[0] += v.x;
          z[1] += v.y;
          z[2] += v.z;
          z[3] += v.w;
        }
        float zh[4], rstd, kx[4], vx[4], ev[4], gg[4];
        ln16(z, eps, zh, rstd);
        load4_bf16(Kt, r0 + ltok, c0, kx);
        load4_bf16(Vt, r0 + ltok, c0, vx);
        float sg = 0.f, sgz = 0.f, se = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ev[i] = fmaf(gam[i], zh[i], bet[i]) + (kx[i] - vx[i]);  // f(k) − v
          gg[i] = gam[i] * ev[i];
          sg += gg[i];
          sgz = fmaf(gg[i], zh[i], sgz);
          se = fmaf(ev[i], ev[i], se);
        }
        const float mg = sum16(sg) * (1.f / 64.f), mgz = sum16(sgz) * (1.f / 64.f);
        float sv[4], sl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sv[i] = ltok < nval ? -lr * (rstd * (gg[i] - mg - zh[i] * mgz)) : 0.f;  // padding: no gradient
          sl[i] = sv[i] - __bfloat162float(__float2bfloat16_rn(sv[i]));
        }
        store4_bf16(sm.S[0], ltok, c0, sv);  // rounds to the hi part
        store4_bf16(sm.S[1], ltok, c0, sl);
        if (LOSS) {
          se = sum16(se);
          if ((lane & 15) == 0) a.loss[(size_t)bh * T + (size_t)s * kTileTokI + r0 + ltok] = se;
        }
      }
      // Outputs of tokens 2w, 2w+1: q + γ·LN(Σ partial Zᵀ of the queries) + β.
      auto query_outputs = [&]() {
        float zq[4] = {0.f, 0.f, 0.f, 0.f}, qh[4], qr, qx[4], y[4];
#pragma unroll
        for (int p = 0; p < kMlpWarps; ++p) {
          const float4 v = *reinterpret_cast<const float4*>(&sm.red[1][p][ltok][c0]);
          zq[0] += v.x;
          zq[1] += v.y;
          zq[2] += v.z;
          zq[3] += v.w;
        }
        ln16(zq, eps, qh, qr);
        load4_bf16(Qt, r0 + ltok, c0, qx);
#pragma unroll
        for (int i = 0; i < 4; ++i) y[i] = qx[i] + fmaf(gam[i], qh[i], bet[i]);
        store4_bf16(obuf, r0 + ltok, c0, y);
      };
      if (kQNow) query_outputs();
      compute_sync<kMlpWarps>();

      // ---- backward, every warp for its hidden slice; gradients at the step's starting weights
      // dHᵀ = (W2[slice, :]·Sᵀ) ⊙ GELU'(H): W2 as the A operand, transposed from the W2ᵀ slice.
      float dh[2][2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) dh[mt][nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 4; ks += 2) {
        uint32_t sb[2][2][4];  // Sᵀ B fragments (columns x tokens): [hi, lo][token n-tile]
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) ldsm4(sbase[p] + swz128_bf16(8 * nt + ri, 16 * ks + 8 * mi), sb[p][nt]);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int fk = ks + kk;  // 16-column k-step = W2ᵀ feature m-tile
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            uint32_t w[4];
            w[0] = movm_t(pack_bf16(a2[fk][2 * mt][0], a2[fk][2 * mt][1]));
            w[1] = movm_t(pack_bf16(a2[fk][2 * mt + 1][0], a2[fk][2 * mt + 1][1]));
            w[2] = movm_t(pack_bf16(a2[fk][2 * mt][2], a2[fk][2 * mt][3]));
            w[3] = movm_t(pack_bf16(a2[fk][2 * mt + 1][2], a2[fk][2 * mt + 1][3]));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int p = 0; p < 2; ++p) mma_bf16(dh[mt][nt], w, sb[p][nt][2 * kk], sb[p][nt][2 * kk + 1]);
          }
        }
      }
      // dHᵀ = dh ⊙ GELU'(H) as A fragments (hidden x tokens), S already carrying −η/b.
      uint32_t da[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        da[mt][0] = pack_bf16(dh[mt][0][0] * dact[mt][0][0], dh[mt][0][1] * dact[mt][0][1]);
        da[mt][1] = pack_bf16(dh[mt][0][2] * dact[mt][0][2], dh[mt][0][3] * dact[mt][0][3]);
        da[mt][2] = pack_bf16(dh[mt][1][0] * dact[mt][1][0], dh[mt][1][1] * dact[mt][1][1]);
        da[mt][3] = pack_bf16(dh[mt][1][2] * dact[mt][1][2], dh[mt][1][3] * dact[mt][1][3]);
      }
      if (HAS_Q && TW) {
        // Queries' first layer (from the forward pass): Hqᵀ += dHᵀ·Mᵀ with M masked to s ≤ t (the
        // Mᵀ B fragment of token n-tile nt holds row t = 8nt + g of M).
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 8 * nt + g;
          const float m00 = 2 * q <= t ? mm[0][2 * nt] : 0.f, m01 = 2 * q + 1 <= t ? mm[0][2 * nt + 1] : 0.f;
          const float m10 = 2 * q + 8 <= t ? mm[1][2 * nt] : 0.f, m11 = 2 * q + 9 <= t ? mm[1][2 * nt + 1] : 0.f;
          uint32_t bh0, bl0, bh1, bl1;
          hilo2(m00, m01, bh0, bl0);
          hilo2(m10, m11, bh1, bl1);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_bf16(hq[mt][nt], da[mt], bh0, bh1);
            mma_bf16(hq[mt][nt], da[mt], bl0, bl1);
          }
        }
      }
      // W1ᵀ += dHᵀ·K.
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t kb[4];
          ldsm4_t(kbase + swz128_bf16(r0 + 8 * (mi & 1) + ri, 8 * nt + 8 * (mi >> 1)), kb);
          mma_bf16(a1[mt][nt], da[mt], kb[0], kb[1]);
          mma_bf16(a1[mt][nt + 1], da[mt], kb[2], kb[3]);
        }
      }
      // TW: the queries' activation, their Gram matrix with the keys' over this warp's hidden
      // slice, gw[nt][e] = G[g + 8(e>>1)][8nt + 2q + (e&1)] with G = A_q·Aᵀ, and its Mᵀ-style B
      // fragments (masked to s ≤ t, hi and lo).
      uint32_t gbh[2][2], gbl[2][2];
      uint32_t bq[2][2][2];  // the queries' Aᵀ B fragments: [token n-tile][hidden k-step][half]
      if (HAS_Q && TW) {
        uint32_t bk[2][2][2];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            float yq[4], dq;
#pragma unroll
            for (int e = 0; e < 4; ++e) gelu_and_grad(hq[mt][nt][e], yq[e], dq);
            aq[mt][nt][0] = pack_bf16(yq[0], yq[1]);
            aq[mt][nt][1] = pack_bf16(yq[2], yq[3]);
          }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              bq[nt][ks][hh] = movm_t(aq[ks][nt][hh]);
              bk[nt][ks][hh] = movm_t(ak[ks][nt][hh]);
            }
        float gw[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const uint32_t a[4] = {bq[0][ks][0], bq[1][ks][0], bq[0][ks][1], bq[1][ks][1]};  // A_q rows t
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) mma_bf16(gw[nt], a, bk[nt][ks][0], bk[nt][ks][1]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 8 * nt + g;
          const float g00 = 2 * q <= t ? gw[0][2 * nt] : 0.f, g01 = 2 * q + 1 <= t ? gw[0][2 * nt + 1] : 0.f;
          const float g10 = 2 * q + 8 <= t ? gw[1][2 * nt] : 0.f, g11 = 2 * q + 9 <= t ? gw[1][2 * nt + 1] : 0.f;
          hilo2(g00, g01, gbh[nt][0], gbl[nt][0]);
          hilo2(g10, g11, gbh[nt][1], gbl[nt][1]);
        }
      }
      // W2ᵀ += Sᵀ·A: Sᵀ as the A operand (columns x tokens), A (tokens x hidden) as B. With TW,
      // each feature tile first gives the queries' partial Zᵀ from the W2 it holds before the
      // update: W2ᵀ·Aqᵀ + Sᵀ·Gᵀ.
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t sa[2][4];
#pragma unroll
        for (int p = 0; p < 2; ++p) ldsm4_t(sbase[p] + swz128_bf16(8 * (mi >> 1) + ri, 16 * mt + 8 * (mi & 1)), sa[p]);
        if (HAS_Q && TW) {
          uint32_t whi[2][4], wlo[2][4];
          afrag_hilo(a2[mt][0], a2[mt][1], whi[0], wlo[0]);
          afrag_hilo(a2[mt][2], a2[mt][3], whi[1], wlo[1]);
          float* red = &sm.red[1][warp][0][0];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            float zp[4] = {0.f, 0.f, 0.f, 0.f}, z2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              mma_bf16(zp, whi[ks], bq[nt][ks][0], bq[nt][ks][1]);
              mma_bf16(z2, wlo[ks], bq[nt][ks][0], bq[nt][ks][1]);
            }
            mma_bf16(zp, sa[0], gbh[nt][0], gbh[nt][1]);
            mma_bf16(z2, sa[0], gbl[nt][0], gbl[nt][1]);
            mma_bf16(z2, sa[1], gbh[nt][0], gbh[nt][1]);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              red[(8 * nt + 2 * q + (e & 1)) * kRedStride + 16 * mt + g + 8 * (e >> 1)] = zp[e] + z2[e];
          }
        }
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int j = 0; j < 4; ++j) mma_bf16(a2[mt][j], sa[p], ak[j >> 1][0][j & 1], ak[j >> 1][1][j & 1]);
      }
      if (HAS_Q && TW) {
        compute_sync<kMlpWarps>();
        query_outputs();
      }
    }
    // End of the tile: its outputs are complete in shared memory and every warp is done with
    // its inputs, so the slot takes tile s + kStagesM.
    if (HAS_Q) fence_proxy_async_smem();
    compute_sync<kMlpWarps>();
    if (threadIdx.x == 0) {
      if (HAS_Q) {
        tma_store_3d(&tmO, obuf, 0, s * kTileTokI, bh);
        bulk_commit();
      }
      if (issued < ntiles) issue(issued++);
      if (HAS_Q) bulk_wait_read<1>();  // the other staging tile is free again
    }
  }
  if (threadIdx.x == 0) {
    if (HAS_Q) bulk_wait<0>();
    // Nothing may still be landing in shared memory when the CTA exits (after an abort the
    // tiles issued past the last one consumed).
    for (int t = s; t < issued; ++t)
      if (t != a.stall_tile) mbar_wait(&sm.full[t % kStagesM], (t / kStagesM) & 1, a.status, nullptr);
  }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        W1g[(8 * nt + 2 * q + (e & 1)) * kHid + hid0 + 16 * mt + g + 8 * (e >> 1)] = a1[mt][nt][e];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        W2g[(hid0 + 8 * nt + 2 * q + (e & 1)) * 64 + 16 * mt + g + 8 * (e >> 1)] = a2[mt][nt][e];
  __syncthreads();
}

template <bool HAS_Q, bool LOSS, bool TW>
ttt_status launch_inner(ttt_state* st, const CUtensorMap* maps, float* loss, int T, const int2* steps,
                        cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const bool mlp = c.rule == TTT_RULE_MLP_GD, ln = c.rule == TTT_RULE_LINEAR_LN_GD;
  const size_t smem = (mlp ? sizeof(MlpSmem) : sizeof(LnSmem)) + 1024;
  // One bit per instantiation whose shared-memory limit has been raised on this state's device.
  const uint64_t bit = 1ull << (40 + 8 * (mlp ? 2 : ln ? 1 : 0) + 4 * TW + 2 * HAS_Q + LOSS);
  auto kernel = mlp ? k_inner_mlp<HAS_Q, LOSS, TW> : ln ? k_inner_ln<HAS_Q, LOSS, TW, true> : k_inner_ln<HAS_Q, LOSS, TW, false>;
  if (!(st->lin.smem_set & bit)) {
    TTT_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    st->lin.smem_set |= bit;
  }
  const int grid = c.batch * c.heads;
  // Fault injection (tests): the second 64-token tile is never loaded, so the waits for it run out.
  int stall_tile = -1;
  if (st->inject_stall && T > kTileTokI) {
    stall_tile = 1;
    st->inject_stall = 0;
  }
  InnerArgs a{st->lin.W, st->lin.W0, st->lin.ln_gamma, st->lin.ln_beta, loss, steps, T, c.heads, T / kMB,
              c.eta, c.ln_eps, DevStatus{st->status.dev, st->wait_limit_ns, st->status.dev + 1}, stall_tile};
  kernel<<<grid, mlp ? kMlpThreads : kLnThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], a);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace

// One launch over [B·H, T, 64] buffers (T a multiple of 16 when steps is set).
static ttt_status inner_launch(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                               int64_t T, __nv_bfloat16* O, float* loss, const int2* steps, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  // [B·H, T, 64] bf16 views of K, V, Q and O, 64-token boxes with the 128-byte swizzle; the maps
  // of the last few buffer sets are kept (encoding costs microseconds of host time).
  const uint64_t dims[3] = {64, (uint64_t)T, (uint64_t)c.batch * c.heads};
  const uint64_t strides[2] = {128, (uint64_t)T * 128};
  const uint32_t box[3] = {64, (uint32_t)kTileTokI, 1};
  LinearBuffers& lb = st->lin;
  const bool has_q = Q != nullptr;
  const void* key[4] = {K, V, Q, O};
  LinearMapSet* ms = nullptr;
  for (LinearMapSet& m : lb.map_sets)
    if (m.T == T && m.key[0] == key[0] && m.key[1] == key[1] && m.key[2] == key[2] && m.key[3] == key[3]) ms = &m;
  if (ms == nullptr) {
    ms = &lb.map_sets[0];
    for (LinearMapSet& m : lb.map_sets)
      if (m.last_use < ms->last_use) ms = &m;
    ms->T = -1;  // invalid until all four are encoded
    for (int i = 0; i < 4; ++i) {
      const void* base = key[i] != nullptr ? key[i] : key[0];
      TTT_TRY(encode_tmap(&ms->maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_128B));
      ms->key[i] = key[i];
    }
    ms->T = T;
  }
  ms->last_use = ++lb.map_clock;
  // Per-token weights change only the outputs.
  if (has_q && c.token_weights)
    return loss ? launch_inner<true, true, true>(st, ms->maps, loss, (int)T, steps, s)
                : launch_inner<true, false, true>(st, ms->maps, loss, (int)T, steps, s);
  if (has_q)
    return loss ? launch_inner<true, true, false>(st, ms->maps, loss, (int)T, steps, s)
                : launch_inner<true, false, false>(st, ms->maps, loss, (int)T, steps, s);
  return loss ? launch_inner<false, true, false>(st, ms->maps, loss, (int)T, steps, s)
              : launch_inner<false, false, false>(st, ms->maps, loss, (int)T, steps, s);
}

ttt_status inner_scan(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                      int64_t T, __nv_bfloat16* O, float* loss, cudaStream_t s) {
  return inner_launch(st, K, V, Q, T, O, loss, nullptr, s);
}

namespace {

// Row r of the padded [B·H, Tp, 64] layout takes input row rows[b·Tp + t] of its (sequence, head)
// (zero where that is -1). One thread a 16-byte vector.
__global__ void k_gather_heads(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               const int32_t* __restrict__ rows, int H, int T, int Tp, long long nrows) {
  const long long n = nrows * 8;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i >> 3;
    const int c = (int)(i & 7);
    const long long bh = r / Tp;
    const int tp = (int)(r % Tp);
    const int32_t from = rows[(bh / H) * Tp + tp];
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (from >= 0) x = reinterpret_cast<const uint4*>(src + (bh * T + from) * 64)[c];
    reinterpret_cast<uint4*>(dst + r * 64)[c] = x;
  }
}

// The inverse for the outputs (bf16 rows) and the losses (one float a row); padding rows are
// dropped.
__global__ void k_scatter_heads(const __nv_bfloat16* __restrict__ srcO, __nv_bfloat16* __restrict__ dstO,
                                const float* __restrict__ srcL, float* __restrict__ dstL,
                                const int32_t* __restrict__ rows, int H, int T, int Tp, long long nrows) {
  const long long n = nrows * 8;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i >> 3;
    const int c = (int)(i & 7);
    const long long bh = r / Tp;
    const int tp = (int)(r % Tp);
    const int32_t to = rows[(bh / H) * Tp + tp];
    if (to < 0) continue;
    if (srcO != nullptr) reinterpret_cast<uint4*>(dstO + (bh * T + to) * 64)[c] = reinterpret_cast<const uint4*>(srcO + r * 64)[c];
    if (srcL != nullptr && c == 0) dstL[bh * T + to] = srcL[r];
  }
}

int grid_for(long long n) {
  const long long b = (n + 255) / 256;
  return (int)(b < 148 * 16 ? (b < 1 ? 1 : b) : 148 * 16);
}

}  // namespace

void free_packed(ttt_state* st) {
  LinearBuffers& lb = st->lin;
  for (auto*& p : lb.pk) {
    if (p != nullptr) cudaFree(p);
    p = nullptr;
  }
  if (lb.pk_loss != nullptr) cudaFree(lb.pk_loss);
  if (lb.pk_rows != nullptr) cudaFree(lb.pk_rows);
  if (lb.pk_steps != nullptr) cudaFree(lb.pk_steps);
  lb.pk_loss = nullptr;
  lb.pk_rows = nullptr;
  lb.pk_steps = nullptr;
  lb.pk_cap = lb.pk_map_cap = 0;
}

ttt_status inner_scan_packed(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                             int64_t T, __nv_bfloat16* O, float* loss, const int64_t* doc_starts,
                             const int32_t* docs_per_seq, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const int B = c.batch, H = c.heads;
  // Layout: every document padded to whole mini-batches; the sequences padded to the longest.
  std::vector<int64_t> padded(B, 0);
  int64_t off = 0;
  for (int b = 0; b < B; ++b) {
    for (int k = 0; k < docs_per_seq[b]; ++k) {
      const int64_t a = doc_starts[off + k], e = k + 1 < docs_per_seq[b] ? doc_starts[off + k + 1] : T;
      padded[b] += (e - a + kMB - 1) / kMB * kMB;
    }
    off += docs_per_seq[b];
  }
  int64_t Tp = kMB;
  for (int64_t p : padded) Tp = std::max(Tp, p);
  if (Tp > (int64_t)INT32_MAX / 4) return fail(TTT_ERR_UNSUPPORTED, "packed layout too long");
  const int64_t nsteps = Tp / kMB;
  std::vector<int32_t> rows((size_t)(B * Tp), -1);
  std::vector<int2> steps((size_t)(B * nsteps), make_int2(0, 0));
  off = 0;
  for (int b = 0; b < B; ++b) {
    int64_t p = 0;
    for (int k = 0; k < docs_per_seq[b]; ++k) {
      const int64_t a = doc_starts[off + k], e = k + 1 < docs_per_seq[b] ? doc_starts[off + k + 1] : T;
      for (int64_t t0 = a; t0 < e; t0 += kMB, p += kMB) {
        const int n = (int)std::min<int64_t>(kMB, e - t0);
        steps[(size_t)(b * nsteps + p / kMB)] = make_int2(t0 == a ? 1 : 0, n);
        for (int j = 0; j < n; ++j) rows[(size_t)(b * Tp + p + j)] = (int32_t)(t0 + j);
      }
    }
    off += docs_per_seq[b];
  }
  // Scratch, grown on demand.
  LinearBuffers& lb = st->lin;
  const int64_t nrows = (int64_t)B * H * Tp;
  if (nrows > lb.pk_cap || B * Tp > lb.pk_map_cap) {
    free_packed(st);
    const size_t rb = (size_t)nrows * 128;
    for (auto*& p : lb.pk) TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&p), rb));
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&lb.pk_loss), (size_t)nrows * 4));
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&lb.pk_rows), (size_t)(B * Tp) * 4));
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&lb.pk_steps), (size_t)(B * nsteps) * sizeof(int2)));
    lb.pk_cap = nrows;
    lb.pk_map_cap = B * Tp;
  }
  TTT_CUDA(cudaMemcpyAsync(lb.pk_rows, rows.data(), rows.size() * 4, cudaMemcpyHostToDevice, s));
  TTT_CUDA(cudaMemcpyAsync(lb.pk_steps, steps.data(), steps.size() * sizeof(int2), cudaMemcpyHostToDevice, s));
  const int gb = grid_for(nrows * 8);
  k_gather_heads<<<gb, 256, 0, s>>>(K, lb.pk[0], lb.pk_rows, H, (int)T, (int)Tp, nrows);
  k_gather_heads<<<gb, 256, 0, s>>>(V, lb.pk[1], lb.pk_rows, H, (int)T, (int)Tp, nrows);
  st->launches += 2;
  if (Q != nullptr) {
    k_gather_heads<<<gb, 256, 0, s>>>(Q, lb.pk[2], lb.pk_rows, H, (int)T, (int)Tp, nrows);
    st->launches++;
  }
  TTT_CUDA(cudaGetLastError());
  TTT_TRY(inner_launch(st, lb.pk[0], lb.pk[1], Q != nullptr ? lb.pk[2] : nullptr, Tp, Q != nullptr ? lb.pk[3] : nullptr,
                       loss != nullptr ? lb.pk_loss : nullptr, lb.pk_steps, s));
  if (O != nullptr || loss != nullptr) {
    k_scatter_heads<<<gb, 256, 0, s>>>(O != nullptr ? lb.pk[3] : nullptr, O, loss != nullptr ? lb.pk_loss : nullptr, loss,
                                       lb.pk_rows, H, (int)T, (int)Tp, nrows);
    st->launches++;
    TTT_CUDA(cudaGetLastError());
  }
  return TTT_OK;
}

}  // namespace ttt
