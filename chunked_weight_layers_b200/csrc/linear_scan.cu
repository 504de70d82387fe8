// TTT-Linear mini-batch gradient scan ("テスト時学習（Test-Time Training）とは", the TTT layers
// page: the hidden state is the weight W of a linear model and each update is one
// self-supervised gradient step). Per (sequence, head) and inner mini-batch i of b tokens:
//   O_i = Q_i·W_i,   R_i = K_i·W_i − V_i,   L_t = ‖R_i[t]‖²,   W_{i+1} = W_i − (η/b)·K_iᵀ·R_i.
//
// Design (B200):
//  * the per-head state is 64x64 fp32 and never leaves the SM: it lives in mma accumulator
//    registers. Column c of W only ever depends on column c of R (R[:, c] = K·W[:, c] − V[:, c]),
//    so columns are split across warps with no communication inside a step.
//  * k_linear_b16 (b = 16, one CTA per head): four compute warps own sixteen columns each and
//    compute every product transposed, so each accumulator layout is directly the next mma's A
//    operand. Operand fragments are loaded one step ahead; a 64-token tile is four
//    straight-line steps with all waits at its top. A TMA producer warp fills the K/V/Q ring
//    and a writer warp sums loss partials and stores the output tiles, so compute warps never
//    meet at a barrier. Measured on B200 it is faster than splitting a head's columns over two
//    CTAs (eight columns per warp, movmatrix for the B operands) even when SMs are idle: 104
//    against 173 us for B=4 x H=16 x T=8192, 32 against 41 us for a single head.
//  * k_linear_scan (b = 32 or 64): one CTA per head, sixteen columns per warp, W and the update
//    operand fed to the tensor cores as bf16 hi + lo pairs.
//  * for b = 16 the tensor cores see W rounded to bf16 each step and the update operand
//    −(η/b)·R rounded to bf16; W itself and every accumulation stay fp32.
//  * K, V, Q stream through a 4-stage ring of 64-token tiles loaded by TMA (128-byte swizzle,
//    3-D maps over [B·H, T, 64] so a head's last tile is clipped to its own T); outputs are
//    staged in swizzled smem and written by TMA stores. Compute warps wait on a full slot for
//    under 6% of the scan, and an 8-stage ring measured no faster.
//  * the chain per step is latency-bound and tiny (393 kFLOP per head), so it runs on the
//    warp-level mma.sync path: a tcgen05 round trip (issue, commit, mbarrier, tcgen05.ld) per
//    dependent 16x64x64 product costs more than the product itself. Measured on B200:
//    mma.sync m16n8k16 latency ~21 cycles, at most one per ~8.2 cycles per SM sub-partition.
#include "common.cuh"
#include "gate_chunk.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int kStages = 4;        // ring depth (64-token tiles): 96 KB of K/V/Q in flight per SM
constexpr int kTileTok = 64;      // tokens per tile
constexpr int kTileBytes = kTileTok * 128;  // 64 tokens x 64 bf16
constexpr int kComputeWarps = 4;
constexpr int kLossStride = 68;   // floats per row of loss partials (64 tokens + 4: no bank conflicts)
constexpr int kThreads = (kComputeWarps + 1) * 32;

struct __align__(1024) LinearSmem {
  uint8_t K[kStages][kTileBytes];
  uint8_t V[kStages][kTileBytes];
  uint8_t Q[kStages][kTileBytes];
  uint8_t O[2][kTileBytes];
  float lossp[kComputeWarps][kTileTok];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort;       // set by the producer when one of its waits ran out
  int cabort[2];   // set by a compute warp whose wait for tile s ran out (index s & 1)
  int consumed;
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32)); }

// Split two fp32 values into packed bf16 hi and lo words (x ≈ hi + lo to ~2^-17 relative).
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = pack_bf16(x - hf.x, y - hf.y);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
}

// Per-lane shared-memory offsets of the fragments one 16-token step reads or writes. With
// the 128-byte swizzle the XOR pattern depends only on the row's low three bits, so an
// offset computed for rows 0..15 holds for any step starting at a multiple of 16 rows:
// the step adds r0·128.
struct StepOffsets {
  uint32_t kb[2][2];  // Kᵀ (and Qᵀ) B fragments of the product with W: [token n-tile][key pair]
  uint32_t kt[4];     // K B fragments of the update: key n-tile pairs
  uint32_t v;         // −Vᵀ accumulator init for this warp's 16 columns
  uint32_t o;         // output tile rows for stmatrix
};

__device__ __forceinline__ StepOffsets step_offsets(int lane, int col0) {
  const int mi = lane >> 3, ri = lane & 7;
  StepOffsets f;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) f.kb[nt][kp] = swz128_bf16(8 * nt + ri, 32 * kp + 8 * mi);
#pragma unroll
  for (int np = 0; np < 4; ++np) f.kt[np] = swz128_bf16(8 * (mi & 1) + ri, 16 * np + 8 * (mi >> 1));
  f.v = swz128_bf16(8 * (mi >> 1) + ri, col0 + 8 * (mi & 1));
  f.o = swz128_bf16(8 * (mi >> 1) + ri, col0 + 8 * (mi & 1));
  return f;
}

__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}

// Operand fragments of one 16-token inner mini-batch (tile rows r0 .. r0+15) for the warp
// owning W columns [col0, col0+16). They are loaded one step ahead: while a step's dependent
// chain runs, the shared-memory reads of the next step are already in flight.
struct Frag16 {
  uint32_t kb[2][2][4];  // Kᵀ B fragments of the product with W: [token n-tile][key pair]
  uint32_t kt[4][4];     // K B fragments of the update: [key n-tile pair]
  uint32_t vf[4];        // Vᵀ of this warp's columns
  uint32_t qb[2][2][4];  // Qᵀ B fragments of the outputs
};

template <bool HAS_Q>
__device__ __forceinline__ void load_frag16(Frag16& F, uint32_t kbase, uint32_t vbase, uint32_t qbase,
                                            const StepOffsets& f, int r0) {
  const uint32_t rofs = (uint32_t)r0 * 128u;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) ldsm_x4(kbase + rofs + f.kb[nt][kp], F.kb[nt][kp]);
  ldsm_x4_t(vbase + rofs + f.v, F.vf);
#pragma unroll
  for (int np = 0; np < 4; ++np) ldsm_x4_t(kbase + rofs + f.kt[np], F.kt[np]);
  if (HAS_Q) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) ldsm_x4(qbase + rofs + f.kb[nt][kp], F.qb[nt][kp]);
  }
}

// One inner mini-batch from loaded fragments, everything transposed so that each accumulator
// layout is directly the next mma's A operand:
//   Pᵀ = Wᵀ·Kᵀ,  Rᵀ = Pᵀ − Vᵀ,  Wᵀ += Sᵀ·K with S = −(η/b)·R,  Oᵀ = Wᵀ_old·Qᵀ.
// The tensor cores see W and S rounded to bf16; W and every accumulation stay fp32. The
// output products are issued after the update so they do not delay the dependent chain.
template <bool HAS_Q, bool LOSS>
__device__ __forceinline__ void compute16(float (&acc)[8][4], const Frag16& F, uint32_t obase, uint32_t ofs_o,
                                          float* lossp, int r0, int lane, float beta) {
  const int g = lane >> 2, q = lane & 3;
  uint32_t wa[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    wa[ks][0] = pack_bf16(acc[2 * ks][0], acc[2 * ks][1]);
    wa[ks][1] = pack_bf16(acc[2 * ks][2], acc[2 * ks][3]);
    wa[ks][2] = pack_bf16(acc[2 * ks + 1][0], acc[2 * ks + 1][1]);
    wa[ks][3] = pack_bf16(acc[2 * ks + 1][2], acc[2 * ks + 1][3]);
  }
  // Two partial sums per token n-tile (keys 0-15 + 32-47 and 16-31 + 48-63) halve the chain.
  float pp[2][2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) pp[nt][0][e] = pp[nt][1][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
      mma16816(pp[nt][ks & 1], wa[ks], F.kb[nt][ks >> 1][2 * (ks & 1)], F.kb[nt][ks >> 1][2 * (ks & 1) + 1]);
  // The first half of the output products goes into the P products' latency; the second half
  // follows the update, into its latency (both halves are off the dependent chain).
  float o[2][2][4];
  if (HAS_Q) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][0][e] = o[nt][1][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        mma16816(o[nt][ks & 1], wa[ks], F.qb[nt][ks >> 1][2 * (ks & 1)], F.qb[nt][ks >> 1][2 * (ks & 1) + 1]);
  }

  // R = P − V: p[nt][e] is R[token 8nt + 2q + (e&1)][column col0 + g + 8(e>>1)].
  float p[2][4];
  {
    const float2 v0 = unpack_bf16(F.vf[0]), v1 = unpack_bf16(F.vf[1]), v2 = unpack_bf16(F.vf[2]),
                 v3 = unpack_bf16(F.vf[3]);
    const float vv[2][4] = {{v0.x, v0.y, v1.x, v1.y}, {v2.x, v2.y, v3.x, v3.y}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) p[nt][e] = (pp[nt][0][e] + pp[nt][1][e]) - vv[nt][e];
  }
  uint32_t sa[4];
  sa[0] = pack_bf16(-beta * p[0][0], -beta * p[0][1]);
  sa[1] = pack_bf16(-beta * p[0][2], -beta * p[0][3]);
  sa[2] = pack_bf16(-beta * p[1][0], -beta * p[1][1]);
  sa[3] = pack_bf16(-beta * p[1][2], -beta * p[1][3]);
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    mma16816(acc[2 * np], sa, F.kt[np][0], F.kt[np][1]);
    mma16816(acc[2 * np + 1], sa, F.kt[np][2], F.kt[np][3]);
  }

  if (HAS_Q) {
#pragma unroll
    for (int ks = 2; ks < 4; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        mma16816(o[nt][ks & 1], wa[ks], F.qb[nt][ks >> 1][2 * (ks & 1)], F.qb[nt][ks >> 1][2 * (ks & 1) + 1]);
    stsm_x4_t(obase + (uint32_t)r0 * 128u + ofs_o, pack_bf16(o[0][0][0] + o[0][1][0], o[0][0][1] + o[0][1][1]),
              pack_bf16(o[0][0][2] + o[0][1][2], o[0][0][3] + o[0][1][3]),
              pack_bf16(o[1][0][0] + o[1][1][0], o[1][0][1] + o[1][1][1]),
              pack_bf16(o[1][0][2] + o[1][1][2], o[1][0][3] + o[1][1][3]));
  }
  if (LOSS) {
    // Squared residuals of this lane's two columns; the writer warp sums the 32 partials of a
    // token (eight lane groups, four warps), so no reduction sits on the chain.
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float l0 = p[nt][0] * p[nt][0] + p[nt][2] * p[nt][2];
      const float l1 = p[nt][1] * p[nt][1] + p[nt][3] * p[nt][3];
      *reinterpret_cast<float2*>(&lossp[g * kLossStride + r0 + 8 * nt + 2 * q]) = make_float2(l0, l1);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Chunked form of the b = 16 scan. A chunk holds NB inner mini-batches (16-token blocks
// i = 0 .. NB−1) and starts from weight W. Unrolling the steps inside the chunk,
//   W_i = W − β·Σ_{j<i} K_jᵀR_j,   so
//   R_i = K_i·W − V_i − β·Σ_{j<i} (K_i·K_jᵀ)·R_j,
//   O_i = Q_i·W     − β·Σ_{j<i} (Q_i·K_jᵀ)·R_j,
//   W_next = W − β·Σ_i K_iᵀR_i.
// This is the same arithmetic as NB sequential steps, regrouped: every product with W uses the
// weight from the chunk's start, so the NB products P_i = K_i·W are independent and issue back
// to back; what stays sequential is the short correction of each block by the residuals of
// the blocks before it (a 16x16x16 product per pair and warp). The Gram blocks G_ij = K_i·K_jᵀ
// and M_ij = Q_i·K_jᵀ do not depend on W: the four compute warps share them out one tile
// ahead (each computes a quarter into shared memory while it runs the tile before).
// ---------------------------------------------------------------------------------------------

// Chunked form: the Gram blocks K_i·K_jᵀ (and Q_i·K_jᵀ) of the block pairs i > j of every chunk
// of a tile, bf16, each 16x16 block as four 8x8 tiles of 128 bytes ([i half][j half]).
constexpr int kMaxTilePairs = 6;   // a 64-token chunk of four 16-token blocks has six pairs
constexpr int kPairBytes = 1024;   // G block then M block

// Slot of pair (i, j), i > j, among a chunk's pairs: (1,0) (2,0) (2,1) (3,0) (3,1) (3,2).
__host__ __device__ constexpr int pair_slot(int i, int j) { return i * (i - 1) / 2 + j; }

// Per-lane offset of the x4 ldmatrix / stmatrix that reads or writes a Gram block (four 8x8
// tiles of 128 bytes: [i 0-7, j 0-7], [i 0-7, j 8-15], [i 8-15, j 0-7], [i 8-15, j 8-15]).
__device__ __forceinline__ uint32_t gram_lane_ofs(int lane) { return (uint32_t)(lane >> 3) * 128u + (uint32_t)(lane & 7) * 16u; }

// One Gram unit: columns 8nt .. 8nt+7 (tokens of block bj) of X_bi·K_bjᵀ, for X = K (into the G
// block of slot `dst`) and, with queries, X = Q (into its M block). Rows come from a tile in the
// ring (128-byte swizzle), blocks bi, bj counted in 16-token rows of the tile. Every fragment is
// loaded before the first mma so the loads' latencies overlap.
template <bool HAS_Q>
__device__ __forceinline__ void gram_unit(uint32_t kbase, uint32_t qbase, int bi, int bj, int nt, uint32_t dst,
                                          const StepOffsets& f, int lane) {
  constexpr int NX = HAS_Q ? 2 : 1;
  // B fragments of K_bjᵀ for this n-tile: dk 32kp .. 32kp+31.
  uint32_t kb[2][4];
#pragma unroll
  for (int kp = 0; kp < 2; ++kp) ldsm_x4(kbase + (uint32_t)(16 * bj) * 128u + f.kb[nt][kp], kb[kp]);
  const int arow = (lane & 7) + 8 * ((lane >> 3) & 1);
  uint32_t a[NX][4][4];
#pragma unroll
  for (int x = 0; x < NX; ++x)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      ldsm_x4((x == 0 ? kbase : qbase) + (uint32_t)(16 * bi) * 128u + swz128_bf16(arow, 16 * ks + 8 * (lane >> 4)),
              a[x][ks]);
  float c[NX][2][4];
#pragma unroll
  for (int x = 0; x < NX; ++x)
#pragma unroll
    for (int e = 0; e < 4; ++e) c[x][0][e] = c[x][1][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int x = 0; x < NX; ++x)
      mma16816(c[x][ks & 1], a[x][ks], kb[ks >> 1][2 * (ks & 1)], kb[ks >> 1][2 * (ks & 1) + 1]);
#pragma unroll
  for (int x = 0; x < NX; ++x) {
    // stmatrix x2: matrix 0 = rows i 0-7 (tile nt), matrix 1 = rows i 8-15 (tile 2 + nt).
    const uint32_t addr = dst + (uint32_t)x * 512u + (uint32_t)((lane >> 3) & 1) * 256u + (uint32_t)nt * 128u +
                          (uint32_t)(lane & 7) * 16u;
    const uint32_t r0 = pack_bf16(c[x][0][0] + c[x][1][0], c[x][0][1] + c[x][1][1]);
    const uint32_t r1 = pack_bf16(c[x][0][2] + c[x][1][2], c[x][0][3] + c[x][1][3]);
    asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(addr), "r"(r0), "r"(r1) : "memory");
  }
}

// This warp's share of the Gram blocks of one tile (all its chunks of NB blocks).
template <int NB, bool HAS_Q>
__device__ __forceinline__ void gram_tile(uint32_t kbase, uint32_t qbase, uint32_t gmbase, const StepOffsets& f,
                                          int warp, int lane) {
  constexpr int kPPC = NB * (NB - 1) / 2;   // pairs per chunk
  constexpr int kUnits = (64 / (16 * NB)) * kPPC * 2;  // (pair, n-tile) units per tile
#pragma unroll
  for (int u0 = 0; u0 < kUnits; u0 += kComputeWarps) {
    const int u = u0 + warp;
    if (kUnits % kComputeWarps != 0 && u >= kUnits) break;
    const int p = u >> 1, nt = u & 1;
    const int cc = p / kPPC, loc = p % kPPC;
    // loc = i(i−1)/2 + j
    const int i = loc < 1 ? 1 : (loc < 3 ? 2 : 3);
    const int j = loc - pair_slot(i, 0);
    gram_unit<HAS_Q>(kbase, qbase, cc * NB + i, cc * NB + j, nt, gmbase + (uint32_t)p * kPairBytes, f, lane);
  }
}

// Fragments one block of a chunk needs after its product with W: Vᵀ of this warp's columns,
// the K operand of the update, the Qᵀ operand of the outputs, the Gram blocks G(i2, i) that
// carry its residuals into the later blocks i2 and the M(i, j) that carry the earlier blocks'
// residuals into its outputs.
template <int NBLK, bool HAS_Q>
struct BlkFrag {
  uint32_t vf[4];
  uint32_t kt[4][4];
  uint32_t qb[2][2][4];
  uint32_t g[NBLK > 1 ? NBLK - 1 : 1][4];
  uint32_t m[NBLK > 1 ? NBLK - 1 : 1][4];
};

template <int NBLK, bool HAS_Q>
__device__ __forceinline__ void load_blk(BlkFrag<NBLK, HAS_Q>& B, int i, uint32_t kbase, uint32_t vbase, uint32_t qbase,
                                         uint32_t gbase, const StepOffsets& f, uint32_t gl, int r0) {
  const uint32_t rofs = (uint32_t)(r0 + 16 * i) * 128u;
  ldsm_x4_t(vbase + rofs + f.v, B.vf);
#pragma unroll
  for (int i2 = i + 1; i2 < NBLK; ++i2) ldsm_x4(gbase + (uint32_t)pair_slot(i2, i) * kPairBytes + gl, B.g[i2 - i - 1]);
#pragma unroll
  for (int np = 0; np < 4; ++np) ldsm_x4_t(kbase + rofs + f.kt[np], B.kt[np]);
  if (HAS_Q) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) ldsm_x4(qbase + rofs + f.kb[nt][kp], B.qb[nt][kp]);
#pragma unroll
    for (int j = 0; j < i; ++j) ldsm_x4(gbase + (uint32_t)pair_slot(i, j) * kPairBytes + 512u + gl, B.m[j]);
  }
}

__device__ __forceinline__ void load_kb(uint32_t (&kb)[2][2][4], uint32_t rb, const StepOffsets& f) {
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) ldsm_x4(rb + f.kb[nt][kp], kb[nt][kp]);
}

// One chunk of NBLK blocks (tile rows r0 .. r0 + 16·NBLK − 1) for the warp owning W columns
// [col0, col0+16). `gbase` is the chunk's first pair slot. Everything transposed as in compute16:
// Pᵀ_i = Wᵀ·K_iᵀ, Rᵀ_i = Pᵀ_i − V_iᵀ + Σ_{j<i} Sᵀ_j·G_ijᵀ with S = −β·R (bf16), Wᵀ += Σ_i Sᵀ_i·K_i,
// Oᵀ_i = Wᵀ·Qᵀ_i + Σ_{j<i} Sᵀ_j·M_ijᵀ. The tensor cores see W, S and the Gram blocks rounded to bf16;
// W and every accumulation stay fp32.
// Loads and mma keep their program order (both are volatile), so every fragment is loaded one
// phase before its first use: the Kᵀ operand of block i+1 while the products of block i issue,
// block 0's remaining fragments while the last product with W issues, and block i+1's while
// block i's outputs issue.
template <int NBLK, bool HAS_Q, bool LOSS>
__device__ __forceinline__ void chunk_run(float (&acc)[8][4], uint32_t kbase, uint32_t vbase, uint32_t qbase,
                                          uint32_t gbase, uint32_t obase, const StepOffsets& f, float* lossp,
                                          int r0, int lane, float beta) {
  const int g = lane >> 2, q = lane & 3;
  const uint32_t gl = gram_lane_ofs(lane);
  uint32_t kbuf[2][2][2][4];
  load_kb(kbuf[0], kbase + (uint32_t)r0 * 128u, f);
  uint32_t wa[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    wa[ks][0] = pack_bf16(acc[2 * ks][0], acc[2 * ks][1]);
    wa[ks][1] = pack_bf16(acc[2 * ks][2], acc[2 * ks][3]);
    wa[ks][2] = pack_bf16(acc[2 * ks + 1][0], acc[2 * ks + 1][1]);
    wa[ks][3] = pack_bf16(acc[2 * ks + 1][2], acc[2 * ks + 1][3]);
  }
  // P_i for every block of the chunk, two partial sums per token n-tile.
  float pp[NBLK][2][2][4];
  BlkFrag<NBLK, HAS_Q> F[2];
#pragma unroll
  for (int i = 0; i < NBLK; ++i) {
    if (i + 1 < NBLK) load_kb(kbuf[(i + 1) & 1], kbase + (uint32_t)(r0 + 16 * (i + 1)) * 128u, f);
    else load_blk<NBLK, HAS_Q>(F[0], 0, kbase, vbase, qbase, gbase, f, gl, r0);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) pp[i][nt][0][e] = pp[i][nt][1][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        mma16816(pp[i][nt][ks & 1], wa[ks], kbuf[i & 1][nt][ks >> 1][2 * (ks & 1)],
                 kbuf[i & 1][nt][ks >> 1][2 * (ks & 1) + 1]);
  }

  uint32_t sa[NBLK][4];
#pragma unroll
  for (int i = 0; i < NBLK; ++i) {
    BlkFrag<NBLK, HAS_Q>& B = F[i & 1];
    // R_i = P_i − V_i (+ the corrections already accumulated into pp[i][.][0]).
    const float2 v0 = unpack_bf16(B.vf[0]), v1 = unpack_bf16(B.vf[1]), v2 = unpack_bf16(B.vf[2]),
                 v3 = unpack_bf16(B.vf[3]);
    const float vv[2][4] = {{v0.x, v0.y, v1.x, v1.y}, {v2.x, v2.y, v3.x, v3.y}};
    float p[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) p[nt][e] = (pp[i][nt][0][e] + pp[i][nt][1][e]) - vv[nt][e];
    sa[i][0] = pack_bf16(-beta * p[0][0], -beta * p[0][1]);
    sa[i][1] = pack_bf16(-beta * p[0][2], -beta * p[0][3]);
    sa[i][2] = pack_bf16(-beta * p[1][0], -beta * p[1][1]);
    sa[i][3] = pack_bf16(-beta * p[1][2], -beta * p[1][3]);
    // Corrections of the later blocks by this block's residuals (the chain's critical step).
#pragma unroll
    for (int i2 = i + 1; i2 < NBLK; ++i2) {
      mma16816(pp[i2][0][0], sa[i], B.g[i2 - i - 1][0], B.g[i2 - i - 1][1]);
      mma16816(pp[i2][1][0], sa[i], B.g[i2 - i - 1][2], B.g[i2 - i - 1][3]);
    }
    // Wᵀ += Sᵀ_i·K_i.
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      mma16816(acc[2 * np], sa[i], B.kt[np][0], B.kt[np][1]);
      mma16816(acc[2 * np + 1], sa[i], B.kt[np][2], B.kt[np][3]);
    }
    if (i + 1 < NBLK) load_blk<NBLK, HAS_Q>(F[(i + 1) & 1], i + 1, kbase, vbase, qbase, gbase, f, gl, r0);
    if (LOSS) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float l0 = p[nt][0] * p[nt][0] + p[nt][2] * p[nt][2];
        const float l1 = p[nt][1] * p[nt][1] + p[nt][3] * p[nt][3];
        *reinterpret_cast<float2*>(&lossp[g * kLossStride + r0 + 16 * i + 8 * nt + 2 * q]) = make_float2(l0, l1);
      }
    }
    if (HAS_Q) {
      float o[2][2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][0][e] = o[nt][1][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
          mma16816(o[nt][ks & 1], wa[ks], B.qb[nt][ks >> 1][2 * (ks & 1)], B.qb[nt][ks >> 1][2 * (ks & 1) + 1]);
#pragma unroll
      for (int j = 0; j < i; ++j) {
        mma16816(o[0][0], sa[j], B.m[j][0], B.m[j][1]);
        mma16816(o[1][0], sa[j], B.m[j][2], B.m[j][3]);
      }
      stsm_x4_t(obase + (uint32_t)(r0 + 16 * i) * 128u + f.o,
                pack_bf16(o[0][0][0] + o[0][1][0], o[0][0][1] + o[0][1][1]),
                pack_bf16(o[0][0][2] + o[0][1][2], o[0][0][3] + o[0][1][3]),
                pack_bf16(o[1][0][0] + o[1][1][0], o[1][0][1] + o[1][1][1]),
                pack_bf16(o[1][0][2] + o[1][1][2], o[1][0][3] + o[1][1][3]));
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Inner mini-batch b = 16, one CTA per head: four compute warps (sixteen columns each), one
// TMA producer warp and one writer warp. The compute warps never wait on each other: tiles
// arrive through full/empty mbarriers, and a finished 64-token tile (outputs in swizzled
// staging, per-warp loss partials) is handed to the writer through an oready mbarrier; the
// writer sums the loss partials, issues the TMA store of the outputs and returns the staging
// buffer through ofree.
// ---------------------------------------------------------------------------------------------

constexpr int kGateWarps = 2;  // alternate tiles: each has two tiles' time for one chunk's statistics
constexpr int kGateRing = 4;   // tiles of losses in flight from the writer to the gate warps
template <bool GATE>
constexpr int b16_threads() { return (kComputeWarps + 2 + (GATE ? kGateWarps : 0)) * 32; }

// Shared memory of one instantiation: arrays a variant does not use shrink to one element, and
// the plain TTT-Linear instantiations (no losses, no gate, one mini-batch a step) keep
// three input stages instead of four: at ~89 KB two CTAs fit on one SM, so with programmatic
// dependent launch every CTA of the next scan is resident (waiting) before this one ends, not
// only those that find an idle SM.
template <bool HAS_Q, bool LOSS, bool GATE, int NB>
struct __align__(1024) B16Smem {
  static constexpr int kS = (!LOSS && !GATE && NB == 1) ? 3 : kStages;  // input ring depth
  static constexpr int kGm = NB > 1 ? 2 : 1;
  uint8_t K[kS][kTileBytes];
  uint8_t V[kS][kTileBytes];
  uint8_t Q[kS][kTileBytes];
  uint8_t O[2][kTileBytes];
  uint8_t gm[kGm][NB > 1 ? kMaxTilePairs : 1][kPairBytes];  // chunked form: Gram blocks of tiles t (t & 1)
  // Per-lane loss partials of tile t (t & 1): [compute warp][lane group g][token], each the sum
  // of the squared residuals of the warp's two columns g, g+8; the writer adds them up.
  float lossp[LOSS ? 2 : 1][kComputeWarps][8][LOSS ? kLossStride : 1];
  float gl[GATE ? kGateRing : 1][kTileTok];  // tiles' losses handed from the writer to the gate warps
  uint64_t full[kS];
  uint64_t empty[kS];
  uint64_t oready[2];
  uint64_t ofree[2];
  uint64_t gmready[2];  // chunked form: the Gram blocks of a tile are complete (all compute lanes)
  uint64_t gready[kGateRing];
  uint64_t gfree[kGateRing];
  int abort;  // set by whichever warp's wait ran out; every other wait then returns at once
  // The gate's sequential state, passed between the gate warps in tile order: gate_turn is the
  // tile whose threshold update and routing may run next.
  float g_tau;
  int g_tau_set;
  int g_routed;
  int gate_turn;
  long long g_tokens;  // tokens gated since reset before this call
};

// The surprisal gate's state and constants for the scan that runs it in its own warps.
struct GateArgs {
  float* tau;         // [B·H] threshold carried between calls
  int32_t* tau_set;   // [B·H] whether τ has been set since reset
  int32_t* entries;   // [B·H, capacity, 3] (sequence, head, token) of routed tokens
  int32_t* counts;    // [B·H, 2] routed since reset, dropped because the cache was full
  int capacity, rank, heads;
  float ema_old, ema_new;
  double lhs, rhs;    // pass ⇔ lhs·S ≥ rhs·τ
  int64_t* tokens;    // [B·H] tokens gated since reset, advanced by this call's T
};

// Warp-uniform bounded wait: false (with abort set) if the phase did not complete in time.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const DevStatus& status, int* abort) {
  bool ok = mbar_wait(bar, parity, status, abort);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *reinterpret_cast<volatile int*>(abort) = 1;
  return ok;
}

// Bounded wait until *turn == want (a shared-memory counter advanced by another warp).
__device__ __forceinline__ bool wait_turn(const int* turn, int want, const DevStatus& status, int* abort) {
  const volatile int* tv = turn;
  const volatile int* av = abort;
  if (*tv == want) return true;
  const uint64_t t0 = globaltimer();
  while (*tv != want) {
    if (*av) return false;
    if (globaltimer() - t0 > status.limit_ns) {
      record_status(status, kDevTimeout, kSiteCounter | (int)((reinterpret_cast<uintptr_t>(turn) >> 2) & 0xFFFFu));
      *const_cast<volatile int*>(av) = 1;
      return false;
    }
  }
  return true;
}

// NB = inner mini-batches per chunk: 1 runs the steps one by one (compute16), 2 or 4 the chunked
// form (chunk_run) with the Gram blocks shared through shared memory one tile ahead.
template <bool HAS_Q, bool LOSS, bool GATE, int NB>
__global__ void __launch_bounds__(b16_threads<true>(), 1)
    k_linear_b16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 float* __restrict__ Wstate, float* __restrict__ loss, int T, float beta, const DevStatus status,
                 const GateArgs ga, int stall_tile) {
  static_assert(!GATE || LOSS, "the gate reads the losses");
  extern __shared__ uint8_t smem_raw[];
  using Smem = B16Smem<HAS_Q, LOSS, GATE, NB>;
  constexpr int kStages = Smem::kS;  // shadows the file-wide depth inside this kernel
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Loss partials of tile t for this warp (null without losses: the helpers then never use it).
  auto lossp_of = [&](int t, int w) -> float* { return LOSS ? &sm.lossp[t & 1][w][0][0] : nullptr; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int ntiles = (T + kTileTok - 1) / kTileTok;
  float* Wg = Wstate + (size_t)bh * 64 * 64;

  // Set-up that reads nothing a kernel before this one in the stream may still be writing runs
  // first: with programmatic dependent launch it overlaps the end of that kernel.
  if (warp == kComputeWarps && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (HAS_Q) tma_prefetch_desc(&tmQ);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kComputeWarps * 32);  // every compute lane arrives
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.oready[i], kComputeWarps * 32);
      mbar_init(&sm.ofree[i], 1);
      mbar_init(&sm.gmready[i], kComputeWarps * 32);
    }
    for (int i = 0; i < kGateRing; ++i) {
      mbar_init(&sm.gready[i], 1);
      mbar_init(&sm.gfree[i], 1);
    }
    sm.abort = 0;
    sm.gate_turn = 0;
    fence_barrier_init();
  }
  __syncthreads();  // the barriers exist for every warp
  // Wait for the kernel before this one (a no-op without programmatic dependent launch), then
  // let the next one start its own set-up: it waits in turn before reading what this one writes.
  // After the wait each role starts at once: the producer's first loads are in flight while the
  // compute warps read their slice of W.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp == kComputeWarps) {
    // ---------------- producer: TMA loads of K, V (and Q) tiles ----------------
    if (lane == 0) {
      const uint32_t stage_bytes = (HAS_Q ? 3u : 2u) * kTileBytes;
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int slot = t % kStages;
        if (t >= kStages && !mbar_wait(&sm.empty[slot], ((t / kStages) - 1) & 1, status, &sm.abort)) break;
        if (t != stall_tile) {
          mbar_arrive_expect_tx(&sm.full[slot], stage_bytes);
          tma_load_3d(sm.K[slot], &tmK, &sm.full[slot], 0, t * kTileTok, bh);
          tma_load_3d(sm.V[slot], &tmV, &sm.full[slot], 0, t * kTileTok, bh);
          if (HAS_Q) tma_load_3d(sm.Q[slot], &tmQ, &sm.full[slot], 0, t * kTileTok, bh);
        }
        issued = t + 1;
      }
      // Nothing may still be landing in shared memory when the CTA exits.
      for (int t = issued - kStages; t < issued; ++t) {
        if (t < 0 || t == stall_tile) continue;
        mbar_wait(&sm.full[t % kStages], (t / kStages) & 1, status, nullptr);
      }
    }
    return;
  }

  if (warp == kComputeWarps + 1) {
    // ---------------- writer: losses and output stores per tile ----------------
    for (int t = 0; t < ntiles; ++t) {
      const int b = t & 1;
      if (!warp_wait(&sm.oready[b], (t >> 1) & 1, status, &sm.abort)) break;
      float v0 = 0.f, v1 = 0.f;  // losses of tokens lane and lane + 32 of the tile
      if (LOSS) {
        const int ntok = min(kTileTok, T - t * kTileTok);
        float* Lt = loss + (size_t)bh * T + (size_t)t * kTileTok;
        // Each warp's sixteen columns as a pairwise tree over the lane groups, then the warps.
        auto token_loss = [&](int i) {
          float w[kComputeWarps];
#pragma unroll
          for (int cw = 0; cw < kComputeWarps; ++cw) {
            const float* x = lossp_of(b, cw) + i;
            w[cw] = ((x[0 * kLossStride] + x[1 * kLossStride]) + (x[2 * kLossStride] + x[3 * kLossStride])) +
                    ((x[4 * kLossStride] + x[5 * kLossStride]) + (x[6 * kLossStride] + x[7 * kLossStride]));
          }
          return (w[0] + w[1]) + (w[2] + w[3]);
        };
        if (lane < ntok) {
          v0 = token_loss(lane);
          Lt[lane] = v0;
        }
        if (lane + 32 < ntok) {
          v1 = token_loss(lane + 32);
          Lt[lane + 32] = v1;
        }
      }
      if (HAS_Q && lane == 0) {
        tma_store_3d(&tmO, sm.O[b], 0, t * kTileTok, bh);
        bulk_commit();
        bulk_wait_read<0>();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ofree[b]);
      if (GATE) {
        // Hand the tile's losses to the gate warps (slot t % kGateRing, last read for tile
        // t − kGateRing; a fresh barrier's phase before its first counts as complete).
        const int r = t % kGateRing;
        if (!warp_wait(&sm.gfree[r], ((t / kGateRing) + 1) & 1, status, &sm.abort)) break;
        sm.gl[r][lane] = v0;
        sm.gl[r][lane + 32] = v1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.gready[r]);
      }
    }
    if (HAS_Q && lane == 0) bulk_wait<0>();
    return;
  }

  if (GATE && warp >= kComputeWarps + 2) {
    // ---------------- gate warps: the surprisal gate, one 64-token chunk per tile ----------------
    // With the gate on T is a multiple of 64, so every tile is one gate chunk. Gate warp w takes
    // the tiles t ≡ w (mod kGateWarps): the chunk's percentile and sum are independent of the
    // other chunks; the threshold update and the routing then run in tile order, passed from
    // warp to warp through gate_turn.
    const int w = warp - (kComputeWarps + 2);
    const int seq = bh / ga.heads, head = bh % ga.heads;
    int32_t* E = ga.entries + (size_t)bh * ga.capacity * 3;
    // The gate's carried state, read by gate warp 0 before its first tile; the other gate warps
    // read it only after gate_turn has passed through warp 0 (which fences its writes).
    if (w == 0 && lane == 0) {
      sm.g_tau = ga.tau[bh];
      sm.g_tau_set = ga.tau_set[bh];
      sm.g_routed = ga.counts[2 * bh];
      sm.g_tokens = ga.tokens[bh];
    }
    __syncwarp();
    for (int t = w; t < ntiles; t += kGateWarps) {
      const int r = t % kGateRing;
      if (!warp_wait(&sm.gready[r], (t / kGateRing) & 1, status, &sm.abort)) break;
      const float v0 = sm.gl[r][lane], v1 = sm.gl[r][lane + 32];
      float p;
      double S;
      chunk_stats(sm.gl[r], lane, ga.rank, p, S);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.gfree[r]);
      if (!__all_sync(0xffffffffu, wait_turn(&sm.gate_turn, t, status, &sm.abort))) break;
      __threadfence_block();
      float tau = *reinterpret_cast<volatile float*>(&sm.g_tau);
      const bool set = *reinterpret_cast<volatile int*>(&sm.g_tau_set) != 0;
      const int routed = *reinterpret_cast<volatile int*>(&sm.g_routed);
      const long long tok0 = *reinterpret_cast<volatile long long*>(&sm.g_tokens);
      tau = tau_next(tau, set, p, ga.ema_old, ga.ema_new);
      const bool pass = ga.lhs * S >= ga.rhs * (double)tau;
      const bool f0 = pass && v0 > tau, f1 = pass && v1 > tau;
      const unsigned m0 = __ballot_sync(0xffffffffu, f0), m1 = __ballot_sync(0xffffffffu, f1);
      const unsigned below = (1u << lane) - 1u;
      const int pos0 = routed + __popc(m0 & below), pos1 = routed + __popc(m0) + __popc(m1 & below);
      const int tok = (int)(tok0 + (long long)t * kTileTok) + lane;
      if (f0 && pos0 < ga.capacity) {
        E[3 * pos0 + 0] = seq;
        E[3 * pos0 + 1] = head;
        E[3 * pos0 + 2] = tok;
      }
      if (f1 && pos1 < ga.capacity) {
        E[3 * pos1 + 0] = seq;
        E[3 * pos1 + 1] = head;
        E[3 * pos1 + 2] = tok + 32;
      }
      __syncwarp();
      if (lane == 0) {
        *reinterpret_cast<volatile float*>(&sm.g_tau) = tau;
        *reinterpret_cast<volatile int*>(&sm.g_tau_set) = 1;
        *reinterpret_cast<volatile int*>(&sm.g_routed) = routed + __popc(m0) + __popc(m1);
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&sm.gate_turn) = t + 1;
      }
    }
    // The warp that ran the last tile writes the state back.
    if (ntiles > 0 && w == (ntiles - 1) % kGateWarps && lane == 0 &&
        *reinterpret_cast<volatile int*>(&sm.gate_turn) == ntiles) {
      __threadfence_block();
      const int routed = sm.g_routed;
      ga.tau[bh] = sm.g_tau;
      ga.tau_set[bh] = sm.g_tau_set;
      ga.counts[2 * bh + 0] = routed;
      ga.counts[2 * bh + 1] = routed > ga.capacity ? routed - ga.capacity : 0;
      const long long tokens = sm.g_tokens + (long long)ntiles * kTileTok;
      ga.tokens[bh] = tokens;
      if (tokens > 0x7FFFFFFFll) record_status(status, kDevUnsupported, kSiteTokenLimit | (bh & 0xFFFF));
    }
    return;
  }

  // ---------------- compute warps ----------------
  const int g = lane >> 2, q = lane & 3;
  const int col0 = 16 * warp;
  const StepOffsets offs = step_offsets(lane, col0);
  // This warp's slice of W, in accumulator layout (warp w owns columns 16w .. 16w+15):
  // acc[nt][e] = W[8nt + 2q + (e&1)][16w + g + 8(e>>1)].
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)];

  if constexpr (NB > 1) {
    // ---- chunked form: chunks of NB blocks, Gram blocks one tile ahead ----
    constexpr int kCPT = 64 / (16 * NB);          // chunks per tile
    constexpr int kPPC = NB * (NB - 1) / 2;       // pairs per chunk
    const int nfull = T / kTileTok, rem = (T % kTileTok) / 16;
    const uint32_t gm0 = smem_u32(sm.gm[0]), gm1 = smem_u32(sm.gm[1]);
    auto gram = [&](int tt) {  // this warp's share of tile tt's Gram blocks (a stale slot past the end: unused)
      const int slot = tt % kStages;
      gram_tile<NB, HAS_Q>(smem_u32(sm.K[slot]), smem_u32(sm.Q[slot]), (tt & 1) ? gm1 : gm0, offs, warp, lane);
    };
    bool ok = ntiles > 0 && warp_wait(&sm.full[0], 0, status, &sm.abort);
    if (ok) {
      gram(0);
      mbar_arrive(&sm.gmready[0]);
    }
    int t = 0;
    for (; ok && t < nfull; ++t) {
      // Waits of the tile, tested without a branch (as in the per-step form): the output staging
      // (last used by tile t − 2), the inputs of tile t+1 (read by the Gram share of tile t+1)
      // and the Gram blocks of tile t.
      const int t1 = t + 1;
      const uint32_t pfree = ((t >> 1) + 1) & 1;
      const uint32_t pfull = ((t1 / kStages) + (t1 < ntiles ? 0 : 1)) & 1;
      const uint32_t pgm = (t >> 1) & 1;
      const bool ready = mbar_try_wait(&sm.ofree[t & 1], pfree) & mbar_try_wait(&sm.full[t1 % kStages], pfull) &
                         mbar_try_wait(&sm.gmready[t & 1], pgm);
      if (!__all_sync(0xffffffffu, ready)) {
        ok = warp_wait(&sm.ofree[t & 1], pfree, status, &sm.abort) &&
             warp_wait(&sm.full[t1 % kStages], pfull, status, &sm.abort) &&
             warp_wait(&sm.gmready[t & 1], pgm, status, &sm.abort);
        if (!ok) break;
      }
      const int slot = t % kStages;
      const uint32_t kb = smem_u32(sm.K[slot]), vb = smem_u32(sm.V[slot]), qb = smem_u32(sm.Q[slot]);
      const uint32_t gb = (t & 1) ? gm1 : gm0, ob = smem_u32(sm.O[t & 1]);
#pragma unroll
      for (int cc = 0; cc < kCPT; ++cc)
        chunk_run<NB, HAS_Q, LOSS>(acc, kb, vb, qb, gb + (uint32_t)(cc * kPPC) * kPairBytes, ob, offs,
                                   lossp_of(t, warp), 16 * NB * cc, lane, beta);
      mbar_arrive(&sm.empty[slot]);  // every fragment of tile t has been read
      // Tile t's Gram blocks have all been read by this warp: its share of tile t+1's may go into
      // the other buffer (every warp passed the top of tile t, so none still reads tile t − 1's).
      gram(t1);
      mbar_arrive(&sm.gmready[t1 & 1]);
      if (HAS_Q) fence_proxy_async_smem();
      mbar_arrive(&sm.oready[t & 1]);
    }
    // A last tile of fewer than 64 tokens (rem 16-token blocks; its Gram blocks were made with
    // the tile before, or in the prologue; rows past T were read as zeros).
    if (ok && rem > 0) {
      const bool w_ok = (t < 2 || warp_wait(&sm.ofree[t & 1], ((t >> 1) - 1) & 1, status, &sm.abort)) &&
                        warp_wait(&sm.gmready[t & 1], (t >> 1) & 1, status, &sm.abort);
      if (w_ok) {
        const int slot = t % kStages;
        const uint32_t kb = smem_u32(sm.K[slot]), vb = smem_u32(sm.V[slot]), qb = smem_u32(sm.Q[slot]);
        const uint32_t gb = (t & 1) ? gm1 : gm0, ob = smem_u32(sm.O[t & 1]);
        float* lp = lossp_of(t, warp);
        if (NB == 2) {
          if (rem >= 2) chunk_run<2, HAS_Q, LOSS>(acc, kb, vb, qb, gb, ob, offs, lp, 0, lane, beta);
          if (rem != 2) chunk_run<1, HAS_Q, LOSS>(acc, kb, vb, qb, gb, ob, offs, lp, rem == 1 ? 0 : 32, lane, beta);
        } else {
          if (rem == 1) chunk_run<1, HAS_Q, LOSS>(acc, kb, vb, qb, gb, ob, offs, lp, 0, lane, beta);
          if (rem == 2) chunk_run<2, HAS_Q, LOSS>(acc, kb, vb, qb, gb, ob, offs, lp, 0, lane, beta);
          if (rem == 3) chunk_run<3, HAS_Q, LOSS>(acc, kb, vb, qb, gb, ob, offs, lp, 0, lane, beta);
        }
        mbar_arrive(&sm.empty[slot]);
        if (HAS_Q) fence_proxy_async_smem();
        mbar_arrive(&sm.oready[t & 1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)] = acc[nt][e];
    return;
  }

  // Fragments of step s (rows 16s .. 16s+15) of tile t are loaded one step before they are
  // used. A 64-token tile is four straight-line steps: every wait of the tile sits at its top
  // and the end-of-tile arrivals are made by all lanes, so the steps themselves contain no
  // branch (a branch costs a warp its in-flight mma results: measured on B200, a per-step
  // conditional structure ran 540 cycles a step against 313 for straight-line steps).
  auto load = [&](Frag16& F, int t, int s) {
    const int slot = t % kStages;
    load_frag16<HAS_Q>(F, smem_u32(sm.K[slot]), smem_u32(sm.V[slot]), smem_u32(sm.Q[slot]), offs, 16 * s);
  };
  auto comp = [&](const Frag16& F, int t, int s) {
    compute16<HAS_Q, LOSS>(acc, F, smem_u32(sm.O[t & 1]), offs.o, lossp_of(t, warp), 16 * s, lane, beta);
  };

  const int nfull = T / kTileTok, rem = (T % kTileTok) / 16;
  Frag16 F0, F1;
  bool ok = ntiles > 0 && warp_wait(&sm.full[0], 0, status, &sm.abort);
  if (ok) load(F0, 0, 0);
  int t = 0;
  for (; ok && t < nfull; ++t) {
    // The staging buffer of tile t was last used by tile t − 2; tile t+1's inputs are needed
    // by the last step of this tile. Both are tested without a branch (a phase that has nothing
    // to wait for is given the parity of its completed predecessor: for t < 2 that is the phase
    // before a fresh barrier's first, which counts as complete); only if either is still open
    // does the warp take the bounded waits. A branch here costs the warp its in-flight mma
    // results, so there is one per tile (a two-tile loop body measured slower: its code no
    // longer fits the instruction cache).
    const int t1 = t + 1;
    const uint32_t pfree = ((t >> 1) + 1) & 1;
    const uint32_t pfull = ((t1 / kStages) + (t1 < ntiles ? 0 : 1)) & 1;
    const bool ready = mbar_try_wait(&sm.ofree[t & 1], pfree) & mbar_try_wait(&sm.full[t1 % kStages], pfull);
    if (!__all_sync(0xffffffffu, ready)) {
      ok = warp_wait(&sm.ofree[t & 1], pfree, status, &sm.abort) &&
           warp_wait(&sm.full[t1 % kStages], pfull, status, &sm.abort);
      if (!ok) break;
    }
    load(F1, t, 1);
    comp(F0, t, 0);
    load(F0, t, 2);
    comp(F1, t, 1);
    load(F1, t, 3);
    comp(F0, t, 2);
    mbar_arrive(&sm.empty[t % kStages]);  // every fragment of tile t has been read
    load(F0, t + 1, 0);                   // past the last tile this reads a stale slot, unused
    comp(F1, t, 3);
    if (HAS_Q) fence_proxy_async_smem();
    mbar_arrive(&sm.oready[t & 1]);
  }
  // A last tile of fewer than 64 tokens (its first fragments are already in F0).
  if (ok && rem > 0) {
    if (t < 2 || warp_wait(&sm.ofree[t & 1], ((t >> 1) - 1) & 1, status, &sm.abort)) {
      comp(F0, t, 0);
      for (int s = 1; s < rem; ++s) {
        load(F1, t, s);
        comp(F1, t, s);
      }
      mbar_arrive(&sm.empty[t % kStages]);
      if (HAS_Q) fence_proxy_async_smem();
      mbar_arrive(&sm.oready[t & 1]);
    }
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)] = acc[nt][e];
}

template <int B>
__global__ void __launch_bounds__(kThreads, 1)
    k_linear_scan(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  float* __restrict__ Wstate, float* __restrict__ loss, int T, float beta, int has_q,
                  const DevStatus status) {
  extern __shared__ uint8_t smem_raw[];
  LinearSmem& sm = *reinterpret_cast<LinearSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nstages = (T + kTileTok - 1) / kTileTok;
  const uint32_t stage_bytes = (has_q ? 3u : 2u) * kTileBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kComputeWarps);
    }
    sm.abort = 0;
    sm.cabort[0] = sm.cabort[1] = 0;
    sm.consumed = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ---------------- producer: TMA loads of K, V, Q tiles ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (has_q) tma_prefetch_desc(&tmQ);
      int issued = 0;
      for (int s = 0; s < nstages; ++s) {
        const int slot = s % kStages;
        if (s >= kStages && !mbar_wait(&sm.empty[slot], ((s / kStages) - 1) & 1, status, &sm.abort)) break;
        mbar_arrive_expect_tx(&sm.full[slot], stage_bytes);
        tma_load_3d(sm.K[slot], &tmK, &sm.full[slot], 0, s * kTileTok, bh);
        tma_load_3d(sm.V[slot], &tmV, &sm.full[slot], 0, s * kTileTok, bh);
        if (has_q) tma_load_3d(sm.Q[slot], &tmQ, &sm.full[slot], 0, s * kTileTok, bh);
        issued = s + 1;
      }
      // Nothing may still be landing in shared memory when the CTA exits: wait (bounded) for
      // the newest issued phase of every slot. A phase that already completed returns at once.
      for (int s = issued - kStages; s < issued; ++s) {
        if (s < 0) continue;
        mbar_wait(&sm.full[s % kStages], (s / kStages) & 1, status, nullptr);
      }
    }
    __syncthreads();
    return;
  }

  // ---------------- compute warps ----------------
  const int g = lane >> 2, q = lane & 3;
  const int col0 = 16 * warp;  // first W column owned by this warp
  float* Wg = Wstate + (size_t)bh * 64 * 64;

  // Wᵀ slice in accumulator layout: acc[nt][e] = W[8nt + 2q + (e&1)][col0 + g + 8(e>>1)].
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)];

  const StepOffsets offs = step_offsets(lane, col0);
  constexpr int NT = B / 8;   // token n-tiles per mini-batch
  constexpr int KT = B / 16;  // token k-steps per mini-batch

  for (int s = 0; s < nstages; ++s) {
    const int slot = s % kStages;
    // Every compute warp takes the same exit decision: the flag for tile s is only written
    // before this barrier and only read after it (tile s+2 uses the same flag, but no warp can
    // reach its wait before all warps passed the end-of-tile barriers of tile s+1).
    if (!mbar_wait(&sm.full[slot], (s / kStages) & 1, status, nullptr)) sm.cabort[s & 1] = 1;
    named_sync();
    if (*reinterpret_cast<volatile int*>(&sm.cabort[s & 1])) break;
    const int ntok = min(kTileTok, T - s * kTileTok);
    const uint32_t kbase = smem_u32(sm.K[slot]);
    const uint32_t vbase = smem_u32(sm.V[slot]);
    const uint32_t qbase = smem_u32(sm.Q[slot]);
    uint8_t* obuf = sm.O[s & 1];

    {
      for (int r0 = 0; r0 < ntok; r0 += B) {
        // A fragments of Wᵀ (hi and lo) for the four 16-key k-steps.
        uint32_t whi[4][4], wlo[4][4];
  #pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          split2(acc[2 * ks][0], acc[2 * ks][1], whi[ks][0], wlo[ks][0]);
          split2(acc[2 * ks][2], acc[2 * ks][3], whi[ks][1], wlo[ks][1]);
          split2(acc[2 * ks + 1][0], acc[2 * ks + 1][1], whi[ks][2], wlo[ks][2]);
          split2(acc[2 * ks + 1][2], acc[2 * ks + 1][3], whi[ks][3], wlo[ks][3]);
        }

        // Pᵀ = −Vᵀ + Wᵀ·Kᵀ and Oᵀ = Wᵀ·Qᵀ for the B tokens of this mini-batch.
        float p[NT][4], o[NT][4];
  #pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
          // −V[t][c] for tokens r0+8nt.. (two n-tiles) and this warp's 16 columns.
          uint32_t v[4];
          const int mi = lane >> 3, ri = lane & 7;
          ldsm_x4_t(vbase + swz128_bf16(r0 + 8 * (nt + (mi >> 1)) + ri, col0 + 8 * (mi & 1)), v);
          const float2 v0 = unpack_bf16(v[0]), v1 = unpack_bf16(v[1]), v2 = unpack_bf16(v[2]), v3 = unpack_bf16(v[3]);
          p[nt][0] = -v0.x; p[nt][1] = -v0.y; p[nt][2] = -v1.x; p[nt][3] = -v1.y;
          if (nt + 1 < NT) { p[nt + 1][0] = -v2.x; p[nt + 1][1] = -v2.y; p[nt + 1][2] = -v3.x; p[nt + 1][3] = -v3.y; }
        }
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
  #pragma unroll
          for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
          float p2[4] = {0.f, 0.f, 0.f, 0.f};
  #pragma unroll
          for (int ks = 0; ks < 4; ks += 2) {
            // B fragments of Kᵀ (and Qᵀ): rows = tokens r0+8nt.., keys 16ks .. 16ks+31.
            const int mi = lane >> 3, ri = lane & 7;
            const uint32_t off = swz128_bf16(r0 + 8 * nt + ri, 16 * ks + 8 * mi);
            uint32_t kb[4];
            ldsm_x4(kbase + off, kb);
            mma16816(p[nt], whi[ks], kb[0], kb[1]);
            mma16816(p2, wlo[ks], kb[0], kb[1]);
            mma16816(p[nt], whi[ks + 1], kb[2], kb[3]);
            mma16816(p2, wlo[ks + 1], kb[2], kb[3]);
            if (has_q) {
              uint32_t qb[4];
              ldsm_x4(qbase + off, qb);
              mma16816(o[nt], whi[ks], qb[0], qb[1]);
              mma16816(o[nt], wlo[ks], qb[0], qb[1]);
              mma16816(o[nt], whi[ks + 1], qb[2], qb[3]);
              mma16816(o[nt], wlo[ks + 1], qb[2], qb[3]);
            }
          }
  #pragma unroll
          for (int e = 0; e < 4; ++e) p[nt][e] += p2[e];
        }

        // Per-token loss: this thread holds R for tokens 8nt+2q, 8nt+2q+1 at columns g, g+8.
        if (loss != nullptr) {
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float l0 = p[nt][0] * p[nt][0] + p[nt][2] * p[nt][2];
            float l1 = p[nt][1] * p[nt][1] + p[nt][3] * p[nt][3];
  #pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
              l0 += __shfl_xor_sync(0xffffffffu, l0, m);
              l1 += __shfl_xor_sync(0xffffffffu, l1, m);
            }
            if (g == 0) {
              sm.lossp[warp][r0 + 8 * nt + 2 * q] = l0;
              sm.lossp[warp][r0 + 8 * nt + 2 * q + 1] = l1;
            }
          }
        }

        // Outputs into the swizzled staging tile (row = token in the tile, col = W column).
        if (has_q) {
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = r0 + 8 * nt + 2 * q + (e & 1);
              const int col = col0 + g + 8 * (e >> 1);
              *reinterpret_cast<__nv_bfloat16*>(obuf + swz128_bf16(row, col)) = __float2bfloat16_rn(o[nt][e]);
            }
        }

        // Wᵀ += Sᵀ·K with S = −(η/b)·R, S fed as bf16 hi + lo.
        uint32_t shi[KT][4], slo[KT][4];
  #pragma unroll
        for (int kt = 0; kt < KT; ++kt) {
          split2(-beta * p[2 * kt][0], -beta * p[2 * kt][1], shi[kt][0], slo[kt][0]);
          split2(-beta * p[2 * kt][2], -beta * p[2 * kt][3], shi[kt][1], slo[kt][1]);
          split2(-beta * p[2 * kt + 1][0], -beta * p[2 * kt + 1][1], shi[kt][2], slo[kt][2]);
          split2(-beta * p[2 * kt + 1][2], -beta * p[2 * kt + 1][3], shi[kt][3], slo[kt][3]);
        }
  #pragma unroll
        for (int kt = 0; kt < KT; ++kt) {
  #pragma unroll
          for (int nt = 0; nt < 8; nt += 2) {
            // B fragments of K[token][key]: tokens r0+16kt .. +15, keys 8nt .. 8nt+15 (transposed).
            const int mi = lane >> 3, ri = lane & 7;
            uint32_t kb[4];
            ldsm_x4_t(kbase + swz128_bf16(r0 + 16 * kt + 8 * (mi & 1) + ri, 8 * nt + 8 * (mi >> 1)), kb);
            mma16816(acc[nt], shi[kt], kb[0], kb[1]);
            mma16816(acc[nt], slo[kt], kb[0], kb[1]);
            mma16816(acc[nt + 1], shi[kt], kb[2], kb[3]);
            mma16816(acc[nt + 1], slo[kt], kb[2], kb[3]);
          }
        }
      }
    }
    // End of the tile: outputs and losses of 64 tokens are complete in shared memory.
    if (has_q) fence_proxy_async_smem();
    named_sync();
    if (loss != nullptr && warp == 0) {
      for (int i = lane; i < ntok; i += 32) {
        const float l = (sm.lossp[0][i] + sm.lossp[1][i]) + (sm.lossp[2][i] + sm.lossp[3][i]);
        loss[(size_t)bh * T + (size_t)s * kTileTok + i] = l;
      }
    }
    if (threadIdx.x == 0) {
      if (has_q) {
        tma_store_3d(&tmO, obuf, 0, s * kTileTok, bh);
        bulk_commit();
        bulk_wait_read<1>();  // the other staging tile is free again
      }
      sm.consumed = s + 1;
    }
    named_sync();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
  }

  if (threadIdx.x == 0 && has_q) bulk_wait<0>();
  // Final state.
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)] = acc[nt][e];
  __syncthreads();
}


template <int B>
ttt_status launch(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                  const CUtensorMap& to, float* loss, int T, int has_q, cudaStream_t s) {
  const size_t smem = sizeof(LinearSmem) + 1024;
  const uint64_t bit = 1ull << (8 + B / 32);
  if (!(st->lin.smem_set & bit)) {
    TTT_CUDA(cudaFuncSetAttribute(k_linear_scan<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    st->lin.smem_set |= bit;
  }
  const int grid = st->cfg.batch * st->cfg.heads;
  const float beta = st->cfg.eta / (float)B;
  k_linear_scan<B><<<grid, kThreads, smem, s>>>(tk, tv, tq, to, st->lin.W, loss, T, beta, has_q,
                                                DevStatus{st->status.dev, st->wait_limit_ns, st->status.dev + 1});
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

template <bool HAS_Q, bool LOSS, bool GATE, int NB>
ttt_status launch_b16_nb(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                         const CUtensorMap& to, float* loss, int T, const GateArgs& ga, cudaStream_t s) {
  const size_t smem = sizeof(B16Smem<HAS_Q, LOSS, GATE, NB>) + 1024;
  // One bit per instantiation whose shared-memory limit has been raised on this state's device.
  const uint64_t bit = 1ull << (16 + 8 * (NB == 1 ? 0 : NB == 2 ? 1 : 2) + 4 * GATE + 2 * HAS_Q + LOSS);
  if (!(st->lin.smem_set & bit)) {
    TTT_CUDA(cudaFuncSetAttribute(k_linear_b16<HAS_Q, LOSS, GATE, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem));
    // All of the SM's unified L1/shared memory as shared memory, so that two CTAs of the small
    // instantiation fit on one SM.
    TTT_CUDA(cudaFuncSetAttribute(k_linear_b16<HAS_Q, LOSS, GATE, NB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  (int)cudaSharedmemCarveoutMaxShared));
    st->lin.smem_set |= bit;
  }
  const int grid = st->cfg.batch * st->cfg.heads;
  const float beta = st->cfg.eta / 16.0f;
  // Fault injection (tests): the producer never loads tile 1, so the compute warps' wait for it
  // runs out.
  int stall_tile = -1;
  if (st->inject_stall && T > 64) {
    stall_tile = 1;
    st->inject_stall = 0;
  }
  // Programmatic dependent launch: the kernel's set-up may overlap the end of the kernel before
  // it in the stream (typically the previous scan); it waits for that kernel before reading
  // anything.
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)grid);
  lc.blockDim = dim3((unsigned)b16_threads<GATE>());
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  TTT_CUDA(cudaLaunchKernelEx(&lc, k_linear_b16<HAS_Q, LOSS, GATE, NB>, tk, tv, tq, to, st->lin.W, loss, T, beta,
                              DevStatus{st->status.dev, st->wait_limit_ns, st->status.dev + 1}, ga, stall_tile));
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

template <bool HAS_Q, bool LOSS, bool GATE>
ttt_status launch_b16_impl(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                           const CUtensorMap& to, float* loss, int T, const GateArgs& ga, cudaStream_t s) {
  switch (st->lin.form) {
    case 2: return launch_b16_nb<HAS_Q, LOSS, GATE, 2>(st, tk, tv, tq, to, loss, T, ga, s);
    case 4: return launch_b16_nb<HAS_Q, LOSS, GATE, 4>(st, tk, tv, tq, to, loss, T, ga, s);
    default: return launch_b16_nb<HAS_Q, LOSS, GATE, 1>(st, tk, tv, tq, to, loss, T, ga, s);
  }
}

ttt_status launch_b16(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                      const CUtensorMap& to, float* loss, int T, int has_q, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  GateArgs ga{};
  if (c.gate_enable) {
    ga = GateArgs{st->gate.tau, st->gate.tau_set, st->gate.entries, st->gate.counts, c.cache_capacity,
                  gate_rank(c), c.heads, c.gate_ema_old, c.gate_ema_new, (double)c.gate_mean_den,
                  (double)c.gate_mean_num * kTileTok, st->gate.tokens};
    const ttt_status r = has_q ? launch_b16_impl<true, true, true>(st, tk, tv, tq, to, loss, T, ga, s)
                               : launch_b16_impl<false, true, true>(st, tk, tv, tq, to, loss, T, ga, s);
    if (r != TTT_OK) return r;
    st->gate.t_offset += T;
    return TTT_OK;
  }
  if (has_q) return loss ? launch_b16_impl<true, true, false>(st, tk, tv, tq, to, loss, T, ga, s)
                         : launch_b16_impl<true, false, false>(st, tk, tv, tq, to, loss, T, ga, s);
  return loss ? launch_b16_impl<false, true, false>(st, tk, tv, tq, to, loss, T, ga, s)
              : launch_b16_impl<false, false, false>(st, tk, tv, tq, to, loss, T, ga, s);
}

}  // namespace

ttt_status linear_scan(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                       int64_t T, __nv_bfloat16* O, float* loss, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const uint64_t BH = (uint64_t)c.batch * c.heads;
  const uint64_t dims[3] = {64, (uint64_t)T, BH};
  const uint64_t strides[2] = {128, (uint64_t)T * 128};
  const uint32_t box[3] = {64, (uint32_t)kTileTok, 1};
  LinearBuffers& lb = st->lin;
  const bool has_q = Q != nullptr;
  const void* key[4] = {K, V, Q, O};
  // Look the buffer set up among the cached ones; otherwise encode it into the least recently
  // used entry.
  LinearMapSet* ms = nullptr;
  for (LinearMapSet& m : lb.map_sets)
    if (m.T == T && m.key[0] == key[0] && m.key[1] == key[1] && m.key[2] == key[2] && m.key[3] == key[3]) ms = &m;
  if (ms == nullptr) {
    ms = &lb.map_sets[0];
    for (LinearMapSet& m : lb.map_sets)
      if (m.last_use < ms->last_use) ms = &m;
    ms->T = -1;  // invalid until all four are encoded
    TTT_TRY(encode_tmap(&ms->maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    TTT_TRY(encode_tmap(&ms->maps[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    if (has_q) {
      TTT_TRY(encode_tmap(&ms->maps[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
      TTT_TRY(encode_tmap(&ms->maps[3], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, O, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    } else {
      ms->maps[2] = ms->maps[0];
      ms->maps[3] = ms->maps[0];
    }
    for (int i = 0; i < 4; ++i) ms->key[i] = key[i];
    ms->T = T;
  }
  ms->last_use = ++lb.map_clock;
  const CUtensorMap &tk = ms->maps[0], &tv = ms->maps[1], &tq = ms->maps[2], &to = ms->maps[3];
  switch (c.chunk) {
    case 16: return launch_b16(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    case 32: return launch<32>(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    case 64: return launch<64>(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    default: return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear: mini-batch %d not built", c.chunk);
  }
}

}  // namespace ttt
