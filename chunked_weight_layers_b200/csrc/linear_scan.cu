// TTT-Linear mini-batch gradient scan ("テスト時学習（Test-Time Training）とは", the TTT layers
// page: the hidden state is the weight W of a linear model and each update is one
// self-supervised gradient step). Per (sequence, head) and inner mini-batch i of b tokens:
//   O_i = Q_i·W_i,   R_i = K_i·W_i − V_i,   L_t = ‖R_i[t]‖²,   W_{i+1} = W_i − (η/b)·K_iᵀ·R_i.
//
// Design (B200):
//  * the per-head state is 64x64 fp32 and never leaves the SM: it lives in mma accumulator
//    registers. Column c of W only ever depends on column c of R (R[:, c] = K·W[:, c] − V[:, c]),
//    so columns are split across warps (and, for b = 16, a head's two column halves across
//    two CTAs) with no communication inside a step.
//  * k_linear_b16 (b = 16, one CTA per head): four compute warps own sixteen columns each and
//    compute every product transposed, so each accumulator layout is directly the next mma's A
//    operand. Operand fragments are loaded one step ahead; a 64-token tile is four
//    straight-line steps with all waits at its top. A TMA producer warp fills the K/V/Q ring
//    and a writer warp sums loss partials and stores the output tiles, so compute warps never
//    meet at a barrier.
//  * k_linear_n8 (b = 16 when 2·B·H ≤ SM count): two CTAs per head, four warps per CTA, eight
//    columns per warp, products in their natural orientation with movmatrix.trans turning
//    accumulators into B operands; partial losses of the two halves are added into a zeroed
//    output.
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
#include "internal.h"

namespace ttt {

namespace {

constexpr int kStages = 4;        // ring depth (64-token tiles): 96 KB of K/V/Q in flight per SM
constexpr int kTileTok = 64;      // tokens per tile
constexpr int kTileBytes = kTileTok * 128;  // 64 tokens x 64 bf16
constexpr int kComputeWarps = 4;
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
    float o[2][2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][0][e] = o[nt][1][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        mma16816(o[nt][ks & 1], wa[ks], F.qb[nt][ks >> 1][2 * (ks & 1)], F.qb[nt][ks >> 1][2 * (ks & 1) + 1]);
    stsm_x4_t(obase + (uint32_t)r0 * 128u + ofs_o, pack_bf16(o[0][0][0] + o[0][1][0], o[0][0][1] + o[0][1][1]),
              pack_bf16(o[0][0][2] + o[0][1][2], o[0][0][3] + o[0][1][3]),
              pack_bf16(o[1][0][0] + o[1][1][0], o[1][0][1] + o[1][1][1]),
              pack_bf16(o[1][0][2] + o[1][1][2], o[1][0][3] + o[1][1][3]));
  }
  if (LOSS) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float l0 = p[nt][0] * p[nt][0] + p[nt][2] * p[nt][2];
      float l1 = p[nt][1] * p[nt][1] + p[nt][3] * p[nt][3];
#pragma unroll
      for (int m = 4; m < 32; m <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, m);
        l1 += __shfl_xor_sync(0xffffffffu, l1, m);
      }
      if (g == 0) *reinterpret_cast<float2*>(&lossp[r0 + 8 * nt + 2 * q]) = make_float2(l0, l1);
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

constexpr int kB16Threads = (kComputeWarps + 2) * 32;

struct __align__(1024) B16Smem {
  uint8_t K[kStages][kTileBytes];
  uint8_t V[kStages][kTileBytes];
  uint8_t Q[kStages][kTileBytes];
  uint8_t O[2][kTileBytes];
  float lossp[2][kComputeWarps][kTileTok];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t oready[2];
  uint64_t ofree[2];
  int abort;  // set by whichever warp's wait ran out; every other wait then returns at once
};

// Warp-uniform bounded wait: false (with abort set) if the phase did not complete in time.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* status, int* abort) {
  bool ok = mbar_wait(bar, parity, status, abort);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *reinterpret_cast<volatile int*>(abort) = 1;
  return ok;
}

template <bool HAS_Q, bool LOSS>
__global__ void __launch_bounds__(kB16Threads, 1)
    k_linear_b16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 float* __restrict__ Wstate, float* __restrict__ loss, int T, float beta, int* status) {
  extern __shared__ uint8_t smem_raw[];
  B16Smem& sm = *reinterpret_cast<B16Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int ntiles = (T + kTileTok - 1) / kTileTok;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kComputeWarps * 32);  // every compute lane arrives
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.oready[i], kComputeWarps * 32);
      mbar_init(&sm.ofree[i], 1);
    }
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ---------------- producer: TMA loads of K, V (and Q) tiles ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (HAS_Q) tma_prefetch_desc(&tmQ);
      const uint32_t stage_bytes = (HAS_Q ? 3u : 2u) * kTileBytes;
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int slot = t % kStages;
        if (t >= kStages && !mbar_wait(&sm.empty[slot], ((t / kStages) - 1) & 1, status, &sm.abort)) break;
        mbar_arrive_expect_tx(&sm.full[slot], stage_bytes);
        tma_load_3d(sm.K[slot], &tmK, &sm.full[slot], 0, t * kTileTok, bh);
        tma_load_3d(sm.V[slot], &tmV, &sm.full[slot], 0, t * kTileTok, bh);
        if (HAS_Q) tma_load_3d(sm.Q[slot], &tmQ, &sm.full[slot], 0, t * kTileTok, bh);
        issued = t + 1;
      }
      // Nothing may still be landing in shared memory when the CTA exits.
      for (int t = issued - kStages; t < issued; ++t) {
        if (t < 0) continue;
        mbar_wait(&sm.full[t % kStages], (t / kStages) & 1, status, nullptr);
      }
    }
    return;
  }

  if (warp == kComputeWarps + 1) {
    // ---------------- writer: loss sums and output stores per tile ----------------
    for (int t = 0; t < ntiles; ++t) {
      const int b = t & 1;
      if (!warp_wait(&sm.oready[b], (t >> 1) & 1, status, &sm.abort)) break;
      if (LOSS) {
        const int ntok = min(kTileTok, T - t * kTileTok);
        for (int i = lane; i < ntok; i += 32)
          loss[(size_t)bh * T + (size_t)t * kTileTok + i] =
              (sm.lossp[b][0][i] + sm.lossp[b][1][i]) + (sm.lossp[b][2][i] + sm.lossp[b][3][i]);
      }
      if (HAS_Q && lane == 0) {
        tma_store_3d(&tmO, sm.O[b], 0, t * kTileTok, bh);
        bulk_commit();
        bulk_wait_read<0>();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ofree[b]);
    }
    if (HAS_Q && lane == 0) bulk_wait<0>();
    return;
  }

  // ---------------- compute warps ----------------
  const int g = lane >> 2, q = lane & 3;
  const int col0 = 16 * warp;
  float* Wg = Wstate + (size_t)bh * 64 * 64;
  // Wᵀ slice in accumulator layout: acc[nt][e] = W[8nt + 2q + (e&1)][col0 + g + 8(e>>1)].
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = Wg[(8 * nt + 2 * q + (e & 1)) * 64 + col0 + g + 8 * (e >> 1)];
  const StepOffsets offs = step_offsets(lane, col0);

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
    compute16<HAS_Q, LOSS>(acc, F, smem_u32(sm.O[t & 1]), offs.o, sm.lossp[t & 1][warp], 16 * s, lane, beta);
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
                  int* status) {
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


// ---------------------------------------------------------------------------------------------
// Inner mini-batch b = 16, eight columns per warp, each head split over two CTAs.
//
// Column c of W only depends on column c of R, so a head's 64 columns are split into two
// halves on two CTAs (no communication) and each of a CTA's four warps owns 8 columns. The
// products run in their natural orientation (m16n8k16 with N = 8 columns):
//   P = K·W (A = K from ldmatrix, B = W from the accumulator via movmatrix.trans),
//   R = P − V, loss, S = −(η/b)·R,
//   W += Kᵀ·S (A = Kᵀ from ldmatrix.trans, B = S via movmatrix.trans),  O = Q·W.
// Half the instructions per warp and step of the 16-columns-per-warp form, and the heads
// reach every SM. The per-token loss is the sum of the two halves' partial sums: each CTA
// adds its partial to a zeroed output (two terms onto zero: the result does not depend on
// their order).
// ---------------------------------------------------------------------------------------------

struct N8Offsets {
  uint32_t ka[4];  // K (or Q) A fragments: [16-key k-step]
  uint32_t kt[4];  // Kᵀ A fragments of the update: [16-key m-tile]
  uint32_t v;      // V fragment of this warp's 8 columns
  uint32_t o;      // output staging rows (64-byte rows, 64-byte swizzle)
};

__device__ __forceinline__ N8Offsets n8_offsets(int lane, int vcol, int w) {
  const int mi = lane >> 3, ri = lane & 7;
  N8Offsets f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f.ka[k] = swz128_bf16(8 * (mi & 1) + ri, 16 * k + 8 * (mi >> 1));
    f.kt[k] = swz128_bf16(8 * (mi >> 1) + ri, 16 * k + 8 * (mi & 1));
  }
  f.v = swz128_bf16(8 * (mi & 1) + ri, vcol);
  const int orow = 8 * (mi & 1) + ri;
  f.o = (uint32_t)(orow * 64 + ((w ^ ((orow >> 1) & 3)) << 4));
  return f;
}

__device__ __forceinline__ uint32_t movm_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void stsm_x2(uint32_t addr, uint32_t r0, uint32_t r1) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(addr), "r"(r0), "r"(r1) : "memory");
}

__device__ __forceinline__ void mma_n8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc[mt][e] = W[16mt + g + 8(e>>1)][col0 + 2q + (e&1)] for this warp's 8 columns.
__device__ __forceinline__ void step16_n8(float (&acc)[4][4], uint32_t kbase, uint32_t vbase, uint32_t qbase,
                                          uint32_t obase, const N8Offsets& f, float* lossp, int r0, int lane,
                                          float beta, int has_q, bool want_loss) {
  const int g = lane >> 2;
  const uint32_t rofs = (uint32_t)r0 * 128u;
  uint32_t ka[4][4], kt[4][4], qa[4][4], v0, v1;
#pragma unroll
  for (int k = 0; k < 4; ++k) ldsm_x4(kbase + rofs + f.ka[k], ka[k]);
  ldsm_x2(vbase + rofs + f.v, v0, v1);
#pragma unroll
  for (int k = 0; k < 4; ++k) ldsm_x4_t(kbase + rofs + f.kt[k], kt[k]);
  if (has_q) {
#pragma unroll
    for (int k = 0; k < 4; ++k) ldsm_x4(qbase + rofs + f.ka[k], qa[k]);
  }
  // W as B fragments: movmatrix.trans turns the accumulator layout (key rows, column pairs)
  // into (key pairs, column) per 8x8 block.
  uint32_t wb[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    wb[k][0] = movm_t(pack_bf16(acc[k][0], acc[k][1]));
    wb[k][1] = movm_t(pack_bf16(acc[k][2], acc[k][3]));
  }
  float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f}, o[4] = {0.f, 0.f, 0.f, 0.f};
  mma_n8(pa, ka[0], wb[0][0], wb[0][1]);
  mma_n8(pb, ka[1], wb[1][0], wb[1][1]);
  mma_n8(pa, ka[2], wb[2][0], wb[2][1]);
  mma_n8(pb, ka[3], wb[3][0], wb[3][1]);
  if (has_q) {
#pragma unroll
    for (int k = 0; k < 4; ++k) mma_n8(o, qa[k], wb[k][0], wb[k][1]);
  }
  // R = P − V: p[e] = R[token g + 8(e>>1)][column 2q + (e&1)].
  const float2 va = unpack_bf16(v0), vb = unpack_bf16(v1);
  float p[4];
  p[0] = (pa[0] + pb[0]) - va.x;
  p[1] = (pa[1] + pb[1]) - va.y;
  p[2] = (pa[2] + pb[2]) - vb.x;
  p[3] = (pa[3] + pb[3]) - vb.y;
  // S = −(η/b)·R as B fragments (token pairs, column).
  const uint32_t sb0 = movm_t(pack_bf16(-beta * p[0], -beta * p[1]));
  const uint32_t sb1 = movm_t(pack_bf16(-beta * p[2], -beta * p[3]));
#pragma unroll
  for (int k = 0; k < 4; ++k) mma_n8(acc[k], kt[k], sb0, sb1);

  if (want_loss) {
    float l0 = p[0] * p[0] + p[1] * p[1];
    float l1 = p[2] * p[2] + p[3] * p[3];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if ((lane & 3) == 0) {
      lossp[r0 + g] = l0;
      lossp[r0 + g + 8] = l1;
    }
  }
  if (has_q) stsm_x2(obase + (uint32_t)r0 * 64u + f.o, pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
}

struct __align__(1024) N8Smem {
  uint8_t K[kStages][kTileBytes];
  uint8_t V[kStages][kTileBytes];
  uint8_t Q[kStages][kTileBytes];
  uint8_t O[2][kTileTok * 64];  // this CTA's 32 output columns of a tile (64-byte swizzle)
  float lossp[kComputeWarps][kTileTok];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort;
  int cabort[2];
};

__global__ void __launch_bounds__(kThreads, 1)
    k_linear_n8(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                float* __restrict__ Wstate, float* __restrict__ loss, int T, float beta, int has_q, int* status) {
  extern __shared__ uint8_t smem_raw[];
  N8Smem& sm = *reinterpret_cast<N8Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x >> 1, half = blockIdx.x & 1;
  const int nstages = (T + kTileTok - 1) / kTileTok;
  const uint32_t stage_bytes = (has_q ? 3u : 2u) * kTileBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kComputeWarps);
    }
    sm.abort = 0;
    sm.cabort[0] = sm.cabort[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
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
      for (int s = issued - kStages; s < issued; ++s) {
        if (s < 0) continue;
        mbar_wait(&sm.full[s % kStages], (s / kStages) & 1, status, nullptr);
      }
    }
    __syncthreads();
    return;
  }

  const int g = lane >> 2, q = lane & 3;
  const int col0 = 32 * half + 8 * warp;  // first W column owned by this warp
  float* Wg = Wstate + (size_t)bh * 64 * 64;
  float acc[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = Wg[(16 * mt + g + 8 * (e >> 1)) * 64 + col0 + 2 * q + (e & 1)];
  const N8Offsets offs = n8_offsets(lane, col0, warp);

  for (int s = 0; s < nstages; ++s) {
    const int slot = s % kStages;
    // Every compute warp takes the same exit decision (see k_linear_scan).
    if (!mbar_wait(&sm.full[slot], (s / kStages) & 1, status, nullptr)) sm.cabort[s & 1] = 1;
    named_sync();
    if (*reinterpret_cast<volatile int*>(&sm.cabort[s & 1])) break;
    const int ntok = min(kTileTok, T - s * kTileTok);
    const uint32_t kbase = smem_u32(sm.K[slot]), vbase = smem_u32(sm.V[slot]), qbase = smem_u32(sm.Q[slot]);
    uint8_t* obuf = sm.O[s & 1];
    for (int r0 = 0; r0 < ntok; r0 += 16)
      step16_n8(acc, kbase, vbase, qbase, smem_u32(obuf), offs, sm.lossp[warp], r0, lane, beta, has_q,
                loss != nullptr);
    if (has_q) fence_proxy_async_smem();
    named_sync();
    if (loss != nullptr && warp == 0) {
      for (int i = lane; i < ntok; i += 32) {
        const float l = (sm.lossp[0][i] + sm.lossp[1][i]) + (sm.lossp[2][i] + sm.lossp[3][i]);
        atomicAdd(&loss[(size_t)bh * T + (size_t)s * kTileTok + i], l);
      }
    }
    if (threadIdx.x == 0 && has_q) {
      tma_store_3d(&tmO, obuf, 32 * half, s * kTileTok, bh);
      bulk_commit();
      bulk_wait_read<1>();
    }
    named_sync();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
  }
  if (threadIdx.x == 0 && has_q) bulk_wait<0>();
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) Wg[(16 * mt + g + 8 * (e >> 1)) * 64 + col0 + 2 * q + (e & 1)] = acc[mt][e];
  __syncthreads();
}

template <int B>
ttt_status launch(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                  const CUtensorMap& to, float* loss, int T, int has_q, cudaStream_t s) {
  const size_t smem = sizeof(LinearSmem) + 1024;
  TTT_CUDA(cudaFuncSetAttribute(k_linear_scan<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int grid = st->cfg.batch * st->cfg.heads;
  const float beta = st->cfg.eta / (float)B;
  k_linear_scan<B><<<grid, kThreads, smem, s>>>(tk, tv, tq, to, st->lin.W, loss, T, beta, has_q, st->status.dev);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

template <bool HAS_Q, bool LOSS>
ttt_status launch_b16_impl(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                           const CUtensorMap& to, float* loss, int T, cudaStream_t s) {
  const size_t smem = sizeof(B16Smem) + 1024;
  TTT_CUDA(cudaFuncSetAttribute(k_linear_b16<HAS_Q, LOSS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int grid = st->cfg.batch * st->cfg.heads;
  const float beta = st->cfg.eta / 16.0f;
  k_linear_b16<HAS_Q, LOSS><<<grid, kB16Threads, smem, s>>>(tk, tv, tq, to, st->lin.W, loss, T, beta, st->status.dev);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

ttt_status launch_b16(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                      const CUtensorMap& to, float* loss, int T, int has_q, cudaStream_t s) {
  if (has_q) return loss ? launch_b16_impl<true, true>(st, tk, tv, tq, to, loss, T, s)
                         : launch_b16_impl<true, false>(st, tk, tv, tq, to, loss, T, s);
  return loss ? launch_b16_impl<false, true>(st, tk, tv, tq, to, loss, T, s)
              : launch_b16_impl<false, false>(st, tk, tv, tq, to, loss, T, s);
}

ttt_status launch_n8(ttt_state* st, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                     const CUtensorMap& to, float* loss, int T, int has_q, cudaStream_t s) {
  const size_t smem = sizeof(N8Smem) + 1024;
  TTT_CUDA(cudaFuncSetAttribute(k_linear_n8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int bh = st->cfg.batch * st->cfg.heads;
  if (loss != nullptr) TTT_CUDA(cudaMemsetAsync(loss, 0, (size_t)bh * T * sizeof(float), s));
  const float beta = st->cfg.eta / 16.0f;
  k_linear_n8<<<2 * bh, kThreads, smem, s>>>(tk, tv, tq, to, st->lin.W, loss, T, beta, has_q, st->status.dev);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}
}  // namespace

ttt_status linear_scan(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                       int64_t T, __nv_bfloat16* O, float* loss, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const uint64_t BH = (uint64_t)c.batch * c.heads;
  const uint64_t dims[3] = {64, (uint64_t)T, BH};
  const uint64_t strides[2] = {128, (uint64_t)T * 128};
  const uint32_t box[3] = {64, (uint32_t)kTileTok, 1};
  CUtensorMap tk, tv, tq, to;
  // b = 16: eight columns per warp on two CTAs per head when every half-head gets its own SM;
  // otherwise sixteen columns per warp on one CTA per head (fewer, fuller SMs win then).
  const bool n8 = c.chunk == 16 && 2 * (int64_t)c.batch * c.heads <= st->num_sms;
  TTT_TRY(encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
  TTT_TRY(encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
  const int has_q = Q != nullptr;
  if (has_q) {
    TTT_TRY(encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    if (n8) {
      const uint32_t obox[3] = {32, (uint32_t)kTileTok, 1};
      TTT_TRY(encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, O, dims, strides, obox, CU_TENSOR_MAP_SWIZZLE_64B));
    } else {
      TTT_TRY(encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, O, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    }
  } else {
    tq = tk;
    to = tk;
  }
  switch (c.chunk) {
    case 16: return n8 ? launch_n8(st, tk, tv, tq, to, loss, (int)T, has_q, s)
                       : launch_b16(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    case 32: return launch<32>(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    case 64: return launch<64>(st, tk, tv, tq, to, loss, (int)T, has_q, s);
    default: return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear: mini-batch %d not built", c.chunk);
  }
}

}  // namespace ttt
