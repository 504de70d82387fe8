// In-Place TTT scan on the 5th-generation tensor cores (tcgen05, bf16 in, fp32 accumulate in
// TMEM), for Wdown states too large to stay on chip (d_model 2560 x d_ff 9728 = 99.6 MB fp32).
//
// "In-Place Test-Time Training", §3: chunk c is first applied with the weight from before
// the chunk, O_c = Z_c·W_cᵀ, then the weight is updated from the same chunk (§2),
// W_{c+1} = W_c + η·V̂_cᵀ·Z_c; with fused target generation (§4) V̂ = Conv1D(X0)·Wtarget.
//
// Design (B200):
//  * one persistent, cooperative launch per scan call, one CTA per SM; every chunk is a round
//    in which each CTA works through a tile list of a static schedule computed on the host
//    by longest-processing-time-first, mixing three GEMM tile types of 128x256 outputs:
//      APPLY  O_c tile   = Z_c[128 tok, f] · W_cᵀ            A, B K-major        → bf16 O
//      UPDATE ΔW tile    = V̂_c[:, 128 rows]ᵀ · Z_c[:, 256]   A, B MN-major (K = tokens)
//                          epilogue W += η·ΔW (fp32 read-modify-write) and writes the bf16
//                          copy of W_{c+1} used by the next chunk's APPLY tiles
//      TARGET V̂_{c+1} tile = conv(X0)_{c+1}[128 tok, d] · Wtarget[:, 256]  A K-major, B MN-major
//    The bf16 copy of W rotates through three buffers: chunk c applies with one, its update
//    writes the next, and the third is what chunk c − 1 applied with, so APPLY and UPDATE
//    tiles of neighbouring chunks overlap. Where a tile needs another CTA's work of an earlier
//    chunk, it waits (bounded) on a progress counter per chunk and 256-row block of W: an APPLY
//    tile on the previous chunk's UPDATE tiles of its block, an UPDATE tile on the APPLY
//    tiles of two chunks back (their buffer is the one it overwrites), the W loader on the
//    previous chunk's update of its tile, and with the fused target an UPDATE tile on the
//    previous chunk's TARGET tiles and a TARGET tile on the UPDATE tiles of two chunks back,
//    which read the target buffer it overwrites (targets rotate through three buffers, and
//    TARGET tiles come first in each list). Every wait refers to an earlier chunk, so the CTA
//    furthest behind can always proceed. In round r CTA i runs list (i + 73r) mod 148: the
//    lists' different loads even out over the rounds. The compute-bound APPLY tiles and the HBM-bound UPDATE
//    epilogues overlap on different SMs.
//  * per CTA: warp 0 issues TMA loads (128-byte swizzle) into a 3-stage shared-memory ring,
//    warp 1 allocates 512 TMEM columns and one lane issues tcgen05.mma (M=128, N=256, K=16)
//    into one of two TMEM accumulators, warps 2..9 drain the other accumulator
//    (tcgen05.ld 32x32b) in the epilogue, two warps per TMEM lane quarter, and warp 10
//    streams the fp32 W of UPDATE tiles by TMA into a 3-slot ring of 128x32 sub-tiles while
//    the mainloop runs; warp 11 waits on the progress counters of the tiles ahead (up to
//    four), so the loads of a tile whose inputs are ready start without a round trip to L2.
//    The epilogue adds η·ΔW in shared memory, writes the bf16 copy beside
//    it, and two TMA stores per sub-tile write both back: the read-modify-write of the 99.6 MB
//    state never goes through per-thread global loads.
//  * SM pairs: where the chunk and d_model are multiples of 256 the kernel runs as clusters
//    of two CTAs on neighbouring SMs, each tile 256 rows x 256 columns. Each CTA loads by TMA
//    its own 128 rows of A and its own 128 columns of B (32 KB a k-block instead of 48 KB
//    for the same MMA work per SM, in a 5-stage ring); both CTAs' loads of a stage complete
//    on the first CTA's barrier, which expects the bytes of both, and one lane of the first
//    issues tcgen05.mma with cta_group::2 (M = 256, N = 256), whose commits arrive on the
//    barriers of both CTAs.
//    Each CTA's TMEM holds its own 128 rows of the accumulator, so the epilogue is the same
//    per CTA; the second CTA's epilogue warps release the accumulator on the first's barrier.
//    No load is multicast: every CTA reads its own operands.
//  * every wait is bounded (%globaltimer); a wait that runs out records TTT_ERR_TIMEOUT in the
//    state's status word, the CTA drains its in-flight copies and MMAs (bounded), frees TMEM
//    and returns.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kSt = 3;                      // operand ring depth (k-blocks)
constexpr int kABytes = BM * BK * 2;        // 16 KB
constexpr int kBBytes = BN * BK * 2;        // 32 KB
constexpr int kTileP = 2 * BM;              // rows of an SM-pair tile
constexpr int kStP = 5;                     // operand ring depth of an SM pair (32 KB stages)
constexpr int kStMax = 5;
constexpr int kRingBytes = kStP * (kABytes + kBBytes / 2);
static_assert(kSt * (kABytes + kBBytes) <= kRingBytes, "single-SM stages exceed the operand ring");
constexpr int kWCols = 32;                  // columns of one W sub-tile of an UPDATE tile
constexpr int kWBytes = BM * kWCols * 4;    // 16 KB of fp32 W
constexpr int kShBytes = BM * kWCols * 2;   // 8 KB of its bf16 copy
constexpr int kWSlots = 3;                  // W sub-tile ring depth
constexpr int kEpiWarps = 8;
constexpr int kWarpWload = 2 + kEpiWarps;   // the warp that streams W sub-tiles in
constexpr int kWarpDeps = 3 + kEpiWarps;    // the warp that waits for other CTAs' progress
constexpr int kThreadsTC = (4 + kEpiWarps) * 32;
constexpr int kDepSlots = 4;                // tiles whose dependencies may be cleared ahead of the loads
constexpr int kTmemCols = 512;

enum : int { APPLY = 0, UPDATE = 1, TARGET = 2 };

__host__ __device__ constexpr int32_t tile_code(int type, int m, int n) { return (type << 28) | (m << 14) | n; }
__device__ __forceinline__ int tile_type(int32_t t) { return (t >> 28) & 3; }
__device__ __forceinline__ int tile_m(int32_t t) { return (t >> 14) & 0x3FFF; }
__device__ __forceinline__ int tile_n(int32_t t) { return t & 0x3FFF; }

struct __align__(1024) TCSmem {
  // Operand stages, each A (16 KB) followed by B (32 KB; 16 KB, this CTA's half, in an SM pair).
  uint8_t ring[kRingBytes];
  uint8_t Wr[kWSlots][kWBytes];  // fp32 W sub-tiles (128 rows x 32 columns, 128-byte swizzle)
  uint8_t Sh[2][kShBytes];       // bf16 copy of an updated sub-tile, one per column half (64-byte swizzle)
  uint64_t full[kStMax], empty[kStMax];
  uint64_t tfull[2], tempty[2];
  uint64_t wfull[kWSlots], wempty[kWSlots];
  uint64_t dep_ok[kDepSlots], dep_free[kDepSlots];
  uint32_t tmem_base;
  int abort;
  int cur0;         // the bf16 copy of W that round 0 applies with
  int eflag[2][2];  // per column half: a wait of sub-tile e ran out (index e & 1)
  int tflag[2][2];  // per column half: the accumulator wait of tile t ran out (index t & 1)
};

struct TCArgs {
  const int32_t* sched;  // [grid + 1] CTA offsets followed by the tile codes
  int chunk;             // chunk c of this launch (token offset c·C)
  int target_chunk;      // chunk whose targets the TARGET tiles produce
  int vrow0;             // first V̂ row of chunk c in the tensor map of V̂
  int d, f, C;
  float eta;
  __nv_bfloat16* O;            // outputs [T, d]
  __nv_bfloat16* Vhat_out;     // targets of target_chunk [C, d]
  DevStatus status;
  // Fault injection (tests): the APPLY tiles of this round wait for one more UPDATE than will
  // ever be counted, so that wait runs out; -1 = none.
  int stall_round;
  // Round r runs tile list (list + r·rotate) mod (number of lists); rotate is coprime to that
  // number, so over the rounds every CTA works through a mix of the lists.
  int rotate;
  // Several chunks in one launch: every CTA runs its tile list once per chunk (chunk index
  // chunk + r in round r). The bf16 copy of W rotates through three buffers: round r applies
  // with buffer (cur0 + r) % 3 and its UPDATE tiles write buffer (cur0 + r + 1) % 3, the one
  // round r − 2 applied with. upd_done[r·nbd + b] / app_done[r·nbd + b] count the finished
  // UPDATE / APPLY work of round r on 256-row block b of W; an APPLY tile of round r waits for
  // round r − 1's UPDATE tiles of its block, an UPDATE tile of round r for round r − 2's APPLY
  // tiles of its block. Null counters: one round, no waits.
  int rounds;
  // The bf16 copy round 0 applies with: ring[0] when ring is set, else cur0. With ring set the
  // last CTA to finish adds `advance` to ring[0] (mod 3) once every CTA has read it, counting
  // finished CTAs in ring[1] (left at 0 again), so no index lives on the host between calls.
  int cur0;
  int* ring;
  int advance;
  int nbd;
  int* upd_done;
  int* app_done;
  // Fused target over several chunks: the last round runs sched_last (no TARGET tiles); the
  // TARGET tiles of round r write V̂ of chunk chunk + r + 1 into vhat[(r + 1) % 3], which the
  // UPDATE tiles of round r + 1 read (the buffer they overwrite was read two rounds before);
  // tgt_done[r·nbd + b] counts round r's TARGET work on 256-column block b of V̂ (one per
  // epilogue warp and tile).
  const int32_t* sched_last;
  __nv_bfloat16* vhat[3];
  int* tgt_done;
};

// ---- tcgen05 wrappers -----------------------------------------------------------------

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;  // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, M = m, N = 256.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// PAIR: issued by the first CTA of an SM pair for both (cta_group::2); A and B are read from
// the same shared-memory offsets in both CTAs and D lands in both CTAs' TMEM.
template <bool PAIR>
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  if constexpr (PAIR) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// The mbarrier at this offset arrives once the MMAs issued before have completed; PAIR: the
// arrival goes to the barrier at the same offset in both CTAs of the pair (CTA mask 0b11).
template <bool PAIR>
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  if constexpr (PAIR) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
  } else {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
  }
}

// TMEM allocation by one warp; PAIR: by one warp in each CTA of the pair, same columns in both.
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  if constexpr (PAIR) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
}

template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  if constexpr (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
}

// ---- thread-block clusters (SM pairs) ----------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of both CTAs; what each wrote before is visible to the other after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of this CTA's shared-memory object `p` in the first CTA of the cluster.
__device__ __forceinline__ uint32_t in_first_cta(const void* p) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(a) : "r"(smem_u32(p)));
  return a;
}

// Arrive on the mbarrier at shared::cluster address `addr` (in the other CTA of the pair),
// relaxed: it orders nothing before it. It signals that this thread's tcgen05.ld reads of TMEM
// have finished (tcgen05.wait::ld before it), not writes made visible by it. A release at
// cluster scope would wait for every memory operation the thread has in flight (its output
// stores): measured on B200, a release arrive took ~1400 cycles.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ int kblocks(int type, const TCArgs& a) {
  if (type == APPLY) return (a.f + BK - 1) / BK;
  if (type == UPDATE) return a.C / BK;
  return (a.d + BK - 1) / BK;
}

// Stores 32 consecutive bf16 values of one row (cols col0 .. col0+31, clipped to ncols).
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* row, int col0, int ncols, const float* v) {
  if (col0 + 32 <= ncols) {
    uint4* dst = reinterpret_cast<uint4*>(row + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
      dst[q] = w;
    }
  } else {
    for (int j = 0; j < 32 && col0 + j < ncols; ++j) row[col0 + j] = __float2bfloat16_rn(v[j]);
  }
}

__device__ __forceinline__ const CUtensorMap* pick3(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                                                    int i) {
  return i == 0 ? &a : (i == 1 ? &b : &c);
}

// TMA load of a box into this CTA's shared memory, completing on the mbarrier at shared::cluster
// address `bar`; PAIR: the barrier may be in the other CTA of the pair (cta_group::2 form).
template <bool PAIR>
__device__ __forceinline__ void tma_load_2d_to(void* dst, const CUtensorMap* map, uint32_t bar, int32_t c0, int32_t c1) {
  if constexpr (PAIR) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
  }
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *ctr ≥ want (a counter other CTAs raise); then the async proxy (TMA) may
// read what they published.
__device__ __forceinline__ bool wait_counter(const int* ctr, int want, const DevStatus& status, volatile int* abort) {
  const volatile int* c = ctr;
  if (*c < want) {
    const uint64_t t0 = globaltimer();
    while (*c < want) {
      if (*abort) return false;
      if (globaltimer() - t0 > status.limit_ns) {
        record_status(status, kDevTimeout, kSiteCounter | (int)((reinterpret_cast<uintptr_t>(ctr) >> 2) & 0xFFFFu));
        *abort = 1;
        return false;
      }
      __nanosleep(128);
    }
  }
  __threadfence();
  fence_proxy_async_global();
  return true;
}

// Work expected on 256-row block b of W per round: UPDATE halves (two 128-row tiles per block,
// fewer at the edge, times the f tiles, two column halves each) and APPLY tiles (C/128).
__device__ __forceinline__ int upd_expect(const TCArgs& a, int b) {
  const int mt = (a.d + BM - 1) / BM, nf = (a.f + BN - 1) / BN;
  return (min(2 * b + 2, mt) - 2 * b) * nf * 2;
}

__device__ __forceinline__ void named_sync_half(int half) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + half), "n"(4 * 32) : "memory");
}

// PAIR = false: one CTA per tile of 128 x 256 outputs. PAIR = true: clusters of two CTAs, one
// tile of 256 x 256 outputs per cluster, 128 rows per CTA (see the file comment).
template <bool PAIR>
__global__ void __launch_bounds__(kThreadsTC, 1)
    k_inplace_tc(const __grid_constant__ CUtensorMap tmZk, const __grid_constant__ CUtensorMap tmZm,
                 const __grid_constant__ CUtensorMap tmVm, const __grid_constant__ CUtensorMap tmVm1,
                 const __grid_constant__ CUtensorMap tmVm2,
                 const __grid_constant__ CUtensorMap tmWk0,
                 const __grid_constant__ CUtensorMap tmWk1, const __grid_constant__ CUtensorMap tmWk2,
                 const __grid_constant__ CUtensorMap tmConv, const __grid_constant__ CUtensorMap tmWt,
                 const __grid_constant__ CUtensorMap tmWf, const __grid_constant__ CUtensorMap tmWs0,
                 const __grid_constant__ CUtensorMap tmWs1, const __grid_constant__ CUtensorMap tmWs2,
                 const TCArgs args) {
  constexpr int kStages = PAIR ? kStP : kSt;
  constexpr int kBCols = PAIR ? BN / 2 : BN;         // B columns (N) this CTA loads
  constexpr int kStage = kABytes + kBCols * BK * 2;  // bytes of one stage of this CTA
  extern __shared__ uint8_t smem_raw[];
  TCSmem& sm = *reinterpret_cast<TCSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = PAIR ? (int)cluster_rank() : 0;  // 0: the CTA that issues the MMAs
  const int nlists = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
  const int list_id = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x;
  // In round r the CTA (pair) runs tile list (list_id + r·rotate) mod nlists: over the rounds
  // every CTA works through a mix of the lists, so their different loads even out instead of
  // adding up round after round.
  auto list_of = [&](int rnd) { return (int)(((long)list_id + (long)rnd * args.rotate) % nlists); };
  auto sched_of = [&](int rnd) {
    return (args.sched_last != nullptr && rnd == args.rounds - 1) ? args.sched_last : args.sched;
  };
  // First row of this CTA's 128 rows of tile row-block m (tokens for APPLY and TARGET tiles,
  // rows of W for UPDATE tiles), and the 256-row block of W that an UPDATE tile lies in.
  auto row0_of = [&](int m) { return PAIR ? m * kTileP + rank * BM : m * BM; };
  auto wblock_of = [&](int m) { return PAIR ? m : m / 2; };
  int ntot = 0;  // tiles of this CTA over all rounds
  for (int rnd = 0; rnd < args.rounds; ++rnd) ntot += sched_of(rnd)[list_of(rnd) + 1] - sched_of(rnd)[list_of(rnd)];
  // Walks the CTA's tiles in order: calls f(round, tile code) until it returns false.
  auto for_tiles = [&](auto&& f) {
    for (int rnd = 0; rnd < args.rounds; ++rnd) {
      const int32_t* sch = sched_of(rnd);
      const int li = list_of(rnd);
      const int32_t* tl = sch + nlists + 1;
      for (int ti = sch[li]; ti < sch[li + 1]; ++ti)
        if (!f(rnd, tl[ti])) return;
    }
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.tfull[i], 1);
      // PAIR: the epilogue warps of both CTAs release an accumulator on the first CTA's barrier.
      mbar_init(&sm.tempty[i], PAIR ? 2 * kEpiWarps : kEpiWarps);
    }
    for (int i = 0; i < kWSlots; ++i) {
      mbar_init(&sm.wfull[i], 1);
      mbar_init(&sm.wempty[i], 1);
    }
    for (int i = 0; i < kDepSlots; ++i) {
      mbar_init(&sm.dep_ok[i], 1);
      mbar_init(&sm.dep_free[i], 1);
    }
    sm.abort = 0;
    sm.cur0 = args.ring != nullptr ? __ldcg(args.ring) : args.cur0;
    sm.eflag[0][0] = sm.eflag[0][1] = sm.eflag[1][0] = sm.eflag[1][1] = 0;
    sm.tflag[0][0] = sm.tflag[0][1] = sm.tflag[1][0] = sm.tflag[1][1] = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<PAIR>(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers exist before either arrives remotely
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmZk);
      tma_prefetch_desc(&tmZm);
      tma_prefetch_desc(&tmVm);
      tma_prefetch_desc(&tmWk0);
      uint32_t it = 0, dep_u = 0;
      for_tiles([&](int rnd, int32_t tc) -> bool {
        if (*abort) return false;
        const int type = tile_type(tc), m = tile_m(tc), n = tile_n(tc);
        const int nk = kblocks(type, args);
        const int chunk = args.chunk + rnd;
        const int r0 = row0_of(m);
        const int b0 = n * BN + rank * (BN / 2);  // first B column (N) this CTA loads
        const CUtensorMap* wk = pick3(tmWk0, tmWk1, tmWk2, (sm.cur0 + rnd) % 3);
        if (args.upd_done != nullptr) {
          // The dependency warp has seen this tile's inputs published by other CTAs.
          const int slot = (int)(dep_u % kDepSlots);
          if (!mbar_wait(&sm.dep_ok[slot], (dep_u / kDepSlots) & 1, args.status, abort)) return false;
          fence_proxy_async_global();  // TMA reads after that point see what the counters published
          mbar_arrive(&sm.dep_free[slot]);
          ++dep_u;
        }
        const CUtensorMap* vm = args.tgt_done != nullptr ? pick3(tmVm, tmVm1, tmVm2, rnd % 3) : &tmVm;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= (uint32_t)kStages && !mbar_wait(&sm.empty[s], ((it / kStages) - 1) & 1, args.status, abort))
            return false;
          uint8_t* sa = sm.ring + s * kStage;
          uint8_t* sb = sa + kABytes;
          // SM pair: the loads of both CTAs complete on the first CTA's barrier, which expects
          // the bytes of both (a load may complete before the expectation is posted: the phase
          // cannot end before it is).
          if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], PAIR ? 2 * kStage : kStage);
          const uint32_t fb = PAIR ? in_first_cta(&sm.full[s]) : smem_u32(&sm.full[s]);
          if (type == APPLY) {
            tma_load_2d_to<PAIR>(sa, &tmZk, fb, kb * BK, chunk * args.C + r0);
            tma_load_2d_to<PAIR>(sb, wk, fb, kb * BK, b0);
          } else if (type == UPDATE) {
            for (int j = 0; j < BM / 64; ++j)
              tma_load_2d_to<PAIR>(sa + j * 8192, vm, fb, r0 + j * 64,
                                   args.vrow0 + (args.tgt_done != nullptr ? 0 : rnd * args.C) + kb * BK);
            for (int j = 0; j < kBCols / 64; ++j)
              tma_load_2d_to<PAIR>(sb + j * 8192, &tmZm, fb, b0 + j * 64, chunk * args.C + kb * BK);
          } else {
            tma_load_2d_to<PAIR>(sa, &tmConv, fb, kb * BK, (args.target_chunk + rnd) * args.C + r0);
            for (int j = 0; j < kBCols / 64; ++j)
              tma_load_2d_to<PAIR>(sb + j * 8192, &tmWt, fb, b0 + j * 64, kb * BK);
          }
        }
        return true;
      });
      // Drain: nothing may still land in this CTA's shared memory when it exits.
      const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0;
      if constexpr (!PAIR) {
        for (uint32_t k = first; k < it; ++k)
          mbar_wait(&sm.full[k % kStages], (k / kStages) & 1, args.status, nullptr);
      } else if (!*abort) {
        // Every stage was consumed by MMAs that waited for both CTAs' bytes; the commits that
        // released the last stages arrive on this CTA's barriers too: wait for them.
        for (uint32_t k = first; k < it; ++k)
          mbar_wait(&sm.empty[k % kStages], (k / kStages) & 1, args.status, nullptr);
      } else {
        // After an abort a stage may never complete on the first CTA's barrier (its partner's
        // half missing), so no barrier tells when this CTA's last loads have landed: wait
        // 50 us, far beyond the latency of a TMA load, before the CTA may exit.
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 50000) __nanosleep(1000);
      }
    }
  } else if (warp == kWarpDeps) {
    // ------------- dependencies: waits on other CTAs' progress, ahead of the loads -------------
    // A counter read is an L2 round trip and its fences more; measured on B200, taken in the
    // producer's path they held up the first k-blocks of every UPDATE tile. Here they run up
    // to kDepSlots tiles ahead, and the producer only waits on a shared-memory barrier.
    if (lane == 0 && args.upd_done != nullptr) {
      uint32_t u = 0;
      for_tiles([&](int rnd, int32_t tc) -> bool {
        if (*abort) return false;
        const int type = tile_type(tc), m = tile_m(tc), n = tile_n(tc);
        const int wb = wblock_of(m);
        const int slot = (int)(u % kDepSlots);
        if (u >= (uint32_t)kDepSlots && !mbar_wait(&sm.dep_free[slot], ((u / kDepSlots) - 1) & 1, args.status, abort))
          return false;
        {
          if (type == APPLY && rnd >= 1 &&
              !wait_counter(&args.upd_done[(rnd - 1) * args.nbd + n],
                            upd_expect(args, n) + (rnd == args.stall_round ? 1 : 0), args.status, abort))
            return false;
          if (type == UPDATE && rnd >= 2 &&
              !wait_counter(&args.app_done[(rnd - 2) * args.nbd + wb], args.C / BM, args.status, abort))
            return false;
          if (args.tgt_done != nullptr) {
            // V̂ of this round was produced by the previous round's TARGET tiles; a TARGET tile
            // overwrites the V̂ buffer the previous round's UPDATE tiles of its block read.
            if (type == UPDATE && rnd >= 1 &&
                !wait_counter(&args.tgt_done[(rnd - 1) * args.nbd + wb], kEpiWarps * (args.C / BM), args.status,
                              abort))
              return false;
            if (type == TARGET && rnd >= 2 &&
                !wait_counter(&args.upd_done[(rnd - 2) * args.nbd + n], upd_expect(args, n), args.status, abort))
              return false;
          }
        }
        mbar_arrive(&sm.dep_ok[slot]);
        ++u;
        return true;
      });
    }
  } else if (warp == kWarpWload) {
    // ---------------- W sub-tile loader (fp32 W of UPDATE tiles, 128 x 32) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmWf);
      uint32_t e = 0;
      for_tiles([&](int rnd, int32_t tc) -> bool {
        if (*abort) return false;
        if (tile_type(tc) != UPDATE) return true;
        const int m = tile_m(tc), n = tile_n(tc);
        const int r0 = row0_of(m), wb = wblock_of(m);
        // The round before updated this W tile, possibly on another CTA.
        if (args.upd_done != nullptr && rnd >= 1 &&
            !wait_counter(&args.upd_done[(rnd - 1) * args.nbd + wb], upd_expect(args, wb), args.status, abort))
          return false;
        bool ok = true;
        for (int k = 0; k < BN / kWCols; ++k, ++e) {
          const int s = e % kWSlots;
          if (e >= (uint32_t)kWSlots && !mbar_wait(&sm.wempty[s], ((e / kWSlots) - 1) & 1, args.status, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.wfull[s], kWBytes);
          tma_load_2d(sm.Wr[s], &tmWf, &sm.wfull[s], n * BN + (k & 1) * 128 + (k >> 1) * kWCols, r0);
        }
        return ok;
      });
      for (uint32_t k = (e > (uint32_t)kWSlots ? e - kWSlots : 0); k < e; ++k)
        mbar_wait(&sm.wfull[k % kWSlots], (k / kWSlots) & 1, args.status, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------- MMA issuer -------------------------------
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for_tiles([&](int, int32_t tc) -> bool {
        const int type = tile_type(tc);
        const int nk = kblocks(type, args);
        const int acc = tcount & 1;
        if (tcount >= 2 && !mbar_wait<PAIR>(&sm.tempty[acc], ((tcount >> 1) - 1) & 1, args.status, abort)) {
          ok = false;
          return false;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        constexpr int kM = PAIR ? kTileP : BM;
        const uint32_t idesc = type == APPLY    ? idesc_bf16(kM, 0, 0)
                               : type == UPDATE ? idesc_bf16(kM, 1, 1)
                                                : idesc_bf16(kM, 0, 1);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait<PAIR>(&sm.full[s], (it / kStages) & 1, args.status, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.ring + s * kStage), b0 = a0 + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            uint64_t ad, bd;
            if (type == UPDATE) {
              ad = umma_desc(a0 + kk * 2048, 8192, 1024);
              bd = umma_desc(b0 + kk * 2048, 8192, 1024);
            } else {
              ad = umma_desc(a0 + kk * 32, 16, 1024);
              bd = type == APPLY ? umma_desc(b0 + kk * 32, 16, 1024) : umma_desc(b0 + kk * 2048, 8192, 1024);
            }
            umma<PAIR>(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          umma_commit<PAIR>(&sm.empty[s]);  // frees the stage (of both CTAs) once these MMAs have read it
        }
        if (!ok) return false;
        umma_commit<PAIR>(&sm.tfull[acc]);  // accumulator ready for the epilogue (of both CTAs)
        ++tcount;
        return true;
      });
      // Drain: the last commit covers every MMA issued before it; wait for it before TMEM
      // is freed. After a clean run that is the last accumulator's commit, after an abort
      // the last stage-release commit.
      if (ok && ntot > 0) {
        const uint32_t last = (uint32_t)(ntot - 1);
        mbar_wait(&sm.tfull[last & 1], (last >> 1) & 1, args.status, nullptr);
      } else if (!ok && it > 0) {
        mbar_wait(&sm.empty[(it - 1) % kStages], ((it - 1) / kStages) & 1, args.status, nullptr);
      }
    }
  } else {
    // ------------------------------- epilogue (8 warps) -------------------------------
    const int lq = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;     // which 128 columns of the 256-wide tile
    const bool leader = lq == 0 && lane == 0;  // issues this half's TMA stores
    uint32_t tcount = 0, ecount = 0;      // tiles seen; W sub-tiles consumed by this half
    const int row_in_tile = lq * 32 + lane;
    bool stop = false;
    for_tiles([&](int rnd, int32_t tc) -> bool {
      const int type = tile_type(tc), m = tile_m(tc), n = tile_n(tc);
      const int r0 = row0_of(m);
      const CUtensorMap* ws = pick3(tmWs0, tmWs1, tmWs2, (sm.cur0 + rnd + 1) % 3);
      const int acc = tcount & 1;
      bool ok = mbar_wait(&sm.tfull[acc], (tcount >> 1) & 1, args.status, nullptr);
      ok = __all_sync(0xffffffffu, ok);
      // The four warps of a column half share named barriers, so they leave together: the
      // flag of tile t is written only before this barrier and read only after it.
      if (!ok && lane == 0) sm.tflag[half][tcount & 1] = 1;
      named_sync_half(half);
      if (*reinterpret_cast<volatile int*>(&sm.tflag[half][tcount & 1])) return false;
      tc_fence_after();
      // The accumulator is complete, so every operand of this tile has been read: an APPLY
      // tile no longer needs its buffer of the bf16 copy of W.
      if (type == APPLY && args.app_done != nullptr && warp == 2 && lane == 0) {
        __threadfence();
        atomicAdd(&args.app_done[rnd * args.nbd + n], 1);
      }
      const uint32_t tbase = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(acc * BN + half * 128);
      if (type == UPDATE) {
        // W sub-tiles arrive in smem by TMA; W ← W + η·ΔW in place, the bf16 copy beside it,
        // and both go back to global memory by TMA stores issued by the half's leader.
#pragma unroll 1
        for (int j = 0; j < 4; ++j, ++ecount) {
          const uint32_t e = 8u * (ecount >> 2) + 2u * (uint32_t)j + (uint32_t)half;  // ring entry
          const int slot = e % kWSlots;
          bool okw = mbar_wait(&sm.wfull[slot], (e / kWSlots) & 1, args.status, nullptr);
          okw = __all_sync(0xffffffffu, okw);
          if (okw) {
            uint32_t r[32];
            tmem_ld32(tbase + j * kWCols, r);
            tmem_wait_ld();
            uint8_t* wrow = sm.Wr[slot] + row_in_tile * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float4* p = reinterpret_cast<float4*>(wrow + ((c ^ (row_in_tile & 7)) << 4));
              float4 w = *p;
              w.x = fmaf(args.eta, __uint_as_float(r[4 * c + 0]), w.x);
              w.y = fmaf(args.eta, __uint_as_float(r[4 * c + 1]), w.y);
              w.z = fmaf(args.eta, __uint_as_float(r[4 * c + 2]), w.z);
              w.w = fmaf(args.eta, __uint_as_float(r[4 * c + 3]), w.w);
              *p = w;
              r[4 * c + 0] = __float_as_uint(w.x);
              r[4 * c + 1] = __float_as_uint(w.y);
              r[4 * c + 2] = __float_as_uint(w.z);
              r[4 * c + 3] = __float_as_uint(w.w);
            }
            uint8_t* srow = sm.Sh[half] + row_in_tile * 64;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(r[8 * c + 0]), __uint_as_float(r[8 * c + 1]));
              v.y = pack_bf16(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3]));
              v.z = pack_bf16(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5]));
              v.w = pack_bf16(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7]));
              *reinterpret_cast<uint4*>(srow + ((c ^ ((row_in_tile >> 1) & 3)) << 4)) = v;
            }
            fence_proxy_async_smem();
          } else if (lane == 0) {
            sm.eflag[half][ecount & 1] = 1;
          }
          named_sync_half(half);
          // Every warp of the half takes the same decision: the flag of this sub-tile is only
          // written before the barrier above and only read after it.
          if (*reinterpret_cast<volatile int*>(&sm.eflag[half][ecount & 1])) {
            stop = true;
            break;
          }
          if (leader) {
            const int col = n * BN + half * 128 + j * kWCols;
            tma_store_2d(&tmWf, sm.Wr[slot], col, r0);
            tma_store_2d(ws, sm.Sh[half], col, r0);
            bulk_commit();
            bulk_wait_read<0>();          // both stores have read shared memory
            mbar_arrive(&sm.wempty[slot]);
          }
          named_sync_half(half);          // the bf16 staging tile is free again
        }
        if (stop) return false;
        // The stores of this half of the tile complete, then later rounds may read them.
        if (leader && args.upd_done != nullptr) {
          bulk_wait<0>();
          fence_proxy_async_global();
          __threadfence();
          atomicAdd(&args.upd_done[rnd * args.nbd + wblock_of(m)], 1);
        }
      } else {
        const int row = r0 + row_in_tile;  // token within the chunk
#pragma unroll 1
        for (int jc = 0; jc < 4; ++jc) {
          const int col0 = n * BN + half * 128 + jc * 32;
          uint32_t r[32];
          tmem_ld32(tbase + jc * 32, r);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (type == APPLY)
            store_row_bf16(args.O + ((size_t)(args.chunk + rnd) * args.C + row) * args.d, col0, args.d, v);
          else
            store_row_bf16((args.tgt_done != nullptr ? args.vhat[(rnd + 1) % 3] : args.Vhat_out) + (size_t)row * args.d,
                           col0, args.d, v);
        }
        if (type == TARGET && args.tgt_done != nullptr) {
          __syncwarp();
          if (lane == 0) {
            __threadfence();
            atomicAdd(&args.tgt_done[rnd * args.nbd + n], 1);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && rank != 0)
          mbar_arrive_remote(in_first_cta(&sm.tempty[acc]));
        else
          mbar_arrive(&sm.tempty[acc]);
      }
      ++tcount;
      return true;
    });
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  // PAIR: neither CTA exits (or frees TMEM) while the other may still arrive on its barriers
  // or the MMAs may still write its TMEM.
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<PAIR>(tmem, kTmemCols);
  if (args.ring != nullptr && threadIdx.x == 0) {
    // This CTA read ring[0] before its first barrier.
    __threadfence();
    if (atomicAdd(args.ring + 1, 1) == (int)gridDim.x - 1) {
      args.ring[0] = (sm.cur0 + args.advance) % 3;
      args.ring[1] = 0;
    }
  }
}

// Depthwise future-tap convolution of X0 for the fused target:
// conv[t, i] = Σ_k w[i, k]·X0[t + k, i] over taps whose source t + k lies before the end of t's
// chunk (pad mode 0) or before T (pad mode 1); fp32 arithmetic, stored as bf16.
__global__ void k_target_conv(const __nv_bfloat16* __restrict__ X0, const float* __restrict__ w, __nv_bfloat16* __restrict__ out,
                              int T, int d, int C, int taps, int pad_mode) {
  const int pairs = d / 2;
  const size_t n = (size_t)T * pairs;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(idx / pairs);
    const int i = (int)(idx % pairs) * 2;
    const int end = pad_mode == 0 ? min(T, (t / C + 1) * C) : T;
    float a0 = 0.f, a1 = 0.f;
    for (int k = 0; k < taps && t + k < end; ++k) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(X0 + (size_t)(t + k) * d + i);
      const float2 xf = __bfloat1622float2(x);
      a0 = fmaf(w[i * taps + k], xf.x, a0);
      a1 = fmaf(w[(i + 1) * taps + k], xf.y, a1);
    }
    *reinterpret_cast<uint32_t*>(out + (size_t)t * d + i) = pack_bf16(a0, a1);
  }
}

// ---- host: schedules ------------------------------------------------------------------

struct Plan {
  std::vector<int32_t> host;  // [lists + 1] offsets, then tile codes
  int grid = 0;               // tile lists: CTAs, or SM pairs when tm = 256
};

// Tile lists for up to `lists` CTAs (tm = 128) or SM pairs (tm = 256, tiles of 256 rows).
Plan make_plan(int lists, int tm, int d, int f, int C, bool apply_update, bool target) {
  struct T {
    int32_t code;
    int cost;
  };
  std::vector<T> tl;
  const int mt_tok = C / tm, nt_d = (d + BN - 1) / BN;
  if (apply_update) {
    const int cost_apply = (f + BK - 1) / BK + 2;
    for (int m = 0; m < mt_tok; ++m)
      for (int n = 0; n < nt_d; ++n) tl.push_back({tile_code(APPLY, m, n), cost_apply});
  }
  if (target) {
    const int cost_t = (d + BK - 1) / BK + 2;
    for (int m = 0; m < mt_tok; ++m)
      for (int n = 0; n < nt_d; ++n) tl.push_back({tile_code(TARGET, m, n), cost_t});
  }
  if (apply_update) {
    // The read-modify-write epilogue (fp32 W in and out, bf16 copy out: 320 KB per tile)
    // costs more than the 16-deep mainloop; weigh it in.
    const int cost_u = std::max(C / BK, 20);
    for (int m = 0; m < (d + tm - 1) / tm; ++m)
      for (int n = 0; n < (f + BN - 1) / BN; ++n) tl.push_back({tile_code(UPDATE, m, n), cost_u});
  }
  const int grid = std::max(1, std::min<int>(lists, (int)tl.size()));
  std::stable_sort(tl.begin(), tl.end(), [](const T& a, const T& b) { return a.cost > b.cost; });
  std::vector<std::vector<int32_t>> per(grid);
  std::vector<long> load(grid, 0);
  for (const T& t : tl) {
    int best = 0;
    for (int i = 1; i < grid; ++i)
      if (load[i] < load[best]) best = i;
    per[best].push_back(t.code);
    load[best] += t.cost;
  }
  // Within each CTA: TARGET tiles first (the next chunk's UPDATE tiles, at the start of their
  // round, need them), then UPDATE tiles, and the long APPLY tile last: a round then ends on
  // an epilogue that only stores outputs rather than on a W read-modify-write, and the CTAs
  // holding an APPLY tile stream W while the others do too (measured on B200: 3.59 against
  // 3.68 ms on the T=32768 workload).
  auto rank = [](int32_t code) {
    const int t = (code >> 28) & 3;
    return t == TARGET ? 0 : (t == UPDATE ? 1 : 2);
  };
  for (auto& v : per)
    std::stable_sort(v.begin(), v.end(), [&](int32_t a, int32_t b) { return rank(a) < rank(b); });
  Plan p;
  p.grid = grid;
  p.host.resize(grid + 1);
  int off = 0;
  for (int i = 0; i < grid; ++i) {
    p.host[i] = off;
    off += (int)per[i].size();
  }
  p.host[grid] = off;
  for (int i = 0; i < grid; ++i) p.host.insert(p.host.end(), per[i].begin(), per[i].end());
  return p;
}

ttt_status upload_plan(const Plan& p, int32_t** dev) {
  TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(dev), p.host.size() * sizeof(int32_t)));
  TTT_CUDA(cudaMemcpy(*dev, p.host.data(), p.host.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
  return TTT_OK;
}

ttt_status map2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in, uint32_t box_out,
                 CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                 CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {inner * (dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4u : 2u)};
  const uint32_t box[2] = {box_in, box_out};
  return encode_tmap(m, dt, 2, base, dims, strides, box, sw);
}

static_assert(sizeof(TCSmem) + 1024 <= 232448, "k_inplace_tc exceeds the 227 KB of shared memory per block");

constexpr size_t kSmemTC = sizeof(TCSmem) + 1024;

// Rotation of the tile lists between rounds: the largest step up to half the list count that
// is coprime to it (73 for 148 lists, 35 for 74), so a CTA meets every list and consecutive
// rounds take lists far apart (measured on 148 lists: 73 against 1 and 61).
int list_rotation(int lists) {
  for (int r = lists / 2; r > 1; --r) {
    int a = lists, b = r;
    while (b) {
      const int t = a % b;
      a = b;
      b = t;
    }
    if (a == 1) return r;
  }
  return 1;
}

// Launches k_inplace_tc<pair> on `grid` CTAs (clusters of two when pair). Cooperative launches
// (several rounds whose CTAs wait on one another) check that every CTA is resident; a cluster
// launch is checked against the occupancy query when its lists are planned.
ttt_status launch_tc(bool pair, int grid, bool cooperative, void** params, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsTC);
  cfg.dynamicSmemBytes = kSmemTC;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  if (pair) {
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
  } else {
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = cooperative ? 1 : 0;
  }
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const void* fn = pair ? reinterpret_cast<const void*>(k_inplace_tc<true>) : reinterpret_cast<const void*>(k_inplace_tc<false>);
  TTT_CUDA(cudaLaunchKernelExC(&cfg, fn, params));
  return TTT_OK;
}

}  // namespace

// Per-state tensor-core resources (schedules, conv buffer), created on first use.
struct TCResources {
  int32_t* plan_dev[3] = {nullptr, nullptr, nullptr};  // 0: steady, 1: target only, 2: apply+update only
  int grid[3] = {0, 0, 0};   // CTAs of each plan's launch (two per list with SM pairs)
  int lists[3] = {0, 0, 0};
  bool pair = false;         // tiles of 256 rows on SM pairs
  __nv_bfloat16* conv = nullptr;
  size_t conv_rows = 0;
  int* counters = nullptr;  // per-round progress counters of a multi-chunk launch
  size_t counters_n = 0;
};

static ttt_status ensure_tc(ttt_state* st) {
  if (st->ip.tc != nullptr) return TTT_OK;
  const ttt_config& c = st->cfg;
  TCResources* r = new (std::nothrow) TCResources();
  if (r == nullptr) return fail(TTT_ERR_OOM, "host allocation failed");
  const bool target = c.target_mode == 1;
  ttt_status s = TTT_OK;
  // SM pairs where every tile has two full 128-row halves: the chunk and d_val multiples of 256.
  int lists = st->num_sms;
  r->pair = st->ip.sm_pair != 0 && c.chunk % kTileP == 0 && c.d_val % kTileP == 0;
  if (r->pair) {
    // As many pairs as can be resident at once (an SM left without a partner in its GPC idles).
    cudaError_t e = cudaFuncSetAttribute(k_inplace_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTC);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (st->num_sms / 2));
    cfg.blockDim = dim3(kThreadsTC);
    cfg.dynamicSmemBytes = kSmemTC;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&clusters, k_inplace_tc<true>, &cfg);
    if (e != cudaSuccess) {
      delete r;
      return fail(TTT_ERR_CUDA, "SM-pair occupancy query failed: %s", cudaGetErrorString(e));
    }
    lists = std::min(st->num_sms / 2, clusters);
    if (lists < 1) r->pair = false;
  }
  if (!r->pair) lists = st->num_sms;
  const int tm = r->pair ? kTileP : BM;
  const int per = r->pair ? 2 : 1;
  Plan p0 = make_plan(lists, tm, c.d_val, c.d_key, c.chunk, true, target);
  s = upload_plan(p0, &r->plan_dev[0]);
  r->lists[0] = p0.grid;
  if (s == TTT_OK && target) {
    Plan p1 = make_plan(lists, tm, c.d_val, c.d_key, c.chunk, false, true);
    Plan p2 = make_plan(lists, tm, c.d_val, c.d_key, c.chunk, true, false);
    s = upload_plan(p1, &r->plan_dev[1]);
    if (s == TTT_OK) s = upload_plan(p2, &r->plan_dev[2]);
    r->lists[1] = p1.grid;
    r->lists[2] = p2.grid;
  }
  for (int i = 0; i < 3; ++i) r->grid[i] = per * r->lists[i];
  if (s != TTT_OK) {
    for (int i = 0; i < 3; ++i)
      if (r->plan_dev[i]) cudaFree(r->plan_dev[i]);
    delete r;
    return s;
  }
  st->ip.tc = r;
  return TTT_OK;
}

void free_tc(ttt_state* st) {
  TCResources* r = st->ip.tc;
  if (r == nullptr) return;
  for (int i = 0; i < 3; ++i)
    if (r->plan_dev[i]) cudaFree(r->plan_dev[i]);
  if (r->conv) cudaFree(r->conv);
  if (r->counters) cudaFree(r->counters);
  delete r;
  st->ip.tc = nullptr;
}

ttt_status inplace_bf16_scan(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* targets, int64_t T,
                             __nv_bfloat16* O, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const int d = c.d_val, f = c.d_key, C = c.chunk;
  const bool target = c.target_mode == 1;
  TTT_TRY(ensure_tc(st));
  TCResources* r = st->ip.tc;
  const int nchunks = (int)(T / C);

  CUtensorMap tmZk, tmZm, tmVm_in, tmVm_buf[3], tmWk[3], tmConv, tmWt, tmWf, tmWs[3];
  TTT_TRY(map2d(&tmWf, st->ip.W, f, d, kWCols, BM, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B));
  for (int i = 0; i < 3; ++i) {
    TTT_TRY(map2d(&tmWs[i], st->ip.Wsh[i], f, d, kWCols, BM, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_64B));
    // APPLY B operand: 256 rows of the bf16 W per tile, 128 per CTA of an SM pair.
    TTT_TRY(map2d(&tmWk[i], st->ip.Wsh[i], f, d, BK, r->pair ? BN / 2 : BN));
  }
  TTT_TRY(map2d(&tmZk, Z, f, T, BK, BM));
  TTT_TRY(map2d(&tmZm, Z, f, T, 64, BK));
  if (target) {
    if (r->conv_rows < (size_t)T) {
      if (r->conv) cudaFree(r->conv);
      r->conv = nullptr;
      r->conv_rows = 0;
      TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&r->conv), (size_t)T * d * 2));
      r->conv_rows = (size_t)T;
    }
    TTT_TRY(map2d(&tmConv, r->conv, d, T, BK, BM));
    TTT_TRY(map2d(&tmWt, st->ip.Wtarget, d, d, 64, BK));
    for (int i = 0; i < 3; ++i) TTT_TRY(map2d(&tmVm_buf[i], st->ip.Vhat[i], d, C, 64, BK));
    const size_t pairs = (size_t)T * (d / 2);
    const int blocks = (int)std::min<size_t>((pairs + 255) / 256, (size_t)st->num_sms * 16);
    k_target_conv<<<blocks, 256, 0, s>>>(targets, st->ip.convw, r->conv, (int)T, d, C, c.conv_taps, c.conv_pad_mode);
    st->launches++;
    TTT_CUDA(cudaGetLastError());
  } else {
    TTT_TRY(map2d(&tmVm_in, targets, d, T, 64, BK));
    tmConv = tmZk;
    tmWt = tmZk;
  }

  if (r->pair)
    TTT_CUDA(cudaFuncSetAttribute(k_inplace_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTC));
  else
    TTT_CUDA(cudaFuncSetAttribute(k_inplace_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTC));

  auto args_for = [&](int plan, int chunk, int tchunk, int rounds, int* counters) {
    TCArgs a;
    a.sched = r->plan_dev[plan];
    a.chunk = chunk;
    a.target_chunk = tchunk;
    a.vrow0 = target ? 0 : chunk * C;
    a.d = d;
    a.f = f;
    a.C = C;
    a.eta = c.eta;
    a.O = O;
    a.Vhat_out = target ? st->ip.Vhat[tchunk % 3] : nullptr;
    a.status = DevStatus{st->status.dev, st->wait_limit_ns, st->status.dev + 1};
    a.stall_round = -1;
    if (st->inject_stall && rounds >= 2 && counters != nullptr) {
      a.stall_round = 1;
      st->inject_stall = 0;
    }
    a.rotate = list_rotation(r->lists[plan]);
    a.rounds = rounds;
    a.cur0 = 0;
    a.ring = st->ip.ring;
    a.advance = plan == 1 ? 0 : rounds;  // plan 1 holds TARGET tiles alone
    a.nbd = (d + BN - 1) / BN;
    a.upd_done = counters;
    a.app_done = counters ? counters + (size_t)rounds * a.nbd : nullptr;
    a.sched_last = nullptr;
    a.vhat[0] = a.vhat[1] = a.vhat[2] = nullptr;
    a.tgt_done = nullptr;
    return a;
  };
  auto launch = [&](int plan, TCArgs a, const CUtensorMap& vm) -> ttt_status {
    void* params[] = {&tmZk, &tmZm, const_cast<CUtensorMap*>(&vm), const_cast<CUtensorMap*>(&vm),
                      const_cast<CUtensorMap*>(&vm), &tmWk[0], &tmWk[1], &tmWk[2], &tmConv, &tmWt, &tmWf,
                      &tmWs[0], &tmWs[1], &tmWs[2], &a};
    TTT_TRY(launch_tc(r->pair, r->grid[plan], false, params, s));
    st->launches++;
    return TTT_OK;
  };
  // All chunks in one launch: each CTA runs its tile list once per chunk, waiting on progress
  // counters only where a chunk needs another CTA's result of an earlier chunk, so a chunk's
  // last tiles overlap the next chunk's first. The grid is one CTA (or SM pair) per SM (pair)
  // that can be resident at once: launched cooperatively, or as clusters sized by the
  // occupancy query, so every CTA is resident.
  auto launch_rounds = [&](TCArgs& a, const CUtensorMap& vm0, const CUtensorMap& vm1,
                           const CUtensorMap& vm2) -> ttt_status {
    void* params[] = {&tmZk, &tmZm, const_cast<CUtensorMap*>(&vm0), const_cast<CUtensorMap*>(&vm1),
                      const_cast<CUtensorMap*>(&vm2), &tmWk[0], &tmWk[1], &tmWk[2], &tmConv, &tmWt, &tmWf,
                      &tmWs[0], &tmWs[1], &tmWs[2], &a};
    TTT_TRY(launch_tc(r->pair, r->grid[0], true, params, s));
    st->launches++;
    return TTT_OK;
  };
  const int nbd = (d + BN - 1) / BN;
  auto counters = [&](size_t need) -> ttt_status {
    if (r->counters_n < need) {
      if (r->counters) cudaFree(r->counters);
      r->counters = nullptr;
      r->counters_n = 0;
      TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&r->counters), need * sizeof(int)));
      r->counters_n = need;
    }
    TTT_CUDA(cudaMemsetAsync(r->counters, 0, need * sizeof(int), s));
    return TTT_OK;
  };

  if (!target) {
    TTT_TRY(counters(2 * (size_t)nchunks * nbd));
    TCArgs a = args_for(0, 0, 1, nchunks, r->counters);
    return launch_rounds(a, tmVm_in, tmVm_in, tmVm_in);
  }

  // Fused target: the targets of the first chunk by their own launch, then every chunk in
  // one launch whose rounds also produce the next chunk's targets (the last round runs the
  // schedule without TARGET tiles).
  TTT_TRY(launch(1, args_for(1, 0, 0, 1, nullptr), tmVm_buf[0]));
  if (r->grid[2] == r->grid[0]) {
    TTT_TRY(counters(3 * (size_t)nchunks * nbd));
    TCArgs a = args_for(0, 0, 1, nchunks, r->counters);
    a.sched_last = r->plan_dev[2];
    a.vhat[0] = st->ip.Vhat[0];
    a.vhat[1] = st->ip.Vhat[1];
    a.vhat[2] = st->ip.Vhat[2];
    a.tgt_done = r->counters + 2 * (size_t)nchunks * nbd;
    a.Vhat_out = nullptr;
    return launch_rounds(a, tmVm_buf[0], tmVm_buf[1], tmVm_buf[2]);
  }
  for (int ch = 0; ch < nchunks; ++ch) {
    const bool last = ch + 1 == nchunks;
    const int plan = last ? 2 : 0;
    TTT_TRY(launch(plan, args_for(plan, ch, ch + 1, 1, nullptr), tmVm_buf[ch % 3]));
  }
  return TTT_OK;
}


// ---- target generation into caller-provided scratch -----------------------------------

namespace {

// Round-robin schedule of the TARGET tiles of one block of rows: tile i goes to CTA i % grid.
// Same layout as the host-built schedules: [grid + 1] offsets, then the tile codes.
__global__ void k_target_plan(int32_t* plan, int grid, int mt, int nt) {
  const int n = mt * nt, q = n / grid, r = n % grid;
  for (int c = threadIdx.x; c <= grid; c += blockDim.x) plan[c] = c * q + min(c, r);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int c = i % grid, j = i / grid;
    plan[grid + 1 + c * q + min(c, r) + j] = tile_code(TARGET, i / nt, i % nt);
  }
}

}  // namespace

int target_values_plan_ints(int T, int d, int num_sms) {
  const int ntiles = (T / BM) * ((d + BN - 1) / BN);
  const int grid = std::max(1, std::min(num_sms, ntiles));
  return grid + 1 + ntiles;
}

ttt_status target_values_into(const __nv_bfloat16* X0, const float* convw, const __nv_bfloat16* Wtarget, int T, int d,
                              int C, int taps, int pad_mode, __nv_bfloat16* conv_scratch, int32_t* plan_scratch,
                              __nv_bfloat16* out, int32_t* status, int num_sms, cudaStream_t s) {
  const int mt = T / BM, nt = (d + BN - 1) / BN;
  const int grid = std::max(1, std::min(num_sms, mt * nt));
  const size_t pairs = (size_t)T * (d / 2);
  const int blocks = (int)std::min<size_t>((pairs + 255) / 256, (size_t)num_sms * 16);
  k_target_conv<<<blocks, 256, 0, s>>>(X0, convw, conv_scratch, T, d, C, taps, pad_mode);
  TTT_CUDA(cudaGetLastError());
  k_target_plan<<<1, 256, 0, s>>>(plan_scratch, grid, mt, nt);
  TTT_CUDA(cudaGetLastError());
  CUtensorMap tmConv, tmWt;
  TTT_TRY(map2d(&tmConv, conv_scratch, d, T, BK, BM));
  TTT_TRY(map2d(&tmWt, Wtarget, d, d, 64, BK));
  TCArgs a;
  a.sched = plan_scratch;
  a.chunk = 0;
  a.target_chunk = 0;
  a.vrow0 = 0;
  a.d = d;
  a.f = d;
  a.C = T;
  a.eta = 0.f;
  a.O = nullptr;
  a.Vhat_out = out;
  a.status = DevStatus{status, kWaitLimitNs};
  a.stall_round = -1;
  a.rounds = 1;
  a.cur0 = 0;
  a.ring = nullptr;
  a.advance = 0;
  a.nbd = 0;
  a.upd_done = nullptr;
  a.app_done = nullptr;
  a.sched_last = nullptr;
  a.vhat[0] = a.vhat[1] = a.vhat[2] = nullptr;
  a.tgt_done = nullptr;
  a.rotate = 1;
  TTT_CUDA(cudaFuncSetAttribute(k_inplace_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTC));
  k_inplace_tc<false><<<grid, kThreadsTC, kSmemTC, s>>>(tmConv, tmConv, tmConv, tmConv, tmConv, tmConv, tmConv, tmConv, tmConv, tmWt,
                                              tmConv, tmConv, tmConv, tmConv, a);
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
