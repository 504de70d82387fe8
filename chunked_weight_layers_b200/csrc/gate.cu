// SR-TTT surprisal gate and residual cache ("SR-TTT: Surprisal-Aware Residual Test-Time
// Training", §2.1 Surprisal Filter and Residual Cache; §5 on saturation).
//
// Per (sequence, head), chunks of 64 losses are gated in order:
//   p95  = the ceil(pct·64)-th smallest loss of the chunk (nearest rank; 61st for 0.95),
//   τ    = p95 for the first chunk since reset, else fl32(fl32(a·τ) + fl32(c·p95)) (a = 0.9f,
//          c = 0.1f, each product and the sum rounded to fp32, no fused multiply-add),
//   pass = den·S ≥ (num·64)·τ in double, S the double sum of the chunk's losses in index order
//          (the mean test S/64 ≥ (num/den)·τ with num/den = 4/5),
//   route t ⇔ pass ∧ L_t > τ (strict, fp32).
// Routed (sequence, head, t) are appended in increasing t to the (sequence, head)'s cache
// until it holds `capacity` entries; later routed tokens are counted as dropped.
//
// Only τ is sequential across chunks, so the kernel splits the work by dependency:
//   1. every warp takes p95 and S of its chunks (chunk_stats: counting selection and an
//      exactness-checked tree sum);
//   2. one thread runs the scalar τ recurrence over the block of chunks;
//   3. all threads flag routed tokens and compact them in order with a block-wide scan.
// One CTA per (sequence, head); losses are processed in blocks of 64 chunks (4096 tokens).
// This kernel serves the standalone routing call; the b = 16 TTT-Linear scan runs the same
// gate in its writer warp, tile by tile.
#include "common.cuh"
#include "gate_chunk.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int kGateThreads = 256;
constexpr int kChunk = 64;
constexpr int kBlockChunks = 64;
constexpr int kBlockTok = kChunk * kBlockChunks;
constexpr int kTokPerThread = kBlockTok / kGateThreads;  // 16

struct __align__(16) GateSmem {
  float x[kBlockTok];
  double S[kBlockChunks];
  float p[kBlockChunks];
  float tau[kBlockChunks];
  int pass[kBlockChunks];
  int warp_sum[kGateThreads / 32];
  float tau_carry;
  int tau_set;
  int routed;
  long long tokens;  // tokens gated since reset before this call
};

__global__ void __launch_bounds__(kGateThreads)
    k_gate(const float* __restrict__ loss, int T, int heads, int rank, float ema_old, float ema_new, double lhs_scale,
           double rhs_scale, float* __restrict__ tau_state, int32_t* __restrict__ tau_set_state,
           int32_t* __restrict__ entries, int32_t* __restrict__ counts, int capacity, int64_t* __restrict__ tokens,
           int* status) {
  __shared__ GateSmem sm;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* L = loss + (size_t)bh * T;
  if (tid == 0) {
    sm.tau_carry = tau_state[bh];
    sm.tau_set = tau_set_state[bh];
    sm.routed = counts[2 * bh + 0];
    sm.tokens = tokens[bh];
  }
  __syncthreads();
  const long long t_offset = sm.tokens;

  for (int b0 = 0; b0 < T; b0 += kBlockTok) {
    const int ntok = min(kBlockTok, T - b0);
    const int nch = ntok / kChunk;
    for (int i = tid * 4; i < ntok; i += kGateThreads * 4)
      *reinterpret_cast<float4*>(&sm.x[i]) = *reinterpret_cast<const float4*>(&L[b0 + i]);
    __syncthreads();

    // 1. percentile and sum of every chunk (warp per chunk).
    for (int g = warp; g < nch; g += kGateThreads / 32) {
      float pv;
      double S;
      chunk_stats(&sm.x[g * kChunk], lane, rank, pv, S);
      if (lane == 0) {
        sm.p[g] = pv;
        sm.S[g] = S;
      }
    }
    __syncthreads();

    // 2. the threshold recurrence (sequential over chunks).
    if (tid == 0) {
      float tau = sm.tau_carry;
      int set = sm.tau_set;
      for (int g = 0; g < nch; ++g) {
        tau = tau_next(tau, set, sm.p[g], ema_old, ema_new);
        set = 1;
        sm.tau[g] = tau;
        sm.pass[g] = lhs_scale * sm.S[g] >= rhs_scale * (double)tau;
      }
      sm.tau_carry = tau;
      sm.tau_set = set;
    }
    __syncthreads();

    // 3. flags and ordered compaction: thread i owns tokens [16i, 16i + 16) of the block.
    const int t0 = tid * kTokPerThread;
    unsigned flags = 0;
    for (int j = 0; j < kTokPerThread; ++j) {
      const int t = t0 + j;
      if (t < ntok) {
        const int g = t / kChunk;
        if (sm.pass[g] && sm.x[t] > sm.tau[g]) flags |= 1u << j;
      }
    }
    const int cnt = __popc(flags);
    int incl = cnt;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) sm.warp_sum[warp] = incl;
    __syncthreads();
    int before = sm.routed;
    for (int w = 0; w < warp; ++w) before += sm.warp_sum[w];
    before += incl - cnt;
    int32_t* E = entries + (size_t)bh * capacity * 3;
    const int seq = bh / heads, head = bh % heads;
    for (int j = 0; j < kTokPerThread; ++j) {
      if (flags & (1u << j)) {
        if (before < capacity) {
          E[3 * before + 0] = seq;
          E[3 * before + 1] = head;
          E[3 * before + 2] = (int32_t)(t_offset + b0 + t0 + j);
        }
        ++before;
      }
    }
    __syncthreads();
    if (tid == 0) {
      int total = 0;
      for (int w = 0; w < kGateThreads / 32; ++w) total += sm.warp_sum[w];
      sm.routed += total;
    }
    __syncthreads();
  }

  if (tid == 0) {
    tau_state[bh] = sm.tau_carry;
    tau_set_state[bh] = sm.tau_set;
    counts[2 * bh + 0] = sm.routed;
    counts[2 * bh + 1] = sm.routed > capacity ? sm.routed - capacity : 0;
    tokens[bh] = t_offset + T;
    if (t_offset + T > 0x7FFFFFFFll)
      record_status(DevStatus{status, 0, status + 1}, kDevUnsupported, kSiteTokenLimit | (bh & 0xFFFF));
  }
}

}  // namespace

int gate_rank(const ttt_config& c) {
  // Nearest rank ceil(pct·n), computed in double like the definition.
  const double x = (double)c.gate_pct * kChunk;
  int rank = (int)x;
  if ((double)rank < x - 1e-9) ++rank;
  if (rank < 1) rank = 1;
  if (rank > kChunk) rank = kChunk;
  return rank;
}

ttt_status gate_route(ttt_state* st, const float* loss, int64_t T, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const int rank = gate_rank(c);
  const double lhs = (double)c.gate_mean_den;
  const double rhs = (double)c.gate_mean_num * kChunk;
  k_gate<<<c.batch * c.heads, kGateThreads, 0, s>>>(loss, (int)T, c.heads, rank, c.gate_ema_old, c.gate_ema_new, lhs,
                                                    rhs, st->gate.tau, st->gate.tau_set, st->gate.entries,
                                                    st->gate.counts, c.cache_capacity, st->gate.tokens,
                                                    st->status.dev);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  st->gate.t_offset += T;
  return TTT_OK;
}

}  // namespace ttt
