// Host-side internals of libttt.so: the state object and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "ttt.h"

namespace ttt {

struct TCResources;

// Records `msg` as the calling thread's last error and returns `s`.
ttt_status fail(ttt_status s, const char* fmt, ...);
// Maps a CUDA runtime error to TTT_ERR_CUDA with a message naming `what`.
ttt_status cuda_fail(cudaError_t e, const char* what);

#define TTT_CUDA(call)                                        \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return ::ttt::cuda_fail(e_, #call); \
  } while (0)

#define TTT_TRY(call)                      \
  do {                                     \
    ttt_status s_ = (call);                \
    if (s_ != TTT_OK) return s_;           \
  } while (0)

// Device-visible status words (pinned, mapped host memory): kernels record the first
// failure in host[0] with atomicCAS and where it happened in host[1]; the host reads both in
// ttt_state_poll().
struct StatusWord {
  int* host = nullptr;
  int* dev = nullptr;
};

struct InplaceBuffers {
  float* W = nullptr;            // fp32 master [d, f]
  float* W0 = nullptr;           // pretrained copy [d, f]
  float* Wf32_next = nullptr;    // fp32 path: the next chunk's weight, written beside W (swapped)
  // bf16 copies of W for the apply (BF16 path): chunk c applies with one while its update
  // writes the next; three so that an update never overwrites the copy that the chunk
  // before is still applying with when chunks overlap in one launch.
  __nv_bfloat16* Wsh[3] = {nullptr, nullptr, nullptr};
  // Device words {index of the bf16 copy that holds the current W, CTAs of the running scan
  // launch that have finished}: the scan kernel reads the index and its last CTA advances it,
  // so the host holds no per-call state and a captured call replays correctly.
  int* ring = nullptr;
  __nv_bfloat16* Wtarget = nullptr;  // [d, d]
  float* convw = nullptr;        // [d, taps]
  // Targets of a chunk [C, d] (fused target): chunk c's are produced while chunk c − 1 runs and
  // read by chunk c's update; three buffers so the producer never waits for a reader.
  __nv_bfloat16* Vhat[3] = {nullptr, nullptr, nullptr};
  TCResources* tc = nullptr;     // tensor-core schedules and conv(X0) buffer, built on first use
  // Context-parallel form (TTT_OPT_INPLACE_PREFIX): the chunks' fp32 deltas [n][d][f] and the bf16
  // weights each chunk applies with [n][d][f], grown on demand.
  int prefix_form = 0;
  int sm_pair = 1;               // TTT_OPT_SM_PAIR: tensor-core tiles on SM pairs where shapes allow
  float* prefix_D = nullptr;
  __nv_bfloat16* prefix_Wb = nullptr;
  int prefix_chunks = 0;
  // Packed sequences (ttt_chunk_scan_docs): Z, V̂ and O with every document padded to whole
  // chunks, the padded row → input row map (−1: padding), the first-chunk-of-a-document flags
  // and the chunk deltas' squared Frobenius norms, grown on demand.
  __nv_bfloat16* docs_Z = nullptr;
  __nv_bfloat16* docs_V = nullptr;
  __nv_bfloat16* docs_O = nullptr;
  int32_t* docs_rows = nullptr;
  int32_t* docs_reset = nullptr;
  double* docs_sumsq = nullptr;
  int64_t docs_rows_cap = 0;
  int docs_chunks_cap = 0;
  // With the target made in the scan: the padded layout's conv rows and targets [Tp, d_val]
  // and the target tiles' schedule, grown on demand.
  __nv_bfloat16* docs_conv = nullptr;
  __nv_bfloat16* docs_T = nullptr;
  int32_t* docs_plan = nullptr;
  int64_t docs_target_cap = 0;
  int64_t docs_plan_cap = 0;
};

// Tensor maps of one scan's K, V, Q, O (encoding them costs microseconds of host time, so the
// maps of the last few buffer sets are kept: a caller that cycles through a few sets of buffers
// encodes each set once).
struct LinearMapSet {
  const void* key[4] = {nullptr, nullptr, nullptr, nullptr};
  int64_t T = -1;
  uint64_t last_use = 0;
  CUtensorMap maps[4];
};

struct LinearBuffers {
  float* W = nullptr;   // [B, H, D, D] (TTT-MLP: [B, H, 64·256 + 256·64], W1 then W2 per head)
  float* W0 = nullptr;  // same shape
  float* ln_gamma = nullptr;  // LayerNorm rules: [H, 64] gain and bias of the inner model's LN
  float* ln_beta = nullptr;
  static constexpr int kMapSets = 8;
  LinearMapSet map_sets[kMapSets];
  uint64_t map_clock = 0;
  // Kernels whose shared-memory size has been raised for this state's device.
  uint64_t smem_set = 0;
  // Inner mini-batches per chunk of the b = 16 scan (TTT_OPT_LINEAR_CHUNK): 1 = one step at a
  // time, 2 or 4 = the chunked form; 0 = the library's choice (1).
  int form = 0;
  // Packed sequences (ttt_chunk_scan_packed): K, V, Q, O with every document padded to whole
  // mini-batches [B, H, Tp, 64], the losses [B, H, Tp], the padded row -> input token map
  // [B, Tp] (-1: padding) and the per-(sequence, mini-batch) {reset, real tokens} table,
  // grown on demand.
  __nv_bfloat16* pk[4] = {nullptr, nullptr, nullptr, nullptr};
  float* pk_loss = nullptr;
  int32_t* pk_rows = nullptr;
  int2* pk_steps = nullptr;
  int64_t pk_cap = 0;      // rows of pk[] (B·H·Tp)
  int64_t pk_map_cap = 0;  // entries of pk_rows (B·Tp)
};

struct GateBuffers {
  float* tau = nullptr;       // [B, H]
  int32_t* tau_set = nullptr; // [B, H]
  int32_t* entries = nullptr; // [B, H, cap, 3]
  int32_t* counts = nullptr;  // [B, H, 2]
  // Tokens gated since the last reset, per (sequence, head) on the device: the gating kernels
  // read it and advance it. t_offset counts the same through the calls made on the host; it
  // only gives early errors, since it misses the replays of a captured call.
  int64_t* tokens = nullptr;  // [B, H]
  int64_t t_offset = 0;
};

// ttt_chunk_scan_host: two sets of device buffers for one segment of tokens (keys, targets,
// queries, out, loss), so that a segment's copies in and out overlap the scan of its
// neighbours, and the copy streams and events of that pipeline (created on first use).
struct HostStaging {
  void* buf[2][5] = {};
  size_t bytes[2][5] = {};
  cudaStream_t copy_in = nullptr;
  cudaStream_t copy_out = nullptr;
  cudaEvent_t entry = nullptr;
  cudaEvent_t in_done[2] = {nullptr, nullptr};    // a set's inputs are on the device
  cudaEvent_t scan_done[2] = {nullptr, nullptr};  // a set's scan ended: inputs free, outputs ready
  cudaEvent_t out_done[2] = {nullptr, nullptr};   // a set's outputs are back in host memory
};

}  // namespace ttt

struct ttt_state {
  ttt_config cfg;
  int device = 0;
  int num_sms = 0;
  ttt::StatusWord status;
  ttt::InplaceBuffers ip;
  ttt::LinearBuffers lin;
  ttt::GateBuffers gate;
  ttt::HostStaging staging;
  int64_t launches = 0;
  // Limit of every spin-wait of this state's kernels (TTT_OPT_WAIT_LIMIT_NS), in ns.
  uint64_t wait_limit_ns = 2000000000ull;
  // Fault injection (TTT_OPT_INJECT_STALL, tests): the next scan that can makes one of its
  // bounded waits wait for something that never comes; cleared once used.
  int inject_stall = 0;
};

namespace ttt {

size_t io_size(int dtype);

// ---- kernel launchers (each returns TTT_OK or TTT_ERR_CUDA after the launch) ----------

// In-Place, fp32 SIMT: one chunk of the scan (apply with W, then W += η·V̂ᵀZ).
// Targets V̂ = Conv1D(X0)·Wtarget for T tokens (T a multiple of 128) into `out`, with the
// caller's scratch for the conv rows [T, d] and the tile schedule (target_values_plan_ints).
int target_values_plan_ints(int T, int d, int num_sms);
ttt_status target_values_into(const __nv_bfloat16* X0, const float* convw, const __nv_bfloat16* Wtarget, int T, int d,
                              int C, int taps, int pad_mode, __nv_bfloat16* conv_scratch, int32_t* plan_scratch,
                              __nv_bfloat16* out, int32_t* status, int num_sms, cudaStream_t s);

// y ← y + alpha·x over n fp32 elements (device), on stream s.
ttt_status add_f32(float* y, const float* x, float alpha, size_t n, int num_sms, cudaStream_t s);

ttt_status inplace_f32_chunk(ttt_state* st, const float* Z, const float* Vhat, const float* W, float* Wn, float* O,
                             int C, cudaStream_t s);

// In-Place, bf16 tensor cores: the whole scan over T tokens.
ttt_status inplace_bf16_scan(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* targets,
                             int64_t T, __nv_bfloat16* O, cudaStream_t s);

// In-Place, bf16 tensor cores, context-parallel form: all chunk deltas, their exclusive prefix
// sums, then all chunk outputs (three launches, no cross-chunk waits).
ttt_status inplace_bf16_scan_prefix(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* Vhat, int64_t T,
                                    __nv_bfloat16* O, cudaStream_t s);

// In-Place, bf16, packed sequences: documents laid end to end, each scanned from the
// pretrained weight with its own chunks (a shorter last one), each chunk's delta clipped to
// Frobenius norm `clip` when clip > 0. Context-parallel machinery; doc_starts is host memory.
ttt_status inplace_bf16_scan_docs(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* Vhat, int64_t T,
                                  const int64_t* doc_starts, int ndocs, float clip, __nv_bfloat16* O,
                                  cudaStream_t s);

// Frees the tensor-core resources of a state (no-op if none were built).
void free_tc(ttt_state* st);

// TTT-Linear mini-batch scan over T tokens of every (sequence, head).
ttt_status linear_scan(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V,
                       const __nv_bfloat16* Q, int64_t T, __nv_bfloat16* O, float* loss,
                       cudaStream_t s);

// TTT-Linear with LayerNorm and residual, TTT-MLP, or the plain TTT-Linear rule with per-token
// weights: the scan over T tokens of every (sequence, head), mini-batch 16.
ttt_status inner_scan(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                      int64_t T, __nv_bfloat16* O, float* loss, cudaStream_t s);

// The same over packed sequences: sequence b holds docs_per_seq[b] documents laid end to end
// whose first tokens are the next docs_per_seq[b] entries of doc_starts (host memory); each is
// scanned from W0 with mini-batches counted from its first token.
ttt_status inner_scan_packed(ttt_state* st, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                             int64_t T, __nv_bfloat16* O, float* loss, const int64_t* doc_starts,
                             const int32_t* docs_per_seq, cudaStream_t s);
void free_packed(ttt_state* st);

// Residual-cache read path: out = o_ttt + clamp(α, 0, 1) ⊙ (attention over the visible entries).
ttt_status cache_attention(const ttt_state* st, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                           const __nv_bfloat16* V, const __nv_bfloat16* O_ttt, const float* alpha, int64_t T,
                           __nv_bfloat16* out, cudaStream_t s);

// Surprisal gate over T losses of every (sequence, head).
ttt_status gate_route(ttt_state* st, const float* loss, int64_t T, cudaStream_t s);
// Nearest rank ceil(gate_pct·64) of the gate's percentile (1-based).
int gate_rank(const ttt_config& c);

// Small utility kernels.
ttt_status f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s,
                       ttt_state* st);
ttt_status fill_i32(int32_t* dst, int32_t v, size_t n, cudaStream_t s, ttt_state* st);

// TMA descriptor encoding through the driver entry point (no -lcuda link needed).
ttt_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

}  // namespace ttt
