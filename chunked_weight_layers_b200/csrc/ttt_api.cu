// C ABI of libttt.so: argument validation, state memory, and dispatch to the kernels.
// The semantics of every entry point are documented in include/ttt.h.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <numeric>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace ttt {

static thread_local char g_last_error[512] = "";

ttt_status fail(ttt_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

ttt_status cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();  // clear a sticky launch error so later calls can proceed
  if (e == cudaErrorMemoryAllocation)
    return fail(TTT_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
  return fail(TTT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t io_size(int dtype) { return dtype == TTT_F32 ? 4 : 2; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Allocation that honours the fault-injection switch TTT_INJECT_OOM (tests only).
static ttt_status dev_alloc(void** p, size_t bytes, const char* what) {
  *p = nullptr;
  const char* inj = getenv("TTT_INJECT_OOM");
  if (inj != nullptr && inj[0] == '1') return fail(TTT_ERR_OOM, "%s: injected allocation failure", what);
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    *p = nullptr;
    return cuda_fail(e, what);
  }
  return TTT_OK;
}

static void dev_free(void* p) {
  if (p != nullptr) cudaFree(p);
}

static ttt_status validate(const ttt_config* c) {
  if (c->token_weights != 0 && c->token_weights != 1) return fail(TTT_ERR_INVALID_ARG, "token_weights must be 0 or 1");
  if (c->token_weights && c->rule == TTT_RULE_INPLACE_HEBBIAN)
    return fail(TTT_ERR_UNSUPPORTED, "per-token weights apply to the TTT-Linear family");
  if (c->token_weights && c->rule == TTT_RULE_LINEAR_GD && (c->chunk != 16 || c->gate_enable))
    return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear per-token weights: mini-batch 16, no gate");
  if (c->rule == TTT_RULE_INPLACE_HEBBIAN) {
    if (c->batch != 1 || c->heads != 1)
      return fail(TTT_ERR_UNSUPPORTED, "In-Place scan: batch and heads must be 1 (one Wdown state)");
    if (c->d_key < 1 || c->d_val < 1 || c->chunk < 1)
      return fail(TTT_ERR_INVALID_ARG, "In-Place scan: d_key, d_val and chunk must be positive");
    if (c->io_dtype == TTT_F32) {
      if (c->target_mode != 0)
        return fail(TTT_ERR_UNSUPPORTED, "In-Place fp32: fused target generation needs BF16 io");
      return TTT_OK;
    }
    if (c->io_dtype != TTT_BF16) return fail(TTT_ERR_INVALID_ARG, "unknown io_dtype %d", c->io_dtype);
    if (c->d_key % 8 != 0 || c->d_val % 8 != 0)
      return fail(TTT_ERR_UNSUPPORTED, "In-Place BF16: d_key and d_val must be multiples of 8 (16-byte rows for TMA)");
    if (c->chunk % 128 != 0)
      return fail(TTT_ERR_UNSUPPORTED, "In-Place BF16: chunk must be a multiple of 128");
    if (c->target_mode != 0 && c->target_mode != 1)
      return fail(TTT_ERR_INVALID_ARG, "target_mode must be 0 or 1");
    if (c->target_mode == 1) {
      if (c->conv_taps < 1 || c->conv_taps > 8)
        return fail(TTT_ERR_UNSUPPORTED, "conv_taps must lie in [1, 8]");
      if (c->conv_pad_mode != 0 && c->conv_pad_mode != 1)
        return fail(TTT_ERR_INVALID_ARG, "conv_pad_mode must be 0 or 1");
    }
    if (c->gate_enable) return fail(TTT_ERR_UNSUPPORTED, "the surprisal gate runs on TTT-Linear states");
    return TTT_OK;
  }
  if (c->rule == TTT_RULE_LINEAR_GD) {
    if (c->io_dtype != TTT_BF16) return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear: io_dtype must be BF16");
    if (c->batch < 1 || c->heads < 1) return fail(TTT_ERR_INVALID_ARG, "TTT-Linear: batch and heads must be positive");
    if (c->d_key != 64 || c->d_val != 64)
      return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear: head width must be 64 (d_key = d_val = 64)");
    if (c->chunk != 16 && c->chunk != 32 && c->chunk != 64)
      return fail(TTT_ERR_UNSUPPORTED, "TTT-Linear: inner mini-batch must be 16, 32 or 64");
    if (c->target_mode != 0) return fail(TTT_ERR_INVALID_ARG, "target_mode applies to In-Place only");
    if (c->gate_enable) {
      if (c->gate_chunk != 64) return fail(TTT_ERR_UNSUPPORTED, "gate_chunk must be 64");
      if (c->cache_capacity < 1) return fail(TTT_ERR_INVALID_ARG, "cache_capacity must be positive");
      if (!(c->gate_pct > 0.f && c->gate_pct <= 1.f)) return fail(TTT_ERR_INVALID_ARG, "gate_pct must lie in (0, 1]");
      if (c->gate_mean_num < 0 || c->gate_mean_den < 1)
        return fail(TTT_ERR_INVALID_ARG, "gate mean fraction must be num >= 0, den >= 1");
    }
    return TTT_OK;
  }
  if (c->rule == TTT_RULE_LINEAR_LN_GD || c->rule == TTT_RULE_MLP_GD) {
    const char* name = c->rule == TTT_RULE_MLP_GD ? "TTT-MLP" : "TTT-Linear with LayerNorm";
    if (c->io_dtype != TTT_BF16) return fail(TTT_ERR_UNSUPPORTED, "%s: io_dtype must be BF16", name);
    if (c->batch < 1 || c->heads < 1) return fail(TTT_ERR_INVALID_ARG, "%s: batch and heads must be positive", name);
    if (c->d_key != 64 || c->d_val != 64)
      return fail(TTT_ERR_UNSUPPORTED, "%s: head width must be 64 (d_key = d_val = 64)", name);
    if (c->chunk != 16) return fail(TTT_ERR_UNSUPPORTED, "%s: inner mini-batch must be 16", name);
    if (c->target_mode != 0) return fail(TTT_ERR_INVALID_ARG, "target_mode applies to In-Place only");
    if (c->gate_enable) return fail(TTT_ERR_UNSUPPORTED, "the surprisal gate runs on TTT-Linear states");
    if (!(c->ln_eps > 0.f)) return fail(TTT_ERR_INVALID_ARG, "%s: ln_eps must be positive", name);
    return TTT_OK;
  }
  return fail(TTT_ERR_INVALID_ARG, "unknown rule %d", c->rule);
}

static size_t weight_elems(const ttt_config& c) {
  if (c.rule == TTT_RULE_INPLACE_HEBBIAN) return (size_t)c.d_val * c.d_key;
  if (c.rule == TTT_RULE_MLP_GD) return (size_t)c.batch * c.heads * 2 * 64 * 256;
  return (size_t)c.batch * c.heads * c.d_key * c.d_key;
}

static void free_state(ttt_state* st) {
  if (st == nullptr) return;
  dev_free(st->ip.W);
  dev_free(st->ip.W0);
  dev_free(st->ip.Wf32_next);
  dev_free(st->ip.prefix_D);
  dev_free(st->ip.prefix_Wb);
  dev_free(st->ip.docs_Z);
  dev_free(st->ip.docs_V);
  dev_free(st->ip.docs_O);
  dev_free(st->ip.docs_rows);
  dev_free(st->ip.docs_reset);
  dev_free(st->ip.docs_sumsq);
  dev_free(st->ip.docs_conv);
  dev_free(st->ip.docs_T);
  dev_free(st->ip.docs_plan);
  dev_free(st->ip.Wsh[0]);
  dev_free(st->ip.Wsh[1]);
  dev_free(st->ip.Wsh[2]);
  dev_free(st->ip.ring);
  dev_free(st->ip.Wtarget);
  dev_free(st->ip.convw);
  free_tc(st);
  dev_free(st->ip.Vhat[0]);
  dev_free(st->ip.Vhat[1]);
  dev_free(st->ip.Vhat[2]);
  dev_free(st->lin.W);
  dev_free(st->lin.W0);
  dev_free(st->lin.ln_gamma);
  dev_free(st->lin.ln_beta);
  free_packed(st);
  dev_free(st->gate.tau);
  dev_free(st->gate.tau_set);
  dev_free(st->gate.entries);
  dev_free(st->gate.counts);
  dev_free(st->gate.tokens);
  HostStaging& hs = st->staging;
  for (int j = 0; j < 2; ++j)
    for (int i = 0; i < 5; ++i) dev_free(hs.buf[j][i]);
  cudaEvent_t* evs[] = {&hs.entry, &hs.in_done[0], &hs.in_done[1], &hs.scan_done[0], &hs.scan_done[1],
                        &hs.out_done[0], &hs.out_done[1]};
  for (cudaEvent_t* e : evs)
    if (*e != nullptr) cudaEventDestroy(*e);
  if (hs.copy_in != nullptr) cudaStreamDestroy(hs.copy_in);
  if (hs.copy_out != nullptr) cudaStreamDestroy(hs.copy_out);
  if (st->status.host != nullptr) cudaFreeHost(st->status.host);
  delete st;
}

static ttt_status gate_reset(ttt_state* st, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const size_t bh = (size_t)c.batch * c.heads;
  TTT_CUDA(cudaMemsetAsync(st->gate.tau, 0, bh * sizeof(float), s));
  TTT_CUDA(cudaMemsetAsync(st->gate.tau_set, 0, bh * sizeof(int32_t), s));
  TTT_CUDA(cudaMemsetAsync(st->gate.counts, 0, bh * 2 * sizeof(int32_t), s));
  TTT_CUDA(cudaMemsetAsync(st->gate.tokens, 0, bh * sizeof(int64_t), s));
  TTT_TRY(fill_i32(st->gate.entries, -1, bh * (size_t)c.cache_capacity * 3, s, st));
  st->gate.t_offset = 0;
  return TTT_OK;
}

static ttt_status load_weights(ttt_state* st, const float* W, cudaStream_t s) {
  const size_t n = weight_elems(st->cfg);
  if (st->cfg.rule == TTT_RULE_INPLACE_HEBBIAN) {
    TTT_CUDA(cudaMemcpyAsync(st->ip.W, W, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
    if (st->cfg.io_dtype == TTT_BF16) {
      TTT_CUDA(cudaMemsetAsync(st->ip.ring, 0, 2 * sizeof(int), s));
      TTT_TRY(f32_to_bf16(st->ip.W, st->ip.Wsh[0], n, s, st));
    }
  } else {
    TTT_CUDA(cudaMemcpyAsync(st->lin.W, W, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
  }
  return TTT_OK;
}

static ttt_status create_impl(const ttt_config* cfg, const void* W0, const void* Wtarget,
                              const float* convw, cudaStream_t s, ttt_state** out) {
  TTT_TRY(validate(cfg));
  const ttt_config& c = *cfg;
  if (W0 == nullptr || !aligned16(W0)) return fail(TTT_ERR_INVALID_ARG, "W0 must be a 16-byte aligned device pointer");
  const bool target = c.rule == TTT_RULE_INPLACE_HEBBIAN && c.target_mode == 1;
  if (target) {
    if (Wtarget == nullptr || convw == nullptr || !aligned16(Wtarget) || !aligned16(convw))
      return fail(TTT_ERR_INVALID_ARG, "target_mode 1 needs 16-byte aligned Wtarget and convw");
  } else if (Wtarget != nullptr || convw != nullptr) {
    return fail(TTT_ERR_INVALID_ARG, "Wtarget and convw are only taken with target_mode 1");
  }

  ttt_state* st = new (std::nothrow) ttt_state();
  if (st == nullptr) return fail(TTT_ERR_OOM, "host allocation of the state failed");
  st->cfg = c;
  ttt_status r = TTT_OK;
  auto guard = [&](ttt_status x) {
    if (x != TTT_OK && r == TTT_OK) r = x;
    return r == TTT_OK;
  };
  cudaError_t e = cudaGetDevice(&st->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&st->num_sms, cudaDevAttrMultiProcessorCount, st->device);
  if (e != cudaSuccess) {
    free_state(st);
    return cuda_fail(e, "cudaGetDevice");
  }
  e = cudaHostAlloc(reinterpret_cast<void**>(&st->status.host), 2 * sizeof(int), cudaHostAllocMapped);
  if (e == cudaSuccess) e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&st->status.dev), st->status.host, 0);
  if (e != cudaSuccess) {
    free_state(st);
    return cuda_fail(e, "status word allocation");
  }
  st->status.host[0] = st->status.host[1] = 0;

  const size_t nW = weight_elems(c);
  if (c.rule == TTT_RULE_INPLACE_HEBBIAN) {
    guard(dev_alloc((void**)&st->ip.W, nW * 4, "W")) && guard(dev_alloc((void**)&st->ip.W0, nW * 4, "W0"));
    if (r == TTT_OK && c.io_dtype == TTT_F32) guard(dev_alloc((void**)&st->ip.Wf32_next, nW * 4, "W (next chunk)"));
    if (r == TTT_OK && c.io_dtype == TTT_BF16) {
      guard(dev_alloc((void**)&st->ip.Wsh[0], nW * 2, "W bf16 copy")) &&
          guard(dev_alloc((void**)&st->ip.Wsh[1], nW * 2, "W bf16 copy")) &&
          guard(dev_alloc((void**)&st->ip.Wsh[2], nW * 2, "W bf16 copy")) &&
          guard(dev_alloc((void**)&st->ip.ring, 2 * sizeof(int), "bf16 copy index"));
    }
    if (r == TTT_OK && target) {
      const size_t dd = (size_t)c.d_val * c.d_val;
      guard(dev_alloc((void**)&st->ip.Wtarget, dd * 2, "Wtarget")) &&
          guard(dev_alloc((void**)&st->ip.convw, (size_t)c.d_val * c.conv_taps * 4, "convw")) &&
          guard(dev_alloc((void**)&st->ip.Vhat[0], (size_t)c.chunk * c.d_val * 2, "target buffer")) &&
          guard(dev_alloc((void**)&st->ip.Vhat[1], (size_t)c.chunk * c.d_val * 2, "target buffer")) &&
          guard(dev_alloc((void**)&st->ip.Vhat[2], (size_t)c.chunk * c.d_val * 2, "target buffer"));
    }
  } else {
    guard(dev_alloc((void**)&st->lin.W, nW * 4, "W")) && guard(dev_alloc((void**)&st->lin.W0, nW * 4, "W0"));
    const size_t bh = (size_t)c.batch * c.heads;
    const int cap = c.gate_enable ? c.cache_capacity : 1;
    st->cfg.cache_capacity = cap;
    if (r == TTT_OK && (c.rule == TTT_RULE_LINEAR_LN_GD || c.rule == TTT_RULE_MLP_GD)) {
      guard(dev_alloc((void**)&st->lin.ln_gamma, (size_t)c.heads * 64 * 4, "LayerNorm gain")) &&
          guard(dev_alloc((void**)&st->lin.ln_beta, (size_t)c.heads * 64 * 4, "LayerNorm bias"));
    }
    if (r == TTT_OK) {
      guard(dev_alloc((void**)&st->gate.tau, bh * 4, "tau")) &&
          guard(dev_alloc((void**)&st->gate.tau_set, bh * 4, "tau_set")) &&
          guard(dev_alloc((void**)&st->gate.entries, bh * (size_t)cap * 3 * 4, "cache")) &&
          guard(dev_alloc((void**)&st->gate.counts, bh * 2 * 4, "cache counts")) &&
          guard(dev_alloc((void**)&st->gate.tokens, bh * sizeof(int64_t), "token positions"));
    }
  }
  if (r != TTT_OK) {
    free_state(st);
    return r;
  }
  float* W0dst = c.rule == TTT_RULE_INPLACE_HEBBIAN ? st->ip.W0 : st->lin.W0;
  e = cudaMemcpyAsync(W0dst, W0, nW * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && target) {
    e = cudaMemcpyAsync(st->ip.Wtarget, Wtarget, (size_t)c.d_val * c.d_val * 2, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(st->ip.convw, convw, (size_t)c.d_val * c.conv_taps * 4, cudaMemcpyDeviceToDevice, s);
  }
  if (e != cudaSuccess) {
    free_state(st);
    return cuda_fail(e, "copying the initial weights");
  }
  r = load_weights(st, W0dst, s);
  if (r == TTT_OK && c.rule == TTT_RULE_LINEAR_GD) r = gate_reset(st, s);
  if (r == TTT_OK && st->lin.ln_gamma != nullptr) {
    // γ = 1 (the bits of 1.0f), β = 0.
    r = fill_i32(reinterpret_cast<int32_t*>(st->lin.ln_gamma), 0x3f800000, (size_t)c.heads * 64, s, st);
    if (r == TTT_OK) {
      e = cudaMemsetAsync(st->lin.ln_beta, 0, (size_t)c.heads * 64 * 4, s);
      if (e != cudaSuccess) r = cuda_fail(e, "LayerNorm bias");
    }
  }
  if (r != TTT_OK) {
    free_state(st);
    return r;
  }
  *out = st;
  return TTT_OK;
}

static ttt_status check_device(const ttt_state* st) {
  int dev = -1;
  TTT_CUDA(cudaGetDevice(&dev));
  if (dev != st->device) return fail(TTT_ERR_INVALID_ARG, "current device %d is not the state's device %d", dev, st->device);
  return TTT_OK;
}

// Cache entries hold the token position since the last reset as int32: a gated call must not
// take it past INT32_MAX.
static ttt_status check_token_position(const ttt_state* st, int64_t T) {
  if (st->gate.t_offset + T > (int64_t)INT32_MAX)
    return fail(TTT_ERR_UNSUPPORTED, "the gate's token position would pass 2^31 - 1 (reset the state first)");
  return TTT_OK;
}

static ttt_status scan_impl(ttt_state* st, const void* keys, const void* targets, const void* queries,
                            int64_t T, void* out, float* loss, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  if (T < 0) return fail(TTT_ERR_INVALID_ARG, "T must be non-negative");
  if (T % c.chunk != 0) return fail(TTT_ERR_INVALID_ARG, "T=%lld is not a multiple of the chunk %d", (long long)T, c.chunk);
  if (T > (int64_t)INT32_MAX / 2) return fail(TTT_ERR_UNSUPPORTED, "T too large");
  if (T == 0) return TTT_OK;
  TTT_TRY(check_device(st));
  if (keys == nullptr || targets == nullptr || !aligned16(keys) || !aligned16(targets))
    return fail(TTT_ERR_INVALID_ARG, "keys and targets must be 16-byte aligned device pointers");
  if (c.rule == TTT_RULE_INPLACE_HEBBIAN) {
    if (queries != nullptr || loss != nullptr)
      return fail(TTT_ERR_INVALID_ARG, "In-Place scan takes no queries and no loss output");
    if (out == nullptr || !aligned16(out)) return fail(TTT_ERR_INVALID_ARG, "out must be a 16-byte aligned device pointer");
    if (c.io_dtype == TTT_F32) {
      const float* Z = static_cast<const float*>(keys);
      const float* V = static_cast<const float*>(targets);
      float* O = static_cast<float*>(out);
      // Chunk j reads buffer j mod 2 and writes the other; after an odd number of chunks the
      // weight goes back to ip.W, so that every call starts and ends with it there.
      float* buf[2] = {st->ip.W, st->ip.Wf32_next};
      int64_t j = 0;
      for (int64_t t0 = 0; t0 < T; t0 += c.chunk, ++j)
        TTT_TRY(inplace_f32_chunk(st, Z + t0 * c.d_key, V + t0 * c.d_val, buf[j & 1], buf[(j + 1) & 1],
                                  O + t0 * c.d_val, c.chunk, s));
      if (j & 1)
        TTT_CUDA(cudaMemcpyAsync(st->ip.W, st->ip.Wf32_next, weight_elems(c) * sizeof(float), cudaMemcpyDeviceToDevice, s));
      return TTT_OK;
    }
    if (st->ip.prefix_form)
      return inplace_bf16_scan_prefix(st, static_cast<const __nv_bfloat16*>(keys),
                                      static_cast<const __nv_bfloat16*>(targets), T, static_cast<__nv_bfloat16*>(out), s);
    return inplace_bf16_scan(st, static_cast<const __nv_bfloat16*>(keys),
                             static_cast<const __nv_bfloat16*>(targets), T,
                             static_cast<__nv_bfloat16*>(out), s);
  }
  if ((queries == nullptr) != (out == nullptr))
    return fail(TTT_ERR_INVALID_ARG, "TTT-Linear: out must be given exactly when queries are");
  if (queries != nullptr && (!aligned16(queries) || !aligned16(out)))
    return fail(TTT_ERR_INVALID_ARG, "queries and out must be 16-byte aligned");
  if (loss != nullptr && !aligned16(loss)) return fail(TTT_ERR_INVALID_ARG, "loss_out must be 16-byte aligned");
  if (c.rule != TTT_RULE_LINEAR_GD || c.token_weights)
    return inner_scan(st, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(targets),
                      static_cast<const __nv_bfloat16*>(queries), T, static_cast<__nv_bfloat16*>(out), loss, s);
  if (c.gate_enable) {
    if (loss == nullptr) return fail(TTT_ERR_INVALID_ARG, "the gate needs loss_out");
    if (T % c.gate_chunk != 0) return fail(TTT_ERR_INVALID_ARG, "T must be a multiple of gate_chunk with the gate on");
    TTT_TRY(check_token_position(st, T));
  }
  TTT_TRY(linear_scan(st, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(targets),
                      static_cast<const __nv_bfloat16*>(queries), T, static_cast<__nv_bfloat16*>(out), loss, s));
  // The b = 16 scan runs the gate itself, tile by tile; the other mini-batch sizes hand the
  // losses to the standalone gate kernel.
  if (c.gate_enable && c.chunk != 16) TTT_TRY(gate_route(st, loss, T, s));
  return TTT_OK;
}

static ttt_status ensure_staging(ttt_state* st, int set, int i, size_t bytes) {
  HostStaging& hs = st->staging;
  if (hs.bytes[set][i] >= bytes) return TTT_OK;
  dev_free(hs.buf[set][i]);
  hs.buf[set][i] = nullptr;
  hs.bytes[set][i] = 0;
  TTT_TRY(dev_alloc(&hs.buf[set][i], bytes, "host-call staging buffer"));
  hs.bytes[set][i] = bytes;
  return TTT_OK;
}

static ttt_status ensure_pipeline(ttt_state* st) {
  HostStaging& hs = st->staging;
  if (hs.copy_out != nullptr) return TTT_OK;
  cudaEvent_t* evs[] = {&hs.entry, &hs.in_done[0], &hs.in_done[1], &hs.scan_done[0], &hs.scan_done[1],
                        &hs.out_done[0], &hs.out_done[1]};
  for (cudaEvent_t* e : evs)
    if (*e == nullptr) TTT_CUDA(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
  if (hs.copy_in == nullptr) TTT_CUDA(cudaStreamCreateWithFlags(&hs.copy_in, cudaStreamNonBlocking));
  TTT_CUDA(cudaStreamCreateWithFlags(&hs.copy_out, cudaStreamNonBlocking));
  return TTT_OK;
}

// Tokens of one segment of a host call: about a quarter of T (a few segments keep the copies
// of one busy while the scan of another runs), in whole units of what a call may end on (the
// chunk; the gate's 64-token chunk when the gate is on). The whole call where a call boundary
// would change the result (the fused target's taps past the call end, pad mode 1), and for the
// TTT-Linear family when it copies back less than a fifth of what it copies in: its scan is
// short next to the copies, so with only the losses coming back there is almost nothing for
// the segments to overlap, and each segment costs launches and strided copies of its own.
static int64_t host_segment(const ttt_config& c, int64_t T, size_t in_bytes, size_t out_bytes) {
  if (c.rule == TTT_RULE_INPLACE_HEBBIAN && c.target_mode == 1 && c.conv_pad_mode == 1) return T;
  if (c.rule != TTT_RULE_INPLACE_HEBBIAN && 5 * out_bytes < in_bytes) return T;
  int64_t unit = c.chunk;
  if (c.gate_enable) unit = unit * c.gate_chunk / std::gcd<int64_t>(unit, c.gate_chunk);
  int64_t seg = (T / 4 + unit - 1) / unit * unit;
  return seg < unit ? unit : (seg > T ? T : seg);
}

// Rows of `rows` [.., T, width] blocks (width bytes a token) between host and device memory for
// tokens [t0, t0 + n): the device side is the dense segment [.., n, width].
static ttt_status copy_segment(void* dst, const void* src, size_t width, int64_t T, int64_t t0, int64_t n,
                               size_t rows, bool to_device, cudaStream_t s) {
  if (n == T || rows == 1) {  // one contiguous range
    const size_t off = t0 * width, bytes = rows * n * width;
    if (to_device)
      TTT_CUDA(cudaMemcpyAsync(dst, static_cast<const uint8_t*>(src) + off, bytes, cudaMemcpyHostToDevice, s));
    else
      TTT_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(dst) + off, src, bytes, cudaMemcpyDeviceToHost, s));
    return TTT_OK;
  }
  if (to_device)
    TTT_CUDA(cudaMemcpy2DAsync(dst, n * width, static_cast<const uint8_t*>(src) + t0 * width, T * width, n * width,
                               rows, cudaMemcpyHostToDevice, s));
  else
    TTT_CUDA(cudaMemcpy2DAsync(static_cast<uint8_t*>(dst) + t0 * width, T * width, src, n * width, n * width, rows,
                               cudaMemcpyDeviceToHost, s));
  return TTT_OK;
}

// A named NVTX range around each call that enqueues a scan, so a timeline tool shows the
// library's calls beside their kernels (no cost without such a tool attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

}  // namespace ttt

using namespace ttt;

extern "C" {

int32_t ttt_abi_version(void) { return 2; }

const char* ttt_last_error_string(void) { return ttt::g_last_error; }

ttt_status ttt_config_init(ttt_config* cfg, int32_t rule) {
  if (cfg == nullptr) return fail(TTT_ERR_INVALID_ARG, "cfg is NULL");
  if (rule < TTT_RULE_INPLACE_HEBBIAN || rule > TTT_RULE_MLP_GD) return fail(TTT_ERR_INVALID_ARG, "unknown rule %d", rule);
  memset(cfg, 0, sizeof(*cfg));
  cfg->rule = rule;
  cfg->io_dtype = TTT_BF16;
  cfg->batch = 1;
  cfg->heads = 1;
  cfg->d_key = 64;
  cfg->d_val = 64;
  cfg->chunk = rule == TTT_RULE_INPLACE_HEBBIAN ? 1024 : 16;
  cfg->eta = 1.0f;
  cfg->conv_taps = 3;
  cfg->gate_chunk = 64;
  cfg->cache_capacity = 256;
  cfg->gate_pct = 0.95f;
  cfg->gate_ema_old = 0.9f;
  cfg->gate_ema_new = 0.1f;
  cfg->gate_mean_num = 4;
  cfg->gate_mean_den = 5;
  cfg->ln_eps = 1e-6f;
  return TTT_OK;
}

ttt_status ttt_state_create(const ttt_config* cfg, const void* W0, const void* Wtarget, const float* convw,
                            ttt_stream stream, ttt_state** out) {
  if (out == nullptr) return fail(TTT_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr) return fail(TTT_ERR_INVALID_ARG, "cfg is NULL");
  return create_impl(cfg, W0, Wtarget, convw, reinterpret_cast<cudaStream_t>(stream), out);
}

ttt_status ttt_chunk_scan(ttt_state* st, const void* keys, const void* targets, const void* queries, int64_t T,
                          void* out, float* loss_out, ttt_stream stream) {
  const CallRange range("ttt_chunk_scan");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  return scan_impl(st, keys, targets, queries, T, out, loss_out, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_chunk_scan_docs(ttt_state* st, const void* keys, const void* targets, int64_t T, void* out,
                               const int64_t* doc_starts, int32_t ndocs, float clip_norm, ttt_stream stream) {
  const CallRange range("ttt_chunk_scan_docs");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  const ttt_config& c = st->cfg;
  if (c.rule != TTT_RULE_INPLACE_HEBBIAN || c.io_dtype != TTT_BF16)
    return fail(TTT_ERR_UNSUPPORTED, "packed sequences of this call run In-Place BF16 states");
  if (T < 0 || T > (int64_t)INT32_MAX / 4) return fail(TTT_ERR_INVALID_ARG, "T out of range");
  if (!(clip_norm >= 0.f)) return fail(TTT_ERR_INVALID_ARG, "clip_norm must be >= 0 (0: no clipping)");
  if (T == 0) return TTT_OK;
  if (doc_starts == nullptr || ndocs < 1) return fail(TTT_ERR_INVALID_ARG, "doc_starts must list at least one document");
  if (doc_starts[0] != 0) return fail(TTT_ERR_INVALID_ARG, "the first document must start at token 0");
  for (int32_t k = 1; k < ndocs; ++k)
    if (doc_starts[k] <= doc_starts[k - 1])
      return fail(TTT_ERR_INVALID_ARG, "doc_starts must increase strictly (entry %d)", (int)k);
  if (doc_starts[ndocs - 1] >= T) return fail(TTT_ERR_INVALID_ARG, "every document must start below T");
  if (keys == nullptr || targets == nullptr || out == nullptr || !aligned16(keys) || !aligned16(targets) ||
      !aligned16(out))
    return fail(TTT_ERR_INVALID_ARG, "keys, targets and out must be 16-byte aligned device pointers");
  TTT_TRY(check_device(st));
  return inplace_bf16_scan_docs(st, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(targets),
                                T, doc_starts, (int)ndocs, clip_norm, static_cast<__nv_bfloat16*>(out),
                                reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_chunk_scan_packed(ttt_state* st, const void* keys, const void* targets, const void* queries, int64_t T,
                                 void* out, float* loss_out, const int64_t* doc_starts, const int32_t* docs_per_seq,
                                 ttt_stream stream) {
  const CallRange range("ttt_chunk_scan_packed");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  const ttt_config& c = st->cfg;
  if (c.rule == TTT_RULE_INPLACE_HEBBIAN)
    return fail(TTT_ERR_UNSUPPORTED, "In-Place states take packed sequences through ttt_chunk_scan_docs");
  if (c.chunk != 16 || c.gate_enable)
    return fail(TTT_ERR_UNSUPPORTED, "packed sequences: mini-batch 16, no gate");
  if (T < 0 || T > (int64_t)INT32_MAX / 4) return fail(TTT_ERR_INVALID_ARG, "T out of range");
  if (T == 0) return TTT_OK;
  if (doc_starts == nullptr || docs_per_seq == nullptr)
    return fail(TTT_ERR_INVALID_ARG, "doc_starts and docs_per_seq are required (host memory)");
  int64_t off = 0;
  for (int b = 0; b < c.batch; ++b) {
    const int32_t n = docs_per_seq[b];
    if (n < 1) return fail(TTT_ERR_INVALID_ARG, "sequence %d lists no document", b);
    if (doc_starts[off] != 0) return fail(TTT_ERR_INVALID_ARG, "sequence %d: the first document must start at 0", b);
    for (int32_t k = 1; k < n; ++k)
      if (doc_starts[off + k] <= doc_starts[off + k - 1])
        return fail(TTT_ERR_INVALID_ARG, "sequence %d: document starts must increase strictly", b);
    if (doc_starts[off + n - 1] >= T) return fail(TTT_ERR_INVALID_ARG, "sequence %d: every document must start below T", b);
    off += n;
  }
  if ((queries == nullptr) != (out == nullptr))
    return fail(TTT_ERR_INVALID_ARG, "out must be given exactly when queries are");
  const void* p[5] = {keys, targets, queries, out, loss_out};
  for (int i = 0; i < 5; ++i)
    if ((i < 2 && p[i] == nullptr) || (p[i] != nullptr && !aligned16(p[i])))
      return fail(TTT_ERR_INVALID_ARG, "keys and targets (and queries, out, loss_out when given) must be 16-byte aligned device pointers");
  TTT_TRY(check_device(st));
  return inner_scan_packed(st, static_cast<const __nv_bfloat16*>(keys), static_cast<const __nv_bfloat16*>(targets),
                           static_cast<const __nv_bfloat16*>(queries), T, static_cast<__nv_bfloat16*>(out), loss_out,
                           doc_starts, docs_per_seq, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_chunk_scan_host(ttt_state* st, const void* keys, const void* targets, const void* queries,
                               int64_t T, void* out, float* loss_out, ttt_stream stream) {
  const CallRange range("ttt_chunk_scan_host");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  const ttt_config& c = st->cfg;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T < 0 || T % c.chunk != 0) return fail(TTT_ERR_INVALID_ARG, "T must be a non-negative multiple of the chunk");
  if (T == 0) return TTT_OK;
  if (keys == nullptr || targets == nullptr) return fail(TTT_ERR_INVALID_ARG, "keys and targets are required");
  TTT_TRY(check_device(st));
  // Per token: bytes of a key, target and output row, over `rows` blocks of T tokens each
  // (In-Place: one [T, width] block; the TTT-Linear family: one block per (sequence, head)).
  const size_t es = io_size(c.io_dtype);
  const bool inplace = c.rule == TTT_RULE_INPLACE_HEBBIAN;
  const size_t rows = inplace ? 1 : (size_t)c.batch * c.heads;
  const size_t kw = (size_t)c.d_key * es, vw = (size_t)c.d_val * es, ow = (inplace ? c.d_val : c.d_key) * es;
  const size_t lw = sizeof(float);
  const void* hin[3] = {keys, targets, queries};
  void* hout[2] = {out, loss_out};
  const size_t win[3] = {kw, vw, kw}, wout[2] = {ow, lw};
  size_t in_bytes = 0, out_bytes = 0;
  for (int i = 0; i < 3; ++i) in_bytes += hin[i] != nullptr ? win[i] : 0;
  for (int i = 0; i < 2; ++i) out_bytes += hout[i] != nullptr ? wout[i] : 0;
  const int64_t seg = host_segment(c, T, in_bytes, out_bytes);
  for (int j = 0; j < (seg < T ? 2 : 1); ++j) {
    for (int i = 0; i < 3; ++i)
      if (hin[i] != nullptr) TTT_TRY(ensure_staging(st, j, i, rows * seg * win[i]));
    for (int i = 0; i < 2; ++i)
      if (hout[i] != nullptr) TTT_TRY(ensure_staging(st, j, 3 + i, rows * seg * wout[i]));
  }
  TTT_TRY(ensure_pipeline(st));
  HostStaging& hs = st->staging;
  // Segment k uses buffer set k mod 2. Its inputs go up on the copy-in stream once the scan of
  // segment k - 2 (the set's last reader) has ended; its scan runs on the caller's stream once
  // they are there and segment k - 2's outputs (the set's last contents) are back; its outputs
  // go down on the copy-out stream once its scan has ended. Each segment continues the scan
  // exactly as a separate call would.
  TTT_CUDA(cudaEventRecord(hs.entry, s));
  TTT_CUDA(cudaStreamWaitEvent(hs.copy_in, hs.entry, 0));
  TTT_CUDA(cudaStreamWaitEvent(hs.copy_out, hs.entry, 0));
  ttt_status r = TTT_OK;
  int k = 0;
  for (int64_t t0 = 0; t0 < T && r == TTT_OK; t0 += seg, ++k) {
    const int j = k & 1;
    const int64_t n = std::min<int64_t>(seg, T - t0);
    void** b = hs.buf[j];
    auto step = [&]() -> ttt_status {
      if (k >= 2) TTT_CUDA(cudaStreamWaitEvent(hs.copy_in, hs.scan_done[j], 0));
      for (int i = 0; i < 3; ++i)
        if (hin[i] != nullptr) TTT_TRY(copy_segment(b[i], hin[i], win[i], T, t0, n, rows, true, hs.copy_in));
      TTT_CUDA(cudaEventRecord(hs.in_done[j], hs.copy_in));
      TTT_CUDA(cudaStreamWaitEvent(s, hs.in_done[j], 0));
      if (k >= 2) TTT_CUDA(cudaStreamWaitEvent(s, hs.out_done[j], 0));
      TTT_TRY(scan_impl(st, b[0], b[1], queries ? b[2] : nullptr, n, out ? b[3] : nullptr,
                        loss_out ? static_cast<float*>(b[4]) : nullptr, s));
      TTT_CUDA(cudaEventRecord(hs.scan_done[j], s));
      TTT_CUDA(cudaStreamWaitEvent(hs.copy_out, hs.scan_done[j], 0));
      for (int i = 0; i < 2; ++i)
        if (hout[i] != nullptr) TTT_TRY(copy_segment(hout[i], b[3 + i], wout[i], T, t0, n, rows, false, hs.copy_out));
      TTT_CUDA(cudaEventRecord(hs.out_done[j], hs.copy_out));
      return TTT_OK;
    };
    r = step();
  }
  // Whatever happened, nothing of this call is left in flight when it returns.
  const cudaError_t e1 = cudaStreamSynchronize(hs.copy_in), e2 = cudaStreamSynchronize(s),
                    e3 = cudaStreamSynchronize(hs.copy_out);
  if (r != TTT_OK) return r;
  if (e1 != cudaSuccess) return cuda_fail(e1, "copy-in stream");
  if (e2 != cudaSuccess) return cuda_fail(e2, "scan stream");
  if (e3 != cudaSuccess) return cuda_fail(e3, "copy-out stream");
  return TTT_OK;
}

ttt_status ttt_surprisal_route(ttt_state* st, const float* loss, int64_t T, ttt_stream stream) {
  const CallRange range("ttt_surprisal_route");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  if (st->cfg.rule != TTT_RULE_LINEAR_GD) return fail(TTT_ERR_UNSUPPORTED, "the surprisal gate runs on TTT-Linear states");
  if (!st->cfg.gate_enable) return fail(TTT_ERR_INVALID_ARG, "the state was created with gate_enable = 0");
  if (T < 0 || T % st->cfg.gate_chunk != 0) return fail(TTT_ERR_INVALID_ARG, "T must be a non-negative multiple of gate_chunk");
  if (T == 0) return TTT_OK;
  if (loss == nullptr || !aligned16(loss)) return fail(TTT_ERR_INVALID_ARG, "loss must be a 16-byte aligned device pointer");
  TTT_TRY(check_token_position(st, T));
  TTT_TRY(check_device(st));
  return gate_route(st, loss, T, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_cache_attention(const ttt_state* st, const void* queries, const void* keys, const void* values,
                               const void* o_ttt, const float* alpha, int64_t T, void* out, ttt_stream stream) {
  const CallRange range("ttt_cache_attention");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  if (st->cfg.rule != TTT_RULE_LINEAR_GD || !st->cfg.gate_enable)
    return fail(TTT_ERR_UNSUPPORTED, "the cache read path needs a TTT-Linear state with the gate enabled");
  // T must equal the tokens gated since the reset. That count lives on the device (the kernel
  // checks it and reports a mismatch through ttt_state_poll); the host's count misses replays of
  // captured calls, so it can only show that T is too small.
  if (T <= 0 || T < st->gate.t_offset)
    return fail(TTT_ERR_INVALID_ARG, "T=%lld must equal the tokens scanned since the last reset (at least %lld)",
                (long long)T, (long long)st->gate.t_offset);
  const void* p[6] = {queries, keys, values, o_ttt, alpha, out};
  for (const void* x : p)
    if (x == nullptr || !aligned16(x))
      return fail(TTT_ERR_INVALID_ARG, "queries, keys, values, o_ttt, alpha and out must be 16-byte aligned device pointers");
  TTT_TRY(check_device(st));
  return cache_attention(st, static_cast<const __nv_bfloat16*>(queries), static_cast<const __nv_bfloat16*>(keys),
                         static_cast<const __nv_bfloat16*>(values), static_cast<const __nv_bfloat16*>(o_ttt), alpha, T,
                         static_cast<__nv_bfloat16*>(out), reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_state_reset(ttt_state* st, ttt_stream stream) {
  const CallRange range("ttt_state_reset");
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  TTT_TRY(check_device(st));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TTT_TRY(load_weights(st, st->cfg.rule == TTT_RULE_INPLACE_HEBBIAN ? st->ip.W0 : st->lin.W0, s));
  if (st->cfg.rule == TTT_RULE_LINEAR_GD) TTT_TRY(gate_reset(st, s));
  return TTT_OK;
}

ttt_status ttt_state_get_weights(const ttt_state* st, float* W, ttt_stream stream) {
  if (st == nullptr || W == nullptr) return fail(TTT_ERR_INVALID_ARG, "state and W are required");
  TTT_TRY(check_device(st));
  const float* src = st->cfg.rule == TTT_RULE_INPLACE_HEBBIAN ? st->ip.W : st->lin.W;
  TTT_CUDA(cudaMemcpyAsync(W, src, weight_elems(st->cfg) * 4, cudaMemcpyDeviceToDevice,
                           reinterpret_cast<cudaStream_t>(stream)));
  return TTT_OK;
}

ttt_status ttt_add_f32(float* y, const float* x, float alpha, int64_t n, ttt_stream stream) {
  if (n < 0) return fail(TTT_ERR_INVALID_ARG, "n must be non-negative");
  if (n == 0) return TTT_OK;
  if (y == nullptr || x == nullptr) return fail(TTT_ERR_INVALID_ARG, "y and x must be device pointers");
  int dev = 0, sms = 0;
  TTT_CUDA(cudaGetDevice(&dev));
  TTT_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  return add_f32(y, x, alpha, (size_t)n, sms, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_state_set_weights(ttt_state* st, const float* W, ttt_stream stream) {
  if (st == nullptr || W == nullptr || !aligned16(W)) return fail(TTT_ERR_INVALID_ARG, "state and an aligned W are required");
  TTT_TRY(check_device(st));
  return load_weights(st, W, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_state_set_layernorm(ttt_state* st, const float* gamma, const float* beta, ttt_stream stream) {
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  if (st->lin.ln_gamma == nullptr) return fail(TTT_ERR_UNSUPPORTED, "only the LayerNorm rules have a LayerNorm");
  if (gamma == nullptr || beta == nullptr || !aligned16(gamma) || !aligned16(beta))
    return fail(TTT_ERR_INVALID_ARG, "gamma and beta must be 16-byte aligned device pointers");
  TTT_TRY(check_device(st));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)st->cfg.heads * 64 * 4;
  TTT_CUDA(cudaMemcpyAsync(st->lin.ln_gamma, gamma, bytes, cudaMemcpyDeviceToDevice, s));
  TTT_CUDA(cudaMemcpyAsync(st->lin.ln_beta, beta, bytes, cudaMemcpyDeviceToDevice, s));
  return TTT_OK;
}

ttt_status ttt_cache_read(const ttt_state* st, int32_t* entries, int32_t* counts, ttt_stream stream) {
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  if (st->cfg.rule != TTT_RULE_LINEAR_GD) return fail(TTT_ERR_UNSUPPORTED, "only TTT-Linear states have a residual cache");
  TTT_TRY(check_device(st));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bh = (size_t)st->cfg.batch * st->cfg.heads;
  if (entries != nullptr)
    TTT_CUDA(cudaMemcpyAsync(entries, st->gate.entries, bh * st->cfg.cache_capacity * 3 * 4, cudaMemcpyDeviceToDevice, s));
  if (counts != nullptr) TTT_CUDA(cudaMemcpyAsync(counts, st->gate.counts, bh * 2 * 4, cudaMemcpyDeviceToDevice, s));
  return TTT_OK;
}

ttt_status ttt_gate_read(const ttt_state* st, float* tau, int32_t* tau_set, ttt_stream stream) {
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  if (st->cfg.rule != TTT_RULE_LINEAR_GD) return fail(TTT_ERR_UNSUPPORTED, "only TTT-Linear states have a gate");
  TTT_TRY(check_device(st));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bh = (size_t)st->cfg.batch * st->cfg.heads;
  if (tau != nullptr) TTT_CUDA(cudaMemcpyAsync(tau, st->gate.tau, bh * 4, cudaMemcpyDeviceToDevice, s));
  if (tau_set != nullptr) TTT_CUDA(cudaMemcpyAsync(tau_set, st->gate.tau_set, bh * 4, cudaMemcpyDeviceToDevice, s));
  return TTT_OK;
}

ttt_status ttt_state_poll(ttt_state* st) {
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  TTT_CUDA(cudaDeviceSynchronize());
  volatile int* w = st->status.host;
  const int v = w[0], site = w[1];
  w[0] = 0;
  w[1] = 0;
  if (v == 0) return TTT_OK;
  if (v == TTT_ERR_TIMEOUT)
    return fail(TTT_ERR_TIMEOUT, "a bounded device-side wait ran out (%s 0x%x)",
                (site & 0xF0000) == kSiteCounter ? "progress counter at word" : "mbarrier at shared offset",
                site & 0xFFFF);
  if ((site & 0xF0000) == kSiteTokenLimit)
    return fail(TTT_ERR_UNSUPPORTED, "the gate's token position passed 2^31 - 1 (sequence-head %d; reset the state)",
                site & 0xFFFF);
  if ((site & 0xF0000) == kSiteCacheLength)
    return fail(TTT_ERR_INVALID_ARG, "the cache read's T is not the number of tokens gated since the last reset "
                "(sequence-head %d)", site & 0xFFFF);
  return fail(TTT_ERR_DEVICE, "a device-side check failed (code %d)", v);
}

ttt_status ttt_state_set_option(ttt_state* st, int32_t option, int64_t value) {
  if (st == nullptr) return fail(TTT_ERR_INVALID_ARG, "state is NULL");
  switch (option) {
    case TTT_OPT_LINEAR_CHUNK:
      if (value != 0 && value != 1 && value != 2 && value != 4)
        return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_LINEAR_CHUNK must be 0, 1, 2 or 4 (got %lld)", (long long)value);
      st->lin.form = (int)value;
      return TTT_OK;
    case TTT_OPT_WAIT_LIMIT_NS:
      if (value < 1000 || value > 60000000000ll)
        return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_WAIT_LIMIT_NS must lie in [1000, 6e10] (got %lld)", (long long)value);
      st->wait_limit_ns = (uint64_t)value;
      return TTT_OK;
    case TTT_OPT_INPLACE_PREFIX:
      if (value != 0 && value != 1) return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_INPLACE_PREFIX must be 0 or 1");
      if (value == 1 && (st->cfg.rule != TTT_RULE_INPLACE_HEBBIAN || st->cfg.io_dtype != TTT_BF16 ||
                         st->cfg.target_mode != 0))
        return fail(TTT_ERR_UNSUPPORTED, "the context-parallel form runs In-Place BF16 states with given targets");
      st->ip.prefix_form = (int)value;
      return TTT_OK;
    case TTT_OPT_SM_PAIR:
      if (value != 0 && value != 1) return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_SM_PAIR must be 0 or 1");
      if (st->ip.sm_pair != (int)value) {
        st->ip.sm_pair = (int)value;
        free_tc(st);  // schedules are built per tile shape; rebuilt on the next scan
      }
      return TTT_OK;
    case TTT_OPT_INJECT_STALL:
      if (value != 0 && value != 1) return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_INJECT_STALL must be 0 or 1");
      st->inject_stall = (int)value;
      return TTT_OK;
    case TTT_OPT_GATE_TOKENS: {
      if (st->cfg.rule == TTT_RULE_INPLACE_HEBBIAN || st->gate.tokens == nullptr)
        return fail(TTT_ERR_UNSUPPORTED, "TTT_OPT_GATE_TOKENS applies to TTT-Linear states");
      if (value < 0 || value > (int64_t)INT32_MAX)
        return fail(TTT_ERR_INVALID_ARG, "TTT_OPT_GATE_TOKENS must lie in [0, 2^31 - 1]");
      TTT_TRY(check_device(st));
      const size_t bh = (size_t)st->cfg.batch * st->cfg.heads;
      std::vector<int64_t> v(bh, value);
      TTT_CUDA(cudaDeviceSynchronize());
      TTT_CUDA(cudaMemcpy(st->gate.tokens, v.data(), bh * sizeof(int64_t), cudaMemcpyHostToDevice));
      return TTT_OK;
    }
    default:
      return fail(TTT_ERR_INVALID_ARG, "unknown option %d", option);
  }
}

int64_t ttt_state_launch_count(const ttt_state* st) { return st == nullptr ? 0 : st->launches; }

ttt_status ttt_state_destroy(ttt_state* st) {
  if (st == nullptr) return TTT_OK;
  cudaError_t e = cudaDeviceSynchronize();
  free_state(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize in destroy");
  return TTT_OK;
}

}  // extern "C"
