// Context-parallel form of the In-Place scan ("In-Place Test-Time Training", §6: the chunk
// updates are additive, so every chunk's ΔW_j is computed in parallel, an exclusive prefix sum
// gives each chunk the cumulative update before it, and then every chunk's outputs are
// computed in parallel with its effective weight W_c = W_0 + η·Σ_{j<c} ΔW_j).
//
// Three launches per scan call of n chunks, none of which waits on another chunk:
//   1. k_gemm_tc, batched over the chunks: D_j = η·V̂_jᵀ·Z_j (fp32 [n][d][f]);
//   2. k_prefix_w: W_j = W_0 + Σ_{i<j} D_i, stored as bf16 [n][d][f] (the weight chunk j
//      applies with); the fp32 sum after the last chunk becomes the state's weight;
//   3. k_gemm_tc, batched over the chunks: O_j = Z_j·W_jᵀ (bf16).
// It computes the same outputs and final weight as the sequential scan (the sums are taken in
// the same order; each η·ΔW_j is rounded to fp32 before it is added) and is the form that
// shards the sequence over devices; on one device it moves more data (the n fp32 deltas and
// the n bf16 weights go through HBM) in exchange for launches without cross-chunk waits.
//
// k_gemm_tc is a plain batched GEMM on the 5th-generation tensor cores: one CTA per 128x256
// output tile, TMA loads (128-byte swizzle) into a 3-stage ring, one thread issuing
// tcgen05.mma (M=128, N=256, K=16) into a TMEM accumulator, four epilogue warps (one per TMEM
// lane quarter) scaling and storing rows. Operands are K-major or MN-major as stored.
#include <vector>

#include "internal.h"
#include "tc_common.cuh"

namespace ttt {

namespace {

constexpr int GM = 128, GN = 256, GK = 64, kGSt = 3;
constexpr int kGA = GM * GK * 2;  // 16 KB of A per stage
constexpr int kGB = GN * GK * 2;  // 32 KB of B per stage
constexpr int kGThreads = 6 * 32;  // TMA producer, MMA issuer, 4 epilogue warps
constexpr int kGTmemCols = 256;

struct __align__(1024) GemmSmem {
  uint8_t A[kGSt][kGA];
  uint8_t B[kGSt][kGB];
  uint64_t full[kGSt], empty[kGSt], tfull;
  uint32_t tmem;
  int abort;
};

struct GemmArgs {
  int M, N, K;         // per batch item
  int a_mn, b_mn;      // operand stored MN-major (its M or N index contiguous) rather than K-major
  int a_outer, b_outer;  // outer tensor-map coordinate of batch item 1 (item b starts at b times it)
  void* out;           // [batch][M][ldo], fp32 (out_f32) or bf16
  int out_f32;
  long long out_batch;  // elements between batch items of out
  int ldo;
  float scale;         // out = scale · A·B
  DevStatus status;
};

__global__ void __launch_bounds__(kGThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (g.N + GN - 1) / GN;
  const int tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n, b = blockIdx.y;
  const int nk = (g.K + GK - 1) / GK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGSt; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(&sm.tfull, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tc::alloc(&sm.tmem, kGTmemCols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = sm.tmem;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int s = kb % kGSt;
        if (kb >= kGSt && !mbar_wait(&sm.empty[s], ((kb / kGSt) - 1) & 1, g.status, abort)) break;
        mbar_arrive_expect_tx(&sm.full[s], kGA + kGB);
        if (!g.a_mn) {
          tma_load_2d(sm.A[s], &tmA, &sm.full[s], kb * GK, b * g.a_outer + tm * GM);
        } else {
          for (int j = 0; j < GM / 64; ++j)
            tma_load_2d(sm.A[s] + j * 8192, &tmA, &sm.full[s], tm * GM + j * 64, b * g.a_outer + kb * GK);
        }
        if (!g.b_mn) {
          tma_load_2d(sm.B[s], &tmB, &sm.full[s], kb * GK, b * g.b_outer + tn * GN);
        } else {
          for (int j = 0; j < GN / 64; ++j)
            tma_load_2d(sm.B[s] + j * 8192, &tmB, &sm.full[s], tn * GN + j * 64, b * g.b_outer + kb * GK);
        }
      }
      // Nothing may still be landing in shared memory when the CTA exits.
      for (int k = kb > kGSt ? kb - kGSt : 0; k < kb; ++k) mbar_wait(&sm.full[k % kGSt], (k / kGSt) & 1, g.status, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(GM, GN, g.a_mn, g.b_mn);
      int kb = 0;
      bool ok = true;
      for (; kb < nk; ++kb) {
        const int s = kb % kGSt;
        if (!mbar_wait(&sm.full[s], (kb / kGSt) & 1, g.status, abort)) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t a0 = smem_u32(sm.A[s]), b0 = smem_u32(sm.B[s]);
#pragma unroll
        for (int kk = 0; kk < GK / 16; ++kk) {
          const uint64_t ad = g.a_mn ? tc::smem_desc(a0 + kk * 2048, 8192, 1024) : tc::smem_desc(a0 + kk * 32, 16, 1024);
          const uint64_t bd = g.b_mn ? tc::smem_desc(b0 + kk * 2048, 8192, 1024) : tc::smem_desc(b0 + kk * 32, 16, 1024);
          tc::mma(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        tc::commit(&sm.empty[s]);  // frees the stage once these MMAs have read it
      }
      if (ok) {
        tc::commit(&sm.tfull);
        // The epilogue's wait covers the MMAs; this thread waits too, so TMEM is not freed early.
        mbar_wait(&sm.tfull, 0, g.status, nullptr);
      } else if (kb > 0) {
        mbar_wait(&sm.empty[(kb - 1) % kGSt], ((kb - 1) / kGSt) & 1, g.status, nullptr);
      }
    }
  } else {
    // Epilogue: warp w reads TMEM lane quarter w % 4, i.e. tile rows 32(w % 4) .. +31.
    const int q = warp & 3;
    bool ok = mbar_wait(&sm.tfull, 0, g.status, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc::fence_after();
      const int row = tm * GM + q * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int jc = 0; jc < GN / 32; ++jc) {
        uint32_t r[32];
        tc::ld32(tbase + jc * 32, r);
        tc::wait_ld();
        const int col0 = tn * GN + jc * 32;
        if (row >= g.M || col0 >= g.N) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = g.scale * __uint_as_float(r[j]);
        if (g.out_f32) {
          float* dst = static_cast<float*>(g.out) + b * g.out_batch + (long long)row * g.ldo + col0;
          if (col0 + 32 <= g.N) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<float4*>(dst)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            for (int j = 0; j < 32 && col0 + j < g.N; ++j) dst[j] = v[j];
          }
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.out) + b * g.out_batch + (long long)row * g.ldo + col0;
          if (col0 + 32 <= g.N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 w;
              w.x = pack_bf16(v[8 * j + 0], v[8 * j + 1]);
              w.y = pack_bf16(v[8 * j + 2], v[8 * j + 3]);
              w.z = pack_bf16(v[8 * j + 4], v[8 * j + 5]);
              w.w = pack_bf16(v[8 * j + 6], v[8 * j + 7]);
              reinterpret_cast<uint4*>(dst)[j] = w;
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < g.N; ++j) dst[j] = __float2bfloat16_rn(v[j]);
          }
        }
      }
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 1) tc::dealloc(tmem, kGTmemCols);
}

// W_j (bf16) = W_0 + Σ_{i<j} s_i·D_i for j = 0 .. n−1, then W ← W_0 + Σ_i s_i·D_i (fp32) and
// its bf16 copy. Four consecutive elements a thread; the sum over the chunks runs in chunk
// order. Packed sequences: where reset[j] is set the sum restarts from Wreset (a document's
// first chunk), and with sumsq given s_i = clip / ‖D_i‖_F when that norm exceeds clip (else
// 1, as without sumsq: the plain form's sums are bit for bit those of W + D). The final bf16
// copy goes to the state's current copy, whose index the device holds (ring[0]).
struct BfCopies {
  __nv_bfloat16* w[3];
  const int* ring;
};

__global__ void k_prefix_w(const float* W0, const float* __restrict__ D, __nv_bfloat16* __restrict__ Wb, float* Wout,
                           const BfCopies copies, long long nelem, int n, const int32_t* __restrict__ reset,
                           const float* __restrict__ Wreset, const double* __restrict__ sumsq, float clip) {
  const long long n4 = nelem / 4;
  __nv_bfloat16* Wcopy = copies.w[*copies.ring];
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(W0)[i];
    for (int j = 0; j < n; ++j) {
      if (reset != nullptr && reset[j]) acc = reinterpret_cast<const float4*>(Wreset)[i];
      uint2 w;
      w.x = pack_bf16(acc.x, acc.y);
      w.y = pack_bf16(acc.z, acc.w);
      reinterpret_cast<uint2*>(Wb + (long long)j * nelem)[i] = w;
      float sc = 1.0f;
      if (sumsq != nullptr) {
        const double nrm = sqrt(sumsq[j]);
        if (nrm > (double)clip) sc = (float)((double)clip / nrm);
      }
      const float4 dj = reinterpret_cast<const float4*>(D + (long long)j * nelem)[i];
      acc.x = fmaf(sc, dj.x, acc.x);
      acc.y = fmaf(sc, dj.y, acc.y);
      acc.z = fmaf(sc, dj.z, acc.z);
      acc.w = fmaf(sc, dj.w, acc.w);
    }
    reinterpret_cast<float4*>(Wout)[i] = acc;
    uint2 w;
    w.x = pack_bf16(acc.x, acc.y);
    w.y = pack_bf16(acc.z, acc.w);
    reinterpret_cast<uint2*>(Wcopy)[i] = w;
  }
}

// Row r of the padded layout (`width` bf16 elements, a multiple of 8) ← row rows[r] of the input,
// or zeros where rows[r] < 0 (the padding that fills a document's last chunk).
__global__ void k_gather_rows(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                              const int32_t* __restrict__ rows, long long nrows, int width) {
  const int v = width / 8;  // 16-byte vectors a row
  const long long n = nrows * v;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / v;
    const int c = (int)(i % v);
    const int32_t from = rows[r];
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (from >= 0) x = reinterpret_cast<const uint4*>(src + (long long)from * width)[c];
    reinterpret_cast<uint4*>(dst + r * width)[c] = x;
  }
}

// Row rows[r] of the output ← row r of the padded layout, for every r that is not padding.
__global__ void k_scatter_rows(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               const int32_t* __restrict__ rows, long long nrows, int width) {
  const int v = width / 8;
  const long long n = nrows * v;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / v;
    const int32_t to = rows[r];
    if (to >= 0) reinterpret_cast<uint4*>(dst + (long long)to * width)[i % v] = reinterpret_cast<const uint4*>(src + r * width)[i % v];
  }
}

// sumsq[j] += Σ D_j² over this block's share of chunk j (blockIdx.y), float partials per thread,
// a double per block.
__global__ void k_chunk_sumsq(const float* __restrict__ D, long long nelem, double* __restrict__ sumsq) {
  const float4* d = reinterpret_cast<const float4*>(D + (long long)blockIdx.y * nelem);
  const long long n4 = nelem / 4;
  float acc = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 x = d[i];
    acc = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, acc))));
  }
  __shared__ double part[32];
  double v = acc;
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(&sumsq[blockIdx.y], t);
  }
}

ttt_status map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in, uint32_t box_out) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {inner * 2};
  const uint32_t box[2] = {box_in, box_out};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

ttt_status gemm(ttt_state* st, const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& g, int batch,
                cudaStream_t s) {
  const size_t smem = sizeof(GemmSmem) + 1024;
  TTT_CUDA(cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const dim3 grid((unsigned)(((g.M + GM - 1) / GM) * ((g.N + GN - 1) / GN)), (unsigned)batch);
  k_gemm_tc<<<grid, kGThreads, smem, s>>>(ta, tb, g);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace

ttt_status inplace_bf16_scan_prefix(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* Vhat, int64_t T,
                                    __nv_bfloat16* O, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const int d = c.d_val, f = c.d_key, C = c.chunk;
  const int n = (int)(T / C);
  const size_t nelem = (size_t)d * f;
  InplaceBuffers& ip = st->ip;
  if (ip.prefix_chunks < n) {
    if (ip.prefix_D) cudaFree(ip.prefix_D);
    if (ip.prefix_Wb) cudaFree(ip.prefix_Wb);
    ip.prefix_D = nullptr;
    ip.prefix_Wb = nullptr;
    ip.prefix_chunks = 0;
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&ip.prefix_D), (size_t)n * nelem * 4));
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&ip.prefix_Wb), (size_t)n * nelem * 2));
    ip.prefix_chunks = n;
  }
  const DevStatus ds{st->status.dev, st->wait_limit_ns, st->status.dev + 1};

  // 1. D_j = η·V̂_jᵀ·Z_j: M = d, N = f, K = C; A = V̂ (MN-major), B = Z (MN-major), batch j at token jC.
  CUtensorMap tV, tZm;
  TTT_TRY(map_bf16(&tV, Vhat, d, T, 64, 64));
  TTT_TRY(map_bf16(&tZm, Z, f, T, 64, 64));
  GemmArgs ga{d, f, C, 1, 1, C, C, ip.prefix_D, 1, (long long)nelem, f, c.eta, ds};
  TTT_TRY(gemm(st, tV, tZm, ga, n, s));

  // 2. Exclusive prefix sums: the weight each chunk applies with, and the final weight.
  const long long n4 = (long long)(nelem / 4);
  const int blocks = (int)std::min<long long>((n4 + 255) / 256, (long long)st->num_sms * 8);
  k_prefix_w<<<blocks, 256, 0, s>>>(ip.W, ip.prefix_D, ip.prefix_Wb, ip.W,
                                    BfCopies{{ip.Wsh[0], ip.Wsh[1], ip.Wsh[2]}, ip.ring}, (long long)nelem, n, nullptr,
                                    nullptr, nullptr, 0.f);
  st->launches++;
  TTT_CUDA(cudaGetLastError());

  // 3. O_j = Z_j·W_jᵀ: M = C, N = d, K = f; A = Z (K-major), B = W_j (K-major, rows jd ..).
  CUtensorMap tZk, tW;
  TTT_TRY(map_bf16(&tZk, Z, f, T, 64, 128));
  TTT_TRY(map_bf16(&tW, ip.prefix_Wb, f, (uint64_t)n * d, 64, 256));
  GemmArgs gc{C, d, f, 0, 0, C, d, O, 0, (long long)C * d, d, 1.0f, ds};
  return gemm(st, tZk, tW, gc, n, s);
}

namespace {

template <class T>
ttt_status grow(T** p, size_t count) {
  if (*p) cudaFree(*p);
  *p = nullptr;
  TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T)));
  return TTT_OK;
}

}  // namespace

ttt_status inplace_bf16_scan_docs(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* Vhat, int64_t T,
                                  const int64_t* doc_starts, int ndocs, float clip, __nv_bfloat16* O,
                                  cudaStream_t s) {
  const ttt_config& c = st->cfg;
  const int d = c.d_val, f = c.d_key, C = c.chunk;
  const size_t nelem = (size_t)d * f;
  InplaceBuffers& ip = st->ip;
  // Padded layout: every document starts a chunk and fills its last chunk with zero rows (a
  // zero row of Z and V̂ adds nothing to the delta, and its output row is dropped). With the
  // target made here (`targets` is X0), the targets come from the padded X0: in pad mode 0 the
  // taps stop at each chunk end, which the layout aligns with the documents; in pad mode 1 they
  // stop only at the end of the layout, so each document is followed by at least taps − 1 zero
  // rows (one more chunk of padding where its last chunk has fewer spare rows), which its last
  // tokens' taps read instead of the next document.
  const bool target = c.target_mode == 1;
  const int64_t tail = target && c.conv_pad_mode == 1 ? c.conv_taps - 1 : 0;
  std::vector<int32_t> rows, reset;
  for (int k = 0; k < ndocs; ++k) {
    const int64_t a = doc_starts[k], e = k + 1 < ndocs ? doc_starts[k + 1] : T;
    const int64_t nch = (e - a + tail + C - 1) / C;
    for (int64_t j = 0; j < nch; ++j) {
      reset.push_back(j == 0 ? 1 : 0);
      for (int r = 0; r < C; ++r) {
        const int64_t t = a + j * C + r;
        rows.push_back(t < e ? (int32_t)t : -1);
      }
    }
  }
  const int n = (int)reset.size();
  const int64_t Tp = (int64_t)n * C;
  if (Tp > (int64_t)INT32_MAX / 2) return fail(TTT_ERR_UNSUPPORTED, "padded length too large");
  if (ip.docs_rows_cap < Tp) {
    ip.docs_rows_cap = 0;  // until every buffer below has its new size
    TTT_TRY(grow(&ip.docs_Z, (size_t)Tp * f));
    TTT_TRY(grow(&ip.docs_V, (size_t)Tp * d));
    TTT_TRY(grow(&ip.docs_O, (size_t)Tp * d));
    TTT_TRY(grow(&ip.docs_rows, (size_t)Tp));
    ip.docs_rows_cap = Tp;
  }
  if (ip.docs_chunks_cap < n) {
    ip.docs_chunks_cap = 0;
    TTT_TRY(grow(&ip.docs_reset, (size_t)n));
    TTT_TRY(grow(&ip.docs_sumsq, (size_t)n));
    ip.docs_chunks_cap = n;
  }
  if (ip.prefix_chunks < n) {
    if (ip.prefix_D) cudaFree(ip.prefix_D);
    if (ip.prefix_Wb) cudaFree(ip.prefix_Wb);
    ip.prefix_D = nullptr;
    ip.prefix_Wb = nullptr;
    ip.prefix_chunks = 0;
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&ip.prefix_D), (size_t)n * nelem * 4));
    TTT_CUDA(cudaMalloc(reinterpret_cast<void**>(&ip.prefix_Wb), (size_t)n * nelem * 2));
    ip.prefix_chunks = n;
  }
  // The maps go up with the stream's work (pageable copies: staged by the driver before return).
  TTT_CUDA(cudaMemcpyAsync(ip.docs_rows, rows.data(), rows.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  TTT_CUDA(cudaMemcpyAsync(ip.docs_reset, reset.data(), reset.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  const DevStatus ds{st->status.dev, st->wait_limit_ns, st->status.dev + 1};
  const int gblocks = st->num_sms * 8;
  k_gather_rows<<<gblocks, 256, 0, s>>>(Z, ip.docs_Z, ip.docs_rows, (long long)Tp, f);
  k_gather_rows<<<gblocks, 256, 0, s>>>(Vhat, ip.docs_V, ip.docs_rows, (long long)Tp, d);
  st->launches += 2;
  TTT_CUDA(cudaGetLastError());
  const __nv_bfloat16* Vp = ip.docs_V;  // the padded targets
  if (target) {
    const int64_t plan = target_values_plan_ints((int)Tp, d, st->num_sms);
    if (ip.docs_target_cap < Tp) {
      ip.docs_target_cap = 0;
      TTT_TRY(grow(&ip.docs_conv, (size_t)Tp * d));
      TTT_TRY(grow(&ip.docs_T, (size_t)Tp * d));
      ip.docs_target_cap = Tp;
    }
    if (ip.docs_plan_cap < plan) {
      ip.docs_plan_cap = 0;
      TTT_TRY(grow(&ip.docs_plan, (size_t)plan));
      ip.docs_plan_cap = plan;
    }
    TTT_TRY(target_values_into(ip.docs_V, ip.convw, ip.Wtarget, (int)Tp, d, C, c.conv_taps, c.conv_pad_mode,
                               ip.docs_conv, ip.docs_plan, ip.docs_T, st->status.dev, st->num_sms, s));
    st->launches += 3;
    Vp = ip.docs_T;
  }

  // 1. D_j = η·V̂_jᵀ·Z_j over the padded chunks.
  CUtensorMap tV, tZm;
  TTT_TRY(map_bf16(&tV, Vp, d, Tp, 64, 64));
  TTT_TRY(map_bf16(&tZm, ip.docs_Z, f, Tp, 64, 64));
  GemmArgs ga{d, f, C, 1, 1, C, C, ip.prefix_D, 1, (long long)nelem, f, c.eta, ds};
  TTT_TRY(gemm(st, tV, tZm, ga, n, s));

  // 2. Norms of the deltas (clipping), then the sums restarting at each document's first chunk.
  if (clip > 0.f) {
    TTT_CUDA(cudaMemsetAsync(ip.docs_sumsq, 0, (size_t)n * sizeof(double), s));
    const long long n4 = (long long)(nelem / 4);
    const int bx = (int)std::max<long long>(1, std::min<long long>((n4 + 255) / 256, (st->num_sms * 8 + n - 1) / n));
    k_chunk_sumsq<<<dim3(bx, n), 256, 0, s>>>(ip.prefix_D, (long long)nelem, ip.docs_sumsq);
    st->launches++;
    TTT_CUDA(cudaGetLastError());
  }
  const long long n4 = (long long)(nelem / 4);
  const int blocks = (int)std::min<long long>((n4 + 255) / 256, (long long)st->num_sms * 8);
  k_prefix_w<<<blocks, 256, 0, s>>>(ip.W0, ip.prefix_D, ip.prefix_Wb, ip.W,
                                    BfCopies{{ip.Wsh[0], ip.Wsh[1], ip.Wsh[2]}, ip.ring}, (long long)nelem, n,
                                    ip.docs_reset, ip.W0, clip > 0.f ? ip.docs_sumsq : nullptr, clip);
  st->launches++;
  TTT_CUDA(cudaGetLastError());

  // 3. O_j = Z_j·W_jᵀ over the padded chunks, then the rows of the documents back in place.
  CUtensorMap tZk, tW;
  TTT_TRY(map_bf16(&tZk, ip.docs_Z, f, Tp, 64, 128));
  TTT_TRY(map_bf16(&tW, ip.prefix_Wb, f, (uint64_t)n * d, 64, 256));
  GemmArgs gc{C, d, f, 0, 0, C, d, ip.docs_O, 0, (long long)C * d, d, 1.0f, ds};
  TTT_TRY(gemm(st, tZk, tW, gc, n, s));
  k_scatter_rows<<<gblocks, 256, 0, s>>>(ip.docs_O, O, ip.docs_rows, (long long)Tp, d);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
