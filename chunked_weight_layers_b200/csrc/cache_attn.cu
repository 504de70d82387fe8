// Read path of the SR-TTT residual cache ("SR-TTT: Surprisal-Aware Residual Test-Time Training",
// §2.1, "Residual Cache" and "Alpha Fusion"): the layer's output is the TTT output plus the
// attention output over the cached tokens, weighted by a gate vector α clamped to [0, 1]:
//   out[t] = o_ttt[t] + clamp(α, 0, 1) ⊙ Σ_j softmax_j(q_t·k_j / √64)·v_j,
// over the cache entries j of the token's (sequence, head) that a query at t may see: a token's
// routing is known once its whole 64-token gate chunk has been scanned, so t sees the entries
// whose gate chunk lies before its own. Keys and values are the scan's own K and V rows of the
// cached tokens; a query that sees no entry adds nothing.
//
// Design (B200): the cache stores its tokens in increasing order, so the entries a query block
// of one gate chunk g sees are a prefix of the cache (those with token < 64g). One CTA takes one
// (sequence, head) and kQPerCta consecutive 64-query blocks: it gathers the prefix its last
// block sees (at most the capacity, 256 by default) of cached K and V rows into shared memory
// once, with asynchronous 16-byte copies (cp.async) so every row is in flight at once, and
// loads each block's queries the same way while the block before computes. Each of its four
// warps runs 16 queries through blocks of 64 keys with mma.sync (bf16 operands, fp32
// accumulation): S = Q·Kᵀ, an online softmax in fp32, A += P·V. The work is small against the
// scan (at most 256 keys a query) and has no serial dependence between query blocks, so it
// spreads over all SMs.
#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int kQBlk = 64;       // queries per block (one gate chunk)
constexpr int kQPerCta = 8;     // query blocks per CTA
constexpr int kKBlk = 64;       // keys per online-softmax block
constexpr int kMaxKeys = 256;   // cache capacity this kernel accepts
constexpr int kThreadsCA = 128;

struct __align__(1024) CacheAttnSmem {
  uint8_t Q[2][kQBlk * 128];     // 64 queries x 64 bf16, 128-byte swizzle, double-buffered
  uint8_t K[kMaxKeys * 128];     // cached keys, same layout
  uint8_t V[kMaxKeys * 128];     // cached values
  int warp_seen[kThreadsCA / 32];  // visible entries counted by each warp
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

// Asynchronous copy of 16-byte chunk `chunk` of the 64-element bf16 row `src` into row `row` of
// a swizzled tile.
__device__ __forceinline__ void put_row_async(uint8_t* tile, int row, const __nv_bfloat16* src, int chunk) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(tile + row * 128 + ((chunk ^ (row & 7)) << 4))),
               "l"(src + 8 * chunk)
               : "memory");
}

__device__ __forceinline__ void zero_row(uint8_t* tile, int row, int chunk) {
  *reinterpret_cast<uint4*>(tile + row * 128 + ((chunk ^ (row & 7)) << 4)) = make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// grid (query blocks, batch·heads), 128 threads. `alpha` [heads, 64] fp32 (clamped here).
__global__ void __launch_bounds__(kThreadsCA) k_cache_attn(const __nv_bfloat16* __restrict__ Q,
                                                           const __nv_bfloat16* __restrict__ K,
                                                           const __nv_bfloat16* __restrict__ V,
                                                           const __nv_bfloat16* O_ttt, const float* __restrict__ alpha,
                                                           const int32_t* __restrict__ entries,
                                                           const int32_t* __restrict__ counts,
                                                           const int64_t* __restrict__ tokens, int T, int heads,
                                                           int capacity, __nv_bfloat16* out, const DevStatus status) {
  extern __shared__ uint8_t smem_raw[];
  CacheAttnSmem& sm =
      *reinterpret_cast<CacheAttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = (T + kQBlk - 1) / kQBlk;
  const int qb0 = blockIdx.x * kQPerCta, qb1 = min(nblk, qb0 + kQPerCta);
  const size_t base = (size_t)bh * T * 64;
  const int32_t* E = entries + (size_t)bh * capacity * 3;
  const int n = min(counts[2 * bh], capacity);
  // The cache holds positions of the tokens gated since the reset, which the caller's arrays
  // must span exactly (positions past T are skipped below whatever the outcome).
  if (blockIdx.x == 0 && threadIdx.x == 0 && tokens[bh] != (int64_t)T)
    record_status(status, kDevInvalidArg, kSiteCacheLength | (bh & 0xFFFF));

  // Entries a block at token t0 sees: those of tokens before its gate chunk (a prefix of the
  // cache, which holds its tokens in increasing order).
  auto visible = [&](int t0) {
    int seen = 0;
    for (int j = threadIdx.x; j < n; j += kThreadsCA) seen += E[3 * j + 2] < t0 ? 1 : 0;
    seen = __reduce_add_sync(0xffffffffu, seen);
    __syncthreads();  // the previous use of warp_seen is over
    if (lane == 0) sm.warp_seen[warp] = seen;
    __syncthreads();
    return sm.warp_seen[0] + sm.warp_seen[1] + sm.warp_seen[2] + sm.warp_seen[3];
  };
  // Queries of block qb into buffer qbuf (rows past T zero).
  auto load_q = [&](int qb, int qbuf) {
    const int t0 = qb * kQBlk, nq = min(kQBlk, T - t0);
    for (int i = threadIdx.x; i < kQBlk * 8; i += kThreadsCA) {
      const int r = i / 8, c = i % 8;
      if (r < nq) put_row_async(sm.Q[qbuf], r, Q + base + (size_t)(t0 + r) * 64, c);
      else zero_row(sm.Q[qbuf], r, c);
    }
    cp_async_commit();
  };

  // The keys and values every block of this CTA may need: the prefix its last block sees.
  const int mmax = visible((qb1 - 1) * kQBlk);
  const int mpad_max = (mmax + kKBlk - 1) / kKBlk * kKBlk;
  load_q(qb0, 0);
  for (int i = threadIdx.x; i < mpad_max * 8; i += kThreadsCA) {
    const int r = i / 8, c = i % 8;
    const int tok = r < mmax ? E[3 * r + 2] : -1;
    if (tok >= 0 && tok < T) {
      put_row_async(sm.K, r, K + base + (size_t)tok * 64, c);
      put_row_async(sm.V, r, V + base + (size_t)tok * 64, c);
    } else {
      zero_row(sm.K, r, c);
      zero_row(sm.V, r, c);
    }
  }
  cp_async_commit();

  const int g = lane >> 2, q = lane & 3, mi = lane >> 3, ri = lane & 7;
  const uint32_t ks = smem_u32(sm.K), vs = smem_u32(sm.V);
  const float* al = alpha + (size_t)(bh % heads) * 64;
  // Scores are scaled by 1/√64 = 1/8 and taken in base 2 for exp2f.
  const float kScaleLog2 = 0.125f * 1.4426950408889634f;

  for (int qb = qb0; qb < qb1; ++qb) {
    const int buf = (qb - qb0) & 1;
    const int t0 = qb * kQBlk, nq = min(kQBlk, T - t0);
    const int m = visible(t0);  // also orders the previous block's reads of the other Q buffer
    if (qb + 1 < qb1) {
      load_q(qb + 1, buf ^ 1);
      cp_async_wait<1>();  // everything but the next block's queries has landed
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    if (m == 0) {
      // Nothing visible: out = o_ttt.
      if (out != O_ttt) {
        for (int i = threadIdx.x; i < nq * 8; i += kThreadsCA) {
          const size_t o = base + (size_t)(t0 + i / 8) * 64 + 8 * (i % 8);
          *reinterpret_cast<uint4*>(out + o) = *reinterpret_cast<const uint4*>(O_ttt + o);
        }
      }
      continue;
    }
    const int mpad = (m + kKBlk - 1) / kKBlk * kKBlk;

    // Warp w: queries 16w .. 16w+15 of the block. Thread (g, q) holds rows g and g+8.
    const uint32_t qs = smem_u32(sm.Q[buf]);
    uint32_t qa[4][4];  // A fragments of Q for the four 16-wide k-steps over the head dimension
    {
      const int arow = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int ks_ = 0; ks_ < 4; ++ks_) ldsm_x4(qs + swz128_bf16(arow, 16 * ks_ + 8 * (lane >> 4)), qa[ks_]);
    }
    float mrow[2] = {-INFINITY, -INFINITY};  // running max of scaled scores (base-2 units), rows g, g+8
    float lrow[2] = {0.f, 0.f};              // running sum of exponentials
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;

    for (int k0 = 0; k0 < mpad; k0 += kKBlk) {
      // S = Q·Kᵀ for keys k0 .. k0+63: eight n-tiles of eight keys.
      float s_[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s_[nt][e] = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        uint32_t kb[2][4];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) ldsm_x4(ks + swz128_bf16(k0 + 8 * nt + ri, 32 * kp + 8 * mi), kb[kp]);
#pragma unroll
        for (int ks_ = 0; ks_ < 4; ++ks_)
          mma16816(s_[nt], qa[ks_], kb[ks_ >> 1][2 * (ks_ & 1)], kb[ks_ >> 1][2 * (ks_ & 1) + 1]);
      }
      // Mask keys past the visible prefix; scale into base-2 units.
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = k0 + 8 * nt + 2 * q + (e & 1);
          s_[nt][e] = key < m ? s_[nt][e] * kScaleLog2 : -INFINITY;
        }
      // Online softmax per row (the four lanes of a quad hold one row's 64 scores).
      float mnew[2], corr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mx = mrow[h];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s_[nt][2 * h], s_[nt][2 * h + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mnew[h] = mx;  // finite: every key block holds at least one visible key
        corr[h] = exp2f(mrow[h] - mx);
        mrow[h] = mx;
      }
      uint32_t pa[4][4];  // P as A fragments over the four 16-key k-steps
      float psum[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(s_[nt][0] - mnew[0]), p1 = exp2f(s_[nt][1] - mnew[0]);
        const float p2 = exp2f(s_[nt][2] - mnew[1]), p3 = exp2f(s_[nt][3] - mnew[1]);
        psum[0] += p0 + p1;
        psum[1] += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 1);
        psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 2);
        lrow[h] = lrow[h] * corr[h] + psum[h];
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        acc[nt][0] *= corr[0];
        acc[nt][1] *= corr[0];
        acc[nt][2] *= corr[1];
        acc[nt][3] *= corr[1];
      }
      // A += P·V: B fragments of V (k = key, n = value channel) by transposed loads.
#pragma unroll
      for (int ks_ = 0; ks_ < 4; ++ks_) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t vb[4];
          ldsm_x4_t(vs + swz128_bf16(k0 + 16 * ks_ + 8 * (mi & 1) + ri, 16 * np + 8 * (mi >> 1)), vb);
          mma16816(acc[2 * np], pa[ks_], vb[0], vb[1]);
          mma16816(acc[2 * np + 1], pa[ks_], vb[2], vb[3]);
        }
      }
    }

    // out = o_ttt + clamp(α, 0, 1) ⊙ A, A = acc / l.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = 16 * warp + g + 8 * h;
      if (r >= nq) continue;
      const float inv = 1.f / lrow[h];
      const size_t rowo = base + (size_t)(t0 + r) * 64;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = 8 * nt + 2 * q;
        const float a0 = fminf(fmaxf(al[c], 0.f), 1.f), a1 = fminf(fmaxf(al[c + 1], 0.f), 1.f);
        const float2 ot = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(O_ttt + rowo + c));
        const float o0 = fmaf(a0, acc[nt][2 * h] * inv, ot.x);
        const float o1 = fmaf(a1, acc[nt][2 * h + 1] * inv, ot.y);
        *reinterpret_cast<uint32_t*>(out + rowo + c) = pack_bf16(o0, o1);
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace

ttt_status cache_attention(const ttt_state* st, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                           const __nv_bfloat16* V, const __nv_bfloat16* O_ttt, const float* alpha, int64_t T,
                           __nv_bfloat16* out, cudaStream_t s) {
  const ttt_config& c = st->cfg;
  if (c.cache_capacity > kMaxKeys)
    return fail(TTT_ERR_UNSUPPORTED, "the cache read path takes a cache capacity of at most %d", kMaxKeys);
  const int BH = c.batch * c.heads;
  const size_t smem = sizeof(CacheAttnSmem) + 1024;
  TTT_CUDA(cudaFuncSetAttribute(k_cache_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int nblk = (int)((T + kQBlk - 1) / kQBlk);
  const dim3 grid((unsigned)((nblk + kQPerCta - 1) / kQPerCta), (unsigned)BH);
  k_cache_attn<<<grid, kThreadsCA, smem, s>>>(Q, K, V, O_ttt, alpha, st->gate.entries, st->gate.counts,
                                             st->gate.tokens, (int)T, c.heads, c.cache_capacity, out,
                                             DevStatus{st->status.dev, st->wait_limit_ns, st->status.dev + 1});
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
