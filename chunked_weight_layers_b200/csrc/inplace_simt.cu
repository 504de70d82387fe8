// In-Place TTT scan, fp32 inputs, fp32 SIMT FFMA (the fp32 workload: d_model 256, d_ff 512,
// chunk 512). "In-Place Test-Time Training", §3: for each chunk, O_c = Z_c·W_cᵀ with the
// weight from before the chunk, then W_{c+1} = W_c + η·V̂_cᵀ·Z_c (§2).
//
// Both steps are small GEMMs (0.13 GFLOP per chunk) run as two tiled launches per chunk:
// 64x64 output tiles, 16-deep k slices staged in shared memory, 4x4 outputs per thread.
// Tensor cores are not used here: TF32 would miss the 1e-4 tolerance of this workload and
// the exact-integer checks, and the work is far too small to be throughput-bound.
#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

// C[M,N] (op)= A[M,K]·B[K,N] where A is stored K-contiguous (A_KC) or M-contiguous, and B is
// stored K-contiguous (B_KC, i.e. as [N,K]) or N-contiguous (as [K,N]).
// UPDATE = false: C = acc.  UPDATE = true: C = C + eta·acc (fused multiply-add).
template <bool A_KC, bool B_KC, bool UPDATE>
__global__ void __launch_bounds__(NT) k_sgemm(const float* __restrict__ A, const float* __restrict__ B,
                                              float* __restrict__ Cmat, int M, int N, int K, int lda, int ldb,
                                              int ldc, float eta) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    // Stage the A slice as As[k][m].
    if (A_KC) {
      const int r = tid / 4, kq = (tid % 4) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = m0 + r, k = k0 + kq + j;
        As[kq + j][r] = (m < M && k < K) ? A[(size_t)m * lda + k] : 0.f;
      }
    } else {
      const int kk = tid / 16, mq = (tid % 16) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = m0 + mq + j, k = k0 + kk;
        As[kk][mq + j] = (m < M && k < K) ? A[(size_t)k * lda + m] : 0.f;
      }
    }
    // Stage the B slice as Bs[k][n].
    if (B_KC) {
      const int r = tid / 4, kq = (tid % 4) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + r, k = k0 + kq + j;
        Bs[kq + j][r] = (n < N && k < K) ? B[(size_t)n * ldb + k] : 0.f;
      }
    } else {
      const int kk = tid / 16, nq = (tid % 16) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + nq + j, k = k0 + kk;
        Bs[kk][nq + j] = (n < N && k < K) ? B[(size_t)k * ldb + n] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float* c = Cmat + (size_t)m * ldc + n;
      if (UPDATE)
        *c = fmaf(eta, acc[i][j], *c);
      else
        *c = acc[i][j];
    }
  }
}

}  // namespace

ttt_status inplace_f32_chunk(ttt_state* st, const float* Z, const float* Vhat, float* O, int C, cudaStream_t s) {
  const int d = st->cfg.d_val, f = st->cfg.d_key;
  // Apply: O[C, d] = Z[C, f] · W[d, f]ᵀ — A = Z (K-contiguous), B = W as [N=d, K=f].
  dim3 ga((d + BN - 1) / BN, (C + BM - 1) / BM);
  k_sgemm<true, true, false><<<ga, NT, 0, s>>>(Z, st->ip.W, O, C, d, f, f, f, d, 0.f);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  // Update: W[d, f] += η · V̂[C, d]ᵀ · Z[C, f] — A = V̂ᵀ (M-contiguous), B = Z as [K=C, N=f].
  dim3 gu((f + BN - 1) / BN, (d + BM - 1) / BM);
  k_sgemm<false, false, true><<<gu, NT, 0, s>>>(Vhat, Z, st->ip.W, d, f, C, d, f, f, st->cfg.eta);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
