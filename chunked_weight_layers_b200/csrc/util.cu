// Small utility kernels (weight conversion, fills) and TMA descriptor encoding.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ttt {

__global__ void k_f32_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x * 4;
  for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    if (i + 4 <= n) {
      const float4 v = *reinterpret_cast<const float4*>(src + i);
      uint2 o;
      o.x = pack_bf16(v.x, v.y);
      o.y = pack_bf16(v.z, v.w);
      *reinterpret_cast<uint2*>(dst + i) = o;
    } else {
      for (size_t j = i; j < n; ++j) dst[j] = __float2bfloat16_rn(src[j]);
    }
  }
}

// y ← y + alpha·x, four elements a thread where both are 16-byte aligned, else one.
__global__ void k_add_f32(float* __restrict__ y, const float* __restrict__ x, float alpha, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(x)) & 15u) == 0) {
    const size_t n4 = n / 4;
    for (size_t i = i0; i < n4; i += stride) {
      float4 a = reinterpret_cast<float4*>(y)[i];
      const float4 b = reinterpret_cast<const float4*>(x)[i];
      a.x = fmaf(alpha, b.x, a.x);
      a.y = fmaf(alpha, b.y, a.y);
      a.z = fmaf(alpha, b.z, a.z);
      a.w = fmaf(alpha, b.w, a.w);
      reinterpret_cast<float4*>(y)[i] = a;
    }
    for (size_t i = n4 * 4 + i0; i < n; i += stride) y[i] = fmaf(alpha, x[i], y[i]);
  } else {
    for (size_t i = i0; i < n; i += stride) y[i] = fmaf(alpha, x[i], y[i]);
  }
}

__global__ void k_fill_i32(int32_t* dst, int32_t v, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) dst[i] = v;
}

static int grid_for(size_t work, int threads, const ttt_state* st) {
  size_t blocks = (work + threads - 1) / threads;
  const size_t cap = (size_t)(st->num_sms > 0 ? st->num_sms : 148) * 8;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

ttt_status f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s, ttt_state* st) {
  if (n == 0) return TTT_OK;
  k_f32_to_bf16<<<grid_for((n + 3) / 4, 256, st), 256, 0, s>>>(src, dst, n);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

ttt_status add_f32(float* y, const float* x, float alpha, size_t n, int num_sms, cudaStream_t s) {
  if (n == 0) return TTT_OK;
  size_t blocks = (n / 4 + 255) / 256 + 1;
  const size_t cap = (size_t)(num_sms > 0 ? num_sms : 148) * 8;
  if (blocks > cap) blocks = cap;
  k_add_f32<<<(int)blocks, 256, 0, s>>>(y, x, alpha, n);
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

ttt_status fill_i32(int32_t* dst, int32_t v, size_t n, cudaStream_t s, ttt_state* st) {
  if (n == 0) return TTT_OK;
  k_fill_i32<<<grid_for(n, 256, st), 256, 0, s>>>(dst, v, n);
  st->launches++;
  TTT_CUDA(cudaGetLastError());
  return TTT_OK;
}

// ---- TMA descriptors ---------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

ttt_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encoder();
  if (fn == nullptr) return fail(TTT_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TTT_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return TTT_OK;
}

}  // namespace ttt
