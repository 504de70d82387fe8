// ttt_target_values_noalloc: target generation V̂ = Conv1D(X0)·Wtarget for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need this work done: their
// device memory is owned entirely by another allocator (a framework's caching allocator
// that has reserved the GPU), or they run in a loop that must not allocate after start-up
// (cudaMalloc can block and synchronise the device). The regular path gets its scratch
// buffers from ttt_state_create; this entry point instead keeps its scratch — the conv(X0)
// rows and the tile schedule — in one fixed array of device memory that is part of the
// library image. It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
// routine. The caller passes the inputs and the output.
//
// The fixed array (kScratchBytes, about 8.1 MB) is a module variable: the CUDA runtime
// creates it on a device when the library's module is first loaded there, which with lazy
// module loading (the default since CUDA 12.2) is the first call's cudaGetSymbolAddress, and
// at library load with CUDA_MODULE_LOADING=EAGER. That first call on a device may therefore
// need about 8 MB of free device memory and may synchronise; from then on the device holds
// the array until the process exits. Every call shares it and it keeps the last call's
// contents; every call overwrites all of the scratch it reads, so nothing needs clearing, but
// calls whose GPU work overlaps (on different streams, or from different host threads without
// ordering) race on it.
//
// A bounded device-side wait that runs out is reported through the caller's optional status
// word (a device int32 the call zeroes first), since there is no state to hold it.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

constexpr size_t kMaxConvElems = (size_t)1 << 22;  // T·d ≤ 4,194,304 (8 MB of bf16 conv rows)
constexpr size_t kMaxPlanInts = 16384;              // schedule: CTA offsets + tile codes
constexpr size_t kConvBytes = kMaxConvElems * 2;
constexpr size_t kScratchBytes = kConvBytes + kMaxPlanInts * 4;
constexpr int kMaxDevices = 64;

// In host code this name is only a host-side stand-in for the device array, never a device
// address; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

struct DeviceScratch {
  void* addr = nullptr;
  int num_sms = 0;
};
DeviceScratch g_dev[kMaxDevices];
std::mutex g_mutex;

// Once per device, with that device current: the device address of the fixed array.
ttt_status scratch_for_current_device(DeviceScratch* out) {
  int dev = -1;
  TTT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(TTT_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceScratch& d = g_dev[dev];
  if (d.addr == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the fixed scratch array");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    d.addr = p;
    d.num_sms = sms;
  }
  *out = d;
  return TTT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace ttt

extern "C" ttt_status ttt_target_values_noalloc(const void* X0, const float* convw, const void* Wtarget, int64_t T,
                                                int32_t d_model, int32_t chunk, int32_t conv_taps,
                                                int32_t conv_pad_mode, void* Vhat_out, int32_t* status,
                                                ttt_stream stream) {
  using namespace ttt;
  if (T < 0) return fail(TTT_ERR_INVALID_ARG, "T must be non-negative");
  if (T == 0) return TTT_OK;
  if (X0 == nullptr || convw == nullptr || Wtarget == nullptr || Vhat_out == nullptr || !aligned16(X0) ||
      !aligned16(convw) || !aligned16(Wtarget) || !aligned16(Vhat_out))
    return fail(TTT_ERR_INVALID_ARG, "X0, convw, Wtarget and Vhat_out must be 16-byte aligned device pointers");
  if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) != 0)
    return fail(TTT_ERR_INVALID_ARG, "status must be a 4-byte aligned device pointer or NULL");
  if (d_model < 8 || d_model % 8 != 0) return fail(TTT_ERR_UNSUPPORTED, "d_model must be a positive multiple of 8");
  if (T % 128 != 0) return fail(TTT_ERR_UNSUPPORTED, "T must be a multiple of 128");
  if (chunk < 1) return fail(TTT_ERR_INVALID_ARG, "chunk must be positive");
  if (conv_taps < 1 || conv_taps > 8) return fail(TTT_ERR_UNSUPPORTED, "conv_taps must lie in [1, 8]");
  if (conv_pad_mode != 0 && conv_pad_mode != 1) return fail(TTT_ERR_INVALID_ARG, "conv_pad_mode must be 0 or 1");
  if ((uint64_t)T * (uint64_t)d_model > kMaxConvElems)
    return fail(TTT_ERR_INVALID_ARG,
                "T*d_model = %lld exceeds the fixed scratch of this entry point (%llu elements); "
                "split the tokens into calls of at most that many rows x d_model",
                (long long)(T * (int64_t)d_model), (unsigned long long)kMaxConvElems);
  DeviceScratch ds;
  TTT_TRY(scratch_for_current_device(&ds));
  if ((size_t)target_values_plan_ints((int)T, d_model, ds.num_sms) > kMaxPlanInts)
    return fail(TTT_ERR_INVALID_ARG, "too many tiles for the fixed schedule scratch");
  uint8_t* base = static_cast<uint8_t*>(ds.addr);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (status != nullptr) TTT_CUDA(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
  return target_values_into(static_cast<const __nv_bfloat16*>(X0), convw, static_cast<const __nv_bfloat16*>(Wtarget),
                            (int)T, d_model, chunk, conv_taps, conv_pad_mode, reinterpret_cast<__nv_bfloat16*>(base),
                            reinterpret_cast<int32_t*>(base + kConvBytes), static_cast<__nv_bfloat16*>(Vhat_out),
                            status, ds.num_sms, s);
}
