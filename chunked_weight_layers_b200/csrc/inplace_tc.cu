// In-Place TTT scan on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
#include "common.cuh"
#include "internal.h"

namespace ttt {

ttt_status inplace_bf16_scan(ttt_state* st, const __nv_bfloat16* Z, const __nv_bfloat16* targets, int64_t T,
                             __nv_bfloat16* O, cudaStream_t s) {
  (void)st; (void)Z; (void)targets; (void)T; (void)O; (void)s;
  return fail(TTT_ERR_UNSUPPORTED, "In-Place BF16 scan not built yet");
}

}  // namespace ttt
