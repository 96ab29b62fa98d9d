// Masked prefill attention kernel (tcgen05 / TMEM / TMA), sm_100a.
#include <cuda_runtime.h>

#include "ps_internal.h"
#include "ps_ranges.cuh"

namespace ps {

size_t prefill_workspace_bytes(int64_t batch, int64_t seq, int32_t hq) {
  (void)batch;
  (void)hq;
  return prefill_plan_bytes(seq, prefill_plan_tiles(seq, 0, 1) + 0) + 256;
}

int launch_prefill(const PrefillLaunch& l, cudaStream_t stream) {
  (void)l;
  (void)stream;
  return fail(PS_ERR_UNSUPPORTED, "masked prefill attention not built yet");
}

}  // namespace ps
