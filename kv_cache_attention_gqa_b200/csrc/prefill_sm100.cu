// bf16 prefill on sm_100a (tcgen05 + TMEM + TMA). Placeholder until the kernel lands.
#include "common.cuh"
#include "internal.h"

namespace gqa {
cudaError_t launch_prefill_bf16(const PrefillArgs&, const CUtensorMap*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace gqa
