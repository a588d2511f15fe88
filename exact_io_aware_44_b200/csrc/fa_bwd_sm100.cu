// fa_bwd_sm100.cu -- placeholder until the backward kernels land.
#include "fa_internal.h"

namespace fa {
cudaError_t launch_bwd_bf16(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const BwdParams&, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace fa
