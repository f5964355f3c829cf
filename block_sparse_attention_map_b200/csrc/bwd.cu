// Backward pass: placeholder until the deterministic kernel lands.
#include "internal.h"

namespace bsa {
cudaError_t launch_bwd(const bsa_problem &, const MaskParams &, const bsa_options &,
                       const PlanSignature &, const CUtensorMap &, const CUtensorMap &,
                       const CUtensorMap &, const CUtensorMap &, const void *, const void *,
                       const float *, void *, void *, void *, const WsLayout &, uint8_t *,
                       cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace bsa
