// Backward on the tensor cores (placeholder until the tcgen05 kernels land).
#include "internal.h"

namespace sk {

size_t bwd_tc_workspace_bytes(int T_tot, int Hq, int D) {
  return sizeof(float) * (size_t)T_tot * Hq * D;
}

int launch_bwd_tc(const AttnProblem&, const BwdBuffers&, cudaStream_t) {
  return SINKATTN_ERR_UNSUPPORTED;
}

}  // namespace sk
