// Tensor-core (tcgen05 / TMEM / TMA) MoDA backward for sm_100a.
#include "moda_internal.h"

namespace moda {
bool bwd_tc_supported(const BwdArgs&) { return false; }
cudaError_t launch_bwd_tc(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace moda
