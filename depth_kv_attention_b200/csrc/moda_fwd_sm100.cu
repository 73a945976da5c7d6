// Tensor-core (tcgen05 / TMEM / TMA) MoDA forward for sm_100a.
#include "moda_internal.h"

namespace moda {
bool fwd_tc_supported(const FwdArgs&) { return false; }
cudaError_t launch_fwd_tc(const FwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace moda
