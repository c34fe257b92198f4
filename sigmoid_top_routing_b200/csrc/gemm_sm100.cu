// Prefill-sized grouped expert GEMMs on tcgen05 (filled in by the next step).
#include "internal.h"

namespace moe {

cudaError_t launch_gemm_up(const ExpertArgs&, bool, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_gemm_down(const ExpertArgs&, bool, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace moe
