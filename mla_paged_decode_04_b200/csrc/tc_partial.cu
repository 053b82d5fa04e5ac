// Placeholder until the tensor-core kernel lands.
#include "internal.h"
namespace mla {
cudaError_t launch_tc_partial(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mla
