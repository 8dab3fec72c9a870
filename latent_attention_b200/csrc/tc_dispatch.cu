// Selection of the tensor-core kernels that have not landed yet.
#include "tc.h"

namespace mla {

bool tc_decode_supported(const mla_config&) { return false; }
cudaError_t tc_decode(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mla
