// Selection of the tensor-core kernels that have not landed yet.
#include "tc.h"

namespace mla {

bool tc_attention_supported(const mla_config&) { return false; }
cudaError_t tc_attention(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
bool tc_decode_supported(const mla_config&) { return false; }
cudaError_t tc_decode(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mla
