// Selection of the tensor-core kernels (filled in as they land).
#include "tc.h"

namespace mla {

bool tc_prefill_supported(const mla_config&) { return false; }
bool tc_gemm_supported(const GemmArgs&, int) { return false; }
cudaError_t tc_gemm(const GemmArgs&, cudaStream_t, uint32_t*) { return cudaErrorNotSupported; }
cudaError_t tc_attention(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
bool tc_decode_supported(const mla_config&) { return false; }
cudaError_t tc_decode(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mla
