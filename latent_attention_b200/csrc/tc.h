// Tensor-core (tcgen05 / TMEM / TMA) path for sm_100a, bf16 operands.
#pragma once
#include "internal.h"

namespace mla {

// Column tile width of the tensor-core GEMM.
constexpr int kTcTileN = 256;

// Whether the tensor-core attention kernel takes this configuration.
bool tc_attention_supported(const mla_config& c);
// Whether a single GEMM can run on the tensor-core kernel.
bool tc_gemm_supported(const GemmArgs& a, int dtype);
cudaError_t tc_gemm(const GemmArgs& a, cudaStream_t st, uint32_t* status);
cudaError_t tc_attention(const AttnArgs& a, cudaStream_t st);
bool tc_decode_supported(const mla_config& c);
cudaError_t tc_decode(const DecodeArgs& a, cudaStream_t st);
// Shortest slice of the token stream one CTA pair of the tensor-core decode
// takes (tokens).
int tc_decode_min_slice();

}  // namespace mla
