// Row positions of a packed (THD) prefill.
//
// Megatron-LM MLA guide, 训练支持与并行策略: variable-length sequences are
// packed back to back and described by cumulative lengths cu_seqlens[0..n].
// Row m belongs to the sequence b with cu[b] <= m < cu[b+1] and sits at
// position m - cu[b] (positions restart at 0 in every sequence), which is
// what the RoPE epilogues of the projections need per row.
#include "internal.h"

namespace mla {
namespace {

// One thread per packed row (and per sequence, for the checks).  cu_seqlens
// lives on the device: a malformed array (cu[0] != 0, cu[n] != total, a
// negative or too long sequence) raises kStatusBadCtx, and every position is
// clamped to [0, max_len) so no table read leaves the caller's RoPE tables.
__global__ void packed_positions_kernel(const int32_t* __restrict__ cu, int n_seq, int total,
                                        int max_len, int32_t* __restrict__ pos,
                                        uint32_t* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_seq) {
    const int len = cu[i + 1] - cu[i];
    if (len < 0 || len > max_len) atomicOr(status, kStatusBadCtx);
  }
  if (i == 0 && (cu[0] != 0 || cu[n_seq] != total)) atomicOr(status, kStatusBadCtx);
  if (i >= total) return;
  int lo = 0, hi = n_seq - 1;      // largest b with cu[b] <= i
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= i) lo = mid; else hi = mid - 1;
  }
  pos[i] = min(max(i - cu[lo], 0), max_len - 1);
}

}  // namespace

cudaError_t launch_packed_positions(const int32_t* cu_seqlens, int n_seq, int total, int max_len,
                                    int32_t* pos, uint32_t* status, cudaStream_t st) {
  const int n = total > n_seq ? total : n_seq;
  count_launches();
  packed_positions_kernel<<<(n + 255) / 256, 256, 0, st>>>(cu_seqlens, n_seq, total, max_len,
                                                           pos, status);
  return cudaGetLastError();
}

}  // namespace mla
