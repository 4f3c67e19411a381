// Inputs of the next decode step.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": the
// accepted candidates join the sequence and the heads of the next round read
// the base model's last hidden state, that of the kept (deepest accepted)
// node; "Medusa no contexto de LLMs": the base model's own choice there (the
// bonus token) is the next generated token, i.e. the next tree's root.
//
// One CTA per sequence: h_next[b] = node_hidden[b][kept] (16-byte copies),
// root_next[b] = bonus[b].
#include <cuda_runtime.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

__global__ void __launch_bounds__(128)
    next_step_kernel(const uint4* __restrict__ node_hidden, int N, int row_vecs,
                     const int32_t* __restrict__ accept_len,
                     const int32_t* __restrict__ accepted_nodes, int width,
                     const int32_t* __restrict__ bonus, uint4* __restrict__ h_next,
                     int32_t* __restrict__ root_next, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  const int b = blockIdx.x;
  const int L = accept_len[b];
  const int kept = (L >= 0 && L < width) ? accepted_nodes[(size_t)b * width + L] : -1;
  if (kept < 0 || kept >= N) {
    if (threadIdx.x == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }
  const uint4* src = node_hidden + ((size_t)b * N + kept) * row_vecs;
  uint4* dst = h_next + (size_t)b * row_vecs;
  for (int e = threadIdx.x; e < row_vecs; e += blockDim.x) dst[e] = src[e];
  if (threadIdx.x == 0) root_next[b] = bonus[b];
}

medusa_status_t next_step(const void* node_hidden, int elem_bytes, const int32_t* accept_len,
                          const int32_t* accepted_nodes, const int32_t* bonus, int B, int N,
                          int d, int max_depth, void* h_next, int32_t* root_next,
                          int32_t* status, cudaStream_t stream) {
  const int row_vecs = d * elem_bytes / 16;
  launch(next_step_kernel, B, 128, 0, stream, static_cast<const uint4*>(node_hidden), N, row_vecs,
         accept_len, accepted_nodes, max_depth + 1, bonus, static_cast<uint4*>(h_next), root_next,
         status);
  return check_launch("next_step");
}

}  // namespace medusa
