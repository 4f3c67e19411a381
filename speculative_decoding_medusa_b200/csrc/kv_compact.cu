// KV compaction: the kept branch's K/V move to contiguous cache slots.
//
// "Medusa no contexto de LLMs": an accepted candidate enters the sequence
// without another full pass; "Medusa Heads" glossary: only the longest
// accepted branch is kept.  For j = 0..L, slot P + j <- slot
// P + accepted_nodes[j]; then P grows by L + 1.
//
// One CTA per sequence.  The L + 1 source rows of K and V of as many kv heads
// as fit are staged in shared memory before any destination is written, so
// overlapping source/destination slots cannot race (a destination of one
// step may be the source of another).
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "abi_internal.h"
#include "common.cuh"
#include "kv_compact.cuh"

namespace medusa {

constexpr int kCompactThreads = 512;

// Shared memory that one round of staging may use; heads per round =
// this / (2 * (max_depth + 1) * row bytes), at least one.
constexpr size_t kCompactSmem = 96 * 1024;

__global__ void __launch_bounds__(kCompactThreads)
    kv_compact_kernel(uint8_t* Kc, uint8_t* Vc, int row_bytes, int32_t* prefix_len,
                      const int32_t* __restrict__ accepted_nodes,
                      const int32_t* __restrict__ accept_len, int Hkv, int cap, int max_depth,
                      int heads_per_round, int32_t* __restrict__ compact_src, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  // [heads_per_round][L+1][row] of K, then the same of V
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ int s_src[MEDUSA_MAX_HEADS + 1];
  __shared__ int s_ok;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int W = max_depth + 1;
  // prefix length, accept length and the path's nodes in one round trip
  const int P = prefix_len[b];
  const int L = accept_len[b];
  const int node = tid < W ? accepted_nodes[(size_t)b * W + tid] : 0;
  if (tid == 0) s_ok = (L >= 0 && L <= max_depth && P >= 0) ? 1 : 0;
  __syncthreads();
  if (tid <= L && tid < W) {
    const long long slot = (long long)P + node;
    if (node < tid || slot >= cap) s_ok = 0;  // a depth-j node has index >= j
    s_src[tid] = (int)slot;
  }
  __syncthreads();
  if (!s_ok) {
    if (tid == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }

  const CompactArgs a{Kc, Vc, row_bytes, prefix_len, Hkv, cap, heads_per_round, compact_src};
  compact_sequence(a, b, P, L, s_src, W, reinterpret_cast<uint4*>(stage));
}

bool compact_plan(medusa_dtype_t dt, int dh, int Hkv, int max_depth, int* heads_per_round,
                  size_t* smem) {
  const int row_bytes = dh * (dt == MEDUSA_BF16 ? 2 : 4);
  const size_t per_head = 2 * (size_t)(max_depth + 1) * row_bytes;
  if (per_head > kCompactSmem) return false;
  *heads_per_round = (int)std::min<size_t>((size_t)Hkv, kCompactSmem / per_head);
  *smem = per_head * *heads_per_round;
  return true;
}

medusa_status_t kv_compact(void* Kc, void* Vc, medusa_dtype_t dt, int32_t* prefix_len,
                           const int32_t* accepted_nodes, const int32_t* accept_len, int B,
                           int Hkv, int dh, int cap, int max_depth, int32_t* compact_src,
                           int32_t* status, cudaStream_t stream) {
  const int row_bytes = dh * (dt == MEDUSA_BF16 ? 2 : 4);
  int heads_per_round = 0;
  size_t smem = 0;
  if (!compact_plan(dt, dh, Hkv, max_depth, &heads_per_round, &smem))
    return fail(MEDUSA_ERR_UNSUPPORTED, "kv_compact: (max_depth+1) * row too large");
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kv_compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kCompactSmem) != cudaSuccess)
    return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(kv_compact) failed");
  launch(kv_compact_kernel, B, kCompactThreads, smem, stream, static_cast<uint8_t*>(Kc),
         static_cast<uint8_t*>(Vc), row_bytes, prefix_len, accepted_nodes, accept_len, Hkv, cap,
         max_depth, heads_per_round, compact_src, status);
  return check_launch("kv_compact");
}

}  // namespace medusa
