// KV compaction: the kept branch's K/V move to contiguous cache slots.
//
// "Medusa no contexto de LLMs": an accepted candidate enters the sequence
// without another full pass; "Medusa Heads" glossary: only the longest
// accepted branch is kept.  For j = 0..L, slot P + j <- slot
// P + accepted_nodes[j]; then P grows by L + 1.
//
// One CTA per sequence.  For each kv head the L + 1 source rows of K and V are
// staged in shared memory before any destination is written, so overlapping
// source/destination slots cannot race (a destination of one step may be the
// source of another).
#include <cuda_runtime.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kCompactThreads = 256;

__global__ void __launch_bounds__(kCompactThreads)
    kv_compact_kernel(uint8_t* Kc, uint8_t* Vc, int row_bytes, int32_t* prefix_len,
                      const int32_t* __restrict__ accepted_nodes,
                      const int32_t* __restrict__ accept_len, int Hkv, int cap, int max_depth,
                      int heads_at_once, int32_t* __restrict__ compact_src, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  // [2][max_depth+1][row_bytes], or [2][Hkv][max_depth+1][row_bytes] when
  // every head is staged at once
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
  if (!s_ok) return;

  const int vec_per_row = row_bytes / 16;
  uint4* sk = reinterpret_cast<uint4*>(stage);
  if (heads_at_once > 1) {
    // every kv head staged in one round trip: [Hkv][L+1][row] for K then V
    const int n_vec = Hkv * (L + 1) * vec_per_row;
    uint4* sv = sk + (size_t)Hkv * W * vec_per_row;
    for (int e = tid; e < n_vec; e += kCompactThreads) {
      const int c = e % vec_per_row;
      const int j = (e / vec_per_row) % (L + 1);
      const int h = e / (vec_per_row * (L + 1));
      const size_t src = (((size_t)b * Hkv + h) * cap + s_src[j]) * row_bytes;
      sk[e] = reinterpret_cast<const uint4*>(Kc + src)[c];
      sv[e] = reinterpret_cast<const uint4*>(Vc + src)[c];
    }
    __syncthreads();
    for (int e = tid; e < n_vec; e += kCompactThreads) {
      const int c = e % vec_per_row;
      const int j = (e / vec_per_row) % (L + 1);
      const int h = e / (vec_per_row * (L + 1));
      const size_t dst = (((size_t)b * Hkv + h) * cap + P + j) * row_bytes;
      reinterpret_cast<uint4*>(Kc + dst)[c] = sk[e];
      reinterpret_cast<uint4*>(Vc + dst)[c] = sv[e];
    }
    if (tid < W) compact_src[(size_t)b * W + tid] = tid <= L ? s_src[tid] : -1;
    if (tid == 0) prefix_len[b] = P + L + 1;
    return;
  }
  const int n_vec = (L + 1) * vec_per_row;
  uint4* sv = reinterpret_cast<uint4*>(stage + (size_t)W * row_bytes);
  for (int h = 0; h < Hkv; ++h) {
    const size_t head_base = ((size_t)b * Hkv + h) * cap;  // in rows
    for (int e = tid; e < n_vec; e += kCompactThreads) {
      const int j = e / vec_per_row, c = e - j * vec_per_row;
      const size_t src = (head_base + s_src[j]) * row_bytes;
      sk[e] = reinterpret_cast<const uint4*>(Kc + src)[c];
      sv[e] = reinterpret_cast<const uint4*>(Vc + src)[c];
    }
    __syncthreads();
    for (int e = tid; e < n_vec; e += kCompactThreads) {
      const int j = e / vec_per_row, c = e - j * vec_per_row;
      const size_t dst = (head_base + P + j) * row_bytes;
      reinterpret_cast<uint4*>(Kc + dst)[c] = sk[e];
      reinterpret_cast<uint4*>(Vc + dst)[c] = sv[e];
    }
    __syncthreads();
  }
  if (tid < W) compact_src[(size_t)b * W + tid] = tid <= L ? s_src[tid] : -1;
  if (tid == 0) prefix_len[b] = P + L + 1;
}

medusa_status_t kv_compact(void* Kc, void* Vc, medusa_dtype_t dt, int32_t* prefix_len,
                           const int32_t* accepted_nodes, const int32_t* accept_len, int B,
                           int Hkv, int dh, int cap, int max_depth, int32_t* compact_src,
                           int32_t* status, cudaStream_t stream) {
  const int row_bytes = dh * (dt == MEDUSA_BF16 ? 2 : 4);
  const size_t per_head = 2 * (size_t)(max_depth + 1) * row_bytes;
  if (per_head > 48 * 1024)
    return fail(MEDUSA_ERR_UNSUPPORTED, "kv_compact: (max_depth+1) * row too large");
  const bool all_heads = per_head * Hkv <= 48 * 1024;
  launch(kv_compact_kernel, B, kCompactThreads, all_heads ? per_head * Hkv : per_head, stream,
      static_cast<uint8_t*>(Kc), static_cast<uint8_t*>(Vc), row_bytes, prefix_len, accepted_nodes,
      accept_len, Hkv, cap, max_depth, all_heads ? Hkv : 1, compact_src, status);
  return check_launch("kv_compact");
}

}  // namespace medusa
