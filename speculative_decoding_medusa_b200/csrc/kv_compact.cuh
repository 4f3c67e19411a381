// KV compaction of one sequence by one thread block (shared by the
// compaction kernel and the verification's compaction tail).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace medusa {

// Where the kept branch moves: caches [B][Hkv][cap][row_bytes], the prefix
// lengths (read, then advanced) and the source-slot list written back.
// Kc == nullptr: no compaction.
struct CompactArgs {
  uint8_t* Kc;
  uint8_t* Vc;
  int row_bytes;
  int32_t* prefix_len;
  int Hkv, cap, heads_per_round;
  int32_t* compact_src;
};

// Sequence b, prefix P, kept branch of L + 1 nodes whose source slots are
// s_src[0..L] (shared memory, checked against the capacity by the caller):
// for j = 0..L, slot P + j <- slot s_src[j] in every kv head of K and V, as
// if done for ascending j.  Rounds of heads_per_round kv heads: every source
// row of a round is staged in `stage` (dynamic shared memory) before any
// destination row is written, since a destination of one step may be the
// source of another.  Then compact_src and prefix_len[b] = P + L + 1.  Every
// thread of the block calls it.
__device__ __forceinline__ void compact_sequence(const CompactArgs& a, int b, int P, int L,
                                                 const int* s_src, int W, uint4* stage) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int vec_per_row = a.row_bytes / 16;
  const int per_head = (L + 1) * vec_per_row;
  uint4* sk = stage;
  uint4* sv = sk + (size_t)a.heads_per_round * W * vec_per_row;
  for (int h0 = 0; h0 < a.Hkv; h0 += a.heads_per_round) {
    const int nh = min(a.heads_per_round, a.Hkv - h0);
    const int n_vec = nh * per_head;
    for (int e = tid; e < n_vec; e += nthr) {
      const int hh = e / per_head, r = e - hh * per_head;
      const int j = r / vec_per_row, c = r - j * vec_per_row;
      const size_t src = (((size_t)b * a.Hkv + h0 + hh) * a.cap + s_src[j]) * a.row_bytes;
      sk[e] = reinterpret_cast<const uint4*>(a.Kc + src)[c];
      sv[e] = reinterpret_cast<const uint4*>(a.Vc + src)[c];
    }
    __syncthreads();
    for (int e = tid; e < n_vec; e += nthr) {
      const int hh = e / per_head, r = e - hh * per_head;
      const int j = r / vec_per_row, c = r - j * vec_per_row;
      const size_t dst = (((size_t)b * a.Hkv + h0 + hh) * a.cap + P + j) * a.row_bytes;
      reinterpret_cast<uint4*>(a.Kc + dst)[c] = sk[e];
      reinterpret_cast<uint4*>(a.Vc + dst)[c] = sv[e];
    }
    __syncthreads();
  }
  if (tid < W) a.compact_src[(size_t)b * W + tid] = tid <= L ? s_src[tid] : -1;
  if (tid == 0) a.prefix_len[b] = P + L + 1;
}

}  // namespace medusa
