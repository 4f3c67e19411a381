// Candidate tree: candidate ids, position ids, ancestor mask, retrieve paths.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": the heads'
// top choices combine into candidate continuations that share prefixes and
// form a tree; head 2 proposes the same tokens under every head-1 branch; the
// attention mask lets each candidate see only its ancestors.
//
// One CTA per sequence, one thread per node (N <= 256).  The mask and the
// retrieve paths depend on the tree only; CTA 0 writes them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kMaxWords = MEDUSA_MAX_NODES / 32;

__global__ void __launch_bounds__(MEDUSA_MAX_NODES)
    tree_build_kernel(const int32_t* __restrict__ parent, const int32_t* __restrict__ depth,
                      const int32_t* __restrict__ rank, int N, int max_depth, int n_leaves,
                      const int32_t* __restrict__ root_tok, const int32_t* __restrict__ topk_ids,
                      int K, int kmax, const int32_t* __restrict__ prefix_len,
                      int32_t* __restrict__ cand_ids, int32_t* __restrict__ pos_ids,
                      uint32_t* __restrict__ anc_mask, int32_t* __restrict__ retrieve,
                      int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ int s_parent[MEDUSA_MAX_NODES];
  __shared__ int s_depth[MEDUSA_MAX_NODES];
  __shared__ int s_has_child[MEDUSA_MAX_NODES];
  __shared__ int s_rank[MEDUSA_MAX_NODES];
  __shared__ int s_warp_leaves[MEDUSA_MAX_NODES / 32];
  __shared__ int s_bad;
  extern __shared__ int s_topk[];  // this sequence's K x kmax candidate ids
  const int i = threadIdx.x;
  const int b = blockIdx.x;
  // every input is read in one round trip: the tree, this sequence's
  // candidate table, its prefix length and root token
  if (i == 0) s_bad = 0;
  if (i < N) {
    s_parent[i] = parent[i];
    s_depth[i] = depth[i];
    s_rank[i] = rank[i];
    s_has_child[i] = 0;
  }
  for (int e = i; e < K * kmax; e += blockDim.x) s_topk[e] = topk_ids[(size_t)b * K * kmax + e];
  const int P = prefix_len[b];
  const int root = root_tok[b];
  __syncthreads();

  // structural checks: BFS order, depth chain, rank range
  if (i < N) {
    const int pa = s_parent[i];
    const int dp = s_depth[i];
    bool ok;
    if (i == 0) {
      ok = (pa == -1) && (dp == 0);
    } else {
      const int rk = s_rank[i];
      ok = pa >= 0 && pa < i && dp == s_depth[pa] + 1 && dp <= max_depth && dp <= K && rk >= 0 &&
           rk < kmax;
    }
    if (!ok) atomicOr(&s_bad, 1);
    if (i > 0 && pa >= 0 && pa < i) s_has_child[pa] = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (i == 0 && b == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    if (i < N) {
      cand_ids[(size_t)b * N + i] = -1;
      pos_ids[(size_t)b * N + i] = -1;
    }
    return;
  }

  if (i < N) {
    const int tok = i == 0 ? root : s_topk[(s_depth[i] - 1) * kmax + s_rank[i]];
    cand_ids[(size_t)b * N + i] = tok;
    pos_ids[(size_t)b * N + i] = P + s_depth[i];
  }
  if (b != 0) return;

  // ancestor-or-self mask row of node i
  if (i < N) {
    uint32_t m[kMaxWords];
#pragma unroll
    for (int w = 0; w < kMaxWords; ++w) m[w] = 0u;
    for (int j = i; j >= 0; j = s_parent[j]) {
#pragma unroll
      for (int w = 0; w < kMaxWords; ++w)
        if ((j >> 5) == w) m[w] |= 1u << (j & 31);
    }
    const int words = (N + 31) >> 5;
#pragma unroll
    for (int w = 0; w < kMaxWords; ++w)
      if (w < words) anc_mask[(size_t)i * words + w] = m[w];
  }

  // leaves in node order: exclusive prefix count by warp ballots
  const bool leaf = i < N && !s_has_child[i];
  const unsigned bal = __ballot_sync(0xffffffffu, leaf);
  const int lane = i & 31;
  if (lane == 0) s_warp_leaves[i >> 5] = __popc(bal);
  __syncthreads();
  if (leaf) {
    int idx = __popc(bal & ((1u << lane) - 1u));
    for (int w = 0; w < (i >> 5); ++w) idx += s_warp_leaves[w];
    if (idx < n_leaves) {
      int32_t* row = retrieve + (size_t)idx * (max_depth + 1);
      for (int t = s_depth[i] + 1; t <= max_depth; ++t) row[t] = -1;
      for (int j = i; j >= 0; j = s_parent[j]) row[s_depth[j]] = j;
    }
  }
  if (i == 0) {
    int total = 0;
    for (int w = 0; w < (N + 31) / 32; ++w) total += s_warp_leaves[w];
    if (total != n_leaves) report(status, MEDUSA_ERR_DEVICE_CHECK);
  }
}

medusa_status_t tree_build(const medusa_tree_t& t, const int32_t* root_tok, const int32_t* topk_ids,
                           int K, int kmax, const int32_t* prefix_len, int B, int32_t* cand_ids,
                           int32_t* pos_ids, uint32_t* anc_mask, int32_t* retrieve,
                           int32_t* status, cudaStream_t stream) {
  launch(tree_build_kernel, B, MEDUSA_MAX_NODES, (size_t)K * kmax * sizeof(int), stream, t.parent,
         t.depth, t.rank, t.n_nodes, t.max_depth, t.n_leaves, root_tok, topk_ids, K, kmax,
         prefix_len, cand_ids, pos_ids, anc_mask, retrieve, status);
  return check_launch("tree_build");
}

}  // namespace medusa
