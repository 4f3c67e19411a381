// Candidate tree of one sequence by one thread block (shared by the tree
// build kernel and the top-k merge's tail).
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": the heads'
// top choices combine into candidate continuations that share prefixes and
// form a tree; head 2 proposes the same tokens under every head-1 branch; the
// attention mask lets each candidate see only its ancestors.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/medusa.h"
#include "common.cuh"

namespace medusa {

// Where one step's tree goes.  cand_ids == nullptr: no tree is built.
struct TreeOut {
  const int32_t* parent;
  const int32_t* depth;
  const int32_t* rank;
  int N, max_depth, n_leaves;
  int K, kmax;
  const int32_t* root_tok;    // [B]
  const int32_t* prefix_len;  // [B]
  int32_t* cand_ids;          // [B][N]
  int32_t* pos_ids;           // [B][N]
  uint32_t* anc_mask;         // [N][ceil(N/32)]
  int32_t* retrieve;          // [n_leaves][max_depth+1]
  int32_t* status;
};

constexpr int kTreeThreads = MEDUSA_MAX_NODES;  // one thread per node
constexpr int kTreeMaxWords = MEDUSA_MAX_NODES / 32;

// Sequence b's candidate ids and positions from its K x kmax top-k table
// (row k = head k + 1, read through `topk`, which the caller points at global
// or shared memory); block 0's caller passes with_tree = true to also write
// the mask and the retrieve paths, which depend on the tree only.  Called by
// every thread of a block of kTreeThreads threads.
template <typename TopkAt>
__device__ __forceinline__ void build_tree_sequence(const TreeOut& t, int b, TopkAt topk,
                                                    bool with_tree) {
  __shared__ int s_parent[MEDUSA_MAX_NODES];
  __shared__ int s_depth[MEDUSA_MAX_NODES];
  __shared__ int s_has_child[MEDUSA_MAX_NODES];
  __shared__ int s_rank[MEDUSA_MAX_NODES];
  __shared__ int s_topk[MEDUSA_MAX_HEADS * MEDUSA_MAX_KMAX];
  __shared__ int s_warp_leaves[MEDUSA_MAX_NODES / 32];
  __shared__ int s_bad;
  const int i = threadIdx.x;
  const int N = t.N;
  // every input is read in one round trip: the tree, this sequence's
  // candidate table, its prefix length and root token
  if (i == 0) s_bad = 0;
  if (i < N) {
    s_parent[i] = t.parent[i];
    s_depth[i] = t.depth[i];
    s_rank[i] = t.rank[i];
    s_has_child[i] = 0;
  }
  for (int e = i; e < t.K * t.kmax; e += kTreeThreads) s_topk[e] = topk(e);
  const int P = t.prefix_len[b];
  const int root = t.root_tok[b];
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
      ok = pa >= 0 && pa < i && dp == s_depth[pa] + 1 && dp <= t.max_depth && dp <= t.K &&
           rk >= 0 && rk < t.kmax;
    }
    if (!ok) atomicOr(&s_bad, 1);
    if (i > 0 && pa >= 0 && pa < i) s_has_child[pa] = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (i == 0 && with_tree) report(t.status, MEDUSA_ERR_DEVICE_CHECK);
    if (i < N) {
      t.cand_ids[(size_t)b * N + i] = -1;
      t.pos_ids[(size_t)b * N + i] = -1;
    }
    return;
  }

  if (i < N) {
    const int tok = i == 0 ? root : s_topk[(s_depth[i] - 1) * t.kmax + s_rank[i]];
    t.cand_ids[(size_t)b * N + i] = tok;
    t.pos_ids[(size_t)b * N + i] = P + s_depth[i];
  }
  if (!with_tree) return;

  // ancestor-or-self mask row of node i
  if (i < N) {
    uint32_t m[kTreeMaxWords];
#pragma unroll
    for (int w = 0; w < kTreeMaxWords; ++w) m[w] = 0u;
    for (int j = i; j >= 0; j = s_parent[j]) {
#pragma unroll
      for (int w = 0; w < kTreeMaxWords; ++w)
        if ((j >> 5) == w) m[w] |= 1u << (j & 31);
    }
    const int words = (N + 31) >> 5;
#pragma unroll
    for (int w = 0; w < kTreeMaxWords; ++w)
      if (w < words) t.anc_mask[(size_t)i * words + w] = m[w];
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
    if (idx < t.n_leaves) {
      int32_t* row = t.retrieve + (size_t)idx * (t.max_depth + 1);
      for (int d = s_depth[i] + 1; d <= t.max_depth; ++d) row[d] = -1;
      for (int j = i; j >= 0; j = s_parent[j]) row[s_depth[j]] = j;
    }
  }
  if (i == 0) {
    int total = 0;
    for (int w = 0; w < (N + 31) / 32; ++w) total += s_warp_leaves[w];
    if (total != t.n_leaves) report(t.status, MEDUSA_ERR_DEVICE_CHECK);
  }
}

}  // namespace medusa
