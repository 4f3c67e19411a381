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
#include "tree_build.cuh"

namespace medusa {

__global__ void __launch_bounds__(kTreeThreads)
    tree_build_kernel(TreeOut t, const int32_t* __restrict__ topk_ids) {
  grid_dep_wait();
  grid_dep_launch();
  const int b = blockIdx.x;
  const int32_t* row = topk_ids + (size_t)b * t.K * t.kmax;
  build_tree_sequence(t, b, [row](int e) { return row[e]; }, b == 0);
}

medusa_status_t tree_build(const medusa_tree_t& tree, const int32_t* root_tok,
                           const int32_t* topk_ids, int K, int kmax, const int32_t* prefix_len,
                           int B, int32_t* cand_ids, int32_t* pos_ids, uint32_t* anc_mask,
                           int32_t* retrieve, int32_t* status, cudaStream_t stream) {
  const TreeOut t{tree.parent, tree.depth, tree.rank, tree.n_nodes, tree.max_depth,
                  tree.n_leaves, K, kmax, root_tok, prefix_len, cand_ids, pos_ids, anc_mask,
                  retrieve, status};
  launch(tree_build_kernel, B, kTreeThreads, 0, stream, t, topk_ids);
  return check_launch("tree_build");
}

}  // namespace medusa
