// The sparse candidate tree of the most accurate combinations (host code).
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": a sparse
// tree built from the most accurate combinations of the heads' top choices
// gives a larger speedup than a dense one.  With acc[t-1][r] the probability
// that head t's rank-r token is the base model's choice (one rank at most,
// heads independent), a node whose rank path is (r1..rt) is accepted with
// probability prod acc[i-1][r_i]; the expected accept length of a tree is the
// sum of those over its non-root nodes.  Because a path's product never
// exceeds its prefix's, the best tree of n nodes holds the n-1 paths with the
// largest products: a best-first walk from the root pops exactly those, in
// order (equal products: the lexicographically smaller path first, so a prefix
// always precedes its extensions).  Nodes are then numbered by depth and
// lexicographic path, so parents precede children.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <map>
#include <queue>
#include <vector>

#include "abi_internal.h"

namespace medusa {
namespace {

struct Cand {
  double prob;
  std::vector<int> path;
};

// priority: larger product first, then lexicographically smaller path
struct Worse {
  bool operator()(const Cand& a, const Cand& b) const {
    if (a.prob != b.prob) return a.prob < b.prob;
    return b.path < a.path;
  }
};

}  // namespace

medusa_status_t tree_from_accuracies(const float* acc, int n_heads, int kmax, int n_nodes,
                                     int max_depth, int32_t* parent, int32_t* depth,
                                     int32_t* rank, double* expected_accept_len) {
  const int D = std::min(n_heads, max_depth);
  std::priority_queue<Cand, std::vector<Cand>, Worse> frontier;
  for (int r = 0; r < kmax; ++r) frontier.push(Cand{acc[r], {r}});
  std::vector<std::vector<int>> chosen;
  double expected = 0.0;
  while ((int)chosen.size() < n_nodes - 1 && !frontier.empty()) {
    Cand c = frontier.top();
    frontier.pop();
    expected += c.prob;
    if ((int)c.path.size() < D) {
      const int t = (int)c.path.size();  // children use head t + 1
      for (int r = 0; r < kmax; ++r) {
        Cand k{c.prob * (double)acc[t * kmax + r], c.path};
        k.path.push_back(r);
        frontier.push(std::move(k));
      }
    }
    chosen.push_back(std::move(c.path));
  }
  if ((int)chosen.size() < n_nodes - 1)
    return fail(MEDUSA_ERR_SHAPE, "tree_from_accuracies: fewer rank paths than n_nodes - 1");
  std::sort(chosen.begin(), chosen.end(), [](const std::vector<int>& a, const std::vector<int>& b) {
    return a.size() != b.size() ? a.size() < b.size() : a < b;
  });
  std::map<std::vector<int>, int> index;
  index[std::vector<int>()] = 0;
  parent[0] = -1;
  depth[0] = 0;
  rank[0] = 0;
  for (int i = 0; i < (int)chosen.size(); ++i) {
    const std::vector<int>& p = chosen[i];
    const int node = i + 1;
    index[p] = node;
    const auto it = index.find(std::vector<int>(p.begin(), p.end() - 1));
    if (it == index.end())  // cannot happen: a prefix is popped before its extensions
      return fail(MEDUSA_ERR_DEVICE_CHECK, "tree_from_accuracies: parent missing");
    parent[node] = it->second;
    depth[node] = (int32_t)p.size();
    rank[node] = p.back();
  }
  if (expected_accept_len != nullptr) *expected_accept_len = expected;
  return MEDUSA_OK;
}

}  // namespace medusa
