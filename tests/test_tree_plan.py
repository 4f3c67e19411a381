"""The native tree planner (host code, no GPU) against the oracle's
definition of the tree of the most accurate combinations."""
import numpy as np
import pytest

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W


@pytest.mark.parametrize("K,kmax,n_nodes,max_depth,seed", [
    (4, 10, 64, 4, 0), (5, 10, 64, 5, 1), (3, 4, 40, 3, 2), (2, 3, 9, 2, 3), (4, 10, 256, 4, 4),
    (4, 1, 5, 4, 5), (1, 32, 33, 1, 6)])
def test_planner_equals_oracle(K, kmax, n_nodes, max_depth, seed):
    rng = np.random.default_rng(seed)
    acc = rng.uniform(0, 1, size=(K, kmax)).astype(np.float32)
    if seed % 2:
        acc[:, 0] = 1.0       # ties along paths
        if kmax > 1:
            acc[1:, 1] = acc[0, 1]  # and between paths
    parent, depth, rank, e = M.medusa_tree_from_accuracies(acc, n_nodes, max_depth)
    ref = O.tree_from_accuracies(acc.astype(np.float64), n_nodes, max_depth)
    np.testing.assert_array_equal(parent, ref["parent"])
    np.testing.assert_array_equal(depth, ref["depth"])
    np.testing.assert_array_equal(rank, ref["rank"])
    assert abs(e - ref["expected_accept_len"]) < 1e-12


def test_planner_glossary_tree_and_errors():
    acc = np.array([[0.6, 0.3, 0.0], [0.5, 0.3, 0.2]], dtype=np.float32)
    parent, depth, rank, _ = M.medusa_tree_from_accuracies(acc, 9, 2)
    ref = W.cartesian_tree([2, 3])
    np.testing.assert_array_equal(parent, ref.parent)
    np.testing.assert_array_equal(rank, ref.rank)
    with pytest.raises(M.MedusaError) as e:  # only 3 + 9 paths exist
        M.medusa_tree_from_accuracies(acc, 14, 2)
    assert e.value.status == 2
    with pytest.raises(M.MedusaError) as e:
        M.medusa_tree_from_accuracies(acc * 2.0, 5, 2)
    assert e.value.status == 1


def test_limits_tree_shape():
    """The size-limit tree of the parity tests: the rank-0 chain reaches the
    requested depth, ranks reach kmax - 1, every node's parent precedes it,
    and nodes are in breadth-first order."""
    spec = W.limits_tree(M.MAX_NODES, M.MAX_HEADS, M.MAX_KMAX)
    assert spec.n_nodes == M.MAX_NODES
    assert spec.max_depth == M.MAX_HEADS and spec.rank.max() == M.MAX_KMAX - 1
    assert all(spec.parent[i] < i for i in range(1, spec.n_nodes))
    assert list(spec.depth) == sorted(spec.depth)
    chain = [i for i in range(spec.n_nodes) if all(r == 0 for r in spec.paths[i])]
    assert len(chain) == M.MAX_HEADS + 1
