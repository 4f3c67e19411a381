"""Losslessness of greedy Medusa decoding, by brute force on a toy model.

"Medusa Decoding Heads" overview, "Diepe duik": the base model verifies the
whole tree, so the accepted text is exactly what plain greedy decoding would
produce.  The oracle's tree build, tree attention, greedy acceptance and KV
compaction are composed into Medusa decoding of a one-layer model and compared
with plain token-by-token greedy decoding: same tokens, and a cache that holds
bit-identical K/V for every kept token."""
import numpy as np
import pytest

from oracle.toy_lm import ToyLM, greedy_decode, medusa_decode
from speculative_decoding_medusa_b200 import workloads as W


def _proposer(ar_tokens, K, kmax, V, seed, hit=0.7):
    rng = np.random.default_rng(seed)

    def propose(step, n_done):
        # head t (1-based) guesses the token t places after the root; rank 0
        # is the true continuation with probability ``hit``
        ids = np.zeros((K, kmax), dtype=np.int32)
        for t in range(1, K + 1):
            true = ar_tokens[n_done + t] if n_done + t < len(ar_tokens) else 0
            first = true if rng.uniform() < hit else int(rng.integers(V))
            rest = [x for x in rng.permutation(V) if x != first][: kmax - 1]
            ids[t - 1] = [first] + rest
        return ids

    return propose


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tree", ["cartesian:2,3", "cartesian:3,2,2", "sparse"])
def test_greedy_medusa_equals_greedy_decoding(seed, tree):
    m = ToyLM(seed=seed)
    if tree == "sparse":
        spec = W.sparse_tree(12, 3, 3, seed, max_depth=3)
    else:
        spec = W.cartesian_tree([int(x) for x in tree.split(":")[1].split(",")])
    K = spec.max_depth
    kmax = 3
    prompt = [int(x) for x in np.random.default_rng(100 + seed).integers(0, m.V, size=5)]
    n_new = 24
    ar, _, _ = greedy_decode(m, prompt, n_new + 2 * (K + 1) + 1)
    res = medusa_decode(m, prompt, n_new, spec.parent, spec.depth, spec.rank, kmax,
                        _proposer(ar, K, kmax, m.V, seed))
    assert res["tokens"] == ar[:n_new]
    assert sum(res["accepted_per_step"]) > 0, "no candidate was ever accepted"
    # the compacted cache equals the cache plain decoding writes, bit for bit
    P = res["prefix_len"]
    emitted = P - len(prompt)
    _, Kar, Var = greedy_decode(m, prompt, emitted + 1)
    assert Kar.shape[1] == P
    np.testing.assert_array_equal(res["Kc"][0, :, :P], Kar)
    np.testing.assert_array_equal(res["Vc"][0, :, :P], Var)
