"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a value
the pages print, a closed form, a brute-force enumeration or a library routine
(CPU only)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")
LN3 = math.log(3.0)


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# heads
# ----------------------------------------------------------------------------


def test_zero_init_heads_reproduce_lm_head_exactly():
    """The glossary's example: 3 zero-initialised heads over hidden 256 /
    vocab 1000 each equal lm_head(h) exactly -> [True, True, True]."""
    g = _gold("zero_init_heads.json")
    w = W.WORKLOADS["tiny"]
    assert (w.d, w.V, w.K) == (g["hidden_size"], g["vocab_size"], g["num_heads"])
    inp = W.heads_inputs(w, seed=0, zero_init=True)
    h = inp["h"].double().numpy()
    z = O.head_logits(h, inp["W1"].double().numpy(), inp["b1"].double().numpy(),
                      inp["W2"].double().numpy())
    base = O.lm_head_logits(h, inp["lm_head"].double().numpy())
    got = [bool(np.array_equal(z[:, k, :], base)) for k in range(w.K)]
    assert got == g["printed"]


def test_silu_closed_forms_through_the_head():
    """h = 0, W1 = 0, W2 = I: the logits are SiLU(b1).  sigmoid(ln 3) = 3/4,
    sigmoid(-ln 3) = 1/4, sigmoid(0) = 1/2, so SiLU takes the values below
    (a sign error in the exponent swaps 3/4 and 1/4)."""
    d = 4
    b1 = np.array([[LN3, -LN3, 0.0, 2.0 * LN3]])
    z = O.head_logits(np.zeros((1, d)), np.zeros((1, d, d)), b1, np.eye(d)[None])
    # sigmoid(2 ln 3) = 9/10
    expect = [0.75 * LN3, -0.25 * LN3, 0.0, 0.9 * 2.0 * LN3]
    np.testing.assert_allclose(z[0, 0], expect, rtol=0, atol=1e-15)


def test_head_orientation_residual_and_bias():
    """Hand-computed 2-feature head: W1 = [[0,1],[0,0]] maps feature 1 into
    output feature 0, h = [0, ln 3], b1 = [0, 0]:
    u = [ln 3, 0], y = h + SiLU(u) = [3/4 ln 3, ln 3],
    W2 = [[1,0],[0,1],[1,1]] -> z = [3/4 ln 3, ln 3, 7/4 ln 3].
    A transposed W1 would give z = [0, ln 3, ln 3]; a missing residual
    [3/4 ln 3, 0, 3/4 ln 3]."""
    W1 = np.array([[[0.0, 1.0], [0.0, 0.0]]])
    W2 = np.array([[[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]]])
    z = O.head_logits(np.array([[0.0, LN3]]), W1, np.zeros((1, 2)), W2)
    np.testing.assert_allclose(z[0, 0], [0.75 * LN3, LN3, 1.75 * LN3], atol=1e-15)
    # bias enters before the SiLU: W1 = 0, b1 = [0, ln 3], h = 0 -> y = [0, 3/4 ln 3]
    z = O.head_logits(np.zeros((1, 2)), np.zeros((1, 2, 2)), np.array([[0.0, LN3]]), W2)
    np.testing.assert_allclose(z[0, 0], [0.0, 0.75 * LN3, 0.75 * LN3], atol=1e-15)


def test_head_and_batch_indexing():
    """Two heads, two sequences: head 1's W2 is minus head 0's, so the logits
    of head 1 are minus those of head 0 when the residual blocks agree; each
    sequence's logits depend on its own hidden state only."""
    rng = np.random.default_rng(1)
    d, V = 6, 5
    W1 = np.stack([rng.standard_normal((d, d))] * 2)
    b1 = np.stack([rng.standard_normal(d)] * 2)
    W2a = rng.standard_normal((V, d))
    W2 = np.stack([W2a, -W2a])
    h = rng.standard_normal((2, d))
    z = O.head_logits(h, W1, b1, W2)
    np.testing.assert_array_equal(z[:, 1], -z[:, 0])
    z0 = O.head_logits(h[:1], W1, b1, W2)
    np.testing.assert_allclose(z0[0], z[0], rtol=0, atol=1e-13)
    assert not np.allclose(z[0], z[1])


def test_topk_literal_and_bruteforce():
    ids, vals = O.topk(np.array([3.0, 1.0, 3.0, 2.0, 5.0]), 3)
    assert ids.tolist() == [4, 0, 2] and vals.tolist() == [5.0, 3.0, 3.0]
    rng = np.random.default_rng(2)
    for _ in range(20):
        z = rng.integers(-3, 4, size=(3, 17)).astype(np.float64)  # many ties
        k = int(rng.integers(1, 10))
        ids, _ = O.topk(z, k)
        for r in range(3):
            ref = sorted(range(17), key=lambda i: (-z[r, i], i))[:k]
            assert ids[r].tolist() == ref


# ----------------------------------------------------------------------------
# tree
# ----------------------------------------------------------------------------


def test_cartesian_2x3_tree_from_the_glossary():
    g = _gold("cartesian_2x3.json")
    spec = W.cartesian_tree(g["widths"])
    assert spec.parent.tolist() == g["parent"]
    assert spec.depth.tolist() == g["depth"]
    assert spec.rank.tolist() == g["rank"]
    ex = g["example"]
    topk_ids = np.array([[ex["topk_ids_head1"], ex["topk_ids_head2"]]], dtype=np.int32)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, np.array([ex["root_tok"]]),
                      topk_ids, np.array([ex["prefix_len"]]))
    assert tb["retrieve"].shape[0] == g["n_candidates"] == 6
    assert tb["retrieve"].tolist() == g["retrieve"]
    assert tb["cand"][0].tolist() == ex["cand"]
    assert tb["pos"][0].tolist() == ex["pos"]
    # head 2 proposes the same tokens under each head-1 branch
    assert tb["cand"][0, 3:6].tolist() == tb["cand"][0, 6:9].tolist()
    for i, anc in enumerate(g["ancestor_or_self"]):
        seen = [j for j in range(9) if O.mask_bit(tb["mask"], i, j)]
        assert seen == anc
    # literal mask words: row 3 = bits {0,1,3}, row 6 = bits {0,2,6}
    assert int(tb["mask"][3, 0]) == 0b1011 and int(tb["mask"][6, 0]) == 1 + 4 + 64


def _random_tree(rng, n):
    paths = [()]
    while len(paths) < n:
        p = paths[int(rng.integers(len(paths)))]
        if len(p) >= 4:
            continue
        c = p + (int(rng.integers(3)),)
        if c not in paths:
            paths.append(c)
    return W._spec_from_paths(paths)


def test_mask_equals_transitive_closure_and_paths_are_root_to_leaf():
    """Ancestor-or-self mask vs the reflexive-transitive closure of the
    child->parent relation computed by boolean matrix powers; retrieve rows
    vs brute-force enumeration of root-to-leaf chains."""
    rng = np.random.default_rng(3)
    specs = [_random_tree(rng, n) for n in range(1, 13) for _ in range(3)]
    specs += [W.tree_for(W.WORKLOADS["llama3_8b"]), W.tree_for(W.WORKLOADS["llama3_70b"])]
    for spec in specs:
        N = spec.n_nodes
        A = np.zeros((N, N), dtype=np.int64)
        for i in range(1, N):
            A[i, spec.parent[i]] = 1
        R = np.eye(N, dtype=np.int64)
        P = np.eye(N, dtype=np.int64)
        for _ in range(N):
            P = np.minimum(P @ A, 1)
            R = np.minimum(R + P, 1)
        K = max(1, spec.max_depth)
        tb = O.tree_build(spec.parent, spec.depth, spec.rank, np.array([0]),
                          np.zeros((1, K, 16), np.int32), np.array([0]))
        for i in range(N):
            for j in range(N):
                assert O.mask_bit(tb["mask"], i, j) == bool(R[i, j])
        leaves = [i for i in range(N) if not any(spec.parent[c] == i for c in range(1, N))]
        assert tb["retrieve"].shape == (len(leaves), spec.max_depth + 1) == (spec.n_leaves, spec.max_depth + 1)
        for row, leaf in zip(tb["retrieve"], leaves):
            path = [int(x) for x in row if x >= 0]
            assert path[0] == 0 and path[-1] == leaf
            assert all(spec.parent[path[t + 1]] == path[t] for t in range(len(path) - 1))
            assert all(x == -1 for x in row[len(path):])


def test_tree_shapes_of_the_workloads():
    dense = W.tree_for(W.WORKLOADS["llama3_70b"])
    assert dense.n_nodes == 256
    assert np.bincount(dense.depth).tolist() == [1, 4, 16, 64, 171]
    s16, s64, s128 = (W.sparse_tree(n, 4, 10, 0, max_depth=4) for n in (16, 64, 128))
    assert s64.n_nodes == 64 and s64.max_depth <= 4
    assert set(s16.paths) <= set(s64.paths) <= set(s128.paths)
    v = W.tree_for(W.WORKLOADS["vicuna7b"])
    assert v.n_nodes == 64 and v.max_depth <= 5
    for spec in (dense, s16, s64, s128, v):
        assert all(spec.parent[i] < i for i in range(1, spec.n_nodes))


# ----------------------------------------------------------------------------
# tree attention
# ----------------------------------------------------------------------------


def _attn_case(seed, B=2, N=9, Hq=4, Hkv=2, dh=8, ctx=(5, 11), spec=None):
    rng = np.random.default_rng(seed)
    spec = spec or W.cartesian_tree([2, 3])
    N = spec.n_nodes
    cap = max(ctx) + N + 3
    P = np.array([ctx[b % len(ctx)] for b in range(B)], dtype=np.int32)
    q = rng.standard_normal((B, N, Hq, dh))
    kn = rng.standard_normal((B, N, Hkv, dh))
    vn = rng.standard_normal((B, N, Hkv, dh))
    Kc = rng.standard_normal((B, Hkv, cap, dh))
    Vc = rng.standard_normal((B, Hkv, cap, dh))
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, np.zeros(B, np.int32),
                      np.zeros((B, max(1, spec.max_depth), 16), np.int32), P)
    return spec, q, kn, vn, Kc, Vc, P, tb["mask"]


def test_tree_attention_equals_causal_attention_along_each_path():
    """Node i's output equals ordinary causal attention (a library routine,
    torch SDPA in fp64) for the linear sequence prefix + root->i path, at its
    last position."""
    spec, q, kn, vn, Kc, Vc, P, mask = _attn_case(4)
    B, N, Hq, dh = q.shape
    Hkv = kn.shape[2]
    scale = 1.0 / math.sqrt(dh)
    got = O.tree_attention(q, kn, vn, Kc, Vc, P, mask, scale)["out"]
    for b in range(B):
        for i in range(N):
            path = []
            j = i
            while j >= 0:
                path.append(j)
                j = int(spec.parent[j])
            path.reverse()
            for hq in range(Hq):
                kv = hq // (Hq // Hkv)
                keys = np.concatenate([Kc[b, kv, :P[b]], kn[b, path, kv]], 0)
                vals = np.concatenate([Vc[b, kv, :P[b]], vn[b, path, kv]], 0)
                ref = torch.nn.functional.scaled_dot_product_attention(
                    torch.from_numpy(q[b, i, hq][None, None, None]),
                    torch.from_numpy(keys[None, None]), torch.from_numpy(vals[None, None]),
                    scale=scale)[0, 0, 0].numpy()
                np.testing.assert_allclose(got[b, i, hq], ref, rtol=0, atol=1e-12)


def test_tree_attention_zero_query_is_mean_of_visible_values():
    """q = 0 gives equal weights, so the output is the mean of the values in
    the visible set (prefix plus ancestors-or-self): a closed form that pins
    the size of the visible set."""
    spec, q, kn, vn, Kc, Vc, P, mask = _attn_case(5)
    q[:] = 0.0
    out = O.tree_attention(q, kn, vn, Kc, Vc, P, mask, 0.125)["out"]
    for b in range(q.shape[0]):
        for i in range(spec.n_nodes):
            anc = [j for j in range(spec.n_nodes) if O.mask_bit(mask, i, j)]
            n_vis = P[b] + len(anc)
            for hq in range(q.shape[2]):
                kv = hq // 2
                total = Vc[b, kv, :P[b]].sum(0) + vn[b, anc, kv].sum(0)
                np.testing.assert_allclose(out[b, i, hq], total / n_vis, atol=1e-13)


def test_tree_attention_grouped_query_mapping_and_cache_write():
    """Hq = 4, Hkv = 2: query heads 0,1 read kv head 0 and heads 2,3 read kv
    head 1 (contiguous groups).  Constant values per kv head make the output
    equal that constant.  The tree K/V land at slots P + i."""
    spec, q, kn, vn, Kc, Vc, P, mask = _attn_case(6)
    Vc[:, 0] = 1.5
    Vc[:, 1] = -2.0
    vn[:, :, 0] = 1.5
    vn[:, :, 1] = -2.0
    res = O.tree_attention(q, kn, vn, Kc, Vc, P, mask, 0.3)
    np.testing.assert_allclose(res["out"][:, :, :2], 1.5, atol=1e-13)
    np.testing.assert_allclose(res["out"][:, :, 2:], -2.0, atol=1e-13)
    for b in range(q.shape[0]):
        for i in range(spec.n_nodes):
            np.testing.assert_array_equal(res["Kc"][b, :, P[b] + i], kn[b, i])
            np.testing.assert_array_equal(res["Vc"][b, :, P[b] + i], vn[b, i])
        # slots before the prefix are untouched
        np.testing.assert_array_equal(res["Kc"][b, :, :P[b]], Kc[b, :, :P[b]])


# ----------------------------------------------------------------------------
# verification and acceptance
# ----------------------------------------------------------------------------


def _brute_force_greedy(logits, cand, spec):
    """Enumerate every root->leaf chain; its accepted length is the number of
    successive candidates that equal the model's choice at the previous node.
    The answer is the deepest reachable node (lowest index on ties)."""
    N = spec.n_nodes
    best = 0
    for leaf in range(N):
        path = []
        j = leaf
        while j >= 0:
            path.append(j)
            j = int(spec.parent[j])
        path.reverse()
        L = 0
        while L + 1 < len(path) and int(np.argmax(logits[path[L]])) == cand[path[L + 1]]:
            L += 1
        node = path[L]
        if spec.depth[node] > spec.depth[best] or (spec.depth[node] == spec.depth[best] and node < best):
            best = node
    return best


def test_greedy_acceptance_matches_bruteforce_paths():
    rng = np.random.default_rng(7)
    for trial in range(60):
        spec = _random_tree(rng, int(rng.integers(2, 14))) if trial % 3 else W.cartesian_tree([2, 3])
        N, V = spec.n_nodes, 12
        cand = rng.integers(0, V, size=(1, N)).astype(np.int32)
        logits = rng.standard_normal((1, N, V))
        for i in range(N):  # force agreement on some children
            kids = [c for c in range(1, N) if spec.parent[c] == i]
            if kids and rng.uniform() < 0.7:
                logits[0, i, cand[0, kids[int(rng.integers(len(kids)))]]] = 10.0
        res = O.verify_greedy(logits, cand, spec.parent, spec.depth, spec.max_depth)
        best = _brute_force_greedy(logits[0], cand[0], spec)
        assert res["accept_len"][0] == spec.depth[best]
        assert res["accepted_nodes"][0, res["accept_len"][0]] == best
        assert res["bonus"][0] == int(np.argmax(logits[0, best]))


def test_greedy_acceptance_literal_example():
    """Glossary tree (top-2 x top-3).  The model's choice at the root is node
    2's token and at node 2 it is node 7's token: the kept branch is
    0 -> 2 -> 7, two candidates accepted, then the bonus token."""
    spec = W.cartesian_tree([2, 3])
    cand = np.array([[7, 100, 101, 200, 201, 202, 200, 201, 202]], dtype=np.int32)
    V = 300
    logits = np.zeros((1, 9, V))
    logits[0, 0, 101] = 1.0   # root -> node 2
    logits[0, 2, 201] = 1.0   # node 2 -> node 7
    logits[0, 7, 42] = 1.0    # bonus
    res = O.verify_greedy(logits, cand, spec.parent, spec.depth, 2)
    assert res["accept_len"].tolist() == [2]
    assert res["accepted_nodes"].tolist() == [[0, 2, 7]]
    assert res["accepted_tokens"].tolist() == [[101, 201, 42]]
    assert res["bonus"].tolist() == [42]
    # nothing agrees -> only the root, bonus = model's choice at the root
    logits2 = np.zeros((1, 9, V))
    logits2[0, 0, 5] = 1.0
    res2 = O.verify_greedy(logits2, cand, spec.parent, spec.depth, 2)
    assert res2["accept_len"].tolist() == [0]
    assert res2["accepted_tokens"].tolist() == [[5, -1, -1]]
    # equal maxima: the lowest index is the first choice
    logits3 = np.zeros((1, 9, V))
    logits3[0, 0, [100, 101]] = 1.0
    res3 = O.verify_greedy(logits3, cand, spec.parent, spec.depth, 2)
    assert res3["accepted_nodes"][0, 1] == 1


def test_typical_threshold_closed_forms():
    """Uniform row over V tokens: p = 1/V, H = ln V, thr = min(eps, delta/V),
    so the log-margin is -ln(delta) when delta/V < eps.  Two tokens with
    logits [ln 3, 0] at T = 1: p = (3/4, 1/4), H = ln 4 - (3/4) ln 3; at T = 1/2
    the scaled logits are [2 ln 3, 0] so p = (9/10, 1/10)."""
    spec = W.cartesian_tree([1])          # root + one child
    V = 64
    cand = np.array([[0, 5]], dtype=np.int32)
    logits = np.zeros((1, 2, V))
    m = O.typical_log_margin(logits, cand, spec.parent, 1.0, 1.0, 0.5)
    assert abs(m[0, 1] - math.log(2.0)) < 1e-12
    m = O.typical_log_margin(logits, cand, spec.parent, 1.0, 1.0, 2.0)
    assert abs(m[0, 1] + math.log(2.0)) < 1e-12
    two = np.array([[[LN3, 0.0], [0.0, 0.0]]])
    c0 = np.array([[0, 0]], dtype=np.int32)
    c1 = np.array([[0, 1]], dtype=np.int32)
    H = math.log(4.0) - 0.75 * LN3
    # eps large, delta = 1: thr = exp(-H); margin = ln p - ln thr = ln p + H
    assert abs(O.typical_log_margin(two, c0, spec.parent, 1.0, 10.0, 1.0)[0, 1]
               - (math.log(0.75) + H)) < 1e-12
    assert abs(O.typical_log_margin(two, c1, spec.parent, 1.0, 10.0, 1.0)[0, 1]
               - (math.log(0.25) + H)) < 1e-12
    H2 = -(0.9 * math.log(0.9) + 0.1 * math.log(0.1))
    assert abs(O.typical_log_margin(two, c1, spec.parent, 0.5, 10.0, 1.0)[0, 1]
               - (math.log(0.1) + H2)) < 1e-12
    # eps binds: thr = eps
    assert abs(O.typical_log_margin(two, c0, spec.parent, 1.0, 0.01, 1.0)[0, 1]
               - (math.log(0.75) - math.log(0.01))) < 1e-12


def test_typical_special_cases():
    """eps = 0 or delta = 0 makes the threshold 0: every candidate passes and
    the deepest node (lowest index) is kept.  A threshold above 1 rejects
    everything: only the root, bonus = the model's choice at the root."""
    spec = W.cartesian_tree([2, 3])
    rng = np.random.default_rng(8)
    cand = rng.integers(0, 50, size=(2, 9)).astype(np.int32)
    logits = rng.standard_normal((2, 9, 50))
    for eps, delta in ((0.0, 0.3), (0.09, 0.0)):
        res = O.verify_typical(logits, cand, spec.parent, spec.depth, 2, 0.7, eps, delta)
        assert res["accept_len"].tolist() == [2, 2]
        assert res["accepted_nodes"][:, 2].tolist() == [3, 3]
    res = O.verify_typical(logits, cand, spec.parent, spec.depth, 2, 0.7, 2.0, 1e9)
    assert res["accept_len"].tolist() == [0, 0]
    assert res["bonus"].tolist() == np.argmax(logits[:, 0], -1).tolist()


# ----------------------------------------------------------------------------
# KV compaction
# ----------------------------------------------------------------------------


def test_kv_compact_literal_and_out_of_place_equivalence():
    rng = np.random.default_rng(9)
    Kc = rng.standard_normal((1, 2, 20, 4))
    Vc = rng.standard_normal((1, 2, 20, 4))
    res = O.kv_compact(Kc, Vc, np.array([4]), np.array([[0, 2, 7]]), np.array([2]))
    assert res["prefix_len"].tolist() == [7]
    assert res["compact_src"].tolist() == [[4, 6, 11]]
    np.testing.assert_array_equal(res["Kc"][0, :, 5], Kc[0, :, 6])
    np.testing.assert_array_equal(res["Vc"][0, :, 6], Vc[0, :, 11])
    np.testing.assert_array_equal(res["Kc"][0, :, :4], Kc[0, :, :4])
    # chains whose sources overlap later destinations: in-place ascending
    # equals an out-of-place gather from the untouched cache
    for nodes in ([0, 2, 3, 5], [0, 1, 2, 3], [0, 3, 4, 9], [0, 2, 6, 7]):
        L = len(nodes) - 1
        res = O.kv_compact(Kc, Vc, np.array([6]), np.array([nodes]), np.array([L]))
        for j, n in enumerate(nodes):
            np.testing.assert_array_equal(res["Kc"][0, :, 6 + j], Kc[0, :, 6 + n])
            np.testing.assert_array_equal(res["Vc"][0, :, 6 + j], Vc[0, :, 6 + n])
        np.testing.assert_array_equal(res["Kc"][0, :, 6 + L + 1:], Kc[0, :, 6 + L + 1:])


# ----------------------------------------------------------------------------
# Verification from hidden states (lm_head fused in front of the verify)
# ----------------------------------------------------------------------------


def test_lmhead_verify_planted_basis_rows():
    """lm_head rows are scaled unit vectors (V = 300 < d = 320, so a transposed
    operand cannot even multiply) and every node's hidden state is the unit
    vector of the token its model should choose: the glossary example of the
    greedy literal test is reproduced, and the logits are the planted values."""
    spec = W.cartesian_tree([2, 3])
    V, d = 300, 320
    lm = np.zeros((V, d))
    lm[np.arange(V), np.arange(V)] = 1.0 + np.arange(V) / 1000.0
    cand = np.array([[7, 100, 101, 200, 201, 202, 200, 201, 202]], dtype=np.int32)
    want = {0: 101, 2: 201, 7: 42}
    hidden = np.zeros((1, 9, d))
    for n in range(9):
        hidden[0, n, want.get(n, 250 + n)] = 1.0
    res = O.lmhead_verify(hidden, lm, cand, spec.parent, spec.depth, 2)
    assert res["accept_len"].tolist() == [2]
    assert res["accepted_nodes"].tolist() == [[0, 2, 7]]
    assert res["accepted_tokens"].tolist() == [[101, 201, 42]]
    assert res["logits"].shape == (1, 9, V)
    assert res["logits"][0, 2, 201] == 1.0 + 201 / 1000.0
    assert np.count_nonzero(res["logits"]) == 9


def test_lmhead_verify_logits_bruteforce_and_typical_mode():
    rng = np.random.default_rng(11)
    B, N, d, V = 2, 4, 5, 7
    spec = W.cartesian_tree([3])
    hidden = rng.standard_normal((B, N, d))
    lm = rng.standard_normal((V, d))
    cand = rng.integers(0, V, size=(B, N)).astype(np.int32)
    res = O.lmhead_verify(hidden, lm, cand, spec.parent, spec.depth, 1, "typical", 0.8, 0.3, 0.5)
    for b in range(B):
        for n in range(N):
            for v in range(V):
                s = 0.0
                for j in range(d):
                    s += hidden[b, n, j] * lm[v, j]
                assert abs(res["logits"][b, n, v] - s) < 1e-12
    # the typical decision depends only on the logits: same result as the
    # logits-level verify on the brute-force logits
    z = np.einsum("bnj,vj->bnv", hidden, lm)
    ref = O.verify_typical(z, cand, spec.parent, spec.depth, 1, 0.8, 0.3, 0.5)
    assert res["accept_len"].tolist() == ref["accept_len"].tolist()
    assert res["bonus"].tolist() == ref["bonus"].tolist()


def test_next_step_inputs_take_the_kept_node_and_bonus():
    """Glossary tree, kept branch 0 -> 2 -> 7 for sequence 0 and the root
    only for sequence 1: the next heads read node 7's (resp. node 0's) hidden
    state and the next root is each sequence's bonus token."""
    spec = W.cartesian_tree([2, 3])
    cand = np.array([[7, 100, 101, 200, 201, 202, 200, 201, 202]] * 2, dtype=np.int32)
    V, d = 300, 320
    lm = np.zeros((V, d))
    lm[np.arange(V), np.arange(V)] = 1.0
    hidden = np.zeros((2, 9, d))
    for n, t in {0: 101, 2: 201, 7: 42}.items():
        hidden[0, n, t] = 1.0
    hidden[1, 0, 9] = 1.0
    for n in range(9):
        hidden[:, n, 300 + n % 20] += 0.5  # node-specific tag outside the vocabulary
    res = O.lmhead_verify(hidden, lm, cand, spec.parent, spec.depth, 2)
    h_next, root_next = O.next_step_inputs(hidden, res["accept_len"], res["accepted_nodes"],
                                           res["bonus"])
    np.testing.assert_array_equal(h_next[0], hidden[0, 7])
    np.testing.assert_array_equal(h_next[1], hidden[1, 0])
    assert root_next.tolist() == [42, 9]


# ----------------------------------------------------------------------------
# Sparse tree from head accuracies
# ----------------------------------------------------------------------------


def _ancestor_closed_subsets(paths, size):
    """All subsets of ``paths`` of the given size that contain every prefix
    of each member (brute force, tiny inputs only)."""
    pset = set(paths)
    for combo in itertools.combinations(paths, size):
        s = set(combo)
        if all((p[:-1] in s or len(p) == 1) for p in s) and s <= pset:
            yield s


def test_tree_from_accuracies_maximises_expected_accept_length():
    """Brute force over every ancestor-closed set of rank paths: the tree
    reaches the largest expected accept length (sum of path products)."""
    rng = np.random.default_rng(12)
    for trial in range(12):
        K, kmax = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        acc = rng.uniform(0, 1, size=(K, kmax))
        if trial % 4 == 0:
            acc[:, 0] = 1.0  # products equal along a path: ties
        paths = [p for t in range(1, K + 1) for p in itertools.product(range(kmax), repeat=t)]
        n_nodes = int(rng.integers(1, min(len(paths), 7) + 1)) + 1

        def value(s):
            return sum(np.prod([acc[i, r] for i, r in enumerate(p)]) for p in s)

        best = max(value(s) for s in _ancestor_closed_subsets(paths, n_nodes - 1))
        t = O.tree_from_accuracies(acc, n_nodes, K)
        assert abs(t["expected_accept_len"] - best) < 1e-12
        assert t["parent"].shape == (n_nodes,)
        # a valid tree in BFS order
        for i in range(1, n_nodes):
            assert 0 <= t["parent"][i] < i
            assert t["depth"][i] == t["depth"][t["parent"][i]] + 1


def test_tree_from_accuracies_glossary_shape():
    """Head 1 right with 0.6 / 0.3 for ranks 0 / 1, head 2 with 0.5 / 0.3 /
    0.2 for ranks 0..2 and nothing else: the 9-node tree is the glossary's
    top-2 x top-3 Cartesian tree."""
    acc = np.array([[0.6, 0.3, 0.0], [0.5, 0.3, 0.2]])
    t = O.tree_from_accuracies(acc, 9, 2)
    ref = W.cartesian_tree([2, 3])
    np.testing.assert_array_equal(t["parent"], ref.parent)
    np.testing.assert_array_equal(t["depth"], ref.depth)
    np.testing.assert_array_equal(t["rank"], ref.rank)
    assert abs(t["expected_accept_len"] - (0.9 + 0.9 * 1.0)) < 1e-12


# ----------------------------------------------------------------------------
# Sampled bonus token (Philox4x32-10, inverse CDF)
# ----------------------------------------------------------------------------


def test_philox_known_answers():
    """Known-answer vectors of Philox4x32-10 from the reference distribution
    of Salmon et al., SC 2011 (zero, all-ones and pi-digit counter/key)."""
    assert O.philox4x32_10([0, 0, 0, 0], [0, 0]) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert O.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == \
        [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert O.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344],
                           [0xA4093822, 0x299F31D0]) == \
        [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_sample_bonus_closed_forms():
    """Uniform row: the token is floor(u * V).  A row with one logit far
    above the rest: always that token.  The kept node's row is the one read."""
    B, N, V = 5, 3, 1000
    logits = np.zeros((B, N, V))
    nodes = np.array([[0, 2, -1]] * B, dtype=np.int32)
    acc = np.ones(B, dtype=np.int32)  # kept node 2
    logits[:, 0, 7] = 1e3            # the root row must not be read
    got = O.sample_bonus(logits, acc, nodes, 0.9, 1234, 5)
    for b in range(B):
        assert got[b] == int(O.bonus_uniform(1234, 5, b) * V)
    logits[:, 2, 321] = 200.0
    assert (O.sample_bonus(logits, acc, nodes, 1.0, 99, 0) == 321).all()
    # different offsets give different draws
    us = {O.bonus_uniform(7, off, 0) for off in range(8)}
    assert len(us) == 8


def test_bonus_uniform_literals():
    """The uniform number of a sequence, pinned by literals.

    Counter 0 and key 0 give the first word 0x6627E8D5 (known-answer vector
    above), so the top 24 bits of word 0 give 0x6627E8 * 2^-24: taking
    another word (0xE169C58D) or the low 24 bits (0x27E8D5) fails here.
    The second literal is the generator's first word, 0xE1E5F2BB, for key
    (0x89ABCDEF, 0x01234567) and counter (0x76543210, 0xFEDCBA98, 5, 0),
    computed from the published round function by a separate C program; it
    fixes the counter/key layout of seed, offset and sequence index."""
    assert O.bonus_uniform(0, 0, 0) == 0x6627E8 * 2.0 ** -24
    seed, offset, b = 0x0123456789ABCDEF, 0xFEDCBA9876543210, 5
    assert O.bonus_uniform(seed, offset, b) == 0xE1E5F2 * 2.0 ** -24
    # every plausible misreading of the layout gives another number
    lo, hi = offset & 0xFFFFFFFF, offset >> 32
    klo, khi = seed & 0xFFFFFFFF, seed >> 32
    wrong = [
        O.philox4x32_10([b, hi, lo, 0], [klo, khi])[0],     # offset and b swapped
        O.philox4x32_10([hi, lo, b, 0], [klo, khi])[0],     # offset halves swapped
        O.philox4x32_10([lo, hi, b, 0], [khi, klo])[0],     # key halves swapped
        O.philox4x32_10([lo, hi, 0, b], [klo, khi])[0],     # b in the last word
    ]
    assert all((w >> 8) != 0xE1E5F2 for w in wrong)
