"""GPU parity: medusa_verify_accept (bit-exact from identical logits)."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import TYPICAL_LOG_MARGIN, f64, i64

pytestmark = pytest.mark.gpu


def _cands(w, spec, seed):
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk),
                      np.zeros(w.B, np.int64))
    return tb["cand"]


def _run(logits, cand, spec, mode, T=1.0, eps=0.09, delta=0.3):
    dev = "cuda"
    tree = M.Tree.from_spec(spec)
    B, N = cand.shape
    W1 = spec.max_depth + 1
    out = dict(
        accept_len=torch.full((B,), -9, dtype=torch.int32, device=dev),
        accepted_nodes=torch.full((B, W1), -9, dtype=torch.int32, device=dev),
        accepted_tokens=torch.full((B, W1), -9, dtype=torch.int32, device=dev),
        bonus=torch.full((B,), -9, dtype=torch.int32, device=dev),
    )
    status = M.new_status()
    M.medusa_verify_accept(logits.to(dev), torch.from_numpy(cand).to(dev), tree,
                           out["accept_len"], out["accepted_nodes"], out["accepted_tokens"],
                           out["bonus"], mode, T, eps, delta, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return {k: v.cpu().numpy() for k, v in out.items()}


def _assert_same(got, ref):
    for k in ("accept_len", "accepted_nodes", "accepted_tokens", "bonus"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


@pytest.mark.parametrize("name,B,V,seed", [("tiny", 1, None, 0), ("tiny", 4, None, 1),
                                            ("vicuna7b", 3, 5000, 2), ("llama3_8b", 8, 20001, 3),
                                            ("llama3_70b", 2, 9000, 4)])
def test_greedy_bit_exact(name, B, V, seed):
    w = W.scaled(W.WORKLOADS[name], B=B, V=V or W.WORKLOADS[name].V)
    spec = W.tree_for(w)
    cand = _cands(w, spec, seed)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=seed)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_GREEDY)
    ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref)


def test_greedy_ties_take_the_lowest_index():
    """bf16 logits with many exact ties at the row maximum."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=2, V=9000)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 5)
    g = torch.Generator().manual_seed(5)
    logits = torch.randint(-3, 4, (w.B, spec.n_nodes, w.V), generator=g).to(torch.bfloat16)
    # make some rows' first maximum a child candidate, with later copies of it
    for b in range(w.B):
        for i in range(0, spec.n_nodes, 3):
            kids = [c for c in range(1, spec.n_nodes) if spec.parent[c] == i]
            if kids:
                t = int(cand[b, kids[0]])
                logits[b, i, t] = 3.0
                logits[b, i, :t] = torch.clamp(logits[b, i, :t], max=2.0)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_GREEDY)
    ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref)
    assert ref["accept_len"].max() > 0


def _typical_case(w, spec, seed):
    """Redraw the logits until every candidate's |ln p - ln thr| exceeds the
    margin, so that fp32 and fp64 take the same decision."""
    cand = _cands(w, spec, seed)
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=seed, attempt=attempt)
        m = O.typical_log_margin(f64(logits), cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            return logits, cand
    pytest.skip("no margin-clean draw")


@pytest.mark.parametrize("name,B,V,seed", [("llama3_70b", 2, 6000, 0), ("llama3_70b", 1, 30000, 1),
                                            ("tiny", 2, None, 2)])
def test_typical_bit_exact(name, B, V, seed):
    base = W.WORKLOADS[name]
    w = W.scaled(base, B=B, V=V or base.V, accept="typical", temperature=0.7, eps=0.09,
                 delta=0.3)
    spec = W.tree_for(w)
    logits, cand = _typical_case(w, spec, seed)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_TYPICAL, w.temperature, w.eps, w.delta)
    ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                           w.temperature, w.eps, w.delta)
    _assert_same(got, ref)


@pytest.mark.parametrize("eps,delta,expect", [(0.0, 0.3, "deepest"), (0.09, 0.0, "deepest"),
                                              (2.0, 1e9, "root")])
def test_typical_special_cases(eps, delta, expect):
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=2, V=4000)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 7)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=7)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_TYPICAL, 0.7, eps, delta)
    ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth, 0.7, eps,
                           delta)
    _assert_same(got, ref)
    if expect == "root":
        assert (got["accept_len"] == 0).all()
    else:
        assert (got["accept_len"] == spec.max_depth).all()


@pytest.mark.slow
def test_full_size_greedy_llama3_8b():
    w = W.WORKLOADS["llama3_8b"]
    spec = W.tree_for(w)
    cand = _cands(w, spec, 0)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=0)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_GREEDY)
    ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref)


@pytest.mark.slow
def test_full_size_typical_llama3_70b():
    w = W.WORKLOADS["llama3_70b"]
    spec = W.tree_for(w)
    logits, cand = _typical_case(w, spec, 0)
    got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_TYPICAL, w.temperature, w.eps, w.delta)
    ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                           w.temperature, w.eps, w.delta)
    _assert_same(got, ref)


@pytest.mark.parametrize("mode", ["greedy", "typical"])
def test_deepest_tree_full_acceptance(mode):
    """MAX_NODES nodes at depth MAX_HEADS - 1: sequence 0's logits make the
    whole rank-0 chain the base model's choice, so it keeps the deepest
    node; the others follow the seeded draw."""
    spec = W.limits_tree(M.MAX_NODES, M.MAX_HEADS - 1, M.MAX_KMAX)
    base = W.WORKLOADS["llama3_70b"] if mode == "typical" else W.WORKLOADS["llama3_8b"]
    w = W.scaled(base, B=3, V=5000, K=M.MAX_HEADS, kmax=M.MAX_KMAX, N=spec.n_nodes)
    cand = _cands(w, spec, 11)
    chain = [i for i in range(spec.n_nodes) if all(r == 0 for r in spec.paths[i])]
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=11, attempt=attempt).float()
        for a, c in zip(chain[:-1], chain[1:]):
            logits[0, a, cand[0, c]] = logits[0, a].max() + 8.0
        logits = logits.to(torch.bfloat16)
        if mode == "greedy":
            break
        # typical: redraw until fp32 and fp64 take the same decisions
        m = O.typical_log_margin(f64(logits), cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            break
    else:
        pytest.skip("no margin-clean draw")
    if mode == "greedy":
        got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_GREEDY)
        ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
    else:
        got = _run(logits, cand, spec, M.MEDUSA_ACCEPT_TYPICAL, w.temperature, w.eps, w.delta)
        ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                               w.temperature, w.eps, w.delta)
    _assert_same(got, ref)
    assert ref["accept_len"][0] == M.MAX_HEADS - 1
    np.testing.assert_array_equal(ref["accepted_nodes"][0], chain)


def _status_of(logits, cand, spec, mode, T=0.7, eps=0.09, delta=0.3):
    dev = "cuda"
    tree = M.Tree.from_spec(spec)
    B, N = cand.shape
    W1 = spec.max_depth + 1
    outs = [torch.full(s, -9, dtype=torch.int32, device=dev) for s in ((B,), (B, W1), (B, W1), (B,))]
    status = M.new_status()
    M.medusa_verify_accept(logits.to(dev), torch.from_numpy(cand).to(dev), tree, *outs, mode, T,
                           eps, delta, dev_status=status)
    torch.cuda.synchronize()
    return int(status.item())


@pytest.mark.parametrize("dtype,mode", [(torch.bfloat16, M.MEDUSA_ACCEPT_GREEDY),
                                        (torch.bfloat16, M.MEDUSA_ACCEPT_TYPICAL),
                                        (torch.float32, M.MEDUSA_ACCEPT_GREEDY),
                                        (torch.float32, M.MEDUSA_ACCEPT_TYPICAL)])
def test_nan_logit_is_reported(dtype, mode):
    """A NaN anywhere in the logits (here in the middle of a chunk of one row,
    and in a row's ragged last chunk) is a device-check error, not a result."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=2, V=5000)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 31)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=31).to(dtype)
    assert _status_of(logits, cand, spec, mode) == 0
    for at in ((1, 3, 777), (0, spec.n_nodes - 1, w.V - 2)):
        bad = logits.clone()
        bad[at] = float("nan")
        assert _status_of(bad, cand, spec, mode) == 6, at


@pytest.mark.parametrize("mode", [M.MEDUSA_ACCEPT_GREEDY, M.MEDUSA_ACCEPT_TYPICAL])
def test_candidate_outside_the_vocabulary_is_reported(mode):
    """A candidate id outside [0, V) is reported (status 6); its logit is
    never read."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=2, V=5000)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 32)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=32)
    for bad_id in (w.V, -1):
        c = cand.copy()
        c[1, 5] = bad_id
        assert _status_of(logits, c, spec, mode) == 6, bad_id
