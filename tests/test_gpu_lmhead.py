"""GPU parity: medusa_lmhead_verify (lm_head GEMM reduced in its epilogue,
then the acceptance) against the oracle's lmhead_verify."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import TYPICAL_LOG_MARGIN, f64, i64

pytestmark = pytest.mark.gpu

LOGIT_ABS = 2e-3       # fp32 tensor-core sum of d bf16 products vs fp64


def _cands(w, spec, seed):
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk),
                      np.zeros(w.B, np.int64))
    return tb["cand"]


def _oracle_logits(hidden, lm):
    B, N, d = hidden.shape
    return O.lm_head_logits(f64(hidden).reshape(B * N, d), f64(lm)).reshape(B, N, -1)


def _run(hidden, lm, cand, spec, mode, T=1.0, eps=0.09, delta=0.3, want_logits=False):
    dev = "cuda"
    tree = M.Tree.from_spec(spec)
    B, N = cand.shape
    V = lm.shape[0]
    W1 = spec.max_depth + 1
    out = dict(
        accept_len=torch.full((B,), -9, dtype=torch.int32, device=dev),
        accepted_nodes=torch.full((B, W1), -9, dtype=torch.int32, device=dev),
        accepted_tokens=torch.full((B, W1), -9, dtype=torch.int32, device=dev),
        bonus=torch.full((B,), -9, dtype=torch.int32, device=dev),
    )
    logits = torch.full((B, N, V), float("nan"), device=dev) if want_logits else None
    status = M.new_status()
    M.medusa_lmhead_verify(hidden.to(dev), lm.to(dev), torch.from_numpy(cand).to(dev), tree,
                           out["accept_len"], out["accepted_nodes"], out["accepted_tokens"],
                           out["bonus"], mode, T, eps, delta, logits=logits, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    res = {k: v.cpu().numpy() for k, v in out.items()}
    if want_logits:
        res["logits"] = logits.cpu().double().numpy()
    return res


def _assert_same(got, ref):
    for k in ("accept_len", "accepted_nodes", "accepted_tokens", "bonus"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def _check_logits(got, z):
    """The GEMM's fp32 logits against the fp64 oracle, and its argmax (taken
    by the kernel on those fp32 values) against the oracle's: the same token
    on every row whose oracle top-2 gap exceeds twice the logit tolerance,
    a near-tie within that tolerance elsewhere."""
    zg = got["logits"]
    assert np.abs(zg - z).max() < LOGIT_ABS
    g_gpu = np.argmax(zg, axis=-1)
    g_ora = np.argmax(z, axis=-1)
    zmax = z.max(axis=-1)
    z_at = np.take_along_axis(z, g_gpu[..., None], axis=-1)[..., 0]
    assert (z_at >= zmax - 2 * LOGIT_ABS).all()
    top2 = np.sort(z, axis=-1)[..., -2:]
    clear = top2[..., 1] - top2[..., 0] > 2 * LOGIT_ABS
    np.testing.assert_array_equal(g_gpu[clear], g_ora[clear])


def _without_near_ties(hidden, lm, z, seed):
    """Redraw, from N(0, 1), the hidden state of every tree node whose oracle
    top-2 logit gap is at most twice the logit tolerance, until no such node
    is left (a planted node's top token stands about 8 above the rest, so
    only unplanted nodes are redrawn).  The argmax of every row is then
    unambiguous at the kernel's fp32 accuracy, and the acceptance from the
    hidden states can be compared with the oracle's unconditionally.
    Returns the new hidden states and their oracle logits."""
    gen = torch.Generator().manual_seed(104729 + seed)
    hidden = hidden.clone()
    z = z.copy()
    lmd = f64(lm)
    d = hidden.shape[-1]
    for _ in range(20):
        top2 = np.sort(z, axis=-1)[..., -2:]
        bad = np.argwhere(top2[..., 1] - top2[..., 0] <= 2 * LOGIT_ABS)
        if len(bad) == 0:
            return hidden, z
        for b, i in bad:
            hidden[b, i] = torch.randn(d, generator=gen).to(hidden.dtype)
            z[b, i] = O.lm_head_logits(f64(hidden[b, i])[None], lmd)[0]
    raise AssertionError("rows with a near-tie argmax remain after 20 redraws")


@pytest.mark.parametrize("B,n_nodes,V,d,seed", [
    (2, 64, 3000, 1024, 0),     # 128 columns: one MMA half, ragged last vocabulary tile
    (5, 64, 2600, 512, 1),      # 320 columns: both halves, the second one ragged
    (9, 64, 1000, 256, 2),      # 576 columns: two column blocks
    (1, 9, 129, 64, 3),         # tiny: 9 columns, two vocabulary tiles, d = 64
])
def test_logits_and_greedy_decisions(B, n_nodes, V, d, seed):
    base = W.WORKLOADS["llama3_8b"] if n_nodes == 64 else W.WORKLOADS["tiny"]
    w = W.scaled(base, B=B, V=V, d=d)
    spec = W.tree_for(w)
    cand = _cands(w, spec, seed)
    hidden, lm = W.lmhead_inputs(w, spec, torch.from_numpy(cand), seed=seed)
    hidden, z = _without_near_ties(hidden, lm, _oracle_logits(hidden, lm), seed)
    got = _run(hidden, lm, cand, spec, M.MEDUSA_ACCEPT_GREEDY, want_logits=True)
    _check_logits(got, z)
    # acceptance: bit-exact on the kernel's own logits ...
    ref = O.verify_greedy(got["logits"], cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref)
    # ... and equal to the oracle's from the hidden states (every argmax is
    # unambiguous after the redraw)
    ref2 = O.lmhead_verify(f64(hidden), f64(lm), cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref2)


@pytest.mark.parametrize("B,V,d,seed", [(2, 4000, 512, 4), (3, 1300, 1024, 5)])
def test_typical_decisions(B, V, d, seed):
    w = W.scaled(W.WORKLOADS["llama3_70b"], B=B, V=V, d=d, accept="typical", temperature=0.7,
                 eps=0.09, delta=0.3)
    spec = W.tree_for(w)
    cand = _cands(w, spec, seed)
    for attempt in range(20):
        hidden, lm = W.lmhead_inputs(w, spec, torch.from_numpy(cand), seed=seed, attempt=attempt,
                                     plant=4.0)
        hidden, z = _without_near_ties(hidden, lm, _oracle_logits(hidden, lm), seed + attempt)
        m = O.typical_log_margin(z, cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            break
    else:
        pytest.skip("no margin-clean draw")
    got = _run(hidden, lm, cand, spec, M.MEDUSA_ACCEPT_TYPICAL, w.temperature, w.eps, w.delta,
               want_logits=True)
    _check_logits(got, z)
    ref = O.verify_typical(got["logits"], cand, spec.parent, spec.depth, spec.max_depth,
                           w.temperature, w.eps, w.delta)
    _assert_same(got, ref)
    ref2 = O.lmhead_verify(f64(hidden), f64(lm), cand, spec.parent, spec.depth, spec.max_depth,
                           "typical", w.temperature, w.eps, w.delta)
    _assert_same(got, ref2)
    assert 0 < ref["accept_len"].sum()


def test_same_result_as_verify_on_materialised_logits():
    """Greedy on the GPU's own fp32 logits through medusa_verify_accept gives
    the same outputs as the fused call."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=3, V=5000, d=1024)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 6)
    hidden, lm = W.lmhead_inputs(w, spec, torch.from_numpy(cand), seed=6)
    got = _run(hidden, lm, cand, spec, M.MEDUSA_ACCEPT_GREEDY, want_logits=True)
    dev = "cuda"
    tree = M.Tree.from_spec(spec)
    Wd = spec.max_depth + 1
    outs = [torch.zeros(w.B, dtype=torch.int32, device=dev),
            torch.zeros(w.B, Wd, dtype=torch.int32, device=dev),
            torch.zeros(w.B, Wd, dtype=torch.int32, device=dev),
            torch.zeros(w.B, dtype=torch.int32, device=dev)]
    st = M.new_status()
    M.medusa_verify_accept(torch.from_numpy(got["logits"]).float().to(dev),
                           torch.from_numpy(cand).to(dev), tree, *outs, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k, t in zip(("accept_len", "accepted_nodes", "accepted_tokens", "bonus"), outs):
        np.testing.assert_array_equal(t.cpu().numpy(), got[k], err_msg=k)


def test_rejects_bad_arguments():
    w = W.scaled(W.WORKLOADS["tiny"], B=1, V=100, d=96)
    spec = W.tree_for(w)
    dev = "cuda"
    hidden = torch.zeros(1, spec.n_nodes, 96, dtype=torch.bfloat16, device=dev)
    lm = torch.zeros(100, 96, dtype=torch.bfloat16, device=dev)
    cand = torch.zeros(1, spec.n_nodes, dtype=torch.int32, device=dev)
    outs = [torch.zeros(1, dtype=torch.int32, device=dev),
            torch.zeros(1, spec.max_depth + 1, dtype=torch.int32, device=dev),
            torch.zeros(1, spec.max_depth + 1, dtype=torch.int32, device=dev),
            torch.zeros(1, dtype=torch.int32, device=dev)]
    tree = M.Tree.from_spec(spec)
    with pytest.raises(M.MedusaError) as e:  # d not a multiple of 64
        M.medusa_lmhead_verify(hidden, lm, cand, tree, *outs,
                               ws=M.workspace(1 << 16, dev))
    assert e.value.status == 2
    with pytest.raises(M.MedusaError) as e:  # fp32 inputs
        M.medusa_lmhead_verify(hidden[..., :64].float().contiguous(),
                               lm[:, :64].float().contiguous(), cand, tree, *outs,
                               ws=M.workspace(1 << 16, dev))
    assert e.value.status == 3


@pytest.mark.slow
def test_full_size_greedy_llama3_8b():
    """B 8 x 64 nodes, V 128256, d 4096: decisions against the oracle (fp64
    logits computed in vocabulary chunks), plus sampled rows of the logits."""
    w = W.WORKLOADS["llama3_8b"]
    spec = W.tree_for(w)
    cand = _cands(w, spec, 0)
    hidden, lm = W.lmhead_inputs(w, spec, torch.from_numpy(cand), seed=0, device="cuda")
    h = f64(hidden.cpu()).reshape(-1, w.d)
    z = np.empty((h.shape[0], w.V))
    for v0 in range(0, w.V, 8192):
        z[:, v0:v0 + 8192] = O.lm_head_logits(h, f64(lm[v0:v0 + 8192].cpu()))
    z = z.reshape(w.B, spec.n_nodes, w.V)
    hidden, z = _without_near_ties(hidden.cpu(), lm.cpu(), z, 0)
    got = _run(hidden, lm, cand, spec, M.MEDUSA_ACCEPT_GREEDY, want_logits=True)
    _check_logits(got, z)
    ref = O.verify_greedy(got["logits"], cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref)
    ref2 = O.verify_greedy(z, cand, spec.parent, spec.depth, spec.max_depth)
    _assert_same(got, ref2)
