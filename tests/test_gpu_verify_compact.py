"""GPU parity: medusa_verify_accept_compact, the verification and the KV
compaction in the verification's launches.  Every output (the four
verification outputs, both caches, prefix_len, compact_src) is compared with
the oracle's verification followed by the oracle's compaction, bit for bit,
and with the two separate calls."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import TYPICAL_LOG_MARGIN, f64, i64

pytestmark = pytest.mark.gpu

FIELDS = ("accept_len", "accepted_nodes", "accepted_tokens", "bonus")


def _cands(w, spec, seed):
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk),
                      np.zeros(w.B, np.int64))
    return tb["cand"]


def _caches(B, Hkv, dh, cap, N, dtype, seed):
    rng = np.random.default_rng(seed)
    prefix = rng.integers(0, cap - N + 1, size=B).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    Kc = torch.randn(B, Hkv, cap, dh, generator=g).to(dtype)
    Vc = torch.randn(B, Hkv, cap, dh, generator=g).to(dtype)
    return Kc, Vc, prefix


def _fused(logits, cand, spec, Kc, Vc, prefix, mode, T, eps, delta):
    dev = "cuda"
    tree = M.Tree.from_spec(spec, dev)
    B, Wd = cand.shape[0], spec.max_depth + 1
    out = {k: torch.full(s, -9, dtype=torch.int32, device=dev) for k, s in
           (("accept_len", (B,)), ("accepted_nodes", (B, Wd)), ("accepted_tokens", (B, Wd)),
            ("bonus", (B,)), ("compact_src", (B, Wd)))}
    Kg, Vg = Kc.to(dev), Vc.to(dev)
    pl = torch.from_numpy(prefix).to(dev)
    st = M.new_status()
    M.medusa_verify_accept_compact(logits.to(dev), torch.from_numpy(cand).to(dev), tree,
                                   out["accept_len"], out["accepted_nodes"],
                                   out["accepted_tokens"], out["bonus"], Kg, Vg, pl,
                                   out["compact_src"], mode, T, eps, delta, dev_status=st)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res.update(Kc=Kg.float().cpu().numpy(), Vc=Vg.float().cpu().numpy(),
               prefix_len=pl.cpu().numpy())
    return res, int(st.item())


def _separate(logits, cand, spec, Kc, Vc, prefix, mode, T, eps, delta):
    dev = "cuda"
    tree = M.Tree.from_spec(spec, dev)
    B, Wd = cand.shape[0], spec.max_depth + 1
    out = {k: torch.full(s, -9, dtype=torch.int32, device=dev) for k, s in
           (("accept_len", (B,)), ("accepted_nodes", (B, Wd)), ("accepted_tokens", (B, Wd)),
            ("bonus", (B,)), ("compact_src", (B, Wd)))}
    Kg, Vg = Kc.to(dev), Vc.to(dev)
    pl = torch.from_numpy(prefix).to(dev)
    st = M.new_status()
    M.medusa_verify_accept(logits.to(dev), torch.from_numpy(cand).to(dev), tree,
                           out["accept_len"], out["accepted_nodes"], out["accepted_tokens"],
                           out["bonus"], mode, T, eps, delta, dev_status=st)
    M.medusa_kv_compact(Kg, Vg, pl, out["accepted_nodes"], out["accept_len"],
                        out["compact_src"], st)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res.update(Kc=Kg.float().cpu().numpy(), Vc=Vg.float().cpu().numpy(),
               prefix_len=pl.cpu().numpy())
    return res, int(st.item())


def _oracle(logits, cand, spec, Kc, Vc, prefix, typical, T, eps, delta):
    if typical:
        ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                               T, eps, delta)
    else:
        ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
    kv = O.kv_compact(Kc.float().numpy(), Vc.float().numpy(), prefix,
                      ref["accepted_nodes"].astype(np.int32), ref["accept_len"].astype(np.int32))
    out = {k: ref[k] for k in FIELDS}
    out.update(kv)
    return out


def _assert_equal(got, ref, what):
    for k in FIELDS + ("Kc", "Vc", "prefix_len", "compact_src"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=f"{what}: {k}")


@pytest.mark.parametrize("name,over,seed,n_nodes,kv_dtype,Hkv,dh", [
    # the Llama-3-8B-shaped step: full vocabulary, 8 kv heads of 128
    ("llama3_8b", dict(B=8), 0, None, torch.bfloat16, 8, 128),
    ("tiny", dict(B=4), 1, None, torch.float32, 2, 64),
    ("vicuna7b", dict(B=3, V=5000), 8, None, torch.bfloat16, 32, 128),
    # 128-node tree, f32 caches of dh 256: two staging rounds of K and V
    ("long", dict(B=4, V=20001), 8, 128, torch.float32, 16, 256),
])
def test_greedy_with_compaction(name, over, seed, n_nodes, kv_dtype, Hkv, dh):
    w = W.scaled(W.WORKLOADS[name], **over)
    spec = W.tree_for(w, n_nodes=n_nodes)
    cand = _cands(w, spec, seed)
    dev = "cuda" if w.B * spec.n_nodes * w.V > (1 << 27) else "cpu"
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=seed, device=dev).cpu()
    Kc, Vc, prefix = _caches(w.B, Hkv, dh, spec.n_nodes + 200, spec.n_nodes, kv_dtype, seed)
    args = (logits, cand, spec, Kc, Vc, prefix)
    ref = _oracle(*args, False, 1.0, 0.09, 0.3)
    assert ref["accept_len"].max() > 0
    got, st = _fused(*args, M.MEDUSA_ACCEPT_GREEDY, 1.0, 0.09, 0.3)
    assert st == 0
    _assert_equal(got, ref, "fused vs oracle")
    sep, st = _separate(*args, M.MEDUSA_ACCEPT_GREEDY, 1.0, 0.09, 0.3)
    assert st == 0
    _assert_equal(got, sep, "fused vs separate calls")


def test_typical_with_compaction():
    w = W.scaled(W.WORKLOADS["llama3_70b"], B=2, V=9000, accept="typical", temperature=0.7,
                 eps=0.09, delta=0.3)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 4)
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=4, attempt=attempt)
        m = O.typical_log_margin(f64(logits), cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            break
    else:
        raise AssertionError("no margin-clean typical draw")
    Kc, Vc, prefix = _caches(w.B, 8, 128, 400, spec.n_nodes, torch.bfloat16, 4)
    args = (logits, cand, spec, Kc, Vc, prefix)
    ref = _oracle(*args, True, w.temperature, w.eps, w.delta)
    got, st = _fused(*args, M.MEDUSA_ACCEPT_TYPICAL, w.temperature, w.eps, w.delta)
    assert st == 0
    _assert_equal(got, ref, "fused vs oracle")


def test_chain_tree_overlapping_moves():
    """Two branches under the root, the second a chain.  Sequence 0 keeps
    node 1, already at its own slot; sequence 1 keeps the chain 0, 2, 3, 4, 5,
    each row moving down one slot (every destination is the next move's
    source)."""
    # node 1 and node 2 both children of the root; 3.. a chain under node 2
    parent = np.array([-1, 0, 0, 2, 3, 4], np.int32)
    depth = np.array([0, 1, 1, 2, 3, 4], np.int32)
    rank = np.array([0, 0, 1, 0, 0, 0], np.int32)
    spec = W.TreeSpec(parent, depth, rank, None)
    cand = np.array([[5, 6, 7, 8, 9, 10], [5, 6, 7, 8, 9, 10]], np.int32)
    logits = torch.full((2, 6, 1000), -1.0)
    # b = 0: argmax at the root is node 1's token, then nothing below it
    logits[0, 0, 6] = 4.0
    logits[0, 1, 3] = 4.0
    # b = 1: the chain 0 -> 2 -> 3 -> 4 -> 5 accepted, bonus 11
    for i, t in ((0, 7), (2, 8), (3, 9), (4, 10), (5, 11)):
        logits[1, i, t] = 4.0
    Kc, Vc, prefix = _caches(2, 4, 128, 40, 6, torch.bfloat16, 8)
    args = (logits, cand, spec, Kc, Vc, prefix)
    ref = _oracle(*args, False, 1.0, 0.09, 0.3)
    assert list(ref["accept_len"]) == [1, 4]
    got, st = _fused(*args, M.MEDUSA_ACCEPT_GREEDY, 1.0, 0.09, 0.3)
    assert st == 0
    _assert_equal(got, ref, "fused vs oracle")


def test_slot_beyond_capacity_is_reported_and_left():
    """A sequence whose kept node would read past the cache capacity: status
    MEDUSA_ERR_DEVICE_CHECK, its cache rows and prefix unchanged; the other
    sequences compacted as the oracle does."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=3, V=4000)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 6)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=6)
    cap = spec.n_nodes + 50
    Kc, Vc, prefix = _caches(w.B, 2, 128, cap, spec.n_nodes, torch.bfloat16, 6)
    ref = _oracle(logits, cand, spec, Kc, Vc, prefix, False, 1.0, 0.09, 0.3)
    best = [int(ref["accepted_nodes"][b, ref["accept_len"][b]]) for b in range(w.B)]
    bad = int(np.argmax(best))
    assert best[bad] > 0
    prefix_bad = prefix.copy()
    prefix_bad[bad] = cap - best[bad]          # slot P + best = cap
    got, st = _fused(logits, cand, spec, Kc, Vc, prefix_bad, M.MEDUSA_ACCEPT_GREEDY, 1.0, 0.09,
                     0.3)
    assert st == 6
    for k in FIELDS:                            # the verification itself is unaffected
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    assert got["prefix_len"][bad] == prefix_bad[bad]
    np.testing.assert_array_equal(got["Kc"][bad], Kc[bad].float().numpy())
    np.testing.assert_array_equal(got["Vc"][bad], Vc[bad].float().numpy())
    ok = [b for b in range(w.B) if b != bad]
    for k in ("Kc", "Vc", "prefix_len", "compact_src"):
        np.testing.assert_array_equal(got[k][ok], ref[k][ok], err_msg=k)
