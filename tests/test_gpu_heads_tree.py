"""GPU parity: medusa_heads_topk_tree, the heads' top-k and the tree build in
the heads' launches.  The top-k outputs must equal medusa_heads_topk's bit for
bit (and pass the oracle's top-k check), and the tree outputs must equal the
oracle's tree build from those lists, bit for bit."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import check_topk, f64, i64

pytestmark = pytest.mark.gpu


def _fused(inp, kmax, spec, root, prefix):
    dev = "cuda"
    h, W1, b1, W2 = (inp[k].to(dev) for k in ("h", "W1", "b1", "W2"))
    B, K = h.shape[0], W2.shape[0]
    N = spec.n_nodes
    tree = M.Tree.from_spec(spec, dev)
    o = dict(
        ids=torch.full((B, K, kmax), -7, dtype=torch.int32, device=dev),
        vals=torch.full((B, K, kmax), float("nan"), dtype=torch.float32, device=dev),
        cand=torch.full((B, N), -5, dtype=torch.int32, device=dev),
        pos=torch.full((B, N), -5, dtype=torch.int32, device=dev),
        mask=torch.full((N, (N + 31) // 32), -5, dtype=torch.int32, device=dev),
        retrieve=torch.full((spec.n_leaves, spec.max_depth + 1), -5, dtype=torch.int32,
                            device=dev),
    )
    st = M.new_status()
    M.medusa_heads_topk_tree(h, W1, b1, W2, kmax, o["ids"], o["vals"], tree, root.to(dev),
                             prefix.to(dev), o["cand"], o["pos"], o["mask"], o["retrieve"],
                             dev_status=st)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}, int(st.item())


def _heads_alone(inp, kmax):
    dev = "cuda"
    h, W1, b1, W2 = (inp[k].to(dev) for k in ("h", "W1", "b1", "W2"))
    B, K = h.shape[0], W2.shape[0]
    ids = torch.full((B, K, kmax), -7, dtype=torch.int32, device=dev)
    vals = torch.full((B, K, kmax), float("nan"), dtype=torch.float32, device=dev)
    st = M.new_status()
    M.medusa_heads_topk(h, W1, b1, W2, kmax, ids, vals, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return ids.cpu().numpy(), vals.cpu().numpy()


def _check(got, spec, root, prefix):
    ref = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), got["ids"].astype(np.int64),
                       i64(prefix))
    np.testing.assert_array_equal(got["cand"], ref["cand"], err_msg="cand")
    np.testing.assert_array_equal(got["pos"], ref["pos"], err_msg="pos")
    np.testing.assert_array_equal(got["retrieve"], ref["retrieve"], err_msg="retrieve")
    np.testing.assert_array_equal(got["mask"].view(np.uint32), ref["mask"], err_msg="mask")


@pytest.mark.parametrize("name,over,n_nodes", [
    ("tiny", {}, None),                                   # fp32 CUDA-core heads
    ("vicuna7b", dict(d=512, V=3000), None),              # one sequence, 64-node tree
    ("llama3_8b", dict(d=1024, V=20001), None),           # 8 sequences, ragged vocabulary
    ("llama3_70b", dict(B=4, d=512, V=5000), None),       # 256-node dense tree
    ("long", dict(B=32, d=256, V=3000), 128),             # 32 sequences, 64-wide MMA
])
def test_matches_heads_and_oracle_tree(name, over, n_nodes):
    w = W.scaled(W.WORKLOADS[name], **over)
    spec = W.tree_for(w, n_nodes=n_nodes)
    inp = W.heads_inputs(w, seed=3)
    root = W.random_root_tokens(w, seed=3)
    prefix = W.prefix_lengths(w, seed=3)
    got, st = _fused(inp, w.kmax, spec, root, prefix)
    assert st == 0
    ids, vals = _heads_alone(inp, w.kmax)
    np.testing.assert_array_equal(got["ids"], ids)
    np.testing.assert_array_equal(got["vals"], vals)
    z = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    check_topk(got["ids"], got["vals"], z, w.kmax)
    _check(got, spec, root, prefix)


def test_at_the_limits():
    """MAX_BATCH sequences, MAX_HEADS heads, MAX_KMAX wide lists and a
    MAX_NODES-node tree of depth MAX_HEADS using every rank."""
    spec = W.limits_tree(M.MAX_NODES, M.MAX_HEADS, M.MAX_KMAX)
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=M.MAX_BATCH, d=128, V=700, K=M.MAX_HEADS,
                 kmax=M.MAX_KMAX, N=spec.n_nodes)
    inp = W.heads_inputs(w, seed=5)
    root = W.random_root_tokens(w, seed=5)
    prefix = torch.randint(0, 5000, (w.B,), generator=torch.Generator().manual_seed(5),
                           dtype=torch.int32)
    got, st = _fused(inp, w.kmax, spec, root, prefix)
    assert st == 0
    ids, vals = _heads_alone(inp, w.kmax)
    np.testing.assert_array_equal(got["ids"], ids)
    _check(got, spec, root, prefix)


def test_malformed_tree_reported():
    """A rank past kmax: the device check reports MEDUSA_ERR_DEVICE_CHECK and
    every candidate id is -1, as medusa_tree_build does; the top-k lists are
    still written."""
    w = W.scaled(W.WORKLOADS["vicuna7b"], B=2, d=256, V=2000, K=2, kmax=3)
    spec = W.cartesian_tree([2, 3])
    bad = W.TreeSpec(spec.parent.copy(), spec.depth.copy(), spec.rank.copy(), spec.paths)
    bad.rank[4] = 3
    inp = W.heads_inputs(w, seed=7)
    got, st = _fused(inp, w.kmax, bad, W.random_root_tokens(w, seed=7), W.prefix_lengths(w, 7))
    assert st == 6
    assert (got["cand"] == -1).all()
    ids, _ = _heads_alone(inp, w.kmax)
    np.testing.assert_array_equal(got["ids"], ids)


def test_full_size_llama3_8b():
    """The configuration the benchmark times: d 4096, V 128256, 8 sequences,
    4 heads, the 64-node tree (the heads alone are checked against the oracle
    at this size in test_gpu_heads.py)."""
    w = W.WORKLOADS["llama3_8b"]
    spec = W.tree_for(w)
    inp = W.heads_inputs(w, seed=0, device="cuda")
    root = W.random_root_tokens(w, seed=0)
    prefix = W.prefix_lengths(w, seed=0)
    got, st = _fused(inp, w.kmax, spec, root, prefix)
    assert st == 0
    ids, vals = _heads_alone(inp, w.kmax)
    np.testing.assert_array_equal(got["ids"], ids)
    np.testing.assert_array_equal(got["vals"], vals)
    _check(got, spec, root, prefix)
