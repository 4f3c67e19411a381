"""GPU parity: medusa_tree_build and medusa_kv_compact (bit-exact)."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import i64

pytestmark = pytest.mark.gpu


def _build(spec, root, topk_ids, prefix):
    dev = "cuda"
    tree = M.Tree.from_spec(spec)
    B, N = root.shape[0], spec.n_nodes
    out = dict(
        cand=torch.full((B, N), -5, dtype=torch.int32, device=dev),
        pos=torch.full((B, N), -5, dtype=torch.int32, device=dev),
        mask=torch.full((N, (N + 31) // 32), -5, dtype=torch.int32, device=dev),
        retrieve=torch.full((spec.n_leaves, spec.max_depth + 1), -5, dtype=torch.int32, device=dev),
    )
    status = M.new_status()
    M.medusa_tree_build(tree, root.to(dev), topk_ids.to(dev), prefix.to(dev), out["cand"],
                        out["pos"], out["mask"], out["retrieve"], status)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}, int(status.item())


@pytest.mark.parametrize("name,n_nodes", [("tiny", None), ("vicuna7b", None), ("llama3_8b", None),
                                          ("llama3_70b", None), ("long", 16), ("long", 128)])
def test_tree_build_bit_exact(name, n_nodes):
    w = W.WORKLOADS[name]
    spec = W.tree_for(w, n_nodes=n_nodes)
    root = W.random_root_tokens(w, seed=1)
    topk_ids = W.random_topk_ids(w, seed=1)
    prefix = W.prefix_lengths(w, seed=1)
    got, st = _build(spec, root, topk_ids, prefix)
    assert st == 0
    ref = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk_ids), i64(prefix))
    np.testing.assert_array_equal(got["cand"], ref["cand"])
    np.testing.assert_array_equal(got["pos"], ref["pos"])
    np.testing.assert_array_equal(got["mask"].view(np.uint32), ref["mask"])
    np.testing.assert_array_equal(got["retrieve"], ref["retrieve"])


def test_tree_build_rejects_a_malformed_tree_on_device():
    """A parent index that does not precede its child is caught by the
    kernel's own checks: status MEDUSA_ERR_DEVICE_CHECK, no write outside the
    outputs."""
    spec = W.cartesian_tree([2, 3])
    bad = W.TreeSpec(spec.parent.copy(), spec.depth.copy(), spec.rank.copy(), spec.paths)
    bad.parent[3] = 5
    w = W.WORKLOADS["tiny"]
    got, st = _build(bad, W.random_root_tokens(w), W.random_topk_ids(w), W.prefix_lengths(w))
    assert st == 6
    assert (got["cand"] == -1).all()


def _compact_case(seed, B=3, Hkv=2, dh=128, dtype=torch.bfloat16, max_depth=4, N=40):
    rng = np.random.default_rng(seed)
    cap = 300
    prefix = rng.integers(0, cap - N, size=B).astype(np.int32)
    Kc = torch.randn(B, Hkv, cap, dh, generator=torch.Generator().manual_seed(seed)).to(dtype)
    Vc = torch.randn(B, Hkv, cap, dh, generator=torch.Generator().manual_seed(seed + 1)).to(dtype)
    L = rng.integers(0, max_depth + 1, size=B).astype(np.int32)
    nodes = np.full((B, max_depth + 1), -1, dtype=np.int32)
    for b in range(B):
        # strictly increasing node ids with node[j] >= j, as a BFS path gives
        chain = [0] + sorted(rng.choice(np.arange(1, N), size=int(L[b]), replace=False).tolist())
        nodes[b, :L[b] + 1] = chain
    return Kc, Vc, prefix, nodes, L, max_depth


@pytest.mark.parametrize("seed,dtype,dh,Hkv,max_depth", [
    (0, torch.bfloat16, 128, 2, 4), (1, torch.bfloat16, 64, 2, 4), (2, torch.float32, 64, 2, 4),
    (3, torch.bfloat16, 128, 2, 4),
    (4, torch.bfloat16, 128, 32, 5),   # 32 kv heads staged in one round
    (5, torch.float32, 256, 16, 5),    # 12 KB per head: two rounds of 8 heads
])
def test_kv_compact_bit_exact(seed, dtype, dh, Hkv, max_depth):
    Kc, Vc, prefix, nodes, L, max_depth = _compact_case(seed, dtype=dtype, dh=dh, Hkv=Hkv,
                                                        max_depth=max_depth)
    if seed == 3:  # overlapping chains: every destination is another step's source
        nodes[:] = -1
        for b in range(nodes.shape[0]):
            L[b] = max_depth
            nodes[b] = [0, 1, 2, 3, 4][: max_depth + 1]
            nodes[b, 1:] = [2, 3, 4, 5][:max_depth]
    ref = O.kv_compact(Kc.float().numpy(), Vc.float().numpy(), prefix, nodes, L)
    dev = "cuda"
    Kg, Vg = Kc.to(dev), Vc.to(dev)
    pl = torch.from_numpy(prefix).to(dev)
    src = torch.full(nodes.shape, -9, dtype=torch.int32, device=dev)
    status = M.new_status()
    M.medusa_kv_compact(Kg, Vg, pl, torch.from_numpy(nodes).to(dev), torch.from_numpy(L).to(dev),
                        src, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(Kg.float().cpu().numpy(), ref["Kc"])
    np.testing.assert_array_equal(Vg.float().cpu().numpy(), ref["Vc"])
    np.testing.assert_array_equal(pl.cpu().numpy(), ref["prefix_len"])
    np.testing.assert_array_equal(src.cpu().numpy(), ref["compact_src"])


def test_kv_compact_rejects_out_of_range_path():
    Kc, Vc, prefix, nodes, L, max_depth = _compact_case(5)
    L[0] = max_depth + 3  # longer than the path arrays
    dev = "cuda"
    Kg = Kc.to(dev)
    before = Kg.clone()
    pl = torch.from_numpy(prefix).to(dev)
    status = M.new_status()
    M.medusa_kv_compact(Kg, Vc.to(dev), pl, torch.from_numpy(nodes).to(dev),
                        torch.from_numpy(L).to(dev), torch.empty(nodes.shape, dtype=torch.int32,
                                                                 device=dev), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6
    assert torch.equal(Kg[0], before[0]) and int(pl[0].item()) == prefix[0]


def test_tree_build_at_the_limits():
    """MAX_NODES nodes, a depth of K = MAX_HEADS, ranks up to MAX_KMAX - 1 and
    MAX_BATCH sequences: bit-exact."""
    spec = W.limits_tree(M.MAX_NODES, M.MAX_HEADS, M.MAX_KMAX)
    assert spec.max_depth == M.MAX_HEADS and spec.rank.max() == M.MAX_KMAX - 1
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=M.MAX_BATCH, K=M.MAX_HEADS, kmax=M.MAX_KMAX,
                 N=spec.n_nodes)
    root = W.random_root_tokens(w, seed=9)
    topk_ids = W.random_topk_ids(w, seed=9)
    prefix = W.prefix_lengths(w, seed=9)
    got, st = _build(spec, root, topk_ids, prefix)
    assert st == 0
    ref = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk_ids), i64(prefix))
    for k in ("cand", "pos", "retrieve"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    np.testing.assert_array_equal(got["mask"].view(np.uint32), ref["mask"])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_kv_compact_deepest_path(dtype):
    """max_depth = MAX_HEADS - 1, the deepest path compaction takes: every
    sequence keeps a full-length path, some of them the first nodes (sources
    that are other steps' destinations)."""
    max_depth = M.MAX_HEADS - 1
    B, Hkv, dh, N, cap = 4, 8, 128, 256, 700
    rng = np.random.default_rng(21)
    prefix = rng.integers(0, cap - N, size=B).astype(np.int32)
    g = torch.Generator().manual_seed(21)
    Kc = torch.randn(B, Hkv, cap, dh, generator=g).to(dtype)
    Vc = torch.randn(B, Hkv, cap, dh, generator=g).to(dtype)
    L = np.full(B, max_depth, dtype=np.int32)
    nodes = np.zeros((B, max_depth + 1), dtype=np.int32)
    for b in range(B):
        if b % 2:
            nodes[b] = np.arange(max_depth + 1)  # node j at slot P + j: stays in place
            nodes[b, 1:] += 1                    # shifted by one: overlapping chain
        else:
            nodes[b, 1:] = np.sort(rng.choice(np.arange(1, N), size=max_depth, replace=False))
    ref = O.kv_compact(Kc.float().numpy(), Vc.float().numpy(), prefix, nodes, L)
    dev = "cuda"
    Kg, Vg = Kc.to(dev), Vc.to(dev)
    pl = torch.from_numpy(prefix).to(dev)
    src = torch.full(nodes.shape, -9, dtype=torch.int32, device=dev)
    status = M.new_status()
    M.medusa_kv_compact(Kg, Vg, pl, torch.from_numpy(nodes).to(dev), torch.from_numpy(L).to(dev),
                        src, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(Kg.float().cpu().numpy(), ref["Kc"])
    np.testing.assert_array_equal(Vg.float().cpu().numpy(), ref["Vc"])
    np.testing.assert_array_equal(pl.cpu().numpy(), ref["prefix_len"])
    np.testing.assert_array_equal(src.cpu().numpy(), ref["compact_src"])
