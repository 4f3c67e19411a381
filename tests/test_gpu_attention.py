"""GPU parity: medusa_tree_attention against the oracle."""
import math

import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import ATTN_REL_L2, LOGIT_MAX_ABS, f64, i64, rel_l2

pytestmark = pytest.mark.gpu


def _mask(spec, B):
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, np.zeros(B, np.int64),
                      np.zeros((B, max(1, spec.max_depth), 32), np.int64), np.zeros(B, np.int64))
    return tb["mask"]


def _run_gpu(inp, mask, max_prefix, out_dtype):
    dev = "cuda"
    q, kn, vn, Kc, Vc = (inp[k].to(dev) for k in ("q", "k_new", "v_new", "Kc", "Vc"))
    pl = inp["prefix_len"].to(dev)
    B, N, Hq, dh = q.shape
    out = torch.full((B, N, Hq, dh), float("nan"), dtype=out_dtype, device=dev)
    m = torch.from_numpy(mask.view(np.int32).copy()).to(dev)
    status = M.new_status()
    M.medusa_tree_attention(q, kn, vn, Kc, Vc, pl, m, max_prefix, out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return f64(out), Kc.cpu(), Vc.cpu()


def _compare(inp, spec, max_prefix, out_dtype=torch.float32, rows=None):
    mask = _mask(spec, inp["q"].shape[0])
    got, Kg, Vg = _run_gpu(inp, mask, max_prefix, out_dtype)
    dh = inp["q"].shape[-1]
    P = i64(inp["prefix_len"])
    if rows is None:
        ref = O.tree_attention(f64(inp["q"]), f64(inp["k_new"]), f64(inp["v_new"]), f64(inp["Kc"]),
                               f64(inp["Vc"]), P, mask, 1.0 / math.sqrt(dh))
        out_ref, Kr, Vr = ref["out"], ref["Kc"], ref["Vc"]
        g = got
    else:  # sampled (sequence, node) rows, all heads, the oracle one row at a time
        out_ref = np.stack([_oracle_row(inp, mask, b, i, P[b], dh) for b, i in rows])
        g = np.stack([got[b, i] for b, i in rows])
        Kr = Vr = None
    err = np.abs(g - out_ref).max()
    assert err < LOGIT_MAX_ABS, err
    if out_dtype == torch.float32:
        assert rel_l2(g, out_ref) < ATTN_REL_L2, rel_l2(g, out_ref)
    else:  # bf16 output adds its own rounding (relative 2^-9)
        assert rel_l2(g, out_ref) < 4e-3
    if Kr is not None:  # the tree K/V landed in their cache slots, bit for bit
        np.testing.assert_array_equal(Kg.double().numpy(), Kr)
        np.testing.assert_array_equal(Vg.double().numpy(), Vr)


def _oracle_row(inp, mask, b, i, P, dh):
    """Oracle tree attention for node i of sequence b only (all query heads):
    the oracle is run on a one-node query whose mask row is node i's."""
    N = inp["q"].shape[1]
    # the oracle is given only node i's visible tree nodes (ancestors and
    # itself, in node order) as its tree, every one of them visible
    vis = [j for j in range(N) if O.mask_bit(mask, i, j)]
    kn = f64(inp["k_new"][b:b + 1, vis])
    vn = f64(inp["v_new"][b:b + 1, vis])
    nvis = len(vis)
    mm = np.zeros((nvis, (nvis + 31) // 32), dtype=np.uint32)
    for r in range(nvis):
        for j in range(nvis):
            mm[r, j // 32] |= np.uint32(1 << (j % 32))
    q = np.repeat(f64(inp["q"][b:b + 1, i:i + 1]), nvis, axis=1)
    res = O.tree_attention(q, kn, vn, f64(inp["Kc"][b:b + 1]), f64(inp["Vc"][b:b + 1]),
                           np.array([P]), mm, 1.0 / math.sqrt(dh))
    return res["out"][0, 0]


def test_tiny_fp32():
    w = W.WORKLOADS["tiny"]
    spec = W.tree_for(w)
    inp = W.attention_inputs(w, seed=0)
    _compare(inp, spec, w.ctx_hi)


@pytest.mark.parametrize("B,Hq,Hkv,dh,ctx,tree,seed", [
    (2, 8, 2, 128, (100, 700), "sparse64", 0),     # ragged, split boundaries, GQA 4
    (1, 4, 4, 64, (64, 64), "cart23", 1),          # dh 64, prefix = one tile
    (3, 8, 1, 128, (1, 200), "sparse16", 2),       # MQA, tiny prefixes
    (2, 16, 2, 128, (0, 0), "sparse64", 3),        # empty prefix: tree only
    (1, 8, 8, 128, (1500, 1500), "dense256", 4),   # 256 nodes, 8 mask words
    (2, 6, 2, 128, (50, 300), "sparse16", 5),      # G 3: Q rows gathered by threads
    (1, 16, 1, 64, (200, 200), "sparse64", 6),     # G 16: four query groups of 256 rows
    (256, 2, 1, 64, (0, 40), "sparse16", 7),       # 256 sequences: the schedule table is full
])
def test_bf16_small(B, Hq, Hkv, dh, ctx, tree, seed):
    if tree == "sparse64":
        spec = W.sparse_tree(64, 4, 10, seed, max_depth=4)
    elif tree == "sparse16":
        spec = W.sparse_tree(16, 4, 10, seed, max_depth=4)
    elif tree == "dense256":
        spec = W.cartesian_tree([4, 4, 4, 4], n_nodes=256)
    else:
        spec = W.cartesian_tree([2, 3])
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=B, Hq=Hq, Hkv=Hkv, dh=dh, ctx_lo=ctx[0],
                 ctx_hi=ctx[1], N=spec.n_nodes)
    inp = W.attention_inputs(w, seed=seed)
    _compare(inp, spec, w.ctx_hi)
    _compare(W.attention_inputs(w, seed=seed), spec, w.ctx_hi, out_dtype=torch.bfloat16)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama3_8b", "llama3_70b", "long"])
def test_full_size_sampled_rows(name):
    # llama3_70b: 256-node dense tree (two tree tiles, 8 mask words), G = 8,
    # eight query groups of 256 rows; long: 32 sequences of 32768 cached keys
    w = W.WORKLOADS[name]
    spec = W.tree_for(w)
    inp = W.attention_inputs(w, seed=0)
    rng = np.random.default_rng(0)
    rows = [(int(rng.integers(w.B)), int(rng.integers(w.N))) for _ in range(24)]
    rows += [(0, 0), (w.B - 1, w.N - 1)]
    _compare(inp, spec, w.ctx_hi, rows=rows)


def _scaled_v(inp, b, factor, rows=None, tree=False):
    """V of sequence b (cache rows `rows`, or all; the tree's v_new too when
    `tree`) multiplied by `factor`, rounded to bf16 like any input."""
    out = dict(inp)
    Vc = inp["Vc"].float().clone()
    sl = slice(None) if rows is None else rows
    Vc[b, :, sl] *= factor
    out["Vc"] = Vc.to(inp["Vc"].dtype)
    if tree:
        vn = inp["v_new"].float().clone()
        vn[b] *= factor
        out["v_new"] = vn.to(inp["v_new"].dtype)
    return out


@pytest.mark.parametrize("case", ["large", "tiny", "mixed_tile", "large_tree"])
def test_bf16_v_outside_fp16_range(case):
    """V tiles that fp16 cannot carry (|v| up to about 4e6, or all |v| near
    1e-6) take the bf16 value product; per sequence the output must match the
    oracle to the usual relative bounds, whatever the magnitude."""
    spec = W.sparse_tree(64, 4, 10, 3, max_depth=4)
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=3, Hq=8, Hkv=2, dh=128, ctx_lo=300, ctx_hi=700,
                 N=spec.n_nodes)
    inp = W.attention_inputs(w, seed=11)
    if case == "large":
        inp = _scaled_v(inp, 0, 1e6)
    elif case == "tiny":
        inp = _scaled_v(inp, 1, 1e-6)
    elif case == "mixed_tile":  # a few rows of one tile large, the rest of it normal
        inp = _scaled_v(inp, 2, 3e5, rows=slice(130, 140))
    else:  # the tree's own values large too (the reload reads v_new)
        inp = _scaled_v(inp, 0, 1e6, tree=True)
    mask = _mask(spec, w.B)
    got, Kg, Vg = _run_gpu(inp, mask, w.ctx_hi, torch.float32)
    ref = O.tree_attention(f64(inp["q"]), f64(inp["k_new"]), f64(inp["v_new"]), f64(inp["Kc"]),
                           f64(inp["Vc"]), i64(inp["prefix_len"]), mask, 1.0 / math.sqrt(w.dh))
    for b in range(w.B):
        scale = np.abs(ref["out"][b]).max()
        assert np.abs(got[b] - ref["out"][b]).max() < LOGIT_MAX_ABS * scale, (case, b)
        assert rel_l2(got[b], ref["out"][b]) < ATTN_REL_L2, (case, b, rel_l2(got[b], ref["out"][b]))
    np.testing.assert_array_equal(Kg.double().numpy(), ref["Kc"])
    np.testing.assert_array_equal(Vg.double().numpy(), ref["Vc"])


def test_bf16_v_nan_is_reported():
    """Inf or NaN in V is a device-check error (status 6), not a fault."""
    spec = W.cartesian_tree([2, 3])
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=1, Hq=4, Hkv=1, dh=128, ctx_lo=200, ctx_hi=200,
                 N=spec.n_nodes)
    inp = W.attention_inputs(w, seed=12)
    Vc = inp["Vc"].clone()
    Vc[0, 0, 17, 5] = float("nan")
    inp["Vc"] = Vc
    dev = "cuda"
    mask = _mask(spec, 1)
    out = torch.empty(1, spec.n_nodes, 4, 128, dtype=torch.float32, device=dev)
    status = M.new_status()
    M.medusa_tree_attention(*(inp[k].to(dev) for k in ("q", "k_new", "v_new", "Kc", "Vc")),
                            inp["prefix_len"].to(dev),
                            torch.from_numpy(mask.view(np.int32).copy()).to(dev), w.ctx_hi, out,
                            dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6
