"""GPU: the next-step hand-off (medusa_next_step) against the oracle, and
decode steps chained on the device, eagerly and replayed from one CUDA graph."""
import math

import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from speculative_decoding_medusa_b200.step import DecodeLoop
from tests.helpers import f64

pytestmark = pytest.mark.gpu


def test_next_step_matches_oracle_and_checks_indices():
    dev = "cuda"
    spec = W.cartesian_tree([2, 3])
    B, N, d = 3, spec.n_nodes, 192
    g = torch.Generator().manual_seed(3)
    hidden = torch.randn(B, N, d, generator=g).to(torch.bfloat16)
    # kept branches: 0 -> 2 -> 7, root only, 0 -> 1
    nodes = np.array([[0, 2, 7], [0, -1, -1], [0, 1, -1]], dtype=np.int32)
    acc = np.array([2, 0, 1], dtype=np.int32)
    bonus = np.array([42, 9, 17], dtype=np.int32)
    h_ref, root_ref = O.next_step_inputs(f64(hidden), acc, nodes, bonus)
    h_next = torch.full((B, d), float("nan"), dtype=torch.bfloat16, device=dev)
    root_next = torch.full((B,), -1, dtype=torch.int32, device=dev)
    st = M.new_status()
    M.medusa_next_step(hidden.to(dev), torch.from_numpy(acc).to(dev),
                       torch.from_numpy(nodes).to(dev), torch.from_numpy(bonus).to(dev), h_next,
                       root_next, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(f64(h_next.cpu()), h_ref)  # a copy: bit for bit
    assert root_next.cpu().tolist() == root_ref.tolist()
    # a kept node outside the tree is reported, its sequence left untouched
    nodes[1, 0] = N
    h_next.fill_(0)
    M.medusa_next_step(hidden.to(dev), torch.from_numpy(acc).to(dev),
                       torch.from_numpy(nodes).to(dev), torch.from_numpy(bonus).to(dev), h_next,
                       root_next, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6
    assert float(h_next[1].abs().sum()) == 0.0


def _loop_setup(R, seed=0):
    base = W.WORKLOADS["llama3_8b"]
    w = W.scaled(base, B=2, d=512, V=3000, Hq=8, Hkv=2, ctx_lo=100, ctx_hi=300)
    spec = W.tree_for(w)
    dev = "cuda"
    tree = M.Tree.from_spec(spec, dev)
    heads = W.heads_inputs(w, seed=seed, device=dev)
    max_prefix = w.ctx_hi + R * (spec.max_depth + 1)
    cap = max_prefix + spec.n_nodes
    att = W.attention_inputs(W.scaled(w, ctx_hi=cap - spec.n_nodes), seed=seed, device=dev,
                             n_nodes=spec.n_nodes)
    att["prefix_len"] = W.prefix_lengths(w, seed=seed, device=dev)
    lm = W.randn((w.V, w.d), seed, 77, 1.0 / math.sqrt(w.d), "bf16", dev)
    bm = W.SyntheticBaseModel(w, spec, lm, R, seed=seed, device=dev)
    loop = DecodeLoop(B=w.B, d=w.d, V=w.V, K=w.K, kmax=w.kmax, tree=tree, Hq=w.Hq, Hkv=w.Hkv,
                      dh=w.dh, cap=cap, max_prefix=max_prefix, steps=R, device=dev)
    state = dict(h=heads["h"].clone(), root=W.random_root_tokens(w, seed, device=dev),
                 Kc=att["Kc"], Vc=att["Vc"], prefix_len=att["prefix_len"].clone())
    fixed = dict(W1=heads["W1"], b1=heads["b1"], W2=heads["W2"], lm_head=lm, base_model=bm,
                 q=att["q"], k_new=att["k_new"], v_new=att["v_new"])
    return w, spec, loop, state, fixed


def _step(loop, r, s, f):
    loop.step(r, s["h"], s["root"], f["W1"], f["b1"], f["W2"], f["lm_head"], f["base_model"],
              f["q"], f["k_new"], f["v_new"], s["Kc"], s["Vc"], s["prefix_len"])


def test_chained_steps_hand_off_and_graph_replay():
    R = 4
    w, spec, loop, s, f = _loop_setup(R)
    init = {k: v.clone() for k, v in s.items()}
    # eager, checking every hand-off against the oracle on the step's own data
    for r in range(R):
        p0 = s["prefix_len"].cpu().numpy().copy()
        _step(loop, r, s, f)
        torch.cuda.synchronize()
        assert int(loop.status.item()) == 0
        acc = loop.accept_len.cpu().numpy()
        nodes = loop.accepted_nodes.cpu().numpy()
        bonus = loop.bonus.cpu().numpy()
        hid = f64(f["base_model"].out.cpu())
        h_ref, root_ref = O.next_step_inputs(hid, acc, nodes, bonus)
        np.testing.assert_array_equal(f64(s["h"].cpu()), h_ref)
        assert s["root"].cpu().tolist() == root_ref.tolist()
        np.testing.assert_array_equal(s["prefix_len"].cpu().numpy(), p0 + acc + 1)
        # the kept branch's tokens are the candidates along it, then the bonus
        cand = loop.cand_ids.cpu().numpy()
        toks = loop.accepted_tokens.cpu().numpy()
        for b in range(w.B):
            L = acc[b]
            assert toks[b, :L].tolist() == [cand[b, n] for n in nodes[b, 1:L + 1]]
            assert toks[b, L] == bonus[b]
    eager = {k: v.clone() for k, v in s.items()}
    hist_eager = loop.history.clone()
    assert int(hist_eager.sum()) > 0  # some candidates were accepted
    # the same steps captured once and replayed from the initial state
    for k in s:
        s[k].copy_(init[k])
    loop.history.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for r in range(R):
                _step(loop, r, s, f)
    torch.cuda.current_stream().wait_stream(side)
    for k in s:
        s[k].copy_(init[k])
    graph.replay()
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0
    assert torch.equal(loop.history, hist_eager)
    for k in ("h", "root", "prefix_len", "Kc", "Vc"):
        assert torch.equal(s[k], eager[k]), k
    del graph
