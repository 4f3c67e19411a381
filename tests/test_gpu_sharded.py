"""GPU: vocabulary-sharded heads and verification, the G shards computed one
after another on one GPU and stacked as an all-gather would, against the
oracle and against the unsharded calls (same kernels, same per-token
arithmetic)."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import sharded as S
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import (TYPICAL_LOG_MARGIN, check_topk, f64, i64,
                           oracle_head_logits_chunked)

pytestmark = pytest.mark.gpu


def _cands(w, spec, seed):
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk),
                      np.zeros(w.B, np.int64))
    return tb["cand"]


@pytest.mark.parametrize("G,V", [(2, 3000), (3, 2049), (8, 128256)])
def test_sharded_heads_equal_unsharded(G, V):
    dev = "cuda"
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=4, V=V, d=1024)
    inp = W.heads_inputs(w, seed=G, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    ids = torch.empty(w.B, w.K, w.kmax, **i32)
    vals = torch.empty(w.B, w.K, w.kmax, dtype=torch.float32, device=dev)
    M.medusa_heads_topk(inp["h"], inp["W1"], inp["b1"], inp["W2"], w.kmax, ids, vals)
    local_v, local_i = [], []
    for g in range(G):
        v0, v1 = S.shard_range(V, G, g)
        li = torch.empty(w.B, w.K, w.kmax, **i32)
        lv = torch.empty(w.B, w.K, w.kmax, dtype=torch.float32, device=dev)
        M.medusa_heads_topk(inp["h"], inp["W1"], inp["b1"], inp["W2"][:, v0:v1].contiguous(),
                            w.kmax, li, lv)
        local_v.append(lv)
        local_i.append(li)
    gv, gi = torch.stack(local_v), torch.stack(local_i)  # [G, B, K, kmax]
    offs = torch.tensor(S.shard_offsets(V, G), **i32)
    rows = w.B * w.K
    out_i = torch.empty_like(ids)
    out_v = torch.empty_like(vals)
    M.medusa_topk_merge(gv, gi, rows, G, w.kmax, w.kmax, rows * w.kmax, offs, w.kmax, out_i,
                        out_v)
    torch.cuda.synchronize()
    # the merged shard lists against the oracle's logits of the whole
    # vocabulary ...
    z = oracle_head_logits_chunked(inp["h"].cpu(), inp["W1"].cpu(), inp["b1"].cpu(),
                                   inp["W2"].cpu())
    check_topk(out_i.cpu().numpy(), out_v.cpu().numpy(), z, w.kmax)
    # ... and equal to the unsharded call bit for bit
    assert torch.equal(out_i, ids)
    assert torch.equal(out_v, vals)


def _sharded_verify(logits, cand, spec, G, mode, T=1.0, eps=0.09, delta=0.3):
    dev = "cuda"
    B, N, V = logits.shape
    tree = M.Tree.from_spec(spec)
    cd = torch.from_numpy(cand).to(dev)
    recs, cls = [], []
    st = M.new_status()
    for g in range(G):
        v0, v1 = S.shard_range(V, G, g)
        r = torch.empty(B * N, 4, device=dev)
        c = torch.empty(B * N, device=dev)
        M.medusa_verify_records(logits[..., v0:v1].contiguous(), cd, tree, v0, r, c, mode, T,
                                dev_status=st)
        recs.append(r)
        cls.append(c)
    records = torch.stack(recs)
    cand_logit = torch.stack(cls).max(dim=0).values  # what the max all-reduce gives
    W1 = spec.max_depth + 1
    out = [torch.full((B,), -9, dtype=torch.int32, device=dev),
           torch.full((B, W1), -9, dtype=torch.int32, device=dev),
           torch.full((B, W1), -9, dtype=torch.int32, device=dev),
           torch.full((B,), -9, dtype=torch.int32, device=dev)]
    M.medusa_verify_from_records(records, cand_logit, cd, tree, V, *out, mode, T, eps, delta,
                                 dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return [t.cpu().numpy() for t in out]


def _unsharded(logits, cand, spec, mode, T=1.0, eps=0.09, delta=0.3):
    dev = "cuda"
    B, N, V = logits.shape
    W1 = spec.max_depth + 1
    out = [torch.full((B,), -9, dtype=torch.int32, device=dev),
           torch.full((B, W1), -9, dtype=torch.int32, device=dev),
           torch.full((B, W1), -9, dtype=torch.int32, device=dev),
           torch.full((B,), -9, dtype=torch.int32, device=dev)]
    st = M.new_status()
    M.medusa_verify_accept(logits, torch.from_numpy(cand).to(dev), M.Tree.from_spec(spec), *out,
                           mode, T, eps, delta, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return [t.cpu().numpy() for t in out]


@pytest.mark.parametrize("G,V,dtype", [(2, 9000, torch.bfloat16), (5, 20001, torch.bfloat16),
                                       (8, 128256, torch.bfloat16), (3, 4000, torch.float32)])
def test_sharded_greedy_equals_unsharded(G, V, dtype):
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=3, V=V)
    spec = W.tree_for(w)
    cand = _cands(w, spec, G)
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=G, device="cuda",
                             dtype="bf16" if dtype == torch.bfloat16 else "f32")
    got = _sharded_verify(logits, cand, spec, G, M.MEDUSA_ACCEPT_GREEDY)
    ref = _unsharded(logits, cand, spec, M.MEDUSA_ACCEPT_GREEDY)
    for a, b in zip(got, ref):
        np.testing.assert_array_equal(a, b)
    oracle = O.verify_greedy(f64(logits.cpu()), cand, spec.parent, spec.depth, spec.max_depth)
    for k, a in zip(("accept_len", "accepted_nodes", "accepted_tokens", "bonus"), got):
        np.testing.assert_array_equal(a, oracle[k], err_msg=k)


@pytest.mark.parametrize("G,V", [(2, 6000), (4, 30000)])
def test_sharded_typical_equals_oracle(G, V):
    w = W.scaled(W.WORKLOADS["llama3_70b"], B=2, V=V, accept="typical", temperature=0.7,
                 eps=0.09, delta=0.3)
    spec = W.tree_for(w)
    cand = _cands(w, spec, G)
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=G, attempt=attempt)
        m = O.typical_log_margin(f64(logits), cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            break
    else:
        pytest.skip("no margin-clean draw")
    got = _sharded_verify(logits.cuda(), cand, spec, G, M.MEDUSA_ACCEPT_TYPICAL, w.temperature,
                          w.eps, w.delta)
    ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                           w.temperature, w.eps, w.delta)
    for k, a in zip(("accept_len", "accepted_nodes", "accepted_tokens", "bonus"), got):
        np.testing.assert_array_equal(a, ref[k], err_msg=k)
