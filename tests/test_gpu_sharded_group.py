"""GPU: the vocabulary-sharded heads and verification run as a real group of
two ranks (two processes on the one GPU, gloo collectives staged through
host memory).  Each rank holds only its own W2 rows and verify-logit
columns, runs ShardedHeads / ShardedVerify end to end on a side stream (its
shard's kernels, the exchange, the merge kernels), and every output is
compared with the oracle.  No kernel waits on another rank: the ranks meet
only in the host-side collectives."""
import os
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import TYPICAL_LOG_MARGIN, check_topk, f64, i64

pytestmark = pytest.mark.gpu

WORLD = 2
HEADS = dict(B=4, V=3001, d=512)
GREEDY = dict(B=3, V=9001)
TYPICAL = dict(B=2, V=6000, accept="typical", temperature=0.7, eps=0.09, delta=0.3)


def _cands(w, spec, seed):
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, i64(root), i64(topk),
                      np.zeros(w.B, np.int64))
    return tb["cand"]


def _typical_case():
    """Typical-acceptance logits whose decisions keep the log margin."""
    w = W.scaled(W.WORKLOADS["llama3_70b"], **TYPICAL)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 11)
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=11, attempt=attempt)
        m = O.typical_log_margin(f64(logits), cand, spec.parent, w.temperature, w.eps, w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            return w, spec, cand, logits, attempt
    raise AssertionError("no margin-clean typical draw")


def _rank(rank, port, attempt, out):
    import speculative_decoding_medusa_b200 as M
    from speculative_decoding_medusa_b200 import sharded as S

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=120))
    try:
        dev = "cuda"
        side = torch.cuda.Stream()
        res = {}
        # heads: this rank's W2 rows only
        w = W.scaled(W.WORKLOADS["llama3_8b"], **HEADS)
        inp = W.heads_inputs(w, seed=21)
        v0, v1 = S.shard_range(w.V, WORLD, rank)
        heads = S.ShardedHeads(B=w.B, d=w.d, V=w.V, K=w.K, kmax=w.kmax, device=dev)
        ids, vals = heads.run(inp["h"].to(dev), inp["W1"].to(dev), inp["b1"].to(dev),
                              inp["W2"][:, v0:v1].contiguous().to(dev), stream=side)
        side.synchronize()
        res["heads"] = (ids.cpu().numpy(), vals.cpu().numpy(), int(heads.status.item()))
        # greedy verification: this rank's logit columns only
        for name, w, spec, cand, logits in _verify_cases(attempt):
            tree = M.Tree.from_spec(spec, dev)
            v0, v1 = S.shard_range(w.V, WORLD, rank)
            ver = S.ShardedVerify(B=w.B, N=spec.n_nodes, V=w.V, tree=tree, accept=w.accept,
                                  temperature=w.temperature, eps=w.eps, delta=w.delta, device=dev)
            outs = ver.run(logits[..., v0:v1].contiguous().to(dev),
                           torch.from_numpy(cand).to(dev), stream=side)
            side.synchronize()
            res[name] = ([t.cpu().numpy() for t in outs], int(ver.status.item()))
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _verify_cases(attempt):
    w = W.scaled(W.WORKLOADS["llama3_8b"], **GREEDY)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 12)
    yield "greedy", w, spec, cand, W.verify_logits(w, spec, torch.from_numpy(cand), seed=12)
    w = W.scaled(W.WORKLOADS["llama3_70b"], **TYPICAL)
    spec = W.tree_for(w)
    cand = _cands(w, spec, 11)
    yield "typical", w, spec, cand, W.verify_logits(w, spec, torch.from_numpy(cand), seed=11,
                                                    attempt=attempt)


def test_two_rank_group_matches_oracle():
    _, _, _, _, attempt = _typical_case()
    port = 29600 + os.getpid() % 1000
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(port, attempt, out), nprocs=WORLD, start_method="spawn",
                           join=True)
        res = dict(out)
    assert sorted(res) == list(range(WORLD))
    # heads: the merged lists against the oracle's logits of the whole vocabulary
    w = W.scaled(W.WORKLOADS["llama3_8b"], **HEADS)
    inp = W.heads_inputs(w, seed=21)
    z = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    for rank in range(WORLD):
        ids, vals, st = res[rank]["heads"]
        assert st == 0
        check_topk(ids, vals, z, w.kmax)
    np.testing.assert_array_equal(res[0]["heads"][0], res[1]["heads"][0])
    # verification: every output field equal to the oracle's, on every rank
    for name, w, spec, cand, logits in _verify_cases(attempt):
        if w.accept == "typical":
            ref = O.verify_typical(f64(logits), cand, spec.parent, spec.depth, spec.max_depth,
                                   w.temperature, w.eps, w.delta)
        else:
            ref = O.verify_greedy(f64(logits), cand, spec.parent, spec.depth, spec.max_depth)
        for rank in range(WORLD):
            got, st = res[rank][name]
            assert st == 0
            for k, a in zip(("accept_len", "accepted_nodes", "accepted_tokens", "bonus"), got):
                np.testing.assert_array_equal(a, ref[k], err_msg=f"{name} rank {rank} {k}")
