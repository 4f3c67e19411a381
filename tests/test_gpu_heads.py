"""GPU parity: medusa_heads_topk against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import LOGIT_MAX_ABS, check_topk, f64, i64, oracle_head_logits_chunked

pytestmark = pytest.mark.gpu


def _run(inp, kmax, want_logits=True):
    dev = "cuda"
    h, W1, b1, W2 = (inp[k].to(dev) for k in ("h", "W1", "b1", "W2"))
    B, K, V = h.shape[0], W2.shape[0], W2.shape[1]
    ids = torch.full((B, K, kmax), -7, dtype=torch.int32, device=dev)
    vals = torch.full((B, K, kmax), float("nan"), dtype=torch.float32, device=dev)
    logits = torch.full((B, K, V), float("nan"), device=dev) if want_logits else None
    status = M.new_status()
    M.medusa_heads_topk(h, W1, b1, W2, kmax, ids, vals, logits, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return ids.cpu().numpy(), vals.cpu().numpy(), (None if logits is None else f64(logits))


def _case(name, **over):
    return W.scaled(W.WORKLOADS[name], **over)


@pytest.mark.parametrize("zero_init", [False, True])
def test_tiny_fp32(zero_init):
    w = W.WORKLOADS["tiny"]
    inp = W.heads_inputs(w, seed=0, zero_init=zero_init)
    ids, vals, z = _run(inp, w.kmax)
    zr = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    assert np.abs(z - zr).max() < 1e-4
    check_topk(ids, vals, zr, w.kmax)
    if zero_init:  # every head reproduces lm_head(h)
        base = O.lm_head_logits(f64(inp["h"]), f64(inp["lm_head"]))
        for k in range(w.K):
            assert np.abs(z[:, k] - base).max() < 1e-4


@pytest.mark.parametrize("B,d,V,K,kmax", [
    (1, 256, 1000, 3, 3),       # ragged vocab tile, smallest MMA width
    (3, 512, 3000, 3, 10),      # ragged vocab tail, several k-blocks
    (8, 192, 777, 2, 32),       # d % 128 != 0 (ragged W1 tile), kmax = 32
    (20, 256, 1500, 2, 5),      # 2B = 40 columns -> 64-wide MMA
    (40, 128, 640, 1, 4),       # 128-wide MMA
    (100, 64, 300, 2, 8),       # 256-wide MMA, one k-block
    (4, 2048, 3000, 3, 10),     # stream-K first GEMM: 48 tiles of 32 k-blocks, 11 per CTA
    (20, 2048, 1500, 3, 5),     # the same at 32 columns
    (128, 128, 700, 16, 32),    # the limits: MAX_BATCH sequences, MAX_HEADS heads, MAX_KMAX
])
def test_bf16_small(B, d, V, K, kmax):
    w = _case("vicuna7b", B=B, d=d, V=V, K=K, kmax=kmax)
    inp = W.heads_inputs(w, seed=B * 7 + d)
    ids, vals, z = _run(inp, kmax)
    zr = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    err = np.abs(z - zr).max()
    assert err < LOGIT_MAX_ABS, err
    assert err < 1e-3, f"logit error {err} far above fp32 accumulation"
    check_topk(ids, vals, zr, kmax)


def test_bf16_zero_init_equals_lm_head():
    w = _case("vicuna7b", B=2, d=256, V=2000, K=3, kmax=4)
    inp = W.heads_inputs(w, seed=3, zero_init=True)
    ids, vals, z = _run(inp, w.kmax)
    base = O.lm_head_logits(f64(inp["h"]), f64(inp["lm_head"]))
    for k in range(w.K):
        assert np.abs(z[:, k] - base).max() < LOGIT_MAX_ABS
        np.testing.assert_array_equal(ids[:, k], ids[:, 0])


def test_bf16_topk_without_logits_output():
    w = _case("vicuna7b", B=2, d=256, V=2048, K=2, kmax=10)
    inp = W.heads_inputs(w, seed=11)
    ids, vals, _ = _run(inp, w.kmax, want_logits=False)
    zr = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    check_topk(ids, vals, zr, w.kmax)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["vicuna7b", "llama3_8b", "llama3_70b", "long"])
def test_full_size(name):
    # llama3_70b: d = 8192 (128 k-blocks per tile); long: B = 32, so the
    # second GEMM runs 64 columns (hi and lo of every sequence) per MMA
    w = W.WORKLOADS[name]
    inp = W.heads_inputs(w, seed=0)
    ids, vals, z = _run(inp, w.kmax)
    zr = oracle_head_logits_chunked(inp["h"], inp["W1"], inp["b1"], inp["W2"])
    err = np.abs(z - zr).max()
    assert err < LOGIT_MAX_ABS, err
    check_topk(ids, vals, zr, w.kmax)
