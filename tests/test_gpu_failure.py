"""GPU: failure detection without a fault.  The library's bounded device wait
runs out on a flag that nothing sets: the call returns, the status word says
MEDUSA_ERR_TIMEOUT, and the same process then runs a normal call correctly."""
import time

import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from tests.helpers import check_topk, f64

pytestmark = pytest.mark.gpu

TIMEOUT = 5


def test_wait_on_a_flag_nothing_sets_times_out_and_returns():
    dev = "cuda"
    flag = torch.zeros(1, dtype=torch.int32, device=dev)   # nothing ever sets it
    status = M.new_status(dev)
    t0 = time.perf_counter()
    M.medusa_wait_flag(flag, 1, 2_000_000, status)         # about 1 ms of SM cycles
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(status.item()) == TIMEOUT
    assert waited < 5.0
    # the first error sticks: a second timeout leaves the code as it is
    M.medusa_wait_flag(flag, 1, 1_000_000, status)
    torch.cuda.synchronize()
    assert int(status.item()) == TIMEOUT


def test_wait_on_a_set_flag_returns_ok():
    dev = "cuda"
    flag = torch.full((1,), 7, dtype=torch.int32, device=dev)
    status = M.new_status(dev)
    M.medusa_wait_flag(flag, 7, 0, status)                 # the library's own bound
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_context_usable_after_a_timeout():
    """A timed-out wait, then a heads call in the same process: the status of
    the new call is clean and its top-k lists match the oracle."""
    dev = "cuda"
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    st_wait = M.new_status(dev)
    M.medusa_wait_flag(flag, 1, 1_000_000, st_wait)
    w = W.scaled(W.WORKLOADS["llama3_8b"], B=2, V=2000, d=256)
    inp = W.heads_inputs(w, seed=3)
    g = {k: v.to(dev) for k, v in inp.items()}
    ids = torch.empty(w.B, w.K, w.kmax, dtype=torch.int32, device=dev)
    vals = torch.empty(w.B, w.K, w.kmax, dtype=torch.float32, device=dev)
    st = M.new_status(dev)
    M.medusa_heads_topk(g["h"], g["W1"], g["b1"], g["W2"], w.kmax, ids, vals, dev_status=st)
    torch.cuda.synchronize()
    assert int(st_wait.item()) == TIMEOUT
    assert int(st.item()) == 0
    z = O.head_logits(f64(inp["h"]), f64(inp["W1"]), f64(inp["b1"]), f64(inp["W2"]))
    check_topk(ids.cpu().numpy(), vals.cpu().numpy(), z, w.kmax)
