"""medusa_verify_accept_noalloc: verification for callers that cannot give the
library device memory per call (the library uses its own fixed 4 MiB device
array instead of a workspace).  Its results must equal medusa_verify_accept's,
bit for bit, on consecutive calls that reuse the shared array.

This file is collected last so that a failure here leaves every other test
already run."""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import _lib
from speculative_decoding_medusa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _outputs(B, W1, dev):
    return [torch.full(s, -9, dtype=torch.int32, device=dev) for s in ((B,), (B, W1), (B, W1), (B,))]


def _case(name, B, V, seed, accept, n_nodes=None):
    base = W.WORKLOADS[name]
    w = W.scaled(base, B=B, V=V, accept=accept)
    spec = W.tree_for(w, n_nodes=n_nodes)
    root = W.random_root_tokens(w, seed)
    topk = W.random_topk_ids(w, seed)
    cand = O.tree_build(spec.parent, spec.depth, spec.rank, root.numpy().astype(np.int64),
                        topk.numpy().astype(np.int64), np.zeros(B, np.int64))["cand"]
    # large cases draw their logits on the device (same recipe)
    dev = "cuda" if B * spec.n_nodes * V > (1 << 27) else "cpu"
    logits = W.verify_logits(w, spec, torch.from_numpy(cand), seed=seed, device=dev)
    return w, spec, torch.from_numpy(cand), logits


@pytest.mark.parametrize("name,B,V,seed,accept,n_nodes", [
    ("llama3_8b", 8, 128256, 0, "greedy", None),
    ("llama3_70b", 2, 50000, 1, "typical", None),
    ("tiny", 3, 1000, 2, "greedy", None),
    # the size the header names: 32 x 128 nodes x 32 chunks = 131072 records
    ("long", 32, 128256, 3, "greedy", 128),
    # exactly at the limit: 16 x 256 nodes x 64 chunks = 262144 records = 4 MiB
    ("llama3_70b", 16, 262144, 4, "greedy", 256),
])
def test_noalloc_matches_workspace_call_twice(name, B, V, seed, accept, n_nodes):
    dev = "cuda"
    w, spec, cand, logits = _case(name, B, V, seed, accept, n_nodes)
    tree = M.Tree.from_spec(spec, dev)
    lg, cd = logits.to(dev), cand.to(dev)
    mode = M.MEDUSA_ACCEPT_TYPICAL if accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
    Wd = spec.max_depth + 1
    ref = _outputs(B, Wd, dev)
    st = M.new_status()
    M.medusa_verify_accept(lg, cd, tree, *ref, mode, w.temperature, w.eps, w.delta, dev_status=st)
    for call in range(2):  # the second call finds the first call's data in the array
        got = _outputs(B, Wd, dev)
        # through the C ABI directly
        ct = tree.c()
        rc = _lib.lib().medusa_verify_accept_noalloc(
            ctypes.c_void_p(lg.data_ptr()), _lib._dt(lg), ctypes.c_void_p(cd.data_ptr()),
            ctypes.byref(ct), B, V, mode, w.temperature, w.eps, w.delta,
            *[ctypes.c_void_p(t.data_ptr()) for t in got], ctypes.c_void_p(st.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, _lib.lib().medusa_last_error()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for a, b in zip(got, ref):
            assert torch.equal(a, b), f"call {call}"


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    dev = "cuda"
    spec = W.cartesian_tree([4, 4, 4, 4], n_nodes=256)
    tree = M.Tree.from_spec(spec, dev)
    B, V = 64, 131073           # 64 * 256 * 17 records of 16 bytes > 4 MiB
    tiny = torch.zeros(16, dtype=torch.bfloat16, device=dev)  # never read: rejected first
    outs = _outputs(B, spec.max_depth + 1, dev)
    ct = tree.c()
    rc = _lib.lib().medusa_verify_accept_noalloc(
        ctypes.c_void_p(tiny.data_ptr()), 0, ctypes.c_void_p(outs[0].data_ptr()), ctypes.byref(ct),
        B, V, 0, 1.0, 0.09, 0.3, *[ctypes.c_void_p(t.data_ptr()) for t in outs], None, None)
    assert rc == 7
    assert b"4 MiB" in _lib.lib().medusa_last_error()
    torch.cuda.synchronize()
    assert (outs[0] == -9).all()


def test_noalloc_rejects_one_record_over_the_limit():
    """64 x 128 nodes x 33 chunks = 270336 records: one chunk per row past
    the 4 MiB array (V = 131073 needs 33 chunks of 4096, V = 131072 only 32)."""
    dev = "cuda"
    spec = W.tree_for(W.WORKLOADS["long"], n_nodes=128)
    tree = M.Tree.from_spec(spec, dev)
    tiny = torch.zeros(16, dtype=torch.bfloat16, device=dev)  # never read: rejected first
    outs = _outputs(64, spec.max_depth + 1, dev)
    ct = tree.c()

    def call(V):
        return _lib.lib().medusa_verify_accept_noalloc(
            ctypes.c_void_p(tiny.data_ptr()), 0, ctypes.c_void_p(outs[0].data_ptr()),
            ctypes.byref(ct), 64, V, 0, 1.0, 0.09, 0.3,
            *[ctypes.c_void_p(t.data_ptr()) for t in outs], None, None)

    assert call(131073) == 7
    # a bad shape is reported as the workspace call reports it, not as a
    # scratch overflow: B * n_nodes above 65535
    assert _lib.lib().medusa_verify_accept_noalloc(
        ctypes.c_void_p(tiny.data_ptr()), 0, ctypes.c_void_p(outs[0].data_ptr()),
        ctypes.byref(ct), 1024, 131073, 0, 1.0, 0.09, 0.3,
        *[ctypes.c_void_p(t.data_ptr()) for t in outs], None, None) == 2
    torch.cuda.synchronize()
    assert (outs[0] == -9).all()
