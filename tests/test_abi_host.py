"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import speculative_decoding_medusa_b200 as M
from speculative_decoding_medusa_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MEDUSA_API\s+[\w\s\*]+?\b(medusa_\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from speculative_decoding_medusa_b200 import build
    build.build()
    return M.lib()


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(L, name), name
    assert set(_lib.EXPORTS) <= set(declared)


def test_status_strings_and_version(L):
    assert L.medusa_version() == 10000
    for code in range(9):
        assert L.medusa_status_string(code)
    assert L.medusa_status_string(99) == b"unknown status"


def _call_heads(L, **kw):
    a = dict(h=1024, W1=1024, b1=1024, W2=1024, dt=0, B=1, d=64, V=100, K=1, kmax=4,
             ids=1024, vals=1024, logits=None, ws=4096, ws_bytes=1 << 20, status=None, stream=None)
    a.update(kw)
    v = lambda x: ctypes.c_void_p(x) if x is not None else None
    return L.medusa_heads_topk(v(a["h"]), v(a["W1"]), v(a["b1"]), v(a["W2"]), a["dt"], a["B"], a["d"],
                               a["V"], a["K"], a["kmax"], v(a["ids"]), v(a["vals"]), v(a["logits"]),
                               v(a["ws"]), a["ws_bytes"], v(a["status"]), v(a["stream"]))


def test_heads_topk_host_checks(L):
    # the fake addresses below are never dereferenced: every case fails its
    # host-side check before any launch
    assert _call_heads(L, h=None) == 1
    assert _call_heads(L, dt=7) == 1
    assert _call_heads(L, B=0) == 2
    assert _call_heads(L, B=129) == 2
    assert _call_heads(L, K=17) == 2
    assert _call_heads(L, kmax=33) == 2
    assert _call_heads(L, kmax=101) == 2          # kmax > V
    assert _call_heads(L, d=96) == 2              # bf16 needs d % 64 == 0
    assert _call_heads(L, W2=1032) == 8           # misaligned
    assert _call_heads(L, ws=None) == 7
    assert _call_heads(L, ws_bytes=16) == 7
    assert _call_heads(L, ws=4096 + 16) == 7      # workspace must be 256-byte aligned
    assert b"workspace" in L.medusa_last_error()
    assert _call_heads(L, kmax=0) == 2 and b"kmax" in L.medusa_last_error()


def test_heads_topk_tree_host_checks(L):
    """The fused heads + tree call: the heads' checks, then the tree's, then
    the workspace."""
    v = ctypes.c_void_p
    good = _lib.medusa_tree_t(9, 2, 6, 1024, 1024, 1024)

    def call(h=1024, K=2, t=good, root=1024, ws=4096, ws_bytes=1 << 20):
        return L.medusa_heads_topk_tree(v(h) if h else None, v(1024), v(1024), v(1024), 0, 1, 64,
                                        100, K, 3, v(1024), v(1024), None,
                                        v(ws) if ws else None, ws_bytes, ctypes.byref(t),
                                        v(root) if root else None, v(1024), v(1024), v(1024),
                                        v(1024), v(1024), None, None)

    assert call(h=None) == 1
    assert call(K=17) == 2
    assert call(h=None, t=_lib.medusa_tree_t(0, 0, 1, 1024, 1024, 1024)) == 1  # heads first
    assert call(t=_lib.medusa_tree_t(0, 0, 1, 1024, 1024, 1024)) == 2
    assert call(root=None) == 1
    assert call(K=1) == 2                          # tree deeper than K heads
    assert call(root=None, ws=None) == 1           # the tree before the workspace
    assert call(ws=None) == 7
    assert call(ws_bytes=16) == 7


def test_tree_checks(L):
    good = _lib.medusa_tree_t(9, 2, 6, 1024, 1024, 1024)
    v = ctypes.c_void_p
    args = lambda t, K=2, kmax=3, B=1: (ctypes.byref(t), v(1024), v(1024), K, kmax, v(1024), B,
                                        v(1024), v(1024), v(1024), v(1024), None, None)
    assert L.medusa_tree_build(*args(_lib.medusa_tree_t(0, 0, 1, 1024, 1024, 1024))) == 2
    assert L.medusa_tree_build(*args(_lib.medusa_tree_t(257, 2, 6, 1024, 1024, 1024))) == 2
    assert L.medusa_tree_build(*args(_lib.medusa_tree_t(9, 2, 6, None, 1024, 1024))) == 1
    assert L.medusa_tree_build(*args(good, K=1)) == 2          # deeper than K heads
    assert L.medusa_tree_build(*args(good, kmax=33)) == 2
    assert L.medusa_tree_build(None, v(1024), v(1024), 2, 3, v(1024), 1, v(1024), v(1024),
                               v(1024), v(1024), None, None) == 1


def test_attention_verify_compact_checks(L):
    v = ctypes.c_void_p
    base = [v(1024)] * 7

    def attn(dt=0, B=1, N=9, Hq=4, Hkv=2, dh=128, cap=200, max_prefix=100, scale=0.1,
             ws=v(4096), ws_bytes=1 << 30, q=v(1024)):
        return L.medusa_tree_attention(q, *base[1:], dt, B, N, Hq, Hkv, dh, cap, max_prefix,
                                       scale, v(1024), dt, ws, ws_bytes, None, None)

    assert attn(q=None) == 1
    assert attn(Hq=5, Hkv=2) == 2
    assert attn(N=257) == 2
    assert attn(max_prefix=195) == 2              # max_prefix + N > cap
    assert attn(dh=96) == 2                       # bf16 dh in {64, 128}
    assert attn(dt=1, dh=48) == 2                 # f32 dh % 32
    assert attn(ws=None) == 7
    assert attn(scale=0.0) == 1

    tree = _lib.medusa_tree_t(9, 2, 6, 1024, 1024, 1024)

    def verify(mode=0, T=1.0, eps=0.09, delta=0.3, logits=v(1024), ws=v(4096)):
        return L.medusa_verify_accept(logits, 0, v(1024), ctypes.byref(tree), 1, 1000, mode, T, eps,
                                      delta, v(1024), v(1024), v(1024), v(1024), ws, 1 << 20, None,
                                      None)

    assert verify(logits=None) == 1
    assert verify(mode=3) == 1
    assert verify(mode=1, T=0.0) == 1
    assert verify(mode=1, eps=-1.0) == 1
    assert verify(logits=v(1032)) == 8
    assert verify(ws=None) == 7

    # the workspace-free variant: same argument checks first, then its 4 MiB
    # limit of B * n_nodes * ceil(V / 4096) 16-byte records, before any launch
    tree128 = _lib.medusa_tree_t(128, 4, 64, 1024, 1024, 1024)

    def noalloc(B=64, V=131073, logits=v(1024), t=tree128):
        return L.medusa_verify_accept_noalloc(logits, 0, v(1024), ctypes.byref(t), B, V, 0, 1.0,
                                              0.09, 0.3, v(1024), v(1024), v(1024), v(1024), None,
                                              None)

    assert noalloc() == 7                          # 64 x 128 x 33 = 270336 records
    assert b"4 MiB" in L.medusa_last_error()
    assert noalloc(V=131072) != 7                  # 64 x 128 x 32 = 262144: exactly fits
    assert noalloc(B=1024) == 2                    # B * n_nodes > 65535, as medusa_verify_accept
    assert noalloc(logits=None) == 1
    assert noalloc(logits=v(1032)) == 8
    assert noalloc(t=_lib.medusa_tree_t(300, 4, 64, 1024, 1024, 1024)) == 2

    def compact(max_depth=4, dh=128, Kc=v(1024)):
        return L.medusa_kv_compact(Kc, v(1024), 0, v(1024), v(1024), v(1024), 1, 2, dh, 100,
                                   max_depth, v(1024), None, None)

    assert compact(Kc=None) == 1
    assert compact(max_depth=16) == 2
    assert compact(dh=4) == 2                     # 8-byte rows are not 16-byte multiples
    assert compact(Kc=v(1032)) == 8

    # verification with the compaction: the verification's checks, then the
    # compaction's, then the workspace
    def fused(logits=v(1024), mode=0, Kc=v(1024), kv_dt=0, dh=128, ws=v(4096), ws_bytes=1 << 20):
        return L.medusa_verify_accept_compact(logits, 0, v(1024), ctypes.byref(tree), 1, 1000,
                                              mode, 1.0, 0.09, 0.3, v(1024), v(1024), v(1024),
                                              v(1024), Kc, v(1024), kv_dt, v(1024), 2, dh, 100,
                                              v(1024), ws, ws_bytes, None, None)

    assert fused(logits=None) == 1
    assert fused(mode=3) == 1
    assert fused(logits=v(1032), Kc=None) == 8     # the verification's check comes first
    assert fused(Kc=None) == 1
    assert fused(kv_dt=7) == 1
    assert fused(dh=4) == 2
    assert fused(Kc=v(1032)) == 8
    assert fused(ws=None) == 7
    assert fused(ws_bytes=16) == 7
    assert fused(ws=v(4100)) == 7                  # workspace not 256-byte aligned
    assert fused(kv_dt=1, dh=8192) == 3            # (max_depth + 1) rows of K and V > 96 KB

    def wait(flag=v(1024), budget=1000, status=v(2048)):
        return L.medusa_wait_flag(flag, 1, budget, status, None)

    assert wait(flag=None) == 1
    assert wait(status=None) == 1
    assert wait(flag=v(1026)) == 8
    assert wait(budget=2000000001) == 2           # above the library's own bound


def test_workspace_queries(L):
    assert M.medusa_heads_topk_workspace_size(8, 4096, 128256, 4, 10, 0) > 0
    assert M.medusa_heads_topk_workspace_size(0, 4096, 128256, 4, 10, 0) == 0
    assert M.medusa_tree_attention_workspace_size(8, 64, 32, 8, 128, 8192, 0) > 0
    assert M.medusa_tree_attention_workspace_size(1, 9, 4, 4, 64, 128, 1) == 0  # f32 needs none
    assert M.medusa_verify_accept_workspace_size(8, 64, 128256) > 0


def test_python_limits_match_the_header():
    """The binding's size limits are the header's #defines."""
    src = open(os.path.join(ROOT, "include", "medusa.h")).read()
    defs = dict(re.findall(r"#define MEDUSA_(MAX_\w+)\s+(\d+)", src))
    assert set(defs) == {"MAX_NODES", "MAX_KMAX", "MAX_HEADS", "MAX_BATCH"}, defs
    for name, value in defs.items():
        assert getattr(_lib, name) == int(value), name
