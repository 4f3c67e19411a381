"""ctypes binding of libmedusa_b200.so: one Python function per C entry point,
same names, argument marshalling only (tensor -> pointer and sizes, stream
handle).  Every step of the computation runs in the library's CUDA kernels;
there is no fallback: a missing library or a non-OK status raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmedusa_b200.so")

MEDUSA_BF16 = 0
MEDUSA_F32 = 1
MEDUSA_ACCEPT_GREEDY = 0
MEDUSA_ACCEPT_TYPICAL = 1
MAX_NODES = 256
MAX_KMAX = 32
MAX_HEADS = 16
MAX_BATCH = 128

STATUS_NAMES = {
    0: "MEDUSA_OK", 1: "MEDUSA_ERR_INVALID_ARG", 2: "MEDUSA_ERR_SHAPE",
    3: "MEDUSA_ERR_UNSUPPORTED", 4: "MEDUSA_ERR_CUDA", 5: "MEDUSA_ERR_TIMEOUT",
    6: "MEDUSA_ERR_DEVICE_CHECK", 7: "MEDUSA_ERR_WORKSPACE", 8: "MEDUSA_ERR_ALIGNMENT",
}

# exported symbols declared in include/medusa.h
EXPORTS = (
    "medusa_status_string", "medusa_last_error", "medusa_version",
    "medusa_heads_topk_workspace_size", "medusa_heads_topk",
    "medusa_tree_build",
    "medusa_tree_attention_workspace_size", "medusa_tree_attention",
    "medusa_verify_accept_workspace_size", "medusa_verify_accept",
    "medusa_kv_compact", "medusa_verify_accept_compact", "medusa_heads_topk_tree", "medusa_verify_accept_noalloc",
    "medusa_lmhead_verify_workspace_size", "medusa_lmhead_verify", "medusa_next_step",
    "medusa_tree_from_accuracies", "medusa_sample_bonus", "medusa_topk_merge",
    "medusa_verify_records_workspace_size", "medusa_verify_records", "medusa_verify_from_records",
    "medusa_wait_flag",
)


class MedusaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class medusa_tree_t(ctypes.Structure):
    _fields_ = [("n_nodes", ctypes.c_int32), ("max_depth", ctypes.c_int32),
                ("n_leaves", ctypes.c_int32), ("parent", ctypes.c_void_p),
                ("depth", ctypes.c_void_p), ("rank", ctypes.c_void_p)]


_lib = None

_V, _I, _Z, _F, _U = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load the library (built by ``speculative_decoding_medusa_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m speculative_decoding_medusa_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.medusa_status_string.restype = ctypes.c_char_p
    L.medusa_status_string.argtypes = [_I]
    L.medusa_last_error.restype = ctypes.c_char_p
    L.medusa_last_error.argtypes = []
    L.medusa_version.restype = _I
    L.medusa_heads_topk_workspace_size.restype = _Z
    L.medusa_heads_topk_workspace_size.argtypes = [_I] * 5 + [_I]
    L.medusa_heads_topk.restype = _I
    L.medusa_heads_topk.argtypes = [_V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _V, _V, _V, _V, _Z, _V, _V]
    L.medusa_heads_topk_tree.restype = _I
    L.medusa_heads_topk_tree.argtypes = [_V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _V, _V, _V, _V, _Z,
                                         ctypes.POINTER(medusa_tree_t), _V, _V, _V, _V, _V, _V, _V,
                                         _V]
    L.medusa_tree_build.restype = _I
    L.medusa_tree_build.argtypes = [ctypes.POINTER(medusa_tree_t), _V, _V, _I, _I, _V, _I,
                                    _V, _V, _V, _V, _V, _V]
    L.medusa_tree_attention_workspace_size.restype = _Z
    L.medusa_tree_attention_workspace_size.argtypes = [_I] * 6 + [_I]
    L.medusa_tree_attention.restype = _I
    L.medusa_tree_attention.argtypes = [_V, _V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _I, _I,
                                        _F, _V, _I, _V, _Z, _V, _V]
    L.medusa_verify_accept_workspace_size.restype = _Z
    L.medusa_verify_accept_workspace_size.argtypes = [_I, _I, _I]
    L.medusa_verify_accept.restype = _I
    L.medusa_verify_accept.argtypes = [_V, _I, _V, ctypes.POINTER(medusa_tree_t), _I, _I, _I, _F, _F,
                                       _F, _V, _V, _V, _V, _V, _Z, _V, _V]
    L.medusa_verify_accept_noalloc.restype = _I
    L.medusa_verify_accept_noalloc.argtypes = [_V, _I, _V, ctypes.POINTER(medusa_tree_t), _I, _I, _I,
                                               _F, _F, _F, _V, _V, _V, _V, _V, _V]
    L.medusa_verify_accept_compact.restype = _I
    L.medusa_verify_accept_compact.argtypes = [_V, _I, _V, ctypes.POINTER(medusa_tree_t), _I, _I, _I,
                                               _F, _F, _F, _V, _V, _V, _V, _V, _V, _I, _V, _I, _I,
                                               _I, _V, _V, _Z, _V, _V]
    L.medusa_kv_compact.restype = _I
    L.medusa_kv_compact.argtypes = [_V, _V, _I, _V, _V, _V, _I, _I, _I, _I, _I, _V, _V, _V]
    L.medusa_lmhead_verify_workspace_size.restype = _Z
    L.medusa_lmhead_verify_workspace_size.argtypes = [_I, _I, _I, _I]
    _LL = ctypes.c_longlong
    L.medusa_topk_merge.restype = _I
    L.medusa_topk_merge.argtypes = [_V, _V, _I, _I, _I, _LL, _LL, _V, _I, _V, _V, _V]
    L.medusa_verify_records_workspace_size.restype = _Z
    L.medusa_verify_records_workspace_size.argtypes = [_I, _I, _I]
    L.medusa_verify_records.restype = _I
    L.medusa_verify_records.argtypes = [_V, _I, _V, ctypes.POINTER(medusa_tree_t), _I, _I, _I, _I,
                                        _F, _V, _V, _V, _Z, _V, _V]
    L.medusa_verify_from_records.restype = _I
    L.medusa_verify_from_records.argtypes = [_V, _I, _V, _V, ctypes.POINTER(medusa_tree_t), _I, _I,
                                             _I, _F, _F, _F, _V, _V, _V, _V, _V, _V]
    L.medusa_sample_bonus.restype = _I
    L.medusa_sample_bonus.argtypes = [_V, _I, _V, _V, _I, _I, _I, _I, _F, ctypes.c_uint64,
                                      ctypes.c_uint64, _V, _V, _V, _V]
    L.medusa_tree_from_accuracies.restype = _I
    L.medusa_tree_from_accuracies.argtypes = [_V, _I, _I, _I, _I, _V, _V, _V, _V]
    L.medusa_next_step.restype = _I
    L.medusa_next_step.argtypes = [_V, _I, _V, _V, _V, _I, _I, _I, _I, _V, _V, _V, _V]
    L.medusa_wait_flag.restype = _I
    L.medusa_wait_flag.argtypes = [_V, ctypes.c_int32, ctypes.c_longlong, _V, _V]
    L.medusa_lmhead_verify.restype = _I
    L.medusa_lmhead_verify.argtypes = [_V, _V, _I, _V, ctypes.POINTER(medusa_tree_t), _I, _I, _I,
                                       _I, _F, _F, _F, _V, _V, _V, _V, _V, _V, _Z, _V, _V]
    _lib = L
    return L


def _check(st: int) -> None:
    if st != 0:
        raise MedusaError(st, lib().medusa_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MEDUSA_BF16
    if t.dtype == torch.float32:
        return MEDUSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _req(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A 256-byte aligned byte buffer (torch's caching allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


class Tree:
    """A candidate tree on the device (parent/depth/rank int32 arrays)."""

    def __init__(self, parent, depth, rank, n_leaves: int, device=None):
        dev = device or "cuda"
        self.parent = torch.as_tensor(parent, dtype=torch.int32).to(dev).contiguous()
        self.depth = torch.as_tensor(depth, dtype=torch.int32).to(dev).contiguous()
        self.rank = torch.as_tensor(rank, dtype=torch.int32).to(dev).contiguous()
        self.n_nodes = int(self.parent.numel())
        self.max_depth = int(torch.as_tensor(depth).max().item()) if self.n_nodes else 0
        self.n_leaves = int(n_leaves)

    @classmethod
    def from_spec(cls, spec, device=None) -> "Tree":
        return cls(spec.parent, spec.depth, spec.rank, spec.n_leaves, device)

    def c(self) -> medusa_tree_t:
        return medusa_tree_t(self.n_nodes, self.max_depth, self.n_leaves,
                             self.parent.data_ptr(), self.depth.data_ptr(), self.rank.data_ptr())


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------


def medusa_heads_topk_workspace_size(B: int, d: int, V: int, K: int, kmax: int, dt: int) -> int:
    return int(lib().medusa_heads_topk_workspace_size(B, d, V, K, kmax, dt))


def medusa_heads_topk(h, W1, b1, W2, kmax: int, topk_ids, topk_vals, logits=None, ws=None,
                      dev_status=None, stream=None) -> None:
    """h [B,d], W1 [K,d,d], b1 [K,d], W2 [K,V,d] -> topk_ids/vals [B,K,kmax]
    (and logits [B,K,V] fp32 when given)."""
    for t, n in ((h, "h"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (topk_ids, "topk_ids"),
                 (topk_vals, "topk_vals")):
        _req(t, n)
    B, d = h.shape
    K, V, _ = W2.shape
    dt = _dt(W2)
    if ws is None:
        ws = workspace(medusa_heads_topk_workspace_size(B, d, V, K, kmax, dt), h.device)
    _check(lib().medusa_heads_topk(_p(h), _p(W1), _p(b1), _p(W2), dt, B, d, V, K, kmax,
                                   _p(topk_ids), _p(topk_vals), _p(logits), _p(ws), ws.numel(),
                                   _p(dev_status), _stream(stream)))


def medusa_heads_topk_tree(h, W1, b1, W2, kmax: int, topk_ids, topk_vals, tree: Tree, root_tok,
                           prefix_len, cand_ids, pos_ids, anc_mask, retrieve, logits=None,
                           ws=None, dev_status=None, stream=None) -> None:
    """medusa_heads_topk, then medusa_tree_build of its lists, in the heads'
    launches."""
    for t, n in ((h, "h"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (topk_ids, "topk_ids"),
                 (topk_vals, "topk_vals")):
        _req(t, n)
    B, d = h.shape
    K, V, _ = W2.shape
    dt = _dt(W2)
    if ws is None:
        ws = workspace(medusa_heads_topk_workspace_size(B, d, V, K, kmax, dt), h.device)
    ct = tree.c()
    _check(lib().medusa_heads_topk_tree(_p(h), _p(W1), _p(b1), _p(W2), dt, B, d, V, K, kmax,
                                        _p(topk_ids), _p(topk_vals), _p(logits), _p(ws),
                                        ws.numel(), ctypes.byref(ct), _p(root_tok),
                                        _p(prefix_len), _p(cand_ids), _p(pos_ids), _p(anc_mask),
                                        _p(retrieve), _p(dev_status), _stream(stream)))


def medusa_tree_build(tree: Tree, root_tok, topk_ids, prefix_len, cand_ids, pos_ids, anc_mask,
                      retrieve, dev_status=None, stream=None) -> None:
    B, K, kmax = topk_ids.shape
    ct = tree.c()
    _check(lib().medusa_tree_build(ctypes.byref(ct), _p(root_tok), _p(topk_ids), K, kmax,
                                   _p(prefix_len), B, _p(cand_ids), _p(pos_ids), _p(anc_mask),
                                   _p(retrieve), _p(dev_status), _stream(stream)))


def medusa_tree_attention_workspace_size(B: int, N: int, Hq: int, Hkv: int, dh: int,
                                         max_prefix: int, dt: int) -> int:
    return int(lib().medusa_tree_attention_workspace_size(B, N, Hq, Hkv, dh, max_prefix, dt))


def medusa_tree_attention(q, k_new, v_new, Kc, Vc, prefix_len, anc_mask, max_prefix: int, out,
                          scale: Optional[float] = None, ws=None, dev_status=None,
                          stream=None) -> None:
    """q [B,N,Hq,dh], k_new/v_new [B,N,Hkv,dh], Kc/Vc [B,Hkv,cap,dh] -> out [B,N,Hq,dh]."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (Kc, "Kc"), (Vc, "Vc"),
                 (out, "out")):
        _req(t, n)
    B, N, Hq, dh = q.shape
    Hkv, cap = Kc.shape[1], Kc.shape[2]
    dt = _dt(q)
    if scale is None:
        scale = dh ** -0.5
    if ws is None:
        ws = workspace(medusa_tree_attention_workspace_size(B, N, Hq, Hkv, dh, max_prefix, dt),
                       q.device)
    _check(lib().medusa_tree_attention(_p(q), _p(k_new), _p(v_new), _p(Kc), _p(Vc),
                                       _p(prefix_len), _p(anc_mask), dt, B, N, Hq, Hkv, dh, cap,
                                       max_prefix, float(scale), _p(out), _dt(out), _p(ws),
                                       ws.numel(), _p(dev_status), _stream(stream)))


def medusa_verify_accept_workspace_size(B: int, N: int, V: int) -> int:
    return int(lib().medusa_verify_accept_workspace_size(B, N, V))


def medusa_verify_accept(logits, cand_ids, tree: Tree, accept_len, accepted_nodes,
                         accepted_tokens, bonus, mode: int = MEDUSA_ACCEPT_GREEDY,
                         temperature: float = 1.0, eps: float = 0.09, delta: float = 0.3,
                         ws=None, dev_status=None, stream=None) -> None:
    """logits [B,N,V] -> accept_len [B], accepted_nodes/tokens [B,Dmax+1], bonus [B]."""
    _req(logits, "logits")
    B, N, V = logits.shape
    if ws is None:
        ws = workspace(medusa_verify_accept_workspace_size(B, N, V), logits.device)
    ct = tree.c()
    _check(lib().medusa_verify_accept(_p(logits), _dt(logits), _p(cand_ids), ctypes.byref(ct), B, V,
                                      mode, float(temperature), float(eps), float(delta),
                                      _p(accept_len), _p(accepted_nodes), _p(accepted_tokens),
                                      _p(bonus), _p(ws), ws.numel(), _p(dev_status),
                                      _stream(stream)))


def medusa_kv_compact(Kc, Vc, prefix_len, accepted_nodes, accept_len, compact_src,
                      dev_status=None, stream=None) -> None:
    _req(Kc, "Kc")
    _req(Vc, "Vc")
    B, Hkv, cap, dh = Kc.shape
    max_depth = accepted_nodes.shape[1] - 1
    _check(lib().medusa_kv_compact(_p(Kc), _p(Vc), _dt(Kc), _p(prefix_len), _p(accepted_nodes),
                                   _p(accept_len), B, Hkv, dh, cap, max_depth, _p(compact_src),
                                   _p(dev_status), _stream(stream)))


def medusa_verify_accept_compact(logits, cand_ids, tree: Tree, accept_len, accepted_nodes,
                                 accepted_tokens, bonus, Kc, Vc, prefix_len, compact_src,
                                 mode: int = MEDUSA_ACCEPT_GREEDY, temperature: float = 1.0,
                                 eps: float = 0.09, delta: float = 0.3, ws=None, dev_status=None,
                                 stream=None) -> None:
    """medusa_verify_accept, then medusa_kv_compact of its result, in the
    verification's launches."""
    _req(logits, "logits")
    _req(Kc, "Kc")
    _req(Vc, "Vc")
    B, N, V = logits.shape
    _, Hkv, cap, dh = Kc.shape
    if ws is None:
        ws = workspace(medusa_verify_accept_workspace_size(B, N, V), logits.device)
    ct = tree.c()
    _check(lib().medusa_verify_accept_compact(
        _p(logits), _dt(logits), _p(cand_ids), ctypes.byref(ct), B, V, mode, float(temperature),
        float(eps), float(delta), _p(accept_len), _p(accepted_nodes), _p(accepted_tokens),
        _p(bonus), _p(Kc), _p(Vc), _dt(Kc), _p(prefix_len), Hkv, dh, cap, _p(compact_src),
        _p(ws), ws.numel(), _p(dev_status), _stream(stream)))


def medusa_verify_accept_noalloc(logits, cand_ids, tree: Tree, accept_len, accepted_nodes,
                                 accepted_tokens, bonus, mode: int = MEDUSA_ACCEPT_GREEDY,
                                 temperature: float = 1.0, eps: float = 0.09, delta: float = 0.3,
                                 dev_status=None, stream=None) -> None:
    """medusa_verify_accept without a workspace argument, for callers that
    cannot hand the library device memory per call: the library keeps its
    own fixed 4 MiB scratch on each device.  Calls that overlap on the GPU
    share that scratch and race."""
    _req(logits, "logits")
    B, N, V = logits.shape
    ct = tree.c()
    _check(lib().medusa_verify_accept_noalloc(_p(logits), _dt(logits), _p(cand_ids),
                                              ctypes.byref(ct), B, V, mode, float(temperature),
                                              float(eps), float(delta), _p(accept_len),
                                              _p(accepted_nodes), _p(accepted_tokens), _p(bonus),
                                              _p(dev_status), _stream(stream)))


def medusa_lmhead_verify_workspace_size(B: int, N: int, d: int, V: int) -> int:
    return int(lib().medusa_lmhead_verify_workspace_size(B, N, d, V))


def medusa_lmhead_verify(hidden, lm_head, cand_ids, tree: Tree, accept_len, accepted_nodes,
                         accepted_tokens, bonus, mode: int = MEDUSA_ACCEPT_GREEDY,
                         temperature: float = 1.0, eps: float = 0.09, delta: float = 0.3,
                         logits=None, ws=None, dev_status=None, stream=None) -> None:
    """hidden [B,N,d] bf16, lm_head [V,d] bf16 -> the verify outputs of
    medusa_verify_accept on logits = hidden @ lm_head^T, never materialised
    unless ``logits`` ([B,N,V] fp32) is given."""
    _req(hidden, "hidden")
    _req(lm_head, "lm_head")
    B, N, d = hidden.shape
    V = lm_head.shape[0]
    if ws is None:
        ws = workspace(medusa_lmhead_verify_workspace_size(B, N, d, V), hidden.device)
    ct = tree.c()
    _check(lib().medusa_lmhead_verify(_p(hidden), _p(lm_head), _dt(hidden), _p(cand_ids),
                                      ctypes.byref(ct), B, d, V, mode, float(temperature),
                                      float(eps), float(delta), _p(accept_len),
                                      _p(accepted_nodes), _p(accepted_tokens), _p(bonus),
                                      _p(logits), _p(ws), ws.numel(), _p(dev_status),
                                      _stream(stream)))


def medusa_next_step(node_hidden, accept_len, accepted_nodes, bonus, h_next, root_next,
                     dev_status=None, stream=None) -> None:
    """h_next[b] = node_hidden[b, kept node], root_next[b] = bonus[b]."""
    _req(node_hidden, "node_hidden")
    _req(h_next, "h_next")
    B, N, d = node_hidden.shape
    max_depth = accepted_nodes.shape[1] - 1
    _check(lib().medusa_next_step(_p(node_hidden), _dt(node_hidden), _p(accept_len),
                                  _p(accepted_nodes), _p(bonus), B, N, d, max_depth, _p(h_next),
                                  _p(root_next), _p(dev_status), _stream(stream)))


def medusa_tree_from_accuracies(acc, n_nodes: int, max_depth: int):
    """acc [K, kmax] (array-like, probabilities) -> (parent, depth, rank)
    int32 numpy arrays of the n_nodes-node tree of the most accurate
    combinations, and its expected accept length.  Host only."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(acc, dtype=np.float32))
    K, kmax = a.shape
    out = [np.zeros(n_nodes, dtype=np.int32) for _ in range(3)]
    e = ctypes.c_double(0.0)
    _check(lib().medusa_tree_from_accuracies(a.ctypes.data, K, kmax, n_nodes, max_depth,
                                             out[0].ctypes.data, out[1].ctypes.data,
                                             out[2].ctypes.data, ctypes.byref(e)))
    return out[0], out[1], out[2], e.value


def medusa_sample_bonus(logits, accept_len, accepted_nodes, bonus, accepted_tokens,
                        temperature: float, seed: int, offset: int = 0, dev_status=None,
                        stream=None) -> None:
    """Redraw the bonus token of each sequence from softmax(logits/T) at the
    kept node (Philox4x32-10, inverse CDF); updates bonus and accepted_tokens."""
    _req(logits, "logits")
    B, N, V = logits.shape
    max_depth = accepted_nodes.shape[1] - 1
    _check(lib().medusa_sample_bonus(_p(logits), _dt(logits), _p(accept_len), _p(accepted_nodes),
                                     B, N, V, max_depth, float(temperature), int(seed),
                                     int(offset), _p(bonus), _p(accepted_tokens), _p(dev_status),
                                     _stream(stream)))


def medusa_topk_merge(vals, ids, rows: int, n_lists: int, list_len: int, row_stride: int,
                      list_stride: int, id_offsets, kmax: int, topk_ids, topk_vals,
                      stream=None) -> None:
    """Best kmax of n_lists candidate lists per row (see include/medusa.h)."""
    _req(vals, "vals")
    _req(ids, "ids")
    _check(lib().medusa_topk_merge(_p(vals), _p(ids), rows, n_lists, list_len, int(row_stride),
                                   int(list_stride), _p(id_offsets), kmax, _p(topk_ids),
                                   _p(topk_vals), _stream(stream)))


def medusa_verify_records_workspace_size(B: int, N: int, V_shard: int) -> int:
    return int(lib().medusa_verify_records_workspace_size(B, N, V_shard))


def medusa_verify_records(logits, cand_ids, tree: Tree, v_offset: int, records, cand_logit,
                          mode: int = MEDUSA_ACCEPT_GREEDY, temperature: float = 1.0, ws=None,
                          dev_status=None, stream=None) -> None:
    """This vocabulary shard's row records ([B*N, 4] float32 view of
    medusa_row_record_t) and candidate logits ([B*N] float32)."""
    _req(logits, "logits")
    B, N, Vs = logits.shape
    if ws is None:
        ws = workspace(medusa_verify_records_workspace_size(B, N, Vs), logits.device)
    ct = tree.c()
    _check(lib().medusa_verify_records(_p(logits), _dt(logits), _p(cand_ids), ctypes.byref(ct), B,
                                       Vs, v_offset, mode, float(temperature), _p(records),
                                       _p(cand_logit), _p(ws), ws.numel(), _p(dev_status),
                                       _stream(stream)))


def medusa_verify_from_records(records, cand_logit, cand_ids, tree: Tree, V: int, accept_len,
                               accepted_nodes, accepted_tokens, bonus,
                               mode: int = MEDUSA_ACCEPT_GREEDY, temperature: float = 1.0,
                               eps: float = 0.09, delta: float = 0.3, dev_status=None,
                               stream=None) -> None:
    """Verification from G shards' records [G, B*N, 4] and the candidate
    logits maximised over the shards [B*N] (typical only)."""
    _req(records, "records")
    G = records.shape[0]
    B = cand_ids.shape[0]
    ct = tree.c()
    _check(lib().medusa_verify_from_records(_p(records), G, _p(cand_logit), _p(cand_ids),
                                            ctypes.byref(ct), B, V, mode, float(temperature),
                                            float(eps), float(delta), _p(accept_len),
                                            _p(accepted_nodes), _p(accepted_tokens), _p(bonus),
                                            _p(dev_status), _stream(stream)))


def medusa_wait_flag(flag, value: int, budget_cycles: int, dev_status, stream=None) -> None:
    """Run the library's bounded flag wait on ``flag`` (device int32): returns
    once *flag == value, or writes MEDUSA_ERR_TIMEOUT into dev_status after
    budget_cycles SM clock cycles (<= 0: the library's own bound)."""
    _req(flag, "flag")
    _check(lib().medusa_wait_flag(_p(flag), int(value), int(budget_cycles), _p(dev_status),
                                  _stream(stream)))
