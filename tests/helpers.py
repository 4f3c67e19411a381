"""Shared helpers of the GPU parity tests: tolerances, comparisons and input
marshalling between torch tensors and the oracle's fp64 numpy arrays."""
import math

import numpy as np
import torch

from oracle import medusa_oracle as O

# tolerances of the decode-verify step (bf16 inputs, fp32 accumulation)
LOGIT_MAX_ABS = 2e-2      # head logits and attention outputs, max-abs
ATTN_REL_L2 = 1e-3        # attention outputs, relative L2 (fp32 output)
TOPK_GAP = 1e-2           # top-k ids must match where the oracle's gap exceeds this
TYPICAL_LOG_MARGIN = 1e-3  # typical-acceptance inputs keep |ln p - ln thr| above this


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def i64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").numpy().astype(np.int64)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def check_topk(gpu_ids: np.ndarray, gpu_vals: np.ndarray, z: np.ndarray, kmax: int) -> None:
    """gpu_ids/vals [..., kmax] against oracle logits z [..., V].

    For every prefix length j whose oracle gap z_(j) - z_(j+1) exceeds
    TOPK_GAP the GPU's first j ids must be the oracle's top-j set; every
    returned value must be within LOGIT_MAX_ABS of the oracle logit of that id,
    values must be non-increasing and ids distinct."""
    ref_ids, ref_vals = O.topk(z, kmax + 1)
    flat_ids = gpu_ids.reshape(-1, kmax)
    flat_vals = gpu_vals.reshape(-1, kmax)
    rids = ref_ids.reshape(-1, kmax + 1)
    rvals = ref_vals.reshape(-1, kmax + 1)
    zz = z.reshape(-1, z.shape[-1])
    checked = 0
    for r in range(flat_ids.shape[0]):
        ids = flat_ids[r]
        assert len(set(ids.tolist())) == kmax, f"row {r}: duplicate ids {ids}"
        assert np.all(np.diff(flat_vals[r]) <= 0), f"row {r}: values not sorted"
        np.testing.assert_allclose(flat_vals[r], zz[r, ids], rtol=0, atol=LOGIT_MAX_ABS)
        for j in range(1, kmax + 1):
            if rvals[r, j - 1] - rvals[r, j] > TOPK_GAP:
                assert set(ids[:j].tolist()) == set(rids[r, :j].tolist()), \
                    f"row {r}: top-{j} set differs: gpu {ids[:j]} oracle {rids[r, :j]}"
                checked += 1
    assert checked > 0


def oracle_head_logits_chunked(h, W1, b1, W2, rows: int = 16384) -> np.ndarray:
    """Oracle head logits for large vocabularies: W2 is widened to fp64 a slice
    of rows at a time (the oracle function itself is called per slice)."""
    hh = f64(h)
    K, V, d = W2.shape
    W1d = f64(W1)
    b1d = f64(b1)
    out = np.empty((hh.shape[0], K, V))
    for k in range(K):
        for v0 in range(0, V, rows):
            w2 = f64(W2[k:k + 1, v0:v0 + rows])
            out[:, k:k + 1, v0:v0 + rows] = O.head_logits(hh, W1d[k:k + 1], b1d[k:k + 1], w2)
    return out
