"""GPU: the sampled bonus token (Philox4x32-10 + inverse CDF at the kept node)
against the oracle's definition."""
import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from tests.helpers import f64

pytestmark = pytest.mark.gpu

CDF_TOL = 2e-5  # fp32 chunked scan vs fp64 cumulative sum, relative to the total


def _paths(rng, B, N, width):
    acc = rng.integers(0, width, size=B).astype(np.int32)
    nodes = np.full((B, width), -1, dtype=np.int32)
    for b in range(B):
        nodes[b, :acc[b] + 1] = np.sort(rng.choice(N, size=acc[b] + 1, replace=False))
    return acc, nodes


def _run(logits, acc, nodes, T, seed, offset):
    dev = "cuda"
    B = logits.shape[0]
    bonus = torch.full((B,), -5, dtype=torch.int32, device=dev)
    toks = torch.full((B, nodes.shape[1]), -5, dtype=torch.int32, device=dev)
    st = M.new_status()
    M.medusa_sample_bonus(logits.to(dev), torch.from_numpy(acc).to(dev),
                          torch.from_numpy(nodes).to(dev), bonus, toks, T, seed, offset,
                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return bonus.cpu().numpy(), toks.cpu().numpy()


@pytest.mark.parametrize("dtype,B,N,V,T,seed", [
    (torch.float32, 6, 9, 1000, 1.0, 1), (torch.bfloat16, 4, 64, 128256, 0.7, 2),
    (torch.bfloat16, 3, 17, 31, 2.0, 3), (torch.float32, 2, 5, 5000, 0.3, 4)])
def test_matches_oracle_inverse_cdf(dtype, B, N, V, T, seed):
    rng = np.random.default_rng(seed)
    g = torch.Generator().manual_seed(seed)
    logits = (torch.randn(B, N, V, generator=g) * 2.0).to(dtype)
    acc, nodes = _paths(rng, B, N, 4)
    z = f64(logits)
    exact = 0
    for offset in range(5):
        got, toks = _run(logits, acc, nodes, T, 1000 + seed, offset)
        ref = O.sample_bonus(z, acc, nodes, T, 1000 + seed, offset)
        for b in range(B):
            assert toks[b, acc[b]] == got[b]
            if got[b] == ref[b]:
                exact += 1
                continue
            # a u next to a boundary: the two tokens must be neighbours in the
            # cumulative distribution, with u within the tolerance of their border
            zt = z[b, nodes[b, acc[b]]] / T
            p = np.exp(zt - zt.max())
            cdf = np.cumsum(p) / p.sum()
            u = O.bonus_uniform(1000 + seed, offset, b)
            lo, hi = sorted((int(got[b]), int(ref[b])))
            assert np.all(p[lo + 1:hi] < CDF_TOL)
            assert abs(cdf[lo] - u) < CDF_TOL
    assert exact >= 0.9 * 5 * B


def test_uniform_row_and_frequencies():
    dev = "cuda"
    B, N, V = 1, 3, 8
    acc = np.zeros(B, dtype=np.int32)
    nodes = np.array([[0, -1]], dtype=np.int32)
    logits = torch.zeros(B, N, V)
    for off in range(16):
        got, _ = _run(logits, acc, nodes, 1.0, 5, off)
        assert got[0] == int(O.bonus_uniform(5, off, 0) * V)
    # empirical frequencies over many offsets follow softmax(z)
    z = torch.tensor([0.0, 1.0, 2.0, -1.0, 0.5, 3.0, -2.0, 1.5])
    logits = z.view(1, 1, V).repeat(1, N, 1)
    p = torch.softmax(z.double(), 0).numpy()
    counts = np.zeros(V)
    n_draws = 4000
    bonus = torch.zeros(B, dtype=torch.int32, device=dev)
    toks = torch.zeros(B, 2, dtype=torch.int32, device=dev)
    accd, nodesd, lg = (torch.from_numpy(acc).to(dev), torch.from_numpy(nodes).to(dev),
                        logits.to(dev))
    draws = torch.zeros(n_draws, dtype=torch.int32, device=dev)
    for off in range(n_draws):
        M.medusa_sample_bonus(lg, accd, nodesd, bonus, toks, 1.0, 77, off)
        draws[off] = bonus[0]
    counts = np.bincount(draws.cpu().numpy(), minlength=V)
    expected = p * n_draws
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 40.0  # 7 degrees of freedom: p ~ 1e-6 at 40


def test_bad_kept_node_is_reported():
    dev = "cuda"
    logits = torch.zeros(1, 4, 16, device=dev)
    st = M.new_status()
    M.medusa_sample_bonus(logits, torch.tensor([1], dtype=torch.int32, device=dev),
                          torch.tensor([[0, 9]], dtype=torch.int32, device=dev),
                          torch.zeros(1, dtype=torch.int32, device=dev),
                          torch.zeros(1, 2, dtype=torch.int32, device=dev), 1.0, 1, 0,
                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6
