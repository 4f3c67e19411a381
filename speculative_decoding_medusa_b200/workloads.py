"""Seeded synthetic inputs for the Medusa decode-verify step.

This module only draws inputs: random tensors, tree shapes and the synthetic
verify logits.  It holds none of the method's arithmetic (no head, no top-k,
no attention, no acceptance rule), so that both the CUDA path and the CPU
oracle can be fed from it without sharing any computation.

Workload shapes restate the five configurations the decode-verify step is
measured on (Tiny, Vicuna-7B-shaped, Llama-3-8B-shaped, Llama-3-70B-shaped
with a dense tree, and long context).  Where the pages leave a choice open the
plainest reading is taken:

* weights ~ N(0, 0.02) drawn in fp32 and rounded to the compute dtype, the
  hidden state ~ N(0, 1) (the glossary's code draws it with ``torch.randn``),
  bias ~ N(0, 0.02); the zero-init variant sets W1 = 0, b1 = 0 and
  W2 = lm_head ("Medusa Heads" glossary, "Comment les têtes prédisent les
  tokens suivants");
* the sparse tree is grown greedily from seeded per-depth "accuracies" (the
  glossary's "Attention arborescente et acceptation" builds its 64-node tree
  from the most accurate combinations; the real accuracies need trained heads,
  so seeded stand-ins are used);
* verify logits are N(0, 1) rows in which, for each non-leaf node and with a
  fixed probability, one child's candidate token is lifted to ``rowmax + 1``
  so that the base model "agrees" with that child.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

# ----------------------------------------------------------------------------
# Workload definitions
# ----------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int            # sequences in the batch
    d: int            # hidden size
    V: int            # vocabulary size
    K: int            # Medusa heads
    kmax: int         # top-k width kept per head
    tree: str         # "cartesian:<w1>,<w2>,..." | "sparse" | "dense:<w>,<w>,..."
    N: int            # tree nodes, root included
    Hq: int
    Hkv: int
    dh: int
    ctx_lo: int       # prefix length range (inclusive); equal for fixed context
    ctx_hi: int
    dtype: str        # "bf16" or "f32"
    accept: str       # "greedy" or "typical"
    p_match: float    # probability that a non-leaf's argmax is forced onto a child
    temperature: float = 1.0
    eps: float = 0.09
    delta: float = 0.3
    max_depth: int = 5

    @property
    def cap(self) -> int:
        """Cache slots per (sequence, kv head): longest prefix plus the tree."""
        return self.ctx_hi + self.N


WORKLOADS: Dict[str, Workload] = {
    # batch 1, hidden 256, vocab 1000, 3 heads, fp32; Cartesian top-2 x top-3
    "tiny": Workload("tiny", B=1, d=256, V=1000, K=3, kmax=3,
                     tree="cartesian:2,3", N=9, Hq=4, Hkv=4, dh=64,
                     ctx_lo=128, ctx_hi=128, dtype="f32", accept="greedy",
                     p_match=0.6, max_depth=2),
    # batch 1, hidden 4096, vocab 32000, 5 heads bf16, 64-node sparse tree
    "vicuna7b": Workload("vicuna7b", B=1, d=4096, V=32000, K=5, kmax=10,
                         tree="sparse", N=64, Hq=32, Hkv=32, dh=128,
                         ctx_lo=2048, ctx_hi=2048, dtype="bf16",
                         accept="greedy", p_match=0.6, max_depth=5),
    # batch 8, hidden 4096, vocab 128256, 4 heads, GQA 32/8, ragged 4k..8k
    "llama3_8b": Workload("llama3_8b", B=8, d=4096, V=128256, K=4, kmax=10,
                          tree="sparse", N=64, Hq=32, Hkv=8, dh=128,
                          ctx_lo=4096, ctx_hi=8192, dtype="bf16",
                          accept="greedy", p_match=0.6, max_depth=4),
    # batch 4, hidden 8192, dense 256-node BFS prefix of the (4,4,4,4) tree,
    # typical acceptance at temperature 0.7
    "llama3_70b": Workload("llama3_70b", B=4, d=8192, V=128256, K=4, kmax=4,
                           tree="dense:4,4,4,4", N=256, Hq=64, Hkv=8, dh=128,
                           ctx_lo=4096, ctx_hi=4096, dtype="bf16",
                           accept="typical", p_match=0.5, temperature=0.7,
                           eps=0.09, delta=0.3, max_depth=4),
    # batch 32, Llama-3-8B shape, 32k context (tree size swept 16/64/128)
    "long": Workload("long", B=32, d=4096, V=128256, K=4, kmax=10,
                     tree="sparse", N=64, Hq=32, Hkv=8, dh=128,
                     ctx_lo=32768, ctx_hi=32768, dtype="bf16",
                     accept="greedy", p_match=0.6, max_depth=4),
}


def scaled(w: Workload, **over) -> Workload:
    """A copy of ``w`` with some fields replaced (used for small parity cases)."""
    return dataclasses.replace(w, **over)


# ----------------------------------------------------------------------------
# Seeded random draws
# ----------------------------------------------------------------------------

_TORCH_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPES[name]


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7_919) % (2 ** 63))
    return g


def randn(shape: Sequence[int], seed: int, stream: int, std: float = 1.0,
          dtype: str = "f32", device="cpu") -> torch.Tensor:
    """N(0, std^2) draw in fp32, rounded to ``dtype``.  Deterministic in
    (seed, stream, device)."""
    g = _gen(seed, stream, device)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch_dtype(dtype))


def randint(lo: int, hi: int, shape: Sequence[int], seed: int, stream: int,
            device="cpu") -> torch.Tensor:
    """Integers uniform in [lo, hi] inclusive, int32."""
    g = _gen(seed, stream, device)
    return torch.randint(lo, hi + 1, tuple(shape), generator=g,
                         dtype=torch.int64, device=device).to(torch.int32)


# ----------------------------------------------------------------------------
# Tree shapes (node lists only; the mask, positions and paths that follow from
# them are computed by the method, not here)
# ----------------------------------------------------------------------------


@dataclasses.dataclass
class TreeSpec:
    parent: np.ndarray   # int32 [N]; parent[0] = -1; parent[i] < i
    depth: np.ndarray    # int32 [N]; depth[0] = 0
    rank: np.ndarray     # int32 [N]; rank of the node within its head's top-k
    paths: List[Tuple[int, ...]]  # rank tuple of each node (root = ())

    @property
    def n_nodes(self) -> int:
        return int(self.parent.shape[0])

    @property
    def max_depth(self) -> int:
        return int(self.depth.max()) if self.depth.size else 0

    @property
    def n_leaves(self) -> int:
        has_child = np.zeros(self.n_nodes, dtype=bool)
        has_child[self.parent[1:]] = True
        return int((~has_child).sum())


def _spec_from_paths(paths: List[Tuple[int, ...]]) -> TreeSpec:
    """Order rank tuples breadth-first (depth, then lexicographic) and link
    each node to its parent."""
    paths = sorted(set(paths), key=lambda p: (len(p), p))
    assert paths[0] == (), "the root must be present"
    index = {p: i for i, p in enumerate(paths)}
    n = len(paths)
    parent = np.full(n, -1, dtype=np.int32)
    depth = np.zeros(n, dtype=np.int32)
    rank = np.zeros(n, dtype=np.int32)
    for i, p in enumerate(paths):
        depth[i] = len(p)
        if p:
            parent[i] = index[p[:-1]]  # KeyError if a parent is missing
            rank[i] = p[-1]
    return TreeSpec(parent, depth, rank, paths)


def cartesian_tree(widths: Sequence[int], n_nodes: Optional[int] = None) -> TreeSpec:
    """Full Cartesian-product tree: depth t holds every combination of the top
    ``widths[0]`` x ... x ``widths[t-1]`` ranks.  With ``n_nodes`` only the
    first nodes in breadth-first order are kept."""
    paths: List[Tuple[int, ...]] = [()]
    frontier: List[Tuple[int, ...]] = [()]
    for w in widths:
        frontier = [p + (r,) for p in frontier for r in range(w)]
        paths.extend(frontier)
    paths.sort(key=lambda p: (len(p), p))
    if n_nodes is not None:
        paths = paths[:n_nodes]
    return _spec_from_paths(paths)


def limits_tree(n_nodes: int, depth: int, kmax: int) -> TreeSpec:
    """A tree at the size limits: the chain of rank-0 nodes down to ``depth``,
    then, breadth-first, every other rank 1..kmax-1 under each chain node,
    until ``n_nodes`` nodes.  The deepest node and the largest rank are both
    present whenever n_nodes >= depth + kmax."""
    chain = [tuple([0] * t) for t in range(depth + 1)]
    rest = [tuple([0] * (t - 1)) + (r,) for t in range(1, depth + 1) for r in range(1, kmax)]
    rest.sort(key=lambda p: (len(p), p))
    return _spec_from_paths(chain + rest[: n_nodes - len(chain)])


def sparse_tree(n_nodes: int, n_heads: int, topk: int, seed: int,
                max_depth: int = 5) -> TreeSpec:
    """Seeded stand-in for the accuracy-driven sparse tree.

    Per depth t (1..min(n_heads, max_depth)) draw ``topk`` scores U(0, 1),
    sort them descending and scale by 0.8**t.  Grow from the root, each time
    adding the frontier node whose product of scores along its path is the
    largest (ties: lexicographically smallest rank tuple), until ``n_nodes``
    nodes.  Trees of different sizes from one seed are nested prefixes of one
    growth order."""
    depth_max = min(n_heads, max_depth)
    rng = np.random.default_rng(seed)
    acc = np.sort(rng.uniform(0.0, 1.0, size=(depth_max, topk)), axis=1)[:, ::-1]
    acc = acc * (0.8 ** np.arange(1, depth_max + 1))[:, None]
    chosen: List[Tuple[int, ...]] = [()]
    score = {(): 1.0}
    frontier = {(r,): acc[0, r] for r in range(topk)}
    while len(chosen) < n_nodes and frontier:
        best = max(frontier.items(), key=lambda kv: (kv[1], tuple(-x for x in kv[0])))[0]
        chosen.append(best)
        score[best] = frontier.pop(best)
        if len(best) < depth_max:
            for r in range(topk):
                frontier[best + (r,)] = score[best] * acc[len(best), r]
    return _spec_from_paths(chosen)


def tree_for(w: Workload, seed: int = 0, n_nodes: Optional[int] = None) -> TreeSpec:
    n = w.N if n_nodes is None else n_nodes
    kind, _, arg = w.tree.partition(":")
    if kind == "cartesian":
        return cartesian_tree([int(x) for x in arg.split(",")])
    if kind == "dense":
        return cartesian_tree([int(x) for x in arg.split(",")], n_nodes=n)
    if kind == "sparse":
        return sparse_tree(n, w.K, w.kmax, seed, max_depth=w.max_depth)
    raise ValueError(w.tree)


def children_lists(spec: TreeSpec) -> List[List[int]]:
    ch: List[List[int]] = [[] for _ in range(spec.n_nodes)]
    for i in range(1, spec.n_nodes):
        ch[int(spec.parent[i])].append(i)
    return ch


# ----------------------------------------------------------------------------
# Inputs of each stage
# ----------------------------------------------------------------------------

# stream ids keep every tensor's draw independent of the others
_S_H, _S_W1, _S_B1, _S_W2, _S_LM = 1, 2, 3, 4, 5
_S_Q, _S_KN, _S_VN, _S_KC, _S_VC, _S_PL = 11, 12, 13, 14, 15, 16
_S_LOG, _S_PICK, _S_ROOT, _S_TOPK = 21, 22, 23, 24


def heads_inputs(w: Workload, seed: int = 0, device="cpu", zero_init: bool = False,
                 std: float = 0.02) -> Dict[str, torch.Tensor]:
    """h [B, d], W1 [K, d, d] (row = output feature), b1 [K, d], W2 [K, V, d]
    and, for the zero-init variant and Tiny, lm_head [V, d]."""
    dt = w.dtype
    out = {"h": randn((w.B, w.d), seed, _S_H, 1.0, dt, device)}
    lm = randn((w.V, w.d), seed, _S_LM, std, dt, device) if (zero_init or w.name == "tiny") else None
    if zero_init:
        out["W1"] = torch.zeros((w.K, w.d, w.d), dtype=torch_dtype(dt), device=device)
        out["b1"] = torch.zeros((w.K, w.d), dtype=torch_dtype(dt), device=device)
        out["W2"] = lm.unsqueeze(0).expand(w.K, w.V, w.d).contiguous()
    else:
        out["W1"] = torch.empty((w.K, w.d, w.d), dtype=torch_dtype(dt), device=device)
        out["W2"] = torch.empty((w.K, w.V, w.d), dtype=torch_dtype(dt), device=device)
        for k in range(w.K):  # one head at a time keeps the fp32 staging small
            out["W1"][k] = randn((w.d, w.d), seed, _S_W1 * 100 + k, std, dt, device)
            out["W2"][k] = randn((w.V, w.d), seed, _S_W2 * 100 + k, std, dt, device)
        out["b1"] = randn((w.K, w.d), seed, _S_B1, std, dt, device)
    if lm is not None:
        out["lm_head"] = lm
    return out


def prefix_lengths(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    if w.ctx_lo == w.ctx_hi:
        return torch.full((w.B,), w.ctx_lo, dtype=torch.int32, device=device)
    return randint(w.ctx_lo, w.ctx_hi, (w.B,), seed, _S_PL, device)


def attention_inputs(w: Workload, seed: int = 0, device="cpu",
                     n_nodes: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """q [B, N, Hq, dh], k_new / v_new [B, N, Hkv, dh], caches Kc / Vc
    [B, Hkv, cap, dh] (slots past each prefix hold noise that must not be
    read), prefix_len [B]."""
    n = w.N if n_nodes is None else n_nodes
    dt = "bf16" if w.dtype == "bf16" else "f32"
    cap = w.ctx_hi + n
    return {
        "q": randn((w.B, n, w.Hq, w.dh), seed, _S_Q, 1.0, dt, device),
        "k_new": randn((w.B, n, w.Hkv, w.dh), seed, _S_KN, 1.0, dt, device),
        "v_new": randn((w.B, n, w.Hkv, w.dh), seed, _S_VN, 1.0, dt, device),
        "Kc": randn((w.B, w.Hkv, cap, w.dh), seed, _S_KC, 1.0, dt, device),
        "Vc": randn((w.B, w.Hkv, cap, w.dh), seed, _S_VC, 1.0, dt, device),
        "prefix_len": prefix_lengths(w, seed, device),
    }


def random_root_tokens(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    return randint(0, w.V - 1, (w.B,), seed, _S_ROOT, device)


def random_topk_ids(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """Distinct token ids per (sequence, head): a stand-in top-k list for
    stages fed without running the heads."""
    g = _gen(seed, _S_TOPK, "cpu")
    ids = torch.stack([torch.randperm(w.V, generator=g)[: w.kmax]
                       for _ in range(w.B * w.K)]).view(w.B, w.K, w.kmax)
    return ids.to(torch.int32).to(device)


def verify_logits(w: Workload, spec: TreeSpec, cand_ids: torch.Tensor, seed: int = 0,
                  device="cpu", dtype: Optional[str] = None, attempt: int = 0) -> torch.Tensor:
    """Synthetic base-model logits at every tree node, [B, N, V].

    Rows are N(0, 1).  For each non-leaf node, with probability ``p_match``
    one child is picked uniformly and its candidate token's logit is set to
    the row maximum plus one, so that the row's unique argmax is that child's
    token.  ``attempt`` shifts the seed (used to redraw a whole set)."""
    dt = dtype or w.dtype
    B, N = cand_ids.shape
    logits = randn((B, N, w.V), seed + 7777 * attempt, _S_LOG, 1.0, "f32", device)
    rng = np.random.default_rng(seed * 31 + 17 + attempt)
    ch = children_lists(spec)
    cand = cand_ids.to("cpu").numpy()
    rows_b, rows_i, cols = [], [], []
    for b in range(B):
        for i in range(N):
            if not ch[i]:
                continue
            u = rng.uniform()
            c = ch[i][int(rng.integers(len(ch[i])))]
            if u < w.p_match:
                rows_b.append(b)
                rows_i.append(i)
                cols.append(int(cand[b, c]))
    if rows_b:
        rb = torch.tensor(rows_b, device=device)
        ri = torch.tensor(rows_i, device=device)
        rc = torch.tensor(cols, device=device)
        rowmax = logits[rb, ri].max(dim=-1).values
        logits[rb, ri, rc] = rowmax + 1.0
    return logits.to(torch_dtype(dt))


_S_HID, _S_LMH = 31, 32


def lmhead_inputs(w: Workload, spec: TreeSpec, cand_ids: torch.Tensor, seed: int = 0,
                  device="cpu", attempt: int = 0, plant: float = 8.0,
                  noise: float = 1.0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Synthetic tree-node hidden states and lm_head, bf16.

    lm_head [V, d] rows are N(0, 1/d) (unit length on average); hidden
    [B, N, d] entries are N(0, noise^2), so unplanted scores are about
    N(0, noise^2).  For each non-leaf node, with
    probability ``p_match`` one child is picked uniformly and ``plant`` times
    the lm_head row of its candidate token is added to the node's hidden
    state, so that this token's score stands about ``plant`` above the rest.
    ``attempt`` shifts the seed (used to redraw a whole set)."""
    B, N = cand_ids.shape
    s = seed + 7919 * attempt
    lm = randn((w.V, w.d), s, _S_LMH, 1.0 / math.sqrt(w.d), "f32", device)
    hid = randn((B, N, w.d), s, _S_HID, noise, "f32", device)
    rng = np.random.default_rng(seed * 37 + 5 + attempt)
    ch = children_lists(spec)
    cand = cand_ids.to("cpu").numpy()
    for b in range(B):
        for i in range(N):
            if not ch[i]:
                continue
            u = rng.uniform()
            c = ch[i][int(rng.integers(len(ch[i])))]
            if u < w.p_match:
                hid[b, i] += plant * lm[int(cand[b, c])]
    return hid.to(torch.bfloat16), lm.to(torch.bfloat16)


class SyntheticBaseModel:
    """Stand-in for the base model's forward over the tree, whose transformer
    layers are outside this library: it only produces the tree nodes' last
    hidden states, on the device, from the step's candidate tokens.

    Hidden states are a fixed N(0, noise^2) draw; at step r, each non-leaf
    node is, with probability ``p_match``, given ``plant`` times the lm_head
    row of one (pre-drawn) child's candidate token, so that the verification
    accepts that child.  All picks are drawn up front, so forward() is a few
    device tensor ops that a CUDA graph can capture."""

    def __init__(self, w: Workload, spec: TreeSpec, lm_head: torch.Tensor, steps: int,
                 seed: int = 0, device="cuda", plant: float = 8.0, noise: float = 1.0):
        B, N = w.B, spec.n_nodes
        self.B, self.N, self.d, self.plant = B, N, w.d, plant
        self.lm = lm_head
        self.noise = randn((B, N, w.d), seed, _S_HID, noise, "f32", device)
        rng = np.random.default_rng(seed * 41 + 3)
        ch = children_lists(spec)
        pick = np.zeros((steps, B, N), dtype=np.int64)
        on = np.zeros((steps, B, N, 1), dtype=np.float32)
        for r in range(steps):
            for b in range(B):
                for n in range(N):
                    if ch[n]:
                        pick[r, b, n] = ch[n][int(rng.integers(len(ch[n])))]
                        on[r, b, n, 0] = plant if rng.uniform() < w.p_match else 0.0
        self.pick = torch.from_numpy(pick).to(device)
        self.on = torch.from_numpy(on).to(device)
        self.tmp = torch.empty(B, N, w.d, dtype=torch.float32, device=device)
        self.out = torch.empty(B, N, w.d, dtype=torch.bfloat16, device=device)

    def forward(self, cand_ids: torch.Tensor, r: int) -> torch.Tensor:
        tok = torch.gather(cand_ids.long(), 1, self.pick[r])
        rows = self.lm.index_select(0, tok.reshape(-1)).view(self.B, self.N, self.d)
        torch.addcmul(self.noise, rows.float(), self.on[r], out=self.tmp)
        self.out.copy_(self.tmp)
        return self.out
