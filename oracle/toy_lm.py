"""A one-layer toy language model for the losslessness check (fp64).

TEST INFRASTRUCTURE (part of the oracle): only tests may use it.

"Medusa Decoding Heads" overview, "Diepe duik": because the base model itself
verifies the tree, greedy Medusa decoding is lossless — the accepted text is
exactly what plain greedy decoding would produce, in fewer steps.  This module
provides both sides of that statement for a tiny model:

* ``greedy_decode``: plain autoregressive decoding, one token per forward, with
  its own textbook causal attention (a library softmax over every earlier
  slot), and
* ``medusa_decode``: repeated decode-verify steps built from the oracle's tree
  build, tree attention, greedy acceptance and KV compaction.

The model: token embedding plus learned position embedding, one multi-head
attention block with a residual connection, then lm_head.  K/V of a token
depend only on the token and its position, so a correct compaction leaves the
cache bit-identical to the one plain decoding writes.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, List, Tuple

import numpy as np

from . import medusa_oracle as O


class ToyLM:
    def __init__(self, vocab: int = 48, d: int = 16, heads: int = 2, dh: int = 8,
                 max_pos: int = 256, seed: int = 0):
        rng = np.random.default_rng(seed)
        self.V, self.d, self.H, self.dh = vocab, d, heads, dh
        self.E = rng.standard_normal((vocab, d))
        self.Pe = 0.3 * rng.standard_normal((max_pos, d))
        s = 1.0 / math.sqrt(d)
        self.Wq = s * rng.standard_normal((heads * dh, d))
        self.Wk = s * rng.standard_normal((heads * dh, d))
        self.Wv = s * rng.standard_normal((heads * dh, d))
        self.Wo = s * rng.standard_normal((d, heads * dh))
        self.lm = rng.standard_normal((vocab, d))

    # one token at a time everywhere, so that both decoders run the very same
    # floating-point operations on the same (token, position)
    def embed(self, tok: int, pos: int) -> np.ndarray:
        return self.E[tok] + self.Pe[pos]

    def qkv(self, e: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        return ((self.Wq @ e).reshape(self.H, self.dh), (self.Wk @ e).reshape(self.H, self.dh),
                (self.Wv @ e).reshape(self.H, self.dh))

    def head_out(self, e: np.ndarray, att: np.ndarray) -> np.ndarray:
        """Residual block then lm_head: logits for the next token."""
        hidden = e + self.Wo @ att.reshape(-1)
        return self.lm @ hidden


def _causal_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Textbook attention of one query over every cached slot (all visible)."""
    from scipy.special import softmax
    out = np.empty_like(q)
    for h in range(q.shape[0]):
        w = softmax(scale * (K[h] @ q[h]))
        out[h] = w @ V[h]
    return out


def greedy_decode(m: ToyLM, prompt: List[int], n_new: int) -> Tuple[List[int], np.ndarray, np.ndarray]:
    """Plain greedy decoding.  Returns the generated tokens and the K/V cache
    [H, len, dh] of every token fed to the model."""
    scale = 1.0 / math.sqrt(m.dh)
    Ks: List[np.ndarray] = []
    Vs: List[np.ndarray] = []
    toks = list(prompt)
    out: List[int] = []
    nxt = None
    pos = 0
    while len(out) < n_new:
        feed = toks[pos]
        e = m.embed(feed, pos)
        q, k, v = m.qkv(e)
        Ks.append(k)
        Vs.append(v)
        att = _causal_attention(q, np.stack(Ks, 1), np.stack(Vs, 1), scale)
        logits = m.head_out(e, att)
        nxt = int(np.argmax(logits))
        pos += 1
        if pos >= len(toks):
            toks.append(nxt)
            out.append(nxt)
    return out, np.stack(Ks, 1), np.stack(Vs, 1)


def medusa_decode(m: ToyLM, prompt: List[int], n_new: int, parent: np.ndarray,
                  depth: np.ndarray, rank: np.ndarray, kmax: int,
                  propose: Callable[[int, int], np.ndarray],
                  cap: int = 256) -> Dict[str, object]:
    """Greedy Medusa decoding with the oracle's stages.

    ``propose(step, n_generated)`` returns the top-k lists [K, kmax] standing in
    for the heads' output at that step (any lists are valid: losslessness
    must hold whatever the heads propose).  The prompt is prefilled one token
    at a time; the first root token is the model's prediction after it."""
    scale = 1.0 / math.sqrt(m.dh)
    N = parent.shape[0]
    Kc = np.zeros((1, m.H, cap, m.dh))
    Vc = np.zeros((1, m.H, cap, m.dh))
    # prefill: plain decoding over the prompt fills the cache
    for p, t in enumerate(prompt):
        e = m.embed(t, p)
        q, k, v = m.qkv(e)
        Kc[0, :, p] = k
        Vc[0, :, p] = v
        att = _causal_attention(q, Kc[0, :, :p + 1], Vc[0, :, :p + 1], scale)
        logits = m.head_out(e, att)
    root = int(np.argmax(logits))
    prefix = np.array([len(prompt)], dtype=np.int32)
    out: List[int] = []
    accepted_per_step: List[int] = []
    step = 0
    while len(out) < n_new:
        ids = propose(step, len(out))[None]
        tb = O.tree_build(parent, depth, rank, np.array([root]), ids, prefix)
        cand, pos = tb["cand"], tb["pos"]
        q = np.zeros((1, N, m.H, m.dh))
        kn = np.zeros((1, N, m.H, m.dh))
        vn = np.zeros((1, N, m.H, m.dh))
        es = []
        for i in range(N):
            e = m.embed(int(cand[0, i]), int(pos[0, i]))
            es.append(e)
            q[0, i], kn[0, i], vn[0, i] = m.qkv(e)
        att = O.tree_attention(q, kn, vn, Kc, Vc, prefix, tb["mask"], scale)
        logits = np.stack([m.head_out(es[i], att["out"][0, i]) for i in range(N)])[None]
        acc = O.verify_greedy(logits, cand, parent, depth, int(depth.max()))
        kv = O.kv_compact(att["Kc"], att["Vc"], prefix, acc["accepted_nodes"], acc["accept_len"])
        Kc, Vc, prefix = kv["Kc"], kv["Vc"], kv["prefix_len"]
        L = int(acc["accept_len"][0])
        new = [root] + [int(t) for t in acc["accepted_tokens"][0, :L]]
        out.extend(new)
        accepted_per_step.append(L)
        root = int(acc["bonus"][0])
        step += 1
    return {"tokens": out[:n_new], "Kc": Kc, "Vc": Vc, "prefix_len": int(prefix[0]),
            "accepted_per_step": accepted_per_step, "steps": step}
