"""CPU oracle for one Medusa decode-verify step (fp64, numpy).

TEST INFRASTRUCTURE.  This module is the plain, slow, obviously correct
statement of what the decode-verify path computes.  Only the test suite, the
package smoke check and the benchmark's CPU-baseline leg may import it; the
product path never calls it and shares no code with it.

Sources (web pages on Medusa; page title, then section):
  [GLOSS-HEADS]  "Medusa Heads" glossary, section "Comment les têtes prédisent
                 les tokens suivants" — head = one feed-forward layer with SiLU
                 and a residual connection, then a projection to the
                 vocabulary; W1/b1 start at zero and W2 as a copy of lm_head,
                 so a fresh head reproduces the base model's next-token logits;
                 head k reads the last hidden state and targets t + k + 1.
  [GLOSS-TREE]   same page, "Attention arborescente et acceptation" — top
                 choices of the heads combine into candidate continuations
                 (top-2 of head 1 x top-3 of head 2 = six candidates sharing
                 prefixes); every candidate token is appended to the input and
                 an attention mask lets each token see only its ancestors in
                 the tree; the longest branch the model agrees with is kept;
                 head 2 proposes the same tokens under every head-1 branch; a
                 64-node sparse tree beats a 256-node dense one; greedy
                 acceptance keeps a candidate equal to the model's first
                 choice, typical acceptance keeps one whose base-model
                 probability exceeds an entropy-linked threshold.
  [DECODE-DEEP]  "Medusa Decoding Heads" overview, "Diepe duik" — greedy
                 verification is lossless: the accepted text is exactly what
                 plain greedy decoding produces.
  [DEPLOY-PT]    "Medusa no contexto de LLMs", "o que significa medusa na
                 prática de deploy" — an accepted candidate enters the
                 sequence without another full pass; on rejection the
                 conventionally generated token is used.
  [ABSTRACT]     "Medusa: Simple LLM Inference Acceleration Framework with
                 Multiple Decoding Heads", abstract — tree-based attention
                 verifies several candidate continuations in one decoding step.

Readings taken where the pages are silent are stated at each function.  The
typical-acceptance threshold min(eps, delta * exp(-H(p))) is not printed on
the pages (they only say "a threshold tied to the entropy"); it is the formula
this build's workload statement fixes, with a strict ">" from the glossary's
"dépasse".

Every function takes numpy arrays already widened to float64 (integers as
int64/int32) and returns new arrays; nothing is modified in place.
"""
from __future__ import annotations

import itertools
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# Stage 1: Medusa heads and top-k                                [GLOSS-HEADS]
# ---------------------------------------------------------------------------


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) = x / (1 + e^-x)."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def head_logits(h: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """Logits of every Medusa head for every sequence.

    h [B, d]; W1 [K, d, d] with W1[k][j, :] the weights of output feature j
    (a Linear layer's layout); b1 [K, d]; W2 [K, V, d] (no bias).
    Head k: y = h + SiLU(W1_k h + b1_k);  z_k = W2_k y.      [GLOSS-HEADS]
    Returns z [B, K, V] in fp64."""
    h = np.asarray(h, dtype=np.float64)
    B, d = h.shape
    K, V, _ = W2.shape
    z = np.empty((B, K, V), dtype=np.float64)
    for k in range(K):
        u = h @ np.asarray(W1[k], np.float64).T + np.asarray(b1[k], np.float64)
        y = h + silu(u)
        z[:, k, :] = y @ np.asarray(W2[k], np.float64).T
    return z


def lm_head_logits(h: np.ndarray, lm_head: np.ndarray) -> np.ndarray:
    """Base model's next-token logits lm_head(h) [B, V] (Linear, no bias)."""
    return np.asarray(h, np.float64) @ np.asarray(lm_head, np.float64).T


def topk(z: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Top-k along the last axis: values descending, equal values by
    ascending index.  Returns (ids int32, values fp64), each [..., k]."""
    z = np.asarray(z, dtype=np.float64)
    flat = z.reshape(-1, z.shape[-1])
    ids = np.empty((flat.shape[0], k), dtype=np.int32)
    for r in range(flat.shape[0]):
        order = np.lexsort((np.arange(flat.shape[1]), -flat[r]))
        ids[r] = order[:k]
    vals = np.take_along_axis(flat, ids.astype(np.int64), axis=1)
    return ids.reshape(z.shape[:-1] + (k,)), vals.reshape(z.shape[:-1] + (k,))


# ---------------------------------------------------------------------------
# Stage 2: candidate tree                                          [GLOSS-TREE]
# ---------------------------------------------------------------------------


def tree_build(parent: np.ndarray, depth: np.ndarray, rank: np.ndarray,
               root_tok: np.ndarray, topk_ids: np.ndarray, prefix_len: np.ndarray
               ) -> Dict[str, np.ndarray]:
    """Candidate ids, position ids, ancestor mask and retrieve paths.

    Readings: node 0 is the root and carries the base model's own next token
    (an input); node i at depth t >= 1 carries rank[i] of head t's top-k — the
    same list under every branch [GLOSS-TREE]; the node's position is the
    sequence's prefix length plus its depth; a node attends to its ancestors
    and to itself (the causal convention); a retrieve path lists the nodes
    from the root to one leaf, leaves in node order, padded with -1.

    parent/depth/rank [N] (parent[0] = -1); root_tok [B]; topk_ids [B, K, kmax];
    prefix_len [B].  Returns cand [B, N], pos [B, N], mask [N, ceil(N/32)]
    uint32 (bit j of word j//32 of row i set iff j is i or an ancestor of i),
    retrieve [P, Dmax+1]."""
    parent = np.asarray(parent, np.int64)
    depth = np.asarray(depth, np.int64)
    rank = np.asarray(rank, np.int64)
    N = parent.shape[0]
    B = len(root_tok)
    cand = np.zeros((B, N), dtype=np.int32)
    pos = np.zeros((B, N), dtype=np.int32)
    for b in range(B):
        for i in range(N):
            if i == 0:
                cand[b, i] = root_tok[b]
            else:
                cand[b, i] = topk_ids[b, depth[i] - 1, rank[i]]
            pos[b, i] = prefix_len[b] + depth[i]
    words = (N + 31) // 32
    mask = np.zeros((N, words), dtype=np.uint32)
    for i in range(N):
        j = i
        while j >= 0:
            mask[i, j // 32] |= np.uint32(1 << (j % 32))
            j = parent[j]
    has_child = [False] * N
    for i in range(1, N):
        has_child[parent[i]] = True
    dmax = int(depth.max())
    paths: List[List[int]] = []
    for i in range(N):
        if not has_child[i]:
            path = []
            j = i
            while j >= 0:
                path.append(j)
                j = parent[j]
            path.reverse()
            paths.append(path + [-1] * (dmax + 1 - len(path)))
    retrieve = np.array(paths, dtype=np.int32).reshape(len(paths), dmax + 1)
    return {"cand": cand, "pos": pos, "mask": mask, "retrieve": retrieve}


def tree_from_accuracies(acc: np.ndarray, n_nodes: int, max_depth: int) -> Dict[str, np.ndarray]:
    """The sparse tree of the most accurate combinations.

    [GLOSS-TREE]: a sparse tree built from the most accurate combinations of
    the heads' top choices beats a dense one.  Reading: acc[t-1][r] is the
    probability that head t's rank-r token is the base model's choice (one
    rank at most is right, heads independent), so a node with rank path
    (r1..rt) is accepted with probability prod acc[i-1][r_i], and a tree's
    expected accept length is the sum of that over its non-root nodes.  The
    tree keeps the n_nodes - 1 rank paths of depth <= max_depth with the
    largest products (equal products: lexicographically smaller path first,
    so a prefix precedes its extensions), plus the root.  Node order: by
    depth, then lexicographic rank path (parents precede children).

    Written as the definition: every path of depth <= max_depth is scored and
    sorted.  acc [K, kmax] with values in [0, 1].  Returns parent, depth, rank
    [N] int32 and the expected accept length."""
    acc = np.asarray(acc, np.float64)
    K, kmax = acc.shape
    D = min(K, max_depth)
    scored = []
    for t in range(1, D + 1):
        for path in itertools.product(range(kmax), repeat=t):
            prob = 1.0
            for i, r in enumerate(path):
                prob *= acc[i, r]
            scored.append((-prob, path))
    scored.sort()
    keep = [path for _, path in scored[:n_nodes - 1]]
    nodes = [()] + sorted(keep, key=lambda p: (len(p), p))
    index = {p: i for i, p in enumerate(nodes)}
    parent = np.array([-1] + [index[p[:-1]] for p in nodes[1:]], dtype=np.int32)
    depth = np.array([len(p) for p in nodes], dtype=np.int32)
    rank = np.array([0] + [p[-1] for p in nodes[1:]], dtype=np.int32)
    expected = float(sum(-s for s, _ in scored[:n_nodes - 1]))
    return {"parent": parent, "depth": depth, "rank": rank, "expected_accept_len": expected}


def mask_bit(mask: np.ndarray, i: int, j: int) -> bool:
    return bool((int(mask[i, j // 32]) >> (j % 32)) & 1)


# ---------------------------------------------------------------------------
# Stage 3: tree attention                                 [GLOSS-TREE, ABSTRACT]
# ---------------------------------------------------------------------------


def tree_attention(q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray,
                   Kc: np.ndarray, Vc: np.ndarray, prefix_len: np.ndarray,
                   mask: np.ndarray, scale: float) -> Dict[str, np.ndarray]:
    """Attention of every tree node over the cached prefix and its ancestors.

    The N tree tokens' keys/values are appended to each sequence's cache at
    slots prefix_len[b] + i; node i's query for head h then attends, with
    softmax(scale * q . k) weights, to slots [0, prefix_len[b]) and to slot
    prefix_len[b] + j for every j with mask bit (i, j) set, in ascending slot
    order.  Query head h reads kv head floor(h * Hkv / Hq) (grouped queries).

    q [B, N, Hq, dh]; k_new, v_new [B, N, Hkv, dh]; Kc, Vc [B, Hkv, cap, dh].
    Returns {"out": [B, N, Hq, dh], "Kc": updated copy, "Vc": updated copy}."""
    B, N, Hq, dh = q.shape
    Hkv = k_new.shape[2]
    Kc = np.array(Kc, dtype=np.float64, copy=True)
    Vc = np.array(Vc, dtype=np.float64, copy=True)
    out = np.zeros((B, N, Hq, dh), dtype=np.float64)
    for b in range(B):
        P = int(prefix_len[b])
        Kc[b, :, P:P + N, :] = np.transpose(k_new[b], (1, 0, 2))
        Vc[b, :, P:P + N, :] = np.transpose(v_new[b], (1, 0, 2))
        for i in range(N):
            slots = list(range(P)) + [P + j for j in range(N) if mask_bit(mask, i, j)]
            for hq in range(Hq):
                kv = hq * Hkv // Hq
                keys = Kc[b, kv, slots, :]
                vals = Vc[b, kv, slots, :]
                s = scale * (keys @ np.asarray(q[b, i, hq], np.float64))
                p = np.exp(s - s.max())
                out[b, i, hq] = (p / p.sum()) @ vals
    return {"out": out, "Kc": Kc, "Vc": Vc}


# ---------------------------------------------------------------------------
# Stage 4: verification and acceptance               [GLOSS-TREE, DEPLOY-PT]
# ---------------------------------------------------------------------------


def row_argmax(logits: np.ndarray) -> np.ndarray:
    """The base model's first choice at every node: index of the largest
    logit, the lowest index among equal maxima.  logits [B, N, V]."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int32)


def typical_log_margin(logits: np.ndarray, cand: np.ndarray, parent: np.ndarray,
                       temperature: float, eps: float, delta: float) -> np.ndarray:
    """ln p_parent(cand[c]) - ln thr_parent for every non-root node c.

    p = softmax(logits / T) at the parent node; H = -sum p ln p (nats);
    thr = min(eps, delta * exp(-H)).  The candidate passes iff p > thr, i.e.
    iff the returned margin is > 0.  Entry 0 (the root) is +inf.  When
    thr == 0 the margin is +inf.  [GLOSS-TREE]"""
    logits = np.asarray(logits, np.float64)
    B, N, V = logits.shape
    out = np.full((B, N), np.inf, dtype=np.float64)
    for b in range(B):
        stats = {}
        for c in range(1, N):
            i = int(parent[c])
            if i not in stats:
                zt = logits[b, i] / temperature
                m = zt.max()
                lse = m + math.log(np.exp(zt - m).sum())
                logp = zt - lse
                H = -float((np.exp(logp) * logp).sum())
                thr = min(eps, delta * math.exp(-H))
                stats[i] = (logp, thr)
            logp, thr = stats[i]
            if thr <= 0.0:
                out[b, c] = np.inf
            else:
                out[b, c] = float(logp[cand[b, c]]) - math.log(thr)
    return out


def accept(passes: np.ndarray, parent: np.ndarray, depth: np.ndarray, cand: np.ndarray,
           bonus_rows: np.ndarray, max_depth: int) -> Dict[str, np.ndarray]:
    """Keep the longest accepted branch.

    passes [B, N] bool: node c's candidate token passes the test at its parent.
    The root is always accepted; node c is accepted iff it passes and its
    parent is accepted.  The kept node is the deepest accepted node, the
    lowest index among equally deep ones.  The bonus token is the model's own
    choice at the kept node (the conventionally generated token
    [DEPLOY-PT]).  Outputs: accept_len [B] (candidates kept, root excluded),
    accepted_nodes [B, Dmax+1] (root first, -1 padded), accepted_tokens
    [B, Dmax+1] (kept candidates' tokens then the bonus token, -1 padded),
    bonus [B]."""
    B, N = passes.shape
    W = max_depth + 1
    accept_len = np.zeros(B, dtype=np.int32)
    nodes = np.full((B, W), -1, dtype=np.int32)
    toks = np.full((B, W), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    for b in range(B):
        ok = np.zeros(N, dtype=bool)
        ok[0] = True
        for c in range(1, N):  # parents precede children
            ok[c] = bool(passes[b, c]) and ok[int(parent[c])]
        best = 0
        for c in range(N):
            if ok[c] and depth[c] > depth[best]:
                best = c
        path = []
        j = best
        while j >= 0:
            path.append(j)
            j = int(parent[j])
        path.reverse()
        L = len(path) - 1
        accept_len[b] = L
        nodes[b, :L + 1] = path
        toks[b, :L] = [cand[b, n] for n in path[1:]]
        bonus[b] = bonus_rows[b, best]
        toks[b, L] = bonus[b]
    return {"accept_len": accept_len, "accepted_nodes": nodes,
            "accepted_tokens": toks, "bonus": bonus}


def verify_greedy(logits: np.ndarray, cand: np.ndarray, parent: np.ndarray,
                  depth: np.ndarray, max_depth: int) -> Dict[str, np.ndarray]:
    """Greedy acceptance: candidate c passes iff it equals the base model's
    first choice at its parent node.  [GLOSS-TREE]"""
    g = row_argmax(logits)
    B, N = cand.shape
    passes = np.zeros((B, N), dtype=bool)
    for b in range(B):
        for c in range(1, N):
            passes[b, c] = g[b, int(parent[c])] == cand[b, c]
    res = accept(passes, parent, depth, cand, g, max_depth)
    res["argmax"] = g
    return res


def verify_typical(logits: np.ndarray, cand: np.ndarray, parent: np.ndarray,
                   depth: np.ndarray, max_depth: int, temperature: float,
                   eps: float, delta: float) -> Dict[str, np.ndarray]:
    """Typical acceptance: candidate c passes iff its probability under the
    base model at its parent exceeds min(eps, delta * exp(-H)).  The bonus
    token is the most probable token at the kept node (a deterministic
    reading; sampling it is not part of this path).  [GLOSS-TREE]"""
    margin = typical_log_margin(logits, cand, parent, temperature, eps, delta)
    passes = margin > 0.0
    passes[:, 0] = True
    g = row_argmax(logits)
    res = accept(passes, parent, depth, cand, g, max_depth)
    res["argmax"] = g
    res["margin"] = margin
    return res


# ---------------------------------------------------------------------------
# Stage 5: KV compaction                                 [DEPLOY-PT, GLOSS-TREE]
# ---------------------------------------------------------------------------


def kv_compact(Kc: np.ndarray, Vc: np.ndarray, prefix_len: np.ndarray,
               accepted_nodes: np.ndarray, accept_len: np.ndarray
               ) -> Dict[str, np.ndarray]:
    """Keep only the kept branch in the cache.

    For j = 0..L (L = accept_len[b]), in ascending order, slot P + j takes the
    contents of slot P + accepted_nodes[b, j] (P = prefix_len[b]), every kv
    head, K and V; then P grows by L + 1.  compact_src [B, Dmax+1] lists the
    source slots, -1 padded.  Kc, Vc [B, Hkv, cap, dh]."""
    Kc = np.array(Kc, copy=True)
    Vc = np.array(Vc, copy=True)
    B = Kc.shape[0]
    W = accepted_nodes.shape[1]
    new_prefix = np.array(prefix_len, dtype=np.int32, copy=True)
    src = np.full((B, W), -1, dtype=np.int32)
    for b in range(B):
        P = int(prefix_len[b])
        L = int(accept_len[b])
        for j in range(L + 1):
            s = P + int(accepted_nodes[b, j])
            Kc[b, :, P + j, :] = Kc[b, :, s, :]
            Vc[b, :, P + j, :] = Vc[b, :, s, :]
            src[b, j] = s
        new_prefix[b] = P + L + 1
    return {"Kc": Kc, "Vc": Vc, "prefix_len": new_prefix, "compact_src": src}


# ---------------------------------------------------------------------------
# The whole step
# ---------------------------------------------------------------------------


def philox4x32_10(counter: Sequence[int], key: Sequence[int]) -> List[int]:
    """The Philox4x32-10 counter-based generator as published by Salmon,
    Moraes, Dror and Shaw ("Parallel Random Numbers: As Easy as 1, 2, 3",
    SC 2011): ten rounds of two 32x32 -> 64-bit multiplications with the
    multipliers 0xD2511F53 and 0xCD9E8D57, the high halves xored with the
    other counter words and the key, the key bumped by 0x9E3779B9 and
    0xBB67AE85 after each round.  counter: 4 words, key: 2 words."""
    c = [int(x) & 0xFFFFFFFF for x in counter]
    k = [int(x) & 0xFFFFFFFF for x in key]
    for rnd in range(10):
        p0 = 0xD2511F53 * c[0]
        p1 = 0xCD9E8D57 * c[2]
        hi0, lo0 = p0 >> 32, p0 & 0xFFFFFFFF
        hi1, lo1 = p1 >> 32, p1 & 0xFFFFFFFF
        c = [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]
        if rnd < 9:
            k = [(k[0] + 0x9E3779B9) & 0xFFFFFFFF, (k[1] + 0xBB67AE85) & 0xFFFFFFFF]
    return c


def bonus_uniform(seed: int, offset: int, b: int) -> float:
    """The uniform number of sequence b: the top 24 bits of the first Philox
    word for key (seed low, seed high) and counter (offset low, offset high,
    b, 0), as a multiple of 2^-24 in [0, 1)."""
    x = philox4x32_10([offset & 0xFFFFFFFF, (offset >> 32) & 0xFFFFFFFF, b, 0],
                      [seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF])[0]
    return (x >> 8) * 2.0 ** -24


def sample_bonus(logits: np.ndarray, accept_len: np.ndarray, accepted_nodes: np.ndarray,
                 temperature: float, seed: int, offset: int) -> np.ndarray:
    """A sampled bonus token: at the kept node, the first token whose
    cumulative probability under softmax(logits / T) exceeds the sequence's
    uniform number (inverse CDF).  [DEPLOY-PT]: the token the base model
    generates itself at the kept node - here drawn from its distribution
    rather than taken as its first choice.  logits [B, N, V]."""
    logits = np.asarray(logits, np.float64)
    B = logits.shape[0]
    out = np.zeros(B, dtype=np.int32)
    for b in range(B):
        kept = int(accepted_nodes[b, int(accept_len[b])])
        zt = logits[b, kept] / temperature
        p = np.exp(zt - zt.max())
        cdf = np.cumsum(p) / p.sum()
        u = bonus_uniform(seed, offset, b)
        out[b] = min(int(np.searchsorted(cdf, u, side="right")), logits.shape[2] - 1)
    return out


def next_step_inputs(node_hidden: np.ndarray, accept_len: np.ndarray,
                     accepted_nodes: np.ndarray, bonus: np.ndarray
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """Inputs of the next decode step after a verification.

    [GLOSS-TREE]: the accepted candidates enter the sequence; the heads of
    the next round read the base model's last hidden state, i.e. that of the
    last accepted node (the kept node), and the next round's first token is
    the base model's own choice there (the bonus token; [DEPLOY-PT]: the
    conventionally generated token).  node_hidden [B, N, d] -> (h_next
    [B, d], root_next [B])."""
    node_hidden = np.asarray(node_hidden)
    B = node_hidden.shape[0]
    kept = np.array([accepted_nodes[b, int(accept_len[b])] for b in range(B)], dtype=np.int64)
    h_next = np.stack([node_hidden[b, kept[b]] for b in range(B)])
    return h_next, np.asarray(bonus, dtype=np.int32).copy()


def lmhead_verify(hidden: np.ndarray, lm_head: np.ndarray, cand: np.ndarray,
                  parent: np.ndarray, depth: np.ndarray, max_depth: int,
                  accept_mode: str = "greedy", temperature: float = 1.0,
                  eps: float = 0.09, delta: float = 0.3) -> Dict[str, np.ndarray]:
    """Verification from the base model's last hidden states of the tree
    nodes instead of from materialised logits.

    The verify logits of node n of sequence b are lm_head(hidden[b, n])
    ([GLOSS-TREE]: one forward pass scores every node; [GLOSS-HEADS]: the
    base model's next-token distribution is lm_head of its last hidden
    state).  hidden [B, N, d], lm_head [V, d].  Returns the verify outputs
    plus the logits [B, N, V] (fp64)."""
    hidden = np.asarray(hidden, np.float64)
    B, N, d = hidden.shape
    logits = lm_head_logits(hidden.reshape(B * N, d), lm_head).reshape(B, N, -1)
    if accept_mode == "greedy":
        res = verify_greedy(logits, cand, parent, depth, max_depth)
    else:
        res = verify_typical(logits, cand, parent, depth, max_depth, temperature, eps, delta)
    res["logits"] = logits
    return res


def decode_verify_step(inp: Dict[str, np.ndarray], tree: Dict[str, np.ndarray],
                       kmax: int, accept_mode: str = "greedy", temperature: float = 1.0,
                       eps: float = 0.09, delta: float = 0.3,
                       head_logits_fn=None) -> Dict[str, np.ndarray]:
    """Stages 1-5 in order, on one batch.  ``inp`` holds h, W1, b1, W2,
    root_tok, q, k_new, v_new, Kc, Vc, prefix_len and the verify logits."""
    z = head_logits(inp["h"], inp["W1"], inp["b1"], inp["W2"])
    ids, vals = topk(z, kmax)
    tb = tree_build(tree["parent"], tree["depth"], tree["rank"], inp["root_tok"], ids,
                    inp["prefix_len"])
    dh = inp["q"].shape[-1]
    att = tree_attention(inp["q"], inp["k_new"], inp["v_new"], inp["Kc"], inp["Vc"],
                         inp["prefix_len"], tb["mask"], 1.0 / math.sqrt(dh))
    dmax = int(np.max(tree["depth"]))
    if accept_mode == "greedy":
        acc = verify_greedy(inp["logits"], tb["cand"], tree["parent"], tree["depth"], dmax)
    else:
        acc = verify_typical(inp["logits"], tb["cand"], tree["parent"], tree["depth"], dmax,
                             temperature, eps, delta)
    kv = kv_compact(att["Kc"], att["Vc"], inp["prefix_len"], acc["accepted_nodes"],
                    acc["accept_len"])
    return {"logits": z, "topk_ids": ids, "topk_vals": vals, **tb,
            "attn_out": att["out"], **acc, **kv}
