"""Vocabulary-sharded heads and verification across the ranks of a
torch.distributed group (one GPU per rank, NCCL over NVLink in practice).

Each rank holds the W2 rows and the verify-logit columns of one contiguous
slice of the vocabulary.  The library computes every shard's top-k lists and
row records and merges them; this module only moves those few kilobytes
between ranks (one all-gather each, plus a max all-reduce of the candidate
logits for typical acceptance).  No collective touches the weights or the
logits, and no device buffer of another GPU is read by a kernel.

The exchanges run on the stream the library calls were enqueued on.  Over
NCCL they stay on the device; over gloo (host collectives) the few KB go
through host memory.
"""
from __future__ import annotations

import contextlib
from typing import List, Tuple

import torch
import torch.distributed as dist

from . import _lib as M


def shard_range(V: int, world: int, rank: int) -> Tuple[int, int]:
    """Tokens [v0, v1) of ``rank``: an even split, the first V % world ranks
    one token larger."""
    base, rem = divmod(V, world)
    v0 = rank * base + min(rank, rem)
    return v0, v0 + base + (1 if rank < rem else 0)


def shard_offsets(V: int, world: int) -> List[int]:
    return [shard_range(V, world, r)[0] for r in range(world)]


def _host_staged(t: torch.Tensor, group) -> bool:
    """A device tensor exchanged over a backend without device collectives
    (gloo gathers host tensors only) goes through host memory."""
    return t.is_cuda and dist.get_backend(group) != "nccl"


def gather_stacked(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's ``t`` in rank order (all-gather).

    Runs on the current stream: NCCL orders the collective after the work
    already queued there; a host-staged exchange copies ``t`` to the host
    with a copy that waits for that work."""
    world = dist.get_world_size(group)
    if _host_staged(t, group):
        h = t.to("cpu")
        parts = [torch.empty_like(h) for _ in range(world)]
        dist.all_gather(parts, h.contiguous(), group=group)
        return torch.stack(parts).to(t.device)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def max_over_ranks(t: torch.Tensor, group=None) -> torch.Tensor:
    """Element-wise maximum over the ranks, in place (current stream)."""
    if _host_staged(t, group):
        h = t.to("cpu")
        dist.all_reduce(h, op=dist.ReduceOp.MAX, group=group)
        t.copy_(h)
        return t
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def _on(stream):
    """Context making ``stream`` (if given) torch's current stream, so that
    the exchange is ordered after the library calls enqueued on it and the
    calls after the exchange are ordered after it."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


class ShardedHeads:
    """Heads + top-k with W2 split by vocabulary: local top-k on this rank's
    shard, all-gather of the [B*K, kmax] lists, merge with each shard's token
    offset (medusa_topk_merge)."""

    def __init__(self, *, B: int, d: int, V: int, K: int, kmax: int, group=None, device="cuda"):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.v0, self.v1 = shard_range(V, self.world, self.rank)
        self.B, self.K, self.kmax = B, K, kmax
        Vs = self.v1 - self.v0
        if kmax > Vs:
            raise ValueError("kmax larger than a vocabulary shard")
        i32 = dict(dtype=torch.int32, device=device)
        self.offsets = torch.tensor(shard_offsets(V, self.world), **i32)
        self.local_ids = torch.empty(B, K, kmax, **i32)
        self.local_vals = torch.empty(B, K, kmax, dtype=torch.float32, device=device)
        self.topk_ids = torch.empty(B, K, kmax, **i32)
        self.topk_vals = torch.empty(B, K, kmax, dtype=torch.float32, device=device)
        self.ws = M.workspace(M.medusa_heads_topk_workspace_size(B, d, Vs, K, kmax, M.MEDUSA_BF16),
                              device)
        self.status = torch.zeros(1, **i32)

    def run(self, h, W1, b1, W2_shard, stream=None):
        M.medusa_heads_topk(h, W1, b1, W2_shard, self.kmax, self.local_ids, self.local_vals, None,
                            self.ws, self.status, stream)
        with _on(stream):
            vals = gather_stacked(self.local_vals, self.group)
            ids = gather_stacked(self.local_ids, self.group)
        rows = self.B * self.K
        M.medusa_topk_merge(vals, ids, rows, self.world, self.kmax, self.kmax,
                            rows * self.kmax, self.offsets, self.kmax, self.topk_ids,
                            self.topk_vals, stream)
        return self.topk_ids, self.topk_vals


class ShardedVerify:
    """Verification with the verify logits split by vocabulary: this rank's
    row records and candidate logits, all-gather of the records, max
    all-reduce of the candidate logits (typical), then the acceptance."""

    def __init__(self, *, B: int, N: int, V: int, tree: M.Tree, accept: str = "greedy",
                 temperature: float = 1.0, eps: float = 0.09, delta: float = 0.3, group=None,
                 device="cuda"):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.v0, self.v1 = shard_range(V, self.world, self.rank)
        self.V, self.tree = V, tree
        self.mode = M.MEDUSA_ACCEPT_TYPICAL if accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
        self.temperature, self.eps, self.delta = temperature, eps, delta
        i32 = dict(dtype=torch.int32, device=device)
        W = tree.max_depth + 1
        self.records = torch.empty(B * N, 4, dtype=torch.float32, device=device)
        self.cand_logit = torch.empty(B * N, dtype=torch.float32, device=device)
        self.ws = M.workspace(M.medusa_verify_records_workspace_size(B, N, self.v1 - self.v0),
                              device)
        self.accept_len = torch.empty(B, **i32)
        self.accepted_nodes = torch.empty(B, W, **i32)
        self.accepted_tokens = torch.empty(B, W, **i32)
        self.bonus = torch.empty(B, **i32)
        self.status = torch.zeros(1, **i32)

    def run(self, logits_shard, cand_ids, stream=None):
        M.medusa_verify_records(logits_shard, cand_ids, self.tree, self.v0, self.records,
                                self.cand_logit, self.mode, self.temperature, self.ws,
                                self.status, stream)
        with _on(stream):
            records = gather_stacked(self.records, self.group)
            if self.mode == M.MEDUSA_ACCEPT_TYPICAL:
                max_over_ranks(self.cand_logit, self.group)
        M.medusa_verify_from_records(records, self.cand_logit, cand_ids, self.tree, self.V,
                                     self.accept_len, self.accepted_nodes, self.accepted_tokens,
                                     self.bonus, self.mode, self.temperature, self.eps,
                                     self.delta, self.status, stream)
        return self.accept_len, self.accepted_nodes, self.accepted_tokens, self.bonus
