"""One decode-verify step through the C ABI: buffers plus three calls in order
(heads + top-k with the tree build, tree attention, verify/accept with the KV
compaction; `DecodeLoop` chains the heads with the tree build, the attention, the
lm_head verification, the compaction and the hand-off to the next step).
Argument marshalling only; all arithmetic runs in libmedusa_b200.so."""
from __future__ import annotations

from typing import Optional

import torch
from torch.cuda import nvtx

from . import _lib as M


class DecodeVerifyStep:
    def __init__(self, *, B: int, d: int, V: int, K: int, kmax: int, tree: M.Tree, Hq: int,
                 Hkv: int, dh: int, cap: int, max_prefix: int, dtype: torch.dtype,
                 accept: str = "greedy", temperature: float = 1.0, eps: float = 0.09,
                 delta: float = 0.3, head_logits: bool = False,
                 attn_out_dtype: Optional[torch.dtype] = None, device="cuda"):
        self.B, self.d, self.V, self.K, self.kmax = B, d, V, K, kmax
        self.tree, self.Hq, self.Hkv, self.dh, self.cap = tree, Hq, Hkv, dh, cap
        self.max_prefix = max_prefix
        self.mode = M.MEDUSA_ACCEPT_TYPICAL if accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
        self.temperature, self.eps, self.delta = temperature, eps, delta
        dt = M.MEDUSA_BF16 if dtype == torch.bfloat16 else M.MEDUSA_F32
        N, W = tree.n_nodes, tree.max_depth + 1
        i32 = dict(dtype=torch.int32, device=device)
        self.topk_ids = torch.empty(B, K, kmax, **i32)
        self.topk_vals = torch.empty(B, K, kmax, dtype=torch.float32, device=device)
        self.head_logits = (torch.empty(B, K, V, dtype=torch.float32, device=device)
                            if head_logits else None)
        self.cand_ids = torch.empty(B, N, **i32)
        self.pos_ids = torch.empty(B, N, **i32)
        self.anc_mask = torch.empty(N, (N + 31) // 32, **i32)
        self.retrieve = torch.empty(tree.n_leaves, W, **i32)
        self.attn_out = torch.empty(B, N, Hq, dh, dtype=attn_out_dtype or dtype, device=device)
        self.accept_len = torch.empty(B, **i32)
        self.accepted_nodes = torch.empty(B, W, **i32)
        self.accepted_tokens = torch.empty(B, W, **i32)
        self.bonus = torch.empty(B, **i32)
        self.compact_src = torch.empty(B, W, **i32)
        self.status = torch.zeros(1, **i32)
        self.ws_heads = M.workspace(M.medusa_heads_topk_workspace_size(B, d, V, K, kmax, dt), device)
        self.ws_attn = M.workspace(M.medusa_tree_attention_workspace_size(
            B, N, Hq, Hkv, dh, max_prefix, dt), device)
        self.ws_verify = M.workspace(M.medusa_verify_accept_workspace_size(B, N, V), device)

    def run(self, h, W1, b1, W2, root_tok, q, k_new, v_new, Kc, Vc, prefix_len, verify_logits,
            stream=None) -> None:
        """Enqueue one step on ``stream``.  Kc/Vc/prefix_len are updated in place
        (tree K/V written, then the kept branch compacted, prefix advanced).
        Each call sits in an NVTX range of its name (for ncu --nvtx filters)."""
        with nvtx.range("medusa_heads_topk_tree"):
            M.medusa_heads_topk_tree(h, W1, b1, W2, self.kmax, self.topk_ids, self.topk_vals,
                                     self.tree, root_tok, prefix_len, self.cand_ids, self.pos_ids,
                                     self.anc_mask, self.retrieve, self.head_logits,
                                     self.ws_heads, self.status, stream)
        with nvtx.range("medusa_tree_attention"):
            M.medusa_tree_attention(q, k_new, v_new, Kc, Vc, prefix_len, self.anc_mask,
                                    self.max_prefix, self.attn_out, None, self.ws_attn,
                                    self.status, stream)
        with nvtx.range("medusa_verify_accept_compact"):
            M.medusa_verify_accept_compact(verify_logits, self.cand_ids, self.tree,
                                           self.accept_len, self.accepted_nodes,
                                           self.accepted_tokens, self.bonus, Kc, Vc, prefix_len,
                                           self.compact_src, self.mode, self.temperature,
                                           self.eps, self.delta, self.ws_verify, self.status,
                                           stream)


class DecodeLoop:
    """Decode steps chained on the device (greedy or typical acceptance with
    the verification taken from the tree nodes' hidden states):

        heads + top-k (h) -> tree build (root) -> base model (external; gives
        the nodes' hidden states and tree Q/K/V) -> tree attention ->
        lm_head verify -> KV compaction -> next step (h := kept node's hidden
        state, root := bonus token)

    ``step`` enqueues one step and records its accept_len in ``history``;
    nothing synchronises with the host, so a run of steps can be captured in
    one CUDA graph."""

    def __init__(self, *, B: int, d: int, V: int, K: int, kmax: int, tree: M.Tree, Hq: int,
                 Hkv: int, dh: int, cap: int, max_prefix: int, steps: int,
                 accept: str = "greedy", temperature: float = 1.0, eps: float = 0.09,
                 delta: float = 0.3, device="cuda"):
        self.B, self.d, self.V, self.K, self.kmax = B, d, V, K, kmax
        self.tree, self.Hq, self.Hkv, self.dh = tree, Hq, Hkv, dh
        self.max_prefix = max_prefix
        self.mode = M.MEDUSA_ACCEPT_TYPICAL if accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
        self.temperature, self.eps, self.delta = temperature, eps, delta
        N, W = tree.n_nodes, tree.max_depth + 1
        i32 = dict(dtype=torch.int32, device=device)
        self.topk_ids = torch.empty(B, K, kmax, **i32)
        self.topk_vals = torch.empty(B, K, kmax, dtype=torch.float32, device=device)
        self.cand_ids = torch.empty(B, N, **i32)
        self.pos_ids = torch.empty(B, N, **i32)
        self.anc_mask = torch.empty(N, (N + 31) // 32, **i32)
        self.retrieve = torch.empty(tree.n_leaves, W, **i32)
        self.attn_out = torch.empty(B, N, Hq, dh, dtype=torch.bfloat16, device=device)
        self.accept_len = torch.empty(B, **i32)
        self.accepted_nodes = torch.empty(B, W, **i32)
        self.accepted_tokens = torch.empty(B, W, **i32)
        self.bonus = torch.empty(B, **i32)
        self.compact_src = torch.empty(B, W, **i32)
        self.history = torch.zeros(steps, B, **i32)
        self.tokens = torch.zeros(steps, B, W, **i32)
        self.status = torch.zeros(1, **i32)
        bf = M.MEDUSA_BF16
        self.ws_heads = M.workspace(M.medusa_heads_topk_workspace_size(B, d, V, K, kmax, bf), device)
        self.ws_attn = M.workspace(M.medusa_tree_attention_workspace_size(
            B, N, Hq, Hkv, dh, max_prefix, bf), device)
        self.ws_lm = M.workspace(M.medusa_lmhead_verify_workspace_size(B, N, d, V), device)

    def step(self, r: int, h, root, W1, b1, W2, lm_head, base_model, q, k_new, v_new, Kc, Vc,
             prefix_len, stream=None) -> None:
        """Enqueue step ``r``.  h [B, d] bf16 and root [B] int32 are replaced
        by the next step's; Kc/Vc/prefix_len advance by the kept branch."""
        M.medusa_heads_topk_tree(h, W1, b1, W2, self.kmax, self.topk_ids, self.topk_vals,
                                 self.tree, root, prefix_len, self.cand_ids, self.pos_ids,
                                 self.anc_mask, self.retrieve, None, self.ws_heads, self.status,
                                 stream)
        node_hidden = base_model.forward(self.cand_ids, r)
        M.medusa_tree_attention(q, k_new, v_new, Kc, Vc, prefix_len, self.anc_mask,
                                self.max_prefix, self.attn_out, None, self.ws_attn, self.status,
                                stream)
        M.medusa_lmhead_verify(node_hidden, lm_head, self.cand_ids, self.tree, self.accept_len,
                               self.accepted_nodes, self.accepted_tokens, self.bonus, self.mode,
                               self.temperature, self.eps, self.delta, None, self.ws_lm,
                               self.status, stream)
        M.medusa_kv_compact(Kc, Vc, prefix_len, self.accepted_nodes, self.accept_len,
                            self.compact_src, self.status, stream)
        M.medusa_next_step(node_hidden, self.accept_len, self.accepted_nodes, self.bonus, h, root,
                           self.status, stream)
        self.history[r].copy_(self.accept_len)
        self.tokens[r].copy_(self.accepted_tokens)
