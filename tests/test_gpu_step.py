"""GPU parity of the whole decode-verify step (DecodeVerifyStep: heads with
the tree build, tree attention, verification with the KV compaction) against
the oracle's step, on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import speculative_decoding_medusa_b200 as M
from oracle import medusa_oracle as O
from speculative_decoding_medusa_b200 import workloads as W
from speculative_decoding_medusa_b200.step import DecodeVerifyStep
from tests.helpers import ATTN_REL_L2, LOGIT_MAX_ABS, TYPICAL_LOG_MARGIN, f64, i64, rel_l2

pytestmark = pytest.mark.gpu


def _inputs(w, seed):
    spec = W.tree_for(w)
    for s in range(seed, seed + 10000, 1000):
        # the step is compared end to end, so the oracle's top-k order must be
        # unambiguous at fp32 accuracy: redraw the heads until every gap among
        # the top kmax+1 logits exceeds 1e-4
        hin = W.heads_inputs(w, seed=s)
        z = O.head_logits(f64(hin["h"]), f64(hin["W1"]), f64(hin["b1"]), f64(hin["W2"]))
        ids, vals = O.topk(z, w.kmax + 1)
        if np.diff(-vals, axis=-1).min() > 1e-4:
            break
    ids = ids[..., :w.kmax]
    att = W.attention_inputs(w, seed=seed)
    if "lm_head" in hin:   # the root is the base model's own next token
        root = O.row_argmax(O.lm_head_logits(f64(hin["h"]), f64(hin["lm_head"]))[:, None])[:, 0]
    else:
        root = i64(W.random_root_tokens(w, seed))
    tb = O.tree_build(spec.parent, spec.depth, spec.rank, root, ids, i64(att["prefix_len"]))
    logits = None
    for attempt in range(20):
        logits = W.verify_logits(w, spec, torch.from_numpy(tb["cand"]), seed=seed, attempt=attempt)
        if w.accept != "typical":
            break
        m = O.typical_log_margin(f64(logits), tb["cand"], spec.parent, w.temperature, w.eps,
                                 w.delta)
        if np.abs(m[:, 1:]).min() > TYPICAL_LOG_MARGIN:
            break
    return spec, hin, att, torch.from_numpy(root.astype(np.int32)), logits


@pytest.mark.parametrize("name,over,seed", [
    ("tiny", {}, 0),
    ("tiny", {"B": 3}, 1),
    ("vicuna7b", dict(B=2, d=256, V=3000, ctx_lo=300, ctx_hi=900), 2),
    ("llama3_8b", dict(B=3, d=256, V=2500, ctx_lo=100, ctx_hi=700), 3),
    ("llama3_70b", dict(B=2, d=128, V=2000, ctx_lo=200, ctx_hi=200, Hq=16, Hkv=2), 4),
])
def test_step_matches_oracle(name, over, seed):
    w = W.scaled(W.WORKLOADS[name], **over)
    spec, hin, att, root, logits = _inputs(w, seed)
    dev = "cuda"
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    step = DecodeVerifyStep(B=w.B, d=w.d, V=w.V, K=w.K, kmax=w.kmax, tree=M.Tree.from_spec(spec),
                            Hq=w.Hq, Hkv=w.Hkv, dh=w.dh, cap=w.cap, max_prefix=w.ctx_hi, dtype=dt,
                            accept=w.accept, temperature=w.temperature, eps=w.eps, delta=w.delta,
                            head_logits=True, attn_out_dtype=torch.float32)
    g = {k: v.to(dev) for k, v in {**hin, **att}.items()}
    step.run(g["h"], g["W1"], g["b1"], g["W2"], root.to(dev), g["q"], g["k_new"], g["v_new"],
             g["Kc"], g["Vc"], g["prefix_len"], logits.to(dev))
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0

    inp = {k: f64(v) for k, v in {**hin, **att}.items() if k != "prefix_len"}
    inp.update(prefix_len=i64(att["prefix_len"]), root_tok=i64(root), logits=f64(logits))
    ref = O.decode_verify_step(inp, {"parent": spec.parent, "depth": spec.depth, "rank": spec.rank},
                               w.kmax, w.accept, w.temperature, w.eps, w.delta)
    assert np.abs(f64(step.head_logits) - ref["logits"]).max() < LOGIT_MAX_ABS
    np.testing.assert_array_equal(step.topk_ids.cpu().numpy(), ref["topk_ids"])
    np.testing.assert_array_equal(step.cand_ids.cpu().numpy(), ref["cand"])
    np.testing.assert_array_equal(step.pos_ids.cpu().numpy(), ref["pos"])
    np.testing.assert_array_equal(step.anc_mask.cpu().numpy().view(np.uint32), ref["mask"])
    np.testing.assert_array_equal(step.retrieve.cpu().numpy(), ref["retrieve"])
    out = f64(step.attn_out)
    assert np.abs(out - ref["attn_out"]).max() < LOGIT_MAX_ABS
    assert rel_l2(out, ref["attn_out"]) < ATTN_REL_L2
    for k in ("accept_len", "accepted_nodes", "accepted_tokens", "bonus"):
        np.testing.assert_array_equal(getattr(step, k).cpu().numpy(), ref[k], err_msg=k)
    np.testing.assert_array_equal(step.compact_src.cpu().numpy(), ref["compact_src"])
    np.testing.assert_array_equal(g["prefix_len"].cpu().numpy(), ref["prefix_len"])
    np.testing.assert_array_equal(f64(g["Kc"]), ref["Kc"])
    np.testing.assert_array_equal(f64(g["Vc"]), ref["Vc"])
