"""The bf16 rounding floor of a full-depth forward: where the full-depth
logits bound of the GPU tests comes from.

The tensor-core path rounds to bf16 exactly where an MMA or the cache needs
a bf16 operand: the RMSNorm outputs (inputs of the QKV, gate/up and LM-head
projections), the attention output and the SwiGLU product (inputs of the O
and down projections), Q, K and V (attention operands; K and V are also the
bf16 cache), and the softmax probabilities P (the A operand of P.V).  All
sums stay in fp32 and the residual stream stays fp32.  The weights are the
same bf16 values on both sides, so they add nothing.

This test runs the AR forward of the Qwen3-1.7B shape (28 layers, random
init, the synthetic recipe) twice in plain fp32 torch on the CPU: once
without rounding and once rounding at those points only, and measures the
last 8 rows' logits error.  No kernel runs here; the forward is written out
from the same model definition as the oracle's (paper notes §2.1: a
Qwen3-style decoder; RMSNorm, RoPE with the rotate-half pairing, GQA,
SwiGLU).

On this seed the floor is ~1.9 % of the row's largest |logit| (and of the
row's L2 norm), against < 0.5 % at two layers: the 2e-2 bound that holds for
the two-layer GPU tests is the floor itself at 28 layers.  The full-depth
GPU test therefore bounds its error at 2.5e-2 on both measures; this test
keeps that bound tied to the arithmetic by asserting the floor lies between
1.2e-2 and 2.5e-2 (a floor above the bound would make the bound unreachable
for any bf16-operand implementation; one far below it would make the bound
too loose).
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth

FULL_DEPTH_BOUND = 2.5e-2


def _bf(x):
    return x.to(torch.bfloat16).to(torch.float32)


def _forward(w, tokens, rounding, rows):
    s = w.shape
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    d, nq, nkv, hd = s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim
    r = _bf if rounding else (lambda x: x)
    R = len(tokens)
    inv = 1.0 / (s.rope_theta ** (torch.arange(0, hd, 2, dtype=torch.float64) / hd))
    ang = torch.arange(R, dtype=torch.float64)[:, None] * inv[None]
    cos, sin = torch.cos(ang).float()[:, None], torch.sin(ang).float()[:, None]

    def rope(x):
        x1, x2 = x[..., :hd // 2], x[..., hd // 2:]
        return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], -1)

    def norm(x, g):
        return x * torch.rsqrt((x * x).mean(-1, keepdim=True) + s.rms_eps) * T(g)

    emb = T(w.embed)
    h = emb[torch.as_tensor(tokens, dtype=torch.long)].clone()
    causal = torch.ones(R, R, dtype=torch.bool).tril()
    g = nq // nkv
    for L in w.layers:
        a = r(norm(h, L["attn_norm"]))
        q = r(rope((a @ T(L["wq"]).T).view(R, nq, hd)))
        k = r(rope((a @ T(L["wk"]).T).view(R, nkv, hd))).repeat_interleave(g, 1)
        v = r((a @ T(L["wv"]).T).view(R, nkv, hd)).repeat_interleave(g, 1)
        sc = torch.einsum("rhd,thd->hrt", q, k) / hd ** 0.5
        sc = sc.masked_fill(~causal, float("-inf"))
        p = torch.exp(sc - sc.max(-1, keepdim=True).values)
        o = torch.einsum("hrt,thd->rhd", r(p), v) / p.sum(-1).T[:, :, None]
        h = h + r(o.reshape(R, nq * hd)) @ T(L["wo"]).T
        a = r(norm(h, L["ffn_norm"]))
        f = torch.nn.functional.silu(a @ T(L["w_gate"]).T) * (a @ T(L["w_up"]).T)
        h = h + r(f) @ T(L["w_down"]).T
    a = r(norm(h[-rows:], w.final_norm))
    return (a @ T(w.lm_head).T).double().numpy()


@pytest.fixture(scope="module")
def model():
    return synth.make_weights(synth.QWEN3_1_7B, 0)


def _floor(w, n_layers):
    s = w.shape
    w = dataclasses.replace(w, layers=w.layers[:n_layers])
    prompt = synth.make_prompt(s, 72, 6).tolist()
    torch.set_num_threads(max(1, min(8, torch.get_num_threads())))
    with torch.no_grad():
        ref = _forward(w, prompt, False, 8)
        got = _forward(w, prompt, True, 8)
    rel_max = float((np.abs(got - ref).max(1) / np.abs(ref).max(1)).max())
    rel_l2 = float((np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)).max())
    return rel_max, rel_l2


def test_bf16_floor_two_layers_within_the_bound(model):
    rel_max, rel_l2 = _floor(model, 2)
    assert rel_max < 1e-2 and rel_l2 < 1e-2, (rel_max, rel_l2)


def test_bf16_floor_full_depth_sets_the_bound(model):
    rel_max, rel_l2 = _floor(model, 28)
    print("bf16 floor at 28 layers: max/row-max %.4f, relative L2 %.4f" % (rel_max, rel_l2))
    for e in (rel_max, rel_l2):
        assert 1.2e-2 <= e <= FULL_DEPTH_BOUND, (rel_max, rel_l2)
