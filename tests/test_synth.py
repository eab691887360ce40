"""The seeded input generator: determinism, stream independence and bf16
rounding (checked against torch's own fp32 -> bf16 conversion)."""
import numpy as np
import torch

import synth


def test_deterministic_and_independent():
    a = synth.normal((4, 5), 1.0, 3, "x")
    assert np.array_equal(a, synth.normal((4, 5), 1.0, 3, "x"))
    assert not np.array_equal(a, synth.normal((4, 5), 1.0, 3, "y"))
    assert not np.array_equal(a, synth.normal((4, 5), 1.0, 4, "x"))


def test_bf16_rounding_matches_torch():
    x = synth.normal(100000, 3.0, 0, "bf16")
    ours = synth.round_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, ref)


def test_prompt_excludes_mask_and_weights_recipe():
    s = synth.TINY
    p = synth.make_prompt(s, 5000, 0)
    assert p.min() >= 0 and p.max() < s.mask_id
    w = synth.make_weights(s, 0)
    assert w.embed.shape == (s.vocab, s.hidden) and w.layers[0]["wq"].shape == (s.n_q_heads * s.head_dim, s.hidden)
    d = w.layers[0]["wq_diff"] - w.layers[0]["wq"]
    assert 0.0015 < d.std() < 0.0025 and 0.018 < w.layers[0]["wq"].std() < 0.022
    # a shallower draw is a prefix of the deeper one
    w1 = synth.make_weights(s, 0, n_layers=1)
    assert np.array_equal(w1.layers[0]["w_down"], w.layers[0]["w_down"])
    b = synth.make_weights(synth.MICRO, 0)
    assert b.lm_head is not b.embed
    import dataclasses
    t = synth.make_weights(dataclasses.replace(synth.QWEN3_1_7B, vocab=512, hidden=64), 0, n_layers=0)
    assert t.lm_head is t.embed                      # tied head
    assert np.array_equal(synth.round_bf16(t.embed[:3]), t.embed[:3])
