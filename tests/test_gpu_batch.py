"""Batched decoding on the bf16 tensor-core path, where one GEMM launch
carries many token rows: every row of a step (up to 256, more in tiles of at
most 256) rides on each weight tile as the N of one MMA, so the weights
stream from HBM once per forward whatever the batch.

* a row's projections do not depend on how many rows share its token tile:
  prefills of 20, 100 and 301 tokens (19, 99 and 300 rows in chunks of at
  most 128: token tiles of 32, 128, and 128 + 128 + 64 rows) leave
  bit-identical K/V in every layer for their common first 19 positions;
* greedy Orthrus at batch 16 x K = 32 (512 rows: two tiles of 256) and at
  batch 3 x K = 21 (63 rows) emits exactly the GPU's own batched plain-AR
  streams, sequence by sequence (paper notes §4.2, §9.1);
* the draft logits of a 10-sequence x 30-row step (300 rows: two tiles of
  160) are within 2e-2 of the row's largest |logit| of the fp64 oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

SHAPE = dataclasses.replace(synth.QWEN3_8B, n_layers=2, hidden=512, n_q_heads=4, n_kv_heads=2, ffn=1024, vocab=1000)


@pytest.fixture(scope="module")
def model():
    return synth.make_weights(SHAPE, 7)


def _engine(w, max_batch, max_block, max_seq):
    import dual_view_diffusion_b200 as pkg
    return pkg.Engine(SHAPE, w, max_batch=max_batch, max_block=max_block, max_seq=max_seq, split_tokens=64)


def _kv_rows(eng, b, n):
    pps = eng.pages_per_seq
    k = eng.k_pages[:, b * pps:(b + 1) * pps].permute(0, 1, 3, 2, 4).reshape(eng.n_layers, -1, SHAPE.n_kv_heads,
                                                                             SHAPE.head_dim)
    v = eng.v_pages[:, b * pps:(b + 1) * pps].permute(0, 1, 4, 2, 3).reshape(eng.n_layers, -1, SHAPE.n_kv_heads,
                                                                             SHAPE.head_dim)
    return k[:, :n].clone(), v[:, :n].clone()


def test_prefill_rows_independent_of_token_tile(model):
    eng = _engine(model, 1, 32, 512)
    prompt = synth.make_prompt(SHAPE, 301, 3)
    got = []
    for P in (20, 100, 301):
        eng.k_pages.zero_(); eng.v_pages.zero_()
        eng.prefill(torch.from_numpy(prompt[:P])[None])
        got.append(_kv_rows(eng, 0, 19))
    assert eng.check_error()[0] == 0
    for k, v in got[1:]:
        assert torch.equal(k, got[0][0]) and torch.equal(v, got[0][1])


@pytest.mark.parametrize("B,K,N", [(16, 32, 48), (3, 21, 40)])
def test_batch_orthrus_equals_batch_ar(model, B, K, N):
    eng = _engine(model, B, K, 512)
    lens = [40 + 7 * b for b in range(B)]
    prompts = np.zeros((B, max(lens)), np.int32)
    for b, P in enumerate(lens):
        prompts[b, :P] = synth.make_prompt(SHAPE, P, 100 + b)
    o, st = eng.generate(torch.from_numpy(prompts), K, N, 0.0, 0, lens=lens)
    a, _ = eng.generate(torch.from_numpy(prompts), 0, N, 0.0, 0, lens=lens)
    assert eng.check_error()[0] == 0
    assert torch.equal(o, a), [int((o[b] != a[b]).nonzero()[0]) if (o[b] != a[b]).any() else -1 for b in range(B)]
    assert st["forwards"] == 2 * st["cycles"]


def test_batch_draft_logits_vs_oracle(model):
    B, K = 10, 30
    eng = _engine(model, B, K, 256)
    lens = [33 + 5 * b for b in range(B)]
    prompts = np.zeros((B, max(lens)), np.int32)
    for b, P in enumerate(lens):
        prompts[b, :P] = synth.make_prompt(SHAPE, P, 200 + b)
    anchor = eng.prefill(torch.from_numpy(prompts), lens)
    eng.draft_block(anchor, K)
    dl = eng.debug_logits(1, B, K).cpu().numpy()
    assert eng.check_error()[0] == 0
    m = oracle.Model(model)
    for b in (0, B - 1):
        P = lens[b]
        kc, vc = m.new_cache(P + K)
        t = m.prefill(prompts[b, :P], kc, vc)
        ref = m.forward(1, 1, [int(prompts[b, P - 1])] + [SHAPE.mask_id] * (K - 1), t, kc, vc)
        rel = float((np.abs(dl[b] - ref).max(axis=1) / np.abs(ref).max(axis=1)).max())
        assert rel <= 2e-2, (b, rel)
