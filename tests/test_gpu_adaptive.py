"""Adaptive block length on the GPU (the paper-notes page on "Orthrus", §7.4:
a verify length set by the draft's own uncertainty; §9.6: a dynamic K; the
reading: a cycle verifies the drafted tokens while their draft rows'
entropies stay at or below a threshold h_max), through orthrus_adaptive_len
and orthrus_commit_adaptive.

* tiny fp32 model with peaky weights (entropies vary between rows and
  cycles), h_max in {+inf, 4.3, 4.45, 4.5, -1}: every cycle's row entropies
  within 1e-4 of the oracle's, its verify length kt, accepted length and
  tokens equal to the oracle's step-by-step cycle (a differing kt is only
  excused by an entropy within 1e-4 of h_max, a differing token by an
  argmax margin under 1e-4), and the whole stream equal to the GPU's own
  plain AR stream and to the oracle's adaptive run;
* bf16, two layers of the Qwen3-1.7B shape: adaptive greedy decoding emits
  the GPU's plain AR stream, and the draft rows' entropies agree with the
  oracle's to first order in the measured logit error.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

FP32_MARGIN = 1e-4
SHAPE = dataclasses.replace(synth.TINY, std=0.2, sigma_diff=0.05)


@pytest.fixture(scope="module")
def tiny():
    import dual_view_diffusion_b200 as pkg
    w = synth.make_weights(SHAPE, 0)
    eng = pkg.Engine(SHAPE, w, max_batch=1, max_block=8, max_seq=128, split_tokens=64, page_size=16)
    return w, eng


def _gpu_ar(eng, prompt, N):
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    eng.step.zero_()
    return [int(eng.ar_step(anchor)[0]) for _ in range(N)]


@pytest.mark.parametrize("h_max", [math.inf, 4.3, 4.45, 4.5, -1.0])
def test_tiny_adaptive_cycles_match_oracle(tiny, h_max):
    w, eng = tiny
    K, N = 8, 24
    prompt = synth.make_prompt(SHAPE, 16, 0)
    m = oracle.Model(w)
    kc, vc = m.new_cache(16 + N + 2 * K)
    t = m.prefill(prompt, kc, vc)
    a_o = int(prompt[-1])
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    got, kts = [], []
    diverged = False
    while len(got) < N:
        draft = eng.draft_block(anchor, K)
        kt, ent = eng.adaptive_len(1, K, h_max, entropy=True)
        eng.verify_block(anchor, draft, K)
        n, toks = eng.commit_adaptive(anchor, K, kt)
        kt, ent, n = int(kt[0]), ent[0].cpu().numpy(), int(n[0])
        toks, d_g = toks[0, :n].cpu().tolist(), draft[0].cpu().numpy()
        # the oracle's cycle from the same state
        d_o, _, z, mg = m.draft(kc, vc, t, a_o, K)
        H = np.array([oracle.entropy(z[k]) for k in range(K)])
        assert np.abs(ent - H).max() <= 1e-4, (ent, H)
        kt_o = oracle.adaptive_len(H, h_max)
        if not np.array_equal(d_g, d_o):
            assert mg < FP32_MARGIN, (d_g, d_o, mg)
            diverged = True
            break
        if kt != kt_o:
            j = min(kt, kt_o) - 1        # the row whose entropy decided differently
            assert abs(H[j] - h_max) < FP32_MARGIN, (kt, kt_o, H, h_max)
            diverged = True
            break
        g, _, _, mg_v = m.verify(kc, vc, t, a_o, d_o[:kt_o])
        n_o, emit = oracle.consensus_greedy(d_o[:kt_o], g)
        if n != n_o or toks != emit.tolist():
            assert mg_v < FP32_MARGIN, (n, n_o, toks, emit)
            diverged = True
            break
        got += toks
        kts.append(kt)
        t += n
        a_o = toks[-1]
    assert eng.check_error()[0] == 0
    if not diverged:
        got = got[:N]
        ref = m.generate_adaptive(prompt, K, h_max, N)
        assert got == ref["tokens"].tolist()
        assert kts == ref["k_per_cycle"].tolist()
        assert got == _gpu_ar(eng, prompt, N)          # every verify length is lossless (greedy)
        if math.isinf(h_max):
            assert set(kts) == {K}
        elif h_max < 0:
            assert set(kts) == {1}
        else:
            assert len(set(kts)) >= 2, kts


def test_bf16_adaptive_greedy_equals_plain_ar():
    import dual_view_diffusion_b200 as pkg
    s = synth.QWEN3_1_7B
    w = synth.make_weights(s, 0, n_layers=2)
    eng = pkg.Engine(s, w, max_batch=1, max_block=16, max_seq=256, split_tokens=64)
    K, N, P = 16, 40, 64
    prompt = synth.make_prompt(s, P, 2)
    m = oracle.Model(w)
    kc, vc = m.new_cache(P + K + 8)
    t = m.prefill(prompt, kc, vc)
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    # entropies of the first draft vs the oracle's, to first order in the
    # measured logit error: |dH| <= max|dz| * E_p|z - E_p z| (+ fp32 slack)
    draft = eng.draft_block(anchor, K)
    kt, ent = eng.adaptive_len(1, K, math.inf, entropy=True)
    z_g = eng.debug_logits(1, 1, K)[0].cpu().numpy().astype(np.float64)
    _, _, z_o, _ = m.draft(kc, vc, t, int(prompt[-1]), K)
    ent = ent[0].cpu().numpy()
    for k in range(K):
        zo = z_o[k]
        p = np.exp(zo - zo.max()); p /= p.sum()
        spread = float((p * np.abs(zo - (p * zo).sum())).sum())
        bound = float(np.abs(z_g[k] - zo).max()) * spread + 1e-3
        assert abs(ent[k] - oracle.entropy(zo)) <= bound, (k, ent[k], oracle.entropy(zo), bound)
    h_max = float(np.median(ent))                # a threshold inside the observed range
    # adaptive greedy decoding from the prompt == the GPU's plain AR stream
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    eng.step.zero_()
    got, kts = [], []
    while len(got) < N:
        draft = eng.draft_block(anchor, K)
        kt = eng.adaptive_len(1, K, h_max)
        eng.verify_block(anchor, draft, K)
        n, toks = eng.commit_adaptive(anchor, K, kt)
        got += toks[0, :int(n[0])].cpu().tolist()
        kts.append(int(kt[0]))
    assert eng.check_error()[0] == 0
    assert got[:N] == _gpu_ar(eng, prompt, N)
    assert all(1 <= k <= K for k in kts)
