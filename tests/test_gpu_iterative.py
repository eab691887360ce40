"""The iterative-denoising draft on the GPU (the multi-step variant the
paper-notes page compares against in §5.4.2): the diffusion view re-run on
its own previous drafts, through orthrus_draft_block_iterative.

* tiny fp32 model: the drafts of every pass count (2 and 3 passes, greedy and
  T = 1) equal the oracle's, and a whole sampled decode driven through the
  step API with two-pass drafts equals the oracle's two-pass stream cycle by
  cycle; a divergence is only accepted in a draft (or a cycle) one of whose
  own decisions has an oracle margin below what fp32 rounding can flip;
* bf16, two layers of the Qwen3-1.7B shape: greedy decoding with two-pass
  drafts emits exactly the GPU's own plain-AR stream.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import first_divergent_cycle, step_cycles

pytestmark = pytest.mark.gpu

FP32_MARGIN = 1e-4


@pytest.fixture(scope="module")
def pkg():
    import dual_view_diffusion_b200 as p
    p.lib()
    return p


@pytest.fixture(scope="module")
def tiny(pkg):
    w = synth.make_weights(synth.TINY, 0)
    eng = pkg.Engine(synth.TINY, w, max_batch=1, max_block=8, max_seq=160, split_tokens=64, page_size=16)
    return w, eng


@pytest.mark.parametrize("iterations", [2, 3])
@pytest.mark.parametrize("T,seed", [(0.0, 0), (1.0, 5)])
def test_tiny_iterative_draft_matches_oracle(tiny, iterations, T, seed):
    w, eng = tiny
    prompt = synth.make_prompt(synth.TINY, 16, 1)
    K = 4
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    d = eng.draft_block(anchor, K, temperature=T, seed=seed, iterations=iterations)
    m = oracle.Model(w)
    kc, vc = m.new_cache(64)
    t = m.prefill(prompt, kc, vc)
    ref, _, _, mg = m.draft(kc, vc, t, prompt[-1], K, T, seed, 0, iterations=iterations)
    got = d[0].cpu().numpy()
    assert np.array_equal(got, ref) or mg < FP32_MARGIN, (got, ref, mg)
    assert eng.check_error()[0] == 0


def test_tiny_two_pass_sampled_stream_matches_oracle(tiny):
    w, eng = tiny
    prompt = synth.make_prompt(synth.TINY, 16, 2)
    K, N, T, seed = 4, 24, 1.0, 7
    cyc = step_cycles(eng, prompt[None], [prompt.size], K, N, T, seed, iterations=2)[0]
    ref = oracle.Model(w).generate(prompt, K, N, T, seed, "orthrus", iterations=2)
    c = first_divergent_cycle(cyc, ref, N)
    assert c < 0 or ref["cycle_margin"][c] < FP32_MARGIN, (c, cyc, ref["tokens"])
    assert eng.check_error()[0] == 0


def test_bf16_two_pass_greedy_equals_plain_ar(pkg):
    s = synth.QWEN3_1_7B
    w = synth.make_weights_torch(s, 0, n_layers=2)
    eng = pkg.Engine(s, w, max_batch=1, max_block=32, max_seq=512, split_tokens=128)
    prompt = torch.from_numpy(synth.make_prompt(s, 200, 0))[None]
    K, N = 32, 96
    anchor = eng.prefill(prompt)
    got = []
    while len(got) < N:
        draft = eng.draft_block(anchor, K, iterations=2)
        eng.verify_block(anchor, draft, K)
        n, toks = eng.commit(anchor, K)
        got += toks[0, :int(n[0])].tolist()
    a, _ = eng.generate(prompt, 0, N, 0.0, 0)
    assert got[:N] == a[0].tolist()
    assert eng.check_error()[0] == 0
    del eng, w
    torch.cuda.empty_cache()
