"""The consensus decision and the commit over long blocks (paper notes
§4.1 step 3, §4.2): rows are tested and emitted 32 at a time, so blocks of
more than 32 rows cross that boundary.

* forced lengths n in {1, 31, 32, 33, K} after one verify of a K = 40
  block, batch 3: n, the emitted tokens (the verify's AR argmaxes g of rows
  0 .. n-1), the new anchor (g of row n-1) and the committed length t + n,
  every sequence;
* greedy cycles on a peaked tiny fp32 model with K = 40 (so that some
  blocks are accepted far): n equals 1 + the first row whose draft differs
  from g (all K when none does), recomputed on the host from the draft and
  g the library left, and the emitted tokens are g's first n.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

K = 40


def _engine(shape, B):
    import dual_view_diffusion_b200 as pkg
    w = synth.make_weights(shape, 0)
    return pkg.Engine(shape, w, max_batch=B, max_block=K, max_seq=512, split_tokens=64, page_size=16)


def test_forced_lengths_across_the_warp_boundary():
    B = 3
    eng = _engine(synth.TINY, B)
    lens = [20, 27, 33]
    prompts = np.zeros((B, max(lens)), np.int32)
    for b, P in enumerate(lens):
        prompts[b, :P] = synth.make_prompt(synth.TINY, P, 40 + b)
    anchor = eng.prefill(torch.from_numpy(prompts), lens)
    t0 = eng.seq_lens[:B].clone()
    a0 = anchor.clone()
    draft = eng.draft_block(anchor, K)
    eng.verify_block(anchor, draft, K)
    g, _, _ = eng.debug_rows(0, B, K)
    for n_force in (1, 31, 32, 33, K):
        eng.seq_lens[:B] = t0
        anchor.copy_(a0)
        force = torch.full((B,), n_force, dtype=torch.int32, device=anchor.device)
        n, toks = eng.commit(anchor, K, force_n=force)
        assert eng.check_error()[0] == 0
        assert (n == n_force).all(), (n_force, n)
        assert torch.equal(toks[:, :n_force], g[:, :n_force]), n_force
        assert torch.equal(anchor, g[:, n_force - 1]), n_force
        assert torch.equal(eng.seq_lens[:B], t0 + n_force), n_force


def test_greedy_length_matches_first_mismatch():
    shape = dataclasses.replace(synth.TINY, std=0.2, sigma_diff=0.01)   # peaked, views close: long acceptance
    eng = _engine(shape, 1)
    anchor = eng.prefill(torch.from_numpy(synth.make_prompt(shape, 24, 7))[None])
    eng.step.zero_()
    longest = 0
    for _ in range(8):
        t = int(eng.seq_lens[0])
        draft = eng.draft_block(anchor, K)
        eng.verify_block(anchor, draft, K)
        g, _, _ = eng.debug_rows(0, 1, K)
        d, gg = draft[0].cpu().numpy(), g[0].cpu().numpy()
        miss = np.nonzero(d != gg)[0]
        n_host = int(miss[0]) + 1 if len(miss) else K
        n, toks = eng.commit(anchor, K)
        assert eng.check_error()[0] == 0
        assert int(n[0]) == n_host, (int(n[0]), n_host, d, gg)
        assert toks[0, :n_host].cpu().tolist() == gg[:n_host].tolist()
        assert int(eng.seq_lens[0]) == t + n_host
        longest = max(longest, n_host)
    assert longest >= 2, longest   # the peaked model accepts past the first row somewhere
