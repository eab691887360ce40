"""One decode step of the Qwen3-8B shape on a synthetically filled cache,
over context lengths, batch sizes and block sizes (the long-context step
sweep; paper notes §2.3, §4.1): two layers at full width and vocabulary,
the cache filled with N(0, 1) bf16 (seed 3, no prefill), accepted lengths
forced per sequence from a seeded uniform over 1..K.

Checked: the committed lengths advance by the forced counts, the emitted
tokens are the verify view's argmaxes, the cache before t and from t + K on
is bit-for-bit untouched, and no device check fires.  A sampled (T = 1)
cycle on the same model is replayed from its seed and step counter.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

L_MAX, B_MAX, K_MAX = 8192, 4, 32


@pytest.fixture(scope="module")
def eng8():
    import dual_view_diffusion_b200 as pkg
    s = synth.QWEN3_8B
    w = synth.make_weights_torch(s, 0, n_layers=2)
    eng = pkg.Engine(s, w, max_batch=B_MAX, max_block=K_MAX, max_seq=L_MAX + K_MAX + 64, split_tokens=128)
    yield eng
    del eng, w
    torch.cuda.empty_cache()


def _by_position(eng, pages, b, transposed):
    """Cache of sequence b as [layer, position, kv head, dim]."""
    pps = eng.pages_per_seq
    x = pages[:, b * pps:(b + 1) * pps]
    x = x.permute(0, 1, 4, 2, 3) if transposed else x.permute(0, 1, 3, 2, 4)
    return x.reshape(x.shape[0], -1, x.shape[3], x.shape[4])


def _fill(eng, seed):
    g = torch.Generator(device=eng.device).manual_seed(seed)
    for p in (eng.k_pages, eng.v_pages):
        p.copy_(torch.randn(p.shape, generator=g, device=eng.device, dtype=torch.float32).to(p.dtype))


@pytest.mark.parametrize("K", [4, 32])
@pytest.mark.parametrize("B", [1, 4])
@pytest.mark.parametrize("L", [2048, 8192])
def test_forced_step(eng8, L, B, K):
    eng = eng8
    _fill(eng, 3)
    eng.seq_lens.zero_()
    eng.seq_lens[:B] = L
    rng = np.random.Generator(np.random.Philox(key=3 + 17 * K + 101 * B))
    force = torch.as_tensor(rng.integers(1, K + 1, size=B), dtype=torch.int32, device=eng.device)
    anchor = torch.as_tensor(rng.integers(0, synth.QWEN3_8B.vocab - 1, size=B), dtype=torch.int32, device=eng.device)
    before = [(eng.k_pages.clone(), False), (eng.v_pages.clone(), True)]
    a_draft = anchor.clone()
    draft = eng.draft_block(a_draft, K)
    eng.verify_block(anchor, draft, K)
    vl = eng.debug_logits(0, B, K)
    n, toks = eng.commit(anchor, K, force_n=force)
    torch.cuda.synchronize()
    assert eng.check_error()[0] == 0
    assert torch.equal(n, force)
    assert torch.equal(eng.seq_lens[:B], torch.full((B,), L, dtype=torch.int32, device=eng.device) + force)
    g = vl.argmax(dim=2).to(torch.int32)                       # verify argmaxes per row
    for b in range(B):
        nb = int(force[b])
        assert torch.equal(toks[b, :nb], g[b, :nb])
        assert int(anchor[b]) == int(g[b, nb - 1])
    for (old, tr), new in zip(before, (eng.k_pages, eng.v_pages)):
        for b in range(B_MAX):
            o, w = _by_position(eng, old, b, tr), _by_position(eng, new, b, tr)
            t = L if b < B else 0
            assert torch.equal(o[:, :t], w[:, :t])              # the committed prefix
            if b < B:
                assert not torch.equal(o[:, t:t + K], w[:, t:t + K])   # the verify K/V landed
            assert torch.equal(o[:, t + (K if b < B else 0):], w[:, t + (K if b < B else 0):])


def test_sampled_cycle_replays(eng8):
    """T = 1: every accepted length is in [1, K] and the stream is a function
    of (seed, step counter, state): replaying from the same state gives the
    same tokens."""
    eng = eng8
    K, B, L = 32, 2, 2048
    out = []
    for _ in range(2):
        _fill(eng, 5)
        eng.seq_lens.zero_()
        eng.seq_lens[:B] = L
        eng.step.zero_()
        anchor = torch.tensor([11, 12], dtype=torch.int32, device=eng.device)
        toks_all = []
        for _ in range(3):
            draft = eng.draft_block(anchor, K, temperature=1.0, seed=9)
            eng.verify_block(anchor, draft, K, temperature=1.0)
            n, toks = eng.commit(anchor, K, temperature=1.0, seed=9)
            assert bool(((n >= 1) & (n <= K)).all())
            toks_all.append((n.clone(), toks.clone()))
        assert eng.check_error()[0] == 0
        out.append(toks_all)
    for (n0, t0), (n1, t1) in zip(*out):
        assert torch.equal(n0, n1)
        for b in range(B):
            assert torch.equal(t0[b, :int(n0[b])], t1[b, :int(n1[b])])
