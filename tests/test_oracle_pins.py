"""Pins of the CPU oracle against things other than itself: closed forms,
invariants, library routines (torch, a HuggingFace Llama model), published
known-answer vectors and exact enumeration of the sampled decode.

Passages restated by the oracle: the paper-notes page on "Orthrus:
Memory-Efficient Parallel Token Generation via Dual-View Diffusion", §2.1
(dual-view layer), §3.1-§3.3 (packed anchor blocks, dual-pass block mask,
forward KL), §3.2 (diffusion mask), §4.1-§4.3 (cycle, greedy and sampled
consensus), §5.1 (TPF bounds), §9.1 (losslessness).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ RNG
def test_philox_known_answers():
    path = os.path.join(GOLDEN, "philox4x32_10_kat.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        assert oracle.philox4x32_10(v[0:4], v[4:6]) == v[6:10]


def test_uniform_range_and_moments():
    u = np.array([oracle.uniform(7, 3, r, i, oracle.PURPOSE_DRAFT) for r in range(4) for i in range(5000)])
    assert (u > 0).all() and (u < 1).all()
    assert abs(u.mean() - 0.5) < 0.01 and abs(u.var() - 1 / 12) < 0.005
    # streams of different purposes / rows are different numbers
    a = oracle.uniform(7, 3, 0, 0, oracle.PURPOSE_DRAFT)
    assert a != oracle.uniform(7, 3, 0, 0, oracle.PURPOSE_ACCEPT)
    assert a != oracle.uniform(7, 3, 1, 0, oracle.PURPOSE_DRAFT)
    assert a != oracle.uniform(8, 3, 0, 0, oracle.PURPOSE_DRAFT)


def test_gumbel_max_samples_softmax():
    # Gumbel-max over one uniform per id is an exact sampler of softmax(z/T):
    # chi-square over 20000 draws.
    z = np.array([0.3, -1.0, 1.2, 0.0, 0.7, -0.4])
    T = 0.8
    p = np.exp(z / T - np.max(z / T)); p /= p.sum()
    n = 20000
    cnt = np.zeros(len(z))
    for s in range(n):
        i, _ = oracle.sample_logits(z, T, 11, s, 2, oracle.PURPOSE_DRAFT)
        cnt[i] += 1
    chi2 = ((cnt - n * p) ** 2 / (n * p)).sum()
    assert chi2 < 25.0          # 5 dof: p-value ~1e-4


def test_softmax_t_matches_torch():
    z = np.random.default_rng(9).standard_normal(50) * 3.0
    for T in (0.3, 0.7, 1.0, 2.5):
        want = torch.softmax(torch.from_numpy(z) / T, 0).numpy()
        assert np.allclose(oracle.softmax_t(z, T), want, rtol=1e-13, atol=1e-17)


def test_argmax_lowest_index_and_margin():
    # ties go to the lowest index (the order the greedy decode commits to);
    # the margin is best minus second best, 0 at a tie
    assert oracle.argmax([1.0, 3.0, 3.0, 2.0]) == (1, 0.0)
    assert oracle.argmax([0.5, 2.0, -1.0, 1.5]) == (1, 0.5)
    assert oracle.argmax([4.0, 4.0]) == (0, 0.0)
    assert oracle.argmax([-2.0, -3.0, -1.0]) == (2, 1.0)


# ------------------------------------------------------------------ blocks
def test_rmsnorm_closed_form_and_torch():
    for c in (0.5, -3.0, 1e-4):
        y = oracle.rmsnorm(np.full(64, c), np.ones(64, np.float32), 1e-6)
        assert np.allclose(y, math.copysign(1.0, c) / math.sqrt(1 + 1e-6 / c ** 2), rtol=1e-14, atol=0)
    x = np.random.default_rng(0).standard_normal(64)
    g = np.random.default_rng(1).standard_normal(64).astype(np.float32)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g.astype(np.float64)), 1e-6)
    assert np.allclose(oracle.rmsnorm(x, g, 1e-6), ref.numpy(), rtol=1e-13, atol=1e-15)


def test_silu():
    assert oracle.silu(0.0) == 0.0
    for g in (-5.0, -0.3, 0.9, 4.0):
        assert abs(oracle.silu(g) - torch.nn.functional.silu(torch.tensor(g, dtype=torch.float64)).item()) < 1e-15


def test_rope_identity_norm_relative():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 16)); k = rng.standard_normal((2, 16))
    assert np.array_equal(oracle.rope(q, 0), q)
    for pos in (1, 7, 1000, 131071):
        assert np.allclose(np.linalg.norm(oracle.rope(q, pos), axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    # q.k after RoPE depends only on the position difference
    d1 = (oracle.rope(q, 10) * oracle.rope(k, 3)).sum(1)
    d2 = (oracle.rope(q, 107) * oracle.rope(k, 100)).sum(1)
    assert np.allclose(d1, d2, rtol=1e-11)
    # a wrong pairing (adjacent instead of rotate-half) would break this:
    # pair (0, 8) rotates by pos * theta^0 = pos radians
    e = np.zeros((1, 16)); e[0, 0] = 1.0
    r = oracle.rope(e, 2)
    assert abs(r[0, 0] - math.cos(2)) < 1e-15 and abs(r[0, 8] - math.sin(2)) < 1e-15


def _sdpa_reference(q, kc, vc, kb, vb, mode):
    """torch scaled_dot_product_attention (library) with an explicit mask."""
    R, nq, hd = q.shape
    nkv = kb.shape[1]
    keys = np.concatenate([kc, kb]) if kc is not None else kb
    vals = np.concatenate([vc, vb]) if vc is not None else vb
    t = 0 if kc is None else kc.shape[0]
    g = nq // nkv
    K = torch.from_numpy(np.repeat(keys, g, axis=1)).permute(1, 0, 2)
    Vv = torch.from_numpy(np.repeat(vals, g, axis=1)).permute(1, 0, 2)
    Q = torch.from_numpy(q).permute(1, 0, 2)
    mask = torch.ones(R, t + R, dtype=torch.bool)
    if mode == 0:
        mask[:, t:] = torch.tril(torch.ones(R, R, dtype=torch.bool))
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, Vv, attn_mask=mask)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("t,R,mode", [(0, 1, 0), (0, 5, 1), (37, 4, 0), (37, 4, 1), (130, 8, 0), (130, 8, 1)])
def test_attention_matches_torch_sdpa(t, R, mode):
    rng = np.random.default_rng(t * 10 + R + mode)
    nq, nkv, hd = 8, 2, 16
    q = rng.standard_normal((R, nq, hd))
    kc = rng.standard_normal((t, nkv, hd)) if t else None
    vc = rng.standard_normal((t, nkv, hd)) if t else None
    kb = rng.standard_normal((R, nkv, hd)); vb = rng.standard_normal((R, nkv, hd))
    o = oracle.attention(q, kc, vc, kb, vb, mode)
    assert np.allclose(o, _sdpa_reference(q, kc, vc, kb, vb, mode), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 4, 8)); kb = rng.standard_normal((1, 2, 8)); vb = rng.standard_normal((1, 2, 8))
    # one key: the output is that key's value row for every head of its group
    o = oracle.attention(q, None, None, kb, vb, 0)
    assert np.allclose(o[0, :2], vb[0, 0]) and np.allclose(o[0, 2:], vb[0, 1])
    # identical keys: the output is the mean of the values
    kc = np.repeat(kb, 9, axis=0); vc = rng.standard_normal((9, 2, 8))
    o = oracle.attention(q, kc, vc, kb, vb, 0)
    mean = np.concatenate([vc, vb]).mean(0)
    assert np.allclose(o[0, :2], mean[0], rtol=1e-12) and np.allclose(o[0, 2:], mean[1], rtol=1e-12)
    # with a one-row block the two masks coincide
    o0 = oracle.attention(q, kc, vc, kb, vb, 0); o1 = oracle.attention(q, kc, vc, kb, vb, 1)
    assert np.array_equal(o0, o1)


# ------------------------------------------------------------------ model
def _hf_llama(w):
    from transformers import LlamaConfig, LlamaForCausalLM
    s = w.shape
    cfg = LlamaConfig(vocab_size=s.vocab, hidden_size=s.hidden, intermediate_size=s.ffn,
                      num_hidden_layers=len(w.layers), num_attention_heads=s.n_q_heads,
                      num_key_value_heads=s.n_kv_heads, head_dim=s.head_dim, rms_norm_eps=s.rms_eps,
                      rope_theta=s.rope_theta, attention_bias=False, mlp_bias=False,
                      tie_word_embeddings=False, max_position_embeddings=4096)
    cfg._attn_implementation = "eager"
    m = LlamaForCausalLM(cfg).double().eval()
    T = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(T(w.embed)); m.lm_head.weight.copy_(T(w.lm_head))
        m.model.norm.weight.copy_(T(w.final_norm))
        for l, lw in enumerate(w.layers):
            L = m.model.layers[l]
            L.input_layernorm.weight.copy_(T(lw["attn_norm"])); L.post_attention_layernorm.weight.copy_(T(lw["ffn_norm"]))
            L.self_attn.q_proj.weight.copy_(T(lw["wq"])); L.self_attn.k_proj.weight.copy_(T(lw["wk"]))
            L.self_attn.v_proj.weight.copy_(T(lw["wv"])); L.self_attn.o_proj.weight.copy_(T(lw["wo"]))
            L.mlp.gate_proj.weight.copy_(T(lw["w_gate"])); L.mlp.up_proj.weight.copy_(T(lw["w_up"]))
            L.mlp.down_proj.weight.copy_(T(lw["w_down"]))
    return m


def test_ar_forward_matches_hf_llama():
    """The AR view is a plain pre-norm Llama-style decoder: its prefill logits
    equal those of the HuggingFace Llama model given the same weights (HF
    builds its RoPE table in fp32, hence the 1e-6 tolerance; a dropped term or
    wrong index gives errors of order 0.1)."""
    w = synth.make_weights(synth.TINY, 0, random_gains=True)
    pr = synth.make_prompt(synth.TINY, 40, 0)
    hf = _hf_llama(w)
    with torch.no_grad():
        ref = hf(torch.from_numpy(pr.astype(np.int64))[None]).logits[0].numpy()
    m = oracle.Model(w)
    kc, vc = m.new_cache(64)
    z = m.forward(0, 0, pr, 0, kc, vc)
    assert np.abs(z - ref).max() < 1e-6 * max(1.0, np.abs(ref).max())


def test_ar_greedy_stream_matches_hf_llama():
    """The oracle's plain AR decode (prefill of all but the last prompt token,
    that token as the first anchor, then one cached row per token) emits the
    tokens of a greedy loop over HuggingFace full-sequence forwards.  The
    loop's smallest argmax margin is asserted to stay far above the 1e-6 the
    two models' logits may differ by, so equality is a strict test."""
    w = synth.make_weights(synth.TINY, 0, random_gains=True)
    pr = synth.make_prompt(synth.TINY, 16, 0)
    hf = _hf_llama(w)
    seq, want, margins = [int(x) for x in pr], [], []
    with torch.no_grad():
        for _ in range(24):
            z = hf(torch.tensor([seq], dtype=torch.int64)).logits[0, -1].numpy()
            top2 = np.sort(z)[-2:]
            margins.append(top2[1] - top2[0])
            want.append(int(np.argmax(z)))
            seq.append(want[-1])
    assert min(margins) > 1e-4
    a = oracle.Model(w).generate(pr, 1, 24, 0.0, 0, "ar")
    assert a["tokens"].tolist() == want


def test_ar_law_matches_hf_llama():
    """The exact AR law of the first two tokens at T = 0.7 (the enumeration
    the losslessness pins compare against) is the product of HuggingFace's
    softmax(logits / T) after the prompt and after the prompt plus the first
    token."""
    w = synth.make_weights(synth.MICRO, 0)
    pr = synth.make_prompt(synth.MICRO, 3, 0)
    T, V = 0.7, synth.MICRO.vocab
    hf = _hf_llama(w)

    def p_next(seq):
        with torch.no_grad():
            z = hf(torch.tensor([list(seq)], dtype=torch.int64)).logits[0, -1]
        return torch.softmax(z / T, 0).numpy()

    p1 = p_next(pr)
    want = np.concatenate([p1[x] * p_next(list(pr) + [x]) for x in range(V)])
    got = oracle.Model(w).enumerate_ar(pr, 2, T)
    assert np.allclose(got, want, rtol=0, atol=1e-6)


def test_diffusion_view_is_the_network_with_its_own_projections(tiny_weights, tiny_prompt):
    """Notes §2.1: the diffusion view is the frozen network with only W_Q,
    W_K, W_V replaced by the diffusion copies.  Its forward over a block
    equals the AR-view code path, under the same (bidirectional) mask, of a
    model whose W_Q/W_K/W_V are those copies; with the original model's AR
    weights the result differs."""
    import dataclasses
    w = tiny_weights
    swapped = dataclasses.replace(w, layers=[dict(lw, wq=lw["wq_diff"], wk=lw["wk_diff"], wv=lw["wv_diff"])
                                             for lw in w.layers])
    m, m2 = oracle.Model(w), oracle.Model(swapped)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    mask = synth.TINY.mask_id
    blk = [int(tiny_prompt[-1]), mask, 17, mask, mask]
    a = m.forward(1, 1, blk, t, kc.copy(), vc.copy())
    assert np.array_equal(a, m2.forward(0, 1, blk, t, kc.copy(), vc.copy()))
    assert not np.allclose(a, m.forward(0, 1, blk, t, kc.copy(), vc.copy()), rtol=0, atol=1e-9)


def test_block_rows_equal_single_rows(tiny_weights, tiny_prompt):
    """Row k of a causal block equals the same row run alone after the rows
    before it were committed (bitwise: rows are computed independently)."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    blk = np.array([tiny_prompt[-1], 3, 77, 200, 9], np.int32)
    z_blk = m.forward(0, 0, blk, t, kc.copy(), vc.copy())
    kc2, vc2 = kc.copy(), vc.copy()
    for k, tok in enumerate(blk):
        z1 = m.forward(0, 0, [tok], t + k, kc2, vc2)
        assert np.array_equal(z1[0], z_blk[k])


def test_views_differ_only_by_qkv(tiny_weights, tiny_prompt):
    """Diffusion weights equal to the AR ones make the two views the same
    function when the masks coincide (one-row block)."""
    w = synth.make_weights(synth.TINY, 0, diff_equals_ar=True)
    m = oracle.Model(w)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    a = m.forward(0, 0, [tiny_prompt[-1]], t, kc.copy(), vc.copy())
    b = m.forward(1, 1, [tiny_prompt[-1]], t, kc.copy(), vc.copy())
    assert np.array_equal(a, b)
    # and with the real (perturbed) diffusion weights they differ
    m2 = oracle.Model(tiny_weights)
    c = m2.forward(1, 1, [tiny_prompt[-1]], t, kc.copy(), vc.copy())
    assert not np.array_equal(a, c)


def test_draft_does_not_touch_cache(tiny_weights, tiny_prompt):
    """Diffusion K/V are transient: a draft leaves the cache bit-identical."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    k0, v0 = kc.copy(), vc.copy()
    m.draft(kc, vc, t, tiny_prompt[-1], 4)
    assert np.array_equal(kc, k0) and np.array_equal(vc, v0)


def test_draft_is_the_diffusion_view_of_anchor_and_masks(tiny_weights, tiny_prompt):
    """Notes §4.1 step 1: the draft is one diffusion-view forward of the block
    [anchor, m, ..., m] at positions t .. t+K-1; row k's token is its argmax
    (T = 0) or the Gumbel-max draw of row k's noise (T > 0, which also
    returns q = softmax(z / T)).  Retyping the block through the plain
    forward gives the same logits."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    K, a = 5, int(tiny_prompt[-1])
    ref = m.forward(1, 1, [a] + [synth.TINY.mask_id] * (K - 1), t, kc.copy(), vc.copy())
    d, _, z, _ = m.draft(kc, vc, t, a, K)
    assert np.array_equal(z, ref) and np.array_equal(d, ref.argmax(axis=1))
    T, seed, step = 0.8, 5, 3
    d2, q2, _, _ = m.draft(kc, vc, t, a, K, T, seed, step)
    assert [int(x) for x in d2] == [oracle.sample_logits(ref[k], T, seed, step, k, oracle.PURPOSE_DRAFT)[0]
                                    for k in range(K)]
    assert np.allclose(q2, torch.softmax(torch.from_numpy(ref) / T, 1).numpy(), rtol=1e-12, atol=1e-15)


def test_verify_is_the_ar_view_of_anchor_and_drafts(tiny_weights, tiny_prompt):
    """Notes §4.1 step 2: verification is one causal AR-view forward of
    [anchor, y_1 .. y_{K-1}] at positions t .. t+K-1 that writes those rows'
    K/V into the cache; g_k is row k's argmax."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    a, y = int(tiny_prompt[-1]), [40, 3, 200, 77, 9]
    k2, v2 = kc.copy(), vc.copy()
    ref = m.forward(0, 0, [a] + y[:-1], t, k2, v2)
    g, _, z, _ = m.verify(kc, vc, t, a, y)
    assert np.array_equal(z, ref) and np.array_equal(g, ref.argmax(axis=1))
    assert np.array_equal(kc, k2) and np.array_equal(vc, v2)


# ------------------------------------------------------------------ consensus
def test_consensus_greedy_examples():
    n, e = oracle.consensus_greedy([5, 6, 7, 8], [5, 6, 9, 1])
    assert n == 3 and list(e) == [5, 6, 9]
    n, e = oracle.consensus_greedy([5, 6, 7, 8], [5, 6, 7, 8])
    assert n == 4 and list(e) == [5, 6, 7, 8]
    n, e = oracle.consensus_greedy([4, 6], [5, 6])
    assert n == 1 and list(e) == [5]


def test_accept_and_residual():
    assert oracle.accept_prob(0.2, 0.4) == 0.5 and oracle.accept_prob(0.4, 0.2) == 1.0
    p = np.array([0.5, 0.3, 0.2]); q = np.array([0.2, 0.5, 0.3])
    assert np.allclose(oracle.residual(p, q), [1.0, 0.0, 0.0])
    assert oracle.residual(p, p) is None
    # the identity behind losslessness: q*min(1,p/q) + (1-beta)*r == p
    q = np.array([0.1, 0.6, 0.3]); p = np.array([0.3, 0.3, 0.4])
    beta = sum(q[i] * oracle.accept_prob(p[i], q[i]) for i in range(3))
    r = oracle.residual(p, q)
    assert np.allclose([q[i] * oracle.accept_prob(p[i], q[i]) + (1 - beta) * r[i] for i in range(3)], p, atol=1e-15)


@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_greedy_orthrus_equals_ar(tiny_weights, tiny_prompt, K):
    """Paper notes §4.2/§9.1: greedy Orthrus emits exactly the AR greedy
    stream; every cycle is 2 forwards and emits 1..K tokens (§4.1, §5.1)."""
    m = oracle.Model(tiny_weights)
    a = m.generate(tiny_prompt, K, 32, 0.0, 0, "ar", want_cache=True)
    o = m.generate(tiny_prompt, K, 32, 0.0, 0, "orthrus", want_cache=True)
    assert np.array_equal(a["tokens"], o["tokens"])
    n = o["n_per_cycle"]
    assert (n >= 1).all() and (n <= K).all()
    tpf = n.sum() / (2 * len(n))
    assert 0.5 <= tpf <= K / 2
    # the committed AR K/V are bit-identical to plain AR's
    t = min(a["t"], o["t"])
    assert np.array_equal(a["k_cache"][:, :t], o["k_cache"][:, :t])
    assert np.array_equal(a["v_cache"][:, :t], o["v_cache"][:, :t])


def test_k1_with_shared_weights_always_accepts(tiny_prompt):
    w = synth.make_weights(synth.TINY, 0, diff_equals_ar=True)
    m = oracle.Model(w)
    o = m.generate(tiny_prompt, 1, 12, 0.0, 0, "orthrus")
    assert (o["n_per_cycle"] == 1).all()
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    d, _, _, _ = m.draft(kc, vc, t, tiny_prompt[-1], 1)
    g, _, _, _ = m.verify(kc, vc, t, tiny_prompt[-1], d)
    assert d[0] == g[0]


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_sampled_orthrus_is_lossless_by_enumeration(T):
    """Paper notes §4.3/§9.1: at T>0 the output law equals the AR law.  Exact
    enumeration over every draft tuple and accept/reject branch on a micro
    model (V=8, K=3, first 4 tokens): total variation below 1e-9; planting the
    classic mistake (residual = p instead of norm(max(0, p - q))) breaks it."""
    w = synth.make_weights(synth.MICRO, 0)
    m = oracle.Model(w)
    pr = synth.make_prompt(synth.MICRO, 3, 0)
    pa = m.enumerate_ar(pr, 4, T)
    po = m.enumerate_orthrus(pr, 3, 4, T)
    assert abs(pa.sum() - 1) < 1e-12 and abs(po.sum() - 1) < 1e-12
    assert 0.5 * np.abs(pa - po).sum() < 1e-9
    pb = m.enumerate_orthrus(pr, 3, 4, T, planted_error=True)
    assert 0.5 * np.abs(pa - pb).sum() > 1e-3
    # a one-token block is lossless too (it reduces to one draft and one check)
    assert 0.5 * np.abs(pa - m.enumerate_orthrus(pr, 1, 4, T)).sum() < 1e-9


@pytest.mark.parametrize("iterations", [1, 2])
def test_sampler_matches_ar_law_monte_carlo(iterations):
    """The oracle's real sampled decode (Philox uniforms, Gumbel drafts,
    acceptance test, residual draw; one draft pass or two) against the exact
    AR law of the first two tokens: chi-square over 6000 seeds on the micro
    model."""
    w = synth.make_weights(synth.MICRO, 0)
    m = oracle.Model(w)
    pr = synth.make_prompt(synth.MICRO, 3, 0)
    pa = m.enumerate_ar(pr, 2, 1.0)
    n = 6000
    cnt = np.zeros(64)
    for s in range(n):
        o = m.generate(pr, 3, 2, 1.0, s + 1, "orthrus", iterations=iterations)
        cnt[o["tokens"][0] * 8 + o["tokens"][1]] += 1
    e = n * pa
    keep = e >= 5
    chi2 = (((cnt - e) ** 2 / e)[keep]).sum() + ((cnt[~keep].sum() - e[~keep].sum()) ** 2 / max(e[~keep].sum(), 1e-9))
    dof = keep.sum()
    # p-value ~1e-4 threshold via Wilson-Hilferty
    z = ((chi2 / dof) ** (1 / 3) - (1 - 2 / (9 * dof))) / math.sqrt(2 / (9 * dof))
    assert z < 3.7, (chi2, dof)


# ---------------------------------------------------------------- iterative denoising
# The paper-notes page (§5.4.2) compares single-step drafting with multi-step
# iterative denoising; the iterative variant re-runs the diffusion view on
# its own previous drafts (oc_draft_iter).

def test_sampled_draft_proposal_is_the_last_pass(tiny_weights, tiny_prompt):
    """At T > 0 the proposal q the acceptance test divides by is softmax(z/T)
    of the pass whose drafts are proposed: the last one, whose logits the
    draft returns (retyped through the plain forward on the previous pass's
    drafts)."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    K, T, seed, step, a = 4, 0.9, 7, 1, int(tiny_prompt[-1])
    d1, _, _, _ = m.draft(kc, vc, t, a, K, T, seed, step)
    d2, q2, z2, _ = m.draft(kc, vc, t, a, K, T, seed, step, iterations=2)
    assert np.array_equal(z2, m.forward(1, 1, [a] + list(d1[:K - 1]), t, kc.copy(), vc.copy()))
    assert np.allclose(q2, torch.softmax(torch.from_numpy(z2) / T, 1).numpy(), rtol=1e-12, atol=1e-15)


def test_iterative_draft_one_pass_is_the_draft(tiny_weights, tiny_prompt):
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    for T, seed in ((0.0, 0), (1.0, 3)):
        d1, q1, z1, _ = m.draft(kc, vc, t, tiny_prompt[-1], 4, T, seed, 2)
        di, qi, zi, _ = m.draft(kc, vc, t, tiny_prompt[-1], 4, T, seed, 2, iterations=1)
        assert np.array_equal(d1, di) and np.array_equal(z1, zi)


def test_iterative_draft_second_pass_sees_first_drafts(tiny_weights, tiny_prompt):
    """Pass 2 is the diffusion view on [anchor, y1_1 .. y1_{K-1}]: retyping
    that block by hand through the plain forward gives the same logits."""
    m = oracle.Model(tiny_weights)
    kc, vc = m.new_cache(64)
    t = m.prefill(tiny_prompt, kc, vc)
    K = 4
    d1, _, _, _ = m.draft(kc, vc, t, tiny_prompt[-1], K)
    d2, _, z2, _ = m.draft(kc, vc, t, tiny_prompt[-1], K, iterations=2)
    ref = m.forward(1, 1, [tiny_prompt[-1]] + list(d1[:K - 1]), t, kc.copy(), vc.copy())
    assert np.array_equal(z2, ref)
    assert np.array_equal(d2, ref.argmax(axis=1))


@pytest.mark.parametrize("iterations", [2, 3])
@pytest.mark.parametrize("K", [2, 4])
def test_greedy_iterative_orthrus_equals_ar(tiny_weights, tiny_prompt, K, iterations):
    """Greedy consensus keeps the AR stream whatever the drafts."""
    m = oracle.Model(tiny_weights)
    a = m.generate(tiny_prompt, K, 24, 0.0, 0, "ar")
    o = m.generate(tiny_prompt, K, 24, 0.0, 0, "orthrus", iterations=iterations)
    assert np.array_equal(a["tokens"], o["tokens"])
    assert (o["n_per_cycle"] >= 1).all() and (o["n_per_cycle"] <= K).all()


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_two_pass_orthrus_is_lossless_by_enumeration(T):
    """At T>0 the two-pass draft only changes the proposal: exact enumeration
    over both passes' draft tuples and every accept/reject branch (micro model,
    K = 3, first 4 tokens) gives the AR law within 1e-9; the planted residual
    mistake breaks it."""
    w = synth.make_weights(synth.MICRO, 0)
    m = oracle.Model(w)
    pr = synth.make_prompt(synth.MICRO, 3, 0)
    pa = m.enumerate_ar(pr, 4, T)
    p2 = m.enumerate_orthrus(pr, 3, 4, T, passes=2)
    assert abs(p2.sum() - 1) < 1e-12
    assert 0.5 * np.abs(pa - p2).sum() < 1e-9
    pb = m.enumerate_orthrus(pr, 3, 4, T, planted_error=True, passes=2)
    assert 0.5 * np.abs(pa - pb).sum() > 1e-3
    # the two-pass proposal differs from the one-pass one (the enumeration
    # really walks the second pass): the planted mistake lands elsewhere
    p1b = m.enumerate_orthrus(pr, 3, 4, T, planted_error=True)
    assert 0.5 * np.abs(pb - p1b).sum() > 1e-6


# ------------------------------------------------------------------ training-side pieces (§3.1-§3.3)
def _bm_case(rng, n_blocks=3, K=4, L=12, nq=4, nkv=2, hd=16, anchors=None):
    q = rng.standard_normal((n_blocks * K, nq, hd))
    kc, vc = rng.standard_normal((L, nkv, hd)), rng.standard_normal((L, nkv, hd))
    kb, vb = rng.standard_normal((n_blocks * K, nkv, hd)), rng.standard_normal((n_blocks * K, nkv, hd))
    if anchors is None:
        anchors = rng.integers(0, L + 1, n_blocks)
    return q, kc, vc, kb, vb, np.asarray(anchors, np.int32)


def test_block_mask_equals_per_block_diffusion_attention():
    # each block under the packed mask == the diffusion-view attention of
    # that block alone over the context prefix before its anchor (the
    # oracle's per-sequence formulation, a separate code path)
    rng = np.random.default_rng(11)
    K = 4
    q, kc, vc, kb, vb, a = _bm_case(rng, n_blocks=4, K=K, anchors=[0, 5, 12, 7])
    o = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    for b in range(4):
        s = slice(b * K, (b + 1) * K)
        t = int(a[b])
        ref = oracle.attention(q[s], kc[:t] if t else None, vc[:t] if t else None, kb[s], vb[s], 1)
        assert np.allclose(o[s], ref, rtol=0, atol=1e-12)


def test_block_mask_uniform_scores_average_the_visible_values():
    # every visible key equal -> uniform softmax -> output = mean of the
    # visible value rows (context [0, a_b) and the block's K rows)
    rng = np.random.default_rng(12)
    K, L, nq, nkv, hd = 4, 10, 4, 2, 8
    q, kc, vc, kb, vb, a = _bm_case(rng, n_blocks=3, K=K, L=L, nq=nq, nkv=nkv, hd=hd, anchors=[0, 3, 10])
    k0 = rng.standard_normal(hd)
    kc[:] = k0
    kb[:] = k0
    o = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    g = nq // nkv
    for b in range(3):
        t = int(a[b])
        for h in range(nq):
            vis = np.concatenate([vc[:t, h // g], vb[b * K:(b + 1) * K, h // g]])
            for k in range(K):
                assert np.allclose(o[b * K + k, h], vis.mean(0), atol=1e-12)


def test_block_mask_blocks_are_mutually_invisible_and_anchor_excluded():
    rng = np.random.default_rng(13)
    K = 4
    q, kc, vc, kb, vb, a = _bm_case(rng, n_blocks=2, K=K, anchors=[6, 9])
    o = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    kb2, vb2 = kb.copy(), vb.copy()
    kb2[K:] += 3.0
    vb2[K:] -= 2.0
    o2 = oracle.block_mask_attention(q, kc, vc, kb2, vb2, a, K)
    assert np.array_equal(o[:K], o2[:K])            # block 1 changed, block 0 untouched
    assert not np.allclose(o[K:], o2[K:])
    kc3, vc3 = kc.copy(), vc.copy()
    kc3[6:] += 5.0                                  # at or after block 0's anchor
    vc3[6:] += 5.0
    o3 = oracle.block_mask_attention(q, kc3, vc3, kb, vb, a, K)
    assert np.array_equal(o[:K], o3[:K])
    kc3[5] += 5.0                                   # the last context row before the anchor
    vc3[5] += 5.0
    o4 = oracle.block_mask_attention(q, kc3, vc3, kb, vb, a, K)
    assert not np.allclose(o[:K], o4[:K])


def test_kl_rows_matches_library_relative_entropy():
    from scipy.stats import entropy
    rng = np.random.default_rng(14)
    V, d = 300, 24
    W = rng.standard_normal((V, d)).astype(np.float32)
    hA = rng.standard_normal((5, d))
    hD = hA + 0.4 * rng.standard_normal((5, d))
    kl, la, ld = oracle.kl_rows(hA, hD, W)
    zA, zD = hA @ W.T.astype(np.float64), hD @ W.T.astype(np.float64)
    for r in range(5):
        pA = torch.softmax(torch.from_numpy(zA[r]), 0).numpy()
        pD = torch.softmax(torch.from_numpy(zD[r]), 0).numpy()
        assert math.isclose(kl[r], entropy(pA, pD), rel_tol=1e-10)        # forward KL(p_A || p_D)
        assert math.isclose(la[r], float(torch.logsumexp(torch.from_numpy(zA[r]), 0)), rel_tol=1e-12)
        assert math.isclose(ld[r], float(torch.logsumexp(torch.from_numpy(zD[r]), 0)), rel_tol=1e-12)
        assert not math.isclose(kl[r], entropy(pD, pA), rel_tol=1e-6)     # the reverse direction differs


def test_kl_rows_closed_forms():
    rng = np.random.default_rng(15)
    W = rng.standard_normal((40, 6)).astype(np.float32)
    h = rng.standard_normal((3, 6))
    kl, _, _ = oracle.kl_rows(h, h, W)
    assert np.all(np.abs(kl) < 1e-12)                # identical views
    # two-token vocabulary: KL = p log(p/q) + (1-p) log((1-p)/(1-q))
    W2 = np.array([[1.0, 0.0], [0.0, 1.0]], np.float32)
    hA, hD = np.array([[0.7, -0.4]]), np.array([[-0.2, 0.5]])
    p = 1 / (1 + math.exp(-(0.7 + 0.4)))
    qq = 1 / (1 + math.exp(-(-0.2 - 0.5)))
    want = p * math.log(p / qq) + (1 - p) * math.log((1 - p) / (1 - qq))
    kl2, _, _ = oracle.kl_rows(hA, hD, W2)
    assert math.isclose(kl2[0], want, rel_tol=1e-12)
