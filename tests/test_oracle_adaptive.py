"""Pins of the oracle's adaptive block length (the paper-notes page on
"Orthrus", §7.4: SV's information-gain signal deciding how many drafted
tokens to verify, proposed as complementary to Orthrus; §9.6: dynamic K).
The pages give no rule; the reading here is that a cycle verifies the
drafted tokens while their draft rows' entropies stay at or below a
threshold.  Held against: scipy's entropy and closed forms, worked
examples of the length rule, the fixed-K cycle at an infinite threshold,
plain AR at a negative one, and the AR greedy stream for thresholds in
between (every verify length is lossless, §4.2 / §9.1)."""
import dataclasses
import math

import numpy as np
import pytest

import oracle
import synth

# a peakier tiny model (weights N(0, 0.2^2)), so draft-row entropies vary
# between rows and cycles
SHAPE = dataclasses.replace(synth.TINY, std=0.2, sigma_diff=0.05)


@pytest.fixture(scope="module")
def model():
    return oracle.Model(synth.make_weights(SHAPE, 0)), synth.make_prompt(SHAPE, 16, 0)


def test_entropy_matches_scipy_and_closed_forms():
    from scipy.stats import entropy
    rng = np.random.default_rng(71)
    for _ in range(5):
        z = rng.standard_normal(300) * 2.5
        p = np.exp(z - z.max()); p /= p.sum()
        assert math.isclose(oracle.entropy(z), float(entropy(p)), rel_tol=1e-12)
    assert math.isclose(oracle.entropy(np.zeros(256)), math.log(256), rel_tol=1e-14)   # uniform
    assert oracle.entropy(np.array([1000.0, 0.0, 0.0])) == 0.0                       # certain
    # two ids with logits 0 and log 3: p = (1/4, 3/4)
    assert math.isclose(oracle.entropy(np.array([0.0, math.log(3.0)])),
                        -(0.25 * math.log(0.25) + 0.75 * math.log(0.75)), rel_tol=1e-14)


def test_adaptive_len_worked_examples():
    H = [0.5, 0.2, 3.0, 0.1]          # y_1 from row 0, y_2 from row 1, y_3 from row 2
    assert oracle.adaptive_len(H, 1.0) == 3      # y_1, y_2 verified; row 2 too uncertain
    assert oracle.adaptive_len(H, 5.0) == 4      # everything: the whole block
    assert oracle.adaptive_len(H, 0.3) == 1      # the anchor alone
    assert oracle.adaptive_len(H, 0.5) == 3      # a row at the threshold counts
    assert oracle.adaptive_len([9.0], -1.0) == 1  # K = 1


def test_infinite_threshold_is_the_fixed_block(model):
    m, p = model
    o = m.generate(p, 8, 24, 0.0, 0, "orthrus")
    a = m.generate_adaptive(p, 8, math.inf, 24)
    assert np.array_equal(o["tokens"], a["tokens"]) and np.array_equal(o["n_per_cycle"], a["n_per_cycle"])
    assert (a["k_per_cycle"] == 8).all()


def test_negative_threshold_is_plain_ar(model):
    m, p = model
    ar = m.generate(p, 8, 20, 0.0, 0, "ar")
    a = m.generate_adaptive(p, 8, -1.0, 20)
    assert np.array_equal(ar["tokens"], a["tokens"])
    assert (a["k_per_cycle"] == 1).all() and (a["n_per_cycle"] == 1).all()


@pytest.mark.parametrize("h_max", [4.3, 4.45, 4.5])
def test_adaptive_decoding_equals_ar(model, h_max):
    m, p = model
    ar = m.generate(p, 8, 24, 0.0, 0, "ar", want_cache=True)
    a = m.generate_adaptive(p, 8, h_max, 24, want_cache=True)
    assert np.array_equal(ar["tokens"], a["tokens"])
    k, n = a["k_per_cycle"], a["n_per_cycle"]
    assert ((1 <= n) & (n <= k) & (k <= 8)).all()
    assert len(set(k.tolist())) >= 2                 # the threshold really varies the length
    t = min(ar["t"], a["t"])
    assert np.array_equal(ar["k_cache"][:, :t], a["k_cache"][:, :t])
    assert np.array_equal(ar["v_cache"][:, :t], a["v_cache"][:, :t])


def test_adaptive_cycle_is_its_retyped_steps(model):
    """An adaptive cycle is: the draft at T = 0, scipy's entropy of each
    draft row's softmax, the length rule, one AR verify of [anchor, y_1 ..
    y_{Kt-1}] and the greedy consensus over those Kt rows.  Retyping four
    cycles from those pinned pieces gives generate_adaptive's lengths and
    tokens (no entropy within 1e-9 of the threshold, so the rule cannot flip
    on rounding)."""
    from scipy.special import softmax
    from scipy.stats import entropy
    m, p = model
    K, h_max = 8, 4.4
    kc, vc = m.new_cache(len(p) + 64)
    t = m.prefill(p, kc, vc)
    anchor, out, ns, ks = int(p[-1]), [], [], []
    for _ in range(4):
        d, _, z, _ = m.draft(kc, vc, t, anchor, K)
        H = [float(entropy(softmax(z[k]))) for k in range(K)]
        assert min(abs(h - h_max) for h in H) > 1e-9
        kt = oracle.adaptive_len(H, h_max)
        g, _, _, _ = m.verify(kc, vc, t, anchor, d[:kt])
        n, emit = oracle.consensus_greedy(d[:kt], g)
        t += n
        anchor = int(emit[-1])
        out += [int(x) for x in emit]
        ns.append(int(n))
        ks.append(int(kt))
    assert len(set(ks)) >= 2                            # the threshold does vary the length
    r = m.generate_adaptive(p, K, h_max, len(out))
    assert r["k_per_cycle"][:4].tolist() == ks and r["n_per_cycle"][:4].tolist() == ns
    assert r["tokens"].tolist() == out
