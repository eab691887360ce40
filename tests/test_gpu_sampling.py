"""Sampled consensus on the bf16 tensor-core path against the fp64 oracle
(the paper-notes page on "Orthrus", §4.3: drafts sampled from the diffusion
view, each accepted with probability min(1, p/q), the first rejection
replaced by a draw from norm(max(0, p - q))).

Two layers of the Qwen3-1.7B shape (full width, the 151936-id vocabulary,
tied head), prompt 48, K = 8, at T = 1.0 and T = 0.7, decoded cycle by
cycle through the public step calls.  In every cycle the GPU's per-row
results (orthrus_debug_rows) are held against the oracle's forward of the
same block:

* log-sum-exps LSE_q and LSE_p within max|dz|/T + 2e-4 (LSE is 1-Lipschitz
  in the logits; 2e-4 covers fp32 accumulation over 151936 terms), where dz
  is the row's measured logit error (orthrus_debug_logits against the
  oracle's logits; itself within the 2e-2 relative logits bound);
* log q(y) and log p(y) of the drafted token within |dz_y|/T + that bound;
* the Gumbel-max draft winner, the acceptance test and the residual draw
  equal the oracle's, unless the oracle's decision is close enough that the
  measured errors could flip it: the winner w must match when its score
  minus its error bound beats every other id's score plus that id's bound
  (per-id bounds from the per-id logit errors), and the acceptance when
  |log u - (log p - log q)| exceeds the measured error of log p - log q.

The first close decision that flips ends the comparison (the streams may
legitimately part there); every decision before it must agree, and the
run must cover at least three cycles.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

EPS_G = 1e-4      # fp32 Gumbel noise (-log(-log u) in fp32) against fp64
LSE_SLACK = 2e-4  # fp32 accumulation of the log-sum-exp over the vocabulary


def _lse(x):
    m = x.max()
    return m + np.log(np.exp(x - m).sum())


def _robust_winner(score, err):
    """The id with the largest score, and whether it stays the largest for
    every perturbation of each score by at most err (per id)."""
    w = int(np.argmax(score))
    lo = score[w] - err[w]
    others = np.delete(score + err, w)
    return w, bool(lo > others.max())


@pytest.fixture(scope="module")
def model():
    import dual_view_diffusion_b200 as pkg
    s = synth.QWEN3_1_7B
    w = synth.make_weights(s, 0, n_layers=2)
    eng = pkg.Engine(s, w, max_batch=1, max_block=8, max_seq=256, split_tokens=64, page_size=64)
    return s, w, eng, oracle.Model(w)


@pytest.mark.parametrize("T,seed,pseed", [(1.0, 11, 3), (0.7, 12, 4)])
def test_bf16_sampled_cycles_match_oracle(model, T, seed, pseed):
    s, w, eng, m = model
    K, P, n_cycles = 8, 48, 8
    V = s.vocab
    prompt = synth.make_prompt(s, P, pseed)
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    kc, vc = m.new_cache(P + (n_cycles + 1) * K)
    t = m.prefill(prompt, kc, vc)
    a_o = int(prompt[-1])
    checked, residuals, accepts = 0, 0, 0
    for cyc in range(n_cycles):
        assert int(anchor[0]) == a_o
        # ---------------- draft: diffusion view, Gumbel-max samples
        draft = eng.draft_block(anchor, K, temperature=T, seed=seed)
        y_g, lq_g, lseq_g = (x[0].cpu().numpy() for x in eng.debug_rows(1, 1, K))
        wz_g = eng.debug_logits(1, 1, K)[0].cpu().numpy().astype(np.float64)
        wz_o = m.forward(1, 1, [a_o] + [s.mask_id] * (K - 1), t, kc.copy(), vc.copy())
        assert np.array_equal(draft[0].cpu().numpy(), y_g)
        dw = np.abs(wz_g - wz_o)
        assert (dw.max(axis=1) <= 2e-2 * np.abs(wz_o).max(axis=1)).all()
        close = False
        for k in range(K):
            G = oracle.gumbel_vec(seed, cyc, k, oracle.PURPOSE_DRAFT, V)
            score = wz_o[k] / T + G
            wk, robust = _robust_winner(score, dw[k] / T + EPS_G + 1e-6 * np.abs(score))
            if y_g[k] != wk:
                assert not robust, (cyc, k, int(y_g[k]), wk)
                close = True
                break
            lse_o = _lse(wz_o[k] / T)
            d_lse = dw[k].max() / T + LSE_SLACK
            assert abs(lseq_g[k] - lse_o) <= d_lse, (cyc, k, lseq_g[k], lse_o)
            assert abs(lq_g[k] - (wz_o[k, wk] / T - lse_o)) <= dw[k, wk] / T + d_lse, (cyc, k)
        if close:
            break
        # ---------------- verify: AR view over [anchor, y_1 .. y_{K-1}]
        eng.verify_block(anchor, draft, K, temperature=T)
        g_g, lp_g, lsep_g = (x[0].cpu().numpy() for x in eng.debug_rows(0, 1, K))
        z_g = eng.debug_logits(0, 1, K)[0].cpu().numpy().astype(np.float64)
        z_o = m.forward(0, 0, [a_o] + [int(x) for x in y_g[:K - 1]], t, kc, vc)
        dz = np.abs(z_g - z_o)
        assert (dz.max(axis=1) <= 2e-2 * np.abs(z_o).max(axis=1)).all()
        lp_o, lq_o = np.zeros(K), np.zeros(K)
        p_o, q_o = np.zeros((K, V)), np.zeros((K, V))
        for k in range(K):
            lse_p, lse_q = _lse(z_o[k] / T), _lse(wz_o[k] / T)
            assert abs(lsep_g[k] - lse_p) <= dz[k].max() / T + LSE_SLACK, (cyc, k)
            lp_o[k] = z_o[k, y_g[k]] / T - lse_p
            lq_o[k] = wz_o[k, y_g[k]] / T - lse_q
            assert abs(lp_g[k] - lp_o[k]) <= dz[k, y_g[k]] / T + dz[k].max() / T + LSE_SLACK, (cyc, k)
            p_o[k] = np.exp(z_o[k] / T - lse_p)
            q_o[k] = np.exp(wz_o[k] / T - lse_q)
        # ---------------- consensus (GPU) and its decisions (oracle)
        n_g, toks_g = eng.commit(anchor, K, temperature=T, seed=seed)
        n_g, toks_g = int(n_g[0]), toks_g[0].cpu().numpy()
        j_o = K
        for k in range(K):
            u = oracle.uniform(seed, cyc, k, 0, oracle.PURPOSE_ACCEPT)
            gap = np.log(u) - (lp_o[k] - lq_o[k])
            err = abs((lp_g[k] - lq_g[k]) - (lp_o[k] - lq_o[k])) + 1e-6
            acc_o = gap < 0
            acc_g = k < n_g - 1 or (k == n_g - 1 and toks_g[k] == y_g[k] and n_g == K)
            if acc_o != acc_g:
                assert abs(gap) <= err, (cyc, k, gap, err)
                close = True
                break
            if not acc_o:
                j_o = k
                break
            accepts += 1
        if close:
            break
        assert n_g == min(j_o + 1, K)
        assert np.array_equal(toks_g[:j_o], y_g[:j_o])
        if j_o < K:   # the residual draw at the rejected row
            r = p_o[j_o] - q_o[j_o]
            G = oracle.gumbel_vec(seed, cyc, j_o, oracle.PURPOSE_RESIDUAL, V)
            # GPU p~, q~ within exp(+-e) of the oracle's, e from the measured errors
            ep = dz[j_o] / T + dz[j_o].max() / T + LSE_SLACK + 1e-6
            eq = dw[j_o] / T + dw[j_o].max() / T + LSE_SLACK + 1e-6
            lo = p_o[j_o] * np.exp(-ep) - q_o[j_o] * np.exp(eq)
            hi = p_o[j_o] * np.exp(ep) - q_o[j_o] * np.exp(-eq)
            with np.errstate(divide="ignore", invalid="ignore"):
                s_o = np.where(r > 0, np.log(np.where(r > 0, r, 1.0)) + G, -np.inf)
                s_hi = np.where(hi > 0, np.log(np.where(hi > 0, hi, 1.0)) + G + EPS_G, -np.inf)
                s_lo = np.where(lo > 0, np.log(np.where(lo > 0, lo, 1.0)) + G - EPS_G, -np.inf)
            if np.isfinite(s_o).any():
                wr = int(np.argmax(s_o))
                robust = s_lo[wr] > np.delete(s_hi, wr).max()
                # the oracle's own residual draw (normalised r, same noise)
                res = oracle.residual(p_o[j_o], q_o[j_o])
                with np.errstate(divide="ignore"):
                    want, _ = oracle.sample_logits(np.log(res), 1.0, seed, cyc, j_o, oracle.PURPOSE_RESIDUAL)
                assert want == wr
                if toks_g[j_o] != wr:
                    assert not robust, (cyc, j_o, int(toks_g[j_o]), wr)
                    break
                residuals += 1
            else:
                assert toks_g[j_o] == g_g[j_o]
        checked += 1
        # ---------------- commit on the oracle side: keep rows t .. t+n-1
        t += n_g
        a_o = int(toks_g[n_g - 1])
    assert eng.check_error()[0] == 0
    assert checked >= 3, checked
    print(f"T={T}: {checked} cycles, {accepts} acceptances, {residuals} residual draws compared")

