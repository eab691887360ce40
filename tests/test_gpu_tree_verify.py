"""The tree-masked verify forward on the GPU and whole tree-verified decode
cycles (the paper-notes page on "Orthrus", §7.5: DDTree verifies a
best-first tree of one draft's top prefixes with tree attention in one
forward; §9.6: the same proposed for Orthrus; greedy only).

Each cycle runs the library's own pieces: the draft with the top-W of its
rows taken in the LM-head pass (orthrus_draft_block_topw; or the draft, its
materialised logits and orthrus_tree_topw, which the first test shows to
give the same candidates), the tree (orthrus_tree_build), the tree-masked AR
forward (orthrus_verify_tree) and the walk plus commit (orthrus_tree_commit).  The oracle mirrors each cycle on the tree the GPU
built (the builder itself is pinned exactly in test_gpu_tree.py):

* tiny fp32 model: every node's logits within 1e-4 of the row's largest
  |logit| of oc_forward_tree's, every node's AR argmax equal to the
  oracle's unless the oracle margin is under 1e-4, n and the emitted tokens
  equal to the oracle's walk, the committed cache within 1e-5 of the
  oracle's compacted cache; the tree-decoded stream equals the GPU's plain
  AR stream and the oracle's tree-decoded stream, a differing token excused
  only by an AR decision margin under 1e-4 at that position;
* bf16 (two layers of the Qwen3-1.7B shape, 151936-id vocabulary): node
  logits within 2e-2 of the row's largest |logit| of the oracle's; the
  tree-decoded stream equals the GPU's plain AR stream, a differing token
  excused only by a margin under 0.05 of the GPU's own AR logits there.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

SHAPE = dataclasses.replace(synth.TINY, std=0.2, sigma_diff=0.05)   # peaky: trees of varied depth


def _tree_cycle(eng, anchor, K, W, nodes, epilogue_topw=True):
    """One tree-verified decode cycle through the C ABI (the draft's top-W
    from its LM-head epilogue, or from its materialised logits).  Returns
    the tree (parent, token, n_rows), the GPU's g, its node logits, n and the
    emitted tokens (sequence 0)."""
    D = K - 1
    if epilogue_topw:
        _, ids, vals, lse = eng.draft_block_topw(anchor, K, W, D)
    else:
        eng.draft_block(anchor, K)
        z = eng.debug_logits(1, 1, K)[0, :D].contiguous()
        ids, vals, lse = eng.tree_topw(z, W)
    par, tok, _, _, nr = eng.tree_build(ids.view(1, D, W), vals.view(1, D, W), lse.view(1, D), nodes)
    g = eng.verify_tree(anchor, par, tok)
    zt = eng.debug_logits(0, 1, nodes + 1)[0].cpu().numpy().astype(np.float64)
    n, emit = eng.tree_commit(par, tok, nr, g, anchor)
    R = int(nr[0])
    return (par[0, :R].cpu().numpy(), tok[0, :R].cpu().numpy(), R, g[0, :R].cpu().numpy(), zt[:R], int(n[0]),
            emit[0, :int(n[0])].cpu().tolist())


def _ar_stream(eng, prompt, N, logits=False):
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    eng.step.zero_()
    out, margins = [], []
    for _ in range(N):
        out.append(int(eng.ar_step(anchor)[0]))
        if logits:
            z = np.sort(eng.debug_logits(0, 1, 1)[0, 0].cpu().numpy())
            margins.append(float(z[-1] - z[-2]))
    return out, margins


def _first_diff(a, b):
    for i, (x, y) in enumerate(zip(a, b)):
        if x != y:
            return i
    return -1


@pytest.fixture(scope="module")
def tiny():
    import dual_view_diffusion_b200 as pkg
    w = synth.make_weights(SHAPE, 0)
    eng = pkg.Engine(SHAPE, w, max_batch=1, max_block=16, max_seq=160, split_tokens=64, page_size=16)
    return w, eng


@pytest.mark.parametrize("vocab_shape", ["tiny", "bf16"])
def test_draft_topw_from_epilogue_equals_materialised(tiny, vocab_shape):
    """orthrus_draft_block_topw (top-W inside the LM-head pass) against the
    greedy draft's materialised logits through orthrus_tree_topw: the same
    drafts, ids and logits exactly, log-sum-exps within 1e-5 relative; on
    the tiny fp32 model and on two bf16 layers of the 1.7B shape (151936
    ids, ties included by the integer-valued logits of no row: random)."""
    import dual_view_diffusion_b200 as pkg
    if vocab_shape == "tiny":
        w, eng = tiny
        s, P, K = SHAPE, 16, 8
    else:
        s, P, K = synth.QWEN3_1_7B, 40, 16
        w = synth.make_weights(s, 0, n_layers=2)
        eng = pkg.Engine(s, w, max_batch=1, max_block=K, max_seq=128, split_tokens=64)
    prompt = synth.make_prompt(s, P, 9)
    for W, D in ((1, K - 1), (4, K - 1), (8, K // 2)):
        anchor = eng.prefill(torch.from_numpy(prompt)[None])
        d1, ids1, vals1, lse1 = eng.draft_block_topw(anchor, K, W, D)
        d2 = eng.draft_block(anchor, K)
        z = eng.debug_logits(1, 1, K)[0, :D].contiguous()
        ids2, vals2, lse2 = eng.tree_topw(z, W)
        assert eng.check_error()[0] == 0
        assert torch.equal(d1, d2)
        assert torch.equal(ids1[0], ids2) and torch.equal(vals1[0], vals2), W
        l1, l2 = lse1[0].cpu().numpy(), lse2.cpu().numpy()
        assert (np.abs(l1 - l2) <= 1e-5 * np.maximum(1.0, np.abs(l2))).all(), (l1, l2)


@pytest.mark.parametrize("K,W,nodes", [(8, 3, 12), (6, 2, 15), (4, 4, 9)])
def test_tiny_tree_cycles_match_oracle(tiny, K, W, nodes):
    w, eng = tiny
    N, P = 28, 16
    prompt = synth.make_prompt(SHAPE, P, 1)
    m = oracle.Model(w)
    cap = P + N + nodes + 2
    kc, vc = m.new_cache(cap)
    t = m.prefill(prompt, kc, vc)
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    got, mirror, depths = [], True, []
    while len(got) < N:
        a = int(anchor[0])
        par, tok, R, g, zt, n, emit = _tree_cycle(eng, anchor, K, W, nodes, epilogue_topw=(W != 2))
        depths.append(int(n))
        got += emit
        if not mirror:
            continue
        tk = tok.copy()
        tk[0] = a
        zo = m.forward_tree(tk, par, t, kc, vc)
        assert (np.abs(zt - zo).max(axis=1) <= 1e-4 * np.abs(zo).max(axis=1) + 1e-5).all()
        go = np.zeros(R, np.int32)
        for r in range(R):
            go[r], mg = oracle.argmax(zo[r])
            if go[r] != g[r]:
                assert mg < 1e-4, (r, g[r], go[r], mg)
                mirror = False
        if not mirror:
            continue
        n_o, emit_o, path = oracle.tree_accept(par, tok, go)
        assert n == n_o and emit == emit_o.tolist()
        oracle.tree_commit_kv(kc, vc, t, path)
        t += n_o
    assert eng.check_error()[0] == 0
    got = got[:N]
    # the committed cache against the oracle's compacted one
    if mirror:
        pps = eng.pages_per_seq
        kg = eng.k_pages[:, :pps].permute(0, 1, 3, 2, 4).reshape(eng.n_layers, -1, SHAPE.n_kv_heads, SHAPE.head_dim)
        vg = eng.v_pages[:, :pps].permute(0, 1, 4, 2, 3).reshape(eng.n_layers, -1, SHAPE.n_kv_heads, SHAPE.head_dim)
        tt = int(eng.seq_lens[0])
        assert tt == t
        assert np.abs(kg[:, :t].double().cpu().numpy() - kc[:, :t]).max() <= 1e-5
        assert np.abs(vg[:, :t].double().cpu().numpy() - vc[:, :t]).max() <= 1e-5
    # greedy tree decoding is lossless: the GPU's plain AR stream and the
    # oracle's tree-decoded stream
    ar = m.generate(prompt, K, N, 0.0, 0, "ar")
    gpu_ar, _ = _ar_stream(eng, prompt, N)
    for other in (gpu_ar, oracle.Model(w).generate_tree(prompt, K, W, nodes, N)["tokens"].tolist()):
        i = _first_diff(got, other)
        assert i < 0 or ar["cycle_margin"][i] < 1e-4, (i, got, other)
    assert max(depths) >= 2 or K == 4, depths      # the trees were accepted past their root somewhere


def test_bf16_tree_cycles_match_oracle_and_ar():
    import dual_view_diffusion_b200 as pkg
    s = synth.QWEN3_1_7B
    w = synth.make_weights(s, 0, n_layers=2)
    K, W, nodes, N, P = 8, 2, 15, 24, 64
    eng = pkg.Engine(s, w, max_batch=1, max_block=16, max_seq=256, split_tokens=64)
    m = oracle.Model(w)
    prompt = synth.make_prompt(s, P, 5)
    kc, vc = m.new_cache(P + N + nodes + 2)
    t = m.prefill(prompt, kc, vc)
    eng.step.zero_()
    anchor = eng.prefill(torch.from_numpy(prompt)[None])
    got, checked = [], 0
    while len(got) < N:
        a = int(anchor[0])
        par, tok, R, g, zt, n, emit = _tree_cycle(eng, anchor, K, W, nodes)
        got += emit
        if checked < 2:   # node logits of the first cycles against the oracle (same tree, same cache)
            tk = tok.copy()
            tk[0] = a
            zo = m.forward_tree(tk, par, t, kc, vc)
            rel = np.abs(zt - zo).max(axis=1) / np.abs(zo).max(axis=1)
            assert rel.max() <= 2e-2, rel
            _, _, path = oracle.tree_accept(par, tok, g)
            oracle.tree_commit_kv(kc, vc, t, path)
            t += n
            checked += 1
    assert eng.check_error()[0] == 0
    ar, margins = _ar_stream(eng, prompt, N, logits=True)
    i = _first_diff(got[:N], ar)
    assert i < 0 or margins[i] < 0.05, (i, got, ar, margins[i] if i >= 0 else None)
