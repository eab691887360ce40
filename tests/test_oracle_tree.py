"""Pins of the oracle's tree verification (the paper-notes page on "Orthrus:
Memory-Efficient Parallel Token Generation via Dual-View Diffusion", §7.5:
DDTree expands one diffusion forward's marginals best-first into a tree of
top prefixes and verifies it with tree attention in one pass; §9.6 proposes
the same on Orthrus's K marginals).  Each oracle piece is held against
something other than itself: brute-force enumeration of prefixes, torch's
scaled_dot_product_attention with an explicit ancestor mask, plain causal
forwards of every root path, hand-worked acceptance walks, and the AR
greedy stream (losslessness, §4.2 / §9.1).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def _log_softmax(z):
    z = np.asarray(z, np.float64)
    m = z.max(axis=-1, keepdims=True)
    return z - m - np.log(np.exp(z - m).sum(axis=-1, keepdims=True))


def _brute_force_tree(lp, W, N):
    """Every prefix of depth 1..D over the W best ids per depth (ties: lowest
    id), ordered by score (descending) and then rank sequence; the first N."""
    D, V = lp.shape
    ranked = [sorted(range(V), key=lambda v: (-lp[d][v], v))[:W] for d in range(D)]
    items = []
    for depth in range(1, D + 1):
        for ranks in itertools.product(range(W), repeat=depth):
            toks = tuple(ranked[i][r] for i, r in enumerate(ranks))
            score = 0.0
            for i, tk in enumerate(toks):
                score += lp[i][tk]
            items.append((-score, ranks, toks, score))
    items.sort(key=lambda x: (x[0], x[1]))
    return [(toks, score) for _, _, toks, score in items[:N]]


def _paths(parent, token):
    out = []
    for r in range(len(parent)):
        p, a = [], r
        while a > 0:
            p.append(int(token[a]))
            a = parent[a]
        out.append(tuple(reversed(p)))
    return out


@pytest.mark.parametrize("D,V,W,N,kind", [(3, 7, 3, 10, "normal"), (4, 6, 2, 15, "normal"), (5, 9, 4, 31, "normal"),
                                          (4, 5, 3, 20, "integer ties"), (3, 6, 3, 12, "certain rows")])
def test_tree_build_matches_brute_force(D, V, W, N, kind):
    rng = np.random.default_rng(D * 100 + V * 10 + W)
    if kind == "normal":
        z = rng.standard_normal((D, V)) * 2.0
    elif kind == "integer ties":                      # equal ids in a row and equal path scores
        z = rng.integers(0, 3, size=(D, V)).astype(np.float64)
    else:                                             # a row with probability 1 on one id: log p = 0
        z = rng.standard_normal((D, V))
        z[1, 2] = 1000.0
    lp = _log_softmax(z)
    par, tok, dep, sc = oracle.tree_build(lp, W, N)
    want = _brute_force_tree(lp, W, N)
    assert len(par) == len(want) + 1
    got = _paths(par, tok)[1:]
    assert got == [t for t, _ in want]
    assert list(sc[1:]) == [s for _, s in want]        # same sums in the same order: exact


def test_topw_matches_numpy_and_scipy():
    from scipy.special import logsumexp
    rng = np.random.default_rng(31)
    for z in (rng.standard_normal((4, 300)) * 3.0, rng.integers(-2, 3, size=(4, 50)).astype(np.float64)):
        ids, lse = oracle.topw(z, 6)
        for r in range(z.shape[0]):
            want = np.lexsort((np.arange(z.shape[1]), -z[r]))[:6]    # by value, then lowest id
            assert list(ids[r]) == list(want)
            assert math.isclose(lse[r], float(logsumexp(z[r])), rel_tol=1e-14)


def test_tree_structure_invariants():
    rng = np.random.default_rng(3)
    lp = _log_softmax(rng.standard_normal((6, 11)))
    par, tok, dep, sc = oracle.tree_build(lp, 4, 40)
    assert par[0] == -1 and dep[0] == 0 and sc[0] == 0.0
    paths = _paths(par, tok)
    assert len(set(paths)) == len(paths)               # distinct prefixes
    for r in range(1, len(par)):
        assert 0 <= par[r] < r                         # a parent precedes its children
        assert dep[r] == dep[par[r]] + 1 <= 6
        assert sc[r] <= sc[par[r]]
        assert math.isclose(sc[r], sum(lp[i][t] for i, t in enumerate(paths[r])), rel_tol=0, abs_tol=1e-12)
        assert paths[r][:-1] in paths                  # closed under prefixes
    # fewer prefixes than asked for: all of them
    par2, _, _, _ = oracle.tree_build(lp[:2], 2, 50)
    assert len(par2) == 1 + 2 + 4
    # W = 1: the chain of the rows' argmaxes
    par1, tok1, _, _ = oracle.tree_build(lp, 1, 6)
    assert list(par1) == [-1, 0, 1, 2, 3, 4, 5]
    assert list(tok1[1:]) == [int(np.argmax(lp[d])) for d in range(6)]


def _sdpa_tree(q, kc, vc, kb, vb, parent):
    """torch scaled_dot_product_attention with an explicit ancestor mask."""
    R, nq, hd = q.shape
    nkv = kb.shape[1]
    t = kc.shape[0]
    g = nq // nkv
    keys, vals = np.concatenate([kc, kb]), np.concatenate([vc, vb])
    K = torch.from_numpy(np.repeat(keys, g, axis=1)).permute(1, 0, 2)
    Vv = torch.from_numpy(np.repeat(vals, g, axis=1)).permute(1, 0, 2)
    Q = torch.from_numpy(q).permute(1, 0, 2)
    mask = torch.zeros(R, t + R, dtype=torch.bool)
    mask[:, :t] = True
    for r in range(R):
        a = r
        while a >= 0:
            mask[r, t + a] = True
            a = parent[a]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, Vv, attn_mask=mask)
    return o.permute(1, 0, 2).numpy()


TREE_PARENT = [-1, 0, 0, 1, 2, 2, 3, 0, 5]            # three branches at the root, two under row 2


def test_attention_tree_matches_sdpa_and_chain():
    rng = np.random.default_rng(21)
    nq, nkv, hd, t = 8, 2, 16, 23
    R = len(TREE_PARENT)
    q = rng.standard_normal((R, nq, hd))
    kc, vc = rng.standard_normal((t, nkv, hd)), rng.standard_normal((t, nkv, hd))
    kb, vb = rng.standard_normal((R, nkv, hd)), rng.standard_normal((R, nkv, hd))
    o = oracle.attention_tree(q, kc, vc, kb, vb, TREE_PARENT)
    assert np.allclose(o, _sdpa_tree(q, kc, vc, kb, vb, TREE_PARENT), rtol=1e-12, atol=1e-12)
    # a chain is the causal block mask, key for key
    chain = [-1] + list(range(R - 1))
    assert np.array_equal(oracle.attention_tree(q, kc, vc, kb, vb, chain), oracle.attention(q, kc, vc, kb, vb, 0))
    # every row equals causal attention over its own root path
    for r in range(R):
        path, a = [], r
        while a >= 0:
            path.append(a)
            a = TREE_PARENT[a]
        path = path[::-1]
        oc = oracle.attention(q[path], kc, vc, kb[path], vb[path], 0)
        assert np.array_equal(o[r], oc[-1])


def test_forward_tree_rows_equal_root_path_forwards(tiny_weights, tiny_prompt):
    """Every node's logits and K/V are those of a plain causal AR forward of
    its root path at positions t .. t + depth (positions follow depth, not
    row index; siblings are invisible to one another)."""
    m = oracle.Model(tiny_weights)
    cap = len(tiny_prompt) + 16
    kc, vc = m.new_cache(cap)
    t = m.prefill(tiny_prompt, kc, vc)
    tokens = [int(tiny_prompt[-1]), 11, 12, 40, 41, 42, 7, 200, 3]
    z = m.forward_tree(tokens, TREE_PARENT, t, kc, vc)
    for r in range(len(tokens)):
        path, a = [], r
        while a >= 0:
            path.append(a)
            a = TREE_PARENT[a]
        path = path[::-1]
        k2, v2 = kc.copy(), vc.copy()
        zr = m.forward(0, 0, [tokens[i] for i in path], t, k2, v2)
        assert np.array_equal(z[r], zr[-1])
        d = len(path) - 1
        assert np.array_equal(kc[:, t + r], k2[:, t + d]) and np.array_equal(vc[:, t + r], v2[:, t + d])


def test_tree_accept_worked_examples():
    #   row:     0   1  2  3  4  5  6
    parent = [-1, 0, 0, 1, 2, 3, 3]
    token = [-1, 5, 7, 9, 9, 4, 6]
    # root's argmax 7 -> row 2; row 2's argmax 9 -> row 4; row 4 has no children: emit its argmax 3
    n, emit, path = oracle.tree_accept(parent, token, [7, 0, 9, 0, 3, 0, 0])
    assert (n, list(emit), list(path)) == (3, [7, 9, 3], [0, 2, 4])
    # no child matches at the root: only the AR token
    n, emit, path = oracle.tree_accept(parent, token, [6, 0, 0, 0, 0, 0, 0])
    assert (n, list(emit), list(path)) == (1, [6], [0])
    # the deepest path: 5 -> 9 -> 6, then row 6's argmax 8
    n, emit, path = oracle.tree_accept(parent, token, [5, 9, 0, 6, 0, 0, 8])
    assert (n, list(emit), list(path)) == (4, [5, 9, 6, 8], [0, 1, 3, 6])
    # a chain reduces to the greedy consensus
    rng = np.random.default_rng(2)
    for _ in range(50):
        K = int(rng.integers(1, 9))
        draft = rng.integers(0, 3, K)
        g = rng.integers(0, 3, K)
        chain_tok = [-1] + list(draft[:K - 1])
        n, emit, _ = oracle.tree_accept([-1] + list(range(K - 1)), chain_tok, g)
        n2, emit2 = oracle.consensus_greedy(draft, g)
        assert n == n2 and list(emit) == list(emit2)


def test_tree_commit_kv_moves_the_path():
    rng = np.random.default_rng(8)
    kc = rng.standard_normal((2, 20, 2, 4))
    vc = rng.standard_normal((2, 20, 2, 4))
    k0, v0 = kc.copy(), vc.copy()
    t = 6
    oracle.tree_commit_kv(kc, vc, t, [0, 2, 5, 7])
    for dst, src in ((t + 1, t + 2), (t + 2, t + 5), (t + 3, t + 7)):
        assert np.array_equal(kc[:, dst], k0[:, src]) and np.array_equal(vc[:, dst], v0[:, src])
    untouched = [i for i in range(20) if i not in (t + 1, t + 2, t + 3)]
    assert np.array_equal(kc[:, untouched], k0[:, untouched]) and np.array_equal(vc[:, untouched], v0[:, untouched])


@pytest.mark.parametrize("K", [2, 4, 8])
def test_tree_of_width_one_is_the_orthrus_cycle(tiny_weights, tiny_prompt, K):
    m = oracle.Model(tiny_weights)
    o = m.generate(tiny_prompt, K, 24, 0.0, 0, "orthrus")
    tr = m.generate_tree(tiny_prompt, K, 1, K - 1, 24)
    assert np.array_equal(o["tokens"], tr["tokens"])
    assert np.array_equal(o["n_per_cycle"], tr["n_per_cycle"])


@pytest.mark.parametrize("K,W,nodes", [(4, 2, 3), (4, 3, 7), (8, 2, 12), (8, 4, 20)])
def test_greedy_tree_decoding_equals_ar(tiny_weights, tiny_prompt, K, W, nodes):
    """Lossless: every emitted token is the AR argmax after the accepted
    prefix, and the committed cache is plain AR's, bit for bit."""
    m = oracle.Model(tiny_weights)
    a = m.generate(tiny_prompt, K, 24, 0.0, 0, "ar", want_cache=True)
    tr = m.generate_tree(tiny_prompt, K, W, nodes, 24, want_cache=True)
    assert np.array_equal(a["tokens"], tr["tokens"])
    n = tr["n_per_cycle"]
    assert (n >= 1).all() and (n <= min(K, nodes + 1)).all()
    t = min(a["t"], tr["t"])
    assert np.array_equal(a["k_cache"][:, :t], tr["k_cache"][:, :t])
    assert np.array_equal(a["v_cache"][:, :t], tr["v_cache"][:, :t])


def test_tree_cycle_is_its_retyped_steps(tiny_weights, tiny_prompt):
    """A tree-verified cycle is: the draft at T = 0, numpy's log-softmax of
    its rows 0 .. K-2 (the tokens at depths 1 .. K-1), the best-first tree
    over them, one tree-masked AR forward of the anchor (the root) and the
    nodes, the greedy walk and the K/V compaction.  Retyping four cycles from
    those pinned pieces gives generate_tree's lengths and tokens."""
    m = oracle.Model(tiny_weights)
    K, W, nodes = 6, 3, 10
    kc, vc = m.new_cache(len(tiny_prompt) + 64)
    t = m.prefill(tiny_prompt, kc, vc)
    anchor, out, ns = int(tiny_prompt[-1]), [], []
    for _ in range(4):
        _, _, z, _ = m.draft(kc, vc, t, anchor, K)
        par, tok, _, _ = oracle.tree_build(_log_softmax(z[:K - 1]), W, nodes)
        tok = tok.copy()
        tok[0] = anchor
        g = m.forward_tree(tok, par, t, kc, vc).argmax(axis=1)
        n, emit, path = oracle.tree_accept(par, tok, g)
        oracle.tree_commit_kv(kc, vc, t, path)
        t += n
        anchor = int(emit[-1])
        out += [int(x) for x in emit]
        ns.append(int(n))
    assert max(ns) >= 2                                 # the walk and the compaction do run
    r = m.generate_tree(tiny_prompt, K, W, nodes, len(out))
    assert r["n_per_cycle"][:4].tolist() == ns and r["tokens"].tolist() == out
