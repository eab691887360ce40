"""Tree-verification kernels vs the fp64 oracle (the paper-notes page on
"Orthrus", §7.5: a best-first tree of the top prefixes of one diffusion
forward's marginals, verified in one pass; §9.6).  Decisions are compared
exactly: top-W ids (ties to the lowest id), the tree (parents, tokens,
depths and fp64 scores, built by both sides from the same fp32 candidate
logits and log-sum-exps), the greedy walk, and the committed cache (bit for
bit).  The kernels' own log-sum-exp is held to 1e-5 relative."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _engine(vocab, n_layers=1, max_batch=4, max_block=32, max_seq=512):
    import dual_view_diffusion_b200 as pkg
    s = dataclasses.replace(synth.QWEN3_8B, n_layers=n_layers, hidden=64, ffn=64, vocab=vocab)
    w = synth.make_weights(s, 0, n_layers=n_layers)
    return pkg.Engine(s, w, max_batch=max_batch, max_block=max_block, max_seq=max_seq, split_tokens=128)


@pytest.fixture(scope="module")
def eng_full_vocab():
    e = _engine(synth.QWEN3_8B.vocab)
    yield e
    del e
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def eng_small():
    e = _engine(1000, n_layers=2, max_batch=4, max_block=32, max_seq=640)
    yield e
    del e
    torch.cuda.empty_cache()


def _f32(shape, seed, name, scale=1.0):
    return (synth.normal(shape, scale, seed, name)).astype(np.float32)


@pytest.mark.parametrize("kind", ["normal", "integer ties"])
@pytest.mark.parametrize("W", [1, 4, 8])
def test_topw_matches_oracle(eng_full_vocab, kind, W):
    eng = eng_full_vocab
    V = eng.shape.vocab
    if kind == "normal":
        z = _f32((5, V), 41, "topw", 3.0)
    else:   # many equal logits: ties go to the lowest id
        z = np.floor(_f32((5, V), 42, "topw_ties", 1.5)).astype(np.float32)
    ids, vals, lse = eng.tree_topw(torch.from_numpy(z).cuda(), W)
    assert eng.check_error()[0] == 0
    want_ids, want_lse = oracle.topw(z.astype(np.float64), W)
    ids, vals, lse = ids.cpu().numpy(), vals.cpu().numpy(), lse.cpu().numpy()
    assert np.array_equal(ids, want_ids)
    assert np.array_equal(vals, np.take_along_axis(z, want_ids, axis=1))
    assert (np.abs(lse - want_lse) <= 1e-5 * np.maximum(1.0, np.abs(want_lse))).all()


def test_topw_masked_ids(eng_full_vocab):
    """Masked vocabulary entries (-inf logits, a normal input) leave the
    top-W and a finite log-sum-exp: rows whose leading ids, scattered ids,
    or all but a few ids are -inf (so many threads meet only -inf logits
    before their first finite one)."""
    eng = eng_full_vocab
    V = eng.shape.vocab
    z = _f32((3, V), 44, "topw_masked", 3.0)
    z[0, : V // 2] = -np.inf
    z[1, ::3] = -np.inf
    keep = np.zeros(V, bool)
    keep[[5, 70000, V - 1]] = True
    z[2, ~keep] = -np.inf
    ids, vals, lse = eng.tree_topw(torch.from_numpy(z).cuda(), 3)
    assert eng.check_error()[0] == 0
    want_ids, want_lse = oracle.topw(z.astype(np.float64), 3)
    assert np.array_equal(ids.cpu().numpy(), want_ids)
    assert np.array_equal(vals.cpu().numpy(), np.take_along_axis(z, want_ids, axis=1))
    assert np.isfinite(lse.cpu().numpy()).all()
    assert (np.abs(lse.cpu().numpy() - want_lse) <= 1e-5 * np.maximum(1.0, np.abs(want_lse))).all()


def test_topw_scalar_path():
    """A vocabulary that is not a multiple of 4 takes the kernel's scalar
    loads (the 16-byte path needs whole float4s per row)."""
    eng = _engine(1001)
    z = _f32((3, 1001), 43, "topw_odd", 2.0)
    ids, vals, lse = eng.tree_topw(torch.from_numpy(z).cuda(), 5)
    assert eng.check_error()[0] == 0
    want_ids, want_lse = oracle.topw(z.astype(np.float64), 5)
    assert np.array_equal(ids.cpu().numpy(), want_ids)
    assert np.array_equal(vals.cpu().numpy(), np.take_along_axis(z, want_ids, axis=1))
    assert (np.abs(lse.cpu().numpy() - want_lse) <= 1e-5 * np.maximum(1.0, np.abs(want_lse))).all()
    del eng
    torch.cuda.empty_cache()


@pytest.mark.parametrize("D,W,N", [(7, 2, 7), (7, 4, 20), (31, 3, 31), (5, 8, 60), (3, 2, 40)])
def test_tree_build_matches_oracle(eng_small, D, W, N):
    """Candidates from the GPU top-W kernel (pinned exact above); the
    log-sum-exps both sides use are the oracle's, rounded to fp32; the
    oracle's rows are then log q = z - lse in fp64, as the kernel forms them."""
    eng = eng_small
    B, V = 3, eng.shape.vocab
    z = _f32((B, D, V), 50 + D * 10 + W, "tree_z", 2.0)
    _, lse64 = oracle.topw(z.reshape(-1, V).astype(np.float64), 1)
    lse32 = lse64.astype(np.float32).reshape(B, D)
    ids, vals, _ = eng.tree_topw(torch.from_numpy(z).cuda(), W)
    par, tok, dep, sc, nr = eng.tree_build(ids.view(B, D, W), vals.view(B, D, W), torch.from_numpy(lse32).cuda(), N)
    assert eng.check_error()[0] == 0
    par, tok, dep, sc, nr = (x.cpu().numpy() for x in (par, tok, dep, sc, nr))
    for b in range(B):
        logp = z[b].astype(np.float64) - lse32[b].astype(np.float64)[:, None]
        wp, wt, wd, ws = oracle.tree_build(logp, W, N)
        n = len(wp)
        assert nr[b] == n
        assert np.array_equal(par[b, :n], wp) and np.array_equal(tok[b, :n], wt)
        assert np.array_equal(dep[b, :n], wd) and np.array_equal(sc[b, :n], ws)
        assert (par[b, n:] == -1).all() and (tok[b, n:] == -1).all()


def _positions(eng, pages, b, transposed):
    """Cache of sequence b as [layer, position, kv head, dim] (float64)."""
    pps = eng.pages_per_seq
    x = pages[:, b * pps:(b + 1) * pps].float()
    x = x.permute(0, 1, 4, 2, 3) if transposed else x.permute(0, 1, 3, 2, 4)
    return np.ascontiguousarray(x.reshape(x.shape[0], -1, x.shape[3], x.shape[4]).cpu().numpy(), np.float64)


def test_tree_commit_matches_oracle(eng_small):
    """Three sequences (one tree crossing a page boundary, one root-only
    tree, one deep acceptance): n, the emitted tokens, the anchor, the
    lengths and the whole cache of both layers against oracle.tree_accept
    and oracle.tree_commit_kv."""
    eng = eng_small
    B, R, V = 3, 16, eng.shape.vocab
    g0 = torch.Generator(device="cuda").manual_seed(6)
    for p in (eng.k_pages, eng.v_pages):
        p.copy_(torch.randn(p.shape, generator=g0, device="cuda").to(p.dtype))
    rng = np.random.Generator(np.random.Philox(key=61))
    ts = [58, 100, 300]                     # 58 + 16 rows crosses the 64-slot page
    parents, tokens, gs, nrows = [], [], [], []
    for b in range(B):
        z = rng.standard_normal((8, V)) * (6.0 if b == 2 else 2.0)   # sharper marginals: a deeper tree
        m = z.max(1, keepdims=True)
        lp = z - m - np.log(np.exp(z - m).sum(1, keepdims=True))
        wp, wt, _, _ = oracle.tree_build(lp, 3, R - 1)
        n_b = 1 if b == 1 else len(wp)
        par = np.full(R, -1, np.int32); tok = np.full(R, -1, np.int32)
        par[:len(wp)], tok[:len(wp)] = wp, wt
        g = rng.integers(0, V, R).astype(np.int32)
        follow = 1.0 if b == 2 else 0.6
        for r in range(n_b):                 # steer the AR argmax onto a child (always, for b = 2)
            kids = [c for c in range(r + 1, n_b) if par[c] == r]
            if kids and rng.random() < follow:
                g[r] = tok[kids[int(rng.integers(0, len(kids)))]]
        parents.append(par); tokens.append(tok); gs.append(g); nrows.append(n_b)
    par_h, tok_h, g_h = np.stack(parents), np.stack(tokens), np.stack(gs)
    eng.seq_lens.zero_()
    eng.seq_lens[:B] = torch.tensor(ts, dtype=torch.int32)
    before_k = [_positions(eng, eng.k_pages, b, False) for b in range(B)]
    before_v = [_positions(eng, eng.v_pages, b, True) for b in range(B)]
    anchor = torch.zeros(B, dtype=torch.int32, device="cuda")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    n, emit = eng.tree_commit(dev(par_h), dev(tok_h), dev(np.array(nrows, np.int32)), dev(g_h), anchor)
    assert eng.check_error()[0] == 0
    n, emit, anchor = n.cpu().numpy(), emit.cpu().numpy(), anchor.cpu().numpy()
    lens = eng.seq_lens[:B].cpu().numpy()
    depths = []
    for b in range(B):
        wn, we, wpath = oracle.tree_accept(par_h[b, :nrows[b]], tok_h[b, :nrows[b]], g_h[b, :nrows[b]])
        depths.append(wn)
        assert n[b] == wn and np.array_equal(emit[b, :wn], we) and anchor[b] == we[-1]
        assert lens[b] == ts[b] + wn
        kc, vc = before_k[b].copy(), before_v[b].copy()
        oracle.tree_commit_kv(kc, vc, ts[b], wpath)
        assert np.array_equal(_positions(eng, eng.k_pages, b, False), kc)
        assert np.array_equal(_positions(eng, eng.v_pages, b, True), vc)
    assert depths == [3, 1, 6], depths       # the third path is rows 0, 1, 5, 7, 9, 15


def test_tree_commit_flags_a_malformed_parent(eng_small):
    """A parent row at or after its child is refused by the kernel's own
    check (ORTHRUS_DEVERR_TOKEN); the walk stops there, nothing is read
    out of bounds."""
    eng = eng_small
    eng.seq_lens.zero_()
    eng.seq_lens[0] = 10
    par = np.array([[-1, 0, 5, 1]], np.int32)
    tok = np.array([[-1, 3, 4, 5]], np.int32)
    g = np.array([[7, 0, 0, 0]], np.int32)
    dev = lambda a: torch.from_numpy(a).cuda()
    anchor = torch.zeros(1, dtype=torch.int32, device="cuda")
    eng.tree_commit(dev(par), dev(tok), dev(np.array([4], np.int32)), dev(g), anchor)
    st, bits = eng.check_error()
    assert st != 0 and bits & 0x1
