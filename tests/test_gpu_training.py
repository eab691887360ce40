"""GPU parity of the training-side kernels (paper notes §3.1-§3.3): the
dual-pass block-masked attention of a packed training sequence and the
forward-KL LM-head epilogue, through the C-ABI entry points
orthrus_block_mask_attention and orthrus_kl_lm_head, against the CPU oracle
on the same seeded bf16 inputs."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import attention_engine, write_cache

pytestmark = pytest.mark.gpu

ATOL_ATTN = 1e-2     # attention outputs, max-abs (bf16 in, bf16 out)


def _bf16(a):
    return synth.round_bf16(np.asarray(a, np.float32))


def _dev(a, eng):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(eng.device, eng.tdtype)


def _block_case(seed, n_blocks, K, L, n_q, n_kv, hd, anchors=None):
    rng = np.random.default_rng(seed)
    q = _bf16(rng.standard_normal((n_blocks * K, n_q, hd)))
    kc, vc = _bf16(rng.standard_normal((L, n_kv, hd))), _bf16(rng.standard_normal((L, n_kv, hd)))
    kb, vb = _bf16(rng.standard_normal((n_blocks * K, n_kv, hd))), _bf16(rng.standard_normal((n_blocks * K, n_kv, hd)))
    if anchors is None:
        anchors = rng.integers(0, L - K + 1, n_blocks)
    return q, kc, vc, kb, vb, np.asarray(anchors, np.int32)


def _run_block_mask(eng, q, kc, vc, kb, vb, anchors, K):
    n_q, hd = q.shape[1], q.shape[2]
    n_kv = kb.shape[1]
    nb = anchors.size
    write_cache(eng, 0, 0, kc, vc)            # the packed context on block-table row 0
    qd = _dev(q, eng).reshape(nb, K, n_q, hd)
    kd = _dev(kb, eng).reshape(nb, K, n_kv, hd)
    vd = _dev(vb, eng).reshape(nb, K, n_kv, hd)
    ad = torch.from_numpy(anchors).to(eng.device)
    out = eng.block_mask_attention(0, qd, kd, vd, ad, K)
    torch.cuda.synchronize()
    assert eng.check_error()[1] == 0
    return out.float().cpu().numpy().reshape(nb * K, n_q, hd)


def test_block_mask_attention_matches_oracle_small():
    # 8 blocks of K = 32 over a 512-position context, anchors at both ends
    # and in between, GQA group 4, several tiles and a ragged last tile
    n_blocks, K, L, n_q, n_kv, hd = 8, 32, 512, 8, 2, 128
    q, kc, vc, kb, vb, a = _block_case(21, n_blocks, K, L, n_q, n_kv, hd,
                                       anchors=[0, 1, 63, 64, 200, 333, 479, 512])
    eng = attention_engine(n_q=n_q, n_kv=n_kv, hd=hd, max_batch=n_blocks, max_block=K, max_seq=L + 64,
                           split_tokens=128)
    got = _run_block_mask(eng, q, kc, vc, kb, vb, a, K)
    want = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    assert np.abs(got - want).max() < ATOL_ATTN


def test_block_mask_attention_training_shape_sampled():
    # the pages' training layout: 256 anchor blocks of K = 32 in one packed
    # sequence of L = 2048 (blocks overlap, and never see one another), the
    # 8B attention shape; sampled blocks checked against the oracle
    n_blocks, K, L, n_q, n_kv, hd = 256, 32, 2048, 32, 8, 128
    q, kc, vc, kb, vb, a = _block_case(22, n_blocks, K, L, n_q, n_kv, hd)
    a[0], a[1], a[2] = 0, L - K, 1
    eng = attention_engine(n_q=n_q, n_kv=n_kv, hd=hd, max_batch=128, max_block=K, max_seq=L + 64,
                           split_tokens=128)   # two launches of 128 blocks
    got = _run_block_mask(eng, q, kc, vc, kb, vb, a, K)
    for b in (0, 1, 2, 17, 127, 128, 255):
        s = slice(b * K, (b + 1) * K)
        want = oracle.block_mask_attention(q[s], kc, vc, kb[s], vb[s], a[b:b + 1], K)
        assert np.abs(got[s] - want).max() < ATOL_ATTN, b


def test_block_mask_attention_is_the_diffusion_view_per_block():
    # one block through the training entry point == the decode-time
    # diffusion-view attention of a sequence whose cache is the context
    # prefix before the anchor (same kernel, same inputs): bitwise
    K, L, n_q, n_kv, hd = 32, 256, 8, 2, 128
    q, kc, vc, kb, vb, a = _block_case(23, 1, K, L, n_q, n_kv, hd, anchors=[150])
    eng = attention_engine(n_q=n_q, n_kv=n_kv, hd=hd, max_batch=1, max_block=K, max_seq=L + 64, split_tokens=128)
    got = _run_block_mask(eng, q, kc, vc, kb, vb, a, K)
    eng.seq_lens[0] = 150
    ref = eng.attention(0, 1, _dev(q, eng).reshape(1, K, n_q, hd), _dev(kb, eng).reshape(1, K, n_kv, hd),
                        _dev(vb, eng).reshape(1, K, n_kv, hd), 1, K)
    torch.cuda.synchronize()
    assert np.array_equal(got, ref.float().cpu().numpy().reshape(K, n_q, hd))


def _kl_engine(vocab, hidden, max_batch=1, max_block=32):
    import dual_view_diffusion_b200 as pkg
    s = dataclasses.replace(synth.QWEN3_8B, n_layers=1, hidden=hidden, n_q_heads=8, n_kv_heads=2, head_dim=128,
                            ffn=64, vocab=vocab)
    w = synth.make_weights(s, 0, n_layers=1)
    eng = pkg.Engine(s, w, max_batch=max_batch, max_block=max_block, max_seq=256, split_tokens=128)
    return eng, w.lm_head


def _kl_rows(seed, rows, hidden, spread=3.0, noise=0.6):
    rng = np.random.default_rng(seed)
    hA = _bf16(spread * rng.standard_normal((rows, hidden)))
    hD = _bf16(hA + noise * spread * rng.standard_normal((rows, hidden)))
    return hA, hD


@pytest.mark.parametrize("vocab,hidden,rows", [(1000, 256, 16), (32000, 512, 5)])
def test_kl_lm_head_matches_oracle(vocab, hidden, rows):
    # several vocabulary tiles and a ragged last one (1000 = 7 x 128 + 104),
    # row counts that leave a partial token tile
    eng, W = _kl_engine(vocab, hidden)
    hA, hD = _kl_rows(31, rows, hidden)
    kl, la, ld = eng.kl_lm_head(_dev(hA, eng), _dev(hD, eng))
    torch.cuda.synchronize()
    assert eng.check_error()[1] == 0
    kl_o, la_o, ld_o = oracle.kl_rows(hA, hD, W)
    kl, la, ld = kl.cpu().numpy(), la.cpu().numpy(), ld.cpu().numpy()
    assert np.all(kl_o > 0.05)
    assert np.all(np.abs(kl - kl_o) <= 2e-2 * kl_o + 2e-3), (kl, kl_o)
    assert np.allclose(la, la_o, rtol=1e-4, atol=1e-3) and np.allclose(ld, ld_o, rtol=1e-4, atol=1e-3)


def test_kl_lm_head_full_vocabulary():
    # the 8B head's vocabulary (151936 = 1187 tiles of 128) over 4 row pairs
    eng, W = _kl_engine(151936, 1024)
    hA, hD = _kl_rows(32, 4, 1024)
    kl, la, ld = eng.kl_lm_head(_dev(hA, eng), _dev(hD, eng))
    torch.cuda.synchronize()
    kl_o, la_o, ld_o = oracle.kl_rows(hA, hD, W)
    kl = kl.cpu().numpy()
    assert np.all(np.abs(kl - kl_o) <= 2e-2 * kl_o + 2e-3), (kl, kl_o)
    assert np.allclose(la.cpu().numpy(), la_o, rtol=1e-4, atol=1e-3)


def test_kl_lm_head_identical_views_is_zero():
    eng, _ = _kl_engine(5000, 256)
    hA, _ = _kl_rows(33, 8, 256)
    kl, la, ld = eng.kl_lm_head(_dev(hA, eng), _dev(hA, eng))
    torch.cuda.synchronize()
    assert np.all(kl.cpu().numpy() == 0.0)
    assert torch.equal(la, ld)


def test_block_mask_attention_ragged_shapes():
    # short blocks (K = 8: one partial subtile), a context that is not a
    # multiple of the tile (L = 300), anchors at 0 and at L, more blocks than
    # one launch holds (7 blocks, max_batch 5: launches of 5 and 2)
    n_blocks, K, L, n_q, n_kv, hd = 7, 8, 300, 16, 4, 128
    q, kc, vc, kb, vb, a = _block_case(24, n_blocks, K, L, n_q, n_kv, hd, anchors=[300, 0, 64, 65, 127, 128, 299])
    eng = attention_engine(n_q=n_q, n_kv=n_kv, hd=hd, max_batch=5, max_block=16, max_seq=L + 64, split_tokens=128)
    got = _run_block_mask(eng, q, kc, vc, kb, vb, a, K)
    want = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    assert np.abs(got - want).max() < ATOL_ATTN


def test_kl_lm_head_single_row_ragged_vocab():
    # one row pair, a vocabulary of 129 ids (a full tile plus one id)
    eng, W = _kl_engine(129, 256)
    hA, hD = _kl_rows(34, 1, 256)
    kl, la, ld = eng.kl_lm_head(_dev(hA, eng), _dev(hD, eng))
    torch.cuda.synchronize()
    kl_o, la_o, ld_o = oracle.kl_rows(hA, hD, W)
    assert abs(float(kl[0]) - kl_o[0]) <= 2e-2 * kl_o[0] + 2e-3
    assert np.allclose(la.cpu().numpy(), la_o, rtol=1e-4, atol=1e-3)
    assert np.allclose(ld.cpu().numpy(), ld_o, rtol=1e-4, atol=1e-3)


def test_training_entry_points_fp32_tiny():
    # the same two entry points on the fp32 tiny shape (4/2 heads, head_dim 16,
    # vocab 256): the SIMT attention and SIMT GEMM paths
    import dual_view_diffusion_b200 as pkg
    s = synth.TINY
    w = synth.make_weights(s, 0)
    eng = pkg.Engine(s, w, max_batch=4, max_block=8, max_seq=128, split_tokens=64, page_size=16)
    n_blocks, K, L = 6, 4, 40
    rng = np.random.default_rng(25)
    q = rng.standard_normal((n_blocks * K, s.n_q_heads, s.head_dim)).astype(np.float32)
    kc = rng.standard_normal((L, s.n_kv_heads, s.head_dim)).astype(np.float32)
    vc = rng.standard_normal((L, s.n_kv_heads, s.head_dim)).astype(np.float32)
    kb = rng.standard_normal((n_blocks * K, s.n_kv_heads, s.head_dim)).astype(np.float32)
    vb = rng.standard_normal((n_blocks * K, s.n_kv_heads, s.head_dim)).astype(np.float32)
    a = np.array([0, 5, 16, 17, 39, 40], np.int32)
    got = _run_block_mask(eng, q, kc, vc, kb, vb, a, K)
    want = oracle.block_mask_attention(q, kc, vc, kb, vb, a, K)
    assert np.abs(got - want).max() < 1e-4
    hA = 2.0 * rng.standard_normal((3, s.hidden)).astype(np.float32)
    hD = (hA + 1.0 * rng.standard_normal((3, s.hidden))).astype(np.float32)
    kl, la, ld = eng.kl_lm_head(_dev(hA, eng), _dev(hD, eng))
    torch.cuda.synchronize()
    kl_o, la_o, ld_o = oracle.kl_rows(hA, hD, w.lm_head)
    assert np.allclose(kl.cpu().numpy(), kl_o, rtol=1e-4, atol=1e-6)
    assert np.allclose(la.cpu().numpy(), la_o, rtol=1e-5, atol=1e-5)
    assert np.allclose(ld.cpu().numpy(), ld_o, rtol=1e-5, atol=1e-5)
