"""Dual-view attention kernel vs the fp64 oracle (paper notes §3.2: prefix
plus bidirectional block for the diffusion view; §4.1 step 2: causal block for
AR verification).  Inputs are N(0, 1) bf16 values (seed 2), the Qwen3-8B
attention shape (32 query / 8 KV heads, head_dim 128).  Tolerance: 1e-2
max-abs on the bf16 output."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import attention_engine, bf16_normal, write_cache

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module")
def eng():
    return attention_engine()


def _case(eng, ts, K, mode, seed=2, tag="", check=None):
    """ts: committed length per sequence.  Returns max-abs error over the
    sequences in `check` (default all) and the GPU output."""
    B = len(ts)
    nq, nkv, hd = 32, 8, 128
    q = bf16_normal((B, K, nq, hd), seed, f"q{tag}")
    kb = bf16_normal((B, K, nkv, hd), seed, f"kb{tag}")
    vb = bf16_normal((B, K, nkv, hd), seed, f"vb{tag}")
    kcs, vcs = [], []
    for b, t in enumerate(ts):
        kc = bf16_normal((t, nkv, hd), seed, f"kc{tag}{b}")
        vc = bf16_normal((t, nkv, hd), seed, f"vc{tag}{b}")
        write_cache(eng, 0, b, kc, vc)
        if mode == 0:     # the verify block's own rows live in the cache tail
            write_cache(eng, 0, b, kb[b], vb[b], start=t)
        kcs.append(kc); vcs.append(vc)
    eng.seq_lens[:B] = torch.tensor(ts, dtype=torch.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    out = eng.attention(0, mode, dev(q), dev(kb), dev(vb), B, K).float().cpu().numpy()
    st, bits = eng.check_error()
    assert st == 0, bits
    err = 0.0
    for b, t in enumerate(ts):
        if check is not None and b not in check:
            continue
        ref = oracle.attention(q[b], kcs[b] if t else None, vcs[b] if t else None, kb[b], vb[b], mode)
        err = max(err, float(np.abs(out[b] - ref).max()))
    return err, out


@pytest.mark.parametrize("mode", [0, 1])
def test_config2_layer(eng, mode):
    """L = 4096 committed keys, K = 32 block rows, batch 1."""
    err, _ = _case(eng, [4096], 32, mode)
    assert err <= TOL, err


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("t,K", [(0, 1), (0, 5), (37, 4), (63, 8), (64, 8), (65, 8), (255, 1), (256, 32),
                                 (1000, 16), (4133, 32), (7000, 3)])
def test_edges(eng, mode, t, K):
    err, _ = _case(eng, [t], K, mode, tag=f"e{t}_{K}")
    assert err <= TOL, err


@pytest.mark.parametrize("mode", [0, 1])
def test_ragged_batch(eng, mode):
    err, _ = _case(eng, [100, 1000, 257], 16, mode, tag="rag")
    assert err <= TOL, err


@pytest.fixture(scope="module")
def eng16():
    e = attention_engine(max_batch=16, max_seq=8192 + 32 + 64, split_tokens=128)
    yield e
    del e
    torch.cuda.empty_cache()


@pytest.mark.parametrize("mode", [0, 1])
def test_batch16_long_context(eng16, mode):
    """The benchmark's batched long-context cell in its launch configuration:
    16 sequences at L = 8192 with K = 32 (split 128: one CTA per sequence
    and KV head); the first, a middle and the last sequence are checked
    against the oracle, so a per-sequence offset error shows."""
    err, _ = _case(eng16, [8192] * 16, 32, mode, tag="b16", check=(0, 7, 15))
    assert err <= TOL, err


def test_rows_independent_of_block(eng):
    """A verify row gives bit-identical output whether it sits in a block of
    K = 32 or is the only row at that position (splits aligned to absolute
    positions, masked keys contribute exact zeros)."""
    t, K = 3000, 32
    nq, nkv, hd = 32, 8, 128
    q = bf16_normal((1, K, nq, hd), 5, "iq")
    kb = bf16_normal((1, K, nkv, hd), 5, "ikb")
    vb = bf16_normal((1, K, nkv, hd), 5, "ivb")
    kc = bf16_normal((t, nkv, hd), 5, "ikc"); vc = bf16_normal((t, nkv, hd), 5, "ivc")
    write_cache(eng, 0, 0, kc, vc)
    write_cache(eng, 0, 0, kb[0], vb[0], start=t)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    eng.seq_lens[0] = t
    full = eng.attention(0, 0, dev(q), dev(kb), dev(vb), 1, K)
    for k in (0, 7, 31):
        eng.seq_lens[0] = t + k
        one = eng.attention(0, 0, dev(q[:, k:k + 1]), dev(kb[:, k:k + 1]), dev(vb[:, k:k + 1]), 1, 1)
        assert torch.equal(one[0, 0], full[0, k]), k
