"""The allocation-free dual-view attention entry point.

Some users of this library cannot give it a workspace: a serving runtime that
has already reserved all of HBM for its own pool, or code on a path where a
cudaMalloc/cudaFree (which synchronise the device) is not acceptable.  For
them, orthrus_dual_view_attention_noalloc runs the same attention kernels with
their scratch in a fixed array the library holds on the GPU.  This file checks,
through the C ABI, on two calls in a row (so nothing left over from the first
call leaks into the second):

* that its output is bit-identical to the workspace-based entry point's for
  the same config — it launches the same kernels with the same shapes — on
  the tensor-core path (short contexts, and long ones where a row group is
  spread over several clusters) and on the SIMT path (fp32, and a bf16 shape
  whose query-head group does not divide 128), and within the attention
  tests' 1e-2 of the fp64 oracle;
* that requests whose scratch does not fit the fixed array (the repacked block
  K/V, or the SIMT split partials) are refused before anything is launched.

It lives in its own file, collected last, and works alone in a fresh process
as well as after the other tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import attention_engine, bf16_normal, write_cache

pytestmark = pytest.mark.gpu
TOL = 1e-2     # the attention tests' max-abs tolerance against the oracle


def _inputs(eng, ts, K, mode, tag, nq, nkv, hd):
    B = len(ts)
    q = bf16_normal((B, K, nq, hd), 11, f"na.q{tag}")
    kb = bf16_normal((B, K, nkv, hd), 11, f"na.kb{tag}")
    vb = bf16_normal((B, K, nkv, hd), 11, f"na.vb{tag}")
    kcs, vcs = [], []
    for b, t in enumerate(ts):
        kc, vc = bf16_normal((t, nkv, hd), 11, f"na.kc{tag}{b}"), bf16_normal((t, nkv, hd), 11, f"na.vc{tag}{b}")
        write_cache(eng, 0, b, kc, vc)
        if mode == 0:
            write_cache(eng, 0, b, kb[b], vb[b], start=t)
        kcs.append(kc); vcs.append(vc)
    eng.seq_lens[:B] = torch.tensor(ts, dtype=torch.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(eng.tdtype)
    return (q, kb, vb, kcs, vcs), (dev(q), dev(kb), dev(vb))


def _noalloc(pkg, eng, cfg, mode, q, kb, vb, B, K, err):
    out = torch.empty_like(q)
    st = pkg.lib().orthrus_dual_view_attention_noalloc(
        C.byref(cfg), C.byref(eng.kv), 0, mode, C.c_void_p(q.data_ptr()), C.c_void_p(kb.data_ptr()),
        C.c_void_p(vb.data_ptr()), B, K, C.c_void_p(out.data_ptr()), C.c_void_p(err.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _run_pair(eng, cases, nq, nkv, hd):
    """Each case through both entry points, in a row: bitwise equal, and
    within TOL of the oracle."""
    import dual_view_diffusion_b200 as pkg
    cfg = pkg.Config.from_buffer_copy(eng.cfg)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for ts, K, mode, tag in cases:
        host, (q, kb, vb) = _inputs(eng, ts, K, mode, tag, nq, nkv, hd)
        ref = eng.attention(0, mode, q, kb, vb, len(ts), K)
        assert eng.check_error()[0] == 0
        st, out = _noalloc(pkg, eng, cfg, mode, q, kb, vb, len(ts), K, err)
        torch.cuda.synchronize()
        assert st == 0, (tag, st)
        assert int(err.item()) == 0, tag
        assert torch.equal(out, ref), (tag, (out.float() - ref.float()).abs().max().item())
        qh, kbh, vbh, kcs, vcs = host
        o = out.float().cpu().numpy()
        for b, t in enumerate(ts):
            r = oracle.attention(qh[b], kcs[b] if t else None, vcs[b] if t else None, kbh[b], vbh[b], mode)
            d = float(np.abs(o[b] - r).max())
            assert d <= TOL, (tag, b, d)


def test_noalloc_tensor_core_path_twice():
    """The 8B attention shape (32/8 heads, head_dim 128, bf16): one cluster
    per row group (max_seq < 8192)."""
    eng = attention_engine(max_seq=4096 + 64)
    _run_pair(eng, [([4000], 32, 1, "a"), ([1000, 37], 16, 0, "b")], 32, 8, 128)


def test_noalloc_long_context_clusters_twice():
    """max_seq >= 8192: both entry points spread a row group over several
    clusters merged through memory (the merge tickets live in the fixed
    array and must start at zero on every call)."""
    eng = attention_engine(max_batch=2, max_seq=12288 + 64)
    _run_pair(eng, [([9000], 32, 1, "c"), ([12000, 700], 8, 0, "d")], 32, 8, 128)


def test_noalloc_simt_fp32_twice():
    """fp32 (the SIMT kernel and its split combine; its partials are the
    scratch here)."""
    eng = attention_engine(n_q=4, n_kv=2, hd=16, max_seq=2048, split_tokens=64, page_size=16, dtype="fp32")
    _run_pair(eng, [([1500], 4, 1, "e"), ([700, 33], 3, 0, "f")], 4, 2, 16)


def test_noalloc_simt_bf16_group_not_dividing_128_twice():
    """24 query heads over 8 KV heads (group 3 does not divide the 128-row
    tile): bf16 head_dim 128 on the SIMT path; its partials (32 rows x 24
    heads x 18 splits x 520 B = 7.2 MB) are a large share of the fixed
    array."""
    eng = attention_engine(n_q=24, n_kv=8, max_batch=2, max_block=32, max_seq=4096 + 64, split_tokens=256)
    _run_pair(eng, [([4000], 32, 1, "g"), ([2000, 999], 16, 0, "h")], 24, 8, 128)


def test_noalloc_refuses_oversize_requests():
    import dual_view_diffusion_b200 as pkg
    eng = attention_engine()
    cfg = pkg.Config.from_buffer_copy(eng.cfg)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a block whose repacked K/V alone exceed the fixed array
    K = 4096
    cfg.max_seq = 1 << 20
    q = torch.zeros((1, K, 32, 128), dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros((1, K, 8, 128), dtype=torch.bfloat16, device="cuda")
    st, _ = _noalloc(pkg, eng, cfg, 1, q, kb, kb.clone(), 1, K, err)
    assert st == 3        # ORTHRUS_ERR_CAPACITY, nothing launched
    # SIMT split partials beyond the array: 24/8 heads (group 3), 32 rows,
    # ceil(4160 / 64) + 1 = 66 splits -> 32 * 24 * 66 * (128 * 4 + 8) B = 26.4 MB
    e24 = attention_engine(n_q=24, n_kv=8, max_seq=4096 + 64)
    cfg = pkg.Config.from_buffer_copy(e24.cfg)
    cfg.split_tokens = 64
    q = torch.zeros((1, 32, 24, 128), dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros((1, 32, 8, 128), dtype=torch.bfloat16, device="cuda")
    e24.seq_lens[0] = 100
    st, _ = _noalloc(pkg, e24, cfg, 0, q, kb, kb, 1, 32, err)
    assert st == 3
    torch.cuda.synchronize()
