"""The allocation-free dual-view attention entry point.

Some users of this library cannot give it a workspace: a serving runtime that
has already reserved all of HBM for its own pool, or code on a path where a
cudaMalloc/cudaFree (which synchronise the device) is not acceptable.  For
them, orthrus_dual_view_attention_noalloc runs the same attention kernels with
their scratch in a fixed array the library holds on the GPU.  This file checks,
through the C ABI, that it gives the same output as the workspace-based entry
point on two calls in a row (so nothing left over from the first call leaks
into the second), and that a request too large for the fixed array is refused
before anything is launched.  It lives in its own file, collected last, and
works alone in a fresh process as well as after the other tests.
"""
import ctypes as C
import dataclasses
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_helpers import attention_engine, bf16_normal, write_cache  # noqa: E402

pytestmark = pytest.mark.gpu
TOL = 1e-2     # the attention tests' max-abs tolerance


def _inputs(eng, ts, K, mode, tag):
    B = len(ts)
    nq, nkv, hd = 32, 8, 128
    q = bf16_normal((B, K, nq, hd), 11, f"na.q{tag}")
    kb = bf16_normal((B, K, nkv, hd), 11, f"na.kb{tag}")
    vb = bf16_normal((B, K, nkv, hd), 11, f"na.vb{tag}")
    for b, t in enumerate(ts):
        write_cache(eng, 0, b, bf16_normal((t, nkv, hd), 11, f"na.kc{tag}{b}"),
                    bf16_normal((t, nkv, hd), 11, f"na.vc{tag}{b}"))
        if mode == 0:
            write_cache(eng, 0, b, kb[b], vb[b], start=t)
    eng.seq_lens[:B] = torch.tensor(ts, dtype=torch.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    return dev(q), dev(kb), dev(vb)


def _noalloc(pkg, eng, cfg, mode, q, kb, vb, B, K, err):
    out = torch.empty_like(q)
    st = pkg.lib().orthrus_dual_view_attention_noalloc(
        C.byref(cfg), C.byref(eng.kv), 0, mode, C.c_void_p(q.data_ptr()), C.c_void_p(kb.data_ptr()),
        C.c_void_p(vb.data_ptr()), B, K, C.c_void_p(out.data_ptr()), C.c_void_p(err.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def test_noalloc_matches_workspace_entry_point_twice():
    import dual_view_diffusion_b200 as pkg
    eng = attention_engine()
    # same model shape; a max_seq that keeps the split partials inside the
    # fixed array (the outputs do not depend on max_seq)
    cfg = pkg.Config.from_buffer_copy(eng.cfg)
    cfg.max_seq = 4096 + 64
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = [([4096], 32, 1, "a"), ([1000, 37], 16, 0, "b")]     # two calls in a row, different shapes
    for ts, K, mode, tag in cases:
        q, kb, vb = _inputs(eng, ts, K, mode, tag)
        ref = eng.attention(0, mode, q, kb, vb, len(ts), K)
        st, out = _noalloc(pkg, eng, cfg, mode, q, kb, vb, len(ts), K, err)
        torch.cuda.synchronize()
        assert st == 0, st
        assert int(err.item()) == 0
        d = (out.float() - ref.float()).abs().max().item()
        assert d <= TOL, (tag, d)
        assert torch.isfinite(out.float()).all()


def test_noalloc_refuses_oversize_request():
    import dual_view_diffusion_b200 as pkg
    eng = attention_engine()
    cfg = pkg.Config.from_buffer_copy(eng.cfg)
    K = 4096                                     # a block whose repacked K/V exceed the fixed array
    cfg.max_seq = 1 << 20
    q = torch.zeros((1, K, 32, 128), dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros((1, K, 8, 128), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st, _ = _noalloc(pkg, eng, cfg, 1, q, kb, kb.clone(), 1, K, err)
    assert st == 3        # ORTHRUS_ERR_CAPACITY, nothing launched
