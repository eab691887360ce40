"""The C-ABI library loads, exports every entry point its header declares,
and rejects bad arguments on the host (no GPU needed for any of this)."""
import ctypes as C
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"\b(orthrus_[a-z_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def pkg():
    from dual_view_diffusion_b200 import build
    build.build()
    import dual_view_diffusion_b200 as p
    return p


def test_every_declared_symbol_is_exported(pkg):
    lib = pkg.lib()
    names = _declared()
    assert {"orthrus_prefill", "orthrus_draft_block", "orthrus_verify_block", "orthrus_commit",
            "orthrus_generate"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(pkg):
    lib = pkg.lib()
    for s in range(7):
        assert lib.orthrus_status_string(s)
    assert lib.orthrus_status_string(99) == b"unknown status"


def test_transient_bytes_is_the_pages_figure(pkg):
    """Paper notes §2.3/§9.5: the diffusion view's transient K/V for the
    Qwen3-8B shape at K = 32 is about 4.5 MiB: 36 layers x 32 rows x 8 KV
    heads x 128 dims x (K and V) x 2 bytes = 4,718,592 B, and it does not
    depend on the sequence length."""
    for max_seq in (2048, 8192, 32768, 131072):
        cfg = pkg.make_config(synth.QWEN3_8B, "bf16", 1, 32, max_seq)
        assert pkg.orthrus_transient_bytes(cfg, 1, 32) == 4718592 == 4.5 * 2 ** 20
    cfg = pkg.make_config(synth.QWEN3_1_7B, "bf16", 1, 32, 4096)
    assert pkg.orthrus_transient_bytes(cfg, 1, 32) == 28 * 32 * 8 * 128 * 2 * 2   # 3.5 MiB
    cfg = pkg.make_config(synth.TINY, "fp32", 1, 4, 128)
    assert pkg.orthrus_transient_bytes(cfg, 1, 4) == 2 * 4 * 2 * 16 * 2 * 4        # 2 KiB


def test_workspace_independent_of_sequence_length(pkg):
    """Paper notes §2.3 / §9.5: the diffusion view's transient memory does
    not grow with the sequence length.  On the bf16 tensor-core path the
    whole workspace is the same for a context sized for 8K, 32K or 128K
    tokens (the cache itself is the caller's); only the switch to the
    long-context attention merge at max_seq >= 8192 adds a fixed amount,
    exactly its merge rows, (m, l) and tickets."""
    ws = {L: pkg.orthrus_workspace_size(pkg.make_config(synth.QWEN3_8B, "bf16", 1, 32, L, split_tokens=128))
          for L in (2048, 4096, 8192, 32768, 131072)}
    assert ws[8192] == ws[32768] == ws[131072]
    assert ws[2048] == ws[4096]
    up = lambda x: (x + 255) // 256 * 256
    rows, nq, nkv, hd = 128, 32, 8, 128          # the forward buffers' rows: max(batch x K, 128)
    merge = up(4 * rows * nq * hd * 4) + up(4 * rows * nq * 8) + up(rows * nkv * 8 * 4)
    assert ws[8192] - ws[4096] == merge
    # the SIMT attention (fp32) keeps split partials, which do scale with max_seq
    f = {L: pkg.orthrus_workspace_size(pkg.make_config(synth.TINY, "fp32", 1, 4, L, split_tokens=64))
         for L in (1024, 2048)}
    assert f[2048] > f[1024]


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("n_kv_heads", 3), ("split_tokens", 100),
                                          ("max_block", 0), ("mask_token_id", 256), ("dtype", 7),
                                          ("max_seq", 4), ("max_batch", 1000)])
def test_invalid_config_rejected(pkg, field, value):
    cfg = pkg.make_config(synth.TINY, "fp32", 1, 4, 128, split_tokens=64)
    setattr(cfg, field, value)
    n = C.c_size_t()
    assert pkg.lib().orthrus_workspace_size(C.byref(cfg), C.byref(n)) == 1


def test_null_arguments_rejected(pkg):
    lib = pkg.lib()
    assert lib.orthrus_workspace_size(None, None) == 1
    assert lib.orthrus_create(None, None, None, 0, None) == 1
    assert lib.orthrus_destroy(None) == 1
    assert lib.orthrus_prefill(None, None, None, 0, None, 0, None, None) == 1
    assert lib.orthrus_draft_block(None, None, None, 1, 4, 0.0, 0, None, None, None) == 1
    assert lib.orthrus_verify_block(None, None, None, None, 1, 4, 0.0, None) == 1
    assert lib.orthrus_commit(None, None, 1, 4, 0.0, 0, None, None, None, None, None, None) == 1
    assert lib.orthrus_check_error(None, None, None) == 1


def test_no_cpu_path(pkg, monkeypatch):
    """The product path fails loudly instead of falling back: an engine on a
    CPU device is refused before anything is allocated, and a missing
    library raises instead of loading anything else."""
    w = synth.make_weights(synth.TINY, 0)
    with pytest.raises(ValueError, match="CUDA device only"):
        pkg.Engine(synth.TINY, w, device="cpu")
    monkeypatch.setattr(pkg, "_lib", None)
    monkeypatch.setattr(pkg, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "liborthrus.so"))
    with pytest.raises(ImportError, match="missing"):
        pkg.lib()
