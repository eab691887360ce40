"""Helpers shared by the GPU tests: building engines and filling the paged
cache from host arrays (input marshalling only)."""
import dataclasses

import numpy as np
import torch

import synth


def attention_engine(n_q=32, n_kv=8, hd=128, max_batch=3, max_block=32, max_seq=8192, split_tokens=256,
                     page_size=64, dtype="bf16"):
    """An engine whose only purpose is the standalone attention entry point:
    one layer of the given attention shape, dummy projections."""
    import dual_view_diffusion_b200 as pkg
    s = dataclasses.replace(synth.QWEN3_8B, n_layers=1, hidden=64, n_q_heads=n_q, n_kv_heads=n_kv, head_dim=hd,
                            ffn=64, vocab=256, dtype=dtype)
    w = synth.make_weights(s, 0, n_layers=1)
    return pkg.Engine(s, w, max_batch=max_batch, max_block=max_block, max_seq=max_seq,
                      split_tokens=split_tokens, page_size=page_size)


def write_cache(eng, layer, b, kc, vc, start=0):
    """Write host rows kc/vc [n, n_kv, hd] at positions start .. start+n-1 of
    sequence b (pages b*pps ...)."""
    n = kc.shape[0]
    if n == 0:
        return
    ps = eng.page_size
    kt = torch.from_numpy(np.ascontiguousarray(kc, dtype=np.float32)).to(eng.device, eng.tdtype)
    vt = torch.from_numpy(np.ascontiguousarray(vc, dtype=np.float32)).to(eng.device, eng.tdtype)
    pos = torch.arange(start, start + n, device=eng.device)
    page = eng.block_table[b].long()[pos // ps]
    slot = pos % ps
    eng.k_pages[layer, page, :, slot, :] = kt
    eng.v_pages[layer, page, :, :, slot] = vt          # V pages are [dim][slot]


def read_cache(eng, layer, b, start, n):
    ps = eng.page_size
    pos = torch.arange(start, start + n, device=eng.device)
    page = eng.block_table[b].long()[pos // ps]
    slot = pos % ps
    return (eng.k_pages[layer, page, :, slot, :].float().cpu().numpy(),
            eng.v_pages[layer, page, :, :, slot].float().cpu().numpy())


def bf16_normal(shape, seed, name):
    return synth.round_bf16(synth.normal(shape, 1.0, seed, name))
