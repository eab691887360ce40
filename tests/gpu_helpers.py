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


def step_cycles(eng, prompts, lens, K, N, T, seed, iterations=1):
    """Drive decode cycles through the public step calls (draft, verify,
    commit) until every sequence has N tokens.  prompts: int array [B, S];
    lens: per-sequence prompt lengths.  Returns, per sequence, the list of
    (n, emitted tokens) of each cycle."""
    p = torch.from_numpy(np.ascontiguousarray(prompts, dtype=np.int32))
    B = p.shape[0]
    eng.step.zero_()
    anchor = eng.prefill(p, lens)
    cycles = [[] for _ in range(B)]
    done = [0] * B
    while min(done) < N:
        draft = eng.draft_block(anchor, K, temperature=T, seed=seed, iterations=iterations)
        eng.verify_block(anchor, draft, K, temperature=T)
        n, toks = eng.commit(anchor, K, temperature=T, seed=seed)
        n, toks = n.cpu().numpy(), toks.cpu().numpy()
        for b in range(B):
            cycles[b].append((int(n[b]), toks[b, :n[b]].tolist()))
            done[b] += int(n[b])
    return cycles


def first_divergent_cycle(cycles, ref, N):
    """The first cycle whose (n, emitted tokens) differ from the oracle's
    run (ref: Model.generate's dict), or -1.  Before that cycle both sides
    emitted the same tokens, so their caches, anchors and step counters were
    identical: a divergence there is decided by that cycle's own decisions,
    whose smallest oracle margin is ref["cycle_margin"][c]."""
    pos = 0
    for c, (n, toks) in enumerate(cycles):
        if pos >= N:
            break
        if c >= ref["cycles"]:
            return c
        m = min(n, N - pos)
        if n != int(ref["n_per_cycle"][c]) or list(toks[:m]) != [int(x) for x in ref["tokens"][pos:pos + m]]:
            return c
        pos += n
    return -1
