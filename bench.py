#!/usr/bin/env python
"""Benchmark of the Orthrus dual-view decode step on B200.

Workload (one GPU): the Qwen3-8B shape (36 layers, hidden 4096, 32/8 heads,
head_dim 128, FFN 12288, vocab 151936), random-init bf16 weights, batch 1,
block K = 32, a 2048-token uniform random prompt prefilled before timing,
greedy decoding.  One step = one decode cycle: draft (diffusion view),
verify (AR view), consensus and commit ("Orthrus: Memory-Efficient Parallel
Token Generation via Dual-View Diffusion", paper notes §4.1).

value     committed tokens/s over the timed steps (device time, CUDA events,
          max over ranks; N ranks run independent replicas)
e2e       the same metric with the step's input (anchor id) copied from
          pinned host memory and its result (n and the tokens) read back
          every step, through the library's public calls
roofline  the gate/up GEMM with its fused SwiGLU (the step's largest kernel by
          device time; ~95% of a step's HBM traffic is weight streaming),
          timed live by CUDA events around its launch in one layer of every
          verify forward of the timed region; algorithmic bytes = weights +
          activations in/out.  layer_gemms: the same for the layer's four
          projection GEMMs together, with each one's time
attn      the dual-view attention entry point on the single-layer workload
          (L = 4096, K = 32, batch 1), timed as attn_long_context does;
          in_step: the attention kernel of one layer inside the decode
          step, timed like the roofline GEMM; bytes = prefix K/V + Q + O
attn_long_context  the attention entry point alone at L = 4K (the single-layer
          attention workload: 32/8 heads, head_dim 128, K = 32, batch 1),
          8K, 32K and 128K (both views), and at batch 4 and 16 for L = 8K
          and 32K (cells of the long-context sweep), timed over runs of
          calls on distinct layers' caches that together exceed L2 (K/V
          from HBM)
iterative_draft  the same decode step with a two-pass iterative-denoising draft
tree_kernels  the tree-verification kernels built so far (top-W of the draft
          rows, the best-first build, the walk and K/V compaction), each
          timed alone
train_kernels  the training-side kernels (block-masked attention of a packed
          2048-position sequence with 256 anchor blocks; the forward-KL
          LM-head epilogue over the full vocabulary), each timed alone beside
          the oracle on a sample
cpu_baseline  the CPU oracle, as it stands, timed on a bounded sample (one
          layer of each view at full width plus 1/16 of the LM head) and
          scaled to a full step

Weights and the prompt are larger than L2 (18 GB of weights per step), so no
flush is needed between steps.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "committed tokens/s (batch 1, Qwen3-8B shape, K=32); dual-view attn HBM GB/s"
UNIT = "tokens/s"
P_PROMPT, K_BLOCK, BATCH = 2048, 32, 1
ITER_STEPS = 20   # decode steps timed with the two-pass iterative draft
VARIANT_STEPS = 20   # decode steps timed for each of the other decode loops (sampled, tree, adaptive)
# tokens committed per cycle that this random-init 8B workload gives (the
# mean accepted length measured on the GPU path, 1.00-1.03 over runs: the
# random-init diffusion view almost never agrees with the AR view).  Used
# only by the reference arm, which cannot run the whole model.
N_BAR_WORKLOAD = 1.0
# block rows of the oracle's bounded sample (both CPU legs: the reference arm
# and cpu_baseline), scaled to the 32 rows of a step
ORACLE_ROWS = 8
SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--temperature", type=float, default=0.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", choices=["reduced", "full", "none"], default="reduced",
                    help="long-context step sweep: L at batch 1, K at L = 2K, batch at L = 8K (reduced), every "
                         "(L, batch, K) cell that fits (full), or none")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the other decode loops (sampled, plain AR, tree, adaptive) and the 1.7B config")
    ap.add_argument("--split-tokens", type=int, default=128,
                    help="KV positions per attention split (a run-wide constant)")
    ap.add_argument("--profile-small", action="store_true",
                    help="small case for ncu captures: 2 layers of the 8B shape, vocab 32000, 2 steps; "
                         "its line is marked profile_case and is not a bench result")
    ap.add_argument("--profile-attn", type=int, default=0, metavar="L",
                    help="small case for ncu captures of the attention kernel: the attention entry point "
                         "alone at prefix length L (both views, 2 calls each); its line is marked "
                         "profile_case and is not a bench result")
    ap.add_argument("--profile-train", action="store_true",
                    help="small case for ncu captures of the training-side kernels: train_kernels alone (one "
                         "timed call each, no CPU oracle) on a one-layer engine with the 8B LM head; its line "
                         "is marked profile_case and is not a bench result")
    a = ap.parse_args()
    if a.profile_small:
        a.steps, a.warmup, a.no_cpu_baseline, a.no_e2e, a.sweep, a.no_variants = 2, 1, True, True, "none", True
    return a


# ----------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    def __init__(self, index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={SMI_FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = [l.split(",") for l in open(self.f.name).read().splitlines() if l.strip()]
        os.unlink(self.f.name)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        sm, mx, reasons = [], None, set()
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def gemm_bytes(s, M):
    """Algorithmic HBM bytes of the four projection launches of one layer
    (QKV, O, gate/up, down) for M token rows, bf16: weights once, activations
    in and out, fp32 residual read+write."""
    d, hq, hk, F = s.hidden, s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim, s.ffn
    qkv = (hq + 2 * hk) * d * 2 + M * d * 2 + M * (hq + 2 * hk) * 2
    o = d * hq * 2 + M * hq * 2 + M * d * 4 * 2
    gu = 2 * F * d * 2 + M * d * 2 + M * F * 2
    dn = d * F * 2 + M * F * 2 + M * d * 4 * 2
    return [qkv, o, gu, dn]


def attn_bytes(s, t, K, B=1):
    """Algorithmic bytes of one verify attention call: keys/values [0, t+K)
    of every KV head read once, Q read, O written (bf16)."""
    return B * ((t + K) * s.n_kv_heads * s.head_dim * 2 * 2 + 2 * K * s.n_q_heads * s.head_dim * 2)


def _code_only(text):
    """C++/CUDA source without comments, blank lines or trailing blanks: a
    profile stays valid across comment-only edits of its kernel."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = []
    for line in text.splitlines():
        # drop a // comment unless it sits inside a string literal
        out, in_str = [], False
        i = 0
        while i < len(line):
            c = line[i]
            if c == '"' and (i == 0 or line[i - 1] != "\\"):
                in_str = not in_str
            if not in_str and line.startswith("//", i):
                break
            out.append(c)
            i += 1
        s = "".join(out).rstrip()
        if s:
            lines.append(s)
    return "\n".join(lines)


def source_sha(sources):
    """sha256 of the kernel sources' code (comments and blank lines removed)."""
    h = hashlib.sha256()
    for s in sources:
        h.update(_code_only(open(os.path.join(ROOT, s), encoding="utf-8").read()).encode())
    return h.hexdigest()


GEMM_SOURCES = ("dual_view_diffusion_b200/csrc/gemm_tc.cu", "dual_view_diffusion_b200/csrc/gemm_epilogue.cuh",
                "dual_view_diffusion_b200/csrc/gemm.cu")
ATTN_SOURCES = ("dual_view_diffusion_b200/csrc/attention_tc.cu",)


def kernel_traffic(name, sources, key="dram_bytes_per_layer"):
    """DRAM bytes recorded by an ncu capture (profiles/<name>), valid only
    while the kernel sources are unchanged (their sha256 is recorded with
    it)."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    rec = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            rec[k.strip()] = v.strip()
    if rec.get("kernel_source_sha256") != source_sha(sources):
        return None
    try:
        return float(rec[key])
    except (KeyError, ValueError):
        return None


LONG_CONTEXT_BATCHED = ((8192, 4), (8192, 16), (32768, 4), (32768, 16))


def attn_long_context(hbm, split_tokens, lengths=(4096, 8192, 32768, 131072), batched=LONG_CONTEXT_BATCHED,
                      reps=5):
    """The dual-view attention entry point alone (the attention layer shape
    of the 8B model: 32/8 heads, head_dim 128, block K = 32), at batch 1 for
    each of `lengths` and at the (L, batch) cells of `batched` (every
    sequence of a batch at prefix L), both views, on N(0,1) bf16 inputs,
    timed the way a forward meets it: a run of
    calls over n distinct layers' caches, back to back, whose caches
    together exceed 2.5x L2, so every call reads its K/V from HBM (inputs
    larger than L2: no flush) while code and block tables stay where a
    forward would leave them.  Per-call time = run time / n (CUDA events
    around the run, after a device-side wait that lets the host enqueue the
    whole run first); median of reps runs.  Bytes = prefix K/V + block K/V
    + Q + O."""
    import math
    import torch
    import synth
    import dual_view_diffusion_b200 as pkg
    K = K_BLOCK
    n_q, n_kv, hd = synth.QWEN3_8B.n_q_heads, synth.QWEN3_8B.n_kv_heads, synth.QWEN3_8B.head_dim
    out = []
    for L, B in [(L, 1) for L in lengths] + list(batched):
        byts = B * ((L + K) * n_kv * hd * 2 * 2 + 2 * K * n_q * hd * 2)
        nl = max(2, math.ceil(2.5 * 126e6 / byts))
        s = dataclasses.replace(synth.QWEN3_8B, n_layers=nl, hidden=64, ffn=64, vocab=256)
        w = synth.make_weights(s, 0, n_layers=nl)
        eng = pkg.Engine(s, w, max_batch=B, max_block=K, max_seq=L + K + 64, split_tokens=split_tokens)
        g = torch.Generator(device="cuda").manual_seed(2)
        for pg in (eng.k_pages, eng.v_pages):
            for i in range(pg.shape[0]):   # one layer at a time: bounded fp32 scratch
                pg[i].copy_(torch.randn(pg[i].shape, generator=g, device="cuda").to(pg.dtype))
        q = torch.randn((B, K, n_q, hd), generator=g, device="cuda").to(torch.bfloat16)
        kb = torch.randn((B, K, n_kv, hd), generator=g, device="cuda").to(torch.bfloat16)
        vb = torch.randn((B, K, n_kv, hd), generator=g, device="cuda").to(torch.bfloat16)
        eng.seq_lens[:B] = L
        for mode in (0, 1):
            for layer in range(nl):
                eng.attention(layer, mode, q, kb, vb, B, K)
            ms = []
            for _ in range(reps):
                torch.cuda.synchronize()
                torch.cuda._sleep(int(2e6 + 1e5 * nl))   # device-side wait: the host enqueues the run meanwhile
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for layer in range(nl):
                    eng.attention(layer, mode, q, kb, vb, B, K)
                e1.record()
                torch.cuda.synchronize()
                ms.append(e0.elapsed_time(e1) / nl)
            us = statistics.median(ms) * 1e3
            out.append({"L": L, "batch": B, "view": "draft (mode 1)" if mode else "verify (mode 0)", "us": us,
                        "layers": nl,
                        "achieved": byts / us / 1e3, "frac": byts / us / 1e3 / hbm})
        assert eng.check_error()[0] == 0
        del eng
        torch.cuda.empty_cache()
    return {"unit": "GB/s", "peak": hbm,
            "how": "runs of back-to-back calls over n distinct layers' caches (together > 2.5x L2, so K/V "
                   "come from HBM), per-call time = run time / n, host enqueue hidden behind a device-side "
                   "wait, median of " + str(reps) + " runs",
            "points": out}


def _timed(fn, reps):
    """Median device time (us) of fn() over reps calls, each after a
    device-side wait that hides host enqueue (the callers' inputs exceed L2,
    so no flush is needed)."""
    import torch
    for _ in range(2):
        fn()
    ms = []
    for _ in range(reps):
        torch.cuda.synchronize()
        torch.cuda._sleep(200000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    return statistics.median(ms) * 1e3


def train_kernels(hbm, tflops, eng, reps=10, cpu=True):
    """The training-side kernels of the pages (§3.1-3.3), each timed alone
    (median of reps; each reads more than L2 holds: 176 MB of queries,
    outputs and K/V, and the 1.24 GB head) beside the CPU oracle on a sample.
    block_mask_attention: one packed training sequence, 256 anchor blocks of
    K = 32 over 2048 positions (anchors uniform in [0, 2016], seed 4), the 8B
    attention shape, N(0,1) bf16; bound tensor: useful FLOPs = 4 hd x the
    keys each (row, query head) sees.  kl_lm_head: 16 row pairs (N(0, 3^2)
    bf16 hidden rows, diffusion = AR + N(0, 1.8^2)) through the 8B LM head
    (151936 x 4096, the decode engine's, or a one-layer engine's when eng is
    None); bound HBM: the head's bytes + rows.  cpu=False skips the oracle
    samples."""
    import numpy as np
    import torch
    import oracle
    import synth
    import dual_view_diffusion_b200 as pkg
    out = {}
    # ---- block-masked attention
    nb, K, L = 256, K_BLOCK, 2048
    s = dataclasses.replace(synth.QWEN3_8B, n_layers=1, hidden=64, ffn=64, vocab=256)
    w = synth.make_weights(s, 0, n_layers=1)
    ae = pkg.Engine(s, w, max_batch=128, max_block=K, max_seq=L + 64, split_tokens=128)
    g = torch.Generator(device="cuda").manual_seed(4)
    n_q, n_kv, hd = s.n_q_heads, s.n_kv_heads, s.head_dim
    for pg in (ae.k_pages, ae.v_pages):
        pg.copy_(torch.randn(pg.shape, generator=g, device="cuda").to(pg.dtype))
    q = torch.randn((nb, K, n_q, hd), generator=g, device="cuda").to(torch.bfloat16)
    kb = torch.randn((nb, K, n_kv, hd), generator=g, device="cuda").to(torch.bfloat16)
    vb = torch.randn((nb, K, n_kv, hd), generator=g, device="cuda").to(torch.bfloat16)
    anchors = np.random.default_rng(4).integers(0, L - K + 1, nb).astype(np.int32)
    ad = torch.from_numpy(anchors).cuda()
    us = _timed(lambda: ae.block_mask_attention(0, q, kb, vb, ad, K), reps)
    flops = float(4 * hd * K * n_q * (anchors.astype(np.int64) + K).sum())
    byts = 2 * nb * K * n_q * hd * 2 + 2 * nb * K * n_kv * hd * 2 + 2 * L * n_kv * hd * 2
    ach = flops / us / 1e6
    out["block_mask_attention"] = {
        "workload": "256 anchor blocks x K=32 in one packed 2048-position sequence, 32/8 heads, head_dim 128",
        "us": us, "bound": "tensor", "achieved": ach, "peak": tflops, "unit": "TFLOP/s", "frac": ach / tflops,
        "hbm_gbs": byts / us / 1e3, "algorithmic_flops": flops, "algorithmic_bytes": byts,
        "ncu_dram_bytes_first_launch": kernel_traffic("block_mask_attention_training.txt", ATTN_SOURCES,
                                                      "dram_bytes_per_launch")}
    if cpu:
        _block_mask_cpu(out["block_mask_attention"], ae, q, kb, vb, anchors, nb, K, L)
    del ae
    torch.cuda.empty_cache()
    # ---- forward-KL LM head on the decode engine's 8B head
    own = eng is None
    if own:
        s8 = dataclasses.replace(synth.QWEN3_8B, n_layers=1)
        eng = pkg.Engine(s8, synth.make_weights_torch(s8, 0, n_layers=1), max_batch=1, max_block=K_BLOCK,
                         max_seq=256, split_tokens=128)
    rows, d, V = 16, eng.shape.hidden, eng.shape.vocab
    gk = torch.Generator(device="cuda").manual_seed(5)
    hA = (3.0 * torch.randn((rows, d), generator=gk, device="cuda")).to(torch.bfloat16)
    hD = (hA.float() + 1.8 * torch.randn((rows, d), generator=gk, device="cuda")).to(torch.bfloat16)
    us = _timed(lambda: eng.kl_lm_head(hA, hD), reps)
    byts = V * d * 2 + 2 * rows * d * 2 + rows * 12
    ach = byts / us / 1e3
    out["kl_lm_head"] = {
        "workload": "16 row pairs through the 151936 x 4096 LM head", "us": us, "bound": "hbm",
        "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "algorithmic_bytes": byts,
        "traffic": kernel_traffic("kl_lm_head_qwen3_8b_head.txt", GEMM_SOURCES, "dram_bytes_per_launch")}
    if cpu:
        Vs = 8192
        Wh = eng.lm_head[:Vs].float().cpu().numpy()
        t0 = time.perf_counter()
        oracle.kl_rows(hA[:1].float().cpu().numpy(), hD[:1].float().cpu().numpy(), Wh)
        t_cpu = (time.perf_counter() - t0) * rows * V / Vs
        out["kl_lm_head"]["cpu_baseline"] = {"seconds": t_cpu, "cores": OracleSample.threads(), "kind": "oracle",
                                             "sample": f"1 row pair over the first {Vs} vocabulary ids, scaled"}
    if own:
        del eng
        torch.cuda.empty_cache()
    return out


def tree_kernels(hbm, reps=20):
    """The tree-verification kernels that exist so far (paper notes §7.5 /
    §9.6), each timed alone (median of reps, device time) at the decode
    workload's sizes: top-W (W = 4) and log-sum-exp of the K - 1 = 31 draft
    rows' fp32 logits over the 151936-id vocabulary (HBM: 31 x 151936 x 4 B
    read; no flush between reps, so the 18.8 MB may be L2 hits); the
    best-first build of 31 nodes over depth 31; the walk and the K/V
    compaction of a 32-row tree whose accepted path has 8 nodes, in the
    36-layer, 8-KV-head, head_dim-128 bf16 cache.  Latency-bound except
    top-W."""
    import numpy as np
    import torch
    import synth
    import dual_view_diffusion_b200 as pkg
    K, W, V = K_BLOCK, 4, synth.QWEN3_8B.vocab
    s = dataclasses.replace(synth.QWEN3_8B, hidden=64, ffn=64)
    eng = pkg.Engine(s, synth.make_weights_torch(s, 0), max_batch=1, max_block=K, max_seq=P_PROMPT + 2 * K,
                     split_tokens=128)
    g = torch.Generator(device="cuda").manual_seed(7)
    z = 3.0 * torch.randn((K - 1, V), generator=g, device="cuda")
    ids, vals, lse = eng.tree_topw(z, W)
    us_topw = _timed(lambda: eng.tree_topw(z, W), reps)
    D = K - 1
    us_build = _timed(lambda: eng.tree_build(ids.view(1, D, W), vals.view(1, D, W), lse.view(1, D), K - 1), reps)
    # a 32-row tree: 23 leaves under the root (rows 1..23), then a chain of 8 nodes (rows 24..31) that
    # the AR argmaxes accept, so its K/V move from slots t+24..t+31 to t+1..t+8
    par = np.array([-1] + [0] * 23 + [0] + list(range(24, 31)), np.int32)
    tok = np.array([-1] + [1000 + i for i in range(23)] + [100 + i for i in range(8)], np.int32)
    gg = np.full(K, 7, np.int32)
    gg[0] = 100
    gg[24:31] = np.arange(101, 108)
    dev = lambda a: torch.from_numpy(a[None]).cuda()
    pd, td, gd, nr = dev(par), dev(tok), dev(gg), torch.tensor([K], dtype=torch.int32, device="cuda")
    anchor = torch.zeros(1, dtype=torch.int32, device="cuda")

    def commit():
        eng.seq_lens[0] = P_PROMPT
        eng.tree_commit(pd, td, nr, gd, anchor)
    commit()
    n_acc = int(eng.seq_lens[0].item()) - P_PROMPT
    us_commit = _timed(commit, reps)   # includes the one-element length reset (a copy kernel)
    assert eng.check_error()[0] == 0
    byts = (K - 1) * V * 4
    out = {"topw": {"rows": K - 1, "width": W, "us": us_topw, "bound": "hbm", "achieved": byts / us_topw / 1e3,
                    "peak": hbm, "unit": "GB/s", "frac": byts / us_topw / 1e3 / hbm, "algorithmic_bytes": byts},
           "build": {"nodes": K - 1, "depth": D, "width": W, "us": us_build, "bound": "latency"},
           "commit": {"rows": K, "accepted": n_acc, "layers": s.n_layers, "us": us_commit, "bound": "latency",
                      "moved_bytes": 2 * (n_acc - 1) * s.n_layers * s.n_kv_heads * s.head_dim * 2}}
    _tree_cpu(out, z[:2].cpu().numpy(), W, K, s.n_layers, s.n_kv_heads, s.head_dim, par, tok, gg)
    del eng
    torch.cuda.empty_cache()
    return out


def _tree_cpu(out, z2, W, K, n_layers, n_kv, hd, par, tok, gg):
    """The oracle beside each tree kernel: top-W + log-sum-exp of 2 of the
    31 logits rows (scaled to 31), the best-first build of the same tree
    (D = K - 1 rows of log q over the vocabulary), and the walk plus the
    K/V moves of the same path in an fp64 cache of the same layers and
    heads (capacity K, t = 0)."""
    import numpy as np
    import oracle
    rows = K - 1
    t0 = time.perf_counter()
    ids, lse = oracle.topw(z2.astype(np.float64), W)
    t_topw = (time.perf_counter() - t0) * rows / z2.shape[0]
    logp = np.repeat(z2[:1].astype(np.float64) - lse[0], rows, axis=0)
    t0 = time.perf_counter()
    oracle.tree_build(logp, W, rows)
    t_build = time.perf_counter() - t0
    kc = np.zeros((n_layers, K, n_kv, hd))
    vc = np.zeros_like(kc)
    t0 = time.perf_counter()
    _, _, path = oracle.tree_accept(par, tok, gg)
    oracle.tree_commit_kv(kc, vc, 0, path)
    t_commit = time.perf_counter() - t0
    cores = OracleSample.threads()
    out["topw"]["cpu_baseline"] = {"seconds": t_topw, "cores": cores, "kind": "oracle",
                                   "sample": f"2 of the {rows} rows, scaled"}
    out["build"]["cpu_baseline"] = {"seconds": t_build, "cores": cores, "kind": "oracle",
                                    "sample": "the whole build (one logits row repeated for every depth)"}
    out["commit"]["cpu_baseline"] = {"seconds": t_commit, "cores": cores, "kind": "oracle",
                                     "sample": "the whole walk and the moves of the same path"}


def _block_mask_cpu(rec, ae, q, kb, vb, anchors, nb, K, L):
    """The oracle on 2 of the blocks, scaled by visible keys to all of them."""
    import numpy as np
    import oracle
    n_kv, hd = ae.shape.n_kv_heads, ae.shape.head_dim
    qh, kbh, vbh = (x.float().cpu().numpy() for x in (q[:2], kb[:2], vb[:2]))
    kc = ae.k_pages[0, :L // ae.page_size].float().permute(0, 2, 1, 3).reshape(L, n_kv, hd).cpu().numpy()
    vc = ae.v_pages[0, :L // ae.page_size].float().permute(0, 3, 1, 2).reshape(L, n_kv, hd).cpu().numpy()
    t0 = time.perf_counter()
    for b in range(2):
        oracle.block_mask_attention(qh[b], kc, vc, kbh[b], vbh[b], anchors[b:b + 1], K)
    t_cpu = (time.perf_counter() - t0) / float(anchors[:2].astype(np.int64).sum() + 2 * K) * \
        float(anchors.astype(np.int64).sum() + nb * K)
    rec["cpu_baseline"] = {"seconds": t_cpu, "cores": OracleSample.threads(), "kind": "oracle",
                           "sample": "2 of the 256 blocks, scaled by visible keys"}


def _time_steps(fn, n):
    """Device time (ms) of n calls of fn(i), CUDA events around the run on the
    current stream."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(n):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def decode_variants(eng, anchor, draft, toks, value, ms_step, steps=VARIANT_STEPS):
    """Other decode loops on the benchmark's engine (the 8B shape, batch 1,
    K = 32), each warmed up three steps and then timed over `steps` steps
    with CUDA events:
      sampled   the Orthrus step at T = 1.0 with rejection sampling (paper
                notes §4.3): draft samples, acceptance test, residual draw
      plain_ar  one AR forward per token (the same kernels, K = 1): the
                baseline whose greedy stream Orthrus reproduces (§4.2)
      tree      a tree-verified step (§7.5 / §9.6): draft with the top-4
                candidates of its rows from the LM-head pass, a best-first
                tree of 31 nodes, the tree-masked verify forward (32 rows, as
                the chain's) and the walk plus K/V compaction
      adaptive  the adaptive block length (§7.4 / §9.6, reading R23): the
                verify length from the draft rows' entropies, threshold the
                median entropy of a warm-up draft"""
    import numpy as np
    import torch
    B, K, dev = BATCH, K_BLOCK, anchor.device
    out = {}
    # ---- sampled T = 1.0
    n_s = torch.zeros((steps + 3, B), dtype=torch.int32, device=dev)

    def st_sampled(j):
        eng.draft_block(anchor, K, 1.0, 4321, out=draft)
        eng.verify_block(anchor, draft, K, 1.0)
        eng.commit(anchor, K, 1.0, 4321, n_out=n_s[j], tokens_out=toks)
    for j in range(3):
        st_sampled(steps + j)
    ms = _time_steps(st_sampled, steps)
    tok = int(n_s[:steps].sum())
    out["sampled"] = {"temperature": 1.0, "steps": steps, "ms_per_step": ms / steps,
                      "value": tok / (ms * 1e-3), "unit": UNIT, "mean_accepted_per_cycle": tok / (steps * B),
                      "how": "draft samples (Gumbel-max), acceptance u < p/q, residual draw from max(0, p - q) at "
                             "the first rejection (one extra LM-head pass over two rows); CUDA events"}
    # ---- plain AR
    ar_tok = torch.empty(B, dtype=torch.int32, device=dev)
    for _ in range(3):
        eng.ar_step(anchor, token_out=ar_tok)
    n_ar = 4 * steps
    ms = _time_steps(lambda i: eng.ar_step(anchor, token_out=ar_tok), n_ar)
    ar_val = n_ar * B / (ms * 1e-3)
    out["plain_ar"] = {"steps": n_ar, "ms_per_token": ms / n_ar, "value": ar_val, "unit": UNIT,
                       "orthrus_over_ar": value / ar_val,
                       "modelled_orthrus_over_ar_at_pages_acceptance": 10.8 / (ms_step * 1e-3) / ar_val,
                       "how": "orthrus_ar_step (AR view on one row, argmax, commit 1) back to back; the ratio is "
                              "the greedy decode step's tokens/s (measured acceptance) over this; the modelled "
                              "ratio uses the pages' 10.8 tokens per cycle"}
    # ---- tree-verified step (greedy)
    W, nodes, D = 4, K - 1, K - 1
    n_t = torch.zeros((steps + 3, B), dtype=torch.int32, device=dev)

    def st_tree(j):
        _, ids, vals, lse = eng.draft_block_topw(anchor, K, W, D, out=draft)
        par, tk, _, _, nr = eng.tree_build(ids, vals, lse, nodes)
        g = eng.verify_tree(anchor, par, tk)
        n, _ = eng.tree_commit(par, tk, nr, g, anchor)
        n_t[j].copy_(n)
    for j in range(3):
        st_tree(steps + j)
    ms = _time_steps(st_tree, steps)
    tok = int(n_t[:steps].sum())
    out["tree"] = {"width": W, "nodes": nodes, "steps": steps, "ms_per_step": ms / steps,
                   "value": tok / (ms * 1e-3), "unit": UNIT, "mean_accepted_per_cycle": tok / (steps * B),
                   "how": "draft with the top-W of its rows taken inside the LM-head pass, best-first build, "
                          "tree-masked verify forward, walk + K/V compaction; greedy"}
    # ---- adaptive block length (greedy)
    kt = torch.empty(B, dtype=torch.int32, device=dev)
    eng.draft_block(anchor, K, out=draft)
    _, ent = eng.adaptive_len(B, K, float("inf"), kt=kt, entropy=True)
    h_max = float(ent.float().median())
    n_a = torch.zeros((steps + 3, B), dtype=torch.int32, device=dev)
    k_a = torch.zeros((steps + 3, B), dtype=torch.int32, device=dev)

    def st_adaptive(j):
        eng.draft_block(anchor, K, out=draft)
        eng.adaptive_len(B, K, h_max, kt=kt)
        eng.verify_block(anchor, draft, K)
        eng.commit_adaptive(anchor, K, kt, n_out=n_a[j], tokens_out=toks)
        k_a[j].copy_(kt)
    for j in range(3):
        st_adaptive(steps + j)
    ms = _time_steps(st_adaptive, steps)
    tok = int(n_a[:steps].sum())
    out["adaptive"] = {"h_max": h_max, "steps": steps, "ms_per_step": ms / steps, "value": tok / (ms * 1e-3),
                       "unit": UNIT, "mean_accepted_per_cycle": tok / (steps * B),
                       "mean_verify_rows": float(k_a[:steps].float().mean()),
                       "how": "draft, per-sequence verify length from the draft rows' entropies (threshold: the "
                              "median entropy of a warm-up draft), verify of the block, greedy consensus over the "
                              "first kt rows; the verify forward still runs 32 rows (its cost is weight streaming)"}
    return out


def config_1p7b(split_tokens, steps=VARIANT_STEPS):
    """The Qwen3-1.7B-shaped random-init model (28 layers, hidden 2048, 16/8
    heads, FFN 6144, tied head), prompt 512, K = 32, batch 1, greedy: the
    decode step and plain AR, each timed over `steps` (AR: 4x) steps after
    three warm-up steps."""
    import torch
    import synth
    import dual_view_diffusion_b200 as pkg
    s = synth.QWEN3_1_7B
    P, K, B = 512, K_BLOCK, 1
    w = synth.make_weights_torch(s, 0)
    eng = pkg.Engine(s, w, max_batch=B, max_block=K, max_seq=P + (2 * steps + 12) * K + 4 * steps + 64,
                     split_tokens=split_tokens)
    prompt = torch.from_numpy(synth.make_prompt(s, P, 0))[None].cuda()
    anchor = eng.prefill(prompt)
    eng.step.zero_()
    draft = torch.empty((B, K), dtype=torch.int32, device="cuda")
    toks = torch.empty((B, K), dtype=torch.int32, device="cuda")
    n_h = torch.zeros((steps + 3, B), dtype=torch.int32, device="cuda")

    def st(j):
        eng.draft_block(anchor, K, out=draft)
        eng.verify_block(anchor, draft, K)
        eng.commit(anchor, K, n_out=n_h[j], tokens_out=toks)
    for j in range(3):
        st(steps + j)
    ms = _time_steps(st, steps)
    tok = int(n_h[:steps].sum())
    ar_tok = torch.empty(B, dtype=torch.int32, device="cuda")
    for _ in range(3):
        eng.ar_step(anchor, token_out=ar_tok)
    ms_ar = _time_steps(lambda i: eng.ar_step(anchor, token_out=ar_tok), 4 * steps)
    assert eng.check_error()[0] == 0
    val, ar_val = tok / (ms * 1e-3), 4 * steps / (ms_ar * 1e-3)
    del eng, w
    torch.cuda.empty_cache()
    return {"workload": "qwen3-1.7b-shape decode step, batch 1, K=32, prompt 512, greedy", "steps": steps,
            "ms_per_step": ms / steps, "value": val, "unit": UNIT, "mean_accepted_per_cycle": tok / steps,
            "plain_ar": {"ms_per_token": ms_ar / (4 * steps), "value": ar_val}, "orthrus_over_ar": val / ar_val}


SWEEP_L = (2048, 8192, 32768, 131072)
SWEEP_B = (1, 4, 16)
SWEEP_K = (4, 8, 16, 32)


def sweep_cells(full):
    """The long-context sweep's (L, batch, K) cells: all of them when full,
    else L at batch 1 and K = 32, K at L = 2K and batch 1, batch at L = 8K
    and K = 32."""
    if full:
        return [(L, B, K) for L in SWEEP_L for B in SWEEP_B for K in SWEEP_K]
    cells = [(L, 1, 32) for L in SWEEP_L] + [(2048, 1, K) for K in SWEEP_K[:-1]] + [(8192, B, 32) for B in SWEEP_B[1:]]
    return cells


def step_sweep(w, s, split_tokens, cells, steps=4, warm=2, hbm=None):
    """One 8B-shape decode step (draft + verify + commit) per (L, batch, K)
    cell: every sequence's cache filled with N(0, 1) bf16 K/V (seed 3) up to
    prefix L (no prefill), anchors uniform ids, the accepted length of each
    sequence and step drawn uniformly from 1..K (seed 3, orthrus_commit's
    force_n); `warm` steps, then `steps` timed with CUDA events.  Bytes per
    step: both views' weights (the decode engine's) + every sequence's K/V
    prefix read twice (draft and verify).  A cell whose cache would not fit
    next to the weights with 16 GB to spare is skipped and listed."""
    import numpy as np
    import torch
    import dual_view_diffusion_b200 as pkg
    free, _ = torch.cuda.mem_get_info()
    kv_tok = s.n_layers * s.n_kv_heads * s.head_dim * 2 * 2
    wbytes = sum(x * 2 for x in gemm_bytes_weights(s)) * s.n_layers + 2 * s.vocab * s.hidden * 2
    out, skipped = [], []
    for L, B, K in cells:
        max_seq = L + (warm + steps + 1) * K + 64
        need = B * ((max_seq + 63) // 64 * 64) * kv_tok
        if need > free - 16e9:
            skipped.append({"L": L, "batch": B, "K": K, "kv_bytes": need,
                            "why": f"the paged cache ({need / 2**30:.0f} GiB) does not fit beside the weights"})
            continue
        eng = pkg.Engine(s, w, max_batch=B, max_block=K, max_seq=max_seq, split_tokens=split_tokens, page_size=64)
        g = torch.Generator(device="cuda").manual_seed(3)
        for pg in (eng.k_pages, eng.v_pages):
            for i in range(pg.shape[0]):
                pg[i].normal_(generator=g)
        rng = np.random.Generator(np.random.Philox(key=3))
        anchor = torch.from_numpy(rng.integers(0, s.vocab - 1, B).astype(np.int32)).cuda()
        fn = torch.from_numpy(rng.integers(1, K + 1, (warm + steps, B)).astype(np.int32)).cuda()
        eng.seq_lens[:B] = L
        eng.step.zero_()
        draft = torch.empty((B, K), dtype=torch.int32, device="cuda")
        toks = torch.empty((B, K), dtype=torch.int32, device="cuda")
        nbuf = torch.empty(B, dtype=torch.int32, device="cuda")

        def st(j):
            eng.draft_block(anchor, K, out=draft)
            eng.verify_block(anchor, draft, K)
            eng.commit(anchor, K, force_n=fn[j], n_out=nbuf, tokens_out=toks)
        for j in range(warm):
            st(j)
        ms = _time_steps(lambda i: st(warm + i), steps)
        assert eng.check_error()[0] == 0
        tok = int(fn[warm:].sum())
        mean_t = L + float(fn[:warm].sum()) / B + float(fn[warm:].sum()) / (2 * B)
        byts = wbytes + 2 * B * (mean_t + K) * kv_tok
        rec = {"L": L, "batch": B, "K": K, "ms_per_step": ms / steps, "tokens_per_s": tok / (ms * 1e-3),
               "workspace_bytes": eng.ws_bytes, "achieved_gbs": byts / (ms / steps * 1e-3) / 1e9}
        if hbm:
            rec["frac"] = rec["achieved_gbs"] / hbm
        out.append(rec)
        del eng
        torch.cuda.empty_cache()
    return {"how": "one decode step per cell, cache filled synthetically (N(0,1) bf16, seed 3), accepted length "
                   "forced uniform over 1..K (seed 3), CUDA events over the timed steps; bytes = weights of both "
                   "views + K/V prefix read by both views", "cells": out, "skipped": skipped}


def gemm_bytes_weights(s):
    """Parameters one decode step reads per layer for each projection (QKV,
    O, gate/up, down), both views together: each view reads its own QKV and
    the shared O and FFN once."""
    d, hq, hk, F = s.hidden, s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim, s.ffn
    return [2 * (hq + 2 * hk) * d, 2 * d * hq, 2 * 2 * F * d, 2 * d * F]


# ----------------------------------------------------------------- oracle sample
class OracleSample:
    """The CPU oracle, as it stands, on a bounded sample of one decode step
    of the 8B shape: one layer of each view at full width over n_rows block
    rows against a 2047-row prefix, plus the LM head over 1/head_slice of the
    vocabulary.  The full step is estimated by scaling: x36 layers, x32/n_rows
    rows, x head_slice for the head.  Weights are drawn once, in fp32 (the
    oracle computes in fp64 whatever the stored precision)."""

    def __init__(self, head_slice=16):
        import oracle
        import synth
        s8 = synth.QWEN3_8B
        self.s8, self.head_slice = s8, head_slice
        self.s = dataclasses.replace(s8, vocab=s8.vocab // head_slice, dtype="fp32")
        self.m = oracle.Model(synth.make_weights(self.s, 0, n_layers=1))
        self.t = P_PROMPT - 1
        self.synth = synth

    def step_seconds(self, n_rows=32):
        s, t = self.s, self.t
        cap = t + n_rows
        kc = self.synth.normal((1, cap, s.n_kv_heads, s.head_dim), 1.0, 3, "bench.kc")
        vc = self.synth.normal((1, cap, s.n_kv_heads, s.head_dim), 1.0, 3, "bench.vc")
        prompt = self.synth.make_prompt(s, n_rows, 0)
        draft_blk = [int(prompt[0])] + [s.mask_id] * (n_rows - 1)
        t0 = time.perf_counter()
        self.m.forward(1, 1, draft_blk, t, kc.copy(), vc.copy(), logits=False)
        t1 = time.perf_counter()
        self.m.forward(0, 0, prompt, t, kc.copy(), vc.copy(), logits=False)
        t2 = time.perf_counter()
        self.m.forward(0, 0, prompt, t, kc.copy(), vc.copy(), logits=True)
        t3 = time.perf_counter()
        layer = (t1 - t0) + (t2 - t1)
        head = max(t3 - t2 - (t2 - t1), 0.0)
        scale_rows = 32 / n_rows
        return scale_rows * (self.s8.n_layers * layer + 2 * self.head_slice * head)

    def describe(self, n_rows):
        return (f"one layer of each view of the Qwen3-8B shape at full width, {n_rows} block rows over a "
                f"{self.t}-row prefix, plus the LM head over 1/{self.head_slice} of the vocabulary; scaled "
                f"x{self.s8.n_layers} layers, x{32 / n_rows:g} rows, x{self.head_slice} head")

    @staticmethod
    def threads():
        return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def reduce_replicas(tokens, ms, e2e_value, world, device):
    """Replicas only: every rank decodes its own sequence with its own copy
    of the weights; no data moves between GPUs.  The job's throughput is
    the tokens of all ranks over the slowest rank's device time, and the
    end-to-end throughputs add.  Statistics only (one all-reduce each, after
    the timed region)."""
    if world == 1:
        return tokens, ms, e2e_value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(tokens), float(e2e_value)], dtype=torch.float64, device=device)
    m = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t)
    dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return int(round(t[0].item())), float(m.item()), float(t[1].item())


# ----------------------------------------------------------------- arms
def run_reference(args, rank, world):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    samples, walls = [], []
    sample = OracleSample()
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        est = sample.step_seconds(ORACLE_ROWS)
        if i >= args.warmup:
            samples.append(est)
            walls.append(time.perf_counter() - t0)
    sec = statistics.mean(samples)
    desc, threads = sample.describe(ORACLE_ROWS), sample.threads()
    value = N_BAR_WORKLOAD / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
            "ms_per_step_is": "the measured wall time of one step's bounded oracle sample; value is extrapolated "
                              "from it to a whole decode step (extrapolated_ms_per_full_step)",
            "extrapolated_ms_per_full_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "qwen3-8b-shape decode step, batch 1, K=32, prompt 2048, greedy",
                       "global_batch": BATCH, "seq_len": P_PROMPT, "parallelism": "host cores"},
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": threads,
                             "sample": desc + f"; tokens per step = {N_BAR_WORKLOAD} (this workload's "
                                              "mean accepted length)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import dual_view_diffusion_b200 as pkg
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = synth.QWEN3_8B
    if args.profile_small:
        s = dataclasses.replace(s, n_layers=2, vocab=32000)
    W, K, T = args.warmup, args.steps, args.temperature
    n_e2e = 0 if args.no_e2e else K
    n_iter = 0 if args.profile_small else 3 + ITER_STEPS   # the iterative-draft measurement
    # the other decode loops: sampled, tree and adaptive steps (<= K tokens
    # each), plain AR (1 token each)
    n_var = 0 if args.no_variants else 3 * (VARIANT_STEPS + 4) * K_BLOCK + 4 * VARIANT_STEPS + 8
    max_seq = P_PROMPT + (W + K + n_e2e + n_iter + 2) * K_BLOCK + K_BLOCK + n_var
    w = synth.make_weights_torch(s, 0, device=dev)
    eng = pkg.Engine(s, w, max_batch=BATCH, max_block=K_BLOCK, max_seq=max_seq, split_tokens=args.split_tokens,
                     page_size=64, device=dev)
    prompt = torch.from_numpy(synth.make_prompt(s, P_PROMPT, 100 + rank))[None].to(dev)
    anchor = eng.prefill(prompt)
    eng.step.zero_()
    draft = torch.empty((BATCH, K_BLOCK), dtype=torch.int32, device=dev)
    toks = torch.empty((BATCH, K_BLOCK), dtype=torch.int32, device=dev)
    n_hist = torch.zeros((K + 1, BATCH), dtype=torch.int32, device=dev)

    def step(i_hist):
        eng.draft_block(anchor, K_BLOCK, T, 1234, out=draft)
        eng.verify_block(anchor, draft, K_BLOCK, T)
        eng.commit(anchor, K_BLOCK, T, 1234, n_out=n_hist[i_hist], tokens_out=toks)

    for _ in range(W):
        step(K)
    torch.cuda.synchronize()
    t_start = int(eng.seq_lens[0])

    # live probes: one middle layer of every verify forward
    probe_layer = s.n_layers // 2
    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    g0, g1 = mk(4 * K), mk(4 * K)
    a0, a1 = mk(K), mk(K)
    eng.set_probe(0, probe_layer, 0, g0, g1)
    eng.set_probe(1, probe_layer, 0, a0, a1)
    launches0 = eng.launch_count()

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record()
        for i in range(K):
            step(i)
        ev1.record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = ev0.elapsed_time(ev1)
    launches = eng.launch_count() - launches0
    eng.set_probe(0, 0, 0, [], [])
    eng.set_probe(1, 0, 0, [], [])
    n = n_hist[:K].sum(dim=1).cpu().numpy()          # per step, summed over the batch
    tokens = int(n.sum())
    st, bits = eng.check_error()
    if st != 0:
        raise RuntimeError(f"device error bits {bits:#x}")

    # projections: bytes per launch / live event durations
    gb = gemm_bytes(s, BATCH * K_BLOCK)
    g_ms = np.array([g0[i].elapsed_time(g1[i]) for i in range(4 * K)]).reshape(K, 4)
    g_bytes = sum(gb) * K
    g_time = g_ms.sum() * 1e-3
    # attention: t per step from the committed history
    t_steps = t_start + np.concatenate([[0], np.cumsum(n)[:-1]])
    a_ms = np.array([a0[i].elapsed_time(a1[i]) for i in range(K)])
    a_bytes = sum(attn_bytes(s, int(t), K_BLOCK) for t in t_steps)
    a_time = a_ms.sum() * 1e-3

    # ---------------------------------------------------------------- e2e
    e2e = None
    if n_e2e:
        h_anchor = torch.empty(BATCH, dtype=torch.int32).pin_memory()
        h_res = torch.empty((BATCH, 1 + K_BLOCK), dtype=torch.int32).pin_memory()
        d_res = torch.empty((BATCH, 1 + K_BLOCK), dtype=torch.int32, device=dev)
        h_anchor.copy_(anchor.cpu())
        e2e_tokens = 0
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_e2e):
            anchor.copy_(h_anchor, non_blocking=True)
            eng.draft_block(anchor, K_BLOCK, T, 1234, out=draft)
            eng.verify_block(anchor, draft, K_BLOCK, T)
            eng.commit(anchor, K_BLOCK, T, 1234, n_out=d_res[:, 0], tokens_out=toks)
            d_res[:, 1:].copy_(toks)
            h_res.copy_(d_res, non_blocking=True)
            torch.cuda.current_stream().synchronize()
            nb = h_res[:, 0]
            e2e_tokens += int(nb.sum())
            for b in range(BATCH):   # the host feeds back the last committed token
                h_anchor[b] = h_res[b, int(nb[b])]
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e = {"value": e2e_tokens / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": 4 * BATCH,
               "d2h_bytes_per_step": 4 * BATCH * (1 + K_BLOCK), "ms_per_step": e2e_ms / n_e2e}

    # ---------------------------------------------------------------- iterative draft (next row f1)
    it_line = None
    if n_iter:
        n_it = torch.zeros((ITER_STEPS, BATCH), dtype=torch.int32, device=dev)

        def step_it(j):
            eng.draft_block(anchor, K_BLOCK, T, 1234, out=draft, iterations=2)
            eng.verify_block(anchor, draft, K_BLOCK, T)
            eng.commit(anchor, K_BLOCK, T, 1234, n_out=n_it[j], tokens_out=toks)

        for j in range(3):
            step_it(j)
        torch.cuda.synchronize()
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2.record()
        for j in range(ITER_STEPS):
            step_it(j)
        e3.record()
        torch.cuda.synchronize()
        it_ms = e2.elapsed_time(e3)
        it_tok = int(n_it.sum())
        it_line = {"iterations": 2, "steps": ITER_STEPS, "ms_per_step": it_ms / ITER_STEPS,
                   "value": it_tok / (it_ms * 1e-3), "unit": UNIT,
                   "how": "the same decode step with a two-pass iterative-denoising draft (the diffusion view "
                          "re-run on its own drafts), CUDA events around the steps"}

    # ---------------------------------------------------------------- other decode loops
    variants = None
    if not args.no_variants:
        variants = decode_variants(eng, anchor, draft, toks, tokens / (ms * 1e-3), ms / K)
        st, bits = eng.check_error()
        if st != 0:
            raise RuntimeError(f"device error bits {bits:#x}")

    # ---------------------------------------------------------------- reduce
    tot_tokens, max_ms, e2e_sum = reduce_replicas(tokens, ms, e2e["value"] if e2e else 0.0, world, dev)
    if e2e:
        e2e["value"] = e2e_sum
    if rank != 0:
        return
    hbm, tflops, src = measured_peaks()
    g_ach = g_bytes / g_time / 1e9
    a_ach = a_bytes / a_time / 1e9
    traffic = kernel_traffic("gemm_projection_qwen3_8b_shape.txt", GEMM_SOURCES)
    gu_traffic = kernel_traffic("gemm_projection_qwen3_8b_shape.txt", GEMM_SOURCES, "dram_bytes_gate_up")
    gu_us = float(g_ms[:, 2].mean() * 1e3)
    gu_ach = gb[2] / (gu_us * 1e-6) / 1e9
    a_traffic = kernel_traffic("attention_qwen3_8b_shape.txt", ATTN_SOURCES, "dram_bytes_per_launch")
    value = tot_tokens / (max_ms * 1e-3)
    nbar = tokens / (K * BATCH)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (random-init weights, uniform random prompt)",
        "config": {"workload": "qwen3-8b-shape decode step (draft + verify + commit), batch 1 per GPU, K=32, "
                               "prompt 2048, greedy", "global_batch": BATCH * world, "seq_len": P_PROMPT,
                   "block_K": K_BLOCK, "split_tokens": args.split_tokens, "parallelism": f"replicas x{world}",
                   "l2": "weights (18 GB) and cache exceed L2 every step; no flush"},
        "mean_accepted_per_cycle": nbar, "tokens_per_forward": nbar / 2,
        "modelled_tokens_per_s_at_pages_acceptance": 10.8 / (max_ms / K * 1e-3),
        "roofline": {"kernel": "gate/up projection GEMM with the fused SwiGLU epilogue (gemm_tc_kernel<EPI_SWIGLU>, "
                               "the step's largest kernel by device time), one verify-view layer",
                     "bound": "hbm", "achieved": gu_ach, "peak": hbm, "unit": "GB/s", "frac": gu_ach / hbm,
                     "traffic": gu_traffic, "peak_source": src, "algorithmic_bytes": gb[2], "us_per_launch": gu_us,
                     "layer_gemms": {"kernel": "the four projection GEMMs (QKV, O, gate/up, down) of one layer",
                                     "achieved": g_ach, "frac": g_ach / hbm, "traffic": traffic,
                                     "algorithmic_bytes_per_layer": sum(gb),
                                     "note": "each GEMM is bracketed by its own CUDA events; under programmatic "
                                             "dependent launch a kernel starts while its predecessor drains, so "
                                             "the brackets overlap and are not disjoint times (their sum exceeds "
                                             "the step)",
                                     "ms_per_layer": float(g_ms.sum(axis=1).mean()),
                                     "per_gemm": {n: {"us": float(g_ms[:, i].mean() * 1e3),
                                                      "achieved_gbs": gb[i] / float(g_ms[:, i].mean() * 1e-3) / 1e9}
                                                  for i, n in enumerate(("qkv", "o", "gate_up", "down"))}}},
        "attn": {"kernel": "dual-view attention (cluster split + on-chip combine), verify view, one layer",
                 "bound": "hbm", "achieved": a_ach, "peak": hbm, "unit": "GB/s", "frac": a_ach / hbm,
                 "traffic": a_traffic, "us_per_call": float(a_ms.mean() * 1e3), "mean_prefix": float(t_steps.mean())},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if it_line:
        line["iterative_draft"] = it_line
    if variants:
        line.update(variants)
    if not args.profile_small:
        lc = attn_long_context(hbm, args.split_tokens)
        line["attn_long_context"] = lc
        # the single-layer attention workload (L = 4096, K = 32, batch 1):
        # its verify-view point is the attn headline, the step's own
        # attention (timed inside the decode step) stays beside it
        p4 = [p for p in lc["points"] if p["L"] == 4096 and p["batch"] == 1]
        if p4:
            v, dv = p4[0], (p4[1] if len(p4) > 1 else None)
            in_step = line["attn"]
            line["attn"] = {
                "kernel": "dual-view attention entry point, the single-layer workload (L = 4096 + K = 32, batch 1, "
                          "32/8 heads, head_dim 128), verify view",
                "bound": "hbm", "achieved": v["achieved"], "peak": hbm, "unit": "GB/s", "frac": v["frac"],
                "traffic": kernel_traffic("attention_l4k_single_layer.txt", ATTN_SOURCES, "dram_bytes_per_launch"),
                "us_per_call": v["us"], "how": lc["how"],
                "draft_view": {"achieved": dv["achieved"], "frac": dv["frac"], "us_per_call": dv["us"]} if dv else None,
                "in_step": in_step}
        line["train_kernels"] = train_kernels(hbm, tflops, eng)
        line["tree_kernels"] = tree_kernels(hbm)
    if args.sweep != "none" and world == 1:
        line["step_sweep"] = step_sweep(w, s, args.split_tokens, sweep_cells(args.sweep == "full"), hbm=hbm)
    if not args.no_variants and world == 1:
        line["config_1p7b"] = config_1p7b(args.split_tokens)
    if args.profile_small:
        line = {"profile_case": True, "config": "2 layers of the Qwen3-8B shape, vocab 32000", "value": value,
                "roofline": line["roofline"], "attn": line["attn"]}
    if not args.no_cpu_baseline and world == 1:
        sample = OracleSample()
        ests = [sample.step_seconds(ORACLE_ROWS) for _ in range(3)]
        est = statistics.mean(ests[1:])     # the first sample is the warm-up, as in the reference arm
        line["cpu_baseline"] = {"value": nbar / est, "unit": UNIT, "cores": sample.threads(), "kind": "oracle",
                                "sample": sample.describe(ORACLE_ROWS) + f"; mean of 2 samples after 1 warm-up; "
                                          f"tokens per step = {nbar:.3f} (this run's mean)",
                                "seconds_per_step": est}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.profile_train:
        hbm, tflops, _ = measured_peaks()
        res = train_kernels(hbm, tflops, None, reps=1, cpu=False)
        print(json.dumps({"profile_case": "training-side kernels alone", "train_kernels": res}), flush=True)
        return
    if args.profile_attn:
        hbm, _, _ = measured_peaks()
        res = attn_long_context(hbm, args.split_tokens, lengths=(args.profile_attn,), batched=(), reps=1)
        print(json.dumps({"profile_case": "attention entry point alone", "attn_long_context": res}), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
