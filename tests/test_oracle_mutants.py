"""Mutation check of the oracle's pins.

Each entry below plants one plausible mistake (a dropped term, a wrong sign,
index, operand or comparison) into one function of a copy of the oracle's C
source, builds the copy into a temporary directory and runs the pins named
beside it against that build: at least one of them must fail.  A control
build of the unchanged source passes every pin the catalogue names, so a
failure is the planted mistake's.  The tracked oracle source and its library
are never modified; the binding is pointed at the planted build for the
duration of one check only.

Every planted change keeps all memory accesses inside the buffers the
original touches (the mutants change values, masks and orders, never an
allocation size), so a build cannot crash the test process.
"""
import concurrent.futures as cf
import dataclasses
import os
import re
import subprocess

import pytest

import oracle
import synth
import test_oracle_adaptive as AD
import test_oracle_pins as P
import test_oracle_tree as TR

SRC = os.path.join(os.path.dirname(oracle.__file__), "orthrus_oracle.c")


@dataclasses.dataclass(frozen=True)
class Mutant:
    name: str
    function: str        # the C function the change is confined to
    old: str
    new: str
    pins: tuple          # pin names (see _pins) of which at least one must fail
    count: int = 1       # occurrences of `old` inside the function


MUTANTS = (
    # building blocks of the backbone (notes §2.1)
    Mutant("rmsnorm sums instead of averaging", "oc_rmsnorm", "sqrt(ss / n + eps)", "sqrt(ss + eps)", ("rmsnorm",)),
    Mutant("rmsnorm drops the gain", "oc_rmsnorm", "y[i] = x[i] * inv * (double)gain[i];", "y[i] = x[i] * inv;",
           ("rmsnorm",)),
    Mutant("rope rotates the wrong way", "oc_rope", "v[i] = a * c - b * s;", "v[i] = a * c + b * s;", ("rope",)),
    Mutant("rope frequency exponent halved", "oc_rope", "pow(theta, -2.0 * i / hd)", "pow(theta, -1.0 * i / hd)",
           ("hf_forward",)),
    Mutant("rope pairs adjacent dims", "oc_rope",
           "double a = v[i], b = v[i + half];\n            v[i] = a * c - b * s;\n            v[i + half] = b * c + a * s;",
           "double a = v[2 * i], b = v[2 * i + 1];\n            v[2 * i] = a * c - b * s;\n"
           "            v[2 * i + 1] = b * c + a * s;", ("rope",)),
    Mutant("silu uses the wrong sign", "oc_silu", "exp(-g)", "exp(g)", ("silu",)),
    Mutant("linear transposes the weight", "oc_linear", "const float *w = W + (size_t)o * in;",
           "const float *w = W + (size_t)o;", ("hf_forward",)),
    # attention (notes §3.2, §4.1)
    Mutant("attention scale 1/hd", "oc_attention", "1.0 / sqrt((double)hd)", "1.0 / (double)hd", ("sdpa",)),
    Mutant("draft mask made causal", "oc_attention", "int nblk = (mode == 0) ? r + 1 : R;", "int nblk = r + 1;",
           ("sdpa",)),
    Mutant("verify mask sees the whole block", "oc_attention", "int nblk = (mode == 0) ? r + 1 : R;",
           "int nblk = R;", ("sdpa",)),
    Mutant("cache excluded from the keys", "oc_attention", "int nkeys = t + nblk;", "int nkeys = nblk;", ("sdpa",)),
    Mutant("GQA head map h mod n_kv", "oc_attention", "int kvh = h / g;", "int kvh = h % n_kv;", ("sdpa",)),
    Mutant("values read from the keys", "oc_attention",
           "const double *vv = (j < t) ? vc + ", "const double *vv = (j < t) ? kc + ", ("sdpa",)),
    Mutant("softmax not normalised", "oc_attention", "double p = s[j] / l;", "double p = s[j];",
           ("sdpa", "attn_special")),
    # one forward of either view (notes §2.1, §2.2)
    Mutant("attention residual dropped", "forward_rows",
           "oc_linear(o, R, nq * hd, L->wo, d, y);\n        for (size_t i = 0; i < (size_t)R * d; ++i) h[i] += y[i];",
           "oc_linear(o, R, nq * hd, L->wo, d, y);\n        for (size_t i = 0; i < (size_t)R * d; ++i) h[i] = y[i];",
           ("hf_forward",)),
    Mutant("SwiGLU gates the wrong operand", "forward_rows", "gt[i] = oc_silu(gt[i]) * up[i];",
           "gt[i] = gt[i] * oc_silu(up[i]);", ("hf_forward",)),
    Mutant("FFN norm uses the attention gain", "forward_rows", "L->ffn_norm, d", "L->attn_norm, d", ("hf_forward",)),
    Mutant("final norm skipped", "forward_rows",
           "oc_rmsnorm(h + (size_t)r * d, w->final_norm, d, c->rms_eps, a + (size_t)r * d);",
           "memcpy(a + (size_t)r * d, h + (size_t)r * d, sizeof(double) * d);", ("hf_forward",)),
    Mutant("all rows at position t", "forward_rows", "pos[r] = !parent ? t + r :", "pos[r] = !parent ? t :",
           ("hf_forward",)),
    Mutant("diffusion view keeps the AR W_K", "forward_rows", "view ? L->wk_diff : L->wk", "L->wk", ("views",)),
    Mutant("diffusion view keeps the AR W_V", "forward_rows", "view ? L->wv_diff : L->wv", "L->wv", ("views",)),
    Mutant("prefill skips the first prompt token", "oc_prefill", "prompt, P - 1, 0,", "prompt + 1, P - 1, 0,",
           ("hf_stream",)),
    # the cycle (notes §4.1-§4.3)
    Mutant("draft block without mask tokens", "oc_draft_iter", "s == 0 ? c->mask_id : draft[k - 1]",
           "s == 0 ? anchor : draft[k - 1]", ("draft",)),
    Mutant("verify block shifted by one", "oc_verify", "for (int k = 1; k < K; ++k) blk[k] = draft[k - 1];",
           "for (int k = 1; k < K; ++k) blk[k] = draft[k];", ("verify", "greedy_eq_ar")),
    Mutant("greedy emits the draft at the mismatch", "oc_consensus_greedy", "emit[k] = g[k];",
           "emit[k] = draft[k];", ("greedy_examples",)),
    Mutant("greedy accepts past a mismatch", "oc_consensus_greedy", "if (draft[k] != g[k]) return k + 1;",
           "if (draft[k] != g[k] && k > 0) return k + 1;", ("greedy_examples",)),
    Mutant("acceptance ratio inverted", "oc_accept_prob", "double a = p / q;", "double a = q / p;",
           ("accept_residual",)),
    Mutant("residual of q - p", "oc_residual", "double d = p[i] - q[i];", "double d = q[i] - p[i];",
           ("accept_residual",), count=2),
    Mutant("residual left unnormalised", "oc_residual", "r[i] = (d > 0.0 ? d : 0.0) / s;",
           "r[i] = (d > 0.0 ? d : 0.0);", ("accept_residual",)),
    Mutant("acceptance test inverted", "oc_consensus_sample", "if (u < a)", "if (u > a)", ("sampler_mc",)),
    Mutant("correction drawn from p", "oc_consensus_sample", "lr[i] = r[i] > 0.0 ? log(r[i]) : -INFINITY;",
           "lr[i] = log(pk[i]);", ("sampler_mc",)),
    Mutant("commit keeps the first emitted token as anchor", "oc_generate_iter", "anchor = emit[n - 1];",
           "anchor = emit[0];", ("greedy_eq_ar",)),
    Mutant("commit advances one row", "oc_generate_iter", "t += n;", "t += 1;", ("greedy_eq_ar",)),
    # randomness (Philox4x32-10, Gumbel-max)
    Mutant("philox key schedule constant", "oc_philox4x32_10", "k1 += 0xBB67AE85u;", "k1 += 0xBB67AE86u;",
           ("philox_kat",)),
    Mutant("philox multiplies the wrong word", "oc_philox4x32_10", "(uint64_t)0xD2511F53u * x0",
           "(uint64_t)0xD2511F53u * x1", ("philox_kat",)),
    Mutant("gumbel noise negated", "oc_gumbel", "return -log(-log(", "return log(-log(", ("gumbel_chi2",)),
    Mutant("gumbel-max ignores the temperature", "oc_sample_logits", "double s = z[i] / T + oc_gumbel(",
           "double s = z[i] + oc_gumbel(", ("gumbel_chi2",)),
    Mutant("softmax ignores the temperature", "oc_softmax_t", "p[i] = exp(z[i] / T - m);", "p[i] = exp(z[i] - m);",
           ("softmax_t", "hf_law")),
    Mutant("argmax ties to the highest index", "oc_argmax", "if (x[i] > b)", "if (x[i] >= b)", ("argmax",)),
    # training side (notes §3.1-§3.3)
    Mutant("block mask shows the anchor's context row", "oc_block_mask_attention", "visible = j < anchors[b];",
           "visible = j <= anchors[b];", ("block_mask_invisible",)),
    Mutant("blocks see earlier blocks", "oc_block_mask_attention", "visible = (int)(jb / K) == b;",
           "visible = (int)(jb / K) <= b;", ("block_mask_per_block",)),
    Mutant("reverse KL", "oc_kl_rows", "acc += exp(lpa) * (lpa - lpd);", "acc += exp(lpd) * (lpd - lpa);",
           ("kl_scipy",)),
    Mutant("KL without the p weight", "oc_kl_rows", "acc += exp(lpa) * (lpa - lpd);", "acc += lpa - lpd;",
           ("kl_scipy",)),
    # tree verification (notes §7.5, §9.6)
    Mutant("top-W ties to the highest id", "oc_topw", "z[v] > z[best]", "z[v] >= z[best]", ("topw",)),
    Mutant("top-W log-sum-exp drops the max", "oc_topw", "*lse = m + log(s);", "*lse = log(s);", ("topw",)),
    Mutant("sibling scored from the chosen node", "oc_tree_build", "ps[np] = score[par] + logp[",
           "ps[np] = sc + logp[", ("tree_brute",)),
    Mutant("tree one level too shallow", "oc_tree_build", "if (d < D) {", "if (d < D - 1) {", ("tree_brute",)),
    Mutant("tree walk compares the child's argmax", "oc_tree_accept", "token[c] == g[cur]", "token[c] == g[c]",
           ("tree_accept",)),
    Mutant("tree commit leaves K in place", "oc_tree_commit_kv", "kl + (size_t)(t + path[i]) * kn",
           "kl + (size_t)(t + i) * kn", ("tree_commit",)),
    Mutant("tree mask hides the node itself", "oc_attention_tree",
           "for (int a = r; a >= 0; a = parent[a]) on_path[a] = 1;",
           "for (int a = parent[r]; a >= 0; a = parent[a]) on_path[a] = 1;", ("tree_sdpa",)),
    Mutant("tree mask is the causal mask", "oc_attention_tree", "if (j >= t && !on_path[j - t]) continue;",
           "if (j >= t && j - t > r) continue;", ("tree_sdpa",), count=3),
    Mutant("tree rows at their row positions", "forward_rows", "(r == 0 ? t : pos[parent[r]] + 1)", "t + r",
           ("tree_forward",)),
    Mutant("tree scores from unnormalised logits", "oc_generate_tree", "lp[(size_t)d * V + v] = zr[v] - m - log(s);",
           "lp[(size_t)d * V + v] = zr[v] - m;", ("tree_cycle",)),
    Mutant("tree depths from the next draft row", "oc_generate_tree", "const double *zr = z + (size_t)d * V;",
           "const double *zr = z + (size_t)(d + 1) * V;", ("tree_cycle",)),
    Mutant("tree root is the first draft, not the anchor", "oc_generate_tree", "tok[0] = anchor;",
           "tok[0] = draft[0];", ("tree_eq_ar", "tree_cycle")),
    # adaptive block length (notes §7.4, §9.6)
    Mutant("entropy sign", "oc_entropy", "return lse - e;", "return e - lse;", ("entropy",)),
    Mutant("threshold made strict", "oc_adaptive_len", "H[k - 1] <= h_max", "H[k - 1] < h_max", ("adaptive_len",)),
    Mutant("length rule reads the next row", "oc_adaptive_len", "H[k - 1] <= h_max", "H[k] <= h_max",
           ("adaptive_len",)),
    Mutant("every row's entropy taken from row 0", "oc_generate_adaptive",
           "H[k] = oc_entropy(z + (size_t)k * V, V);", "H[k] = oc_entropy(z, V);", ("adaptive_cycle",)),
    # the iterative draft (notes §5.4.2) and the exact law of the sampled cycle (notes §4.3)
    Mutant("second pass reads the drafts one row late", "oc_draft_iter", "s == 0 ? c->mask_id : draft[k - 1]",
           "s == 0 ? c->mask_id : draft[k]", ("iterative_pass2",)),
    Mutant("two-pass proposal taken from the first pass", "oc_draft_iter", "if (last && q_probs) oc_softmax_t(",
           "if (s == 0 && q_probs) oc_softmax_t(", ("proposal_last_pass", "sampler_mc_2pass")),
    Mutant("enumeration forgets the acceptance so far", "oc_enumerate_orthrus", "double rej = acc * (1.0 - a);",
           "double rej = 1.0 - a;", ("lossless_enum",)),
)

SDPA_CASES = ((0, 1, 0), (0, 5, 1), (37, 4, 0), (37, 4, 1))
TREE_CASES = ((3, 7, 3, 10, "normal"), (4, 5, 3, 20, "integer ties"))


def _adaptive_model():
    return oracle.Model(synth.make_weights(AD.SHAPE, 0)), synth.make_prompt(AD.SHAPE, 16, 0)


def _pins(tw, tp):
    """Pin name -> a call of that pin (the tests of the oracle's pin files)."""
    return {
        "philox_kat": P.test_philox_known_answers,
        "gumbel_chi2": P.test_gumbel_max_samples_softmax,
        "softmax_t": P.test_softmax_t_matches_torch,
        "argmax": P.test_argmax_lowest_index_and_margin,
        "rmsnorm": P.test_rmsnorm_closed_form_and_torch,
        "silu": P.test_silu,
        "rope": P.test_rope_identity_norm_relative,
        "sdpa": lambda: [P.test_attention_matches_torch_sdpa(*c) for c in SDPA_CASES],
        "attn_special": P.test_attention_special_cases,
        "hf_forward": P.test_ar_forward_matches_hf_llama,
        "hf_stream": P.test_ar_greedy_stream_matches_hf_llama,
        "hf_law": P.test_ar_law_matches_hf_llama,
        "views": lambda: P.test_diffusion_view_is_the_network_with_its_own_projections(tw, tp),
        "draft": lambda: P.test_draft_is_the_diffusion_view_of_anchor_and_masks(tw, tp),
        "verify": lambda: P.test_verify_is_the_ar_view_of_anchor_and_drafts(tw, tp),
        "greedy_examples": P.test_consensus_greedy_examples,
        "accept_residual": P.test_accept_and_residual,
        "greedy_eq_ar": lambda: [P.test_greedy_orthrus_equals_ar(tw, tp, K) for K in (1, 2, 4, 8)],
        "sampler_mc": lambda: P.test_sampler_matches_ar_law_monte_carlo(1),
        "sampler_mc_2pass": lambda: P.test_sampler_matches_ar_law_monte_carlo(2),
        "proposal_last_pass": lambda: P.test_sampled_draft_proposal_is_the_last_pass(tw, tp),
        "block_mask_per_block": P.test_block_mask_equals_per_block_diffusion_attention,
        "block_mask_invisible": P.test_block_mask_blocks_are_mutually_invisible_and_anchor_excluded,
        "kl_scipy": P.test_kl_rows_matches_library_relative_entropy,
        "topw": TR.test_topw_matches_numpy_and_scipy,
        "tree_brute": lambda: [TR.test_tree_build_matches_brute_force(*c) for c in TREE_CASES],
        "tree_accept": TR.test_tree_accept_worked_examples,
        "tree_commit": TR.test_tree_commit_kv_moves_the_path,
        "tree_sdpa": TR.test_attention_tree_matches_sdpa_and_chain,
        "tree_forward": lambda: TR.test_forward_tree_rows_equal_root_path_forwards(tw, tp),
        "tree_cycle": lambda: TR.test_tree_cycle_is_its_retyped_steps(tw, tp),
        "tree_eq_ar": lambda: TR.test_greedy_tree_decoding_equals_ar(tw, tp, 8, 4, 20),
        "iterative_pass2": lambda: P.test_iterative_draft_second_pass_sees_first_drafts(tw, tp),
        "lossless_enum": lambda: P.test_sampled_orthrus_is_lossless_by_enumeration(0.7),
        "adaptive_cycle": lambda: AD.test_adaptive_cycle_is_its_retyped_steps(_adaptive_model()),
        "entropy": AD.test_entropy_matches_scipy_and_closed_forms,
        "adaptive_len": AD.test_adaptive_len_worked_examples,
    }


def _function_span(src, name):
    """[start, end) of the definition of C function `name` in src."""
    for m in re.finditer(r"^[A-Za-z][^\n;{}]*\b" + re.escape(name) + r"\(", src, re.MULTILINE):
        brace = src.index("{", m.end())
        if ";" in src[m.end():brace]:
            continue                      # a prototype, not the definition
        depth = 0
        for j in range(brace, len(src)):
            depth += {"{": 1, "}": -1}.get(src[j], 0)
            if depth == 0:
                return m.start(), j + 1
    raise KeyError(name)


def plant(src, mutant):
    a, b = _function_span(src, mutant.function)
    body = src[a:b]
    assert body.count(mutant.old) == mutant.count, (mutant.name, body.count(mutant.old))
    return src[:a] + body.replace(mutant.old, mutant.new) + src[b:]


def _build(text, directory, stem):
    c_path, so_path = os.path.join(directory, stem + ".c"), os.path.join(directory, stem + ".so")
    with open(c_path, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-w", "-o", so_path, c_path, "-lm"])
    return so_path


@pytest.fixture(scope="module")
def planted_builds(tmp_path_factory):
    src = open(SRC).read()
    d = str(tmp_path_factory.mktemp("planted_oracle"))
    jobs = {"control": src}
    jobs.update({f"m{i:02d}": plant(src, m) for i, m in enumerate(MUTANTS)})
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        futs = {k: ex.submit(_build, text, d, k) for k, text in jobs.items()}
        return {k: f.result() for k, f in futs.items()}


def _use_build(monkeypatch, path):
    monkeypatch.setattr(oracle, "build", lambda force=False: path)
    monkeypatch.setattr(oracle, "_lib", None)


def test_catalogue_names_known_pins(tiny_weights, tiny_prompt):
    pins = _pins(tiny_weights, tiny_prompt)
    names = [m.name for m in MUTANTS]
    assert len(set(names)) == len(names)
    for m in MUTANTS:
        assert m.pins and all(p in pins for p in m.pins), m.name


def test_control_build_passes_every_named_pin(planted_builds, monkeypatch, tiny_weights, tiny_prompt):
    _use_build(monkeypatch, planted_builds["control"])
    pins = _pins(tiny_weights, tiny_prompt)
    for name in sorted({p for m in MUTANTS for p in m.pins}):
        pins[name]()


@pytest.mark.parametrize("i", range(len(MUTANTS)), ids=[m.name.replace(" ", "_") for m in MUTANTS])
def test_planted_mistake_fails_a_pin(i, planted_builds, monkeypatch, tiny_weights, tiny_prompt):
    m = MUTANTS[i]
    _use_build(monkeypatch, planted_builds[f"m{i:02d}"])
    pins = _pins(tiny_weights, tiny_prompt)
    failed = []
    for name in m.pins:
        try:
            pins[name]()
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught: {m.name}"
