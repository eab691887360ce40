"""ctypes binding of the plain fp64 CPU oracle (orthrus_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are its only users.  The CUDA product path never
imports it, and it never imports the product package.

The C source follows the paper-notes page on "Orthrus: Memory-Efficient
Parallel Token Generation via Dual-View Diffusion" (§2.1 dual-view layer,
§3.2 diffusion mask, §4.1-4.3 the decode cycle and its consensus; §3.1-3.3
the training-side block mask and forward KL; §7.5 / §9.6 tree verification
of one draft's marginals and the adaptive block length); each C function
cites the passage it restates.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "orthrus_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, ERR_ARG, ERR_NOMEM, ERR_CAPACITY = 0, 1, 2, 3
PURPOSE_DRAFT, PURPOSE_ACCEPT, PURPOSE_RESIDUAL, PURPOSE_AR = 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim",
                                       "ffn", "vocab", "mask_id")] + [("rope_theta", C.c_double),
                                                                      ("rms_eps", C.c_double)]


_LAYER_FIELDS = ("attn_norm", "wq", "wk", "wv", "wq_diff", "wk_diff", "wv_diff",
                 "wo", "ffn_norm", "w_gate", "w_up", "w_down")


class _Layer(C.Structure):
    _fields_ = [(n, C.POINTER(C.c_float)) for n in _LAYER_FIELDS]


class _Model(C.Structure):
    _fields_ = [("embed", C.POINTER(C.c_float)), ("final_norm", C.POINTER(C.c_float)),
                ("lm_head", C.POINTER(C.c_float)), ("layers", C.POINTER(_Layer))]


_D = C.POINTER(C.c_double)
_F = C.POINTER(C.c_float)
_I = C.POINTER(C.c_int32)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            l = C.CDLL(build())
            P = C.POINTER
            l.oc_rmsnorm.argtypes = [_D, _F, C.c_int, C.c_double, _D]
            l.oc_linear.argtypes = [_D, C.c_int, C.c_int, _F, C.c_int, _D]
            l.oc_rope.argtypes = [_D, C.c_int, C.c_int, C.c_int, C.c_double]
            l.oc_silu.argtypes = [C.c_double]
            l.oc_silu.restype = C.c_double
            l.oc_attention.argtypes = [_D, C.c_int, C.c_int, C.c_int, C.c_int, _D, _D, C.c_int, _D, _D, C.c_int, _D]
            l.oc_forward.argtypes = [P(_Cfg), P(_Model), C.c_int, C.c_int, _I, C.c_int, C.c_int,
                                     _D, _D, C.c_int, _D, _D]
            l.oc_prefill.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, _D, _D, C.c_int]
            l.oc_philox4x32_10.argtypes = [P(C.c_uint32), P(C.c_uint32), P(C.c_uint32)]
            l.oc_uniform.argtypes = [C.c_uint64, C.c_uint32, C.c_uint32, C.c_uint32, C.c_uint32]
            l.oc_uniform.restype = C.c_double
            l.oc_gumbel.argtypes = l.oc_uniform.argtypes
            l.oc_gumbel.restype = C.c_double
            l.oc_gumbel_vec.argtypes = [C.c_uint64, C.c_uint32, C.c_uint32, C.c_uint32, C.c_int, _D]
            l.oc_argmax.argtypes = [_D, C.c_int, _D]
            l.oc_softmax_t.argtypes = [_D, C.c_int, C.c_double, _D]
            l.oc_sample_logits.argtypes = [_D, C.c_int, C.c_double, C.c_uint64, C.c_uint32, C.c_uint32,
                                           C.c_uint32, _D]
            l.oc_consensus_greedy.argtypes = [_I, _I, C.c_int, _I]
            l.oc_accept_prob.argtypes = [C.c_double, C.c_double]
            l.oc_accept_prob.restype = C.c_double
            l.oc_residual.argtypes = [_D, _D, C.c_int, _D]
            l.oc_draft.argtypes = [P(_Cfg), P(_Model), _D, _D, C.c_int, C.c_int, C.c_int32, C.c_int,
                                   C.c_double, C.c_uint64, C.c_uint32, _I, _D, _D, _D]
            l.oc_draft_iter.argtypes = [P(_Cfg), P(_Model), _D, _D, C.c_int, C.c_int, C.c_int32, C.c_int,
                                        C.c_int, C.c_double, C.c_uint64, C.c_uint32, _I, _D, _D, _D]
            l.oc_verify.argtypes = [P(_Cfg), P(_Model), _D, _D, C.c_int, C.c_int, C.c_int32, _I, C.c_int,
                                    C.c_double, _I, _D, _D, _D]
            l.oc_consensus_sample.argtypes = [_D, _D, _I, _I, C.c_int, C.c_int, C.c_uint64, C.c_uint32, _I, _D]
            l.oc_generate.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_int, C.c_double,
                                      C.c_uint64, C.c_int, _I, _I, P(C.c_int), _D, _D, _D, P(C.c_int)]
            l.oc_generate_iter.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_int, C.c_double,
                                           C.c_uint64, C.c_int, C.c_int, _I, _I, P(C.c_int), _D, _D, _D,
                                           P(C.c_int), _D]
            l.oc_enumerate_ar.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_double, _D]
            l.oc_enumerate_orthrus.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_int,
                                               C.c_double, C.c_int, _D]
            l.oc_enumerate_orthrus_2pass.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_int,
                                                     C.c_double, C.c_int, _D]
            l.oc_block_mask_attention.argtypes = [_D, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _D, _D,
                                                  C.c_int, _D, _D, _I, _D]
            l.oc_kl_rows.argtypes = [_D, _D, C.c_int, C.c_int, _F, C.c_int, _D, _D, _D]
            l.oc_attention_tree.argtypes = [_D, C.c_int, C.c_int, C.c_int, C.c_int, _D, _D, C.c_int, _D, _D, _I,
                                            _D]
            l.oc_forward_tree.argtypes = [P(_Cfg), P(_Model), _I, _I, C.c_int, C.c_int, _D, _D, C.c_int, _D]
            l.oc_topw.argtypes = [_D, C.c_int, C.c_int, _I, _D]
            l.oc_entropy.argtypes = [_D, C.c_int]
            l.oc_entropy.restype = C.c_double
            l.oc_adaptive_len.argtypes = [_D, C.c_int, C.c_double]
            l.oc_generate_adaptive.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_double, C.c_int, _I,
                                               _I, _I, P(C.c_int), _D, _D, P(C.c_int)]
            l.oc_tree_build.argtypes = [_D, C.c_int, C.c_int, C.c_int, C.c_int, _I, _I, _I, _D]
            l.oc_tree_accept.argtypes = [_I, _I, C.c_int, _I, _I, _I]
            l.oc_tree_commit_kv.argtypes = [_D, _D, C.c_int, C.c_int, C.c_int, C.c_int, _I, C.c_int]
            l.oc_generate_tree.argtypes = [P(_Cfg), P(_Model), _I, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                           _I, _I, P(C.c_int), _D, _D, P(C.c_int)]
            _lib = l
    return _lib


def _dp(a):
    return a.ctypes.data_as(_D) if a is not None else None


def _fp(a):
    return a.ctypes.data_as(_F)


def _ip(a):
    return a.ctypes.data_as(_I) if a is not None else None


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


# ---------------------------------------------------------------- primitives
def rmsnorm(x, gain, eps=1e-6):
    x = _f64(x); g = _f32(gain); y = np.empty_like(x)
    lib().oc_rmsnorm(_dp(x), _fp(g), x.size, eps, _dp(y))
    return y


def linear(x, W):
    x = _f64(np.atleast_2d(x)); W = _f32(W)
    y = np.empty((x.shape[0], W.shape[0]))
    lib().oc_linear(_dp(x), x.shape[0], x.shape[1], _fp(W), W.shape[0], _dp(y))
    return y


def rope(x, pos, theta=1e6):
    """x [n_heads, hd] -> rotated copy."""
    x = _f64(np.atleast_2d(x)).copy()
    lib().oc_rope(_dp(x), x.shape[0], x.shape[1], int(pos), float(theta))
    return x


def silu(g):
    return lib().oc_silu(float(g))


def attention(q, kc, vc, kb, vb, mode):
    """q [R, n_q, hd]; kc/vc [t, n_kv, hd]; kb/vb [R, n_kv, hd]; mode 0 = AR
    causal block, 1 = diffusion bidirectional block.  Returns o [R, n_q, hd]."""
    q, kb, vb = _f64(q), _f64(kb), _f64(vb)
    R, nq, hd = q.shape
    nkv = kb.shape[1]
    t = 0 if kc is None else kc.shape[0]
    kc = _f64(kc) if t else np.zeros((1, nkv, hd))
    vc = _f64(vc) if t else np.zeros((1, nkv, hd))
    o = np.empty_like(q)
    lib().oc_attention(_dp(q), R, nq, nkv, hd, _dp(kc), _dp(vc), t, _dp(kb), _dp(vb), int(mode), _dp(o))
    return o


def block_mask_attention(q, kctx, vctx, kblk, vblk, anchors, K):
    """Diffusion-pass attention of one packed training sequence under the
    dual-pass block mask.  q [n_blocks*K, n_q, hd]; kctx/vctx [L, n_kv, hd]
    (clean context, AR view); kblk/vblk [n_blocks*K, n_kv, hd] (the blocks'
    diffusion K/V); anchors [n_blocks].  Returns o [n_blocks*K, n_q, hd]."""
    q, kblk, vblk = _f64(q), _f64(kblk), _f64(vblk)
    rows, nq, hd = q.shape
    nkv = kblk.shape[1]
    L = 0 if kctx is None else kctx.shape[0]
    kctx = _f64(kctx) if L else np.zeros((1, nkv, hd))
    vctx = _f64(vctx) if L else np.zeros((1, nkv, hd))
    a = _i32(anchors)
    nb = a.size
    assert rows == nb * K
    o = np.empty_like(q)
    lib().oc_block_mask_attention(_dp(q), nb, K, nq, nkv, hd, _dp(kctx), _dp(vctx), L, _dp(kblk), _dp(vblk),
                                  _ip(a), _dp(o))
    return o


def kl_rows(hA, hD, W):
    """Forward KL(softmax(W hA) || softmax(W hD)) per row, and both
    log-sum-exps.  hA/hD [rows, d] (final-normed hidden rows), W [V, d]."""
    hA, hD, W = _f64(np.atleast_2d(hA)), _f64(np.atleast_2d(hD)), _f32(W)
    rows, d = hA.shape
    kl, la, ld = np.empty(rows), np.empty(rows), np.empty(rows)
    lib().oc_kl_rows(_dp(hA), _dp(hD), rows, d, _fp(W), W.shape[0], _dp(kl), _dp(la), _dp(ld))
    return kl, la, ld


def attention_tree(q, kc, vc, kb, vb, parent):
    """Tree-masked attention: row r sees the cache and the rows of its own
    root path (parent[0] = -1, parent[r] < r).  Shapes as attention()."""
    q, kb, vb, par = _f64(q), _f64(kb), _f64(vb), _i32(parent)
    R, nq, hd = q.shape
    nkv = kb.shape[1]
    t = 0 if kc is None else kc.shape[0]
    kc = _f64(kc) if t else np.zeros((1, nkv, hd))
    vc = _f64(vc) if t else np.zeros((1, nkv, hd))
    o = np.empty_like(q)
    lib().oc_attention_tree(_dp(q), R, nq, nkv, hd, _dp(kc), _dp(vc), t, _dp(kb), _dp(vb), _ip(par), _dp(o))
    return o


def topw(z, W):
    """The W largest entries of each row of z (ties: lowest id) and each
    row's log-sum-exp: (ids int32 [rows, W], lse [rows])."""
    z = _f64(np.atleast_2d(z))
    rows, V = z.shape
    ids = np.zeros((rows, W), np.int32)
    lse = np.zeros(rows)
    for r in range(rows):
        out = C.c_double()
        lib().oc_topw(_dp(z[r]), V, int(W), _ip(ids[r]), C.byref(out))
        lse[r] = out.value
    return ids, lse


def entropy(z):
    """Entropy (nats) of softmax(z) at T = 1."""
    z = _f64(z)
    return lib().oc_entropy(_dp(z), z.size)


def adaptive_len(H, h_max):
    """The adaptive verify length for draft-row entropies H [K]."""
    H = _f64(H)
    return lib().oc_adaptive_len(_dp(H), H.size, float(h_max))


def tree_build(logp, W, N):
    """Best-first draft tree over logp [D, V] (row d: log-probabilities of
    the token at depth d + 1), W candidates per depth, N prefixes.  Returns
    (parent, token, depth, score) of the root plus the chosen nodes, in
    selection order."""
    lp = _f64(np.atleast_2d(logp))
    D, V = lp.shape
    par, tok, dep = (np.zeros(N + 1, np.int32) for _ in range(3))
    sc = np.zeros(N + 1)
    n = lib().oc_tree_build(_dp(lp), D, V, int(W), int(N), _ip(par), _ip(tok), _ip(dep), _dp(sc))
    if n < 0:
        raise ValueError(f"oc_tree_build failed: {-n}")
    return par[:n], tok[:n], dep[:n], sc[:n]


def tree_accept(parent, token, g):
    """Greedy walk of a verified tree: returns (n, emitted tokens, path rows)."""
    par, tok, g = _i32(parent), _i32(token), _i32(g)
    R = par.size
    emit, path = np.zeros(R, np.int32), np.zeros(R, np.int32)
    n = lib().oc_tree_accept(_ip(par), _ip(tok), R, _ip(g), _ip(emit), _ip(path))
    return n, emit[:n], path[:n]


def tree_commit_kv(kc, vc, t, path):
    """In place: path row path[i]'s K/V (slot t + path[i]) to slot t + i.
    kc/vc [n_layers, cap, n_kv, hd] float64 C-contiguous."""
    assert kc.dtype == np.float64 and kc.flags.c_contiguous and vc.flags.c_contiguous
    p = _i32(path)
    nl, cap = kc.shape[:2]
    kn = int(np.prod(kc.shape[2:]))
    lib().oc_tree_commit_kv(_dp(kc), _dp(vc), nl, cap, kn, int(t), _ip(p), p.size - 1)


def philox4x32_10(ctr, key):
    c = (C.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (C.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (C.c_uint32 * 4)()
    lib().oc_philox4x32_10(c, k, o)
    return [o[i] for i in range(4)]


def uniform(seed, step, row, id_, purpose):
    return lib().oc_uniform(seed, step, row, id_, purpose)


def gumbel(seed, step, row, id_, purpose):
    return lib().oc_gumbel(seed, step, row, id_, purpose)


def gumbel_vec(seed, step, row, purpose, n):
    """gumbel(seed, step, row, i, purpose) for i = 0 .. n-1."""
    g = np.empty(n)
    lib().oc_gumbel_vec(seed, step, row, purpose, int(n), _dp(g))
    return g


def argmax(x):
    x = _f64(x); m = C.c_double()
    i = lib().oc_argmax(_dp(x), x.size, C.byref(m))
    return i, m.value


def softmax_t(z, T):
    z = _f64(z); p = np.empty_like(z)
    lib().oc_softmax_t(_dp(z), z.size, float(T), _dp(p))
    return p


def sample_logits(z, T, seed, step, row, purpose):
    z = _f64(z); m = C.c_double()
    i = lib().oc_sample_logits(_dp(z), z.size, float(T), seed, step, row, purpose, C.byref(m))
    return i, m.value


def consensus_greedy(draft, g):
    draft, g = _i32(draft), _i32(g)
    emit = np.zeros_like(g)
    n = lib().oc_consensus_greedy(_ip(draft), _ip(g), draft.size, _ip(emit))
    return n, emit[:n]


def accept_prob(p, q):
    return lib().oc_accept_prob(float(p), float(q))


def residual(p, q):
    p, q = _f64(p), _f64(q); r = np.zeros_like(p)
    none = lib().oc_residual(_dp(p), _dp(q), p.size, _dp(r))
    return None if none else r


# ---------------------------------------------------------------- the model
class Model:
    """Oracle view of one model: synth.Weights (fp32 host arrays) + shape."""

    def __init__(self, w):
        s = w.shape
        self.shape = s
        self.cfg = _Cfg(s.n_layers if not w.layers else len(w.layers), s.hidden, s.n_q_heads,
                        s.n_kv_heads, s.head_dim, s.ffn, s.vocab, s.mask_id, s.rope_theta, s.rms_eps)
        self._keep = []

        def k(a):
            a = _f32(a)
            self._keep.append(a)
            return _fp(a)

        n = len(w.layers)
        self._layers = (_Layer * n)()
        for i, lw in enumerate(w.layers):
            for f in _LAYER_FIELDS:
                setattr(self._layers[i], f, k(lw[f]))
        self.model = _Model(k(w.embed), k(w.final_norm), k(w.lm_head), self._layers)
        self.n_layers = n

    # cache helpers -----------------------------------------------------
    def new_cache(self, cap):
        s = self.shape
        sz = (self.n_layers, cap, s.n_kv_heads, s.head_dim)
        return np.zeros(sz), np.zeros(sz)

    def forward(self, view, mode, tokens, t, kc, vc, want_hidden=False, logits=True):
        """One forward of a block; kc/vc are modified in place (mode 0 writes
        rows t .. t+R-1).  Returns logits [R, V] (and final hidden rows);
        logits=False skips the LM head and returns None for them."""
        tok = _i32(tokens)
        R = tok.size
        cap = kc.shape[1]
        logits = np.empty((R, self.shape.vocab)) if logits else None
        hid = np.empty((R, self.shape.hidden)) if want_hidden else None
        rc = lib().oc_forward(C.byref(self.cfg), C.byref(self.model), int(view), int(mode), _ip(tok), R,
                              int(t), _dp(kc), _dp(vc), cap, _dp(logits), _dp(hid))
        if rc:
            raise RuntimeError(f"oc_forward failed: {rc}")
        return (logits, hid) if want_hidden else logits

    def prefill(self, prompt, kc, vc):
        p = _i32(prompt)
        t = lib().oc_prefill(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, _dp(kc), _dp(vc),
                             kc.shape[1])
        if t < 0:
            raise RuntimeError(f"oc_prefill failed: {-t}")
        return t

    def draft(self, kc, vc, t, anchor, K, T=0.0, seed=0, step=0, iterations=1):
        """iterations > 1: the iterative-denoising draft (oc_draft_iter)."""
        V = self.shape.vocab
        d = np.zeros(K, np.int32)
        q = np.zeros((K, V)) if T > 0 else None
        z = np.zeros((K, V))
        mg = C.c_double(np.inf)
        rc = lib().oc_draft_iter(C.byref(self.cfg), C.byref(self.model), _dp(kc), _dp(vc), kc.shape[1], int(t),
                                 int(anchor), int(K), int(iterations), float(T), seed, step, _ip(d), _dp(q),
                                 _dp(z), C.byref(mg))
        if rc:
            raise RuntimeError(f"oc_draft failed: {rc}")
        return d, q, z, mg.value

    def verify(self, kc, vc, t, anchor, draft, T=0.0):
        V = self.shape.vocab
        K = len(draft)
        g = np.zeros(K, np.int32)
        p = np.zeros((K, V)) if T > 0 else None
        z = np.zeros((K, V))
        mg = C.c_double(np.inf)
        dr = _i32(draft)
        rc = lib().oc_verify(C.byref(self.cfg), C.byref(self.model), _dp(kc), _dp(vc), kc.shape[1], int(t),
                             int(anchor), _ip(dr), K, float(T), _ip(g), _dp(p), _dp(z), C.byref(mg))
        if rc:
            raise RuntimeError(f"oc_verify failed: {rc}")
        return g, p, z, mg.value

    def generate(self, prompt, K, N, T=0.0, seed=0, method="orthrus", want_cache=False, iterations=1):
        """method 'orthrus' or 'ar'; iterations = diffusion passes per draft.
        Returns a dict with tokens, n_per_cycle, cycles, min_margin,
        cycle_margin (the smallest decision margin of each cycle), t and
        (optionally) the committed cache."""
        p = _i32(prompt)
        out = np.zeros(N, np.int32)
        npc = np.zeros(N, np.int32)
        cmg = np.zeros(N)
        cyc = C.c_int()
        mg = C.c_double()
        tt = C.c_int()
        cap = p.size + N + K
        kc = vc = None
        if want_cache:
            kc, vc = self.new_cache(cap)
        rc = lib().oc_generate_iter(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, int(K), int(N),
                                    float(T), seed, 1 if method == "orthrus" else 0, int(iterations), _ip(out),
                                    _ip(npc), C.byref(cyc), C.byref(mg), _dp(kc), _dp(vc), C.byref(tt), _dp(cmg))
        if rc:
            raise RuntimeError(f"oc_generate failed: {rc}")
        res = {"tokens": out, "n_per_cycle": npc[:cyc.value], "cycles": cyc.value, "min_margin": mg.value,
               "cycle_margin": cmg[:cyc.value], "t": tt.value}
        if want_cache:
            res["k_cache"], res["v_cache"] = kc, vc
        return res

    def forward_tree(self, tokens, parent, t, kc, vc):
        """AR forward of a draft tree (rows = nodes, parent[0] = -1); K/V
        written at slots t .. t+R-1 of kc/vc (in place).  Returns logits."""
        tok, par = _i32(tokens), _i32(parent)
        z = np.empty((tok.size, self.shape.vocab))
        rc = lib().oc_forward_tree(C.byref(self.cfg), C.byref(self.model), _ip(tok), _ip(par), tok.size, int(t),
                                   _dp(kc), _dp(vc), kc.shape[1], _dp(z))
        if rc:
            raise RuntimeError(f"oc_forward_tree failed: {rc}")
        return z

    def generate_tree(self, prompt, K, W, nodes, N, want_cache=False):
        """Greedy decoding with best-first tree verification (W candidates
        per depth, `nodes` prefixes per cycle).  Returns a dict like
        generate()."""
        p = _i32(prompt)
        out = np.zeros(N, np.int32)
        npc = np.zeros(N, np.int32)
        cyc = C.c_int()
        tt = C.c_int()
        cap = p.size + N + nodes + 1
        kc = vc = None
        if want_cache:
            kc, vc = self.new_cache(cap)
        rc = lib().oc_generate_tree(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, int(K), int(W),
                                    int(nodes), int(N), _ip(out), _ip(npc), C.byref(cyc), _dp(kc), _dp(vc),
                                    C.byref(tt))
        if rc:
            raise RuntimeError(f"oc_generate_tree failed: {rc}")
        res = {"tokens": out, "n_per_cycle": npc[:cyc.value], "cycles": cyc.value, "t": tt.value}
        if want_cache:
            res["k_cache"], res["v_cache"] = kc, vc
        return res

    def generate_adaptive(self, prompt, K, h_max, N, want_cache=False):
        """Greedy decoding whose cycles verify only the drafted tokens whose
        draft rows have entropy <= h_max (at most K rows).  Returns a dict
        like generate() plus k_per_cycle."""
        p = _i32(prompt)
        out = np.zeros(N, np.int32)
        npc = np.zeros(N, np.int32)
        kpc = np.zeros(N, np.int32)
        cyc = C.c_int()
        tt = C.c_int()
        kc = vc = None
        if want_cache:
            kc, vc = self.new_cache(p.size + N + K)
        rc = lib().oc_generate_adaptive(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, int(K), float(h_max),
                                        int(N), _ip(out), _ip(npc), _ip(kpc), C.byref(cyc), _dp(kc), _dp(vc),
                                        C.byref(tt))
        if rc:
            raise RuntimeError(f"oc_generate_adaptive failed: {rc}")
        res = {"tokens": out, "n_per_cycle": npc[:cyc.value], "k_per_cycle": kpc[:cyc.value], "cycles": cyc.value,
               "t": tt.value}
        if want_cache:
            res["k_cache"], res["v_cache"] = kc, vc
        return res

    def enumerate_ar(self, prompt, N, T):
        p = _i32(prompt)
        dist = np.zeros(self.shape.vocab ** N)
        rc = lib().oc_enumerate_ar(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, int(N), float(T),
                                   _dp(dist))
        if rc:
            raise RuntimeError(f"oc_enumerate_ar failed: {rc}")
        return dist

    def enumerate_orthrus(self, prompt, K, N, T, planted_error=False, passes=1):
        """passes = 1 (single-step draft) or 2 (two-pass iterative draft)."""
        p = _i32(prompt)
        dist = np.zeros(self.shape.vocab ** N)
        fn = lib().oc_enumerate_orthrus if passes == 1 else lib().oc_enumerate_orthrus_2pass
        if passes not in (1, 2):
            raise ValueError("passes must be 1 or 2")
        rc = fn(C.byref(self.cfg), C.byref(self.model), _ip(p), p.size, int(K), int(N), float(T),
                int(bool(planted_error)), _dp(dist))
        if rc:
            raise RuntimeError(f"oc_enumerate_orthrus failed: {rc}")
        return dist
