"""Python binding of liborthrus.so, the B200 dual-view decode library.

Argument marshalling only: every step of the decode cycle runs in the
library's CUDA kernels ("Orthrus: Memory-Efficient Parallel Token Generation
via Dual-View Diffusion", paper notes §4.1: parallel projection, AR
verification, consensus and commit).  PyTorch provides device memory and
streams.  There is no CPU fallback: without the built library, or without a
CUDA device, the calls raise.

The functions named ``orthrus_*`` mirror include/orthrus.h one to one;
``Engine`` owns the torch allocations a run needs (weights, the paged KV
cache, the workspace) and calls them.
"""
from __future__ import annotations

import ctypes as C
import os

__all__ = ["lib", "Config", "Engine", "OrthrusError", "library_path", "DTYPE_BF16", "DTYPE_FP32"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liborthrus.so")
_lib = None

DTYPE_BF16, DTYPE_FP32 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "capacity exceeded", 4: "CUDA error",
          5: "device-side check failed", 6: "non-finite log-sum-exp"}


class OrthrusError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn",
                                         "vocab", "mask_token_id", "dtype", "max_batch", "max_block",
                                         "max_seq", "split_tokens")] + [("rope_theta", C.c_float),
                                                                        ("rms_eps", C.c_float)]


LAYER_FIELDS = ("attn_norm", "wq", "wk", "wv", "wq_diff", "wk_diff", "wv_diff", "wo", "ffn_norm", "w_gate",
                "w_up", "w_down")


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in LAYER_FIELDS]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p),
                ("layers", C.POINTER(LayerWeights))]


class KV(C.Structure):
    _fields_ = [("k_pages", C.c_void_p), ("v_pages", C.c_void_p), ("block_table", C.c_void_p),
                ("seq_lens", C.c_void_p), ("num_pages", C.c_int32), ("page_size", C.c_int32),
                ("max_pages_per_seq", C.c_int32)]


class Stats(C.Structure):
    _fields_ = [("cycles", C.c_int64), ("forwards", C.c_int64), ("tokens", C.c_int64), ("min_tokens", C.c_int64)]


_P = C.c_void_p
_I = C.c_int32
_SIGS = {
    "orthrus_workspace_size": [C.POINTER(Config), C.POINTER(C.c_size_t)],
    "orthrus_transient_bytes": [C.POINTER(Config), _I, _I, C.POINTER(C.c_size_t)],
    "orthrus_create": [C.POINTER(Config), C.POINTER(Weights), _P, C.c_size_t, C.POINTER(_P)],
    "orthrus_destroy": [_P],
    "orthrus_prefill": [_P, C.POINTER(KV), _P, _I, C.POINTER(_I), _I, _P, _P],
    "orthrus_draft_block": [_P, C.POINTER(KV), _P, _I, _I, C.c_float, C.c_uint64, _P, _P, _P],
    "orthrus_draft_block_iterative": [_P, C.POINTER(KV), _P, _I, _I, _I, C.c_float, C.c_uint64, _P, _P, _P],
    "orthrus_verify_block": [_P, C.POINTER(KV), _P, _P, _I, _I, C.c_float, _P],
    "orthrus_commit": [_P, C.POINTER(KV), _I, _I, C.c_float, C.c_uint64, _P, _P, _P, _P, _P, _P],
    "orthrus_ar_step": [_P, C.POINTER(KV), _I, C.c_float, C.c_uint64, _P, _P, _P, _P],
    "orthrus_generate": [_P, C.POINTER(KV), _P, _I, C.POINTER(_I), _I, _I, _I, C.c_float, C.c_uint64, _P,
                         C.POINTER(Stats), _P],
    "orthrus_dual_view_attention": [_P, C.POINTER(KV), _I, _I, _P, _P, _P, _I, _I, _P, _P],
    "orthrus_block_mask_attention": [_P, C.POINTER(KV), _I, _P, _P, _P, _P, _I, _I, _P, _P],
    "orthrus_kl_lm_head": [_P, _P, _P, _I, _P, _P, _P, _P],
    "orthrus_tree_topw": [_P, _P, _I, _I, _P, _P, _P, _P],
    "orthrus_tree_build": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P],
    "orthrus_tree_commit": [_P, C.POINTER(KV), _I, _I, _P, _P, _P, _P, _P, _P, _P, _P],
    "orthrus_verify_tree": [_P, C.POINTER(KV), _P, _P, _P, _I, _I, _P, _P],
    "orthrus_draft_block_topw": [_P, C.POINTER(KV), _P, _I, _I, _I, _I, _P, _P, _P, _P, _P],
    "orthrus_debug_logits": [_P, _I, _I, _I, _P, _P],
    "orthrus_debug_rows": [_P, _I, _I, _I, _P, _P, _P, _P],
    "orthrus_adaptive_len": [_P, _I, _I, C.c_float, _P, _P, _P],
    "orthrus_commit_adaptive": [_P, C.POINTER(KV), _I, _I, _P, _P, _P, _P, _P, _P],
    "orthrus_check_error": [_P, _P, C.POINTER(C.c_uint32)],
    "orthrus_set_probe": [_P, _I, _I, _I, C.POINTER(_P), C.POINTER(_P), _I],
    "orthrus_dual_view_attention_noalloc": [C.POINTER(Config), C.POINTER(KV), _I, _I, _P, _P, _P, _I, _I, _P, _P,
                                            _P],
}


def lib():
    """Load liborthrus.so (raises if it was never built: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing; build it with "
                              "`python -m dual_view_diffusion_b200.build` (nvcc, sm_100a)")
        l = C.CDLL(_LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(l, name)
            f.argtypes = args
            f.restype = C.c_int
        l.orthrus_launch_count.argtypes = [_P]
        l.orthrus_launch_count.restype = C.c_uint64
        l.orthrus_status_string.argtypes = [C.c_int]
        l.orthrus_status_string.restype = C.c_char_p
        _lib = l
    return _lib


def _check(name, status):
    if status != 0:
        raise OrthrusError(name, status)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


# ------------------------------------------------------------- C-ABI mirrors
def orthrus_workspace_size(cfg: Config) -> int:
    n = C.c_size_t()
    _check("orthrus_workspace_size", lib().orthrus_workspace_size(C.byref(cfg), C.byref(n)))
    return n.value


def orthrus_transient_bytes(cfg: Config, batch: int, K: int) -> int:
    n = C.c_size_t()
    _check("orthrus_transient_bytes", lib().orthrus_transient_bytes(C.byref(cfg), batch, K, C.byref(n)))
    return n.value


def make_config(shape, dtype, max_batch, max_block, max_seq, split_tokens=256) -> Config:
    """Config from any object with the model-shape attributes (n_layers,
    hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, rope_theta,
    rms_eps); the mask id is vocab - 1."""
    return Config(shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.ffn,
                  shape.vocab, shape.vocab - 1, DTYPE_BF16 if dtype == "bf16" else DTYPE_FP32, max_batch,
                  max_block, max_seq, split_tokens, shape.rope_theta, shape.rms_eps)


def _need(x, dtype, name):
    """Marshalling check: a contiguous device tensor of the dtype the C call reads."""
    if x.dtype != dtype or not x.is_cuda or not x.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {x.dtype} on {x.device}")


class Engine:
    """One model on one CUDA device: weights, a paged KV cache and a
    context.  `weights` is either host arrays (attributes embed, final_norm,
    lm_head, layers = list of dicts keyed like LAYER_FIELDS) or the same
    structure of device torch tensors already in the model dtype."""

    def __init__(self, shape, weights, *, dtype=None, max_batch=1, max_block=32, max_seq=4096,
                 split_tokens=256, page_size=64, device="cuda"):
        import torch
        self.torch = torch
        self.shape = shape
        self.dtype_name = dtype or shape.dtype
        self.tdtype = torch.bfloat16 if self.dtype_name == "bf16" else torch.float32
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError(f"Engine runs on a CUDA device only (got {self.device}); the library has no CPU path")
        n_layers = len(weights.layers)
        shape_l = type("S", (), {k: getattr(shape, k) for k in ("hidden", "n_q_heads", "n_kv_heads", "head_dim",
                                                                  "ffn", "vocab", "rope_theta", "rms_eps")})()
        shape_l.n_layers = n_layers
        self.cfg = make_config(shape_l, self.dtype_name, max_batch, max_block, max_seq, split_tokens)
        self.n_layers = n_layers

        def dev(a):
            if isinstance(a, torch.Tensor):
                return a.to(self.device, self.tdtype).contiguous()
            return torch.from_numpy(a).to(self.device).to(self.tdtype).contiguous()

        self._keep = []
        embed = dev(weights.embed)
        head = embed if weights.lm_head is weights.embed else dev(weights.lm_head)
        fnorm = dev(weights.final_norm)
        self._keep += [embed, head, fnorm]
        self._layers = (LayerWeights * n_layers)()
        self.layer_tensors = []
        for i, lw in enumerate(weights.layers):
            tl = {}
            for f in LAYER_FIELDS:
                t = dev(lw[f])
                tl[f] = t
                setattr(self._layers[i], f, t.data_ptr())
            self.layer_tensors.append(tl)
        self.embed, self.lm_head, self.final_norm = embed, head, fnorm
        self._w = Weights(embed.data_ptr(), fnorm.data_ptr(), head.data_ptr(), self._layers)

        # paged cache: sequence b owns pages [b * pps, (b + 1) * pps)
        self.page_size = page_size
        self.pages_per_seq = (max_seq + page_size - 1) // page_size
        num_pages = max_batch * self.pages_per_seq
        # K pages [slot][dim], V pages transposed [dim][slot] (see orthrus_kv_t)
        kshape = (n_layers, num_pages, shape.n_kv_heads, page_size, shape.head_dim)
        vshape = (n_layers, num_pages, shape.n_kv_heads, shape.head_dim, page_size)
        self.k_pages = torch.zeros(kshape, dtype=self.tdtype, device=self.device)
        self.v_pages = torch.zeros(vshape, dtype=self.tdtype, device=self.device)
        self.block_table = torch.arange(num_pages, dtype=torch.int32, device=self.device).view(max_batch, -1)
        self.seq_lens = torch.zeros(max_batch, dtype=torch.int32, device=self.device)
        self.kv = KV(self.k_pages.data_ptr(), self.v_pages.data_ptr(), self.block_table.data_ptr(),
                     self.seq_lens.data_ptr(), num_pages, page_size, self.pages_per_seq)

        self.ws_bytes = orthrus_workspace_size(self.cfg)
        self.workspace = torch.empty(self.ws_bytes + 256, dtype=torch.uint8, device=self.device)
        base = self.workspace.data_ptr()
        self._ws_ptr = (base + 255) & ~255
        ctx = C.c_void_p()
        _check("orthrus_create", lib().orthrus_create(C.byref(self.cfg), C.byref(self._w), C.c_void_p(self._ws_ptr),
                                                      C.c_size_t(self.ws_bytes), C.byref(ctx)))
        self.ctx = ctx
        self.step = torch.zeros(1, dtype=torch.int64, device=self.device)

    def __del__(self):
        try:
            if getattr(self, "ctx", None):
                lib().orthrus_destroy(self.ctx)
                self.ctx = None
        except Exception:
            pass

    # -------------------------------------------------------------- calls
    def _i32(self, x):
        t = self.torch
        if isinstance(x, t.Tensor):
            return x.to(self.device, t.int32).contiguous()
        return t.as_tensor(x, dtype=t.int32, device=self.device).contiguous()

    def prefill(self, prompts, lens=None):
        """prompts: [B, S] ids; lens: per-sequence lengths (default S)."""
        p = self._i32(prompts)
        if p.dim() == 1:
            p = p[None]
        B, S = p.shape
        lens = [S] * B if lens is None else list(lens)
        L = (C.c_int32 * B)(*lens)
        anchor = self.torch.empty(B, dtype=self.torch.int32, device=self.device)
        _check("orthrus_prefill", lib().orthrus_prefill(self.ctx, C.byref(self.kv), _ptr(p), S, L, B, _ptr(anchor),
                                                        _stream()))
        return anchor

    def draft_block(self, anchor, K, temperature=0.0, seed=0, step=None, out=None, iterations=1):
        """iterations > 1: the iterative-denoising draft (diffusion view re-run
        on its own previous drafts)."""
        B = anchor.numel()
        draft = out if out is not None else self.torch.empty((B, K), dtype=self.torch.int32, device=self.device)
        st = self.step if step is None else step
        if iterations == 1:
            _check("orthrus_draft_block", lib().orthrus_draft_block(
                self.ctx, C.byref(self.kv), _ptr(anchor), B, K, float(temperature), seed, _ptr(st), _ptr(draft),
                _stream()))
        else:
            _check("orthrus_draft_block_iterative", lib().orthrus_draft_block_iterative(
                self.ctx, C.byref(self.kv), _ptr(anchor), B, K, int(iterations), float(temperature), seed, _ptr(st),
                _ptr(draft), _stream()))
        return draft

    def draft_block_topw(self, anchor, K, width, depth=None, out=None):
        """Greedy draft plus, for draft rows k < depth (default K - 1), the
        `width` best ids and logits and each row's log-sum-exp, taken inside
        the LM-head pass: (draft [B, K], ids [B, depth, width], vals, lse
        [B, depth])."""
        t = self.torch
        B = anchor.numel()
        depth = K - 1 if depth is None else depth
        draft = out if out is not None else t.empty((B, K), dtype=t.int32, device=self.device)
        ids = t.empty((B, depth, width), dtype=t.int32, device=self.device)
        vals = t.empty((B, depth, width), dtype=t.float32, device=self.device)
        lse = t.empty((B, depth), dtype=t.float32, device=self.device)
        _check("orthrus_draft_block_topw", lib().orthrus_draft_block_topw(
            self.ctx, C.byref(self.kv), _ptr(anchor), B, K, int(width), int(depth), _ptr(draft), _ptr(ids),
            _ptr(vals), _ptr(lse), _stream()))
        return draft, ids, vals, lse

    def verify_block(self, anchor, draft, K, temperature=0.0):
        B = anchor.numel()
        _check("orthrus_verify_block", lib().orthrus_verify_block(self.ctx, C.byref(self.kv), _ptr(anchor),
                                                                  _ptr(draft), B, K, float(temperature), _stream()))

    def commit(self, anchor, K, temperature=0.0, seed=0, step=None, force_n=None, n_out=None, tokens_out=None):
        """Consensus + commit; anchor is updated in place.  Returns (n, tokens)."""
        B = anchor.numel()
        t = self.torch
        n = n_out if n_out is not None else t.empty(B, dtype=t.int32, device=self.device)
        toks = tokens_out if tokens_out is not None else t.empty((B, K), dtype=t.int32, device=self.device)
        _check("orthrus_commit", lib().orthrus_commit(self.ctx, C.byref(self.kv), B, K, float(temperature), seed,
                                                      _ptr(self.step if step is None else step), _ptr(force_n),
                                                      _ptr(n), _ptr(toks), _ptr(anchor), _stream()))
        return n, toks

    def adaptive_len(self, B, K, h_max, kt=None, entropy=False):
        """Per-sequence verify length after a greedy draft (rows whose
        entropy is at most h_max extend it).  Returns kt [B] (and the draft
        rows' entropies [B, K] when entropy=True)."""
        t = self.torch
        kt = kt if kt is not None else t.empty(B, dtype=t.int32, device=self.device)
        ent = t.empty((B, K), dtype=t.float32, device=self.device) if entropy else None
        _check("orthrus_adaptive_len", lib().orthrus_adaptive_len(self.ctx, B, K, float(h_max), _ptr(kt), _ptr(ent),
                                                                  _stream()))
        return (kt, ent) if entropy else kt

    def commit_adaptive(self, anchor, K, kt, step=None, n_out=None, tokens_out=None):
        """Greedy consensus over the first kt[b] verified rows + commit;
        anchor is updated in place.  Returns (n, tokens)."""
        B = anchor.numel()
        t = self.torch
        n = n_out if n_out is not None else t.empty(B, dtype=t.int32, device=self.device)
        toks = tokens_out if tokens_out is not None else t.empty((B, K), dtype=t.int32, device=self.device)
        _check("orthrus_commit_adaptive", lib().orthrus_commit_adaptive(
            self.ctx, C.byref(self.kv), B, K, _ptr(kt), _ptr(self.step if step is None else step), _ptr(n),
            _ptr(toks), _ptr(anchor), _stream()))
        return n, toks

    def ar_step(self, anchor, temperature=0.0, seed=0, step=None, token_out=None):
        B = anchor.numel()
        t = self.torch
        tok = token_out if token_out is not None else t.empty(B, dtype=t.int32, device=self.device)
        _check("orthrus_ar_step", lib().orthrus_ar_step(self.ctx, C.byref(self.kv), B, float(temperature), seed,
                                                        _ptr(self.step if step is None else step), _ptr(tok),
                                                        _ptr(anchor), _stream()))
        return tok

    def generate(self, prompts, K, max_new, temperature=0.0, seed=0, lens=None):
        """K = 0 runs plain AR decoding.  Returns (tokens [B, max_new], stats)."""
        p = self._i32(prompts)
        if p.dim() == 1:
            p = p[None]
        B, S = p.shape
        lens = [S] * B if lens is None else list(lens)
        L = (C.c_int32 * B)(*lens)
        out = self.torch.zeros((B, max_new), dtype=self.torch.int32, device=self.device)
        st = Stats()
        _check("orthrus_generate", lib().orthrus_generate(self.ctx, C.byref(self.kv), _ptr(p), S, L, B, K, max_new,
                                                          float(temperature), seed, _ptr(out), C.byref(st),
                                                          _stream()))
        return out, {"cycles": st.cycles, "forwards": st.forwards, "tokens": st.tokens,
                     "min_tokens": st.min_tokens}

    def attention(self, layer, mode, q, k_blk, v_blk, B, K):
        out = self.torch.empty_like(q)
        _check("orthrus_dual_view_attention", lib().orthrus_dual_view_attention(
            self.ctx, C.byref(self.kv), layer, mode, _ptr(q), _ptr(k_blk), _ptr(v_blk), B, K, _ptr(out),
            _stream()))
        return out

    def block_mask_attention(self, layer, q, k_blk, v_blk, anchors, K):
        """Training-side block-masked attention of one packed sequence:
        block b (rows [b*K, (b+1)*K) of q) sees context positions
        [0, anchors[b]) of block-table row 0 and its own K rows.
        anchors: device int32 [n_blocks]."""
        n_blocks = int(anchors.numel())
        out = self.torch.empty_like(q)
        _check("orthrus_block_mask_attention", lib().orthrus_block_mask_attention(
            self.ctx, C.byref(self.kv), layer, _ptr(q), _ptr(k_blk), _ptr(v_blk), _ptr(anchors), n_blocks, K,
            _ptr(out), _stream()))
        return out

    def kl_lm_head(self, h_ar, h_diff):
        """Forward KL(softmax(W h_ar) || softmax(W h_diff)) per row through the
        LM head, with both log-sum-exps: three fp32 [rows] tensors."""
        rows = int(h_ar.shape[0])
        kl = self.torch.empty(rows, dtype=self.torch.float32, device=self.device)
        la, ld = self.torch.empty_like(kl), self.torch.empty_like(kl)
        _check("orthrus_kl_lm_head", lib().orthrus_kl_lm_head(
            self.ctx, _ptr(h_ar), _ptr(h_diff), rows, _ptr(kl), _ptr(la), _ptr(ld), _stream()))
        return kl, la, ld

    def tree_topw(self, logits, width):
        """The `width` best ids and logits of each fp32 logits row, and the
        row's log-sum-exp: (ids int32 [rows, width], vals fp32, lse fp32)."""
        t = self.torch
        _need(logits, t.float32, "logits")
        z = logits.reshape(-1, logits.shape[-1]).contiguous()
        if int(z.shape[1]) != self.shape.vocab:
            raise ValueError(f"logits rows must have {self.shape.vocab} entries")
        rows = int(z.shape[0])
        ids = t.empty((rows, width), dtype=t.int32, device=self.device)
        vals = t.empty((rows, width), dtype=t.float32, device=self.device)
        lse = t.empty(rows, dtype=t.float32, device=self.device)
        _check("orthrus_tree_topw", lib().orthrus_tree_topw(self.ctx, _ptr(z), rows, width, _ptr(ids), _ptr(vals),
                                                            _ptr(lse), _stream()))
        return ids, vals, lse

    def tree_build(self, ids, vals, lse, nodes):
        """Best-first draft trees from per-depth candidates ids/vals [B, D, W]
        and lse [B, D]: (parent, token, depth, score [B, nodes + 1], n_rows [B])."""
        t = self.torch
        for name, x, dt in (("ids", ids, t.int32), ("vals", vals, t.float32), ("lse", lse, t.float32)):
            _need(x, dt, name)
        B, D, W = (int(x) for x in ids.shape)
        par, tok, dep = (t.empty((B, nodes + 1), dtype=t.int32, device=self.device) for _ in range(3))
        sc = t.empty((B, nodes + 1), dtype=t.float64, device=self.device)
        nr = t.empty(B, dtype=t.int32, device=self.device)
        _check("orthrus_tree_build", lib().orthrus_tree_build(
            self.ctx, _ptr(ids), _ptr(vals), _ptr(lse), B, D, W, nodes, _ptr(par), _ptr(tok), _ptr(dep), _ptr(sc),
            _ptr(nr), _stream()))
        return par, tok, dep, sc, nr

    def verify_tree(self, anchor, parent, token):
        """Tree-masked AR verification of trees parent/token [B, rows] (row 0
        the anchor): returns each row's AR argmax g [B, rows]."""
        t = self.torch
        for name, x in (("anchor", anchor), ("parent", parent), ("token", token)):
            _need(x, t.int32, name)
        B, R = (int(x) for x in parent.shape)
        g = t.empty((B, R), dtype=t.int32, device=self.device)
        _check("orthrus_verify_tree", lib().orthrus_verify_tree(self.ctx, C.byref(self.kv), _ptr(anchor), _ptr(parent),
                                                                _ptr(token), B, R, _ptr(g), _stream()))
        return g

    def tree_commit(self, parent, token, n_rows, g, anchor):
        """Greedy acceptance on verified trees [B, rows] and the commit of the
        accepted paths' K/V; anchor [B] is updated in place.  Returns
        (n [B], emitted tokens [B, rows])."""
        t = self.torch
        for name, x in (("parent", parent), ("token", token), ("n_rows", n_rows), ("g", g), ("anchor", anchor)):
            _need(x, t.int32, name)
        B, R = (int(x) for x in parent.shape)
        n = t.empty(B, dtype=t.int32, device=self.device)
        emit = t.full((B, R), -1, dtype=t.int32, device=self.device)
        _check("orthrus_tree_commit", lib().orthrus_tree_commit(
            self.ctx, C.byref(self.kv), B, R, _ptr(parent), _ptr(token), _ptr(n_rows), _ptr(g), _ptr(n), _ptr(emit),
            _ptr(anchor), _stream()))
        return n, emit

    def debug_logits(self, which, B, K, out=None):
        """fp32 logits [B, K, vocab] of the last verify (which = 0) or draft
        (which = 1), from the final hidden rows they kept."""
        if out is None:
            out = self.torch.empty((B, K, self.shape.vocab), dtype=self.torch.float32, device=self.device)
        _need(out, self.torch.float32, "out")
        _check("orthrus_debug_logits", lib().orthrus_debug_logits(self.ctx, which, B, K, _ptr(out), _stream()))
        return out

    def debug_rows(self, which, B, K):
        """(tokens int32, log-probability of the row's token, log-sum-exp)
        [B, K] of the last verify (which = 0: AR argmax, log p(y_k)) or draft
        (which = 1: drafted token, log q(y_k))."""
        t = self.torch
        tok = t.empty((B, K), dtype=t.int32, device=self.device)
        lp, lse = t.empty((B, K), dtype=t.float32, device=self.device), t.empty((B, K), dtype=t.float32,
                                                                              device=self.device)
        _check("orthrus_debug_rows", lib().orthrus_debug_rows(self.ctx, which, B, K, _ptr(tok), _ptr(lp), _ptr(lse),
                                                              _stream()))
        return tok, lp, lse

    def check_error(self):
        bits = C.c_uint32()
        st = lib().orthrus_check_error(self.ctx, _stream(), C.byref(bits))
        return st, bits.value

    def set_probe(self, family, layer, view, starts, stops):
        """Record torch.cuda.Event pairs around the launches of one kernel
        family in one layer of every forward of `view` (see
        orthrus_set_probe); empty lists disable it."""
        n = len(starts)
        for e in list(starts) + list(stops):
            if not e.cuda_event:       # torch creates the CUDA event on first record
                e.record()
        S = (C.c_void_p * max(n, 1))(*[e.cuda_event for e in starts])
        E = (C.c_void_p * max(n, 1))(*[e.cuda_event for e in stops])
        _check("orthrus_set_probe", lib().orthrus_set_probe(self.ctx, family, layer, view, S, E, n))

    def launch_count(self):
        return int(lib().orthrus_launch_count(self.ctx))

    def transient_bytes(self, batch, K):
        return orthrus_transient_bytes(self.cfg, batch, K)
