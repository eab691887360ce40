"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module only draws numbers and formats them (fp32 / bf16 rounding of the
draws).  It holds none of the decoding method's arithmetic: no norm, no
projection, no attention, no sampling rule.  Every random number that the
method itself draws at run time (Gumbel noise, acceptance uniforms) is not
made here: each side implements the counter-based Philox4x32-10 generator
from its published definition.

Recipe (the workloads of "Orthrus: Memory-Efficient Parallel Token Generation
via Dual-View Diffusion", whose evaluation prompts are reasoning benchmarks
that are not available here; uniform random prompts of the stated lengths
stand in for them):

* every AR matrix (embedding, W_Q/W_K/W_V/W_O, gate/up/down, LM head) is
  N(0, 0.02), drawn in fp64 and rounded once to the model dtype
  (fp32, or bf16 through fp32 with round-to-nearest-even at both steps);
* the diffusion-view W_Q/W_K/W_V of each layer are the AR draw plus
  N(0, sigma_diff) noise, added in fp64 before the single rounding;
* norm gains are 1 unless a test asks for random gains;
* prompt ids are uniform over [0, vocab - 1), so the mask id vocab - 1 never
  appears in a prompt.

Streams are keyed by (seed, name); the name is hashed with CRC-32 so that the
key does not depend on the order in which tensors are drawn.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "ModelShape", "TINY", "MICRO", "QWEN3_1_7B", "QWEN3_8B", "shape_by_name",
    "rng", "normal", "uniform_ids", "round_bf16", "round_fp32", "bf16_bits",
    "bits_to_f32", "make_weights", "make_prompt",
]


@dataclass(frozen=True)
class ModelShape:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    tied: bool
    dtype: str            # "fp32" or "bf16"
    sigma_diff: float     # std of the noise added to the AR copy for W^diff
    std: float = 0.02
    rope_theta: float = 1e6
    rms_eps: float = 1e-6

    @property
    def mask_id(self) -> int:
        return self.vocab - 1

    @property
    def qkv_out(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim


# The tiny fp32 model, the Qwen3-1.7B and Qwen3-8B shapes (random init), and
# a micro model small enough for exact enumeration of the sampled decode.
TINY = ModelShape("tiny", 2, 64, 4, 2, 16, 128, 256, False, "fp32", 0.002)
MICRO = ModelShape("micro", 1, 16, 2, 1, 8, 32, 8, False, "fp32", 0.05, std=0.3)
QWEN3_1_7B = ModelShape("qwen3-1.7b", 28, 2048, 16, 8, 128, 6144, 151936, True, "bf16", 1e-3)
QWEN3_8B = ModelShape("qwen3-8b", 36, 4096, 32, 8, 128, 12288, 151936, False, "bf16", 1e-3)

_SHAPES = {s.name: s for s in (TINY, MICRO, QWEN3_1_7B, QWEN3_8B)}


def shape_by_name(name: str) -> ModelShape:
    return _SHAPES[name]


def rng(seed: int, name: str) -> np.random.Generator:
    """Independent stream for (seed, name): numpy's Philox bit generator keyed
    by seed in the high word and CRC-32(name) in the low word."""
    key = (int(seed) << 32) | zlib.crc32(name.encode())
    return np.random.Generator(np.random.Philox(key=key))


def round_fp32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns of x (fp64 -> fp32 -> bf16, each round to
    nearest even; finite inputs only)."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    b = f.view(np.uint32)          # finite values: b + 0x8000 never overflows 32 bits
    r = (b >> 16) & 1
    r += 0x7FFF
    r += b
    r >>= 16
    return r.astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """x rounded to bf16, returned as fp32 (exactly representable values)."""
    return bits_to_f32(bf16_bits(x))


def normal(shape, std: float, seed: int, name: str) -> np.ndarray:
    """fp64 N(0, std^2) draws (not yet rounded)."""
    return rng(seed, name).standard_normal(size=shape, dtype=np.float64) * std


def uniform_ids(n: int, high: int, seed: int, name: str) -> np.ndarray:
    """n ids uniform over [0, high)."""
    return rng(seed, name).integers(0, high, size=n, dtype=np.int64).astype(np.int32)


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(x) if dtype == "bf16" else round_fp32(x)


@dataclass
class Weights:
    """Host copies of one model's weights, every matrix row-major [out][in]
    (the nn.Linear convention), values already rounded to the model dtype
    and held as fp32.  Per-layer lists are indexed by layer."""
    shape: ModelShape
    embed: np.ndarray
    final_norm: np.ndarray
    lm_head: np.ndarray
    layers: list = field(default_factory=list)


LAYER_KEYS = ("attn_norm", "wq", "wk", "wv", "wq_diff", "wk_diff", "wv_diff",
              "wo", "ffn_norm", "w_gate", "w_up", "w_down")


def make_weights(s: ModelShape, seed: int, n_layers: int | None = None,
                 random_gains: bool = False, diff_equals_ar: bool = False) -> Weights:
    """Draw one model.  n_layers overrides the depth (same per-layer recipe,
    so a shallower model is a prefix of the deeper one)."""
    L = s.n_layers if n_layers is None else n_layers
    d, hq, hkv, hd, F, V = s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab
    embed = _round(normal((V, d), s.std, seed, "embed"), s.dtype)
    lm_head = embed if s.tied else _round(normal((V, d), s.std, seed, "lm_head"), s.dtype)

    def gain(name):
        if not random_gains:
            return np.ones(d, dtype=np.float32)
        return _round(1.0 + 0.25 * rng(seed, name).standard_normal(d), s.dtype)

    layers = []
    for l in range(L):
        lw = {"attn_norm": gain(f"L{l}.attn_norm"), "ffn_norm": gain(f"L{l}.ffn_norm")}
        for key, rows in (("wq", hq * hd), ("wk", hkv * hd), ("wv", hkv * hd)):
            base = normal((rows, d), s.std, seed, f"L{l}.{key}")
            lw[key] = _round(base, s.dtype)
            if diff_equals_ar:
                lw[key + "_diff"] = lw[key]
            else:
                noise = normal((rows, d), s.sigma_diff, seed, f"L{l}.{key}_diff_noise")
                lw[key + "_diff"] = _round(base + noise, s.dtype)
        lw["wo"] = _round(normal((d, hq * hd), s.std, seed, f"L{l}.wo"), s.dtype)
        lw["w_gate"] = _round(normal((F, d), s.std, seed, f"L{l}.w_gate"), s.dtype)
        lw["w_up"] = _round(normal((F, d), s.std, seed, f"L{l}.w_up"), s.dtype)
        lw["w_down"] = _round(normal((d, F), s.std, seed, f"L{l}.w_down"), s.dtype)
        layers.append(lw)
    return Weights(s, embed, gain("final_norm"), lm_head, layers)


def make_prompt(s: ModelShape, length: int, seed: int, name: str = "prompt") -> np.ndarray:
    """Uniform random prompt over [0, vocab - 1) (the mask id never appears)."""
    return uniform_ids(length, s.vocab - 1, seed, name)


def make_weights_torch(s: ModelShape, seed: int, device="cuda", n_layers: int | None = None):
    """Device-side draw of the same recipe for shapes too large for the host
    generator (the 8B shape has 9.1e9 parameters): torch's Philox generator
    on the device, seeded per tensor from (seed, name); values drawn in fp32,
    the diffusion copy formed in fp32 and rounded once to the model dtype.
    The values differ from make_weights' (a different generator) but follow
    the same distributions; tests that compare against the oracle copy the
    pieces they need back to the host."""
    import torch
    L = s.n_layers if n_layers is None else n_layers
    d, hq, hkv, hd, F, V = s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab
    dt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device)

    def draw(shape, std, name):
        gen.manual_seed((int(seed) << 32) | zlib.crc32(name.encode()))
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).mul_(std)

    embed = draw((V, d), s.std, "embed").to(dt)
    lm_head = embed if s.tied else draw((V, d), s.std, "lm_head").to(dt)
    ones = torch.ones(d, device=device, dtype=dt)
    layers = []
    for l in range(L):
        lw = {"attn_norm": ones, "ffn_norm": ones}
        for key, rows in (("wq", hq * hd), ("wk", hkv * hd), ("wv", hkv * hd)):
            base = draw((rows, d), s.std, f"L{l}.{key}")
            lw[key] = base.to(dt)
            lw[key + "_diff"] = base.add_(draw((rows, d), s.sigma_diff, f"L{l}.{key}_diff_noise")).to(dt)
            del base
        lw["wo"] = draw((d, hq * hd), s.std, f"L{l}.wo").to(dt)
        lw["w_gate"] = draw((F, d), s.std, f"L{l}.w_gate").to(dt)
        lw["w_up"] = draw((F, d), s.std, f"L{l}.w_up").to(dt)
        lw["w_down"] = draw((d, F), s.std, f"L{l}.w_down").to(dt)
        layers.append(lw)
    return Weights(s, embed, ones, lm_head, layers)
