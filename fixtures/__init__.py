"""Seeded synthetic inputs for the decode step (shared by the oracle's tests and the GPU path).

This module constructs inputs only: weight matrices, prefilled KV caches, token
ids and context lengths, all regenerated bit-identically from (seed, tensor id,
element index) by the counter-based generator in ``fx.c``.  It contains none of
the decode step's arithmetic.

Tensor ids::

    tid = (slot << 40) | (role << 32) | expert

``slot`` is 0 for model-global tensors and ``layer + 1`` for per-layer ones;
``expert`` is ``e + 1`` for the tensors of MoE expert ``e`` and 0 otherwise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .configs import CONFIGS, ModelConfig  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfx.so")
_lib = None

# roles
EMBED, FINAL_NORM, LM_HEAD = 0, 1, 2
ATTN_NORM, WQ, WK, WV, Q_NORM, K_NORM, WO, MLP_NORM, W_GATE, W_UP, W_DOWN, ROUTER = range(10, 22)
K_CACHE, V_CACHE = 30, 31
TOKENS, SEQ_LENS = 40, 41

BF16_ONE = 0x3F80
DEFAULT_SEED = 0


def build(force: bool = False) -> str:
    """Compile libfx.so next to this file (gcc, OpenMP, no fast-math)."""
    src = os.path.join(_HERE, "fx.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-o", tmp, src,
                               "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, f64 = ctypes.c_uint64, ctypes.c_double
        lib.fx_splitmix64.restype = u64
        lib.fx_splitmix64.argtypes = [u64]
        lib.fx_normal_bf16.restype = None
        lib.fx_normal_bf16.argtypes = [u64, u64, u64, u64, f64, ctypes.c_void_p]
        lib.fx_uniform_int.restype = None
        lib.fx_uniform_int.argtypes = [u64, u64, u64, u64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.fx_fill_u16.restype = None
        lib.fx_fill_u16.argtypes = [ctypes.c_uint16, u64, ctypes.c_void_p]
        _lib = lib
    return _lib


def tid(role: int, layer: int = -1, expert: int = -1) -> int:
    return ((layer + 1) << 40) | (role << 32) | (expert + 1)


def splitmix64(z: int) -> int:
    return int(_load().fx_splitmix64(z & 0xFFFFFFFFFFFFFFFF))


def normal_bf16(seed: int, tensor_id: int, n: int, sigma: float, offset: int = 0, out=None) -> np.ndarray:
    """bf16 bit patterns (uint16) of sigma * N(0,1)-shaped draws for elements [offset, offset+n)."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _load().fx_normal_bf16(seed, tensor_id, offset, n, sigma, out.ctypes.data)
    return out


def uniform_ints(seed: int, tensor_id: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    """Uniform integers in [lo, hi] (inclusive) as int32."""
    out = np.empty(n, dtype=np.int32)
    _load().fx_uniform_int(seed, tensor_id, offset, n, lo, hi, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------------------------
# Model recipe: every tensor of a config with its shape and how it is drawn.
# --------------------------------------------------------------------------------------------


class TensorSpec:
    """One model tensor: where it lives, its shape, and how its values are drawn."""

    __slots__ = ("name", "layer", "role", "expert", "shape", "sigma")

    def __init__(self, name, layer, role, expert, shape, sigma):
        self.name, self.layer, self.role, self.expert = name, layer, role, expert
        self.shape, self.sigma = tuple(shape), sigma   # sigma None -> constant bf16 1.0

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n

    @property
    def tensor_id(self) -> int:
        return tid(self.role, self.layer, self.expert)

    def __repr__(self):
        return f"TensorSpec({self.name}, layer={self.layer}, shape={self.shape})"


def layer_specs(cfg: ModelConfig, layer: int, gains: str = "ones"):
    """Specs of one layer's tensors, keyed by name.

    gains: "ones" (all configs) or "random" (tests: N(0,1)-shaped gains exercise the multiply).
    """
    H, hd, s = cfg.hidden, cfg.head_dim, cfg.weight_sigma
    g = None if gains == "ones" else 1.0
    d = {
        "attn_norm": TensorSpec("attn_norm", layer, ATTN_NORM, -1, (H,), g),
        "wq": TensorSpec("wq", layer, WQ, -1, (cfg.q_dim, H), s),
        "wk": TensorSpec("wk", layer, WK, -1, (cfg.kv_dim, H), s),
        "wv": TensorSpec("wv", layer, WV, -1, (cfg.kv_dim, H), s),
        "wo": TensorSpec("wo", layer, WO, -1, (H, cfg.q_dim), s),
        "mlp_norm": TensorSpec("mlp_norm", layer, MLP_NORM, -1, (H,), g),
    }
    if cfg.qk_norm:
        d["q_norm"] = TensorSpec("q_norm", layer, Q_NORM, -1, (hd,), g)
        d["k_norm"] = TensorSpec("k_norm", layer, K_NORM, -1, (hd,), g)
    if cfg.n_experts:
        E, Ie = cfg.n_experts, cfg.expert_ffn_dim
        d["router"] = TensorSpec("router", layer, ROUTER, -1, (E, H), s)
    else:
        I = cfg.ffn_dim
        d["w_gate"] = TensorSpec("w_gate", layer, W_GATE, -1, (I, H), s)
        d["w_up"] = TensorSpec("w_up", layer, W_UP, -1, (I, H), s)
        d["w_down"] = TensorSpec("w_down", layer, W_DOWN, -1, (H, I), s)
    return d


def expert_specs(cfg: ModelConfig, layer: int, expert: int):
    """Specs of one MoE expert's SwiGLU weights (gate, up: [Ie][H]; down: [H][Ie])."""
    H, Ie, s = cfg.hidden, cfg.expert_ffn_dim, cfg.weight_sigma
    return {
        "w_gate": TensorSpec("w_gate", layer, W_GATE, expert, (Ie, H), s),
        "w_up": TensorSpec("w_up", layer, W_UP, expert, (Ie, H), s),
        "w_down": TensorSpec("w_down", layer, W_DOWN, expert, (H, Ie), s),
    }


def global_specs(cfg: ModelConfig, gains: str = "ones"):
    H, V, s = cfg.hidden, cfg.vocab, cfg.weight_sigma
    g = None if gains == "ones" else 1.0
    d = {
        "embed": TensorSpec("embed", -1, EMBED, -1, (V, H), s),
        "final_norm": TensorSpec("final_norm", -1, FINAL_NORM, -1, (H,), g),
    }
    if not cfg.tied_embeddings:
        d["lm_head"] = TensorSpec("lm_head", -1, LM_HEAD, -1, (V, H), s)
    return d


def materialize(spec: TensorSpec, seed: int = DEFAULT_SEED, row0: int = 0, rows: int | None = None) -> np.ndarray:
    """Host bf16 bit patterns of spec (or of rows [row0, row0+rows) of its leading dim)."""
    shape = list(spec.shape)
    inner = spec.numel // shape[0]
    if rows is None:
        rows = shape[0] - row0
    shape[0] = rows
    n = rows * inner
    out = np.empty(n, dtype=np.uint16)
    if spec.sigma is None:
        _load().fx_fill_u16(BF16_ONE, n, out.ctypes.data)
    else:
        normal_bf16(seed, spec.tensor_id, n, spec.sigma, offset=row0 * inner, out=out)
    return out.reshape(shape)


def context_lengths(cfg: ModelConfig, seed: int = DEFAULT_SEED) -> np.ndarray:
    """Prefilled tokens per sequence before the first decode step (int32[B])."""
    if cfg.ragged:
        return uniform_ints(seed, tid(SEQ_LENS), cfg.batch, cfg.ctx_lo, cfg.ctx_hi)
    return np.full(cfg.batch, cfg.ctx, dtype=np.int32)


def tokens(cfg: ModelConfig, seed: int = DEFAULT_SEED) -> np.ndarray:
    """Teacher-forced token ids, int32[steps][B], uniform over the vocabulary."""
    return uniform_ints(seed, tid(TOKENS), cfg.steps * cfg.batch, 0, cfg.vocab - 1).reshape(cfg.steps, cfg.batch)


BF16_NAN = 0x7FC0


def kv_prefill(cfg: ModelConfig, layer: int, which: int, seq_lens, seed: int = DEFAULT_SEED,
               poison: bool = False) -> np.ndarray:
    """Prefilled cache of one layer, bf16 bits [B][n_kv][max_ctx][hd].

    Positions p < seq_lens[b] hold kv_sigma * N(0,1)-shaped draws at generator index
    ((b*n_kv + h)*max_ctx + p)*hd + d; later positions hold 0, or NaN when poison is set
    (so that a read past the valid range shows up).
    """
    B, nkv, T, hd = cfg.batch, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim
    out = np.full((B, nkv, T, hd), BF16_NAN if poison else 0, dtype=np.uint16)
    t = tid(K_CACHE if which == 0 else V_CACHE, layer)
    for b in range(B):
        S = int(seq_lens[b])
        for h in range(nkv):
            if S:
                normal_bf16(seed, t, S * hd, cfg.kv_sigma, offset=((b * nkv + h) * T) * hd,
                            out=out[b, h, :S].reshape(-1))
    return out
