"""Python binding of the CPU oracle (``oracle.c``): marshalling only.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the GPU path.

The oracle is the mid-state test oracle of ForgeMegakernel (arXiv 2609.12379,
abstract): fp64 arithmetic over bf16-stored weights and KV cache, dumping
every layer's hidden states, the appended K/V rows, MoE routing and logits.

Parity status of each oracle function (what pins it, in ``tests/test_oracle_pins.py``):
every primitive and the whole-model step are pinned by closed forms,
invariants, library routines and brute force; the end-to-end numbers are
pinned only through those, because the pages print no worked example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double


class _Desc(ctypes.Structure):
    _fields_ = [(n, _I) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab",
                                  "n_experts", "top_k", "expert_ffn_dim", "qk_norm", "batch", "max_ctx")] + \
               [("rms_eps", _D), ("rope_theta", _D), ("fp8_block", _I)]


FP8_MATRICES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")  # in ora_layer's order of fp8 forms


class _Layer(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm", "w_gate",
                                  "w_up", "w_down", "router")] + \
               [(f"{n}_fp8_{part}", _P) for n in FP8_MATRICES for part in ("codes", "scale")]


_EXPERT_FN = ctypes.CFUNCTYPE(_P, _P, _I, _I, _I)


class _Model(ctypes.Structure):
    _fields_ = [("d", _Desc), ("embed", _P), ("final_norm", _P), ("lm_head", _P), ("layers", ctypes.POINTER(_Layer)),
                ("expert", _EXPERT_FN), ("expert_ctx", _P)]


def build(force: bool = False, extra_flags=()) -> str:
    """Compile liboracle.so (gcc, -O2, no fast-math, no FMA contraction)."""
    src = os.path.join(_HERE, "oracle.c")
    hdr = os.path.join(_HERE, "oracle.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", *extra_flags,
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def build_variant(path: str, defines=()) -> ctypes.CDLL:
    """Compile a separate copy of the oracle with extra -D flags (used by tests that plant mistakes)."""
    src = os.path.join(_HERE, "oracle.c")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           *[f"-D{d}" for d in defines], "-o", path, src, "-lm"])
    return _setup(ctypes.CDLL(path))


def _setup(lib):
    u16p = _P
    lib.ora_bf16_to_double.restype = _D
    lib.ora_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.ora_double_to_bf16.restype = ctypes.c_uint16
    lib.ora_double_to_bf16.argtypes = [_D]
    lib.ora_rmsnorm.argtypes = [_P, _I, u16p, _D, _P]
    lib.ora_rope.argtypes = [_P, _I, _I, _D]
    lib.ora_gemv.argtypes = [u16p, _I, _I, _P, _P]
    lib.ora_silu.restype = _D
    lib.ora_silu.argtypes = [_D]
    lib.ora_attention.argtypes = [_P, u16p, u16p, _I, _I, _P, _P]
    lib.ora_swiglu.argtypes = [u16p, u16p, u16p, _I, _I, _P, _P]
    lib.ora_topk.argtypes = [_P, _I, _I, _P, _P]
    lib.ora_layer_forward.restype = _I
    lib.ora_layer_forward.argtypes = [ctypes.POINTER(_Model), _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.ora_decode_step.restype = _I
    lib.ora_decode_step.argtypes = [ctypes.POINTER(_Model), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.ora_lm_head.argtypes = [ctypes.POINTER(_Model), _P, _P]
    lib.ora_e4m3_to_double.restype = _D
    lib.ora_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.ora_e2m1_to_double.restype = _D
    lib.ora_e2m1_to_double.argtypes = [ctypes.c_uint8]
    lib.ora_gemv_fp8.argtypes = [_P, _P, _I, _I, _I, _P, _P]
    lib.ora_gemv_nvfp4.argtypes = [_P, _P, ctypes.c_float, _I, _I, _P, _P]
    for f in ("ora_rmsnorm", "ora_rope", "ora_gemv", "ora_attention", "ora_swiglu", "ora_topk", "ora_lm_head",
              "ora_gemv_fp8", "ora_gemv_nvfp4"):
        getattr(lib, f).restype = None
    return lib


def lib():
    global _lib
    if _lib is None:
        _lib = _setup(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---- primitives --------------------------------------------------------------------------------

def bf16_to_double(h: int, L=None) -> float:
    return (L or lib()).ora_bf16_to_double(int(h))


def double_to_bf16(x: float, L=None) -> int:
    return int((L or lib()).ora_double_to_bf16(float(x)))


def rmsnorm(x, gain, eps, L=None):
    x = _f64(x); gain = _u16(gain)
    out = np.empty_like(x)
    (L or lib()).ora_rmsnorm(_ptr(x), x.size, _ptr(gain), eps, _ptr(out))
    return out


def rope(v, pos, theta, L=None):
    v = _f64(v).copy()
    (L or lib()).ora_rope(_ptr(v), v.size, int(pos), float(theta))
    return v


def gemv(w, x, L=None):
    w = _u16(w); x = _f64(x)
    y = np.empty(w.shape[0], dtype=np.float64)
    (L or lib()).ora_gemv(_ptr(w), w.shape[0], w.shape[1], _ptr(x), _ptr(y))
    return y


def e4m3_to_double(code: int, L=None) -> float:
    return (L or lib()).ora_e4m3_to_double(int(code))


def e2m1_to_double(nibble: int, L=None) -> float:
    return (L or lib()).ora_e2m1_to_double(int(nibble))


def gemv_fp8(w, scale, block, x, L=None):
    """w uint8 [rows][cols] E4M3 codes, scale fp32 [rows][ceil(cols / block)] -> y [rows]."""
    w = np.ascontiguousarray(w, dtype=np.uint8); scale = np.ascontiguousarray(scale, dtype=np.float32)
    x = _f64(x)
    y = np.empty(w.shape[0], dtype=np.float64)
    (L or lib()).ora_gemv_fp8(_ptr(w), _ptr(scale), w.shape[0], w.shape[1], int(block), _ptr(x), _ptr(y))
    return y


def gemv_nvfp4(w, scale, tensor_scale, x, L=None):
    """w uint8 [rows][cols / 2] E2M1 pairs, scale uint8 [rows][cols / 16] E4M3 -> y [rows]."""
    w = np.ascontiguousarray(w, dtype=np.uint8); scale = np.ascontiguousarray(scale, dtype=np.uint8)
    x = _f64(x)
    rows, cols = w.shape[0], 2 * w.shape[1]
    y = np.empty(rows, dtype=np.float64)
    (L or lib()).ora_gemv_nvfp4(_ptr(w), _ptr(scale), float(tensor_scale), rows, cols, _ptr(x), _ptr(y))
    return y


def silu(z, L=None):
    return (L or lib()).ora_silu(float(z))


def attention(q, k, v, L=None):
    """q [d] float; k, v [n][d] bf16 bits -> (out [d], probs [n])."""
    q = _f64(q); k = _u16(k); v = _u16(v)
    n, d = k.shape
    out = np.empty(d, dtype=np.float64)
    probs = np.empty(max(n, 1), dtype=np.float64)
    (L or lib()).ora_attention(_ptr(q), _ptr(k), _ptr(v), n, d, _ptr(out), _ptr(probs))
    return out, probs[:n]


def swiglu(wg, wu, wd, xn, L=None):
    wg, wu, wd = _u16(wg), _u16(wu), _u16(wd); xn = _f64(xn)
    ffn, hidden = wg.shape
    y = np.empty(hidden, dtype=np.float64)
    (L or lib()).ora_swiglu(_ptr(wg), _ptr(wu), _ptr(wd), ffn, hidden, _ptr(xn), _ptr(y))
    return y


def topk(logits, k, L=None):
    logits = _f64(logits)
    sel = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    (L or lib()).ora_topk(_ptr(logits), logits.size, k, _ptr(sel), _ptr(w))
    return sel, w


# ---- model ---------------------------------------------------------------------------------------

class Model:
    """Host weights of one model (bf16 bit patterns as numpy uint16) bound for the oracle.

    layers: list of dicts with keys attn_norm, wq, wk, wv, wo, mlp_norm and either w_gate, w_up,
    w_down (dense) or router (MoE), plus q_norm, k_norm when qk_norm.  expert_fn(layer, e) returns a
    dict with w_gate, w_up, w_down for MoE configs.
    """

    def __init__(self, cfg, embed, final_norm, lm_head, layers, expert_fn=None, L=None, fp8_block=0):
        if fp8_block and cfg.n_experts:
            raise ValueError("fp8 weights are modelled for the attention projections and the dense MLP only, "
                             "not for a mixture-of-experts model")
        self.cfg = cfg
        self.L = L or lib()
        self._keep = [embed, final_norm, lm_head]
        self._layers = (_Layer * cfg.n_layers)()
        for i, lw in enumerate(layers):
            if lw is None:
                continue
            for name in _Layer._fields_:
                if "_fp8_" in name[0]:
                    continue
                a = lw.get(name[0])
                if a is not None:
                    a = _u16(a)
                    self._keep.append(a)
                    setattr(self._layers[i], name[0], a.ctypes.data)
            if fp8_block:  # fp8 forms: lw[name + "_fp8"] = (E4M3 codes uint8 [out][in], fp32 scales)
                for n in FP8_MATRICES:
                    codes, scale = lw[n + "_fp8"]
                    codes = np.ascontiguousarray(codes, dtype=np.uint8)
                    scale = np.ascontiguousarray(scale, dtype=np.float32)
                    self._keep += [codes, scale]
                    setattr(self._layers[i], n + "_fp8_codes", codes.ctypes.data)
                    setattr(self._layers[i], n + "_fp8_scale", scale.ctypes.data)
        self._expert_fn = expert_fn
        self._expert_cache = {}
        self._cb = _EXPERT_FN(self._expert)
        d = _Desc(cfg.n_layers, cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn_dim, cfg.vocab,
                  cfg.n_experts, cfg.top_k, cfg.expert_ffn_dim, int(cfg.qk_norm), cfg.batch, cfg.max_ctx,
                  cfg.rms_eps, cfg.rope_theta, int(fp8_block))
        lm = embed if lm_head is None else lm_head
        self.m = _Model(d, embed.ctypes.data, final_norm.ctypes.data, lm.ctypes.data, self._layers, self._cb, None)

    def _expert(self, ctx, layer, e, which):
        key = (layer, e)
        if key not in self._expert_cache:
            w = self._expert_fn(layer, e)
            self._expert_cache[key] = [_u16(w["w_gate"]), _u16(w["w_up"]), _u16(w["w_down"])]
        return self._expert_cache[key][which].ctypes.data

    def clear_expert_cache(self):
        self._expert_cache.clear()

    def decode_step(self, k_cache, v_cache, tokens, positions, seq_lens):
        """One step; mutates k_cache/v_cache ([L][B][nkv][T][hd] uint16).  Returns the dumps."""
        c = self.cfg
        B, H, L = c.batch, c.hidden, c.n_layers
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        pos = np.ascontiguousarray(positions, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
        out = {"h_attn": np.empty((L, B, H)), "h_mlp": np.empty((L, B, H)), "logits": np.empty((B, c.vocab))}
        if c.n_experts:
            out["router_logits"] = np.empty((L, B, c.n_experts))
            out["sel"] = np.empty((L, B, c.top_k), dtype=np.int32)
            out["sel_w"] = np.empty((L, B, c.top_k))
        rc = self.L.ora_decode_step(ctypes.byref(self.m), k_cache.ctypes.data, v_cache.ctypes.data, _ptr(tok),
                                    _ptr(pos), _ptr(sl), _ptr(out["h_attn"]), _ptr(out["h_mlp"]),
                                    _ptr(out.get("router_logits")), _ptr(out.get("sel")), _ptr(out.get("sel_w")),
                                    _ptr(out["logits"]))
        if rc != 0:
            raise ValueError(f"oracle decode step failed ({rc})")
        return out

    def layer_forward(self, layer, x, k_cache_layer, v_cache_layer, positions, seq_lens):
        """One layer on residual x [B][H] (float64, updated in place); caches of this layer."""
        c = self.cfg
        x = np.ascontiguousarray(x, dtype=np.float64)
        pos = np.ascontiguousarray(positions, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        out = {"h_attn": np.empty((c.batch, c.hidden))}
        if c.n_experts:
            out["router_logits"] = np.empty((c.batch, c.n_experts))
            out["sel"] = np.empty((c.batch, c.top_k), dtype=np.int32)
            out["sel_w"] = np.empty((c.batch, c.top_k))
        rc = self.L.ora_layer_forward(ctypes.byref(self.m), layer, _ptr(x), k_cache_layer.ctypes.data,
                                      v_cache_layer.ctypes.data, _ptr(pos), _ptr(sl), _ptr(out["h_attn"]),
                                      _ptr(out.get("router_logits")), _ptr(out.get("sel")), _ptr(out.get("sel_w")))
        if rc != 0:
            raise ValueError(f"oracle layer forward failed ({rc})")
        out["h_mlp"] = x
        return out

    def lm_head(self, x_row):
        x_row = _f64(x_row)
        logits = np.empty(self.cfg.vocab)
        self.L.ora_lm_head(ctypes.byref(self.m), _ptr(x_row), _ptr(logits))
        return logits
