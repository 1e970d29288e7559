"""ctypes binding of libmk.so with the names of the C ABI in include/mk.h (marshalling only).

Every step of the decode path runs in the CUDA library; nothing here computes.
The library is loaded from this package's directory; if it is missing the
import fails (build it with ``python -m auto_regressive_decode_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_UNSUPPORTED = -2
MK_ERR_CUDA = -3
MK_ERR_DEVICE_TIMEOUT = -4
MK_ERR_RANGE = -5

MK_STATE_HIDDEN = 0
MK_STATE_ROUTER = 1
MK_STATE_SELECTION = 2
MK_STATE_SEL_WEIGHT = 3
MK_STATE_EXPERT_COUNT = 4
MK_STATE_TRACE = 5
MK_STATE_COUNTERS = 6

OP_NAMES = {0: "nop", 1: "embed", 2: "qkv", 3: "attn", 4: "oproj", 5: "gateup", 6: "down", 7: "lmhead",
            8: "router", 9: "exp_gateup", 10: "exp_down"}

_i32, _u64, _f32, _P = ctypes.c_int32, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p


class mk_model_desc(ctypes.Structure):
    _fields_ = [(n, _i32) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab",
                                    "n_experts", "top_k", "expert_ffn_dim", "qk_norm", "tied_embeddings")] + \
               [("rms_eps", _f32), ("rope_theta", _f32), ("batch", _i32), ("max_ctx", _i32),
                ("wait_timeout_ns", _u64)]


class mk_layer_weights(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm", "w_gate",
                                  "w_up", "w_down", "router")]


class mk_weights(ctypes.Structure):
    _fields_ = [("embed", _P), ("final_norm", _P), ("lm_head", _P), ("layers", ctypes.POINTER(mk_layer_weights))]


class mk_kv(ctypes.Structure):
    _fields_ = [("k", _P), ("v", _P), ("block_table", _P), ("page_size", _i32), ("n_pages", _i32)]


class mk_instr(ctypes.Structure):
    _fields_ = [(n, _i32) for n in ("op_layer", "wait_idx", "wait_count", "sig_idx", "a", "b", "c", "d")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmk.so not found at {LIB_PATH}; build it with `python -m auto_regressive_decode_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    H = _P
    sig = {
        "mk_create": (_i32, [ctypes.POINTER(mk_model_desc), ctypes.POINTER(mk_weights), ctypes.POINTER(mk_kv),
                             ctypes.POINTER(H)]),
        "mk_decode_step": (_i32, [H, _P, _P, _P, _P, _P]),
        "mk_decode_greedy": (_i32, [H, _i32, _P, _P, _P, _P, _P]),
        "mk_get_status": (_i32, [H, _P]),
        "mk_destroy": (_i32, [H]),
        "mk_status_string": (ctypes.c_char_p, [_i32]),
        "mk_read_state": (_i32, [H, _i32, _P, ctypes.c_size_t, _P]),
        "mk_state_bytes": (ctypes.c_size_t, [H, _i32]),
        "mk_decode_step_noalloc": (_i32, [ctypes.POINTER(mk_model_desc), ctypes.POINTER(mk_weights),
                                          ctypes.POINTER(mk_kv), _P, _P, _P, _P, _P]),
        "mk_plan_create": (_i32, [ctypes.POINTER(mk_model_desc), _i32, ctypes.POINTER(H)]),
        "mk_plan_n_sm": (_i32, [H]),
        "mk_plan_n_counters": (_i32, [H]),
        "mk_plan_n_instrs": (_i32, [H]),
        "mk_plan_copy": (_i32, [H, _P, _P]),
        "mk_plan_counter_targets": (_i32, [H, _P]),
        "mk_plan_attn_chunk": (_i32, [H, ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
        "mk_plan_attn_pieces": (_i32, [H, _P, _P, _i32, ctypes.POINTER(_i32)]),
        "mk_plan_destroy": (_i32, [H]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()

# Same names as the C ABI -----------------------------------------------------------------------
mk_create = lib.mk_create
mk_decode_step = lib.mk_decode_step
mk_decode_greedy = lib.mk_decode_greedy
mk_get_status = lib.mk_get_status
mk_destroy = lib.mk_destroy
mk_read_state = lib.mk_read_state
mk_state_bytes = lib.mk_state_bytes
mk_decode_step_noalloc = lib.mk_decode_step_noalloc
mk_plan_create = lib.mk_plan_create
mk_plan_n_sm = lib.mk_plan_n_sm
mk_plan_n_counters = lib.mk_plan_n_counters
mk_plan_n_instrs = lib.mk_plan_n_instrs
mk_plan_copy = lib.mk_plan_copy
mk_plan_counter_targets = lib.mk_plan_counter_targets
mk_plan_attn_chunk = lib.mk_plan_attn_chunk
mk_plan_attn_pieces = lib.mk_plan_attn_pieces
mk_plan_destroy = lib.mk_plan_destroy


def mk_status_string(code: int) -> str:
    return lib.mk_status_string(code).decode()


class MkError(RuntimeError):
    def __init__(self, code, what=""):
        super().__init__(f"{what}: {mk_status_string(code)} ({code})")
        self.code = code


def check(code, what=""):
    if code != MK_OK:
        raise MkError(code, what)
    return code


def model_desc(cfg, batch=None, max_ctx=None, wait_timeout_ns=0) -> mk_model_desc:
    """mk_model_desc of a model config (any object with the fixture config's field names)."""
    return mk_model_desc(cfg.n_layers, cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn_dim,
                         cfg.vocab, cfg.n_experts, cfg.top_k, cfg.expert_ffn_dim, int(cfg.qk_norm),
                         int(cfg.tied_embeddings), cfg.rms_eps, cfg.rope_theta,
                         cfg.batch if batch is None else batch, cfg.max_ctx if max_ctx is None else max_ctx,
                         wait_timeout_ns)


# ---- host-only lowering ------------------------------------------------------------------------

class Plan:
    """The per-SM instruction lists mk_create would build for n_sm SMs (no GPU needed)."""

    def __init__(self, desc: mk_model_desc, n_sm: int):
        import numpy as np
        h = _P()
        check(mk_plan_create(ctypes.byref(desc), n_sm, ctypes.byref(h)), "mk_plan_create")
        try:
            n = mk_plan_n_instrs(h)
            nc = mk_plan_n_counters(h)
            self.instrs = np.zeros((max(n, 1), 8), dtype=np.int32)[:n]
            self.offsets = np.zeros(n_sm + 1, dtype=np.int32)
            buf = np.zeros((max(n, 1), 8), dtype=np.int32)
            check(mk_plan_copy(h, buf.ctypes.data, self.offsets.ctypes.data), "mk_plan_copy")
            self.instrs = buf[:n]
            self.targets = np.zeros(nc, dtype=np.int32)
            check(mk_plan_counter_targets(h, self.targets.ctypes.data), "mk_plan_counter_targets")
            c, nch = _i32(), _i32()
            check(mk_plan_attn_chunk(h, ctypes.byref(c), ctypes.byref(nch)), "mk_plan_attn_chunk")
            self.chunk, self.n_chunks = c.value, nch.value
            self.n_sm = n_sm
        finally:
            mk_plan_destroy(h)
        self._desc = desc

    def attn_pieces(self, seq_lens):
        """int32[n][7] (slot, b, row, first unit, end unit, piece index in row, pieces of row) for one step."""
        import numpy as np
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        h = _P()
        check(mk_plan_create(ctypes.byref(self._desc), self.n_sm, ctypes.byref(h)), "mk_plan_create")
        try:
            n = _i32()
            mk_plan_attn_pieces(h, sl.ctypes.data, None, 0, ctypes.byref(n))
            out = np.zeros((max(n.value, 1), 7), dtype=np.int32)
            check(mk_plan_attn_pieces(h, sl.ctypes.data, out.ctypes.data, n.value, ctypes.byref(n)),
                  "mk_plan_attn_pieces")
            return out[:n.value]
        finally:
            mk_plan_destroy(h)

    def sm_list(self, s):
        return self.instrs[self.offsets[s]:self.offsets[s + 1]]

    @staticmethod
    def op(row):
        return int(row[0]) & 0xFF

    @staticmethod
    def layer(row):
        return int(row[0]) >> 8


# ---- device handle (torch tensors for memory and streams) ---------------------------------------

class Decoder:
    """Owns one mk_handle.  weights: dict of device tensors (see include/mk.h for shapes);
    k_cache / v_cache: device bf16 tensors [L][B][n_kv][max_ctx][hd]."""

    def __init__(self, cfg, weights, k_cache, v_cache, wait_timeout_ns=0, block_table=None, page_size=0):
        """block_table (device int32 [B][ceil(max_ctx/page_size)]) with page_size: k_cache / v_cache are
        page pools [L][n_pages][n_kv][page_size][hd]."""
        import torch
        self.cfg = cfg
        self._keep = (weights, k_cache, v_cache, block_table)
        self.desc = model_desc(cfg, wait_timeout_ns=wait_timeout_ns)
        L = cfg.n_layers
        layers = (mk_layer_weights * L)()

        def ptr(t):
            return None if t is None else t.data_ptr()
        for l in range(L):
            lw = weights["layers"][l]
            for name, _ in mk_layer_weights._fields_:
                setattr(layers[l], name, ptr(lw.get(name)))
        self._layers = layers
        w = mk_weights(ptr(weights["embed"]), ptr(weights["final_norm"]), ptr(weights.get("lm_head")), layers)
        if block_table is None:
            kv = mk_kv(k_cache.data_ptr(), v_cache.data_ptr(), None, 0, 0)
        else:
            kv = mk_kv(k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(), page_size, k_cache.shape[1])
        h = _P()
        check(mk_create(ctypes.byref(self.desc), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(h)), "mk_create")
        self.h = h
        self.torch = torch

    def step(self, tokens, positions, seq_lens, logits, stream=None):
        """Asynchronous decode step; all arguments are device tensors (int32, int32, int32, float32)."""
        s = (stream or self.torch.cuda.current_stream()).cuda_stream
        check(mk_decode_step(self.h, tokens.data_ptr(), positions.data_ptr(), seq_lens.data_ptr(), s,
                             logits.data_ptr()), "mk_decode_step")

    def greedy(self, n_steps, tokens, seq_lens, out_tokens, logits=None, stream=None):
        """n_steps greedy steps on the device (asynchronous); out_tokens int32 [n_steps][B] device tensor."""
        s = (stream or self.torch.cuda.current_stream()).cuda_stream
        check(mk_decode_greedy(self.h, n_steps, tokens.data_ptr(), seq_lens.data_ptr(), s, out_tokens.data_ptr(),
                               None if logits is None else logits.data_ptr()), "mk_decode_greedy")

    def status(self, stream=None):
        s = (stream or self.torch.cuda.current_stream()).cuda_stream
        return mk_get_status(self.h, s)

    def read_state(self, which, dst, stream=None):
        s = (stream or self.torch.cuda.current_stream()).cuda_stream
        check(mk_read_state(self.h, which, dst.data_ptr(), dst.numel() * dst.element_size(), s), "mk_read_state")
        return dst

    def hidden_states(self):
        """float32 [2L+1][B][H] residual stream of the last step."""
        c = self.cfg
        out = self.torch.empty((2 * c.n_layers + 1, c.batch, c.hidden), dtype=self.torch.float32, device="cuda")
        return self.read_state(MK_STATE_HIDDEN, out)

    def routing(self):
        """MoE routing of the last step (host numpy): router logits float32 [L][B][E], picks int32
        [L][B][k] (best first), their weights float32 [L][B][k], distinct experts int32 [L]."""
        c, torch = self.cfg, self.torch
        L, B, E, K = c.n_layers, c.batch, c.n_experts, c.top_k
        r = self.read_state(MK_STATE_ROUTER, torch.empty((L, B, E), dtype=torch.float32, device="cuda"))
        sel = self.read_state(MK_STATE_SELECTION, torch.empty((L, B, K), dtype=torch.int32, device="cuda"))
        w = self.read_state(MK_STATE_SEL_WEIGHT, torch.empty((L, B, K), dtype=torch.float32, device="cuda"))
        n = self.read_state(MK_STATE_EXPERT_COUNT, torch.empty((L,), dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        return r.cpu().numpy(), sel.cpu().numpy(), w.cpu().numpy(), n.cpu().numpy()

    def counters(self):
        """uint32 dependency counters after the last step (host numpy), in mk_plan_counter_targets order."""
        import numpy as np
        n = mk_state_bytes(self.h, MK_STATE_COUNTERS) // 4
        c = self.read_state(MK_STATE_COUNTERS, self.torch.empty((n,), dtype=self.torch.int32, device="cuda"))
        self.torch.cuda.synchronize()
        return c.cpu().numpy().view(np.uint32)

    def close(self):
        if getattr(self, "h", None):
            mk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def weight_structs(cfg, weights, k_cache, v_cache):
    """(mk_model_desc, mk_weights, mk_kv, keep-alive) for a stateless call such as mk_decode_step_noalloc."""
    L = cfg.n_layers
    layers = (mk_layer_weights * L)()
    for l in range(L):
        lw = weights["layers"][l]
        for name, _ in mk_layer_weights._fields_:
            t = lw.get(name)
            setattr(layers[l], name, None if t is None else t.data_ptr())
    lm = weights.get("lm_head")
    w = mk_weights(weights["embed"].data_ptr(), weights["final_norm"].data_ptr(),
                   None if lm is None else lm.data_ptr(), layers)
    kv = mk_kv(k_cache.data_ptr(), v_cache.data_ptr(), None, 0, 0)
    return model_desc(cfg), w, kv, (layers, weights, k_cache, v_cache)


def decoder_trace(dec):
    """int64 [n_instr][8] timestamps of the last step (handle created with MK_TRACE=1)."""
    import torch
    n = mk_state_bytes(dec.h, MK_STATE_TRACE)
    if n == 0:
        raise MkError(MK_ERR_INVALID_ARG, "handle was not created with MK_TRACE=1")
    out = torch.empty(n // 8, dtype=torch.int64, device="cuda")
    dec.read_state(MK_STATE_TRACE, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(-1, 8)
