"""Materialise a config's seeded inputs as CUDA tensors (torch is used for device memory only).

Values are generated on the host by the same counter-based generator as for the
oracle (chunk by chunk, through a pinned buffer) and copied to the device, so
both sides see bit-identical weights, caches and tokens.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (BF16_NAN, DEFAULT_SEED, K_CACHE, V_CACHE, _load, context_lengths, expert_specs, global_specs,
               layer_specs, normal_bf16, tid)

_CHUNK = 1 << 25  # elements per host chunk (64 MB of bf16)


class _Staging:
    def __init__(self, n=_CHUNK):
        self.host = torch.empty(n, dtype=torch.int16, pin_memory=True)
        self.np = self.host.numpy().view(np.uint16)


def _fill(dst: torch.Tensor, spec, seed, stg: _Staging, row0=0):
    """dst: contiguous device bf16 tensor receiving spec's values (rows from row0)."""
    flat = dst.view(torch.int16).view(-1)
    n = flat.numel()
    inner = spec.numel // spec.shape[0]
    base = row0 * inner
    done = 0
    while done < n:
        m = min(_CHUNK, n - done)
        buf = stg.np[:m]
        if spec.sigma is None:
            _load().fx_fill_u16(0x3F80, m, buf.ctypes.data)
        else:
            normal_bf16(seed, spec.tensor_id, m, spec.sigma, offset=base + done, out=buf)
        flat[done:done + m].copy_(stg.host[:m], non_blocking=False)
        done += m


def _alloc_filled(spec, seed, stg, device):
    t = torch.empty(spec.shape, dtype=torch.bfloat16, device=device)
    _fill(t, spec, seed, stg)
    return t


def device_model(cfg, seed=DEFAULT_SEED, gains="ones", device="cuda"):
    """{'embed','final_norm','lm_head'(None if tied),'layers':[{name: tensor}]} on the device."""
    stg = _Staging()
    out = {k: _alloc_filled(s, seed, stg, device) for k, s in global_specs(cfg, gains).items()}
    out.setdefault("lm_head", None)
    layers = []
    for l in range(cfg.n_layers):
        lw = {k: _alloc_filled(s, seed, stg, device) for k, s in layer_specs(cfg, l, gains).items()}
        if cfg.n_experts:
            E, Ie, H = cfg.n_experts, cfg.expert_ffn_dim, cfg.hidden
            lw["w_gate"] = torch.empty((E, Ie, H), dtype=torch.bfloat16, device=device)
            lw["w_up"] = torch.empty((E, Ie, H), dtype=torch.bfloat16, device=device)
            lw["w_down"] = torch.empty((E, H, Ie), dtype=torch.bfloat16, device=device)
            for e in range(E):
                es = expert_specs(cfg, l, e)
                for k in ("w_gate", "w_up", "w_down"):
                    _fill(lw[k][e], es[k], seed, stg)
        layers.append(lw)
    out["layers"] = layers
    return out


def device_caches(cfg, seq_lens=None, seed=DEFAULT_SEED, poison=False, device="cuda"):
    """(k, v) bf16 caches [L][B][n_kv][max_ctx][hd]; positions >= seq_lens[b] hold 0 (or NaN if poison)."""
    if seq_lens is None:
        seq_lens = context_lengths(cfg, seed)
    L, B, nkv, T, hd = cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim
    fill = np.int16(np.uint16(BF16_NAN).view(np.int16)) if poison else 0
    stg = _Staging()
    caches = []
    for role in (K_CACHE, V_CACHE):
        c = torch.full((L, B, nkv, T, hd), int(fill), dtype=torch.int16, device=device)
        for l in range(L):
            t = tid(role, l)
            for b in range(B):
                S = int(seq_lens[b])
                if S == 0:
                    continue
                for h in range(nkv):
                    n = S * hd
                    buf = stg.np[:n]
                    normal_bf16(seed, t, n, cfg.kv_sigma, offset=((b * nkv + h) * T) * hd, out=buf)
                    c[l, b, h, :S].view(-1).copy_(stg.host[:n])
        caches.append(c.view(torch.bfloat16))
    return caches[0], caches[1]
