"""Shared test helpers: materialise seeded host models and compare mid-states."""
from __future__ import annotations

import numpy as np

import fixtures as fx


def host_model(cfg, seed=fx.DEFAULT_SEED, gains="ones", layers=None):
    """Host bf16 weights of cfg: (globals dict, [per-layer dict or None]).

    layers: iterable of layer indices to materialise (default all).
    """
    g = {k: fx.materialize(s, seed) for k, s in fx.global_specs(cfg, gains).items()}
    if cfg.tied_embeddings:
        g["lm_head"] = None
    want = range(cfg.n_layers) if layers is None else set(layers)
    ls = []
    for l in range(cfg.n_layers):
        if l in want:
            ls.append({k: fx.materialize(s, seed) for k, s in fx.layer_specs(cfg, l, gains).items()})
        else:
            ls.append(None)
    return g, ls


def expert_loader(cfg, seed=fx.DEFAULT_SEED):
    def load(layer, e):
        return {k: fx.materialize(s, seed) for k, s in fx.expert_specs(cfg, layer, e).items()}
    return load


def host_caches(cfg, seq_lens, seed=fx.DEFAULT_SEED, poison=False, layers=None):
    """Model caches [L][B][nkv][T][hd] (bf16 bits) prefilled from the generator."""
    L = cfg.n_layers
    shape = (L, cfg.batch, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim)
    kc = np.zeros(shape, dtype=np.uint16)
    vc = np.zeros(shape, dtype=np.uint16)
    for l in (range(L) if layers is None else layers):
        kc[l] = fx.kv_prefill(cfg, l, 0, seq_lens, seed, poison)
        vc[l] = fx.kv_prefill(cfg, l, 1, seq_lens, seed, poison)
    return kc, vc


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def bf16_f64(a):
    return fx.bf16_to_f32(np.asarray(a, dtype=np.uint16)).astype(np.float64)
