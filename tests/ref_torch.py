"""A second, independent fp64 reference of the decode step, written with PyTorch library routines.

It exists only to pin the C oracle: it shares no code with it and is built
from different primitives (torch.nn.functional.rms_norm, scaled_dot_product_attention,
silu, torch.topk / softmax, complex-number RoPE via torch.polar).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F


def w64(a):
    """bf16 bit patterns (uint16 numpy) -> float64 torch tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64)


def to_bf16_bits(x64: torch.Tensor) -> np.ndarray:
    return x64.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def rope_complex(x: torch.Tensor, pos: int, theta: float) -> torch.Tensor:
    """Rotate-half RoPE written as a complex multiply: z_i = x_i + i x_{i+d/2}, z_i *= e^{i pos w_i}."""
    d = x.shape[-1]
    half = d // 2
    w = theta ** (-torch.arange(half, dtype=torch.float64) * 2.0 / d)
    rot = torch.polar(torch.ones(half, dtype=torch.float64), pos * w)
    z = torch.complex(x[..., :half], x[..., half:]) * rot
    return torch.cat([z.real, z.imag], dim=-1)


def decode_step(cfg, g, layers, kc, vc, tokens, positions, seq_lens, expert_fn=None):
    """Returns dumps like the oracle; kc/vc (numpy uint16 [L][B][nkv][T][hd]) are updated in place."""
    B, H, L = cfg.batch, cfg.hidden, cfg.n_layers
    nq, nkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    emb = w64(g["embed"])
    x = emb[torch.as_tensor(np.asarray(tokens, dtype=np.int64))].clone()      # [B][H]
    h_attn, h_mlp, rl, sels, sws = [], [], [], [], []
    for l in range(L):
        W = layers[l]
        xn = F.rms_norm(x, (H,), w64(W["attn_norm"]), eps=cfg.rms_eps)
        q = F.linear(xn, w64(W["wq"])).view(B, nq, hd)
        k = F.linear(xn, w64(W["wk"])).view(B, nkv, hd)
        v = F.linear(xn, w64(W["wv"])).view(B, nkv, hd)
        if cfg.qk_norm:
            q = F.rms_norm(q, (hd,), w64(W["q_norm"]), eps=cfg.rms_eps)
            k = F.rms_norm(k, (hd,), w64(W["k_norm"]), eps=cfg.rms_eps)
        att = torch.empty(B, nq, hd, dtype=torch.float64)
        for b in range(B):
            S, p = int(seq_lens[b]), int(positions[b])
            qb = rope_complex(q[b], p, cfg.rope_theta)
            kb = rope_complex(k[b], p, cfg.rope_theta)
            kc[l, b, :, S] = to_bf16_bits(kb)
            vc[l, b, :, S] = to_bf16_bits(v[b])
            K = w64(kc[l, b, :, : S + 1])            # [nkv][S+1][hd]
            V = w64(vc[l, b, :, : S + 1])
            o = F.scaled_dot_product_attention(qb[:, None, :], K, V, enable_gqa=True)   # [nq][1][hd]
            att[b] = o[:, 0]
        x = x + F.linear(att.reshape(B, nq * hd), w64(W["wo"]))
        h_attn.append(x.clone())
        xn = F.rms_norm(x, (H,), w64(W["mlp_norm"]), eps=cfg.rms_eps)
        if not cfg.n_experts:
            y = F.linear(F.silu(F.linear(xn, w64(W["w_gate"]))) * F.linear(xn, w64(W["w_up"])), w64(W["w_down"]))
        else:
            r = F.linear(xn, w64(W["router"]))                       # [B][E]
            rl.append(r.clone())
            y = torch.zeros(B, H, dtype=torch.float64)
            sel_l, sw_l = [], []
            for b in range(B):
                # stable descending sort keeps the lower index first among equal logits
                order = torch.sort(r[b], descending=True, stable=True).indices[: cfg.top_k]
                p = torch.softmax(r[b], dim=0)[order]
                p = p / p.sum()
                sel_l.append(order.numpy().astype(np.int32))
                sw_l.append(p.numpy())
                for j, e in enumerate(order.tolist()):
                    ew = expert_fn(l, e)
                    ye = F.linear(F.silu(F.linear(xn[b], w64(ew["w_gate"]))) * F.linear(xn[b], w64(ew["w_up"])),
                                  w64(ew["w_down"]))
                    y[b] += p[j] * ye
            sels.append(np.stack(sel_l))
            sws.append(np.stack(sw_l))
        x = x + y
        h_mlp.append(x.clone())
    xf = F.rms_norm(x, (H,), w64(g["final_norm"]), eps=cfg.rms_eps)
    lm = g["lm_head"] if g.get("lm_head") is not None else g["embed"]
    logits = F.linear(xf, w64(lm))
    out = {"h_attn": torch.stack(h_attn).numpy(), "h_mlp": torch.stack(h_mlp).numpy(), "logits": logits.numpy()}
    if cfg.n_experts:
        out["router_logits"] = torch.stack(rl).numpy()
        out["sel"] = np.stack(sels)
        out["sel_w"] = np.stack(sws)
    return out
