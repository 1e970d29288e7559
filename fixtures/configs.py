"""Synthetic decode workloads: model shapes and the seeded input recipe.

Each workload is one decoder-only transformer shape plus the decode run it is
measured on (batch, prefilled context lengths, number of decode steps).  The
shapes follow the model sizes the ForgeMegakernel abstract evaluates
("0.6B-13B parameters", dense and MoE families; arxivdaily 2609.12379,
English abstract).  Where a shape leaves a value open the plainest common
choice is taken: RMSNorm eps 1e-6, RoPE theta 1e4, norm gains 1, untied
embeddings unless stated.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int            # dense SwiGLU width (0 for MoE)
    vocab: int
    n_experts: int = 0      # 0 -> dense SwiGLU MLP
    top_k: int = 0
    expert_ffn_dim: int = 0
    qk_norm: bool = False
    tied_embeddings: bool = False
    rms_eps: float = 1e-6
    rope_theta: float = 1e4
    # decode run
    batch: int = 1
    ctx: int = 0            # fixed prefilled context (when ctx_lo == ctx_hi == 0)
    ctx_lo: int = 0         # ragged contexts: uniform integers in [ctx_lo, ctx_hi]
    ctx_hi: int = 0
    steps: int = 1
    weight_sigma: float = 0.02
    kv_sigma: float = 1.0

    @property
    def ragged(self) -> bool:
        return self.ctx_hi > 0

    @property
    def max_prefill(self) -> int:
        return self.ctx_hi if self.ragged else self.ctx

    @property
    def max_ctx(self) -> int:
        """Cache capacity: the largest prefill plus one slot per decode step."""
        return self.max_prefill + self.steps

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def replace(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)

    def weight_bytes(self) -> int:
        """bf16 bytes of every weight tensor (all experts counted)."""
        H, L = self.hidden, self.n_layers
        per = 2 * H + self.q_dim * H * 2 + self.kv_dim * H * 2
        if self.qk_norm:
            per += 2 * self.head_dim
        if self.n_experts:
            per += self.n_experts * 3 * self.expert_ffn_dim * H + self.n_experts * H
        else:
            per += 3 * self.ffn_dim * H
        tot = L * per + H + self.vocab * H * (1 if self.tied_embeddings else 2)
        return 2 * tot


TINY = ModelConfig("tiny", n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn_dim=688,
                   vocab=1024, rms_eps=1e-6, rope_theta=1e4, batch=1, ctx=128, steps=16)

QWEN_0_6B = ModelConfig("dense-0.6b", n_layers=28, hidden=1024, n_q_heads=16, n_kv_heads=8, head_dim=128,
                        ffn_dim=3072, vocab=151936, qk_norm=True, tied_embeddings=True, batch=1, ctx=1024,
                        steps=64)

LLAMA_8B = ModelConfig("dense-8b", n_layers=32, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                       ffn_dim=14336, vocab=128256, rope_theta=5e5, batch=1, ctx=4096, steps=128)

DENSE_13B = ModelConfig("dense-13b-b8", n_layers=40, hidden=5120, n_q_heads=40, n_kv_heads=40, head_dim=128,
                        ffn_dim=13824, vocab=32000, batch=8, ctx_lo=256, ctx_hi=4096, steps=64)

MOE = ModelConfig("moe-128x8", n_layers=48, hidden=2048, n_q_heads=32, n_kv_heads=4, head_dim=128, ffn_dim=0,
                  vocab=151936, n_experts=128, top_k=8, expert_ffn_dim=768, batch=4, ctx_lo=512, ctx_hi=2048,
                  steps=32)

CONFIGS = {c.name: c for c in (TINY, QWEN_0_6B, LLAMA_8B, DENSE_13B, MOE)}
