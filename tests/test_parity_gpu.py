"""GPU decode step vs the CPU oracle, through the C ABI, teacher-forced on seeded inputs."""
import os

import numpy as np
import pytest

import fixtures as fx
from tests.gpu_harness import assert_parity, run_teacher_forced

pytestmark = pytest.mark.gpu


def test_tiny_all_steps():
    res = run_teacher_forced(fx.CONFIGS["tiny"])
    assert_parity(res)


@pytest.mark.parametrize("kw,gains", [
    ({"qk_norm": True, "tied_embeddings": True, "rope_theta": 5e5}, "random"),
    ({"ctx": 0, "steps": 3}, "ones"),                      # empty cache: position 0
    ({"ctx": 255, "steps": 3}, "random"),                  # new token crosses a chunk boundary
    ({"n_q_heads": 8, "n_kv_heads": 1}, "ones"),           # 8 query heads per KV head
    ({"n_q_heads": 2, "n_kv_heads": 2}, "ones"),           # MHA
])
def test_tiny_variants(kw, gains):
    res = run_teacher_forced(fx.CONFIGS["tiny"].replace(**kw), steps=kw.get("steps", 4), gains=gains)
    assert_parity(res)


def test_tiny_head_dim_128_small_chunks(monkeypatch):
    monkeypatch.setenv("MK_ATTN_CHUNK", "40")            # many chunks, ragged last sub-chunk
    cfg = fx.CONFIGS["tiny"].replace(n_q_heads=4, n_kv_heads=2, head_dim=128, ctx=200, steps=3)
    assert_parity(run_teacher_forced(cfg, gains="random"))


def test_tiny_last_cache_slot():
    cfg = fx.CONFIGS["tiny"].replace(ctx=141, steps=3)   # writes slots 141..143 of 144
    assert_parity(run_teacher_forced(cfg))


def test_dense_0_6b_first_steps():
    assert_parity(run_teacher_forced(fx.CONFIGS["dense-0.6b"], steps=3))
