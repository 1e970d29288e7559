"""The stored oracle outputs in tests/golden: the oracle still reproduces them, and the GPU step matches them.

tiny_step0.json holds the oracle's step 0 of the tiny model (written by
tests/golden/make_golden.py, which calls only the oracle and the seeded input
generator).  The first test makes any change to the oracle's arithmetic show
up; the second checks the CUDA path against the stored values with the same
tolerances as the live parity tests, without running the oracle.
"""
import json
import os

import numpy as np
import pytest

import fixtures as fx
from tests.helpers import rel_l2

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_step0.json")


def load():
    with open(GOLDEN) as f:
        return json.load(f)


def test_golden_provenance():
    d = load()
    cfg = fx.CONFIGS[d["config"]]
    assert "make_golden.py" in d["what"] and "oracle" in d["source"]
    assert np.asarray(d["h_attn"]).shape == (cfg.n_layers, cfg.batch * cfg.hidden)
    assert np.asarray(d["h_mlp"]).shape == (cfg.n_layers, cfg.batch * cfg.hidden)
    assert len(d["logits"]) == cfg.batch * cfg.vocab
    assert d["tokens"] == [int(t) for t in fx.tokens(cfg)[0]]


def test_oracle_reproduces_golden():
    from tests.golden.make_golden import tiny_step0
    d = load()
    cfg, tok, S, out = tiny_step0()
    assert [int(t) for t in tok] == d["tokens"] and [int(s) for s in S] == d["positions"]
    for key in ("h_attn", "h_mlp"):
        got = out[key].reshape(cfg.n_layers, -1)
        assert rel_l2(got, np.asarray(d[key])) < 1e-12, key
    assert rel_l2(out["logits"].reshape(-1), np.asarray(d["logits"])) < 1e-12


@pytest.mark.gpu
def test_gpu_step_matches_golden():
    import torch

    import auto_regressive_decode_b200.mk as mk
    from fixtures.device import device_caches, device_model
    from tests.gpu_harness import TOL_HIDDEN, TOL_LOGITS_ABS
    d = load()
    cfg = fx.CONFIGS[d["config"]]
    S = np.asarray(d["positions"], dtype=np.int32)
    w = device_model(cfg, gains=d["gains"])
    kc, vc = device_caches(cfg, S)
    dec = mk.Decoder(cfg, w, kc, vc)
    logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    dt = torch.tensor(d["tokens"], dtype=torch.int32, device="cuda")
    ds = torch.from_numpy(S.copy()).cuda()
    dec.step(dt, ds, ds, logits)
    assert dec.status() == 0
    hid = dec.hidden_states().cpu().numpy().astype(np.float64)
    for l in range(cfg.n_layers):
        assert rel_l2(hid[2 * l + 1].reshape(-1), np.asarray(d["h_attn"][l])) <= TOL_HIDDEN
        assert rel_l2(hid[2 * l + 2].reshape(-1), np.asarray(d["h_mlp"][l])) <= TOL_HIDDEN
    lg = logits.cpu().numpy().astype(np.float64).reshape(-1)
    assert np.max(np.abs(lg - np.asarray(d["logits"]))) <= TOL_LOGITS_ABS
    dec.close()
