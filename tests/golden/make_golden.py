"""Write tiny_step0.json: the oracle's outputs for the first decode step of the tiny model.

The pages print no worked example of the decode step, so the stored values are
the oracle's own (oracle/oracle.c, fp64), from the seeded generator's inputs
(fixtures, master seed 0): tokens of step 0 at the prefilled length, the
residual stream after every attention and MLP block, and the logits.  Nothing
here touches the CUDA path.  Re-run after a change to the oracle's arithmetic
that a passage of the pages justifies, and say which in the commit.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import fixtures as fx  # noqa: E402
import oracle as ora  # noqa: E402
from tests.helpers import host_caches, host_model  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_step0.json")


def tiny_step0():
    """Inputs and oracle outputs of step 0 of the tiny model (gains "random")."""
    cfg = fx.CONFIGS["tiny"]
    g, ls = host_model(cfg, gains="random")
    S = fx.context_lengths(cfg)
    kc, vc = host_caches(cfg, S)
    model = ora.Model(cfg, g["embed"], g["final_norm"], g["lm_head"], ls)
    tok = fx.tokens(cfg)[0]
    out = model.decode_step(kc, vc, tok, S, S)
    return cfg, tok, S, out


def main():
    cfg, tok, S, out = tiny_step0()
    doc = {
        "what": "oracle outputs of decode step 0 of the tiny model; written by tests/golden/make_golden.py",
        "source": "oracle/oracle.c (fp64); inputs from fixtures (seed 0, gains random); no page prints a worked example",
        "config": cfg.name,
        "gains": "random",
        "tokens": [int(t) for t in tok],
        "positions": [int(s) for s in S],
        "h_attn": [[float(v) for v in row] for row in out["h_attn"].reshape(cfg.n_layers, -1)],
        "h_mlp": [[float(v) for v in row] for row in out["h_mlp"].reshape(cfg.n_layers, -1)],
        "logits": [float(v) for v in out["logits"].reshape(-1)],
    }
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=0)
        f.write("\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()
