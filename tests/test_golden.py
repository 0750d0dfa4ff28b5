"""The stored LM-head goldens agree with the generator and the oracle."""
import json
from pathlib import Path

import numpy as np
import pytest

import oracle
from tree_verification_jsv_b200 import synth

GOLD = Path(__file__).resolve().parent / "golden"


def load_golden(name):
    return json.loads((GOLD / f"lmhead_{name}.json").read_text())


@pytest.mark.parametrize("name", list(synth.SHAPES))
def test_tokens_are_planted_from_stored_argmax(name):
    g = load_golden(name)
    wl = synth.make_workload(name, values=False, lmhead=False)
    assert g["T"] == wl.T and g["seed"] == wl.seed
    tok = synth.plant_tokens(wl, np.asarray(g["argmax"]))
    assert tok.tolist() == g["tokens"]
    assert g["min_margin_ratio"] > 1.0


def test_tiny_golden_recomputes_from_oracle():
    g = load_golden("tiny")
    wl = synth.make_workload("tiny", values=False, redraws={int(k): v for k, v in g["redraws"].items()})
    a, t1, t2 = oracle.lmhead_top2(wl.hidden, wl.w)
    ok, _ = oracle.certify_margin(wl.hidden, wl.w, a, t1, t2)
    assert ok.all() and a.tolist() == g["argmax"]
