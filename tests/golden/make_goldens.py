"""Write the certified LM-head goldens for the named synthetic workloads.

Calls only ``oracle`` and the seeded generator.  For each workload:

1. draw the inputs (``tree_verification_jsv_b200.synth``);
2. compute every node's fp64 greedy choice with ``oracle.lmhead_top2``;
3. certify with ``oracle.certify_margin`` that the choice cannot flip under
   any fp32 summation order; redraw the hidden row of every uncertified node
   from its next sub-stream and repeat until all are certified;
4. plant the tree tokens from the certified choices and store, as JSON:
   the redraw counts, the argmax of every node, the planted tokens, the
   oracle walk's accept length and bonus token per request, and the
   smallest margin/bound ratio.

Temperature-0 greedy selection by the target's own logits follows the
JetSpec README ("JetSpec / Overview"; ``temperature=0.0`` in its examples).

Usage: python tests/golden/make_goldens.py [names...]
"""
import json
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
from tree_verification_jsv_b200 import synth  # noqa: E402

HERE = Path(__file__).resolve().parent


def make(name: str) -> dict:
    t0 = time.time()
    wl = synth.make_workload(name, values=False, lmhead=True)
    T, d = wl.T, wl.d
    wmax = oracle.w_row_norm_max(wl.w)
    arg = np.zeros(T, dtype=np.int64)
    ratio = np.zeros(T)
    redraws: dict[int, int] = {}
    rows = np.arange(T)
    H = wl.hidden
    rounds = 0
    while len(rows):
        a, t1, t2 = oracle.lmhead_top2(H, wl.w, rows=rows)
        ok, r = oracle.certify_margin(H, wl.w, a, t1, t2, rows=rows, wmax=wmax)
        arg[rows[ok]] = a[ok]
        ratio[rows[ok]] = r[ok]
        bad = rows[~ok]
        for t in bad:
            redraws[int(t)] = redraws.get(int(t), 0) + 1
            H[t] = synth.normal_bf16(wl.seed, "hidden_redraw", d, 1.0 / np.sqrt(d), int(t), redraws[int(t)])
        rows = bad
        rounds += 1
    wl.redraws = redraws
    assert np.array_equal(synth.hidden_rows(wl.seed, T, d, redraws), H)
    tokens = synth.plant_tokens(wl, arg)
    walk = oracle.accept_batch(wl.node_offsets, wl.parent, tokens, arg)
    out = {
        "workload": name,
        "seed": wl.seed,
        "T": T,
        "d": d,
        "V": wl.V,
        "source": "tests/golden/make_goldens.py (oracle.lmhead_top2 + oracle.certify_margin)",
        "certification": "l1 - l2 > 4 * d * 2^-24 * (A_v1 + |H|_2 max_v |W_v|_2)",
        "redraw_rounds": rounds,
        "redraws": {str(k): v for k, v in sorted(redraws.items())},
        "min_margin_ratio": float(ratio.min()),
        "argmax": [int(x) for x in arg],
        "tokens": [int(x) for x in tokens],
        "accept_len": [int(w[1]) for w in walk],
        "bonus": [int(w[2]) for w in walk],
        "seconds": round(time.time() - t0, 1),
    }
    return out


if __name__ == "__main__":
    names = sys.argv[1:] or list(synth.SHAPES)
    for n in names:
        g = make(n)
        (HERE / f"lmhead_{n}.json").write_text(json.dumps(g, separators=(",", ":")) + "\n")
        print(n, "T", g["T"], "redrawn", len(g["redraws"]), "rounds", g["redraw_rounds"],
              "min ratio %.3f" % g["min_margin_ratio"], "%.1fs" % g["seconds"], flush=True)
