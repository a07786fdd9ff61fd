"""Writes oracle_tiny_snapshot.json: the fp64 oracle's kept sets, candidate counts
and sampled outputs on the seeded tiny workload (first 192 tokens, three update
intervals of 64, both kv-head streams). It calls only oracle/ and the seeded input
generator; no value comes from the CUDA path.

This is a regression snapshot of the oracle, not a pin: the oracle is pinned by
tests/test_oracle_pins.py against closed forms, brute force and special cases.
The snapshot catches unintended drift. A deliberate change to the oracle's
arithmetic regenerates it, and the commit names the passage that justifies the
change.

    python tests/golden/make_oracle_snapshot.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from hybrid_linear_attention_lola_b200 import workloads as wl  # noqa: E402

T = 192
SAMPLES = [(0, 5, 0, 0), (0, 63, 1, 7), (0, 64, 0, 31), (0, 100, 1, 62), (0, 127, 0, 13),
           (0, 128, 1, 0), (0, 150, 0, 44), (0, 191, 1, 63)]   # (b, t, q-head, dim)


def compute():
    w = wl.WORKLOADS["tiny"]
    q, k, v, _ = wl.make_inputs(w, T=T)
    W = wl.make_W(w)
    ints = [w.chunk] * (T // w.chunk)
    r = oracle.run(q, k, v, W, window=w.window, lambda_=w.lambda_, intervals=ints, eps=w.eps)
    return {
        "workload": "tiny (B 1, Hq 2, Hkv 2, d 64, D 64, window 64, lambda 32, chunk 64), first %d tokens" % T,
        "intervals": ints,
        "nq": r.nq.tolist(),
        "nkept": r.nkept.tolist(),
        "kept": [[[int(x) for x in r.kept[i, s, :r.nkept[i, s]]] for s in range(r.kept.shape[1])]
                 for i in range(len(ints))],
        "out_samples": [[list(ix), float(r.out[ix])] for ix in SAMPLES],
        "out_abs_sum": float(np.abs(r.out).sum()),
    }


if __name__ == "__main__":
    snap = compute()
    with open(os.path.join(HERE, "oracle_tiny_snapshot.json"), "w") as f:
        json.dump(snap, f, indent=1)
        f.write("\n")
    print("wrote", os.path.join(HERE, "oracle_tiny_snapshot.json"))
