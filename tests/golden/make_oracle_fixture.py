"""Writes tests/golden/oracle_tiny.json: the fp64 oracle's outputs on two tiny seeded cases, stored
as exact hex floats. It calls only oracle/ (and the input generator), so the stored values never
come from the CUDA path. Re-run only when a change to the oracle's arithmetic is justified by the
pages; tests/test_golden.py then fails until the fixture is rewritten.

    python tests/golden/make_oracle_fixture.py
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from mhc_hyper_connection_02_b200 import inputs  # noqa: E402

CASES = [dict(T=2, H=8, seed=7), dict(T=3, H=13, seed=8)]


def hexlist(a):
    return [float(v).hex() for v in np.asarray(a, dtype=np.float64).ravel()]


def main():
    out = []
    for c in CASES:
        w = inputs.custom(c["T"], c["H"], c["seed"])
        r = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                       post_mult=w.post_mult, iters=w.iters, eps=w.eps)
        p32 = r["post"].astype(np.float32)
        c32 = r["comb"].astype(np.float32)
        o = oracle.post(w.x, w.R, p32, c32)
        out.append({"case": c, **{k: hexlist(r[k]) for k in ("rstd", "logits", "pre", "post", "comb", "y")},
                    "post_out": hexlist(o)})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
