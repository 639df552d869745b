"""Golden fixtures under tests/golden/: values the pages print (cited in the JSON) and an oracle
regression fixture written by tests/golden/make_oracle_fixture.py (which calls only oracle/)."""

import json
import os

import numpy as np

import oracle
from mhc_hyper_connection_02_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_mix_layout_from_the_pages():
    g = load("pages_constants.json")
    lay = g["mix_layout"]
    assert lay["hc"] * (2 + lay["hc"]) == lay["mix"] == inputs.MIX
    assert lay["pre"] == [0, 4] and lay["post"] == [4, 8] and lay["comb"] == [8, 24]
    for hc, v in g["mix_hc"]["values"].items():
        assert (2 + int(hc)) * int(hc) == v
    assert g["mix_hc"]["values"]["4"] == g["mix_hc"]["max_kernel_mix"]
    s = g["mix_scratch_bytes"]
    assert 256 * inputs.MIX * s["bytes_per_entry"] * s["sites"] == s["at_256_tokens"]
    assert 1024 * inputs.MIX * s["bytes_per_entry"] * s["sites"] == s["at_1024_tokens"]


def test_oracle_logit_layout_matches_pages():
    """A logit placed at pre/post/comb offsets of the page layout lands in that output."""
    w = inputs.custom(1, 8, 3)
    base = np.zeros(24, np.float32)
    base[2] = 5.0     # pre[2]
    base[4 + 1] = -5.0  # post[1]
    out = oracle.pre(np.zeros((1, 4, 8), np.uint16), np.zeros((32, 24), np.float32),
                     np.ones(3, np.float32), base)
    assert out["pre"][0, 2] > 0.99 and out["post"][0, 1] < 0.02
    del w


def test_oracle_matches_stored_fixture():
    for case in load("oracle_tiny.json"):
        c = case["case"]
        w = inputs.custom(c["T"], c["H"], c["seed"])
        r = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                       post_mult=w.post_mult, iters=w.iters, eps=w.eps)
        for k in ("rstd", "logits", "pre", "post", "comb", "y"):
            want = np.array([float.fromhex(v) for v in case[k]])
            np.testing.assert_array_equal(r[k].ravel(), want, err_msg=k)
        o = oracle.post(w.x, w.R, r["post"].astype(np.float32), r["comb"].astype(np.float32))
        np.testing.assert_array_equal(o.ravel(), [float.fromhex(v) for v in case["post_out"]])
