"""Write the oracle's regression fixtures (tests/golden/oracle_regression.json).

This script calls only the fp64 oracle and the seeded input generator.  The
fixtures record what the oracle computes today on small seeded cases of every
function it offers, so that a later change to its arithmetic shows up in
tests/test_golden.py; such a change must then name the passage that justifies
it and regenerate the file with this script.  They pin the oracle against its
own past, not against the method: the correctness pins are the closed forms,
limits and identities of tests/test_oracle_pins.py.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402

OUT = os.path.join(HERE, "oracle_regression.json")


def cases():
    """(name, workload, seed, extra oracle keywords) of every fixture."""
    return [
        ("fwd_f32", I.Workload("g", 1, 3, 9, 4, "f32"), 1, {}),
        ("fwd_bf16", I.Workload("g", 2, 2, 7, 16, "bf16"), 2, {}),
        ("fwd_h0", I.Workload("g", 1, 2, 6, 4, "f32"), 3, {"h0": True}),
        ("fwd_conv", I.Workload("g", 1, 2, 8, 4, "f32"), 4, {"conv": 3}),
        ("fwd_zoh", I.Workload("g", 1, 2, 8, 4, "f32"), 5, {"zoh": True}),
        ("bwd", I.Workload("g", 2, 2, 6, 4, "f32"), 6, {"bwd": True}),
    ]


def run(w, seed, extra):
    x = I.make_inputs(w, seed=seed)
    args = (x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    if extra.get("bwd"):
        dy = I.fill(seed, 12, (w.batch, w.dim, w.seqlen)).astype(np.float64)
        g = oracle.scan_bwd(*args, dy=dy, nthreads=1)
        return {k: v.tolist() for k, v in g.items() if v is not None}
    kw = {"nthreads": 1}
    if extra.get("h0"):
        kw["h0"] = I.make_state(w.batch, w.dim, w.dstate, seed=seed)
    if extra.get("conv"):
        kw["conv_weight"], kw["conv_bias"] = I.make_conv(w.dim, extra["conv"], seed=seed)
    if extra.get("zoh"):
        kw["zoh"] = True
    y, h = oracle.scan_fwd(*args, **kw)
    return {"y": y.tolist(), "last_state": h.tolist()}


def main():
    data = {}
    for name, w, seed, extra in cases():
        data[name] = {"workload": [w.batch, w.dim, w.seqlen, w.dstate, w.dtype], "seed": seed,
                      "extra": extra, "outputs": run(w, seed, extra)}
    with open(OUT, "w") as f:
        json.dump(data, f, indent=0)
        f.write("\n")
    print(f"wrote {OUT}")


if __name__ == "__main__":
    main()
