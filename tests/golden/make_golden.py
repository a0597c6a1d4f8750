"""Write tests/golden/tiny_f32.json: oracle forward + backward on the tiny fp32 workload.

A regression snapshot of the CPU oracle (it calls nothing but ``oracle/`` and the seeded input
generator), so that any later change to the oracle's arithmetic shows up as a diff here.
Run from the repository root:  python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

import oracle
from deformable_slide_attention_b200 import inputs

ITEMS = [0, 1, 37, 63, 64, 130, 255, 256, 300, 511]  # h*N + n, N = 256


def main():
    w = inputs.BY_NAME["tiny-f32"]
    inp = inputs.make(w, "cpu", with_dout=True)
    out, lse = oracle.forward(inp["q"], inp["k"], inp["v"], inp["offsets"], w.dims, w.window, ITEMS)
    dq, doff, dk, dv = oracle.backward(inp["q"], inp["k"], inp["v"], inp["offsets"], inp["dout"],
                                       w.dims, w.window, ITEMS, ITEMS)
    rec = {
        "what": "3D-DSA oracle outputs on the tiny-f32 workload (seeded; dO drawn after offsets)",
        "source": "oracle/dsa3d_oracle.c via tests/golden/make_golden.py",
        "workload": w.name, "items": ITEMS,
        "out": out.tolist(), "lse": [float(x) for x in lse],
        "dq": dq.tolist(), "doff": doff.tolist(), "dk": dk.tolist(), "dv": dv.tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32.json")
    with open(path, "w") as f:
        json.dump(rec, f)
    print("wrote", path, "max|out|", float(np.abs(out).max()))


if __name__ == "__main__":
    main()
