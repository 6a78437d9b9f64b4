"""Write the oracle regression fixtures of this folder.

The pages on the method print no worked numeric example, so every stored value
here comes from the fp64 oracle (and only from it) on a small seeded workload.
The fixtures guard the oracle against unnoticed changes to its arithmetic;
what pins the oracle to the method is test_oracle_pins.py.

Run from the repository root:  python tests/golden/make_golden.py
"""

import os
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import bpt_inputs as bi  # noqa: E402
import oracle  # noqa: E402

CASES = {
    # name: (shape, rows to store)
    "tiny_causal_bf16": (bi.LayerShape(1, 64, 64, 2, 16, 32, True), [0, 1, 15, 16, 33, 63]),
    "tiny_noncausal_f32": (bi.LayerShape(2, 32, 64, 1, 8, 8, False, "f32"), [0, 7, 31, 32, 50, 63]),
}


def compute(name):
    shp, rows = CASES[name]
    inp = {k: bi.to_f64(v) for k, v in bi.make_inputs(shp, seed=0).items()}
    a = tuple(inp[k] for k in ("x", "Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2"))
    y = oracle.layer_forward(*a, heads=shp.heads, causal=shp.causal, threads=1)
    return shp, rows, y.reshape(-1, shp.h)[rows]


def main():
    here = os.path.dirname(os.path.abspath(__file__))
    for name in CASES:
        shp, rows, vals = compute(name)
        with open(os.path.join(here, f"{name}.txt"), "w") as f:
            f.write(f"# oracle output rows of the seeded workload {shp} (seed 0)\n")
            f.write("# written by tests/golden/make_golden.py from oracle/ only; format: row, then h values\n")
            for r, v in zip(rows, vals):
                f.write(f"{r} " + " ".join(repr(float(t)) for t in v) + "\n")


if __name__ == "__main__":
    main()
