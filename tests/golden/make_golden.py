"""Writes tests/golden/tiny_step.txt: the oracle's loss and per-tensor
gradient norms on the tiny workload (bf16 weights from seed 0, uniform token
ids from seed 1).  Calls only the oracle and the seeded input generators."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    wl = synth.WORKLOADS["tiny"]
    _, w = synth.make_weights(wl.model, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1)
    loss, g = oracle.step(wl.model, w, tok, tgt)
    G = oracle.views(wl.model, g)
    with open(os.path.join(HERE, "tiny_step.txt"), "w") as f:
        f.write("# oracle loss and gradient L2 norms, tiny workload; written by make_golden.py\n")
        f.write(f"loss {float(loss)!r}\n")
        for name, arr in G.items():
            f.write(f"norm.{name} {float(np.linalg.norm(arr))!r}\n")


if __name__ == "__main__":
    main()
