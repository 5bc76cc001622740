"""Writes tests/golden/oracle_small.json: a small seeded case and the oracle's
output for it.  Calls only oracle/ (and numpy for the seeded inputs); the file
is a regression guard for the oracle's arithmetic, whose correctness is pinned
separately by closed forms and special cases in tests/test_oracle_pins.py."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.Generator(np.random.PCG64(20261202))
    B, T, H, dk, dv = 1, 6, 2, 3, 2
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, T, H, dv))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(B, T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    S0 = 0.01 * rng.normal(size=(B, H, dk, dv))
    o, S = oracle.forward(q, k, v, g, b, S0)
    out = {
        "what": "KDA token recurrence, fp64 oracle output (regression guard)",
        "inputs": {"q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "log_alpha": g.tolist(),
                   "beta": b.tolist(), "init_state": S0.tolist()},
        "o": o.tolist(),
        "final_state": S.tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
