"""Write oracle_tiny.json by calling only the oracle (regression fixture)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def case(gate, seed):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 6, 1, 3, 4
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    gs = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = (-0.5 * np.log1p(np.exp(rng.standard_normal(gs)))).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((B, T, H))))).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((B, H, dv, dk))).astype(np.float32)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, S0.astype(np.float64), gate=gate, nthreads=1)
    return dict(gate=gate, seed=seed, q=q.tolist(), k=k.tolist(), v=v.tolist(), g=g.tolist(),
                beta=beta.tolist(), S0=S0.tolist(), o=o.tolist(), S_T=S_T.tolist())


if __name__ == "__main__":
    out = dict(note="written by tests/golden/make_golden.py from oracle.gdr_fwd",
               cases=[case("scalar", 1), case("channel", 2)])
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(out, f, indent=1)
