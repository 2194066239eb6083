"""Write oracle_siblings_tiny.json by calling only the oracle (regression
fixture for gated linear attention, the DPLR transition, the backward and
the prologue)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def inputs(seed):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 6, 1, 3, 4
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    q, k, v, a, b = f(B, T, H, dk), f(B, T, H, dk), f(B, T, H, dv), f(B, T, H, dk), f(B, T, H, dk)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a *= 0.2
    b *= 0.2
    g = (-0.5 * np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((B, T, H))))).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((B, H, dv, dk))).astype(np.float32)
    dout = f(B, T, H, dv)
    return dict(q=q, k=k, v=v, a=a, b=b, g=g, beta=beta, S0=S0, dout=dout)


def results(x):
    S0 = x["S0"].astype(np.float64)
    o_gla, S_gla = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], S0, gate="channel", nthreads=1)
    o_dp, S_dp = oracle.dplr_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["g"], S0,
                                 gate="channel", nthreads=1)
    gr = oracle.gdr_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dout"], S0, None,
                        gate="channel", nthreads=1)
    gs = np.array([0.1], np.float32)
    o_pr, S_pr = oracle.gdr_fwd_prologue(x["q"], x["k"], x["v"], x["g"][..., 0], x["beta"], gs,
                                         S0, nthreads=1)
    return dict(o_gla=o_gla, S_gla=S_gla, o_dplr=o_dp, S_dplr=S_dp, o_pro=o_pr, S_pro=S_pr,
                **{k: v for k, v in gr.items()})


if __name__ == "__main__":
    x = inputs(3)
    r = results(x)
    out = dict(note="written by tests/golden/make_golden_siblings.py from oracle/",
               inputs={k: v.tolist() for k, v in x.items()},
               results={k: np.asarray(v).tolist() for k, v in r.items()})
    with open(os.path.join(HERE, "oracle_siblings_tiny.json"), "w") as f:
        json.dump(out, f, indent=1)
