"""Shared helpers for the parity tests: tolerance metrics and oracle calls on
the exact tensors the CUDA path received."""
import numpy as np
import torch

import oracle
from gated_delta_rule_85_b200.workloads import to_f64

# Bounds stated for the operator: fp32 inputs rel-L2 <= 1e-4; bf16 inputs
# rel-L2 <= 1e-2 and max-abs <= 5e-2 on o and on the final state.
TOL = {torch.float32: dict(rel_l2=1e-4, max_abs=None), torch.bfloat16: dict(rel_l2=1e-2, max_abs=5e-2)}


def rel_l2(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.linalg.norm(y.ravel())
    return float(np.linalg.norm((x - y).ravel()) / (den if den > 0 else 1.0))


def max_abs(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.abs(x - y))) if x.size else 0.0


def assert_close(got, want, dtype, what=""):
    tol = TOL[dtype]
    r = rel_l2(got, want)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite values"
    assert r <= tol["rel_l2"], f"{what}: rel-L2 {r:.3e} > {tol['rel_l2']:.0e}"
    if tol["max_abs"] is not None:
        m = max_abs(got, want)
        assert m <= tol["max_abs"], f"{what}: max-abs {m:.3e} > {tol['max_abs']:.0e}"
    return r


def oracle_prefill(d, heads=None):
    """Oracle on the inputs dict (optionally a subset of heads, selected on the
    device before widening to float64).  Returns (o, S) float64."""
    keys = ["q", "k", "v", "log_alpha", "beta"]

    def pick(x, state=False):
        if x is None:
            return None
        if heads is not None:
            idx = torch.as_tensor(heads, device=x.device)
            x = x.index_select(1 if state else 2, idx)
        return to_f64(x)

    arrs = [pick(d[x]) for x in keys]
    s0 = pick(d.get("init_state"), state=True)
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    return oracle.forward(*arrs, init_state=s0, cu_seqlens=cu)
