"""Shared test helpers: tolerances and seeded case builders.

The tolerances are the parity bar for this library (fixed before any kernel
existed): fp32 max |err| <= 1e-5; bf16 max |err| <= 2e-2 and mean |err| <= 2e-3;
INT4 (against an oracle fed the identically dequantised K/V) max |err| <= 2e-2;
cache contents and INT4 codes bit-exact.

INT4 outputs are bf16.  The 4-bit workload has x10 outlier channels, so an
output element can reach |O| ~ 40, and bf16 cannot hold such a value to within
2e-2: rounding alone moves it by up to half an ulp, 2^-9 |O| (0.078 at 40).
The INT4 bound is therefore the absolute 2e-2 plus that half-ulp of the
reference value, 2e-2 + 2^-9 |ref|, elementwise.  No other slack is allowed.
"""

import numpy as np
import torch

BF16_HALF_ULP_REL = 2.0 ** -9

TOL = {
    "f32": dict(max=1e-5, mean=None, bf16_rounding=False),
    "bf16": dict(max=2e-2, mean=2e-3, bf16_rounding=False),
    "int4": dict(max=2e-2, mean=None, bf16_rounding=True),
}


def parity_errors(got, ref, bf16_rounding=False):
    """(max, mean) of |got - ref|; with bf16_rounding the error of each
    element first loses the output's own rounding allowance, 2^-9 |ref|, so
    that the result compares directly with the absolute bound."""
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, dtype=np.float64)
    err = np.abs(g - r)
    if bf16_rounding:
        err = np.maximum(err - BF16_HALF_ULP_REL * np.abs(r), 0.0)
    return float(err.max()), float(err.mean())


def assert_parity(got, ref, kind, what=""):
    tol = TOL[kind]
    mx, mean = parity_errors(got, ref, tol["bf16_rounding"])
    assert np.isfinite(mx), "%s: non-finite output" % what
    assert mx <= tol["max"], "%s: max |err| %.3g > %.3g%s" % (
        what, mx, tol["max"], " (+ 2^-9 |ref|)" if tol["bf16_rounding"] else "")
    if tol["mean"] is not None:
        assert mean <= tol["mean"], "%s: mean |err| %.3g > %.3g" % (what, mean, tol["mean"])
    return mx, mean


def raw_max_error(got, ref):
    """Plain max |got - ref| (reported next to the bound in test output)."""
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    return float(np.abs(g - np.asarray(ref, dtype=np.float64)).max())


def seeded_mask(seed, n_kv, n_ret):
    g = torch.Generator().manual_seed(seed)
    m = torch.zeros(n_kv, dtype=torch.uint8)
    m[torch.randperm(n_kv, generator=g)[:n_ret]] = 1
    return m


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()
