"""Shared helpers for the GPU parity tests: device inputs, error metrics and
the tolerances, each stated once.

Tolerances (floating point; bf16 outputs against the fp64 oracle):
  O:   max |err| <= 1e-2 and ||err||_2 / ||ref||_2 <= 5e-3
  LSE: max |err| <= 1e-3
  dQ, dK, dV: ||err||_2 / ||ref||_2 <= 1e-2; where the reference gradient is
              exactly zero (e.g. dQ and dK with a single key, where dS = 0),
              the relative error is undefined and max |g| <= 1e-3 is used
              instead (a quarter of a bf16 ulp at unit magnitude).
"""
import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def has_gpu():
    return torch.cuda.is_available() and torch.cuda.get_device_capability()[0] == 10


def to_dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def max_abs(a, ref):
    a = np.asarray(a, np.float64)
    return float(np.max(np.abs(a - ref))) if a.size else 0.0


def rel_l2(a, ref):
    a = np.asarray(a, np.float64)
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(a - ref)) / max(den, 1e-300)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_o(O, ref, what=""):
    ma, rl = max_abs(O, ref), rel_l2(O, ref)
    assert ma <= O_MAX_ABS and rl <= O_REL_L2, f"{what} O max-abs {ma:.3e} rel-L2 {rl:.3e}"
    return ma, rl


def assert_lse(L, ref, what=""):
    L = np.asarray(L, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(L), np.isneginf(ref)), f"{what} LSE -inf pattern differs"
    ma = max_abs(L[fin], ref[fin])
    assert ma <= LSE_ABS, f"{what} LSE max-abs {ma:.3e}"
    return ma


ZERO_GRAD_ABS = 1e-3


def assert_grad(g, ref, name, what=""):
    if not np.any(ref):
        ma = float(np.max(np.abs(np.asarray(g, np.float64))))
        assert ma <= ZERO_GRAD_ABS, f"{what} {name} should be zero, max |g| {ma:.3e}"
        return ma
    rl = rel_l2(g, ref)
    assert rl <= GRAD_REL_L2, f"{what} {name} rel-L2 {rl:.3e}"
    return rl
