"""Helpers shared by the GPU parity tests (host-side marshalling and the
tolerance rule; no arithmetic of the scan itself)."""
from __future__ import annotations

import numpy as np

import oracle

# y tolerance per io dtype and the state tolerance (fp32 state in both cases)
RTOL_Y = {"f32": 1e-5, "bf16": 2e-2}
RTOL_STATE = 1e-6
# gradients: per-element rule for the activation gradients (io dtype), and
# the parameter / state gradients (fp32 sums over all tokens)
RTOL_GRAD = {"f32": 1e-5, "bf16": 2e-2, "param": 1e-5}


def to_dev(a, device="cuda"):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_f64(t) -> np.ndarray:
    """Device tensor -> float64 numpy, widening bf16 exactly."""
    import torch
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return oracle.decode(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy().astype(np.float64)


def c12(got, want, rtol):
    """Per-element |got - want| <= rtol * (|want| + rms(want)); returns (ok, worst ratio)."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return True, 0.0
    rms = float(np.sqrt(np.mean(want * want)))
    bound = rtol * (np.abs(want) + rms)
    err = np.abs(got - want)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    worst = float(np.max(ratio))
    return bool(np.all(np.isfinite(got)) and worst <= 1.0), worst


def state_norm_err(got, want):
    """Normwise error of cached states: for every [D, N] cache slice,
    max|got - want| / max|want|; returns the worst slice."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return 0.0
    g2 = got.reshape(-1, got.shape[-2] * got.shape[-1])
    w2 = want.reshape(-1, want.shape[-2] * want.shape[-1])
    num = np.max(np.abs(g2 - w2), axis=1)
    den = np.max(np.abs(w2), axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(den > 0, num / den, np.where(num > 0, np.inf, 0.0))
    return float(np.max(r)) if np.all(np.isfinite(got)) else float("inf")


# every state check of the session: (what, normwise error / rtol, worst
# per-element ratio against rtol * (|o| + rms(o))); printed at the end of the run
STATE_LOG = []


def assert_state(got, want, what="", rtol=RTOL_STATE):
    """Cached states (fp32) match the oracle to rtol normwise per [D, N] cache.
    The per-element ratio |g - o| / (rtol (|o| + rms(o))) is computed beside it
    and logged (not asserted: an fp32 state recurrence cannot meet a
    per-element bound at 1e-6)."""
    err = state_norm_err(got, want)
    _, per_elem = c12(got, want, rtol)
    STATE_LOG.append((what, err / rtol, per_elem))
    assert err <= rtol, f"{what}: normwise state error {err:.3g} > {rtol} (per-element ratio {per_elem:.3g})"
    return err


def assert_c12(got, want, rtol, what=""):
    ok, worst = c12(got, want, rtol)
    assert ok, f"{what}: worst error is {worst:.3g}x the tolerance (rtol {rtol})"
    return worst
