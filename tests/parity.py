"""Helpers shared by the GPU parity tests: tolerances and the per-head
bridge between torch tensors and the oracle's numpy arrays."""
from __future__ import annotations

import numpy as np
import torch

# Floating-point bar for bf16 outputs and gradients: max-abs 2e-2 and
# rel-L2 5e-3.  The max-abs bound is applied to |x - y| / max(1, |y|): bf16
# storage alone rounds by up to 2^-9 |y|, which passes 2e-2 in absolute
# terms once |y| > 10, and outputs here reach |y| ~ 50 (heavy tokens).
MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


# Every assert_close call appends one row here (the test, the quantity, the
# plain max-abs |x - y|, the envelope-scaled max-abs, rel-L2, and the share
# of elements within the plain 2e-2); conftest writes the rows of a GPU run
# to tests/results/parity_errors.json at the end of the session.
RECORDS: list[dict] = []


def close_report(got, want, env=None):
    """(max |x - y| / max(1, env), rel-L2).  env is the magnitude of what was
    summed to make y (|y| itself by default; for a sum of rounded terms, the
    sum of the terms' magnitudes, since each term carries its own rounding)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    env = np.abs(want) if env is None else np.asarray(env, dtype=np.float64)
    err = np.abs(got - want)
    scaled = float(np.max(err / np.maximum(1.0, env))) if err.size else 0.0
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)) if err.size else 0.0
    return scaled, rel


def record(got, want, name, env=None):
    """Append the plain and scaled error figures of one comparison to RECORDS."""
    import os
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    scaled, rel = close_report(got, want, env)
    err = np.abs(got - want)
    RECORDS.append({
        "test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
        "quantity": name, "elements": int(err.size),
        "max_abs": float(err.max()) if err.size else 0.0,
        "max_abs_scaled": scaled, "rel_l2": rel,
        "frac_within_plain_2e-2": float(np.mean(err <= MAX_ABS)) if err.size else 1.0,
        "max_abs_ref": float(np.abs(want).max()) if want.size else 0.0})
    return scaled, rel


def assert_close(got, want, name, max_abs=MAX_ABS, rel_l2=REL_L2, env=None):
    scaled, rel = record(got, want, name, env)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert scaled <= max_abs and rel <= rel_l2, f"{name}: max-abs(scaled) {scaled:.3e}, rel-L2 {rel:.3e}"
    return scaled, rel


def bf16_ulp(x):
    """One unit in the last place of bf16 at |x| (x != 0), as fp64."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.where(x > 0, x, 1.0))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


def head(x: torch.Tensor, b: int, h: int) -> np.ndarray:
    """[B, N, H, d] tensor -> one head's [N, d] fp64 array."""
    return np.ascontiguousarray(x[b, :, h, :].to(torch.float64).cpu().numpy())


def attn_bwd_envelopes(qg, kg, vg, dog, scale, chunk=256, rows=None):
    """Magnitude envelopes of the attention gradients: the sums that make
    each gradient with every term replaced by its magnitude.  dS = P dP - P D
    is formed from two products, so its envelope is P (|dP| + |D|):
    scale P(|dP|+|D|) |K|, scale (P(|dP|+|D|))^T |Q| and P^T |dO| (fp64).
    ``rows`` restricts the query rows (exact for those rows' dQ, and for the
    dK / dV columns that only those rows reach)."""
    S = qg.shape[0]
    eq, ek, ev = np.zeros_like(qg), np.zeros_like(kg), np.zeros_like(vg)
    cols = np.arange(S)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    for a in range(0, rows.shape[0], chunk):
        r = rows[a:a + chunk]
        s = (qg[r] @ kg.T) * scale
        s[cols[None, :] > r[:, None]] = -np.inf
        pr = np.exp(s - s.max(axis=1)[:, None])
        pr /= pr.sum(axis=1)[:, None]
        dp = dog[r] @ vg.T
        dd = np.abs((pr * dp).sum(axis=1))[:, None]
        ds = pr * (np.abs(dp) + dd)
        eq[r] = scale * (ds @ np.abs(kg))
        ek += scale * (ds.T @ np.abs(qg[r]))
        ev += pr.T @ np.abs(dog[r])
    return eq, ek, ev


def attn_envelopes_full(qg, kg, vg, dog, scale, chunk=256):
    """All four magnitude envelopes of one head's attention over every row, in
    one pass with each row block restricted to its causal key prefix: P|V|
    (output), and the three gradient envelopes of attn_bwd_envelopes."""
    S = qg.shape[0]
    eo = np.zeros_like(vg)
    eq, ek, ev = np.zeros_like(qg), np.zeros_like(kg), np.zeros_like(vg)
    cols = np.arange(S)
    aq, ak, av, ado = np.abs(qg), np.abs(kg), np.abs(vg), np.abs(dog)
    for a in range(0, S, chunk):
        r = np.arange(a, min(a + chunk, S))
        hi = int(r[-1]) + 1
        s = (qg[r] @ kg[:hi].T) * scale
        s[cols[None, :hi] > r[:, None]] = -np.inf
        pr = np.exp(s - s.max(axis=1)[:, None])
        pr /= pr.sum(axis=1)[:, None]
        eo[r] = pr @ av[:hi]
        dp = dog[r] @ vg[:hi].T
        dd = np.abs((pr * dp).sum(axis=1))[:, None]
        ds = pr * (np.abs(dp) + dd)
        eq[r] = scale * (ds @ ak[:hi])
        ek[:hi] += scale * (ds.T @ aq[r])
        ev[:hi] += pr.T @ ado[r]
    return eo, eq, ek, ev
