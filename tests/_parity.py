"""Comparison rules shared by the GPU parity tests.

Tolerance: the GPU computes in fp32 (FFMA or 3xTF32 tensor-core products, fp32 accumulation);
the oracle in fp64. A bound matches when |gpu - oracle| <= 1e-4 * (|oracle| + 1).

Decisions taken from floating point: the adaptive lower slope of an unstable ReLU jumps from
0 to 1 where u = -l. When a neuron's |u + l| / (u - l) is within 1e-5 of that tie in the
oracle's own bounds, fp32 and fp64 may take different (both correct) branches and every
later bound of that centre may differ by a finite amount. Such centres are compared on what
stays unique -- both results must be sound on sampled inputs -- instead of element-wise.
All other stable/unstable switches are continuous in (l, u) and need no special case.
"""
from __future__ import annotations

import numpy as np

import oracle.lbp as O

REL_TOL = 1e-4
TIE_TOL = 1e-5


def tol(oracle_vals):
    return REL_TOL * (np.abs(oracle_vals) + 1.0)


def max_violation(gpu, ora):
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    return float(np.max(np.abs(gpu - ora) / tol(ora))) if ora.size else 0.0


def ambiguous_centres(res: "O.OracleResult", net, alphas=None) -> np.ndarray:
    """Centres with an adaptive-slope decision within TIE_TOL of its tie (relative)."""
    alphas = alphas or {}
    B = res.lb.shape[0]
    amb = np.zeros(B, bool)
    for k in [v for v, nd in enumerate(net) if nd.op == "relu"]:
        if k in alphas:
            continue
        l, u = res.pre_bounds[k]
        unst = (l < 0) & (u > 0)
        ratio = np.where(unst, np.abs(u + l) / np.maximum(u - l, 1e-300), np.inf)
        amb |= (ratio < TIE_TOL).any(axis=1)
    return amb


def sound_on_samples(net, centres, eps, C, lb, ub=None, n=2000, seed=0):
    """Every sampled network output (uniform in the box plus random vertices) lies within the bounds
    (up to the fp32 tolerance)."""
    rng = np.random.default_rng(seed)
    for b in range(centres.shape[0]):
        c = centres[b].astype(np.float64)
        xs = np.concatenate([c + eps * (2 * rng.random((n, c.size)) - 1), c + eps * rng.choice([-1.0, 1.0], (n // 4, c.size))])
        Cb = C[b if C.shape[0] > 1 else 0].astype(np.float64)
        y = O.forward(net, xs)[-1] @ Cb.T
        if np.any(y < lb[b] - tol(y)):
            return False
        if ub is not None and np.any(y > ub[b] + tol(y)):
            return False
    return True


def kink_sensitive_rows(run, centres, eps, rows, rel=1e-6):
    """Rows (centre b, row r) at a kink of an iterative computation: `run(centre_batch, eps)` -> [b, R] is the
    oracle's result (fp64). A row whose result moves by more than the parity tolerance when eps changes by a
    relative `rel` -- a change far below any tolerance, about the size of fp32 rounding in the inputs -- has a
    discontinuity there (a branch of a decision flips), so fp32 and fp64 may legitimately end on different
    branches. Returns a boolean mask over `rows` (a list of (b, r))."""
    out = np.zeros(len(rows), bool)
    by_centre = {}
    for i, (b, r) in enumerate(rows):
        by_centre.setdefault(b, []).append((i, r))
    for b, items in by_centre.items():
        base = run(centres[b:b + 1], eps)[0]
        hi = run(centres[b:b + 1], eps * (1 + rel))[0]
        lo = run(centres[b:b + 1], eps * (1 - rel))[0]
        for i, r in items:
            t = REL_TOL * (abs(base[r]) + 1.0)
            out[i] = abs(hi[r] - base[r]) > t or abs(lo[r] - base[r]) > t
    return out
