"""Parity at the benchmark's full workload sizes, in the configuration bench.py times.

The GPU runs the whole batch in one vf_verify_batch call (the workspace bench.py uses, so the same row
blocking and kernels); the oracle then computes a sample of centres one by one. Every centre's bounds
depend only on that centre, so a sampled centre's oracle result is exactly what the full run must match.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, sound_on_samples

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")

BENCH_WORKSPACE = 16 << 30


def _check_sampled(w, sample, both=False):
    net = vf.Net(w.net, workspace_bytes=BENCH_WORKSPACE)
    c = torch.from_numpy(w.centres).cuda()
    C = torch.from_numpy(w.C).cuda()
    out = net.verify(c, w.eps, C, crown_relus=w.crown_relus, both_sides=both)
    torch.cuda.synchronize()
    net.check()
    lb = out["lb"].cpu().numpy()
    ub = out["ub"].cpu().numpy() if both else None
    Cs = w.C[sample] if w.C.shape[0] > 1 else w.C
    ora = O.verify(w.net, w.centres[sample], w.eps, Cs, crown_relus=w.crown_relus, both_sides=both)
    amb = ambiguous_centres(ora, w.net)
    viol = np.max(np.abs(lb[sample] - ora.lb) / (1e-4 * (np.abs(ora.lb) + 1.0)), axis=1)
    if both:
        viol = np.maximum(viol, np.max(np.abs(ub[sample] - ora.ub) / (1e-4 * (np.abs(ora.ub) + 1.0)), axis=1))
    bad = viol > 1.0
    assert not np.any(bad & ~amb), f"full-size parity violated at centres {np.asarray(sample)[bad & ~amb]}: {viol}"
    assert (bad & amb).sum() <= max(1, len(sample) // 4)
    if bad.any():
        idx = np.asarray(sample)[bad]
        assert sound_on_samples(w.net, w.centres[idx], w.eps, w.C[idx] if w.C.shape[0] > 1 else w.C, lb[idx],
                                ub[idx] if both else None, n=500)
    assert np.isfinite(lb).all()
    return out


def test_cfg1_full():
    w = synth.workload(1)
    _check_sampled(w, list(range(64)), both=True)


def test_cfg2_full_size_sampled():
    w = synth.workload(2)
    _check_sampled(w, [0, 1, 255, 511, 512, 777, 1022, 1023])


def test_cfg3_full_size_sampled():
    w = synth.workload(3)
    _check_sampled(w, [0, 128, 255])


@pytest.mark.parametrize("eps", [0.5 / 255, 1.0 / 255, 2.0 / 255])
def test_cfg5_full_size_sampled(eps):
    w = synth.workload(5, eps=eps)
    # eight centres (about a second of oracle time each): with 8 x 1024 IBP-substituted neurons per centre, a
    # centre often holds an adaptive-slope near-tie, and at most a quarter of the sample may sit there
    _check_sampled(w, [0, 1, 1023, 2047, 2048, 3071, 4094, 4095])


@pytest.mark.slow
def test_cfg4_full_size_one_centre():
    w = synth.workload(4)
    _check_sampled(w, [31])
