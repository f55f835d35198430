"""vf_concretize_dense_noalloc: the entry point for callers that cannot allocate device memory (their
device memory belongs to another allocator, or they run under a fixed budget, or they must avoid the
synchronisation that cudaMalloc/cudaFree can cause). Its scratch is a fixed array inside the library.

It must give the same bounds as the fp64 oracle's back-substitution through the layer followed by its
concretisation, and as the handle-based path -- vf_crown_backward from the dense layer followed by
vf_concretize -- within the parity tolerance, on two calls in a row (the shared scratch keeps the
previous call's contents, so the second call checks that nothing stale leaks in). This file is named so
that pytest collects it last; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _rel_violation(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(got - ref) / (1e-4 * (np.abs(ref) + 1.0))))


@pytest.mark.parametrize("shared_rows", [False, True])
def test_noalloc_matches_crown_backward_then_concretize_twice(shared_rows):
    rng = np.random.default_rng(2024)
    net = synth.mlp([784, 256, 10], rng)  # node 1: dense 784 -> 256, fed by the input
    B, R, eps = 37, 21, float(np.float32(2.0 / 255.0))
    centres = torch.from_numpy(rng.random((B, 784)).astype(np.float32)).cuda()
    lam_np = rng.standard_normal((1 if shared_rows else B, R, 256)).astype(np.float32)
    lam = torch.from_numpy(lam_np).cuda()

    g = vf.Net(net)
    lb_all, ub_all = g.ibp(centres, eps)
    lam_in, cst = g.crown_backward(1, lam, lb_all, ub_all, B)
    ref = vf.concretize(lam_in, cst, centres, eps)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()

    # the oracle: rows over z = W x + b back to the input (one dense node on the input), then concretised
    c_np = centres.cpu().numpy()
    ora = np.stack([O.concretize(*O.backward(net[:2], 1, lam_np[0 if shared_rows else i].astype(np.float64), {}),
                                 c_np[i], eps) for i in range(B)])
    assert _rel_violation(ref, ora) <= 1.0

    W = torch.from_numpy(np.ascontiguousarray(net[1].W)).cuda()
    b = torch.from_numpy(np.ascontiguousarray(net[1].b)).cuda()
    out = torch.empty(B, R, device="cuda")
    for call in range(2):
        out.fill_(float("nan"))
        vf.concretize_dense_noalloc(lam, W, b, centres, eps, out=out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}: unwritten outputs"
        assert _rel_violation(got, ora) <= 1.0, f"call {call}: against the oracle"
        assert _rel_violation(got, ref) <= 1.0, f"call {call}: against the handle path"


def test_noalloc_rejects_requests_beyond_its_fixed_scratch():
    L = vf.lib()
    tiny = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(tiny.data_ptr())
    # B*R = 600000 rows with n_in = 784 needs 600000 * (1 + 7) floats > 2^22: rejected before any launch
    rc = L.vf_concretize_dense_noalloc(p, 0, 600000, p, p, p, 0.01, 1, 784, 256, p, None)
    assert rc == vf.VF_ERR_WORKSPACE
    assert b"fixed scratch" in L.vf_last_error()
    torch.cuda.synchronize()
