"""GPU parity of the forward products on the tensor cores (tcgen05 kind::tf32 with the 3xTF32 split, the kernel of
the dense back-substitution read through an identity relaxation row). By default they serve the alpha ascent's
G W^T + b (products of 32 output tiles or more; VF_FWD_TC=all: every product the shapes allow), tested in
test_gpu_alpha.py and by the rule below. VF_FWD_TC=ibp also puts the IBP centre W c + b and radius |W| r of dense
layers [SNNV §2.1] there; that option is tested here against the fp64 oracle through the C ABI, with the FFMA kernel
(VF_FWD_TC=0) as a second path. It is off by default because on the 3072-1024x8-100 network its bounds drift to the
edge of the parity tolerance after eight layers. The shapes cover ragged row tiles (M not a multiple of 128), ragged column tiles (N = 1000 in four tiles of
256), layers the kernel does not take (K < 32, N < 16: FFMA) in the same network, and the smallest M it takes."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, max_violation

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


CASES = [([784, 256, 256, 10], 300), ([64, 48, 36, 20, 5], 128), ([32, 1000, 16], 257), ([784, 256, 10], 127)]


@pytest.mark.parametrize("dims,B", CASES, ids=[f"{'-'.join(map(str, d))}_B{b}" for d, b in CASES])
def test_ibp_forward_products_match_oracle(monkeypatch, dims, B):
    rng = np.random.default_rng(sum(dims) + B)
    net = synth.mlp(dims, rng)
    centres = rng.random((B, dims[0])).astype(np.float32)
    eps = float(np.float32(0.01))
    ib = O.ibp(net, centres, eps)
    got = {}
    for fwd in ("ibp", "0"):
        monkeypatch.setenv("VF_FWD_TC", fwd)
        g = vf.Net(net)
        g.profile(True)
        g.profile_read(reset=True)
        lb, ub = g.ibp(_dev(centres), eps)
        torch.cuda.synchronize()
        g.check()
        n_tc = g.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC)[0]
        assert (n_tc > 0) == (fwd == "ibp" and B >= 128), n_tc
        for v in range(len(net)):
            gl = g.node_block(lb, v, B).cpu().numpy()
            gu = g.node_block(ub, v, B).cpu().numpy()
            assert max_violation(gl, ib[0][v] - ib[1][v]) <= 1.0, (fwd, v)
            assert max_violation(gu, ib[0][v] + ib[1][v]) <= 1.0, (fwd, v)
            got[(fwd, v)] = (gl, gu)
    for v in range(len(net)):  # the two paths within the tolerance of each other as well
        for a, b in zip(got[("ibp", v)], got[("0", v)]):
            assert max_violation(a, b.astype(np.float64)) <= 1.0, v


def test_verify_with_forward_products_on_tensor_cores(monkeypatch):
    """The whole verify step at 256 centres of the 784-256x3-10 network with the IBP products on the tensor
    cores: final and intermediate bounds element-wise against the oracle on sampled centres."""
    monkeypatch.setenv("VF_FWD_TC", "ibp")
    w = synth.workload(2, B=256)
    g = vf.Net(w.net)
    g.profile(True)
    g.profile_read(reset=True)
    out = g.verify(_dev(w.centres), w.eps, _dev(w.C), want_pre=True)
    torch.cuda.synchronize()
    g.check()
    assert g.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC)[0] > 0
    pick = np.sort(np.random.default_rng(3).choice(256, 6, replace=False))
    C = w.C[pick] if w.C.shape[0] > 1 else w.C
    ora = O.verify(w.net, w.centres[pick], w.eps, C)
    ok = ~ambiguous_centres(ora, w.net)  # an adaptive slope at its tie may flip between fp32 and fp64
    assert ok.sum() >= 3
    lb = out["lb"].cpu().numpy()[pick]
    assert max_violation(lb[ok], ora.lb[ok]) <= 1.0
    for k, (l, u) in ora.pre_bounds.items():
        src = w.net[k].src
        gl = g.node_block(out["pre_lb"], src, 256).cpu().numpy()[pick]
        gu = g.node_block(out["pre_ub"], src, 256).cpu().numpy()[pick]
        assert max_violation(gl[ok], l[ok]) <= 1.0, k
        assert max_violation(gu[ok], u[ok]) <= 1.0, k


def test_default_rule_by_tile_count(monkeypatch):
    """By default only the alpha ascent's products take the tensor cores, and only with 32 output tiles or more:
    the gradient of 1024 centres x 9 rows through 256 neurons (72 tiles) does, that of 16 centres (2 tiles) does
    not, and the IBP of 4096 centres through 1024 neurons (128 tiles) stays on the FFMA kernel."""
    monkeypatch.delenv("VF_FWD_TC", raising=False)
    for B, want in ((1024, True), (16, False)):
        w = synth.workload(2, B=B)
        g = vf.Net(w.net)
        R = w.C.shape[1]
        alpha = torch.full((g.alpha_size(B, R),), 0.5, device="cuda")
        g.profile(True)
        g.profile_read(reset=True)
        g.alpha_grad(_dev(w.centres), w.eps, _dev(w.C), alpha)
        torch.cuda.synchronize()
        g.check()
        assert (g.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC)[0] > 0) == want, B
    rng = np.random.default_rng(4096)
    net = synth.mlp([256, 1024, 1024, 10], rng)
    g = vf.Net(net)
    g.profile(True)
    g.profile_read(reset=True)
    g.ibp(_dev(rng.random((4096, 256)).astype(np.float32)), 0.01)
    torch.cuda.synchronize()
    assert g.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC)[0] == 0
