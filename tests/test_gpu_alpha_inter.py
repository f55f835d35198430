"""GPU parity of alpha-CROWN for the intermediate bounds (vf_opts.alpha_inter_iters) against the fp64 oracle's
``verify(..., alpha_inter_iters=...)``, through the C ABI.

Every refined pre-activation bound and every final lower bound is compared element-wise at the parity tolerance.
The ascent takes the sign of gradient entries (Adam's first steps move a slope by lr * sign(g)), a decision made
in floating point, so a value may leave the oracle's only where the oracle's own result jumps when eps changes
by 1e-6 relative (a kink of the optimisation, as for the specification ascent); those values are listed and
must stay few. Centres with an adaptive-slope near-tie are compared by soundness only."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import relu_ids
from tests._parity import REL_TOL, ambiguous_centres, sound_on_samples, tol

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _mlp(seed=41, B=4):
    rng = np.random.default_rng(seed)
    net = synth.mlp([8, 16, 16, 16, 4], rng)
    centres = rng.random((B, 8)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 4, B), 4)
    return net, centres, C, float(np.float32(0.15))


def _wl(config, B):
    w = synth.workload(config, B=B)
    return w.net, w.centres, w.C, w.eps


CASES = {"mlp8-16x3-4": (_mlp, 6), "mlp784-256x3-10": (lambda: _wl(2, 2), 3), "cnn3x32x32": (lambda: _wl(3, 1), 2)}


def _values(net, pre_l, pre_u, lb):
    """One vector per centre: the bounds of every ReLU's source (lower, upper), then the final lower bounds."""
    parts = []
    for k in relu_ids(net):
        parts += [pre_l[k], pre_u[k]]
    return np.concatenate(parts + [lb], axis=1)


def _oracle(net, centres, eps, C, iters, splits=None):
    res = O.verify(net, centres, eps, C, alpha_inter_iters=iters, alpha_inter_lr=0.1, splits=splits)
    return res, _values(net, {k: res.pre_bounds[k][0] for k in res.pre_bounds},
                        {k: res.pre_bounds[k][1] for k in res.pre_bounds}, res.lb)


def _gpu(g, net, centres, eps, C, iters, splits=None):
    B = centres.shape[0]
    sp = None if splits is None else {k: _dev(v.astype(np.int8)) for k, v in splits.items()}
    out = g.verify(_dev(centres), eps, _dev(C), want_pre=True, alpha_inter_iters=iters, alpha_inter_lr=0.1, splits=sp)
    torch.cuda.synchronize()
    g.check()
    pl = {k: g.node_block(out["pre_lb"], net[k].src, B).cpu().numpy() for k in relu_ids(net)}
    pu = {k: g.node_block(out["pre_ub"], net[k].src, B).cpu().numpy() for k in relu_ids(net)}
    return out, pl, pu, _values(net, pl, pu, out["lb"].cpu().numpy())


def _assert_parity_off_kinks(net, centres, eps, C, iters, gv, ov, ok, splits=None, max_kink_frac=0.1):
    viol = np.abs(gv - ov) / tol(ov)
    kinks = 0
    for b in np.nonzero(ok)[0]:
        off = np.nonzero(viol[b] > 1.0)[0]
        if off.size == 0:
            continue
        Cb = C[b:b + 1] if C.shape[0] > 1 else C
        sp = None if splits is None else {k: v[b:b + 1] for k, v in splits.items()}
        hi = _oracle(net, centres[b:b + 1], eps * (1 + 1e-6), Cb, iters, sp)[1][0]
        lo = _oracle(net, centres[b:b + 1], eps * (1 - 1e-6), Cb, iters, sp)[1][0]
        t = REL_TOL * (np.abs(ov[b]) + 1.0)
        sens = (np.abs(hi - ov[b]) > t) | (np.abs(lo - ov[b]) > t)
        bad = off[~sens[off]]
        assert bad.size == 0, f"centre {b}: values {bad[:8]} off the oracle without a kink (worst {viol[b].max():.3g})"
        kinks += off.size
    assert kinks <= max_kink_frac * ov[ok].size, f"{kinks} of {ov[ok].size} values at kinks"


@pytest.mark.parametrize("case", list(CASES))
def test_alpha_inter_matches_oracle(case):
    make, iters = CASES[case]
    net, centres, C, eps = make()
    res, ov = _oracle(net, centres, eps, C, iters)
    g = vf.Net(net)
    out, pl, pu, gv = _gpu(g, net, centres, eps, C, iters)
    ok = ~ambiguous_centres(res, net)
    assert ok.sum() >= max(1, centres.shape[0] // 2)
    _assert_parity_off_kinks(net, centres, eps, C, iters, gv, ov, ok)
    # never looser than the plain bounds of the same device path, and sound on samples
    plain = g.verify(_dev(centres), eps, _dev(C), want_pre=True)
    torch.cuda.synchronize()
    B = centres.shape[0]
    tightened = 0
    for k in relu_ids(net):
        p0 = g.node_block(plain["pre_lb"], net[k].src, B).cpu().numpy()
        q0 = g.node_block(plain["pre_ub"], net[k].src, B).cpu().numpy()
        assert np.all(pl[k] >= p0) and np.all(pu[k] <= q0), k
        tightened += int(np.sum(pl[k] > p0) + np.sum(pu[k] < q0))
    assert tightened > 0
    lb = out["lb"].cpu().numpy()
    assert sound_on_samples(net, centres, eps, C, lb, None, n=2000)


def test_alpha_inter_with_splits_matches_oracle():
    """Branch-and-bound subdomains: split constraints on the first ReLU layer; the intermediate ascent then also
    optimises the split multipliers beta of the earlier layers."""
    net, centres, C, eps = _mlp(seed=43, B=4)
    rng = np.random.default_rng(5)
    k1 = relu_ids(net)[0]
    # the signs of z at one input of each box, on a random half of the neurons: no subdomain is empty
    x0 = centres + eps * (2 * rng.random(centres.shape) - 1)
    z = O.forward(net, x0.astype(np.float64))[net[k1].src]
    sp = {k1: (np.where(z >= 0, 1, -1) * (rng.random(z.shape) < 0.5)).astype(np.int8)}
    res, ov = _oracle(net, centres, eps, C, 5, sp)
    g = vf.Net(net)
    _, _, _, gv = _gpu(g, net, centres, eps, C, 5, sp)
    ok = ~ambiguous_centres(res, net)
    assert ok.sum() >= 2
    _assert_parity_off_kinks(net, centres, eps, C, 5, gv, ov, ok, splits=sp)


def test_alpha_crown_on_refined_intermediate_bounds():
    """vf_alpha_crown with alpha_inter_iters: the specification ascent runs on the refined intermediate bounds,
    against the oracle's alpha_crown with the same options (rows at kinks excepted)."""
    net, centres, C, eps = _mlp(seed=44, B=3)
    g = vf.Net(net)
    r = g.alpha_crown(_dev(centres), eps, _dev(C), iters=4, lr=0.1, alpha_inter_iters=4, alpha_inter_lr=0.1)
    torch.cuda.synchronize()
    g.check()
    lb = r["lb"].cpu().numpy()
    best, _ = O.alpha_crown(net, centres, eps, C, iters=4, lr=0.1, alpha_inter_iters=4, alpha_inter_lr=0.1)
    res = O.verify(net, centres, eps, C, alpha_inter_iters=4, alpha_inter_lr=0.1)
    ok = ~ambiguous_centres(res, net)
    viol = np.abs(lb - best) / tol(best)
    for b in np.nonzero(ok)[0]:
        off = np.nonzero(viol[b] > 1.0)[0]
        if off.size == 0:
            continue
        run = lambda e: O.alpha_crown(net, centres[b:b + 1], e, C[b:b + 1], iters=4, lr=0.1, alpha_inter_iters=4,
                                      alpha_inter_lr=0.1)[0][0]
        hi, lo = run(eps * (1 + 1e-6)), run(eps * (1 - 1e-6))
        t = REL_TOL * (np.abs(best[b]) + 1.0)
        sens = (np.abs(hi - best[b]) > t) | (np.abs(lo - best[b]) > t)
        assert np.all(sens[off]), f"centre {b}: rows {off[~sens[off]]} off the oracle without a kink"
    assert sound_on_samples(net, centres, eps, C, lb, None, n=2000)


def test_alpha_inter_rejects_unsupported_options():
    net, centres, C, eps = _mlp(B=2)
    g = vf.Net(net)
    for kw, code in ((dict(alpha_inter_iters=-1), vf.VF_ERR_ARG), (dict(alpha_inter_iters=2, sound=True), vf.VF_ERR_UNSUPPORTED),
                     (dict(alpha_inter_iters=2, no_host_sync=True), vf.VF_ERR_UNSUPPORTED),
                     (dict(alpha_inter_iters=2, alpha_inter_lr=float("nan")), vf.VF_ERR_NONFINITE)):
        with pytest.raises(vf.VfError) as e:
            g.verify(_dev(centres), eps, _dev(C), **kw)
        assert e.value.code == code, kw
    rng = np.random.default_rng(7)
    rnet = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(3, 4, 5), fc=6, classes=4)
    gr = vf.Net(rnet)
    with pytest.raises(vf.VfError) as e:
        gr.verify(_dev(rng.random((1, 192)).astype(np.float32)), 0.02, _dev(synth.margin_spec(np.array([0]), 4)),
                  alpha_inter_iters=2)
    assert e.value.code == vf.VF_ERR_UNSUPPORTED
