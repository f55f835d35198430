"""GPU parity of alpha-CROWN (vf_alpha_grad, vf_alpha_crown) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, kink_sensitive_rows, sound_on_samples

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _viol(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(got - ref) / (1e-4 * (np.abs(ref) + 1.0))


def _oracle_relax(net, res, b):
    return {k: O.relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b])
            for k, nd in enumerate(net) if nd.op == "relu"}


@pytest.mark.parametrize("config,B", [(1, 16), (2, 6), (2, 16), (3, 2)])
def test_alpha_grad_matches_oracle(monkeypatch, config, B):
    """Bound and slope gradient element-wise. Workload 2 at 16 centres has 144 rows per pass, so with the forward
    products on the tensor cores whenever the shapes allow (VF_FWD_TC=all) the gradient's G W^T + b runs there
    (at 6 centres, 54 rows, on the FFMA kernel). The down pass's contractions take the tensor cores whenever the
    shapes allow as well (VF_DENSE_KERNEL=tc)."""
    monkeypatch.setenv("VF_FWD_TC", "all")
    monkeypatch.setenv("VF_DENSE_KERNEL", "tc")
    w = synth.workload(config, B=B)
    net, R = w.net, w.C.shape[1]
    rng = np.random.default_rng(5)
    g = vf.Net(net)
    relus = g.relu_ids
    alpha = rng.random(g.alpha_size(B, R)).astype(np.float32)  # seeded slopes, from the test
    g.profile(True)
    g.profile_read(reset=True)
    lb, grad = g.alpha_grad(_dev(w.centres), w.eps, _dev(w.C), _dev(alpha))
    torch.cuda.synchronize()
    g.check()
    fwd_tc = g.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC)[0]
    assert (fwd_tc > 0) == (config == 2 and B * R >= 128), fwd_tc
    lb, grad = lb.cpu().numpy(), grad.cpu().numpy()
    res = O.verify(net, w.centres, w.eps, w.C)
    amb = ambiguous_centres(res, net)
    off = 0
    blocks = {}
    for k in relus:
        n = g.sizes[k]
        blocks[k] = (off, n)
        off += B * R * n
    checked = 0
    for b in range(B):
        if amb[b]:
            continue
        relax = _oracle_relax(net, res, b)
        a = {k: alpha[o + b * R * n: o + (b + 1) * R * n].reshape(R, n).astype(np.float64)
             for k, (o, n) in blocks.items()}
        Cb = w.C[b if w.C.shape[0] > 1 else 0]
        olb, og = O.spec_bound_alpha(net, w.centres[b], w.eps, Cb, relax, a)
        assert _viol(lb[b], olb).max() <= 1.0, f"centre {b}"
        for k, (o, n) in blocks.items():
            gg = grad[o + b * R * n: o + (b + 1) * R * n].reshape(R, n)
            # every gradient entry at the parity tolerance (the gradient is a chain of fp32 contractions
            # like the bound itself; the measured worst entry is well inside it)
            assert _viol(gg, og[k]).max() <= 1.0, f"centre {b} relu {k}: {_viol(gg, og[k]).max()}"
        checked += 1
    assert checked >= B // 2


@pytest.mark.parametrize("config,B", [(1, 64), (2, 16), (3, 3)])
def test_alpha_crown_improves_soundly_and_tracks_oracle(config, B):
    w = synth.workload(config, B=B)
    net = w.net
    g = vf.Net(net)
    out = g.alpha_crown(_dev(w.centres), w.eps, _dev(w.C), iters=5, lr=0.1)
    torch.cuda.synchronize()
    g.check()
    lb, lb0 = out["lb"].cpu().numpy(), out["lb_start"].cpu().numpy()
    assert np.all(lb >= lb0)
    # the adaptive start is exactly the CROWN bound of vf_verify_batch's specification pass
    res = O.verify(net, w.centres, w.eps, w.C)
    amb = ambiguous_centres(res, net)
    ok = ~amb
    assert _viol(lb0[ok], res.lb_crown[ok]).max() <= 1.0
    # the same 5 Adam steps in fp64 end within tolerance on every row that is not at a kink of the
    # trajectory: a row may leave the oracle's value only if the oracle's own value jumps under a 1e-6
    # relative change of eps (a slope step or a slope choice flips there)
    best, start = O.alpha_crown(net, w.centres, w.eps, w.C, iters=5, lr=0.1)
    _assert_off_rows_at_kinks(net, w.centres, w.eps, w.C, lb, best, ok, iters=5)
    assert sound_on_samples(net, w.centres[:4], w.eps, w.C[:4] if w.C.shape[0] > 1 else w.C, lb[:4], None, n=2000)


def _assert_off_rows_at_kinks(net, centres, eps, C, lb, best, ok, iters, splits=None, starts=None):
    """Every row of a centre without an adaptive-slope near-tie matches the oracle's optimised bound, or
    sits at a kink of the optimisation (kink_sensitive_rows)."""
    off = [(b, r) for b in range(lb.shape[0]) if ok[b] for r in range(lb.shape[1])
           if _viol(lb[b, r], best[b, r]) > 1.0]
    if not off:
        return

    by_b = {}
    for b, r in off:
        by_b.setdefault(b, []).append(r)
    bad = []
    for b, rs in by_b.items():
        Cb = C[b:b + 1] if C.shape[0] > 1 else C
        sp = None if splits is None else {k: v[b:b + 1] for k, v in splits.items()}
        st = None if starts is None else [starts[b]]
        kink = kink_sensitive_rows(lambda c, e: O.alpha_crown(net, c, e, Cb, iters=iters, lr=0.1, splits=sp,
                                                              starts=st)[0],
                                   centres[b:b + 1], eps, [(0, r) for r in rs])
        bad += [(b, r) for r, k in zip(rs, kink) if not k]
    assert not bad, f"rows off the oracle's trajectory without a kink: {bad[:8]} (of {len(off)} off)"


def _small_residual(seed=7, B=2):
    rng = np.random.default_rng(seed)
    net = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(3, 4, 5), fc=6, classes=4)
    centres = rng.random((B, 3 * 8 * 8)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 4, B), 4)
    return net, centres, C, 0.02


def test_alpha_grad_matches_oracle_residual():
    """The graph form of the slope gradient (residual adds, identity and 1x1-convolution shortcuts)."""
    net, centres, C, eps = _small_residual()
    B, R = centres.shape[0], C.shape[1]
    g = vf.Net(net)
    rng = np.random.default_rng(9)
    alpha = rng.random(g.alpha_size(B, R)).astype(np.float32)
    lb, grad = g.alpha_grad(_dev(centres), eps, _dev(C), _dev(alpha))
    torch.cuda.synchronize()
    g.check()
    lb, grad = lb.cpu().numpy(), grad.cpu().numpy()
    res = O.verify(net, centres, eps, C)
    amb = ambiguous_centres(res, net)
    off, checked = 0, 0
    blocks = {}
    for k in g.relu_ids:
        blocks[k] = (off, g.sizes[k])
        off += B * R * g.sizes[k]
    for b in range(B):
        if amb[b]:
            continue
        relax = _oracle_relax(net, res, b)
        a = {k: alpha[o + b * R * n: o + (b + 1) * R * n].reshape(R, n).astype(np.float64) for k, (o, n) in blocks.items()}
        olb, og = O.spec_bound_alpha(net, centres[b], eps, C[b], relax, a)
        assert _viol(lb[b], olb).max() <= 1.0, f"centre {b}"
        for k, (o, n) in blocks.items():
            gg = grad[o + b * R * n: o + (b + 1) * R * n].reshape(R, n)
            assert _viol(gg, og[k]).max() <= 1.0, f"centre {b} relu {k}: {_viol(gg, og[k]).max()}"
        checked += 1
    assert checked >= 1


def test_alpha_crown_residual_improves_soundly():
    net, centres, C, eps = _small_residual(B=3)
    g = vf.Net(net)
    out = g.alpha_crown(_dev(centres), eps, _dev(C), iters=5, lr=0.1)
    torch.cuda.synchronize()
    g.check()
    lb, lb0 = out["lb"].cpu().numpy(), out["lb_start"].cpu().numpy()
    assert np.all(lb >= lb0)
    res = O.verify(net, centres, eps, C)
    ok = ~ambiguous_centres(res, net)
    assert _viol(lb0[ok], res.lb_crown[ok]).max() <= 1.0
    best, start = O.alpha_crown(net, centres, eps, C, iters=5, lr=0.1)
    _assert_off_rows_at_kinks(net, centres, eps, C, lb, best, ok, iters=5)
    assert sound_on_samples(net, centres, eps, C, lb, None, n=2000)


def test_alpha_rejects_both_sides():
    w = synth.workload(2, B=2)
    g = vf.Net(w.net)
    o, keep = g._opts()
    o.both_sides = 1
    B, R = 2, w.C.shape[1]
    lb = torch.empty(B, R, device="cuda")
    code = vf.lib().vf_alpha_crown(g.h, vf._ptr(_dev(w.centres)), B, float(w.eps), vf._ptr(_dev(w.C)), R, 0,
                                   vf.ctypes.byref(o), 1, 0.1, vf._ptr(lb), None, None, vf._stream_ptr())
    assert code == vf.VF_ERR_UNSUPPORTED
