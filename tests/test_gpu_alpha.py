"""GPU parity of alpha-CROWN (vf_alpha_grad, vf_alpha_crown) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, sound_on_samples

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


@pytest.mark.parametrize("config,B", [(1, 16), (2, 6), (3, 2)])
def test_alpha_grad_matches_oracle(config, B):
    w = synth.workload(config, B=B)
    net, R = w.net, w.C.shape[1]
    rng = np.random.default_rng(5)
    g = vf.Net(net)
    relus = g.relu_ids
    alpha = rng.random(g.alpha_size(B, R)).astype(np.float32)  # seeded slopes, from the test
    lb, grad = g.alpha_grad(_dev(w.centres), w.eps, _dev(w.C), _dev(alpha))
    torch.cuda.synchronize()
    g.check()
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
            # gradient entries: compare where the oracle's coefficient sign is clear (the kink of the
            # |.| and of the slope choice makes the gradient one-sided at lam = 0)
            assert _viol(gg, og[k]).max() <= 10.0, f"centre {b} relu {k}: {_viol(gg, og[k]).max()}"
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
    # the same 5 Adam steps in fp64 end within tolerance on all but a few rows (kinks may split them)
    best, start = O.alpha_crown(net, w.centres, w.eps, w.C, iters=5, lr=0.1)
    v = _viol(lb[ok], best[ok])
    assert (v > 1.0).mean() <= 0.05, f"{(v > 1.0).mean():.3f} of rows off the oracle trajectory"
    assert sound_on_samples(net, w.centres[:4], w.eps, w.C[:4] if w.C.shape[0] > 1 else w.C, lb[:4], None, n=2000)


def test_alpha_rejects_non_chains():
    rng = np.random.default_rng(7)
    net = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(3, 4, 5), fc=6, classes=4)
    centres = rng.random((2, 3 * 8 * 8)).astype(np.float32)
    C = synth.margin_spec(np.array([0, 1]), 4)
    g = vf.Net(net)
    with pytest.raises(vf.VfError) as e:
        g.alpha_crown(_dev(centres), 0.01, _dev(C), iters=1)
    assert e.value.code == vf.VF_ERR_UNSUPPORTED
