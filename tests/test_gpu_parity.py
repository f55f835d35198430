"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on seeded inputs.

Sizes are chosen so that the oracle finishes in seconds while the GPU kernels still see
several tiles and ragged tails (row counts and widths that are not multiples of the tiles).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, max_violation, sound_on_samples

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_both(net, centres, eps, C, crown_relus=None, alphas=None, both=False, workspace=0):
    ora = O.verify(net, centres, eps, C, crown_relus=crown_relus, alphas=alphas, both_sides=both)
    g = vf.Net(net, workspace_bytes=workspace)
    a_dev = {k: _dev(v.astype(np.float32)) for k, v in (alphas or {}).items()} or None
    out = g.verify(_dev(centres), eps, _dev(C), crown_relus=crown_relus, alpha=a_dev, both_sides=both, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    out = {k: v.cpu().numpy() for k, v in out.items()}
    return g, ora, out


def _row_violation(gpu, ora):
    """Per-centre max of |gpu - oracle| / tol."""
    gpu = np.asarray(gpu, np.float64).reshape(gpu.shape[0], -1)
    ora = np.asarray(ora, np.float64).reshape(ora.shape[0], -1)
    return np.max(np.abs(gpu - ora) / (1e-4 * (np.abs(ora) + 1.0)), axis=1)


def assert_parity(net, centres, eps, C, g, ora, out, alphas=None, both=False):
    """Element-wise parity on every centre; a centre may differ only if the oracle's bounds put an
    adaptive-slope decision within rounding of its tie, and then its bounds must still be sound."""
    amb = ambiguous_centres(ora, net, alphas)
    B = centres.shape[0]
    bad = _row_violation(out["lb"], ora.lb) > 1.0
    assert max_violation(out["lb_ibp"], ora.lb_ibp) <= 1.0
    if both:
        bad |= _row_violation(out["ub"], ora.ub) > 1.0
    for k in [v for v, nd in enumerate(net) if nd.op == "relu"]:
        p = net[k].src
        gl = g.node_block(torch.from_numpy(out["pre_lb"]), p, B).numpy()
        gu = g.node_block(torch.from_numpy(out["pre_ub"]), p, B).numpy()
        bad |= _row_violation(gl, ora.pre_bounds[k][0]) > 1.0
        bad |= _row_violation(gu, ora.pre_bounds[k][1]) > 1.0
    assert not np.any(bad & ~amb), f"parity violated on centres {np.nonzero(bad & ~amb)[0]}"
    assert (bad & amb).sum() <= max(1, B // 4), f"too many tie-ambiguous centres differ: {(bad & amb).sum()}"
    ok = ~bad
    clear = ok[:, None] & (np.abs(ora.lb) > 1e-4 * (np.abs(ora.lb) + 1))
    assert np.array_equal(out["verified"][clear].astype(bool), ora.verified[clear])
    if bad.any():
        assert sound_on_samples(net, centres[bad], eps, C[bad] if C.shape[0] > 1 else C, out["lb"][bad],
                                out.get("ub")[bad] if both else None)


def test_cfg1_full():
    w = synth.workload(1)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C, both=True)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out, both=True)


def test_cfg2_subset_ragged():
    w = synth.workload(2, B=19)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)


@pytest.mark.parametrize("windows", ["1", "0"])
def test_cfg3_subset(monkeypatch, windows):
    monkeypatch.setenv("VF_CONV_WINDOWS", windows)
    w = synth.workload(3, B=3)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)


@pytest.mark.parametrize("windows", ["1", "0"])
def test_resnet_small_all_paths(monkeypatch, windows):
    monkeypatch.setenv("VF_CONV_WINDOWS", windows)
    rng = np.random.default_rng(41)
    net = synth.resnet_cfg4(rng, image=(3, 12, 12), widths=(5, 6, 7), fc=20, classes=7)
    centres = rng.random((3, 3 * 12 * 12)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 7, 3), 7)
    g, ora, out = run_both(net, centres, np.float32(0.01).item(), C, both=True)
    assert_parity(net, centres, 0.01, C, g, ora, out, both=True)


def _conv_flops(net, centres, eps, C, both):
    g = vf.Net(net)
    g.profile(True)
    g.profile_read(reset=True)
    out = g.verify(_dev(centres), eps, _dev(C), both_sides=both, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    fl = g.profile_read(kind=3, reset=False)[2] + g.profile_read(kind=4)[2]  # whole-map + windowed
    return fl, {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("kernel", ["tile", "warp", "auto"])
def test_whole_map_convolution_kernels(monkeypatch, kernel):
    """Whole-map rows (windows off) through the tiled kernel, through the windowed kernel with the whole map as
    the window, and the default choice between them: all match the oracle on a CNN and a residual net."""
    monkeypatch.setenv("VF_CONV_WINDOWS", "0")
    monkeypatch.setenv("VF_CONV_KERNEL", kernel)
    w = synth.workload(3, B=2)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)
    rng = np.random.default_rng(45)
    net = synth.resnet_cfg4(rng, image=(3, 16, 16), widths=(4, 5, 6), fc=10, classes=5)
    centres = rng.random((2, 3 * 16 * 16)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, 2), 5)
    g, ora, out = run_both(net, centres, 0.01, C, both=True)
    assert_parity(net, centres, 0.01, C, g, ora, out, both=True)


def test_window_kernels_on_mixed_geometries(monkeypatch):
    """Convolutions with 5x5 stride-1, 3x3 stride-2 and 4x4 stride-4 kernels: the stride/tap combinations
    without a position-blocked instance take the per-position windowed kernel, the others the blocked
    one; both window kernels and the whole-map path match the oracle."""
    rng = np.random.default_rng(44)
    net = [synth.Node(synth.INPUT, shape=(3, 16, 16))]
    v = synth._relu(net, synth._conv(net, rng, 0, 3, 4, 5, 1, 2))
    v = synth._relu(net, synth._conv(net, rng, v, 4, 6, 3, 2, 1))
    v = synth._relu(net, synth._conv(net, rng, v, 6, 5, 4, 4, 0))
    v = synth._relu(net, synth._dense(net, rng, v, 5 * 2 * 2, 9))
    synth._dense(net, rng, v, 9, 4)
    B = 3
    centres = rng.random((B, 3 * 16 * 16)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 4, B), 4)
    eps = 0.01
    ora = O.verify(net, centres, eps, C, both_sides=True)
    for windows, kernel in (("1", "2"), ("1", "1"), ("0", "2")):
        monkeypatch.setenv("VF_CONV_WINDOWS", windows)
        monkeypatch.setenv("VF_CONV_WIN_KERNEL", kernel)
        g = vf.Net(net)
        out = g.verify(_dev(centres), eps, _dev(C), both_sides=True, want_pre=True)
        torch.cuda.synchronize()
        g.check()
        out = {k: v.cpu().numpy() for k, v in out.items()}
        assert_parity(net, centres, eps, C, g, ora, out, both=True)


@pytest.mark.parametrize("kernel", ["2", "1"])
def test_receptive_field_windows_through_residual_adds(monkeypatch, kernel):
    """A residual net on a map large enough that windows survive the residual adds (union of the two
    branches' windows, identity shortcuts that share rows, windows that outgrow the map and return to
    whole-map rows). Windowed and whole-map passes both match the oracle, and the windowed run does
    less convolution work."""
    rng = np.random.default_rng(43)
    net = synth.resnet_cfg4(rng, image=(3, 20, 20), widths=(3, 4, 5), fc=12, classes=5)
    B = 2
    centres = rng.random((B, 3 * 20 * 20)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, B), 5)
    eps = 0.01
    monkeypatch.setenv("VF_CONV_WIN_KERNEL", kernel)
    ora = O.verify(net, centres, eps, C, both_sides=True)
    res = {}
    for windows in ("1", "0"):
        monkeypatch.setenv("VF_CONV_WINDOWS", windows)
        fl, out = _conv_flops(net, centres, eps, C, True)
        g = vf.Net(net)
        assert_parity(net, centres, eps, C, g, ora, out, both=True)
        res[windows] = fl
    assert res["1"] < 0.7 * res["0"], res


@pytest.mark.parametrize("compact", ["1", "0"])
@pytest.mark.parametrize("eps", [0.3 / 255, 1e-6])
def test_unstable_compaction_dense(monkeypatch, compact, eps):
    """Intermediate passes over the IBP-unstable neurons only (gathered +-W rows for a dense start): at
    eps 0.3/255 the first refined layer is ~37% unstable and compacted, the second stays plain; at 1e-6
    almost no neuron is unstable and the compacted passes are a few rows per centre."""
    monkeypatch.setenv("VF_COMPACT", compact)
    w = synth.workload(2, B=7, eps=eps)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)


@pytest.mark.parametrize("compact", ["1", "0"])
def test_unstable_compaction_conv(monkeypatch, compact):
    monkeypatch.setenv("VF_COMPACT", compact)
    w = synth.workload(3, B=2)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)


def test_verify_graph_replays_match_plain_calls():
    """A verify call captured in a CUDA graph gives the plain call's bounds, also after new inputs are
    written into its buffers."""
    w = synth.workload(2, B=38)
    net = vf.Net(w.net)
    c_all, C = _dev(w.centres), _dev(w.C)
    a, b = c_all[:19].contiguous(), c_all[19:].contiguous()
    vg = vf.VerifyGraph(net, a, w.eps, C)
    for batch in (a, b, a):
        vg.centres.copy_(batch)
        got = {k: v.clone() for k, v in vg.replay().items()}
        ref = net.verify(batch, w.eps, C)
        torch.cuda.synchronize()
        net.check()
        for k in ("lb", "lb_ibp", "verified"):
            assert torch.equal(got[k], ref[k]), k


def test_verify_graph_cnn_with_windows_and_compaction_off():
    """The captured call runs plain (uncompacted) passes; on a CNN its bounds match the plain call's
    compacted ones and the oracle."""
    w = synth.workload(3, B=2)
    net = vf.Net(w.net)
    c, C = _dev(w.centres), _dev(w.C)
    vg = vf.VerifyGraph(net, c, w.eps, C)
    got = {k: v.cpu().numpy() for k, v in vg.replay().items()}
    ref = {k: v.cpu().numpy() for k, v in net.verify(c, w.eps, C).items()}
    np.testing.assert_allclose(got["lb"], ref["lb"], rtol=1e-6, atol=1e-6)
    ora = O.verify(w.net, w.centres, w.eps, w.C)
    assert max_violation(got["lb"], ora.lb) <= 1.0


@pytest.mark.parametrize("eps", [0.5 / 255, 1.0 / 255, 2.0 / 255])
def test_cfg5_subset_each_eps(eps):
    w = synth.workload(5, B=2, eps=eps)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C, crown_relus=w.crown_relus)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out)


@pytest.mark.parametrize("kernel", ["tc", "ffma", "default"])
def test_cfg2_both_dense_kernels(monkeypatch, kernel):
    """The tensor-core (3xTF32) contraction on every launch the shapes allow, FFMA only, and the default choice
    (launches of few tiles on the K-split FFMA kernel) each match the oracle on the bench network."""
    if kernel == "default":
        monkeypatch.delenv("VF_DENSE_KERNEL", raising=False)
    else:
        monkeypatch.setenv("VF_DENSE_KERNEL", kernel)
    w = synth.workload(2, B=11)
    g, ora, out = run_both(w.net, w.centres, w.eps, w.C, both=True)
    assert_parity(w.net, w.centres, w.eps, w.C, g, ora, out, both=True)


@pytest.mark.parametrize("B,min_tiles,want_tc", [(2, "100000", False), (2, "0", True), (64, None, True)])
def test_dense_kernel_choice_by_tile_count(monkeypatch, B, min_tiles, want_tc):
    """A dense back-substitution takes the tensor cores only when its launch has at least VF_DENSE_TC_MIN_TILES
    output tiles (128 rows x up to 256 columns): with an unreachable minimum every launch runs on the FFMA kernel,
    with 0 every launch the shapes allow runs on the tensor cores, and with the default the intermediate passes of
    64 centres of the 784-256x3-10 network (64 x 512 rows, 256 tiles and more) do. The bounds match the oracle
    either way."""
    monkeypatch.delenv("VF_DENSE_KERNEL", raising=False)
    if min_tiles is None:
        monkeypatch.delenv("VF_DENSE_TC_MIN_TILES", raising=False)
    else:
        monkeypatch.setenv("VF_DENSE_TC_MIN_TILES", min_tiles)
    w = synth.workload(2, B=B)
    g = vf.Net(w.net)
    g.profile(True)
    g.profile_read(reset=True)
    out = g.verify(_dev(w.centres), w.eps, _dev(w.C))
    torch.cuda.synchronize()
    g.check()
    n_tc = g.profile_read(kind=vf.VF_KERNEL_DENSE_TC, reset=False)[0]
    n_ffma = g.profile_read(kind=vf.VF_KERNEL_DENSE_FFMA)[0]
    assert (n_tc > 0) == want_tc, (n_tc, n_ffma)
    assert n_ffma > 0  # the specification pass's first step (K = 10) is always FFMA
    # the K-split FFMA launches reduce their partial tiles in a fixed order: a second call is bitwise identical
    again = g.verify(_dev(w.centres), w.eps, _dev(w.C))
    torch.cuda.synchronize()
    assert torch.equal(again["lb"], out["lb"])
    nb = min(B, 4)  # rows are independent across centres: the oracle checks the first few
    ora = O.verify(w.net, w.centres[:nb], w.eps, w.C[:nb])
    amb = ambiguous_centres(ora, w.net)
    lb = out["lb"].cpu().numpy()
    for b in range(nb):
        if not amb[b]:
            assert max_violation(lb[b], ora.lb[b]) <= 1.0, b


def test_tc_path_wide_mlp_shapes(monkeypatch):
    """Shapes that hit the tensor-core tiling edge cases: K not a multiple of 32, N not a multiple
    of the N tile, N below 16 (falls back), several N tiles with concretisation partials. The launches here
    have few tiles, so the tensor cores are forced (VF_DENSE_KERNEL=tc)."""
    monkeypatch.setenv("VF_DENSE_KERNEL", "tc")
    rng = np.random.default_rng(11)
    net = synth.mlp([300, 196, 68, 260, 36, 12], rng)
    B = 3
    centres = rng.random((B, 300)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 12, B), 12)
    g, ora, out = run_both(net, centres, 0.02, C, both=True)
    assert_parity(net, centres, 0.02, C, g, ora, out, both=True)


def test_odd_mlp_given_alpha_and_chunking_is_bitwise_stable():
    rng = np.random.default_rng(7)
    net = synth.mlp([13, 37, 29, 33, 7], rng)
    B = 5
    centres = rng.random((B, 13)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 7, B), 7)
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    alphas = {relus[1]: rng.random((B, 29)) * 1.4 - 0.2}
    g, ora, out = run_both(net, centres, 0.08, C, alphas=alphas, both=True)
    assert_parity(net, centres, 0.08, C, g, ora, out, alphas=alphas, both=True)
    # a workspace so small that every pass runs in many row blocks: bitwise identical
    g2, _, out2 = run_both(net, centres, 0.08, C, alphas=alphas, both=True, workspace=300_000)
    for k in ("lb", "ub", "pre_lb", "pre_ub"):
        assert np.array_equal(out[k], out2[k]), k
    # repeated call on the same handle: bitwise identical
    a_dev = {k: _dev(v.astype(np.float32)) for k, v in alphas.items()}
    o3 = g.verify(_dev(centres), 0.08, _dev(C), alpha=a_dev, both_sides=True)
    assert np.array_equal(o3["lb"].cpu().numpy(), out["lb"])


def test_ibp_entry_point():
    w = synth.workload(3, B=4)
    g = vf.Net(w.net)
    lb, ub = g.ibp(_dev(w.centres), w.eps)
    torch.cuda.synchronize()
    ib = O.ibp(w.net, w.centres, w.eps)
    for v in range(len(w.net)):
        gl = g.node_block(lb, v, 4).cpu().numpy()
        gu = g.node_block(ub, v, 4).cpu().numpy()
        assert max_violation(gl, ib[0][v] - ib[1][v]) <= 1.0, v
        assert max_violation(gu, ib[0][v] + ib[1][v]) <= 1.0, v


def test_crown_backward_and_concretize_entry_points():
    w = synth.workload(2, B=6)
    g = vf.Net(w.net)
    cen = _dev(w.centres)
    lb, ub = g.ibp(cen, w.eps)
    last = len(w.net) - 1
    lam_in, cst = g.crown_backward(last, _dev(w.C), lb, ub, 6)
    lbc = vf.concretize(lam_in, cst, cen, w.eps)
    torch.cuda.synchronize()
    ib = O.ibp(w.net, w.centres, w.eps)
    for b in range(6):
        relax = {k: O.relax_params(ib[0][w.net[k].src][b] - ib[1][w.net[k].src][b],
                                   ib[0][w.net[k].src][b] + ib[1][w.net[k].src][b])
                 for k, nd in enumerate(w.net) if nd.op == "relu"}
        L, c = O.backward(w.net, last, w.C[b].astype(np.float64), relax)
        assert max_violation(lam_in[b].cpu().numpy(), L) <= 1.0
        assert max_violation(cst[b].cpu().numpy(), c) <= 1.0
        assert max_violation(lbc[b].cpu().numpy(), O.concretize(L, c, w.centres[b], w.eps)) <= 1.0


def test_concretize_ragged_sizes():
    rng = np.random.default_rng(3)
    for (B, R, n0) in [(1, 1, 1), (3, 5, 33), (2, 7, 1000)]:
        lam = rng.standard_normal((B, R, n0)).astype(np.float32)
        cst = rng.standard_normal((B, R)).astype(np.float32)
        c = rng.random((B, n0)).astype(np.float32)
        got = vf.concretize(_dev(lam), _dev(cst), _dev(c), 0.1).cpu().numpy()
        ref = np.stack([O.concretize(lam[b].astype(np.float64), cst[b], c[b], np.float32(0.1).item()) for b in range(B)])
        assert max_violation(got, ref) <= 1.0


def test_errors_are_codes_not_faults():
    w = synth.workload(1, B=4)
    g = vf.Net(w.net)
    bad = w.centres.copy()
    bad[1, 2] = np.nan
    with pytest.raises(vf.VfError) as e:
        g.verify(_dev(bad), w.eps, _dev(w.C))
    assert e.value.code == vf.VF_ERR_NONFINITE
    with pytest.raises(vf.VfError) as e:
        g.verify(_dev(w.centres), float("nan"), _dev(w.C))
    assert e.value.code == vf.VF_ERR_NONFINITE
    tiny = vf.Net(w.net, workspace_bytes=4096)
    with pytest.raises(vf.VfError) as e:
        tiny.verify(_dev(w.centres), w.eps, _dev(w.C))
    assert e.value.code == vf.VF_ERR_WORKSPACE
    # the handle still works after errors
    out = g.verify(_dev(w.centres), w.eps, _dev(w.C))
    torch.cuda.synchronize()
    assert torch.isfinite(out["lb"]).all()


def test_host_fault_injection(monkeypatch):
    w = synth.workload(2, B=3)
    monkeypatch.setenv("VF_TEST_FAIL_AT", "5")
    g = vf.Net(w.net)
    with pytest.raises(vf.VfError) as e:
        g.verify(_dev(w.centres), w.eps, _dev(w.C))
    assert e.value.code == vf.VF_ERR_CUDA and "injected" in str(e.value)
    monkeypatch.delenv("VF_TEST_FAIL_AT")
    g2 = vf.Net(w.net)
    out = g2.verify(_dev(w.centres), w.eps, _dev(w.C))
    vf.sync()
    assert torch.isfinite(out["lb"]).all()


def test_bounded_wait_expiry_is_reported_and_context_survives(monkeypatch):
    """A tensor-core launch whose copy is withheld (test hook) gives up its bounded wait after about
    two seconds of clock, frees its resources and raises the device flag: vf_net_check reports
    VF_ERR_TIMEOUT. The context stays usable: a fresh handle then matches the oracle."""
    w = synth.workload(2, B=4)
    monkeypatch.setenv("VF_DENSE_KERNEL", "tc")  # few tiles per launch: force the tensor-core kernel
    monkeypatch.setenv("VF_TEST_TC_STALL", "1")
    g = vf.Net(w.net)
    g.verify(_dev(w.centres), w.eps, _dev(w.C))
    torch.cuda.synchronize()
    with pytest.raises(vf.VfError) as e:
        g.check()
    assert e.value.code == vf.VF_ERR_TIMEOUT
    g.check()  # the flag was cleared by the first check
    monkeypatch.delenv("VF_TEST_TC_STALL")
    g2, ora, out = run_both(w.net, w.centres, w.eps, w.C)
    assert_parity(w.net, w.centres, w.eps, w.C, g2, ora, out)
