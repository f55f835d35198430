"""GPU parity of the tensor-core convolution step against the fp64 oracle, through the C ABI. Two kernels do it,
both tcgen05 implicit GEMMs with the 3xTF32 split: conv_back_tc (tap shifts, the default) and conv_back_tcn (taps
in the N dimension, chosen with VF_CONV_TC=tapn where its shapes allow; measured slower, kept tested).

The kernel takes every convolution back-substitution whose input has a multiple of 16 channels (up to 128) or,
at stride 1, fewer than 16 (a 3-channel stem, padded to 16 with zero weights),
kernel size up to 8 and stride 1 or 2: whole-map rows, receptive-field windows, stored, accumulated (residual
adds) and concretised against the input box (a convolution fed by a 16-channel input). The networks below
are chosen so that each of those cases runs (1x1 stride-2 shortcuts leave whole stride classes empty; a 5x5
stride-1 convolution has a gap of four lines and columns around each row's slab), at sizes the oracle
finishes in seconds, with windows and unstable-neuron compaction on and off.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import max_violation
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _resnet(seed=61, B=2):
    rng = np.random.default_rng(seed)
    net = synth.resnet_cfg4(rng, image=(16, 8, 8), widths=(16, 32, 64), fc=24, classes=5)
    centres = rng.random((B, 16 * 8 * 8)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, B), 5)
    return net, centres, C, float(np.float32(0.004))


def _mixed(seed=63, B=2):
    """5x5 stride-1 and 3x3 stride-2 convolutions on 16 and 16 input channels, then a dense head."""
    rng = np.random.default_rng(seed)
    net = [synth.Node(synth.INPUT, shape=(16, 12, 12))]
    v = synth._relu(net, synth._conv(net, rng, 0, 16, 16, 5, 1, 2))
    v = synth._relu(net, synth._conv(net, rng, v, 16, 32, 3, 2, 1))
    v = synth._relu(net, synth._dense(net, rng, v, 32 * 6 * 6, 12))
    synth._dense(net, rng, v, 12, 4)
    centres = rng.random((B, 16 * 12 * 12)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 4, B), 4)
    return net, centres, C, float(np.float32(0.003))


def _cnn(seed=62, B=2):
    rng = np.random.default_rng(seed)
    net = synth.cnn_cfg3(rng, image=(16, 16, 16), c1=16, c2=32, hidden=20, classes=5)
    centres = rng.random((B, 16 * 16 * 16)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, B), 5)
    return net, centres, C, float(np.float32(0.004))


def _stem_cnn(seed=64, B=2):
    """A 3-channel input whose 4x4 stride-2 stem stays on the FFMA kernels (the rest on the tensor cores)."""
    rng = np.random.default_rng(seed)
    net = synth.cnn_cfg3(rng, image=(3, 16, 16), c1=16, c2=32, hidden=20, classes=5)
    centres = rng.random((B, 3 * 16 * 16)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, B), 5)
    return net, centres, C, float(np.float32(0.004))


def _stem_resnet(seed=65, B=2):
    """A 3-channel 3x3 stride-1 stem before residual blocks of 16, 32 and 64 channels."""
    rng = np.random.default_rng(seed)
    net = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(16, 32, 64), fc=24, classes=5)
    centres = rng.random((B, 3 * 8 * 8)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, B), 5)
    return net, centres, C, float(np.float32(0.004))


CASES = {"resnet16-32-64": _resnet, "conv5x5-conv3x3s2": _mixed, "cnn16-32-k4s2": _cnn, "stem3-cnn": _stem_cnn,
         "stem3-resnet": _stem_resnet}


def _run(net, centres, eps, C, both=True, workspace=0):
    g = vf.Net(net, workspace_bytes=workspace)
    g.profile(True)
    g.profile_read(reset=True)
    out = g.verify(_dev(centres), eps, _dev(C), both_sides=both, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    tc = g.profile_read(kind=vf.VF_KERNEL_CONV_TC, reset=False)[0] + g.profile_read(kind=vf.VF_KERNEL_CONV_TC_PAD)[0]
    return g, {k: v.cpu().numpy() for k, v in out.items()}, tc


@pytest.mark.parametrize("kernel", ["1", "tapn"])
@pytest.mark.parametrize("compact", ["1", "0"])
@pytest.mark.parametrize("windows", ["1", "0"])
@pytest.mark.parametrize("case", list(CASES))
def test_conv_tc_matches_oracle(monkeypatch, case, windows, compact, kernel):
    monkeypatch.setenv("VF_CONV_WINDOWS", windows)
    monkeypatch.setenv("VF_COMPACT", compact)
    monkeypatch.setenv("VF_CONV_TC", kernel)
    net, centres, C, eps = CASES[case]()
    ora = O.verify(net, centres, eps, C, both_sides=True)
    g, out, tc = _run(net, centres, eps, C)
    assert tc > 0, "the tensor-core convolution did not run"
    assert_parity(net, centres, eps, C, g, ora, out, both=True)


@pytest.mark.parametrize("kernel", ["1", "tapn"])
@pytest.mark.parametrize("case", list(CASES))
def test_conv_tc_row_blocks_are_bitwise_stable(monkeypatch, case, kernel):
    """Each row's arithmetic depends only on its own window: the same bounds, bit for bit, when a pass is
    cut into many small row blocks (a small workspace), i.e. when rows share tensor-core groups with other
    rows and sit at other places in them."""
    monkeypatch.setenv("VF_CONV_TC", kernel)
    net, centres, C, eps = CASES[case]()
    _, a, _ = _run(net, centres, eps, C)
    _, b, _ = _run(net, centres, eps, C, workspace=6 << 20)
    for k in ("lb", "ub", "pre_lb", "pre_ub"):
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("config,B", [(3, 6), (4, 1)])
def test_conv_tc_and_ffma_agree_on_workloads(monkeypatch, config, B):
    """The CNN and residual workloads with the tensor-core convolution on and off: the same bounds within the
    parity tolerance, and the oracle's on the centres it finishes quickly."""
    w = synth.workload(config, B=B)
    res = {}
    for on in ("1", "tapn", "0"):
        monkeypatch.setenv("VF_CONV_TC", on)
        _, out, tc = _run(w.net, w.centres, w.eps, w.C, both=False)
        assert (tc > 0) == (on != "0")
        res[on] = out
    for on in ("1", "tapn"):
        assert max_violation(res[on]["lb"], res["0"]["lb"]) <= 1.0
        assert max_violation(res[on]["pre_lb"], res["0"]["pre_lb"]) <= 1.0
        assert max_violation(res[on]["pre_ub"], res["0"]["pre_ub"]) <= 1.0
    if config == 3:
        ora = O.verify(w.net, w.centres[:2], w.eps, w.C[:2])
        assert max_violation(res["1"]["lb"][:2], ora.lb) <= 1.0
