"""Seeded synthetic networks, input centres and specification matrices.

This module only draws numbers and lays out data: it holds none of the bound
propagation arithmetic, so the fp64 oracle (``oracle/``) and the CUDA path can
both be fed from it without sharing any method code.

The workloads mirror the kinds of models the page "Scaling Neural Network
Verification with Tensor Parallelism and Fully Sharded Data Parallelism"
(technical summary, §4.2 and §4.3) verifies -- wide MLPs, CNNs and a ResNet
on CIFAR-100 -- with MNIST-shaped (784) and CIFAR-shaped (3x32x32, 100
classes) inputs. Those models and datasets are not available here, so every
weight and input is drawn from a seeded generator:

* generator: numpy ``PCG64(1000 * config + stream)``; stream 0 = weights,
  1 = centres, 2 = labels;
* weights: He-normal, ``N(0, 2 / fan_in)`` with ``fan_in = C_in * k * k`` for
  convolutions and ``n_in`` for dense layers, drawn in fp64 and rounded to fp32;
  in the residual network every convolution inside a block (both 3x3 and the
  1x1 shortcut) is further scaled by ``1/sqrt(2)``;
* biases: ``N(0, 0.01^2)`` for every layer;
* centres: ``U[0, 1)`` per input coordinate;
* labels: uniform in ``0..K-1``; specification rows ``e_y - e_j`` for every
  ``j != y`` in increasing ``j``.

A network is a list of :class:`Node` in topological order (every ``src`` index
is smaller than the node's own index). Node 0 is the input. Activations are
flattened in C order (channel, row, column).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "Node", "Net", "Workload", "rng_for", "mlp", "cnn_cfg3", "resnet_cfg4",
    "margin_spec", "identity_spec", "workload", "node_shapes", "WORKLOAD_NAMES",
]

INPUT, DENSE, CONV, RELU, ADD = "input", "dense", "conv", "relu", "add"


@dataclasses.dataclass
class Node:
    op: str
    src: int = -1
    src2: int = -1
    W: Optional[np.ndarray] = None  # dense: [n_out, n_in]; conv: [C_out, C_in, k, k]
    b: Optional[np.ndarray] = None  # dense: [n_out]; conv: [C_out]
    stride: int = 1
    pad: int = 0
    shape: Tuple[int, ...] = ()  # input node only: (n,) or (C, H, W)


Net = List[Node]


def rng_for(config: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * config + stream))


def node_shapes(net: Sequence[Node]) -> List[Tuple[int, ...]]:
    """Output shape of every node (pure bookkeeping, no arithmetic on values)."""
    shapes: List[Tuple[int, ...]] = []
    for v, nd in enumerate(net):
        if nd.op == INPUT:
            shapes.append(tuple(nd.shape))
        elif nd.op == DENSE:
            shapes.append((nd.W.shape[0],))
        elif nd.op == CONV:
            c, h, w = shapes[nd.src]
            k = nd.W.shape[2]
            ho = (h + 2 * nd.pad - k) // nd.stride + 1
            wo = (w + 2 * nd.pad - k) // nd.stride + 1
            shapes.append((nd.W.shape[0], ho, wo))
        elif nd.op in (RELU,):
            shapes.append(shapes[nd.src])
        elif nd.op == ADD:
            assert shapes[nd.src] == shapes[nd.src2], (v, shapes[nd.src], shapes[nd.src2])
            shapes.append(shapes[nd.src])
        else:
            raise ValueError(nd.op)
    return shapes


def _he(rng, shape, fan_in, scale=1.0):
    std = math.sqrt(2.0 / fan_in) * scale
    return (rng.standard_normal(shape) * std).astype(np.float32)


def _bias(rng, n):
    return (rng.standard_normal(n) * 0.01).astype(np.float32)


def mlp(widths: Sequence[int], rng: np.random.Generator) -> Net:
    """ReLU MLP ``widths[0] - widths[1] - ... - widths[-1]`` (no ReLU on the output)."""
    net: Net = [Node(INPUT, shape=(widths[0],))]
    for i in range(len(widths) - 1):
        W = _he(rng, (widths[i + 1], widths[i]), widths[i])
        b = _bias(rng, widths[i + 1])
        net.append(Node(DENSE, src=len(net) - 1, W=W, b=b))
        if i + 1 < len(widths) - 1:
            net.append(Node(RELU, src=len(net) - 1))
    return net


def _conv(net, rng, src, c_in, c_out, k, stride, pad, scale=1.0):
    W = _he(rng, (c_out, c_in, k, k), c_in * k * k, scale)
    b = _bias(rng, c_out)
    net.append(Node(CONV, src=src, W=W, b=b, stride=stride, pad=pad))
    return len(net) - 1


def _dense(net, rng, src, n_in, n_out):
    net.append(Node(DENSE, src=src, W=_he(rng, (n_out, n_in), n_in), b=_bias(rng, n_out)))
    return len(net) - 1


def _relu(net, src):
    net.append(Node(RELU, src=src))
    return len(net) - 1


def cnn_cfg3(rng: np.random.Generator, image=(3, 32, 32), c1=16, c2=32, hidden=100, classes=10) -> Net:
    """conv c_in->c1 4x4 s2 p1, ReLU, conv c1->c2 4x4 s2 p1, ReLU, fc, ReLU, fc."""
    net: Net = [Node(INPUT, shape=tuple(image))]
    v = _relu(net, _conv(net, rng, 0, image[0], c1, 4, 2, 1))
    v = _relu(net, _conv(net, rng, v, c1, c2, 4, 2, 1))
    flat = c2 * (image[1] // 4) * (image[2] // 4)
    v = _relu(net, _dense(net, rng, v, flat, hidden))
    _dense(net, rng, v, hidden, classes)
    return net


def resnet_cfg4(rng: np.random.Generator, image=(3, 32, 32), widths=(16, 32, 64), fc=512,
                classes=100) -> Net:
    """Stem conv 3x3, then residual blocks (conv3x3(s) -> ReLU -> conv3x3(1)) + shortcut -> ReLU.

    Block ``i`` has ``widths[i]`` channels and stride 1 for the first block, 2 after;
    the shortcut is the identity when the shape is unchanged, else a 1x1 conv of
    the same stride. Padding 1 for the 3x3 convs, 0 for the 1x1. No batch norm.
    """
    s = 1.0 / math.sqrt(2.0)
    net: Net = [Node(INPUT, shape=tuple(image))]
    v = _relu(net, _conv(net, rng, 0, image[0], widths[0], 3, 1, 1))
    c_prev, hw = widths[0], image[1]
    for i, c in enumerate(widths):
        stride = 1 if i == 0 else 2
        x = v
        a = _relu(net, _conv(net, rng, x, c_prev, c, 3, stride, 1, s))
        bconv = _conv(net, rng, a, c, c, 3, 1, 1, s)
        if stride == 1 and c == c_prev:
            sc = x
        else:
            sc = _conv(net, rng, x, c_prev, c, 1, stride, 0, s)
        net.append(Node(ADD, src=bconv, src2=sc))
        v = _relu(net, len(net) - 1)
        c_prev, hw = c, hw // stride
    flat = c_prev * hw * (image[2] * hw // image[1])
    v = _relu(net, _dense(net, rng, v, flat, fc))
    _dense(net, rng, v, fc, classes)
    return net


def margin_spec(labels: np.ndarray, classes: int) -> np.ndarray:
    """Rows ``e_y - e_j`` for all ``j != y`` in increasing ``j``: shape [B, classes-1, classes]."""
    B = labels.shape[0]
    C = np.zeros((B, classes - 1, classes), np.float32)
    for bi, y in enumerate(labels):
        r = 0
        for j in range(classes):
            if j == y:
                continue
            C[bi, r, y] = 1.0
            C[bi, r, j] = -1.0
            r += 1
    return C


def identity_spec(n: int) -> np.ndarray:
    """C = I_n shared by all centres: shape [1, n, n]."""
    return np.eye(n, dtype=np.float32)[None]


@dataclasses.dataclass
class Workload:
    name: str
    net: Net
    centres: np.ndarray  # [B, n0] fp32
    eps: float  # fp32 value held in a Python float
    C: np.ndarray  # [B or 1, R, n_L] fp32
    labels: Optional[np.ndarray]
    crown_relus: Optional[List[int]]  # relu node ids whose pre-activation bounds use CROWN; None = all
    both_sides: bool


WORKLOAD_NAMES = {
    1: "mlp_8-32-32-4_B64",
    2: "mlp_784-256x3-10_B1024",
    3: "cnn_3x32x32_c16-c32-fc100-fc10_B256",
    4: "resnet_cifar100_16-32-64_fc512_B32",
    5: "mlp_3072-1024x8-100_B4096",
}


def _relu_ids(net):
    return [v for v, nd in enumerate(net) if nd.op == RELU]


def workload(config: int, B: Optional[int] = None, eps: Optional[float] = None) -> Workload:
    """The five benchmark workloads, fully determined by ``config`` (and an optional batch override).

    ``B`` smaller than the configured batch keeps the first ``B`` centres (and labels), so
    a subset is always a prefix of the full workload.
    """
    wr = rng_for(config, 0)
    cr = rng_for(config, 1)
    lr = rng_for(config, 2)
    if config == 1:
        net = mlp([8, 32, 32, 4], wr)
        Bf, e, classes = 64, 0.05, None
    elif config == 2:
        net = mlp([784, 256, 256, 256, 10], wr)
        Bf, e, classes = 1024, 2.0 / 255.0, 10
    elif config == 3:
        net = cnn_cfg3(wr)
        Bf, e, classes = 256, 2.0 / 255.0, 10
    elif config == 4:
        net = resnet_cfg4(wr)
        Bf, e, classes = 32, 1.0 / 255.0, 100
    elif config == 5:
        net = mlp([3072] + [1024] * 8 + [100], wr)
        Bf, e, classes = 4096, 1.0 / 255.0, 100
    else:
        raise ValueError(config)
    n0 = int(np.prod(net[0].shape))
    centres = cr.random((Bf, n0)).astype(np.float32)
    labels = None
    if classes is None:
        C = identity_spec(net[-1].W.shape[0])
    else:
        labels = lr.integers(0, classes, Bf)
        C = margin_spec(labels, classes)
    if B is not None:
        assert 0 < B <= Bf, (B, Bf)
        centres = centres[:B]
        if labels is not None:
            labels = labels[:B]
            C = C[:B]
    relus = _relu_ids(net)
    crown = relus[-2:] if config == 5 else None
    return Workload(name=WORKLOAD_NAMES[config], net=net, centres=np.ascontiguousarray(centres),
                    eps=float(np.float32(e if eps is None else eps)), C=np.ascontiguousarray(C),
                    labels=labels, crown_relus=crown, both_sides=(config == 1))
