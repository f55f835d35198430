"""Seeded random networks for the fuzz tests and the oracle's pins: plain and residual CNNs with random kernel
sizes, strides and paddings and a dense head, and dense ReLU chains of random widths. Inputs only: no bound
arithmetic lives here."""
from __future__ import annotations

import numpy as np

from linear_bound_propagation_b200 import synth


def _out_hw(h, k, s, p):
    return (h + 2 * p - k) // s + 1


def random_net(seed):
    """A random network of this library's node kinds; returns (net, input shape, classes)."""
    rng = np.random.default_rng(10_000 + seed)
    c, h = int(rng.integers(1, 4)), int(rng.integers(6, 13))
    net = [synth.Node(synth.INPUT, shape=(c, h, h))]
    v = 0
    for _ in range(int(rng.integers(1, 4))):
        if rng.random() < 0.35 and h >= 4:  # residual block: conv-relu-conv + shortcut, add, relu
            co = int(rng.integers(1, 5))
            s = int(rng.choice([1, 2]))
            ho = _out_hw(h, 3, s, 1)
            a = synth._relu(net, synth._conv(net, rng, v, c, co, 3, s, 1, 0.7))
            b = synth._conv(net, rng, a, co, co, 3, 1, 1, 0.7)
            sc = v if (s == 1 and co == c) else synth._conv(net, rng, v, c, co, 1, s, 0, 0.7)
            net.append(synth.Node(synth.ADD, src=b, src2=sc))
            v = synth._relu(net, len(net) - 1)
            c, h = co, ho
        else:
            k = int(rng.integers(1, min(5, h) + 1))
            s = int(rng.choice([1, 2, 2, 4])) if h > k else 1
            p = int(rng.integers(0, k))
            if _out_hw(h, k, s, p) < 1 or s * (_out_hw(h, k, s, p) - 1) > h - 1 + p:
                p = 0
            co = int(rng.integers(1, 6))
            v = synth._relu(net, synth._conv(net, rng, v, c, co, k, s, p))
            c, h = co, _out_hw(h, k, s, p)
    hidden, classes = int(rng.integers(3, 12)), int(rng.integers(2, 6))
    v = synth._relu(net, synth._dense(net, rng, v, c * h * h, hidden))
    synth._dense(net, rng, v, hidden, classes)
    return net, net[0].shape, classes


def random_mlp(seed):
    rng = np.random.default_rng(30_000 + seed)
    widths = [int(rng.choice([5, 8, 13, 32, 48, 64, 100]))]
    for _ in range(int(rng.integers(1, 5))):
        widths.append(int(rng.choice([4, 7, 16, 32, 36, 64, 96, 128])))
    widths.append(int(rng.integers(2, 8)))
    return synth.mlp(widths, rng), widths
