"""Thin ctypes binding of libvf.so (include/vf.h): argument marshalling only.

Every step of the bound computation runs in the CUDA library; this module only passes
device pointers (``tensor.data_ptr()``), sizes and the current CUDA stream. PyTorch is
used for device memory and streams. If the library is missing the first call raises --
there is no other implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvf.so")

VF_OK, VF_ERR_ARG, VF_ERR_SHAPE, VF_ERR_WORKSPACE, VF_ERR_NONFINITE, VF_ERR_CUDA, VF_ERR_TIMEOUT, \
    VF_ERR_UNSUPPORTED = range(8)
VF_INPUT, VF_DENSE, VF_CONV2D, VF_RELU, VF_ADD = range(5)
(VF_KERNEL_ALL, VF_KERNEL_DENSE_TC, VF_KERNEL_DENSE_FFMA, VF_KERNEL_CONV, VF_KERNEL_CONV_WIN, VF_KERNEL_CONV_TC,
 VF_KERNEL_DENSE_FWD_TC, VF_KERNEL_CONV_TC_PAD) = range(8)

SYMBOLS = ["vf_net_create", "vf_net_destroy", "vf_net_node_size", "vf_net_total_size", "vf_ibp",
           "vf_crown_backward", "vf_concretize", "vf_verify_batch", "vf_sync", "vf_last_error",
           "vf_profile_enable", "vf_profile_read", "vf_launch_count", "vf_net_check",
           "vf_concretize_dense_noalloc", "vf_alpha_crown", "vf_alpha_grad", "vf_alpha_beta_grad",
           "vf_net_node_info", "vf_bab_verify", "vf_bab_search", "vf_abi_layout"]
NOALLOC_SCRATCH_FLOATS = 1 << 22


class VfError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"vf error {code}: {msg}")
        self.code = code


class NodeDesc(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int), ("src", ctypes.c_int), ("src2", ctypes.c_int),
                ("c", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int),
                ("n_out", ctypes.c_int), ("k", ctypes.c_int), ("stride", ctypes.c_int), ("pad", ctypes.c_int),
                ("W", ctypes.c_void_p), ("b", ctypes.c_void_p)]


class Opts(ctypes.Structure):
    _fields_ = [("relu_crown", ctypes.POINTER(ctypes.c_int)), ("alpha", ctypes.POINTER(ctypes.c_void_p)),
                ("both_sides", ctypes.c_int), ("skip_finite_check", ctypes.c_int),
                ("pre_lb", ctypes.c_void_p), ("pre_ub", ctypes.c_void_p), ("no_host_sync", ctypes.c_int),
                ("split", ctypes.POINTER(ctypes.c_void_p)), ("sound", ctypes.c_int),
                ("alpha_inter_iters", ctypes.c_int), ("alpha_inter_lr", ctypes.c_float),
                ("alpha_rows_init", ctypes.c_void_p), ("beta_rows_init", ctypes.c_void_p),
                ("beta_rows_out", ctypes.c_void_p)]


class BabOpts(ctypes.Structure):
    _fields_ = [("max_domains", ctypes.c_int), ("batch", ctypes.c_int), ("alpha_iters", ctypes.c_int),
                ("lr", ctypes.c_float), ("relu_crown", ctypes.POINTER(ctypes.c_int)),
                ("trace", ctypes.POINTER(ctypes.c_int)), ("trace_cap", ctypes.c_int),
                ("alpha_inter_iters", ctypes.c_int), ("alpha_inter_lr", ctypes.c_float), ("cold_start", ctypes.c_int)]


class BabResult(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int), ("domains", ctypes.c_longlong), ("rounds", ctypes.c_int),
                ("max_depth", ctypes.c_int), ("lb", ctypes.c_float)]


BAB_STATUS = {1: "verified", -1: "falsified", 0: "unknown"}
BOUND_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_byte),
                            ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libvf.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m linear_bound_propagation_b200._build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    L.vf_net_create.argtypes = [ctypes.POINTER(NodeDesc), I, ctypes.c_size_t, ctypes.POINTER(P)]
    L.vf_net_destroy.argtypes = [P]
    L.vf_net_destroy.restype = None
    L.vf_net_node_size.argtypes = [P, I]
    L.vf_net_total_size.argtypes = [P]
    L.vf_net_total_size.restype = LL
    L.vf_ibp.argtypes = [P, P, I, F, P, P, P]
    L.vf_crown_backward.argtypes = [P, I, P, I, LL, P, P, ctypes.POINTER(P), I, P, P, P]
    L.vf_concretize.argtypes = [P, P, P, F, I, I, I, P, P]
    L.vf_verify_batch.argtypes = [P, P, I, F, P, I, LL, ctypes.POINTER(Opts), P, P, P, P, P]
    L.vf_sync.argtypes = [P]
    L.vf_last_error.restype = ctypes.c_char_p
    L.vf_profile_enable.argtypes = [P, I]
    L.vf_profile_read.argtypes = [P, I, ctypes.POINTER(LL), ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_double), I]
    L.vf_net_check.argtypes = [P]
    L.vf_concretize_dense_noalloc.argtypes = [P, LL, I, P, P, P, F, I, I, I, P, P]
    L.vf_alpha_crown.argtypes = [P, P, I, F, P, I, LL, ctypes.POINTER(Opts), I, F, P, P, P, P]
    L.vf_alpha_grad.argtypes = [P, P, I, F, P, I, LL, ctypes.POINTER(Opts), P, P, P, P]
    L.vf_alpha_beta_grad.argtypes = [P, P, I, F, P, I, LL, ctypes.POINTER(Opts), P, P, P, P, P, P]
    L.vf_net_node_info.argtypes = [P, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(LL)]
    L.vf_bab_verify.argtypes = [P, P, F, P, I, ctypes.POINTER(BabOpts), ctypes.POINTER(BabResult), P]
    L.vf_bab_search.argtypes = [BOUND_FN, P, I, I, ctypes.POINTER(BabResult)]
    L.vf_launch_count.argtypes = [P]
    L.vf_launch_count.restype = LL
    _lib = L
    return L


def _check(code):
    if code != VF_OK:
        raise VfError(code, lib().vf_last_error().decode())


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


class Net:
    """A network handle on the current CUDA device (vf_net_create / vf_net_destroy)."""

    def __init__(self, nodes: Sequence, workspace_bytes: int = 0):
        L = lib()
        descs = (NodeDesc * len(nodes))()
        keep = []
        for v, nd in enumerate(nodes):
            d = descs[v]
            d.src, d.src2 = -1, -1
            if nd.op == "input":
                d.op = VF_INPUT
                shp = tuple(nd.shape)
                d.c, d.h, d.w = (shp + (1, 1))[:3] if len(shp) == 1 else shp
            elif nd.op in ("dense", "conv"):
                W = np.ascontiguousarray(nd.W, np.float32)
                b = np.ascontiguousarray(nd.b, np.float32)
                keep += [W, b]
                d.op = VF_DENSE if nd.op == "dense" else VF_CONV2D
                d.src = nd.src
                d.n_out = W.shape[0]
                if nd.op == "conv":
                    d.k, d.stride, d.pad = W.shape[2], nd.stride, nd.pad
                d.W = W.ctypes.data
                d.b = b.ctypes.data
            elif nd.op == "relu":
                d.op, d.src = VF_RELU, nd.src
            elif nd.op == "add":
                d.op, d.src, d.src2 = VF_ADD, nd.src, nd.src2
            else:
                raise ValueError(nd.op)
        h = ctypes.c_void_p()
        _check(L.vf_net_create(descs, len(nodes), workspace_bytes, ctypes.byref(h)))
        self.h = h
        self.n_nodes = len(nodes)
        self.sizes = [L.vf_net_node_size(h, v) for v in range(len(nodes))]
        self.total = L.vf_net_total_size(h)
        self.relu_ids = [v for v, nd in enumerate(nodes) if nd.op == "relu"]

    def close(self):
        if getattr(self, "h", None):
            lib().vf_net_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def offset(self, v: int, B: int) -> int:
        return B * sum(self.sizes[:v])

    # --------------------------------------------------------------------- entry points
    def ibp(self, centres: torch.Tensor, eps: float, stream=None):
        B = centres.shape[0]
        lb = torch.empty(B * self.total, device=centres.device, dtype=torch.float32)
        ub = torch.empty_like(lb)
        _check(lib().vf_ibp(self.h, _ptr(centres), B, float(eps), _ptr(lb), _ptr(ub), _stream_ptr(stream)))
        return lb, ub

    def node_block(self, flat: torch.Tensor, v: int, B: int) -> torch.Tensor:
        o = self.offset(v, B)
        return flat[o:o + B * self.sizes[v]].view(B, self.sizes[v])

    def crown_backward(self, start_node: int, lambda0: torch.Tensor, lb_all, ub_all, B: int,
                       alpha: Optional[Dict[int, torch.Tensor]] = None, stream=None):
        R = lambda0.shape[-2]
        bstride = 0 if lambda0.dim() == 2 or lambda0.shape[0] == 1 else R * lambda0.shape[-1]
        lam_in = torch.empty(B, R, self.sizes[0], device=lambda0.device, dtype=torch.float32)
        cst = torch.empty(B, R, device=lambda0.device, dtype=torch.float32)
        arr = self._alpha_array(alpha)
        _check(lib().vf_crown_backward(self.h, start_node, _ptr(lambda0), R, bstride, _ptr(lb_all), _ptr(ub_all),
                                       arr, B, _ptr(lam_in), _ptr(cst), _stream_ptr(stream)))
        return lam_in, cst

    def _alpha_array(self, alpha):
        if not alpha:
            return None
        arr = (ctypes.c_void_p * self.n_nodes)()
        for v, a in alpha.items():
            arr[v] = a.data_ptr()
        return arr

    def verify(self, centres: torch.Tensor, eps: float, C: torch.Tensor, crown_relus: Optional[Sequence[int]] = None,
               alpha: Optional[Dict[int, torch.Tensor]] = None, both_sides: bool = False, want_pre: bool = False,
               skip_finite_check: bool = False, no_host_sync: bool = False, stream=None, out=None,
               splits: Optional[Dict[int, torch.Tensor]] = None, sound: bool = False, alpha_inter_iters: int = 0,
               alpha_inter_lr: float = 0.1):
        """vf_verify_batch. C: [B or 1, R, n_L]. splits: ReLU node -> int8 [B, n] signs (+1: z >= 0,
        -1: z <= 0, 0: free), one subdomain per centre row. sound: bounds that hold despite fp32 rounding.
        alpha_inter_iters > 0: alpha-CROWN for the intermediate bounds (vf_opts). Returns dict of device tensors."""
        B = centres.shape[0]
        R = C.shape[1]
        dev = centres.device
        bstride = 0 if C.shape[0] == 1 else R * C.shape[2]
        if out is None:
            out = {"lb": torch.empty(B, R, device=dev), "lb_ibp": torch.empty(B, R, device=dev),
                   "verified": torch.empty(B, R, device=dev, dtype=torch.uint8)}
            if both_sides:
                out["ub"] = torch.empty(B, R, device=dev)
            if want_pre:
                out["pre_lb"] = torch.empty(B * self.total, device=dev)
                out["pre_ub"] = torch.empty(B * self.total, device=dev)
        o = Opts()
        keep = []
        if crown_relus is not None:
            flags = (ctypes.c_int * self.n_nodes)()
            for v in crown_relus:
                flags[v] = 1
            o.relu_crown = ctypes.cast(flags, ctypes.POINTER(ctypes.c_int))
            keep.append(flags)
        arr = self._alpha_array(alpha)
        if arr is not None:
            o.alpha = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
            keep.append(arr)
        o.both_sides = 1 if both_sides else 0
        o.skip_finite_check = 1 if skip_finite_check else 0
        o.no_host_sync = 1 if no_host_sync else 0
        o.sound = 1 if sound else 0
        o.alpha_inter_iters = int(alpha_inter_iters)
        o.alpha_inter_lr = float(alpha_inter_lr)
        sarr = self._split_array(splits)
        if sarr is not None:
            o.split = ctypes.cast(sarr, ctypes.POINTER(ctypes.c_void_p))
            keep.append(sarr)
        o.pre_lb = out["pre_lb"].data_ptr() if "pre_lb" in out else None
        o.pre_ub = out["pre_ub"].data_ptr() if "pre_ub" in out else None
        _check(lib().vf_verify_batch(self.h, _ptr(centres), B, float(eps), _ptr(C), R, bstride, ctypes.byref(o),
                                     _ptr(out["lb"]), _ptr(out.get("ub")), _ptr(out.get("lb_ibp")),
                                     _ptr(out.get("verified")), _stream_ptr(stream)))
        return out

    def _split_array(self, splits):
        if not splits:
            return None
        arr = (ctypes.c_void_p * self.n_nodes)()
        for v, sg in splits.items():
            assert sg.dtype == torch.int8 and sg.is_cuda and sg.is_contiguous(), "splits: contiguous CUDA int8"
            arr[v] = sg.data_ptr()
        return arr

    def _opts(self, crown_relus=None, splits=None, alpha_inter_iters=0, alpha_inter_lr=0.1):
        o = Opts()
        o.alpha_inter_iters = int(alpha_inter_iters)
        o.alpha_inter_lr = float(alpha_inter_lr)
        keep = []
        if crown_relus is not None:
            flags = (ctypes.c_int * self.n_nodes)()
            for v in crown_relus:
                flags[v] = 1
            o.relu_crown = ctypes.cast(flags, ctypes.POINTER(ctypes.c_int))
            keep.append(flags)
        sarr = self._split_array(splits)
        if sarr is not None:
            o.split = ctypes.cast(sarr, ctypes.POINTER(ctypes.c_void_p))
            keep.append(sarr)
        return o, keep

    def alpha_size(self, B: int, R: int) -> int:
        """Length of a per-row slope array: one [B, R, n_v] block per ReLU node v in node order."""
        return B * R * sum(self.sizes[v] for v in self.relu_ids)

    def alpha_crown(self, centres: torch.Tensor, eps: float, C: torch.Tensor, iters: int = 20, lr: float = 0.1,
                    crown_relus=None, want_alpha: bool = False, stream=None, splits=None, alpha_inter_iters: int = 0,
                    alpha_inter_lr: float = 0.1, alpha_init: Optional[torch.Tensor] = None,
                    beta_init: Optional[torch.Tensor] = None, want_beta: bool = False):
        """vf_alpha_crown: returns dict(lb=best bound [B, R], lb_start=[B, R], alpha=final slopes or None,
        beta=final split multipliers or None). With splits (see verify) the split multipliers beta are optimised
        with the slopes; alpha_inter_iters > 0 optimises the intermediate bounds first; alpha_init / beta_init
        (alpha_size(B, R) floats, device) are start states (a negative slope entry: the adaptive slope)."""
        B, R = centres.shape[0], C.shape[1]
        bstride = 0 if C.shape[0] == 1 else R * C.shape[2]
        lb = torch.empty(B, R, device=centres.device)
        lb0 = torch.empty(B, R, device=centres.device)
        al = torch.empty(self.alpha_size(B, R), device=centres.device) if want_alpha else None
        be = torch.empty(self.alpha_size(B, R), device=centres.device) if want_beta else None
        o, keep = self._opts(crown_relus, splits, alpha_inter_iters, alpha_inter_lr)
        for t in (alpha_init, beta_init):
            if t is not None:
                assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and t.numel() == self.alpha_size(B, R)
        o.alpha_rows_init = alpha_init.data_ptr() if alpha_init is not None else None
        o.beta_rows_init = beta_init.data_ptr() if beta_init is not None else None
        o.beta_rows_out = be.data_ptr() if be is not None else None
        _check(lib().vf_alpha_crown(self.h, _ptr(centres), B, float(eps), _ptr(C), R, bstride, ctypes.byref(o), iters,
                                    float(lr), _ptr(lb), _ptr(lb0), _ptr(al), _stream_ptr(stream)))
        return {"lb": lb, "lb_start": lb0, "alpha": al, "beta": be}

    def alpha_grad(self, centres: torch.Tensor, eps: float, C: torch.Tensor, alpha: torch.Tensor, crown_relus=None,
                   stream=None):
        """vf_alpha_grad: (lb [B, R], grad with alpha's layout) at the given per-row slopes."""
        B, R = centres.shape[0], C.shape[1]
        bstride = 0 if C.shape[0] == 1 else R * C.shape[2]
        lb = torch.empty(B, R, device=centres.device)
        grad = torch.empty_like(alpha)
        o, keep = self._opts(crown_relus)
        _check(lib().vf_alpha_grad(self.h, _ptr(centres), B, float(eps), _ptr(C), R, bstride, ctypes.byref(o),
                                   _ptr(alpha), _ptr(lb), _ptr(grad), _stream_ptr(stream)))
        return lb, grad

    def alpha_beta_grad(self, centres: torch.Tensor, eps: float, C: torch.Tensor, alpha: torch.Tensor,
                        beta: Optional[torch.Tensor], splits, crown_relus=None, stream=None):
        """vf_alpha_beta_grad: (lb [B, R], d lb / d alpha, d lb / d beta) at the given slopes and split
        multipliers (both in alpha's layout)."""
        B, R = centres.shape[0], C.shape[1]
        bstride = 0 if C.shape[0] == 1 else R * C.shape[2]
        lb = torch.empty(B, R, device=centres.device)
        ga = torch.empty_like(alpha)
        gb = torch.empty_like(alpha)
        o, keep = self._opts(crown_relus, splits)
        _check(lib().vf_alpha_beta_grad(self.h, _ptr(centres), B, float(eps), _ptr(C), R, bstride, ctypes.byref(o),
                                        _ptr(alpha), _ptr(beta), _ptr(lb), _ptr(ga), _ptr(gb), _stream_ptr(stream)))
        return lb, ga, gb

    def bab(self, centre: torch.Tensor, eps: float, C: torch.Tensor, max_domains: int = 1000, batch: int = 16,
            alpha_iters: int = 20, lr: float = 0.1, crown_relus=None, stream=None, trace: bool = False,
            alpha_inter_iters: int = 0, alpha_inter_lr: float = 0.1, warm_start: bool = True):
        """vf_bab_verify on one box: centre [n0], C [R, n_L] (device). Returns dict(status, domains, rounds,
        max_depth, lb), plus, with trace, the branching neuron of every bounded subdomain in the order bounded
        (search-wide index, -1 if none). alpha_inter_iters > 0: intermediate bounds of every subdomain by
        alpha-CROWN with the split multipliers (vf_opts). warm_start: children start their ascent from the
        parent's last slopes and multipliers."""
        o = BabOpts(max_domains=max_domains, batch=batch, alpha_iters=alpha_iters, lr=float(lr),
                    alpha_inter_iters=int(alpha_inter_iters), alpha_inter_lr=float(alpha_inter_lr),
                    cold_start=0 if warm_start else 1)
        tbuf = None
        if trace:
            tbuf = (ctypes.c_int * max_domains)()
            o.trace = ctypes.cast(tbuf, ctypes.POINTER(ctypes.c_int))
            o.trace_cap = max_domains
        keep = None
        if crown_relus is not None:
            keep = (ctypes.c_int * self.n_nodes)()
            for v in crown_relus:
                keep[v] = 1
            o.relu_crown = ctypes.cast(keep, ctypes.POINTER(ctypes.c_int))
        r = BabResult()
        C2 = C.reshape(-1, C.shape[-1]).contiguous()
        _check(lib().vf_bab_verify(self.h, _ptr(centre.contiguous()), float(eps), _ptr(C2), C2.shape[0],
                                   ctypes.byref(o), ctypes.byref(r), _stream_ptr(stream)))
        out = {"status": BAB_STATUS[r.status], "domains": r.domains, "rounds": r.rounds, "max_depth": r.max_depth,
               "lb": r.lb}
        if trace:
            out["trace"] = [tbuf[i] for i in range(min(r.domains, max_domains))]
        return out

    def profile(self, enable: bool):
        _check(lib().vf_profile_enable(self.h, 1 if enable else 0))

    def profile_read(self, kind: int = 0, reset: bool = True):
        """(launches, total device ms, algorithmic flops) of one contraction kind since the last reset:
        0 all, 1 dense tensor-core (3xTF32), 2 dense FFMA, 3 whole-map convolution, 4 windowed convolution,
        5 tensor-core convolution (3xTF32, whole maps and windows), 6 dense tensor-core forward product,
        7 tensor-core convolution of a stem with its channels padded to 16."""
        n = ctypes.c_longlong()
        ms = ctypes.c_double()
        fl = ctypes.c_double()
        _check(lib().vf_profile_read(self.h, kind, ctypes.byref(n), ctypes.byref(ms), ctypes.byref(fl),
                                     1 if reset else 0))
        return n.value, ms.value, fl.value

    def check(self):
        """Synchronise and raise if a kernel of this handle gave up a bounded wait."""
        _check(lib().vf_net_check(self.h))

    def launch_count(self) -> int:
        return lib().vf_launch_count(self.h)


class VerifyGraph:
    """One vf_verify_batch call captured in a CUDA graph and replayed.

    Shapes, eps, options and the device buffers are fixed at capture: write the next batch into
    ``self.centres`` / ``self.C`` in place, call ``replay()`` and read ``self.out``. The captured call
    never synchronises its stream (``no_host_sync``: no NaN/Inf scan, no unstable-neuron compaction),
    which leaves the bounds unchanged. It uses the handle's workspace, so no other call on the same
    handle may run while a replay is in flight.
    """

    def __init__(self, net: Net, centres: torch.Tensor, eps: float, C: torch.Tensor,
                 crown_relus: Optional[Sequence[int]] = None, both_sides: bool = False):
        self.net = net
        self.centres = centres.clone()
        self.C = C.clone()
        kw = dict(crown_relus=crown_relus, both_sides=both_sides, no_host_sync=True)
        side = torch.cuda.Stream(device=centres.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # warm-up outside the capture: host caches, kernel attributes
            self.out = net.verify(self.centres, eps, self.C, **kw)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize(centres.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, capture_error_mode="relaxed"):
            net.verify(self.centres, eps, self.C, out=self.out, **kw)

    def replay(self):
        self.graph.replay()
        return self.out


def concretize(lam: torch.Tensor, cst: Optional[torch.Tensor], centres: torch.Tensor, eps: float, stream=None):
    B, R, n0 = lam.shape
    lb = torch.empty(B, R, device=lam.device)
    _check(lib().vf_concretize(_ptr(lam), _ptr(cst), _ptr(centres), float(eps), B, R, n0, _ptr(lb),
                               _stream_ptr(stream)))
    return lb


def concretize_dense_noalloc(lam: torch.Tensor, W: torch.Tensor, b: torch.Tensor, centres: torch.Tensor, eps: float,
                             out: Optional[torch.Tensor] = None, stream=None):
    """vf_concretize_dense_noalloc: rows lam [B or 1, R, n_out] over z = W x + b, x in centres +/- eps.
    The library allocates nothing for this call (its scratch is a fixed device array); `out` may be
    passed to keep the call free of any allocation on the Python side too."""
    for name, t in (("lam", lam), ("W", W), ("b", b), ("centres", centres)):
        if t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32, got {t.dtype}")
    if W.dim() != 2 or centres.dim() != 2 or lam.dim() not in (2, 3):
        raise ValueError("W [n_out, n_in], centres [B, n_in] and lam [B or 1, R, n_out] (or [R, n_out]) expected")
    B = centres.shape[0]
    R = lam.shape[-2]
    n_out, n_in = W.shape
    if centres.shape[1] != n_in or lam.shape[-1] != n_out or b.numel() != n_out:
        raise ValueError(f"shapes do not match W [{n_out}, {n_in}]: centres {tuple(centres.shape)}, "
                         f"lam {tuple(lam.shape)}, b {tuple(b.shape)}")
    if lam.dim() == 3 and lam.shape[0] not in (1, B):
        raise ValueError(f"lam has {lam.shape[0]} centre blocks for {B} centres")
    bstride = 0 if lam.dim() == 2 or lam.shape[0] == 1 else R * n_out
    if out is None:
        out = torch.empty(B, R, device=centres.device)
    elif out.dtype != torch.float32 or tuple(out.shape) != (B, R):
        raise ValueError(f"out must be float32 [{B}, {R}], got {out.dtype} {tuple(out.shape)}")
    _check(lib().vf_concretize_dense_noalloc(_ptr(lam), bstride, R, _ptr(W), _ptr(b), _ptr(centres), float(eps), B,
                                             n_in, n_out, _ptr(out), _stream_ptr(stream)))
    return out


def bab_search(evaluate, max_domains: int, batch: int):
    """vf_bab_search with a Python bound function: evaluate(list of subdomains, each a dict neuron -> sign in
    the order its splits were made) -> one (lowest row bound, holds no input, neuron to split next or None)
    per subdomain. Returns dict(status, domains, rounds, max_depth, lb). Runs on the host."""
    err = []

    def cb(user, n, off, cnt, nid, sg, lb, branch, empty):
        try:
            doms = [{nid[off[i] + k]: sg[off[i] + k] for k in range(cnt[i])} for i in range(n)]
            for i, (l, e, b) in enumerate(evaluate(doms)):
                lb[i] = l
                branch[i] = -1 if b is None else int(b)
                empty[i] = 1 if e else 0
            return VF_OK
        except Exception as ex:  # reported after the call returns
            err.append(ex)
            return VF_ERR_ARG

    fn = BOUND_FN(cb)
    r = BabResult()
    code = lib().vf_bab_search(fn, None, max_domains, batch, ctypes.byref(r))
    if err:
        raise err[0]
    _check(code)
    return {"status": BAB_STATUS[r.status], "domains": r.domains, "rounds": r.rounds, "max_depth": r.max_depth,
            "lb": r.lb}


def sync(stream=None):
    _check(lib().vf_sync(_stream_ptr(stream)))


def verify_host(net: Net, centres_host: torch.Tensor, eps: float, C_host: torch.Tensor, **kw):
    """End-to-end call with host inputs: copies centres and C to the device (from pinned host
    memory when given), runs vf_verify_batch, and copies lb and verified back to the host."""
    dev = torch.device("cuda")
    centres = centres_host.to(dev, non_blocking=True)
    C = C_host.to(dev, non_blocking=True)
    out = net.verify(centres, eps, C, **kw)
    return {k: v.to("cpu") for k, v in out.items() if k in ("lb", "ub", "verified")}
