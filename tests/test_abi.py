"""The C ABI library loads on a machine without a GPU and exports every entry point that
include/vf.h declares (no compute calls here)."""
import ctypes
import os
import re
import subprocess

from linear_bound_propagation_b200 import _build, vf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "vf.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vf_[a-z_0-9]+)\s*\(", text)))


def test_library_builds_and_loads():
    path = _build.build()
    assert os.path.exists(path)
    ctypes.CDLL(path)


def test_every_declared_symbol_is_exported():
    path = _build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (vf_\w+)$", out, flags=re.M))
    decl = declared_symbols()
    assert decl, "no declarations parsed"
    missing = [s for s in decl if s not in exported]
    assert not missing, missing
    assert set(vf.SYMBOLS) <= set(decl)
    L = vf.lib()
    for s in decl:
        assert hasattr(L, s)


def test_last_error_without_gpu_call():
    L = vf.lib()
    assert isinstance(L.vf_last_error(), bytes)


def test_new_entry_points_reject_null_arguments_without_a_gpu():
    """Branch and bound, the split multipliers' gradient and the node query validate their arguments on the
    host before any device work: a NULL handle or missing option block is an error code, not a crash."""
    L = vf.lib()
    res = vf.BabResult()
    o = vf.BabOpts(max_domains=10, batch=4, alpha_iters=0, lr=0.1)
    assert L.vf_bab_verify(None, None, 0.1, None, 1, vf.ctypes.byref(o), vf.ctypes.byref(res), None) == vf.VF_ERR_ARG
    assert b"NULL" in L.vf_last_error()
    assert L.vf_alpha_beta_grad(None, None, 1, 0.1, None, 1, 0, None, None, None, None, None, None, None) == vf.VF_ERR_ARG
    op = vf.ctypes.c_int()
    assert L.vf_net_node_info(None, 0, vf.ctypes.byref(op), None, None, None) == vf.VF_ERR_ARG


def test_struct_layouts_match_the_binding():
    """Every ctypes mirror of a C struct (node descriptors, vf_opts, vf_bab_opts, vf_bab_result) has the C
    struct's size and every field at the C offset, as the library reports them (vf_abi_layout, no device
    work): a field added on one side only would shift every later one."""
    L = vf.lib()
    L.vf_abi_layout.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    out = ctypes.c_size_t()
    for which, S in enumerate((vf.NodeDesc, vf.Opts, vf.BabOpts, vf.BabResult)):
        assert L.vf_abi_layout(which, -1, ctypes.byref(out)) == vf.VF_OK
        assert out.value == ctypes.sizeof(S), S.__name__
        for i, (name, _) in enumerate(S._fields_):
            assert L.vf_abi_layout(which, i, ctypes.byref(out)) == vf.VF_OK, (S.__name__, name)
            assert out.value == getattr(S, name).offset, (S.__name__, name)
        assert L.vf_abi_layout(which, len(S._fields_), ctypes.byref(out)) == vf.VF_ERR_ARG, S.__name__
