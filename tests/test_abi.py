"""The C-ABI library loads and exports every symbol include/*.h declares, and
host-side validation works without a GPU."""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADERS = glob.glob(os.path.join(ROOT, "include", "*.h"))


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from packed_mxfp4_w4a16_b200 import _lib
    return _lib.load()


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("moe_create", "moe_load_packed", "moe_route", "moe_forward"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from packed_mxfp4_w4a16_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    declared = declared_functions()
    assert declared, "no declarations parsed"
    missing = declared - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    # the binding declares exactly the header's functions
    bound = {name for name, _, _ in _lib.SIGNATURES}
    assert bound == declared
    # nothing but the C ABI leaks out of the library
    extra = {s for s in exported if s.startswith("moe_")} - declared
    assert not extra


def test_create_validates_shapes(lib):
    h = C.c_void_p()
    ok = [(64, 2048, 1536, 4), (16, 512, 384, 4), (1, 32, 32, 1), (8, 64, 96, 8)]
    for E, H, I, k in ok:
        assert lib.moe_create(E, H, I, k, C.byref(h)) == 0 and h.value
        assert lib.moe_destroy(h) == 0
    bad = [(0, 2048, 1536, 4), (64, 2047, 1536, 4), (64, 2048, 1530, 4), (64, 2048, 1536, 0),
           (64, 2048, 1536, 9), (3, 64, 64, 4), (2000, 64, 64, 4), (64, 16, 64, 1)]
    for E, H, I, k in bad:
        h = C.c_void_p(123)
        assert lib.moe_create(E, H, I, k, C.byref(h)) == -1
        assert h.value is None
    assert lib.moe_create(64, 2048, 1536, 4, None) == -1
    assert lib.moe_destroy(None) == 0


def test_bytes_per_expert_closed_form(lib):
    h = C.c_void_p()
    assert lib.moe_create(64, 2048, 1536, 4, C.byref(h)) == 0
    n = C.c_size_t()
    assert lib.moe_bytes_per_expert(h, C.byref(n)) == 0
    # 3*2048*1536 weights at 0.5 + 1/32 byte each
    assert n.value == 5013504
    ws = C.c_size_t()
    assert lib.moe_workspace_bytes(h, 1, C.byref(ws)) == 0 and ws.value > 0
    ws4 = C.c_size_t()
    assert lib.moe_workspace_bytes(h, 4, C.byref(ws4)) == 0 and ws4.value > ws.value
    assert lib.moe_workspace_bytes(h, 0, C.byref(ws)) == -1
    lib.moe_destroy(h)


def test_calls_fail_cleanly_without_weights_or_device(lib):
    h = C.c_void_p()
    assert lib.moe_create(16, 512, 384, 4, C.byref(h)) == 0
    # no workspace / weights: forward and route refuse before touching CUDA
    assert lib.moe_forward(h, None, 1, None, None, None, None) in (-1, -2)
    assert lib.moe_route(h, None, 1, None, None, None, None, None) in (-1, -2)
    assert lib.moe_forward(h, None, 0, None, None, None, None) == -1
    st = C.c_uint()
    assert lib.moe_get_status(h, C.byref(st)) == -2
    hp, op = C.c_void_p(), C.c_void_p()
    assert lib.moe_get_intermediates(h, C.byref(hp), C.byref(op)) == -2
    assert lib.moe_set_tuning(h, 1, 0) == 0
    lib.moe_destroy(h)


def test_forward_flags_are_validated_on_the_host(lib):
    """Flag combinations that exclude each other, unknown bits and a forced
    tcgen05 path without contiguous weights are refused (MOE_ERR_ARG) before
    any device work; a valid combination gets as far as the missing weights
    (MOE_ERR_NOT_LOADED)."""
    from packed_mxfp4_w4a16_b200 import (FWD_FORCE_DECODE, FWD_FORCE_GROUPED, FWD_FORCE_MMA,
                                         FWD_FORCE_TCGEN05, FWD_PHASE_DOWN, FWD_PHASE_GATEUP)
    h = C.c_void_p()
    assert lib.moe_create(64, 2048, 1536, 4, C.byref(h)) == 0
    try:
        def fwd(flags, T=64):
            return lib.moe_forward_ex(h, None, T, None, None, None, None, flags, None)
        for bad in (0x80, 1 << 31, FWD_FORCE_MMA | FWD_FORCE_TCGEN05,
                    FWD_FORCE_MMA | FWD_FORCE_DECODE, FWD_FORCE_TCGEN05 | FWD_FORCE_DECODE,
                    FWD_FORCE_DECODE | FWD_FORCE_GROUPED, FWD_PHASE_GATEUP | FWD_PHASE_DOWN,
                    FWD_FORCE_TCGEN05):  # no contiguous weights bound
            assert fwd(bad) == -1, hex(bad)
        assert fwd(0, T=0) == -1
        for good in (0, FWD_FORCE_MMA, FWD_FORCE_GROUPED, FWD_FORCE_DECODE, FWD_PHASE_GATEUP):
            assert fwd(good) == -2, hex(good)
    finally:
        lib.moe_destroy(h)


def test_status_strings(lib):
    for code in range(-8, 1):
        s = lib.moe_status_string(code).decode()
        assert s.startswith("MOE_")
    assert lib.moe_status_string(-99).decode() == "unknown moe status"


def test_stack_calls_validate_on_the_host(lib):
    """moe_stack_* refuse bad arguments before any device work."""
    out = C.c_void_p(123)
    assert lib.moe_stack_create(None, 1, None, None, C.byref(out)) == -1 and out.value is None
    h = C.c_void_p()
    assert lib.moe_create(64, 2048, 1536, 4, C.byref(h)) == 0
    try:
        arr = (C.c_void_p * 1)(h.value)
        rws = (C.c_void_p * 1)(None)
        assert lib.moe_stack_create(arr, 0, rws, None, C.byref(out)) == -1
        assert lib.moe_stack_create(arr, 65, rws, None, C.byref(out)) == -1
        # weights not bound yet
        assert lib.moe_stack_create(arr, 1, rws, None, C.byref(out)) == -2
        assert lib.moe_stack_create(arr, 1, rws, None, None) == -1
    finally:
        lib.moe_destroy(h)
    assert lib.moe_stack_destroy(None) == 0
    assert lib.moe_stack_decode(None, None, None, None, None, None, None, None) == -1
    assert lib.moe_stack_set_spin_limit(None, 0) == -1
    n = C.c_size_t()
    assert lib.moe_stack_workspace_bytes(None, C.byref(n)) == -1
    st = C.c_uint()
    assert lib.moe_stack_get_status(None, None, C.byref(st)) == -1
    assert lib.moe_forward_noalloc_status(None, None) == -1


def test_noalloc_wrapper_checks_every_tensor_against_the_shape():
    """The Python wrapper of moe_forward_noalloc checks sizes, dtypes,
    contiguity and device of every tensor before the C call (which takes bare
    pointers): here on CPU tensors against device 'cpu'."""
    import torch

    import packed_mxfp4_w4a16_b200 as moe
    E, H, I, k, T = 4, 64, 32, 2, 3
    t = dict(codes=torch.zeros(E * 3 * I * H // 2, dtype=torch.uint8),
             scales=torch.zeros(E * 3 * I * H // 32, dtype=torch.uint8),
             x=torch.zeros(T, H, dtype=torch.bfloat16),
             topk_ids=torch.zeros(T, k, dtype=torch.int32),
             topk_w=torch.zeros(T, k, dtype=torch.float32),
             residual=None, y=torch.zeros(T, H, dtype=torch.bfloat16))

    def run(**over):
        a = dict(t, **over)
        return moe._noalloc_args_ok(E, H, I, k, a["codes"], a["scales"], a["x"], a["topk_ids"],
                                    a["topk_w"], a["residual"], a["y"], device="cpu")

    assert run() == T
    assert run(residual=torch.zeros(T, H, dtype=torch.bfloat16)) == T
    bad = [dict(codes=t["codes"][:-1]), dict(scales=torch.zeros(7, dtype=torch.uint8)),
           dict(x=torch.zeros(T, H + 32, dtype=torch.bfloat16)),
           dict(x=torch.zeros(T, H, dtype=torch.float32)),
           dict(topk_ids=torch.zeros(T, k + 1, dtype=torch.int32)),
           dict(topk_ids=torch.zeros(T, k, dtype=torch.int64)),
           dict(topk_w=torch.zeros(T - 1, k, dtype=torch.float32)),
           dict(y=torch.zeros(T + 1, H, dtype=torch.bfloat16)),
           dict(y=torch.zeros(H, T, dtype=torch.bfloat16).t()),
           dict(residual=torch.zeros(T, H - 32, dtype=torch.bfloat16))]
    for over in bad:
        with pytest.raises(moe.MoEError):
            run(**over)
    with pytest.raises(moe.MoEError):  # tensors on another device than asked
        moe._noalloc_args_ok(E, H, I, k, t["codes"], t["scales"], t["x"], t["topk_ids"],
                             t["topk_w"], None, t["y"], device="meta")
