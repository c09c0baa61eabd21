"""The C-ABI library builds, loads and exports what include/*.h declares (CPU only).

No compute call is made here (there is no GPU); the GPU suite covers that.
"""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def libvgqa():
    from varlen_gqa_split_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("attn_plan", "attn_plan_ex", "attn_plan_info", "attn_run", "attn_run_strided", "attn_run_paged",
              "attn_merge_lse", "attn_check_error", "attn_destroy", "attn_strerror", "attn_run_noalloc"):
        assert n in names


def test_library_exports_every_declared_symbol(libvgqa):
    lib, path = libvgqa
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported by {path}"


def test_library_exports_only_the_boundary(libvgqa):
    _, path = libvgqa
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    text_syms = [l.split()[-1] for l in out.splitlines() if len(l.split()) == 3 and l.split()[1] == "T"]
    ours = [s for s in text_syms if s.startswith("attn_")]
    assert sorted(ours) == declared_functions()


def test_library_targets_sm100a(libvgqa):
    # the build flags name the sm_100a target and only that one
    from varlen_gqa_split_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_strerror_and_host_errors_without_gpu(libvgqa):
    import varlen_gqa_split_b200 as vg
    assert vg.strerror(0) == "success"
    assert "alignment" in vg.strerror(-4)
    assert vg.strerror(12345) == "unknown error code"
    lib, _ = libvgqa
    lib.attn_plan.argtypes = [ctypes.POINTER(ctypes.c_void_p)] + [ctypes.c_int] * 6
    h = ctypes.c_void_p()
    # argument checks come before any device query
    assert lib.attn_plan(ctypes.byref(h), 0, 128, 4, 1, 64, 1) == -1       # B_max < 1
    assert lib.attn_plan(ctypes.byref(h), 2, 128, 6, 4, 64, 1) == -1       # Hq % Hkv
    assert lib.attn_plan(ctypes.byref(h), 2, 128, 4, 1, 96, 1) == -2       # head dim
    lib.attn_run.argtypes = [ctypes.c_void_p] * 9
    assert lib.attn_run(None, None, None, None, None, None, None, None, None) == -5
    lib.attn_run_strided.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
    assert lib.attn_run_strided(None, None, None, None, None, None, None, None, 1024, 1024, None) == -5
    lib.attn_run_paged.argtypes = ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 2 + [ctypes.c_int] * 2 +
                                   [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 5)
    assert lib.attn_run_paged(None, None, None, None, 2048, 256, 16, 4, None, 8, None, None, None, None,
                              None) == -5
    lib.attn_merge_lse.argtypes = ([ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p] +
                                   [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3)
    assert lib.attn_merge_lse(2, None, None, 4, None, 1, 8, 128, None, None, None) == -3   # no GPU touched
    lib.attn_plan_info.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    buf = ctypes.create_string_buffer(256)
    assert lib.attn_plan_info(ctypes.c_void_p(0x1234), buf) == -5          # unknown handle


def test_no_silent_fallback_without_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import varlen_gqa_split_b200 as vg
    with pytest.raises(vg.AttnError):
        vg.Plan(2, 128, 4, 1, 64, 1)
