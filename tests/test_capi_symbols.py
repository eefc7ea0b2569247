"""The C-ABI library loads and exports every function include/gpt2.h declares (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gpt2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(gpt2_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def libpath():
    from train_step_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("gpt2_create", "gpt2_forward_backward", "gpt2_step", "gpt2_get_params", "gpt2_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (gpt2_\w+)", out))
    assert set(declared_functions()) <= exported


def test_binding_covers_the_header(libpath):
    import train_step_b200 as tsb
    assert set(declared_functions()) == set(tsb.exported_symbols())
    tsb.lib()  # loads without a GPU


def test_library_is_built_for_sm100a(libpath):
    # the build flags name the architecture; the binary itself is not inspected
    from train_step_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


def test_attention_ds_workspace_size(libpath):
    """gpt2_attention_ds_bytes: B*NH tiles of 128 x 128 bf16 per (key block, query block),
    nqb = T / 128 rounded up; 0 for an empty shape. Pure host arithmetic, no GPU."""
    lib = ctypes.CDLL(libpath)
    f = lib.gpt2_attention_ds_bytes
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    f.restype = ctypes.c_size_t
    for B, T, NH in [(16, 1024, 12), (1, 1000, 2), (4, 1024, 25), (3, 129, 1), (1, 1, 1)]:
        nqb = (T + 127) // 128
        assert f(B, T, NH) == B * NH * nqb * nqb * 128 * 128 * 2
    assert f(16, 1024, 12) == 402653184  # the 124M step's workspace: 384 MiB
    assert f(0, 1024, 12) == 0 and f(1, 0, 12) == 0 and f(1, 1024, 0) == 0
