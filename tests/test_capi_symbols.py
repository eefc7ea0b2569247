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
