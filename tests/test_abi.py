"""The C-ABI library loads and exports every symbol include/fa.h declares
(CPU only: no compute call needs a GPU here)."""
import ctypes
import os
import re

import pytest

from io_aware_attention_flashattention_b200 import build
from io_aware_attention_flashattention_b200 import _lib

HEADER = os.path.join(build.INCLUDE, "fa.h")


@pytest.fixture(scope="module")
def libfa():
    build.build_library()
    return ctypes.CDLL(build.LIB)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("fa_forward", "fa_backward", "fa_backward_workspace_size", "fa_forward_f32",
                 "fa_backward_f32", "fa_get_status", "fa_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(libfa):
    for name in declared_functions():
        assert hasattr(libfa, name), f"{name} declared in fa.h but not exported"


def test_binding_covers_the_header():
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def test_host_only_entry_points(libfa):
    libfa.fa_version.restype = ctypes.c_char_p
    assert b"sm_100a" in libfa.fa_version()
    libfa.fa_status_string.restype = ctypes.c_char_p
    assert libfa.fa_status_string(4) == b"kernel watchdog timeout"
    f = libfa.fa_backward_workspace_size
    f.restype = ctypes.c_size_t
    # L2 and D padded to 128 rows, plus the fp32 dQ accumulator
    assert f(1, 8, 16384, 128) == 2 * (8 * 16384 * 4) + 8 * 16384 * 128 * 4
    assert f(1, 1, 100, 64) == 2 * 512 + 25600
    assert f(1, 1, 100, 96) == 0
    assert f(0, 1, 100, 64) == 0


def test_argument_errors_need_no_gpu(libfa):
    fn = libfa.fa_forward
    fn.restype = ctypes.c_int
    fn.argtypes = _lib.SIGNATURES["fa_forward"][1]
    assert fn(None, None, None, None, None, 1, 1, 128, 64, 0.1, 0, None) == 1
    assert fn(None, None, None, None, None, 1, 1, 128, 80, 0.1, 0, None) == 2
    assert fn(None, None, None, None, None, 1, 1, 0, 64, 0.1, 0, None) == 0  # empty: no-op


def test_no_cpu_fallback_in_product_path():
    """The product package never imports the oracle."""
    pkg = os.path.dirname(build.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(root, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
