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


def test_launch_plan_refuses_bad_shapes_before_any_device_call(libfa):
    """fa_launch_plan validates the shape first: a refused shape returns its status
    without touching a GPU (this host has none) and writes no output."""
    f = _fn(libfa, "fa_launch_plan")
    out = [ctypes.c_int(-7) for _ in range(3)]
    ptrs = [ctypes.addressof(o) for o in out]
    assert f(1, 1, 100, 96, 0, *ptrs) == 2        # d = 96: FA_ERR_UNSUPPORTED
    assert f(0, 1, 100, 64, 0, *ptrs) == 1        # B = 0
    assert f(1, 1, 100, 64, 2, *ptrs) == 1        # causal must be 0 or 1
    assert f(1, 1, 2**30 + 1, 64, 0, *ptrs) == 2  # N beyond 2^30: FA_ERR_UNSUPPORTED
    assert [o.value for o in out] == [-7, -7, -7]


def test_host_only_entry_points(libfa):
    libfa.fa_version.restype = ctypes.c_char_p
    assert b"sm_100a" in libfa.fa_version()
    libfa.fa_status_string.restype = ctypes.c_char_p
    assert libfa.fa_status_string(4) == b"kernel watchdog timeout"
    f = libfa.fa_backward_workspace_size
    f.restype = ctypes.c_size_t
    # L2 and D padded to 128 rows and the fp32 dQ accumulator, each region rounded up
    # to 256 bytes; launches of at most 592 key tiles with N padded to 4096 or more add
    # room for the fp32 dK/dV partials (2 segments x 128 rows x d, twice) and arrival
    # counters of min(key tiles, 160) split key tiles. 1024 key tiles, or short rows,
    # get no split slots:
    assert f(1, 8, 16384, 128) == 2 * (8 * 16384 * 4) + 8 * 16384 * 128 * 4
    assert f(1, 1, 100, 64) == 2 * 512 + 25600
    assert f(1, 2, 1000, 64) == 2 * 8192 + 512000
    # 512 key tiles: 160 slots; 32 key tiles (N = 4000 pads to 4096): 32 slots
    assert f(1, 8, 8192, 128) == (2 * (8 * 8192 * 4) + 8 * 8192 * 128 * 4
                                  + 160 * 4 * 128 * 128 * 4 + 768)
    assert f(1, 1, 4000, 64) == 2 * 16384 + 4000 * 64 * 4 + 32 * 4 * 128 * 64 * 4 + 256
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


def _fn(libfa, name):
    f = getattr(libfa, name)
    f.restype, f.argtypes = _lib.SIGNATURES[name]
    return f


def test_host_validation_of_every_entry_point(libfa):
    """Each entry point rejects bad arguments on the host, before any CUDA call, with
    the documented status (1 invalid argument, 2 unsupported); no GPU is needed."""
    P = 0x10000  # a 16-byte-aligned stand-in address; a rejected call never touches it
    fwd = _fn(libfa, "fa_forward")
    assert fwd(P, P, P, P, P, 1, 1, (1 << 30) + 1, 128, 0.1, 0, None) == 2  # N > 2^30
    assert fwd(P, P, P, P, P, 1 << 14, 1 << 13, 128, 128, 0.1, 0, None) == 2  # B*H = 2^27 tiles
    assert fwd(P, P, P, P, P, 1 << 16, 1 << 16, 0, 64, 0.1, 0, None) == 2  # B*H = 2^32
    assert fwd(P, P, P, P, P, 1, 1, 128, 64, float("nan"), 0, None) == 1
    assert fwd(P, P, P, P, P, 1, 1, 128, 64, 0.0, 0, None) == 1
    assert fwd(P, P, P, P, P, 1, 1, 128, 64, 0.1, 2, None) == 1
    assert fwd(P, P, P, P, P, 0, 1, 128, 64, 0.1, 0, None) == 1
    assert fwd(P, P, P, P, P, 1, 1, -1, 64, 0.1, 0, None) == 1
    assert fwd(P + 8, P, P, P, P, 1, 1, 128, 64, 0.1, 0, None) == 1  # misaligned
    f16 = _fn(libfa, "fa_forward_f16")
    assert f16(P, P, P, P, P, 1, 1, 128, 32, 0.1, 0, None) == 2
    masked = _fn(libfa, "fa_forward_masked")
    big_n = 4097 * 128  # a block mask of more than 4096 x 4096 tiles
    assert masked(P, P, P, P, P, 1, 1, big_n, 64, 0.1, 0, -1, -1, P, None) == 2
    assert masked(P, P, P, P, P, 1, 1, 256, 64, 0.1, 3, 4, 4, None, None) == 1
    drop = _fn(libfa, "fa_forward_dropout")
    for p in (1.0, -0.25, float("nan"), float("inf")):
        assert drop(P, P, P, P, P, 1, 1, 256, 64, 0.1, 0, -1, -1, None, p, 7, 0, None) == 1
    # a rate below 1/256 would round down to no dropout at all: refused
    assert drop(P, P, P, P, P, 1, 1, 256, 64, 0.1, 0, -1, -1, None, 0.003, 7, 0, None) == 2
    dheads = _fn(libfa, "fa_forward_dropout_heads")
    assert dheads(P, P, P, P, P, 1, 1, 256, 64, 0.1, 0, -1, -1, None, 0.1, 7, 0, -1, None) == 1
    assert dheads(P, P, P, P, P, 1, 1, 256, 64, 0.1, 0, -1, -1, None, 1.5, 7, 0, 3, None) == 1
    ws = _fn(libfa, "fa_backward_workspace_size")(1, 2, 384, 64)
    bwd = _fn(libfa, "fa_backward")
    assert bwd(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, P, ws - 1, None) == 1
    assert bwd(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, None, ws, None) == 1
    assert bwd(P, P, P, P, P, None, P, P, P, 1, 2, 384, 64, 0.1, 0, P, ws, None) == 1
    bwd16 = _fn(libfa, "fa_backward_f16")
    assert bwd16(P, P, P, P, P, P, P, P, P, 1, 2, 384, 96, 0.1, 0, P, ws, None) == 2
    noalloc = _fn(libfa, "fa_backward_noalloc")
    # B1 H8 N16384 d128 needs 68 MB of workspace, more than the 32 MiB built in
    assert noalloc(P, P, P, P, P, P, P, P, P, 1, 8, 16384, 128, 0.1, 0, None) == 2
    bdrop = _fn(libfa, "fa_backward_dropout")
    assert bdrop(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, -1, -1, None, 1.5, 1, 0,
                 P, ws, None) == 1
    f32 = _fn(libfa, "fa_backward_f32")
    assert f32(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, P, ws - 1, None) == 1
    bdrop_ok = bdrop(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, -1, -1, None, 0.001, 1, 0,
                     P, ws, None)
    assert bdrop_ok == 2
    bheads = _fn(libfa, "fa_backward_dropout_heads")
    assert bheads(P, P, P, P, P, P, P, P, P, 1, 2, 384, 64, 0.1, 0, -1, -1, None, 0.1, 1, 0,
                  -5, P, ws, None) == 1


def test_dropout_rate_is_the_byte_threshold(libfa):
    """fa_dropout_rate returns the drop probability the kernels apply: p rounded down
    to a multiple of 1/256; -1 for a rate the dropout calls refuse."""
    rate = _fn(libfa, "fa_dropout_rate")
    assert rate(0.0) == 0.0
    assert rate(0.1) == 25 / 256
    assert rate(0.5) == 0.5
    assert rate(255.9 / 256) == 255 / 256
    for p in (0.001, 1.0, -0.5, float("nan")):
        assert rate(p) == -1.0


def test_binding_runs_each_call_on_its_tensors_gpu():
    """Every entry point of the binding makes its tensors' GPU current (the library
    launches on the current device) and refuses tensors spread over two GPUs."""
    import types

    import torch

    from io_aware_attention_flashattention_b200 import api

    on = lambda i: types.SimpleNamespace(device=torch.device("cuda", i))  # noqa: E731
    with pytest.raises(ValueError, match="one GPU"):
        api._one_device(on(0), on(1))
    ctx = api._one_device(on(1), on(1), torch.zeros(1), 7, None)
    assert isinstance(ctx, torch.cuda.device) and ctx.idx == 1
    assert not isinstance(api._one_device(torch.zeros(1), 3.0), torch.cuda.device)
    for name in api.__all__:
        fn = getattr(api, name)
        if name.startswith("fa_") and callable(fn) and name not in (
                "fa_version", "fa_backward_workspace_size", "fa_dropout_rate",
                "fa_launch_plan"):  # no tensors: host-only, or (the plan) the current GPU
            assert getattr(fn, "__wrapped__", None) is not None, f"{name} is not device-guarded"
