"""Python front of the fp64 exact-attention oracle (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path never does: it has no CPU
fallback. The oracle shares no code with the CUDA library.

All arithmetic lives in ``attn_oracle.cpp`` (plain fp64 loops, OpenMP over rows);
this module only builds that file with gcc, loads it with ctypes and marshals
numpy arrays. Inputs are any array-likes; they are converted to contiguous
float64 [B, H, N, d] arrays (the caller passes values already rounded to the
run's dtype, so the oracle sees exactly the bits the GPU sees, upcast to fp64).

Definitions followed (titles of the sources, see the header of attn_oracle.cpp):
  * attention definition S = QK^T, P = Softmax(S), O = PV: "A survey of key
    techniques of large language model pre-training systems", Journal of
    Software 2026(1), p.218;
  * scaling by 1/sqrt(d): "FlashAttention optimisation: breaking the
    performance bottleneck of standard attention", section 1;
  * safe softmax: "From GPU memory access to code: how FlashAttention makes
    large-model training 3x faster", section 2.1;
  * causal masking (key j visible to query i iff j <= i): "Flash Attention-2:
    acceleration principle and GPU memory optimisation in deployment", causal
    mask item;
  * sliding window (i - left <= j <= i + right) from the sliding-window example
    of the same item, and a block mask over 128 x 128 blocks (block-sparse
    FlashAttention, "FlashAttention optimisation: breaking the performance
    bottleneck of standard attention", section 7). Every entry point takes
    ``window=(left, right)`` (negative = unbounded side; None = no window) and
    ``block_mask`` (uint8 [ceil(N/128), ceil(N/128)], shared by all heads; None =
    every block); they combine with ``causal`` by AND. A row that sees no key has
    O = 0, L = -inf and zero gradients;
  * dropout on P ([jos] lists it among the fused operations), with the keep/drop
    decision from a byte of Philox-4x32-10 (Salmon et al., "Parallel random numbers:
    as easy as 1, 2, 3", SC 2011) against floor(256 p), so p acts rounded down to a
    multiple of 1/256. ``dropout=(p, seed, offset)``; see attn_oracle.cpp.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "attn_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int64)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64
_c = ctypes.c_int
_MASK = [_c, _i64, _i64, _U8]  # causal, window left, window right, block mask
_DROP = [ctypes.c_double, ctypes.c_uint64, ctypes.c_uint32]  # p, seed, offset

BLOCK = 128  # block-mask granularity


def _mask(N: int, causal: bool, window, block_mask):
    """(ctypes argument list, array to keep alive) for the masks of one call."""
    left, right = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    blocks = None
    if block_mask is not None:
        nb = (N + BLOCK - 1) // BLOCK
        blocks = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
        if blocks.shape != (nb, nb):
            raise ValueError(f"block_mask must be [{nb}, {nb}] for N={N}")
    ptr = blocks.ctypes.data_as(_U8) if blocks is not None else None
    return [int(bool(causal)), left, right, ptr], blocks


def _drop(dropout):
    """ctypes arguments of a dropout spec (p, seed, offset); None = no dropout."""
    if dropout is None:
        return [0.0, 0, 0]
    p, seed, offset = dropout
    return [float(p), int(seed) & ((1 << 64) - 1), int(offset) & 0xFFFFFFFF]


def _compile(src: str, out: str) -> None:
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", src, "-o", out + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(force: bool = False) -> str:
    """Compile attn_oracle.cpp into liboracle.so beside it (gcc, -O2, OpenMP).

    No fast-math: the oracle keeps IEEE fp64 semantics."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
            _compile(SOURCE, _LIB)
    return _LIB


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _pi(a: np.ndarray):
    return a.ctypes.data_as(_I)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _shape4(Q):
    if Q.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    return Q.shape


class Oracle:
    """The oracle's entry points over one compiled copy of attn_oracle.cpp.

    The module-level functions use the copy built from the committed source. The
    test suite also builds copies with a deliberately planted mistake (see
    ``Oracle.from_source``) to show that its pins catch such mistakes."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        f = ctypes.c_double
        lib.oracle_attention_probs.argtypes = [_D, _D, _i64, _i64, f] + _MASK + [_D]
        lib.oracle_attention_forward.argtypes = (
            [_D, _D, _D, _i64, _i64, _i64, _i64, f] + _MASK + _DROP + [_D, _D])
        lib.oracle_attention_backward.argtypes = (
            [_D, _D, _D, _D, _i64, _i64, _i64, _i64, f] + _MASK + _DROP + [_D, _D, _D, _D, _D])
        lib.oracle_attention_forward_rows.argtypes = (
            [_D, _D, _D, _i64, _i64, _i64, _i64, f] + _MASK + _DROP + [_i64, _I, _I, _D, _D])
        lib.oracle_attention_backward_dq_rows.argtypes = (
            [_D, _D, _D, _D, _i64, _i64, _i64, _i64, f] + _MASK + _DROP
            + [_i64, _I, _I, _D, _D])
        lib.oracle_attention_backward_dkdv_rows.argtypes = (
            [_D, _D, _D, _D, _i64, _i64, _i64, _i64, f] + _MASK + _DROP
            + [_i64, _D, _D, _i64, _I, _D, _D])
        _U32 = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_philox4x32_10.argtypes = [_U32, ctypes.c_uint32, ctypes.c_uint32, _U32]
        lib.oracle_philox4x32_10.restype = None
        for name in ("oracle_attention_probs", "oracle_attention_forward",
                     "oracle_attention_backward", "oracle_attention_forward_rows",
                     "oracle_attention_backward_dq_rows",
                     "oracle_attention_backward_dkdv_rows"):
            getattr(lib, name).restype = ctypes.c_int
        self._lib = lib
        self.path = lib_path

    @classmethod
    def from_source(cls, source_text: str, workdir: str) -> "Oracle":
        """Compile ``source_text`` (a variant of attn_oracle.cpp) in ``workdir``."""
        os.makedirs(workdir, exist_ok=True)
        src = os.path.join(workdir, "attn_oracle_variant.cpp")
        out = os.path.join(workdir, "liboracle_variant.so")
        with open(src, "w") as f:
            f.write(source_text)
        _compile(src, out)
        return cls(out)

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self._lib.oracle_set_num_threads(int(n))

    def probs(self, q, k, scale: float, causal: bool, window=None,
              block_mask=None) -> np.ndarray:
        """P = softmax(scale * q k^T) (masked) of one head; q, k are [N, d]."""
        q, k = _f64(q), _f64(k)
        N, d = q.shape
        P = np.empty((N, N), dtype=np.float64)
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_probs(_p(q), _p(k), N, d, float(scale), *m, _p(P)),
               "probs")
        return P

    def philox(self, counter, key):
        """Philox-4x32-10 of one counter (4 words) under one key (2 words)."""
        ctr = np.ascontiguousarray(counter, dtype=np.uint32)
        out = np.zeros(4, dtype=np.uint32)
        U32 = ctypes.POINTER(ctypes.c_uint32)
        self._lib.oracle_philox4x32_10(ctr.ctypes.data_as(U32), int(key[0]), int(key[1]),
                                       out.ctypes.data_as(U32))
        return out

    def forward(self, Q, K, V, scale: float, causal: bool, window=None, block_mask=None,
                dropout=None):
        """(O, L): O [B,H,N,d] fp64, L [B,H,N] fp64 natural-log log-sum-exp."""
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, H, N, d = _shape4(Q)
        O = np.empty_like(Q)
        L = np.empty((B, H, N), dtype=np.float64)
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_forward(_p(Q), _p(K), _p(V), B, H, N, d, float(scale),
                                                  *m, *_drop(dropout), _p(O), _p(L)), "forward")
        return O, L

    def backward(self, Q, K, V, dO, scale: float, causal: bool, with_check: bool = False,
                 window=None, block_mask=None, dropout=None):
        """(dQ, dK, dV, D[, Dcheck]) for the loss <dO, O>."""
        Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
        B, H, N, d = _shape4(Q)
        dQ, dK, dV = np.empty_like(Q), np.empty_like(Q), np.empty_like(Q)
        D = np.empty((B, H, N), dtype=np.float64)
        Dc = np.empty((B, H, N), dtype=np.float64) if with_check else None
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_backward(
            _p(Q), _p(K), _p(V), _p(dO), B, H, N, d, float(scale), *m, *_drop(dropout),
            _p(dQ), _p(dK), _p(dV), _p(D), _p(Dc) if with_check else None), "backward")
        return (dQ, dK, dV, D, Dc) if with_check else (dQ, dK, dV, D)

    def forward_rows(self, Q, K, V, scale: float, causal: bool, heads, rows, window=None,
                     block_mask=None, dropout=None):
        """O and L of selected (head, row) pairs, head = b * H + h: ([R, d], [R])."""
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, H, N, d = _shape4(Q)
        heads = np.ascontiguousarray(heads, dtype=np.int64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = heads.shape[0]
        O = np.empty((R, d), dtype=np.float64)
        L = np.empty((R,), dtype=np.float64)
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_forward_rows(
            _p(Q), _p(K), _p(V), B, H, N, d, float(scale), *m, *_drop(dropout), R, _pi(heads),
            _pi(rows), _p(O), _p(L)), "forward_rows")
        return O, L

    def backward_dq_rows(self, Q, K, V, dO, scale: float, causal: bool, heads, rows,
                         window=None, block_mask=None, dropout=None):
        """dQ and D of selected (head, row) pairs: ([R, d], [R])."""
        Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
        B, H, N, d = _shape4(Q)
        heads = np.ascontiguousarray(heads, dtype=np.int64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = heads.shape[0]
        dQ = np.empty((R, d), dtype=np.float64)
        D = np.empty((R,), dtype=np.float64)
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_backward_dq_rows(
            _p(Q), _p(K), _p(V), _p(dO), B, H, N, d, float(scale), *m, *_drop(dropout), R,
            _pi(heads), _pi(rows), _p(dQ), _p(D)), "backward_dq_rows")
        return dQ, D

    def backward_dkdv_rows(self, Q, K, V, dO, scale: float, causal: bool, head: int, L_head,
                           D_head, keys, window=None, block_mask=None, dropout=None):
        """dK and dV of selected key rows of one head, given that head's L and D as
        computed by this oracle (forward_rows / backward_dq_rows over all rows)."""
        Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
        B, H, N, d = _shape4(Q)
        L_head, D_head = _f64(L_head), _f64(D_head)
        if L_head.shape != (N,) or D_head.shape != (N,):
            raise ValueError("L_head and D_head must be [N]")
        keys = np.ascontiguousarray(keys, dtype=np.int64)
        R = keys.shape[0]
        dK = np.empty((R, d), dtype=np.float64)
        dV = np.empty((R, d), dtype=np.float64)
        m, keep = _mask(N, causal, window, block_mask)
        _check(self._lib.oracle_attention_backward_dkdv_rows(
            _p(Q), _p(K), _p(V), _p(dO), B, H, N, d, float(scale), *m, *_drop(dropout), int(head),
            _p(L_head), _p(D_head), R, _pi(keys), _p(dK), _p(dV)), "backward_dkdv_rows")
        return dK, dV


_default = None


def default() -> Oracle:
    """The oracle built from the committed attn_oracle.cpp."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def probs(*a, **k):
    return default().probs(*a, **k)


def forward(*a, **k):
    return default().forward(*a, **k)


def backward(*a, **k):
    return default().backward(*a, **k)


def forward_rows(*a, **k):
    return default().forward_rows(*a, **k)


def backward_dq_rows(*a, **k):
    return default().backward_dq_rows(*a, **k)


def backward_dkdv_rows(*a, **k):
    return default().backward_dkdv_rows(*a, **k)
