"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances (max absolute error against the oracle fed the same rounded inputs):
  bf16 path:  |dO| <= 1e-2, |dLSE| <= 1e-3, each of dQ, dK, dV <= 5e-2 * max|oracle grad|
  fp32 path:  |dO| <= 1e-5, |dLSE| <= 1e-5, each grad <= 1e-5 * max|oracle grad|
  f16 path:   |dO| <= 2e-3, |dLSE| <= 1e-3, each grad <= 1e-2 * max|oracle grad|
The f16 bounds are the bf16 ones scaled by the ratio of the two formats' unit
roundoffs (2^-11 / 2^-8 = 1/8) and then loosened by about 1.6x, except LSE, which
is computed from fp32 logits of exactly representable inputs in both formats.
O is stored in bf16 (f16): rounding to the output format alone moves a value in
[2^e, 2^(e+1)) by up to 2^(e-8), which exceeds 1e-2 once |O| > 2.56 (near-one-hot
attention, as with the x8 logits, gives |O| ~ 4). The O bound is therefore read as
applying to the result before that final rounding: per element, the bound plus
half an ulp of the output format at the oracle value.
Where the oracle's gradient is identically zero (N = 1 gives dQ = dK = 0), the
relative bound would demand exact zeros from rounded arithmetic; there the bound
is an absolute floor (1e-3 bf16, 1e-6 fp32), far below
the gradients' natural scale (|dO| ~ 1).
Outputs are pre-filled with NaN so that an unwritten element fails the check.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_attention_flashattention_b200 import api
from io_aware_attention_flashattention_b200.inputs import (WORKLOADS, make_inputs,
                                                         make_inputs_device, workload_inputs)

pytestmark = pytest.mark.gpu

TOL_BF16 = dict(O=1e-2, L=1e-3, grad=5e-2, floor=1e-3)
TOL_F32 = dict(O=1e-5, L=1e-5, grad=1e-5, floor=1e-6)
TOL_F16 = dict(O=2e-3, L=1e-3, grad=1e-2, floor=2e-4)
TOL = {torch.bfloat16: TOL_BF16, torch.float16: TOL_F16, torch.float32: TOL_F32}


def grad_tol(tol, want):
    return max(tol["grad"] * float(np.abs(want).max()) if np.size(want) else 0.0, tol["floor"])


# significant bits and smallest normal exponent of the 16-bit output formats
_FORMAT = {torch.bfloat16: (8, -126), torch.float16: (11, -14)}


def half_ulp(x, dtype=torch.bfloat16):
    """Half the spacing of the output format's grid at |x| (fixed below the normals)."""
    bits, emin = _FORMAT[dtype]
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.maximum(np.floor(np.log2(np.where(x > 0, x, 1.0))), emin)
    return np.where(x > 0, np.exp2(e - bits), 0.0)


def assert_close_o(name, got, want, tol, dtype=torch.bfloat16):
    """O check: tol plus half an ulp of the output format at the oracle value,
    element by element."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), f"{name}: non-finite values (unwritten or overflow)"
    if not got.size:
        return 0.0
    excess = np.abs(got - want) - (tol + half_ulp(want, dtype))
    worst = int(np.argmax(excess))
    err = float(np.abs(got - want).flat[worst])
    assert excess.flat[worst] <= 0, (
        f"{name}: error {err:.3e} at |O|={abs(want.flat[worst]):.3f} exceeds "
        f"{tol:.1e} + half-ulp {half_ulp(want.flat[worst], dtype):.2e}")
    return float(np.max(np.abs(got - want)))


def _dev(*ts):
    return [t.cuda() for t in ts]


def _nan_like(t):
    return torch.full_like(t, float("nan"))


def run_forward(q, k, v, scale, causal):
    B, H, N, d = q.shape
    o = _nan_like(q)
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    {torch.bfloat16: api.fa_forward, torch.float16: api.fa_forward_f16,
     torch.float32: api.fa_forward_f32}[q.dtype](q, k, v, o, lse, scale, causal)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    return o, lse


def run_backward(q, k, v, o, lse, do, scale, causal):
    dq, dk, dv = _nan_like(q), _nan_like(k), _nan_like(v)
    ws = api.workspace_for(q)
    ws.fill_(0xFF)  # the workspace's contents on entry must not matter
    {torch.bfloat16: api.fa_backward, torch.float16: api.fa_backward_f16,
     torch.float32: api.fa_backward_f32}[q.dtype](q, k, v, o, do, lse, dq, dk, dv, scale,
                                                  causal, ws)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    return dq, dk, dv


def _np(t):
    return t.detach().double().cpu().numpy()


def assert_close(name, got, want, tol):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), f"{name}: non-finite values (unwritten or overflow)"
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    assert err <= tol, f"{name}: max abs error {err:.3e} > {tol:.3e}"
    return err


def check_full(q, k, v, do, scale, causal, tol, backward=True):
    """Every element of O, LSE (and dQ, dK, dV) against the full oracle."""
    qc, kc, vc, doc = _dev(q, k, v, do)
    o, lse = run_forward(qc, kc, vc, scale, causal)
    O_ref, L_ref = oracle.forward(q, k, v, scale, causal)
    if q.dtype in _FORMAT:
        assert_close_o("O", _np(o), O_ref, tol["O"], q.dtype)
    else:
        assert_close("O", _np(o), O_ref, tol["O"])
    assert_close("LSE", _np(lse), L_ref, tol["L"])
    if not backward:
        return
    dq, dk, dv = run_backward(qc, kc, vc, o, lse, doc, scale, causal)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, causal)
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got), want, grad_tol(tol, want))


# ------------------------------------------------------------------ small shapes


SMALL = [
    # (B, H, N, d, causal)
    (1, 1, 128, 64, False),
    (1, 1, 256, 128, False),
    (2, 3, 384, 64, True),
    (1, 2, 512, 128, True),
    (1, 1, 1, 64, False),       # a single key
    (1, 1, 1, 128, True),
    (1, 2, 77, 64, False),      # one ragged tile
    (2, 1, 200, 128, True),     # ragged tail
    (1, 1, 129, 128, False),    # one row into the second tile
    (1, 2, 1000, 64, True),     # several tiles + ragged tail
    (1, 1, 640, 128, False),    # odd number of 128-row tiles (half-empty last CTA)
]


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_bf16_small_full_parity(B, H, N, d, causal):
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=7 + N + d + int(causal))
    check_full(q, k, v, do, 1.0 / math.sqrt(d), causal, TOL_BF16)


# Non-causal launches of few key tiles with 32 or more query tiles each run some or
# all of them as two CTAs, one per half of the query tiles, whose fp32 dK/dV partials
# are summed by the second to end.
SPLIT = [
    (1, 1, 4000, 128, False),   # 32 key tiles, all split; ragged tail
    (1, 5, 4000, 64, False),    # 160 key tiles, the last 12 split
]


@pytest.mark.parametrize("B,H,N,d,causal", SPLIT)
def test_split_key_tiles_full_parity(B, H, N, d, causal):
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=41 + N + d)
    check_full(q, k, v, do, 1.0 / math.sqrt(d), causal, TOL_BF16)


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 1, 256, 64, False), (1, 2, 200, 128, True),
                                            (2, 1, 1, 64, True), (1, 1, 100, 64, False)])
def test_f32_small_full_parity(B, H, N, d, causal):
    q, k, v, do = make_inputs(B, H, N, d, torch.float32, seed=11 + N)
    check_full(q, k, v, do, 1.0 / math.sqrt(d), causal, TOL_F32)


F16_SMALL = [
    (1, 1, 128, 64, False),
    (1, 1, 256, 128, False),
    (2, 3, 384, 64, True),
    (1, 1, 1, 128, True),
    (2, 1, 200, 128, True),
    (1, 2, 1000, 64, True),
    (1, 1, 640, 128, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", F16_SMALL)
def test_f16_small_full_parity(B, H, N, d, causal):
    q, k, v, do = make_inputs(B, H, N, d, torch.float16, seed=17 + N + d + int(causal))
    check_full(q, k, v, do, 1.0 / math.sqrt(d), causal, TOL_F16)


# Launches of more items than SMs whose items average few key tiles run the
# persistent forward: each CTA walks several items, reusing its Q, S, P and O
# buffers (and the K/V rings) from one item to the next. Their backward, with more
# key tiles than SMs, runs the persistent backward the same way (K/V, dK/dV in TMEM,
# the Q/dO ring).
PERSISTENT = [
    # (B, H, N, d, causal, dtype)
    (4, 16, 1024, 64, True, torch.bfloat16),    # 256 pair items, 1 to 8 key tiles each
    (4, 16, 1024, 64, True, torch.float16),
    (2, 40, 900, 128, True, torch.bfloat16),    # ragged tail; single-tile items too
    (3, 64, 256, 128, False, torch.bfloat16),   # 192 items of 2 key tiles
]


@pytest.mark.parametrize("B,H,N,d,causal,dtype", PERSISTENT)
def test_persistent_forward_full_parity(B, H, N, d, causal, dtype):
    q, k, v, do = make_inputs(B, H, N, d, dtype, seed=61 + N + d + int(causal))
    tol = TOL_F16 if dtype == torch.float16 else TOL_BF16
    check_full(q, k, v, do, 1.0 / math.sqrt(d), causal, tol)


def test_f16_large_logits_online_rescale():
    q, k, v, do = make_inputs(1, 2, 512, 128, torch.float16, seed=98, qk_gain=8.0)
    check_full(q, k, v, do, 1.0 / math.sqrt(128), True, TOL_F16)
    check_full(q, k, v, do, 1.0 / math.sqrt(128), False, TOL_F16)


def test_bf16_large_logits_online_rescale():
    """Logits spanning +-hundreds force many rescales of the running max."""
    q, k, v, do = make_inputs(1, 2, 512, 128, torch.bfloat16, seed=99, qk_gain=8.0)
    check_full(q, k, v, do, 1.0 / math.sqrt(128), True, TOL_BF16)
    check_full(q, k, v, do, 1.0 / math.sqrt(128), False, TOL_BF16)


def test_empty_sequence_is_noop():
    z = torch.zeros((1, 1, 0, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 0), dtype=torch.float32, device="cuda")
    api.fa_forward(z, z, z, z, lse, 0.125, False)
    assert api.fa_get_status() == 0


# ------------------------------------------------------------------ the named workloads


def test_workload_oracle_f32_n256_d64():
    w = WORKLOADS["oracle_f32_n256_d64"]
    q, k, v, do = workload_inputs(w)
    check_full(q, k, v, do, w.scale, w.causal, TOL_F32)


def _sampled_rows(rng, BH, N, per_head, extra_head_rows=()):
    heads, rows = [], []
    for h in range(BH):
        r = rng.choice(N, size=min(per_head, N), replace=False)
        heads.extend([h] * len(r))
        rows.extend(r.tolist())
    for h, rs in extra_head_rows:
        heads.extend([h] * len(rs))
        rows.extend(list(rs))
    return np.array(heads), np.array(rows)


def check_sampled(w, per_head=16, full_heads=(0,), dq_rows=True, dkdv_head=None, n_keys=64):
    """Full-size workload on the GPU (the launch the benchmark times), checked
    against the oracle on sampled elements: ``per_head`` random rows of every head,
    plus the first and last 128 rows of each head in ``full_heads`` (O, LSE, dQ),
    and dK/dV of ``n_keys`` random keys plus the first and last 32 keys of head
    ``dkdv_head``. A fast pre-check; test_gpu_full_parity.py compares every element
    of the same launches."""
    q, k, v, do = workload_inputs(w)
    tol = TOL[w.dtype]
    B, H, N, d = q.shape
    BH = B * H
    qc, kc, vc, doc = _dev(q, k, v, do)
    o, lse = run_forward(qc, kc, vc, w.scale, w.causal)
    o_np = _np(o).reshape(BH, N, d)
    l_np = _np(lse).reshape(BH, N)
    assert np.all(np.isfinite(o_np)) and np.all(np.isfinite(l_np))
    rng = np.random.default_rng(w.seed)
    # first and last 128 rows of the full heads: diagonal tiles and the tail
    extra = [(h, list(range(0, 128)) + list(range(N - 128, N))) for h in full_heads]
    heads, rows = _sampled_rows(rng, BH, N, per_head, extra)
    O_ref, L_ref = oracle.forward_rows(q, k, v, w.scale, w.causal, heads, rows)
    assert_close_o("O rows", o_np[heads, rows], O_ref, tol["O"], w.dtype)
    assert_close("LSE rows", l_np[heads, rows], L_ref, tol["L"])
    if not w.backward:
        return
    dq, dk, dv = run_backward(qc, kc, vc, o, lse, doc, w.scale, w.causal)
    dq_np, dk_np, dv_np = (_np(t).reshape(BH, N, d) for t in (dq, dk, dv))
    for name, g in (("dQ", dq_np), ("dK", dk_np), ("dV", dv_np)):
        assert np.all(np.isfinite(g)), f"{name}: non-finite"
    if dq_rows:
        dQ_ref, _ = oracle.backward_dq_rows(q, k, v, do, w.scale, w.causal, heads, rows)
        assert_close("dQ rows", dq_np[heads, rows], dQ_ref, grad_tol(tol, dQ_ref))
    if dkdv_head is not None:
        h = dkdv_head
        all_rows = np.arange(N)
        _, L_h = oracle.forward_rows(q, k, v, w.scale, w.causal, np.full(N, h), all_rows)
        _, D_h = oracle.backward_dq_rows(q, k, v, do, w.scale, w.causal, np.full(N, h), all_rows)
        keys = np.unique(np.concatenate([np.arange(0, 32), np.arange(N - 32, N),
                                         rng.choice(N, n_keys, replace=False)]))
        dK_ref, dV_ref = oracle.backward_dkdv_rows(q, k, v, do, w.scale, w.causal, h, L_h, D_h,
                                                   keys)
        assert_close("dK rows", dk_np[h, keys], dK_ref, grad_tol(tol, dK_ref))
        assert_close("dV rows", dv_np[h, keys], dV_ref, grad_tol(tol, dV_ref))
    # properties at full size: sum_j dK_j = 0 and sum_i dV_i = sum_i dO_i per head
    do_np = _np(doc).reshape(BH, N, d)
    sum_dv = dv_np.sum(axis=1)
    sum_do = do_np.sum(axis=1)
    assert np.max(np.abs(sum_dv - sum_do)) <= 5e-2 * np.abs(sum_do).max() + 1e-2 * math.sqrt(N)
    sum_dk = dk_np.sum(axis=1)
    assert np.max(np.abs(sum_dk)) <= 5e-2 * np.abs(dk_np).max() * math.sqrt(N)


def test_workload_gpt2_causal_b8h12_n1024_d64():
    w = WORKLOADS["gpt2_causal_b8h12_n1024_d64"]
    q, k, v, do = workload_inputs(w)
    # two whole heads through the full oracle (first and last)
    for h in (0, w.B * w.H - 1):
        b, hh = divmod(h, w.H)
        sl = (slice(b, b + 1), slice(hh, hh + 1))
        qc, kc, vc, doc = _dev(q, k, v, do)
        o, lse = run_forward(qc, kc, vc, w.scale, w.causal)
        dq, dk, dv = run_backward(qc, kc, vc, o, lse, doc, w.scale, w.causal)
        O_ref, L_ref = oracle.forward(q[sl], k[sl], v[sl], w.scale, w.causal)
        dQ, dK, dV, _ = oracle.backward(q[sl], k[sl], v[sl], do[sl], w.scale, w.causal)
        assert_close_o("O", _np(o[sl]), O_ref, TOL_BF16["O"])
        assert_close("LSE", _np(lse[sl]), L_ref, TOL_BF16["L"])
        for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
            assert_close(name, _np(got[sl]), want, grad_tol(TOL_BF16, want))
    check_sampled(w, per_head=8, full_heads=(5,), dkdv_head=17)


def test_workload_mid_b1h8_n4096_d128():
    check_sampled(WORKLOADS["mid_b1h8_n4096_d128"], per_head=64, full_heads=(0, 7), dkdv_head=3)


def test_workload_stress_causal_b2h16_n8192_d128_qk8():
    check_sampled(WORKLOADS["stress_causal_b2h16_n8192_d128_qk8"], per_head=16, full_heads=(0, 31))


def test_workload_mid_b1h8_n4096_d128_in_f16():
    w = dataclasses.replace(WORKLOADS["mid_b1h8_n4096_d128"], dtype=torch.float16)
    check_sampled(w, per_head=32, full_heads=(2,), dkdv_head=6)


@pytest.mark.slow
def test_workload_long_b1h8_n16384_d128_causal():
    """The long workload's shape with the causal mask (tiles above the diagonal never
    loaded; the forward's pair/single split differs from the non-causal one)."""
    w = dataclasses.replace(WORKLOADS["long_b1h8_n16384_d128"], causal=True)
    check_sampled(w, per_head=24, full_heads=(1,), dkdv_head=6, n_keys=32)


def test_workload_stress_causal_b2h16_n8192_d128_qk8_in_f16():
    """The x8-logit causal stress shape with f16 inputs (forward only)."""
    w = dataclasses.replace(WORKLOADS["stress_causal_b2h16_n8192_d128_qk8"], dtype=torch.float16)
    check_sampled(w, per_head=12, full_heads=(3,))


@pytest.mark.slow
def test_workload_long_b1h8_n16384_d128():
    check_sampled(WORKLOADS["long_b1h8_n16384_d128"], per_head=32, full_heads=(0, 7),
                  dkdv_head=5, n_keys=32)


def test_tensors_beyond_2p31_elements():
    """Offsets are 64-bit: B1 H1040 N16384 d128 puts 2.18e9 elements in each tensor
    (4.4 GB of bf16), so the last head starts past element 2^31. Its O, LSE, dQ, dK
    and dV are compared with the oracle on that head's inputs (the definition is per
    head, so one head is a [1, 1, N, d] problem)."""
    B, H, N, d = 1, 1040, 16384, 128
    if torch.cuda.mem_get_info()[0] < (64 << 30):
        pytest.skip("needs about 50 GB of free device memory")
    assert (H - 1) * N * d > 2 ** 31
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = make_inputs_device(B, H, N, d, torch.bfloat16, seed=2031)
    o, lse = run_forward(q, k, v, scale, False)
    dq, dk, dv = run_backward(q, k, v, o, lse, do, scale, False)
    sl = (slice(0, 1), slice(H - 1, H))
    qh, kh, vh, doh = (t[sl].cpu() for t in (q, k, v, do))
    O_ref, L_ref = oracle.forward(qh, kh, vh, scale, False)
    assert_close_o("O", _np(o[sl]), O_ref, TOL_BF16["O"])
    assert_close("LSE", _np(lse[sl]), L_ref, TOL_BF16["L"])
    dQ, dK, dV, _ = oracle.backward(qh, kh, vh, doh, scale, False)
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got[sl]), want, grad_tol(TOL_BF16, want))
    # every head was written (NaN-prefilled outputs)
    for t in (o, lse, dq, dk, dv):
        assert not torch.isnan(t).any()


# ------------------------------------------------------------------ behaviour


def test_dk_dv_deterministic():
    q, k, v, do = _dev(*make_inputs(1, 4, 1024, 128, torch.bfloat16, seed=5))
    o, lse = run_forward(q, k, v, 0.088, True)
    a = run_backward(q, k, v, o, lse, do, 0.088, True)
    b = run_backward(q, k, v, o, lse, do, 0.088, True)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2)


def test_split_key_tiles_are_deterministic():
    """B1 H8 N8192 d128 (512 key tiles on 148 SMs) runs 68 key tiles as two CTAs each,
    whose fp32 dK/dV partials are added in a fixed order: dK and dV are the same bits
    every run."""
    q, k, v, do = _dev(*make_inputs(1, 8, 8192, 128, torch.bfloat16, seed=13))
    o, lse = run_forward(q, k, v, 0.088, False)
    a = run_backward(q, k, v, o, lse, do, 0.088, False)
    b = run_backward(q, k, v, o, lse, do, 0.088, False)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_argument_errors_launch_nothing():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    lib = api.lib()
    p = q.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.fa_forward(p, p, p, p, lse.data_ptr(), 1, 1, 128, 96, 0.1, 0, s) == 2  # d
    assert lib.fa_forward(p, p, p, p, lse.data_ptr(), 1, 1, 128, 64, -1.0, 0, s) == 1  # scale
    assert lib.fa_forward(p, p, p, p, lse.data_ptr(), 1, 1, 128, 64, float("nan"), 0, s) == 1
    assert lib.fa_forward(p + 2, p, p, p, lse.data_ptr(), 1, 1, 128, 64, 0.1, 0, s) == 1  # align
    assert lib.fa_forward(p, p, p, p, None, 1, 1, 128, 64, 0.1, 0, s) == 1  # null
    assert lib.fa_forward(p, p, p, p, lse.data_ptr(), 0, 1, 128, 64, 0.1, 0, s) == 1  # B
    assert lib.fa_forward(p, p, p, p, lse.data_ptr(), 1, 1, 128, 64, 0.1, 2, s) == 1  # causal
    ws_need = api.fa_backward_workspace_size(1, 1, 128, 64)
    assert lib.fa_backward(p, p, p, p, p, lse.data_ptr(), p, p, p, 1, 1, 128, 64, 0.1, 0,
                           p, ws_need - 1, s) == 1
    assert api.fa_get_status() == 0


def test_call_on_a_second_gpu_while_the_first_is_current():
    """The binding makes the tensors' GPU current for the call, so the library's
    per-GPU state (status word, SM count, shared-memory attributes, work split) is
    that GPU's. Needs two GPUs."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    q, k, v, do = make_inputs(1, 2, 384, 128, torch.bfloat16, seed=31)
    with torch.cuda.device(0):
        qc, kc, vc, doc = (t.to("cuda:1") for t in (q, k, v, do))
        o, lse = api.forward(qc, kc, vc, causal=True)
        dq, dk, dv = api.backward(qc, kc, vc, o, lse, doc, causal=True)
        assert torch.cuda.current_device() == 0
        torch.cuda.synchronize(1)
        assert api.fa_get_status(torch.cuda.current_stream(1)) == 0
    scale = 1.0 / math.sqrt(128)
    O_ref, L_ref = oracle.forward(q, k, v, scale, True)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, True)
    assert_close_o("O", _np(o), O_ref, TOL_BF16["O"])
    assert_close("LSE", _np(lse), L_ref, TOL_BF16["L"])
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))


def test_watchdog_timeout_is_reported_and_context_survives():
    api.fa_watchdog_selftest(50)
    assert api.fa_get_status() == 4  # FA_ERR_TIMEOUT
    assert api.fa_get_status() == 0  # cleared by the read
    q, k, v, do = make_inputs(1, 1, 256, 64, torch.bfloat16, seed=3)
    check_full(q, k, v, do, 0.125, False, TOL_BF16)


def test_autograd_function_matches_oracle():
    q, k, v, do = make_inputs(1, 2, 256, 128, torch.bfloat16, seed=21)
    qc, kc, vc = (t.cuda().requires_grad_() for t in (q, k, v))
    out = api.attention(qc, kc, vc, causal=True)
    out.backward(do.cuda())
    O_ref, _ = oracle.forward(q, k, v, 1 / math.sqrt(128), True)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, 1 / math.sqrt(128), True)
    assert_close_o("O", _np(out), O_ref, TOL_BF16["O"])
    for name, got, want in (("dQ", qc.grad, dQ), ("dK", kc.grad, dK), ("dV", vc.grad, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))


def test_launch_plan_matches_the_measured_choices():
    """The launch forms the host picks on a 148-SM B200 for the named shapes."""
    props = torch.cuda.get_device_properties(0)
    if props.multi_processor_count != 148:
        pytest.skip("the expected plans are for 148 SMs")
    plan = api.fa_launch_plan
    # long rows: one CTA per forward item; more key tiles than SMs: persistent backward
    assert plan(1, 8, 16384, 128, False) == {"fwd_persistent": False, "bwd_persistent": True,
                                             "bwd_split": 0}
    # GPT-2 shape: short causal rows run persistent in both directions
    assert plan(8, 12, 1024, 64, True) == {"fwd_persistent": True, "bwd_persistent": True,
                                           "bwd_split": 0}
    # 512 key tiles of 64 steps: 68 split over two CTAs each, one CTA per tile
    assert plan(1, 8, 8192, 128, False) == {"fwd_persistent": False, "bwd_persistent": False,
                                            "bwd_split": 68}
    # 256 items/tiles: the forward's 128 pairs fill one wave; the backward is persistent
    assert plan(1, 8, 4096, 128, False) == {"fwd_persistent": False, "bwd_persistent": True,
                                            "bwd_split": 0}
    assert plan(1, 8, 0, 128, False) == {"fwd_persistent": False, "bwd_persistent": False,
                                         "bwd_split": 0}
