"""GPU parity of fa_forward_dropout / fa_backward_dropout against the fp64 oracle with
the same dropout spec (p, seed, offset).

The keep/drop decision is an integer compare of a Philox-4x32-10 word on both sides,
so the kept set must match exactly; the values are held to the bf16 tolerances of
test_gpu_parity.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_attention_flashattention_b200 import api
from io_aware_attention_flashattention_b200.inputs import make_inputs
from test_gpu_parity import TOL_BF16, _np, assert_close, assert_close_o, grad_tol

pytestmark = pytest.mark.gpu


def run_dropout(q, k, v, do, scale, causal, dropout, window=None, blocks=None):
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    bm = None if blocks is None else torch.from_numpy(blocks).cuda()
    o = torch.full_like(qc, float("nan"))
    lse = torch.full(qc.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    api.fa_forward_dropout(qc, kc, vc, o, lse, scale, causal, dropout, window, bm)
    dq, dk, dv = (torch.full_like(qc, float("nan")) for _ in range(3))
    ws = api.workspace_for(qc)
    ws.fill_(0xFF)
    api.fa_backward_dropout(qc, kc, vc, o, doc, lse, dq, dk, dv, scale, causal, ws, dropout,
                            window, bm)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    return o, lse, dq, dk, dv


CASES = [
    # (B, H, N, d, causal, p, seed, offset, window, block density)
    (1, 2, 256, 64, False, 0.2, 1234, 0, None, None),
    (1, 1, 1000, 128, True, 0.5, 2**40 + 17, 3, None, None),
    (2, 1, 384, 128, False, 0.1, 99, 2**31 + 5, (100, 50), None),
    (1, 2, 640, 64, True, 0.3, 7, 1, None, 0.6),
    (1, 1, 77, 128, False, 0.9, 5, 5, None, None),
    # 192 items of 1 to 5 key tiles: the persistent forward
    (2, 32, 640, 64, True, 0.2, 11, 0, None, None),
]


@pytest.mark.parametrize("B,H,N,d,causal,p,seed,offset,window,density", CASES)
def test_dropout_full_parity(B, H, N, d, causal, p, seed, offset, window, density):
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=300 + N + d)
    scale = 1.0 / math.sqrt(d)
    blocks = None
    if density is not None:
        T = (N + 127) // 128
        blocks = (np.random.default_rng(N).random((T, T)) < density).astype(np.uint8)
        np.fill_diagonal(blocks, 1)
    drop = (p, seed, offset)
    o, lse, dq, dk, dv = run_dropout(q, k, v, do, scale, causal, drop, window, blocks)
    kw = dict(window=window, block_mask=blocks, dropout=drop)
    O_ref, L_ref = oracle.forward(q, k, v, scale, causal, **kw)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, causal, **kw)
    live = np.isfinite(L_ref)
    assert_close_o("O", _np(o)[live], O_ref[live], TOL_BF16["O"])
    assert_close("LSE", _np(lse)[live], L_ref[live], TOL_BF16["L"])
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))


def test_dropout_keep_pattern_is_exact():
    """With V = I the output is Pd itself: its zeros are exactly the dropped keys of
    the oracle's generator (P > 0 everywhere at these logits)."""
    N = d = 128
    g = torch.Generator().manual_seed(8)
    q = (torch.randn(1, 1, N, d, generator=g) * 0.2).to(torch.bfloat16)
    k = (torch.randn(1, 1, N, d, generator=g) * 0.2).to(torch.bfloat16)
    v = torch.eye(N, dtype=torch.bfloat16)[None, None]
    drop = (0.37, 0xDEADBEEF12345678, 42)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qc)
    lse = torch.empty((1, 1, N), dtype=torch.float32, device="cuda")
    api.fa_forward_dropout(qc, kc, vc, o, lse, 0.1, False, drop)
    torch.cuda.synchronize()
    O_ref, _ = oracle.forward(q, k, v, 0.1, False, dropout=drop)
    got = _np(o)[0, 0] != 0
    want = O_ref[0, 0] != 0
    assert np.array_equal(got, want), f"{int((got != want).sum())} keep decisions differ"
    kept = want.mean()
    assert abs(kept - 0.63) < 0.05


def test_dropout_zero_is_masked_path_and_offsets_differ():
    q, k, v, _ = (t.cuda() for t in make_inputs(1, 2, 512, 128, torch.bfloat16, seed=4))
    scale = 1 / math.sqrt(128)
    o0 = torch.empty_like(q)
    l0 = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    api.fa_forward_masked(q, k, v, o0, l0, scale, True, (200, -1), None)
    o1, l1 = torch.empty_like(o0), torch.empty_like(l0)
    api.fa_forward_dropout(q, k, v, o1, l1, scale, True, (0.0, 5, 6), (200, -1), None)
    o2, l2 = torch.empty_like(o0), torch.empty_like(l0)
    api.fa_forward_dropout(q, k, v, o2, l2, scale, True, (0.25, 5, 6), (200, -1), None)
    o3, l3 = torch.empty_like(o0), torch.empty_like(l0)
    api.fa_forward_dropout(q, k, v, o3, l3, scale, True, (0.25, 5, 7), (200, -1), None)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1), "p = 0 must be the masked path"
    assert torch.equal(l0, l2), "LSE does not depend on dropout"
    assert not torch.equal(o2, o3), "a different offset must draw a different mask"


def test_dropout_workload_b1h8_n4096_d128_causal_p01():
    B, H, N, d = 1, 8, 4096, 128
    drop = (0.1, 20261202, 0)
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=1012)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = run_dropout(q, k, v, do, scale, True, drop)
    BH = B * H
    rng = np.random.default_rng(9)
    heads = np.repeat(np.arange(BH), 12)
    rows = np.concatenate([rng.choice(N, 12, replace=False) for _ in range(BH)])
    kw = dict(dropout=drop)
    O_ref, L_ref = oracle.forward_rows(q, k, v, scale, True, heads, rows, **kw)
    dQ_ref, _ = oracle.backward_dq_rows(q, k, v, do, scale, True, heads, rows, **kw)
    assert_close_o("O rows", _np(o).reshape(BH, N, d)[heads, rows], O_ref, TOL_BF16["O"])
    assert_close("LSE rows", _np(lse).reshape(BH, N)[heads, rows], L_ref, TOL_BF16["L"])
    assert_close("dQ rows", _np(dq).reshape(BH, N, d)[heads, rows], dQ_ref,
                 grad_tol(TOL_BF16, dQ_ref))
    h = 2
    all_rows = np.arange(N)
    _, L_h = oracle.forward_rows(q, k, v, scale, True, np.full(N, h), all_rows, **kw)
    _, D_h = oracle.backward_dq_rows(q, k, v, do, scale, True, np.full(N, h), all_rows, **kw)
    keys = np.array([0, 1, 2, 3, 127, 128, 2049, 4094, 4095])
    dK_ref, dV_ref = oracle.backward_dkdv_rows(q, k, v, do, scale, True, h, L_h, D_h, keys, **kw)
    assert_close("dK rows", _np(dk).reshape(BH, N, d)[h, keys], dK_ref, grad_tol(TOL_BF16, dK_ref))
    assert_close("dV rows", _np(dv).reshape(BH, N, d)[h, keys], dV_ref, grad_tol(TOL_BF16, dV_ref))


def test_dropout_argument_errors():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    lib = api.lib()
    p = q.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    for bad in (1.0, -0.1, float("nan")):
        assert lib.fa_forward_dropout(p, p, p, p, lse.data_ptr(), 1, 1, 128, 64, 0.1, 0, -1, -1,
                                      None, bad, 1, 0, s) == 1
    assert api.fa_get_status() == 0


def test_autograd_with_window_and_dropout_matches_oracle():
    """The differentiable wrapper carries the window and the dropout spec into its
    backward."""
    q, k, v, do = make_inputs(1, 2, 300, 128, torch.bfloat16, seed=77)
    drop, window = (0.2, 31337, 4), (100, -1)
    qc, kc, vc = (t.cuda().requires_grad_() for t in (q, k, v))
    out = api.attention(qc, kc, vc, causal=True, window=window, dropout=drop)
    out.backward(do.cuda())
    scale = 1 / math.sqrt(128)
    kw = dict(window=window, dropout=drop)
    O_ref, _ = oracle.forward(q, k, v, scale, True, **kw)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, True, **kw)
    assert_close_o("O", _np(out), O_ref, TOL_BF16["O"])
    for name, got, want in (("dQ", qc.grad, dQ), ("dK", kc.grad, dK), ("dV", vc.grad, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))
