"""GPU parity of the masked entry points (fa_forward_masked / fa_backward_masked)
against the fp64 oracle given the same masks.

Masks: a sliding window (left, right) and a 128 x 128 block mask, ANDed with
causal. Tolerances are the bf16 ones of test_gpu_parity. Rows that see no key must
come back exactly as O = 0, LSE = -inf, dQ = 0; keys no query sees get dK = dV = 0.
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


def _blocks(N, density, seed, zero_row=None, zero_col=None):
    T = (N + 127) // 128
    rng = np.random.default_rng(seed)
    m = (rng.random((T, T)) < density).astype(np.uint8)
    if zero_row is not None:
        m[zero_row, :] = 0
    if zero_col is not None:
        m[:, zero_col] = 0
    return m


def run_masked(q, k, v, do, scale, causal, window, blocks):
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    bm = None if blocks is None else torch.from_numpy(blocks).cuda()
    o = torch.full_like(qc, float("nan"))
    lse = torch.full(qc.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    api.fa_forward_masked(qc, kc, vc, o, lse, scale, causal, window, bm)
    dq, dk, dv = (torch.full_like(qc, float("nan")) for _ in range(3))
    ws = api.workspace_for(qc)
    ws.fill_(0xFF)
    api.fa_backward_masked(qc, kc, vc, o, doc, lse, dq, dk, dv, scale, causal, ws, window, bm)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    return o, lse, dq, dk, dv


def check_masked_full(B, H, N, d, causal, window, blocks, seed):
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=seed)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = run_masked(q, k, v, do, scale, causal, window, blocks)
    O_ref, L_ref = oracle.forward(q, k, v, scale, causal, window, blocks)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, causal, window=window,
                                    block_mask=blocks)
    o_np, l_np = _np(o), _np(lse)
    live = np.isfinite(L_ref)
    assert_close_o("O", o_np[live], O_ref[live], TOL_BF16["O"])
    assert_close("LSE", l_np[live], L_ref[live], TOL_BF16["L"])
    if not live.all():  # rows that see no key
        assert np.all(o_np[~live] == 0.0), "O of rows that see no key"
        assert np.all(l_np[~live] == -np.inf), "LSE of rows that see no key"
        assert np.all(_np(dq)[~live] == 0.0), "dQ of rows that see no key"
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))
    return live


WINDOW_CASES = [
    # (B, H, N, d, causal, window)
    (1, 2, 1000, 64, False, (100, 50)),
    (1, 2, 1000, 128, True, (300, -1)),
    (1, 1, 777, 128, False, (0, 0)),        # the diagonal only
    (2, 1, 640, 64, False, (-1, 129)),      # unbounded left, right past a tile edge
    (1, 1, 512, 128, True, (127, 0)),       # exactly one tile wide
    (1, 2, 384, 128, False, (5000, 5000)),  # wider than N: plain attention
    # more items than SMs, few key tiles each: the persistent forward
    (2, 32, 1024, 64, True, (100, 0)),
    (1, 40, 1000, 128, False, (64, 64)),
]


@pytest.mark.parametrize("B,H,N,d,causal,window", WINDOW_CASES)
def test_sliding_window_full_parity(B, H, N, d, causal, window):
    check_masked_full(B, H, N, d, causal, window, None, seed=40 + N + d)


BLOCK_CASES = [
    # (B, H, N, d, causal, window, density, zero_row, zero_col)
    (1, 2, 640, 128, False, None, 0.5, None, None),
    (1, 2, 640, 64, True, None, 0.6, None, None),
    (1, 1, 1000, 128, False, None, 0.4, 2, 4),    # a query tile and a key tile that see nothing
    (1, 2, 900, 64, False, (150, 150), 0.7, 6, None),  # empty rows inside walked tiles
    (2, 1, 300, 128, True, (200, -1), 1.0, None, 1),
]


@pytest.mark.parametrize("B,H,N,d,causal,window,density,zero_row,zero_col", BLOCK_CASES)
def test_block_mask_full_parity(B, H, N, d, causal, window, density, zero_row, zero_col):
    blocks = _blocks(N, density, seed=N + d, zero_row=zero_row, zero_col=zero_col)
    live = check_masked_full(B, H, N, d, causal, window, blocks, seed=60 + N)
    if zero_row is not None:
        assert not live.all()


def test_no_mask_equals_unmasked_entry_point():
    """With no window and no block mask the masked entry point is fa_forward."""
    q, k, v, do = (t.cuda() for t in make_inputs(1, 2, 700, 128, torch.bfloat16, seed=3))
    o1, l1 = api.forward(q, k, v, causal=True)
    o2 = torch.empty_like(q)
    l2 = torch.empty_like(l1)
    api.fa_forward_masked(q, k, v, o2, l2, 1 / math.sqrt(128), True, None, None)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_window_workload_b1h8_n4096_d128_causal_w512():
    """The sliding-window shape of the deployment page's example (window (512, 512)
    with is_causal) at B1 H8 N4096 d128, sampled rows and keys against the oracle."""
    B, H, N, d = 1, 8, 4096, 128
    causal, window = True, (512, 512)
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=1010)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = run_masked(q, k, v, do, scale, causal, window, None)
    BH = B * H
    rng = np.random.default_rng(5)
    heads = np.repeat(np.arange(BH), 24)
    rows = np.concatenate([rng.choice(N, 24, replace=False) for _ in range(BH)])
    rows[:8] = [0, 1, 511, 512, 513, 4095, 4094, 2048]
    kw = dict(window=window)
    O_ref, L_ref = oracle.forward_rows(q, k, v, scale, causal, heads, rows, **kw)
    dQ_ref, _ = oracle.backward_dq_rows(q, k, v, do, scale, causal, heads, rows, **kw)
    assert_close_o("O rows", _np(o).reshape(BH, N, d)[heads, rows], O_ref, TOL_BF16["O"])
    assert_close("LSE rows", _np(lse).reshape(BH, N)[heads, rows], L_ref, TOL_BF16["L"])
    assert_close("dQ rows", _np(dq).reshape(BH, N, d)[heads, rows], dQ_ref,
                 grad_tol(TOL_BF16, dQ_ref))
    h = 3
    all_rows = np.arange(N)
    _, L_h = oracle.forward_rows(q, k, v, scale, causal, np.full(N, h), all_rows, **kw)
    _, D_h = oracle.backward_dq_rows(q, k, v, do, scale, causal, np.full(N, h), all_rows, **kw)
    keys = np.array([0, 1, 100, 511, 512, 2047, 3583, 3584, 4000, 4095])
    dK_ref, dV_ref = oracle.backward_dkdv_rows(q, k, v, do, scale, causal, h, L_h, D_h, keys, **kw)
    assert_close("dK rows", _np(dk).reshape(BH, N, d)[h, keys], dK_ref, grad_tol(TOL_BF16, dK_ref))
    assert_close("dV rows", _np(dv).reshape(BH, N, d)[h, keys], dV_ref, grad_tol(TOL_BF16, dV_ref))


@pytest.mark.slow
def test_block_sparse_workload_b1h8_n16384_d128():
    """A 25%-dense random block mask (diagonal kept) at B1 H8 N16384 d128, causal:
    sampled rows and keys against the oracle."""
    B, H, N, d = 1, 8, 16384, 128
    T = N // 128
    rng = np.random.default_rng(77)
    blocks = (rng.random((T, T)) < 0.25).astype(np.uint8)
    np.fill_diagonal(blocks, 1)
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=1011)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = run_masked(q, k, v, do, scale, True, None, blocks)
    BH = B * H
    heads = np.repeat(np.arange(BH), 8)
    rows = np.concatenate([rng.choice(N, 8, replace=False) for _ in range(BH)])
    kw = dict(block_mask=blocks)
    O_ref, L_ref = oracle.forward_rows(q, k, v, scale, True, heads, rows, **kw)
    dQ_ref, _ = oracle.backward_dq_rows(q, k, v, do, scale, True, heads, rows, **kw)
    assert_close_o("O rows", _np(o).reshape(BH, N, d)[heads, rows], O_ref, TOL_BF16["O"])
    assert_close("LSE rows", _np(lse).reshape(BH, N)[heads, rows], L_ref, TOL_BF16["L"])
    assert_close("dQ rows", _np(dq).reshape(BH, N, d)[heads, rows], dQ_ref,
                 grad_tol(TOL_BF16, dQ_ref))
    h = 6
    all_rows = np.arange(N)
    _, L_h = oracle.forward_rows(q, k, v, scale, True, np.full(N, h), all_rows, **kw)
    _, D_h = oracle.backward_dq_rows(q, k, v, do, scale, True, np.full(N, h), all_rows, **kw)
    keys = np.unique(np.concatenate([[0, 127, 128, 16383], rng.choice(N, 12, replace=False)]))
    dK_ref, dV_ref = oracle.backward_dkdv_rows(q, k, v, do, scale, True, h, L_h, D_h, keys, **kw)
    assert_close("dK rows", _np(dk).reshape(BH, N, d)[h, keys], dK_ref, grad_tol(TOL_BF16, dK_ref))
    assert_close("dV rows", _np(dv).reshape(BH, N, d)[h, keys], dV_ref, grad_tol(TOL_BF16, dV_ref))


def test_masked_argument_errors():
    q = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 256), dtype=torch.float32, device="cuda")
    lib = api.lib()
    p = q.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    big = 4097 * 128  # block mask of more than 4096 x 4096 tiles
    assert lib.fa_forward_masked(p, p, p, p, lse.data_ptr(), 1, 1, big, 64, 0.1, 0, -1, -1,
                                 p, s) == 2
    assert lib.fa_forward_masked(p, p, p, p, lse.data_ptr(), 1, 1, 256, 64, 0.1, 3, 4, 4,
                                 None, s) == 1  # causal must be 0 or 1
    assert api.fa_get_status() == 0
