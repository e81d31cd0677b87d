"""The fp64 oracle against its pins (CPU only; see tests/pins.py)."""
import numpy as np
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=[p.__name__ for p in pins.ALL_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_row_functions_match_full_functions(orc):
    """The row-restricted entry points (used at sizes where the full oracle is too
    slow) agree with the full ones, which the pins above tie down."""
    rng = np.random.default_rng(21)
    B, H, N, d = 2, 3, 37, 8
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    for causal in (False, True):
        O, L = orc.forward(Q, K, V, 0.4, causal)
        dQ, dK, dV, D = orc.backward(Q, K, V, dO, 0.4, causal)
        heads = rng.integers(0, B * H, 20)
        rows = rng.integers(0, N, 20)
        Or, Lr = orc.forward_rows(Q, K, V, 0.4, causal, heads, rows)
        np.testing.assert_allclose(Or, O.reshape(B * H, N, d)[heads, rows], atol=1e-13)
        np.testing.assert_allclose(Lr, L.reshape(B * H, N)[heads, rows], atol=1e-13)
        dQr, Dr = orc.backward_dq_rows(Q, K, V, dO, 0.4, causal, heads, rows)
        np.testing.assert_allclose(dQr, dQ.reshape(B * H, N, d)[heads, rows], atol=1e-13)
        np.testing.assert_allclose(Dr, D.reshape(B * H, N)[heads, rows], atol=1e-13)
        head = 4
        keys = np.array([0, 5, 36, 17])
        dKr, dVr = orc.backward_dkdv_rows(Q, K, V, dO, 0.4, causal, head,
                                          L.reshape(B * H, N)[head], D.reshape(B * H, N)[head], keys)
        np.testing.assert_allclose(dKr, dK.reshape(B * H, N, d)[head, keys], atol=1e-13)
        np.testing.assert_allclose(dVr, dV.reshape(B * H, N, d)[head, keys], atol=1e-13)


def test_row_functions_match_full_functions_with_masks(orc):
    """The same agreement under a sliding window and a block mask (one block row
    empty, so some rows see no key), with and without dropout."""
    rng = np.random.default_rng(22)
    B, H, N, d = 1, 2, 260, 4
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    blocks = [[1, 0, 1], [1, 1, 0], [0, 0, 0]]
    for causal, window, dropout in ((False, (40, 7), None), (True, (90, -1), None),
                                    (False, (40, 7), (0.3, 1234, 9))):
        kw = dict(window=window, block_mask=blocks, dropout=dropout)
        O, L = orc.forward(Q, K, V, 0.4, causal, **kw)
        dQ, dK, dV, D = orc.backward(Q, K, V, dO, 0.4, causal, **kw)
        heads = rng.integers(0, B * H, 30)
        rows = rng.integers(0, N, 30)
        Or, Lr = orc.forward_rows(Q, K, V, 0.4, causal, heads, rows, **kw)
        np.testing.assert_allclose(Or, O.reshape(B * H, N, d)[heads, rows], atol=1e-13)
        np.testing.assert_array_equal(np.isinf(Lr), np.isinf(L.reshape(B * H, N)[heads, rows]))
        fin = np.isfinite(Lr)
        np.testing.assert_allclose(Lr[fin], L.reshape(B * H, N)[heads, rows][fin], atol=1e-13)
        dQr, Dr = orc.backward_dq_rows(Q, K, V, dO, 0.4, causal, heads, rows, **kw)
        np.testing.assert_allclose(dQr, dQ.reshape(B * H, N, d)[heads, rows], atol=1e-13)
        np.testing.assert_allclose(Dr, D.reshape(B * H, N)[heads, rows], atol=1e-13)
        head = 1
        keys = np.array([0, 5, 130, 255, 259, 200])
        dKr, dVr = orc.backward_dkdv_rows(Q, K, V, dO, 0.4, causal, head,
                                          L.reshape(B * H, N)[head], D.reshape(B * H, N)[head],
                                          keys, **kw)
        np.testing.assert_allclose(dKr, dK.reshape(B * H, N, d)[head, keys], atol=1e-13)
        np.testing.assert_allclose(dVr, dV.reshape(B * H, N, d)[head, keys], atol=1e-13)


def test_bad_arguments_rejected(orc):
    with pytest.raises(RuntimeError):
        orc.forward_rows(np.zeros((1, 1, 4, 2)), np.zeros((1, 1, 4, 2)), np.zeros((1, 1, 4, 2)),
                         1.0, False, [0], [4])


def test_empty_sequence(orc):
    Z = np.zeros((1, 2, 0, 4))
    O, L = orc.forward(Z, Z, Z, 1.0, True)
    assert O.shape == (1, 2, 0, 4) and L.shape == (1, 2, 0)
