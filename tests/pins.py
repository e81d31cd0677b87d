"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` takes an oracle object (``oracle.Oracle``) and raises AssertionError
when the oracle disagrees with:
  * the two-block softmax decomposition m = max(m1, m2),
    l = e^(m1-m) l1 + e^(m2-m) l2 of "A survey of key techniques of large language
    model pre-training systems" (Journal of Software 2026(1), p.218), and the
    two-pass tiled softmax of "From GPU memory access to code: how FlashAttention
    makes large-model training 3x faster", section 2.1;
  * closed forms (rows of P sum to 1; a constant key gives the mean of V; one key
    gives O = V; a two-level logit pattern has an exact weighted mean);
  * the blockwise online loop of "Flash Attention-2: acceleration principle and
    GPU memory optimisation in deployment" (its "Flash Attention-2 blockwise
    computation" listing, restated here in numpy), which that page says equals
    standard attention exactly;
  * a library routine computing the same function (torch fp64 CPU
    scaled_dot_product_attention and its autograd backward);
  * central finite differences of the loss <dO, O>;
  * invariants of the gradient (sum_j dK_j = 0, sum_i dV_i = sum_i dO_i, D two ways).

The same pins run against variants of the oracle with a planted mistake
(tests/test_oracle_mutants.py); each such variant must fail at least one pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs error {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------- softmax


def pin_two_block_decomposition(orc):
    """The oracle's softmax row equals the two-block decomposition and the two-pass
    tiled softmax, for unequal splits and logits up to +-800 (where skipping the
    max subtraction overflows fp64)."""
    rng = _rng(11)
    cases = [(7, 3, 1.0), (16, 1, 50.0), (33, 20, 300.0), (64, 63, 300.0), (9, 4, 800.0)]
    for N, split, spread in cases:
        x = rng.uniform(-spread, spread, N)
        # d = 1, q = 1, k_j = x_j, scale = 1: every row's logits are exactly x.
        q = np.ones((N, 1))
        k = x.reshape(N, 1)
        P = orc.probs(q, k, 1.0, False)
        x1, x2 = x[:split], x[split:]
        m1, m2 = x1.max(), x2.max()
        f1, f2 = np.exp(x1 - m1), np.exp(x2 - m2)
        l1, l2 = f1.sum(), f2.sum()
        m = max(m1, m2)
        f = np.concatenate([np.exp(m1 - m) * f1, np.exp(m2 - m) * f2])
        l = np.exp(m1 - m) * l1 + np.exp(m2 - m) * l2
        want = f / l
        for i in (0, N // 2, N - 1):
            _close(P[i], want, 1e-14, f"two-block softmax N={N} split={split}")
        # two-pass tiled softmax: global max over blocks, then the sum, then divide
        blocks = [x[a:a + 5] for a in range(0, N, 5)]
        gmax = max(b.max() for b in blocks)
        total = sum(np.exp(b - gmax).sum() for b in blocks)
        tiled = np.concatenate([np.exp(b - gmax) / total for b in blocks])
        _close(P[0], tiled, 1e-14, "two-pass tiled softmax")
        # the log-sum-exp the forward returns is m + ln l of the decomposition
        V = rng.standard_normal((1, 1, N, 1))
        _, L = orc.forward(q.reshape(1, 1, N, 1), k.reshape(1, 1, N, 1), V, 1.0, False)
        _close(L[0, 0], np.full(N, m + math.log(l)), 1e-12 * max(1.0, abs(m)),
               "log-sum-exp from the decomposition")


def pin_rows_sum_to_one(orc):
    """Softmax = f / l: every row of P sums to 1; causal rows put no weight above
    the diagonal and some weight on it."""
    rng = _rng(12)
    N, d = 50, 8
    q = rng.standard_normal((N, d)) * 3
    k = rng.standard_normal((N, d)) * 3
    for causal in (False, True):
        P = orc.probs(q, k, 0.5, causal)
        _close(P.sum(axis=1), np.ones(N), 1e-12, "row sums")
        assert np.all(P >= 0)
        if causal:
            assert np.all(np.triu(P, 1) == 0.0), "weight above the diagonal"
            assert np.all(np.diag(P) > 0.0), "no weight on the diagonal"


# --------------------------------------------------------------------------- forward


def pin_constant_key(orc):
    """All keys equal: P is uniform over the visible keys, so O_i is the mean of
    V_0..V_{N-1} (causal: of V_0..V_i) and L_i = scale <q_i, k> + ln(count)."""
    rng = _rng(13)
    B, H, N, d = 2, 2, 24, 8
    scale = 0.3
    Q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, 1, d))
    K = np.repeat(k, N, axis=2)
    V = rng.standard_normal((B, H, N, d))
    for causal in (False, True):
        O, L = orc.forward(Q, K, V, scale, causal)
        if causal:
            counts = np.arange(1, N + 1, dtype=np.float64)
            want_O = np.cumsum(V, axis=2) / counts[None, None, :, None]
        else:
            counts = np.full(N, float(N))
            want_O = np.broadcast_to(V.mean(axis=2, keepdims=True), V.shape)
        want_L = scale * np.einsum("bhnd,bhd->bhn", Q, k[:, :, 0, :]) + np.log(counts)
        _close(O, want_O, 1e-12, f"constant key O (causal={causal})")
        _close(L, want_L, 1e-12, f"constant key L (causal={causal})")


def pin_single_key(orc):
    """N = 1: O = V, L = scale <q, k>; the gradient is dQ = dK = 0, dV = dO."""
    rng = _rng(14)
    B, H, N, d = 3, 2, 1, 16
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    for causal in (False, True):
        O, L = orc.forward(Q, K, V, 0.7, causal)
        _close(O, V, 1e-15, "N=1 O")
        _close(L, 0.7 * np.sum(Q * K, axis=-1), 1e-13, "N=1 L")
        dQ, dK, dV, D = orc.backward(Q, K, V, dO, 0.7, causal)
        _close(dQ, np.zeros_like(dQ), 1e-15, "N=1 dQ")
        _close(dK, np.zeros_like(dK), 1e-15, "N=1 dK")
        _close(dV, dO, 1e-15, "N=1 dV")


def pin_two_level_logits(orc):
    """Logits a on one key pi(i) per row and 0 elsewhere (pi a permutation):
    O_i = (e^a V_pi(i) + sum_{j != pi(i)} V_j) / (e^a + N - 1), L_i = ln(e^a + N - 1)."""
    rng = _rng(15)
    N = 12
    perm = rng.permutation(N)
    V = rng.standard_normal((1, 1, N, N))  # the oracle takes one head width for Q, K, V
    for a in (3.0, 60.0):
        scale = 0.5
        Q = np.zeros((1, 1, N, N))
        Q[0, 0, np.arange(N), perm] = a / scale
        K = np.eye(N).reshape(1, 1, N, N)
        O, L = orc.forward(Q, K, V, scale, False)
        total = V[0, 0].sum(axis=0)
        ea = math.exp(a)
        want = (ea * V[0, 0, perm] + (total[None, :] - V[0, 0, perm])) / (ea + N - 1)
        _close(O[0, 0], want, 1e-13, f"two-level logits O (a={a})")
        _close(L[0, 0], np.full(N, math.log(ea + N - 1)), 1e-13, f"two-level logits L (a={a})")


def blockwise_forward(Q, K, V, scale, causal, Br, Bc):
    """The blockwise online-softmax loop (outer loop over query blocks, inner over
    key/value blocks, running max m and sum l, rescale by exp(m_old - m_new), divide
    by l at the end), in fp64 numpy. Independent of the oracle's code."""
    B, H, N, d = Q.shape
    O = np.zeros_like(Q)
    L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, Br):
                qi = Q[b, h, i0:i0 + Br]
                r = qi.shape[0]
                rows = np.arange(i0, i0 + r)
                m = np.full(r, -np.inf)
                l = np.zeros(r)
                acc = np.zeros((r, d))
                for j0 in range(0, N, Bc):
                    if causal and j0 > rows[-1]:
                        break
                    kj = K[b, h, j0:j0 + Bc]
                    vj = V[b, h, j0:j0 + Bc]
                    s = (qi @ kj.T) * scale
                    if causal:
                        cols = np.arange(j0, j0 + kj.shape[0])
                        s = np.where(cols[None, :] > rows[:, None], -np.inf, s)
                    m_new = np.maximum(m, s.max(axis=1))
                    p = np.exp(s - m_new[:, None])
                    alpha = np.exp(m - m_new)
                    l = l * alpha + p.sum(axis=1)
                    acc = acc * alpha[:, None] + p @ vj
                    m = m_new
                O[b, h, i0:i0 + r] = acc / l[:, None]
                L[b, h, i0:i0 + r] = m + np.log(l)
    return O, L


def pin_blockwise_loop(orc):
    """The oracle equals the blockwise online loop (ragged last blocks, unequal
    Br and Bc, causal and not) to 1e-12."""
    rng = _rng(16)
    B, H, N, d = 2, 3, 100, 16
    Q, K, V = (rng.standard_normal((B, H, N, d)) * 2 for _ in range(3))
    for causal in (False, True):
        O, L = orc.forward(Q, K, V, 0.25, causal)
        Ob, Lb = blockwise_forward(Q, K, V, 0.25, causal, Br=32, Bc=48)
        _close(O, Ob, 1e-12, f"blockwise O (causal={causal})")
        _close(L, Lb, 1e-12, f"blockwise L (causal={causal})")


# --------------------------------------------------------------------------- library


def pin_torch_sdpa(orc):
    """fp64 torch SDPA on the CPU (forward and autograd backward) agrees to 1e-12."""
    rng = _rng(17)
    B, H, N, d = 2, 2, 40, 16
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    for causal in (False, True):
        scale = 1.0 / math.sqrt(d)
        O, L = orc.forward(Q, K, V, scale, causal)
        qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
        ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal,
                                                              scale=scale)
        ot.backward(torch.tensor(dO))
        _close(O, ot.detach().numpy(), 1e-12, "SDPA O")
        # L against the library's logsumexp of the masked logits
        s = torch.einsum("bhid,bhjd->bhij", torch.tensor(Q), torch.tensor(K)) * scale
        if causal:
            s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
        _close(L, torch.logsumexp(s, dim=-1).numpy(), 1e-12, "logsumexp L")
        dQ, dK, dV, D = orc.backward(Q, K, V, dO, scale, causal)
        _close(dQ, qt.grad.numpy(), 1e-12, "SDPA dQ")
        _close(dK, kt.grad.numpy(), 1e-12, "SDPA dK")
        _close(dV, vt.grad.numpy(), 1e-12, "SDPA dV")


# --------------------------------------------------------------------------- backward


def pin_finite_differences(orc):
    """Central differences (h = 1e-6) of l = <dO, O> over every element of Q, K, V
    at N <= 16, d <= 8, causal and not: relative error <= 1e-6 of max|grad|."""
    rng = _rng(18)
    for (N, d, causal) in ((16, 8, False), (13, 4, True), (5, 8, True)):
        B, H = 1, 2
        Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
        scale = 1.0 / math.sqrt(d)
        dQ, dK, dV, _ = orc.backward(Q, K, V, dO, scale, causal)

        def loss(q, k, v):
            O, _ = orc.forward(q, k, v, scale, causal)
            return float(np.sum(O * dO))

        h = 1e-6
        for which, grad in ((0, dQ), (1, dK), (2, dV)):
            num = np.zeros_like(grad)
            for idx in np.ndindex(*grad.shape):
                args_p = [Q.copy(), K.copy(), V.copy()]
                args_m = [Q.copy(), K.copy(), V.copy()]
                args_p[which][idx] += h
                args_m[which][idx] -= h
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            ref = max(1e-3, float(np.max(np.abs(num))))
            err = float(np.max(np.abs(num - grad)))
            assert err <= 1e-6 * ref, (
                f"finite differences of {'QKV'[which]} (N={N}, d={d}, causal={causal}): "
                f"{err:.3e} > 1e-6 * {ref:.3e}")


def pin_gradient_invariants(orc):
    """Rows of dS sum to 0, so sum_j dK_j = 0; sum_i dV_i = sum_i dO_i (columns of
    P^T sum to 1); D = rowsum(P o dP) equals rowsum(dO o O)."""
    rng = _rng(19)
    B, H, N, d = 2, 2, 48, 16
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) * 1.5 for _ in range(4))
    for causal in (False, True):
        dQ, dK, dV, D, Dc = orc.backward(Q, K, V, dO, 0.25, causal, with_check=True)
        _close(dK.sum(axis=2), np.zeros((B, H, d)), 1e-12 * N * max(1.0, np.abs(dK).max()),
               "sum_j dK_j")
        _close(dV.sum(axis=2), dO.sum(axis=2), 1e-12 * N, "sum_i dV_i")
        _close(D, Dc, 1e-12 * max(1.0, np.abs(D).max()), "D two ways")
        O, _ = orc.forward(Q, K, V, 0.25, causal)
        _close(D, np.sum(dO * O, axis=-1), 1e-12 * max(1.0, np.abs(D).max()), "D = rowsum(dO o O)")


# --------------------------------------------------------------------------- masks
#
# Sliding window (keep i - left <= j <= i + right; "Flash Attention-2: acceleration
# principle and GPU memory optimisation in deployment", sliding-window example of
# its causal-mask item) and a block mask over 128 x 128 blocks (block-sparse
# FlashAttention, "FlashAttention optimisation: breaking the performance bottleneck
# of standard attention", section 7), both ANDed with the causal mask.


def library_mask(N, causal, window, blocks):
    """The kept (i, j) pairs built with library routines: a band from torch's
    triu/tril, the block pattern from numpy's Kronecker product."""
    keep = torch.ones(N, N, dtype=torch.bool)
    if causal:
        keep = keep.tril(0)
    if window is not None:
        left, right = window
        if left >= 0:
            keep = keep.triu(-left)
        if right >= 0:
            keep = keep.tril(right)
    if blocks is not None:
        full = np.kron(np.asarray(blocks, dtype=np.uint8), np.ones((128, 128), np.uint8))
        keep = keep & torch.from_numpy(full[:N, :N] != 0)
    return keep


MASK_CASES = [
    # (N, causal, window, block pattern or None)
    (40, False, (3, 5), None),
    (40, True, (7, -1), None),
    (40, False, (0, 0), None),           # the diagonal only
    (40, False, (-1, 2), None),          # unbounded on the left
    (300, False, None, [[1, 0, 1], [0, 1, 0], [1, 1, 0]]),
    (300, True, (150, -1), [[1, 0, 0], [1, 0, 0], [0, 1, 1]]),
    (260, False, (20, 20), [[0, 1, 1], [1, 0, 1], [0, 0, 0]]),  # empty rows (last block)
]


def pin_masks_match_library(orc):
    """Windowed and block-masked attention equals fp64 torch SDPA given the library-
    built boolean mask (forward, logsumexp, autograd gradients) to 1e-12; rows that
    see no key have O = 0, L = -inf and zero dQ, and P vanishes exactly where the
    mask hides a key."""
    rng = _rng(21)
    for N, causal, window, blocks in MASK_CASES:
        B, H, d = 1, 2, 8
        Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
        scale = 0.4
        keep = library_mask(N, causal, window, blocks)
        what = f"N={N} causal={causal} window={window} blocks={blocks}"
        P = orc.probs(Q[0, 0], K[0, 0], scale, causal, window, blocks)
        assert np.array_equal(P > 0, keep.numpy()), f"{what}: support of P"
        O, L = orc.forward(Q, K, V, scale, causal, window, blocks)
        dQ, dK, dV, _ = orc.backward(Q, K, V, dO, scale, causal, window=window,
                                     block_mask=blocks)
        live = keep.any(dim=1).numpy()
        qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
        ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=keep,
                                                              scale=scale)
        # rows with no visible key are NaN in the library; they are not part of the loss
        ot_live = ot[:, :, torch.from_numpy(live)]
        ot_live.backward(torch.tensor(dO[:, :, live]))
        _close(O[:, :, live], ot_live.detach().numpy(), 1e-12, f"{what}: O")
        s = torch.einsum("bhid,bhjd->bhij", torch.tensor(Q), torch.tensor(K)) * scale
        lse = torch.logsumexp(s.masked_fill(~keep, -math.inf), dim=-1).numpy()
        _close(L[:, :, live], lse[:, :, live], 1e-12, f"{what}: L")
        _close(dQ[:, :, live], qt.grad.numpy()[:, :, live], 1e-12, f"{what}: dQ")
        _close(dK, kt.grad.numpy(), 1e-12, f"{what}: dK")
        _close(dV, vt.grad.numpy(), 1e-12, f"{what}: dV")
        if not live.all():
            dead = ~live
            assert np.all(O[:, :, dead] == 0.0), f"{what}: O of empty rows"
            assert np.all(L[:, :, dead] == -np.inf), f"{what}: L of empty rows"
            assert np.all(dQ[:, :, dead] == 0.0), f"{what}: dQ of empty rows"


def pin_window_closed_forms(orc):
    """With every key equal, P is uniform over the visible keys, so O_i is the mean
    of V over the window max(0, i-left) .. min(N-1, i+right) (causal: .. i) and
    L_i = s + ln(count); the count of visible keys is the window's length."""
    rng = _rng(22)
    N, d = 50, 4
    for causal, (left, right) in ((False, (4, 9)), (True, (6, -1)), (False, (0, 0)),
                                  (True, (-1, 3)), (False, (60, 1))):
        q = rng.standard_normal((N, d))
        k = np.tile(rng.standard_normal((1, d)), (N, 1))
        v = rng.standard_normal((N, d))
        O, L = orc.forward(q[None, None], k[None, None], v[None, None], 0.5, causal,
                           (left, right))
        for i in range(N):
            lo = 0 if left < 0 else max(0, i - left)
            hi = N - 1 if right < 0 else min(N - 1, i + right)
            if causal:
                hi = min(hi, i)
            s = 0.5 * float(q[i] @ k[0])
            what = f"row {i} causal={causal} window=({left},{right})"
            _close(O[0, 0, i], v[lo:hi + 1].mean(axis=0), 1e-13, what + ": O")
            _close(L[0, 0, i], s + math.log(hi - lo + 1), 1e-12, what + ": L")


def pin_masked_finite_differences(orc):
    """Central differences of <dO, O> through windowed and block-masked attention
    (a sample of elements at N = 140, all of them at N = 12): error <= 1e-6 of
    max|grad|."""
    rng = _rng(23)
    cases = [(12, 3, False, (2, 1), None, None),
             (12, 3, True, (4, -1), None, None),
             (140, 2, False, (30, 5), [[1, 1], [0, 1]], 24)]
    for N, d, causal, window, blocks, n_sample in cases:
        Q, K, V, dO = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
        scale = 0.7
        grads = orc.backward(Q, K, V, dO, scale, causal, window=window, block_mask=blocks)[:3]

        def loss(q, k, v):
            O, _ = orc.forward(q, k, v, scale, causal, window, blocks)
            return float(np.sum(O * dO))

        h = 1e-6
        for which, grad in enumerate(grads):
            idxs = list(np.ndindex(*grad.shape))
            if n_sample is not None:
                idxs = [idxs[t] for t in rng.choice(len(idxs), n_sample, replace=False)]
            ref = max(1e-3, float(np.max(np.abs(grad))))
            for idx in idxs:
                args_p = [Q.copy(), K.copy(), V.copy()]
                args_m = [Q.copy(), K.copy(), V.copy()]
                args_p[which][idx] += h
                args_m[which][idx] -= h
                num = (loss(*args_p) - loss(*args_m)) / (2 * h)
                assert abs(num - grad[idx]) <= 1e-6 * ref, (
                    f"masked finite differences of {'QKV'[which]}{idx} (N={N}, "
                    f"window={window}, blocks={blocks}): {num:.6e} vs {grad[idx]:.6e}")


# --------------------------------------------------------------------------- dropout
#
# Dropout on P ("A survey of key techniques of large language model pre-training
# systems", p.218, lists it among the operations fused into the attention kernel):
# Pd = P o Z / (1 - t/256) with t = floor(256 p). Z[i][j] = 0 iff byte j % 4 of word
# i % 4 of Philox-4x32-10 at counter (j / 4, i / 4, bh, offset) under key (seed low,
# seed high) is below t.

# Philox-4x32-10 known-answer vectors published with the generator (Salmon, Moraes,
# Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011; the Random123
# distribution's known-answer tests): (counter, key, output).
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


def philox_py(ctr, key):
    """Philox-4x32-10 written out from its definition (Salmon et al., SC 2011, cited above)."""
    m = 0xFFFFFFFF
    x0, x1, x2, x3 = ctr
    k0, k1 = key
    for r in range(10):
        if r:
            k0, k1 = (k0 + 0x9E3779B9) & m, (k1 + 0xBB67AE85) & m
        a, b = 0xD2511F53 * x0, 0xCD9E8D57 * x2
        x0, x1, x2, x3 = (b >> 32) ^ x1 ^ k0, b & m, (a >> 32) ^ x3 ^ k1, a & m
    return (x0, x1, x2, x3)


def dropout_threshold(p):
    """The byte threshold t = floor(256 p); the drop probability is t / 256."""
    return min(math.floor(p * 256.0), 255)


def dropout_keep(N, bh, p, seed, offset):
    """Z of one head, [N, N] of 0/1, from philox_py: the block at counter
    (j // 4, i // 4, bh, offset) gives query i its word i % 4 and key j byte j % 4 of
    it; a byte below floor(256 p) drops the pair."""
    t = dropout_threshold(p)
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    Z = np.zeros((N, N))
    for i4 in range((N + 3) // 4):
        for j4 in range((N + 3) // 4):
            w = philox_py((j4, i4, bh, offset), key)
            for r in range(4):
                for b in range(4):
                    i, j = 4 * i4 + r, 4 * j4 + b
                    if i < N and j < N:
                        Z[i, j] = 1.0 if (w[r] >> (8 * b)) & 0xFF >= t else 0.0
    return Z


def dropout_scale(p):
    """1 / (1 - t/256): the kept values' factor for the rounded drop probability."""
    return 256.0 / (256.0 - dropout_threshold(p))


def pin_philox_known_answers(orc):
    """The oracle's Philox-4x32-10 reproduces the published known-answer vectors and
    agrees with the definition written out here on random counters and keys."""
    for ctr, key, want in PHILOX_KAT:
        assert tuple(int(x) for x in orc.philox(ctr, key)) == want, f"Philox KAT {ctr}"
        assert philox_py(ctr, key) == want
    rng = _rng(31)
    for _ in range(64):
        ctr = tuple(int(x) for x in rng.integers(0, 2**32, 4))
        key = tuple(int(x) for x in rng.integers(0, 2**32, 2))
        assert tuple(int(x) for x in orc.philox(ctr, key)) == philox_py(ctr, key)


def pin_dropout_reduces_to_softmax_and_generator(orc):
    """With dropout, O = (P o Z / (1 - t/256)) V with P from the (pinned) softmax, Z
    from the generator above and t = floor(256 p), L is the logits' log-sum-exp
    without dropout, and p = 0 is exactly no dropout."""
    rng = _rng(32)
    B, H, N, d = 1, 2, 37, 6
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    for causal, p, seed, offset in ((False, 0.3, 0x1234_5678_9ABC_DEF0, 7),
                                    (True, 0.75, 42, 0), (False, 0.05, 2**63 + 5, 2**31)):
        O, L = orc.forward(Q, K, V, 0.6, causal, dropout=(p, seed, offset))
        O0, L0 = orc.forward(Q, K, V, 0.6, causal)
        _close(L, L0, 0.0, "L does not depend on dropout")
        for bh in range(B * H):
            P = orc.probs(Q[0, bh], K[0, bh], 0.6, causal)
            Z = dropout_keep(N, bh, p, seed, offset)
            _close(O[0, bh], (P * Z * dropout_scale(p)) @ V[0, bh], 1e-13,
                   f"dropout O (p={p}, head {bh})")
    Op, Lp = orc.forward(Q, K, V, 0.6, True, dropout=(0.0, 99, 3))
    Oz, Lz = orc.forward(Q, K, V, 0.6, True)
    assert np.array_equal(Op, Oz) and np.array_equal(Lp, Lz), "p = 0 must be no dropout"


def pin_dropout_keep_rate(orc):
    """The kept fraction matches 1 - t/256 within 5 binomial standard deviations, and
    different offsets give different masks."""
    N = 160
    assert [dropout_threshold(p) for p in (0.0, 0.1, 0.5, 0.9, 0.999)] == [0, 25, 128, 230, 255]
    for p in (0.1, 0.5, 0.9):
        Z = dropout_keep(N, 3, p, 2024, 11)
        n, pe = Z.size, dropout_threshold(p) / 256.0
        sigma = math.sqrt(n * pe * (1 - pe))
        assert abs(Z.sum() - n * (1 - pe)) <= 5 * sigma, f"keep rate at p={p}"
    # the keep rate of every byte position of every word is the same
    Z = dropout_keep(N, 1, 0.5, 7, 0)
    for r in range(4):
        for b in range(4):
            sub = Z[r::4, b::4]
            sigma = math.sqrt(sub.size * 0.25)
            assert abs(sub.sum() - sub.size * 0.5) <= 5 * sigma, f"word {r} byte {b}"
    # the oracle's masks: rows of P o Z are zero exactly where Z is
    rng = _rng(33)
    q = rng.standard_normal((1, 1, N, N)) * 0.1  # one head width d = N for Q, K and V
    k = rng.standard_normal((1, 1, N, N)) * 0.1
    eye = np.eye(N)[None, None]  # V = I exposes Pd itself as O
    O1, _ = orc.forward(q, k, eye, 0.5, False, dropout=(0.5, 2024, 11))
    O2, _ = orc.forward(q, k, eye, 0.5, False, dropout=(0.5, 2024, 12))
    Z = dropout_keep(N, 0, 0.5, 2024, 11)
    assert np.array_equal(O1[0, 0] != 0, Z != 0), "zeros of Pd are the dropped keys"
    assert not np.array_equal(O1 != 0, O2 != 0), "offsets must change the mask"


def pin_dropout_finite_differences(orc):
    """Central differences of <dO, O> through dropout (Z fixed by the seed) at N <= 12,
    and D = rowsum(dO o O) computed both ways."""
    rng = _rng(34)
    for N, d, causal, p in ((12, 3, False, 0.4), (9, 4, True, 0.2)):
        Q, K, V, dO = (rng.standard_normal((1, 2, N, d)) for _ in range(4))
        drop = (p, 77, 5)
        dQ, dK, dV, D, Dc = orc.backward(Q, K, V, dO, 0.5, causal, with_check=True,
                                         dropout=drop)
        O, _ = orc.forward(Q, K, V, 0.5, causal, dropout=drop)
        _close(D, np.sum(dO * O, axis=-1), 1e-12, "D = rowsum(dO o O) with dropout")
        _close(D, Dc, 1e-12, "D two ways with dropout")

        def loss(q, k, v):
            o, _ = orc.forward(q, k, v, 0.5, causal, dropout=drop)
            return float(np.sum(o * dO))

        h = 1e-6
        for which, grad in ((0, dQ), (1, dK), (2, dV)):
            num = np.zeros_like(grad)
            for idx in np.ndindex(*grad.shape):
                ap = [Q.copy(), K.copy(), V.copy()]
                am = [Q.copy(), K.copy(), V.copy()]
                ap[which][idx] += h
                am[which][idx] -= h
                num[idx] = (loss(*ap) - loss(*am)) / (2 * h)
            ref = max(1e-3, float(np.max(np.abs(num))))
            err = float(np.max(np.abs(num - grad)))
            assert err <= 1e-6 * ref, (
                f"dropout finite differences of {'QKV'[which]} (N={N}, p={p}): {err:.3e}")


# --------------------------------------------------------------------------- row functions


def pin_row_functions_agree(orc):
    """The row-restricted entry points (used where whole heads are too slow) equal the
    full ones, which the pins above tie down: plain, causal with a window and a block
    mask, and with dropout."""
    rng = _rng(41)
    B, H, N, d = 1, 2, 140, 4
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    blocks = [[1, 0], [1, 1]]
    cases = [dict(), dict(window=(50, -1), block_mask=blocks), dict(dropout=(0.3, 99, 2))]
    for causal, kw in zip((False, True, False), cases):
        O, L = orc.forward(Q, K, V, 0.5, causal, **kw)
        dQ, dK, dV, D = orc.backward(Q, K, V, dO, 0.5, causal, **kw)
        heads = rng.integers(0, B * H, 24)
        rows = rng.integers(0, N, 24)
        Or, Lr = orc.forward_rows(Q, K, V, 0.5, causal, heads, rows, **kw)
        _close(Or, O.reshape(B * H, N, d)[heads, rows], 1e-13, f"forward_rows O {kw}")
        _close(Lr, L.reshape(B * H, N)[heads, rows], 1e-13, f"forward_rows L {kw}")
        dQr, Dr = orc.backward_dq_rows(Q, K, V, dO, 0.5, causal, heads, rows, **kw)
        _close(dQr, dQ.reshape(B * H, N, d)[heads, rows], 1e-13, f"backward_dq_rows dQ {kw}")
        _close(Dr, D.reshape(B * H, N)[heads, rows], 1e-13, f"backward_dq_rows D {kw}")
        head, keys = 1, np.array([0, 3, 64, 127, 128, 139])
        dKr, dVr = orc.backward_dkdv_rows(Q, K, V, dO, 0.5, causal, head,
                                          L.reshape(B * H, N)[head], D.reshape(B * H, N)[head],
                                          keys, **kw)
        _close(dKr, dK.reshape(B * H, N, d)[head, keys], 1e-13, f"backward_dkdv_rows dK {kw}")
        _close(dVr, dV.reshape(B * H, N, d)[head, keys], 1e-13, f"backward_dkdv_rows dV {kw}")


# --------------------------------------------------------------------------- golden


def pin_golden_fixtures(orc):
    """Hand-worked examples stored under tests/golden/ (each with its derivation)."""
    for name in sorted(os.listdir(GOLDEN)):
        if not name.endswith(".json"):
            continue
        with open(os.path.join(GOLDEN, name)) as f:
            fx = json.load(f)
        env = {"math": math, "ln": math.log, "exp": math.exp}

        def ev(x):
            if isinstance(x, list):
                return [ev(y) for y in x]
            return float(eval(x, env)) if isinstance(x, str) else float(x)

        for case in fx["cases"]:
            Q = np.array(ev(case["Q"]), dtype=np.float64)[None, None]
            K = np.array(ev(case["K"]), dtype=np.float64)[None, None]
            V = np.array(ev(case["V"]), dtype=np.float64)[None, None]
            O, L = orc.forward(Q, K, V, float(case["scale"]), bool(case["causal"]))
            _close(O[0, 0], np.array(ev(case["O"])), 1e-13, f"{name}:{case['name']} O")
            _close(L[0, 0], np.array(ev(case["L"])), 1e-13, f"{name}:{case['name']} L")


ALL_PINS = [
    pin_two_block_decomposition,
    pin_rows_sum_to_one,
    pin_constant_key,
    pin_single_key,
    pin_two_level_logits,
    pin_blockwise_loop,
    pin_torch_sdpa,
    pin_finite_differences,
    pin_gradient_invariants,
    pin_golden_fixtures,
    pin_masks_match_library,
    pin_window_closed_forms,
    pin_masked_finite_differences,
    pin_philox_known_answers,
    pin_dropout_reduces_to_softmax_and_generator,
    pin_dropout_keep_rate,
    pin_dropout_finite_differences,
    pin_row_functions_agree,
]
