"""Stream order across back-to-back launches.

Every kernel of the library is launched with programmatic stream serialization: its
CTAs may be placed, and run their set-up, while the grid before it on the stream is
still finishing, and each waits for that grid before its first global memory access.
These tests queue calls with no synchronisation between them, so that a kernel that
touched memory too early would read a buffer before it was written (the backward's
preprocess reading O, a block mask built by the kernel just before) or overwrite one
that the grid before still reads (the next forward writing O and LSE, the next
backward zeroing the shared workspace). Each result is compared with the same calls
run one at a time, with a device synchronisation after each: dK, dV, O and LSE bit
for bit (their kernels are deterministic), dQ within two units in the last place of
bf16 (its fp32 atomic adds may land in another order).
"""
import math

import pytest
import torch

from io_aware_attention_flashattention_b200 import api
from io_aware_attention_flashattention_b200.inputs import make_inputs_device

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, d, seed, dtype=torch.bfloat16):
    return make_inputs_device(B, H, N, d, dtype, seed)


def _assert_dq_close(got, want):
    g, w = got.float(), want.float()
    assert torch.isfinite(g).all()
    bound = 2.0 ** -6 * w.abs() + 1e-6 * float(w.abs().max())
    worst = float(((g - w).abs() - bound).max())
    assert worst <= 0.0, (
        f"dQ differs from the one-call-at-a-time run by more than 2 ulp ({worst:.3e})")


def _chain(sets, B, H, N, d, causal, sync, fwd, bwd, dtype=torch.bfloat16, **kw):
    """forward(i) then backward(i) for each input set i, into one O / LSE / workspace."""
    dev = sets[0][0].device
    O = torch.full((B, H, N, d), float("nan"), dtype=dtype, device=dev)
    LSE = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    ws = api.workspace_for(sets[0][0])
    scale = 1.0 / math.sqrt(d)
    grads = []
    torch.cuda.synchronize()
    for Q, K, V, dO in sets:
        dQ, dK, dV = (torch.full_like(Q, float("nan")) for _ in range(3))
        fwd(Q, K, V, O, LSE, scale, causal, **kw)
        if sync:
            torch.cuda.synchronize()
        bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, scale, causal, ws, **kw)
        if sync:
            torch.cuda.synchronize()
        grads.append((dQ, dK, dV))
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    return O, LSE, grads


def _compare(a, b):
    Oa, La, ga = a
    Ob, Lb, gb = b
    assert torch.equal(Oa, Ob) and torch.equal(La, Lb), "O / LSE of the last forward differ"
    for (dqa, dka, dva), (dqb, dkb, dvb) in zip(ga, gb):
        assert torch.equal(dka, dkb), "dK differs"
        assert torch.equal(dva, dvb), "dV differs"
        _assert_dq_close(dqa, dqb)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 8, 4096, 128, False),   # one-CTA forward, persistent backward
    (8, 12, 1024, 64, True),    # persistent forward and backward
    (1, 2, 4096, 128, False),   # backward with split key tiles
])
def test_back_to_back_calls_match_one_at_a_time(B, H, N, d, causal):
    sets = [_inputs(B, H, N, d, seed) for seed in (11, 12, 11, 13)]
    queued = _chain(sets, B, H, N, d, causal, False, api.fa_forward, api.fa_backward)
    single = _chain(sets, B, H, N, d, causal, True, api.fa_forward, api.fa_backward)
    _compare(queued, single)


def test_block_mask_built_just_before_the_call():
    B, H, N, d = 1, 4, 2048, 128
    T = (N + 127) // 128
    sets = [_inputs(B, H, N, d, seed) for seed in (21, 22)]

    def run(sync):
        g = torch.Generator(device="cuda").manual_seed(5)
        # built by torch kernels queued right before the library's launches
        bm = (torch.rand((T, T), generator=g, device="cuda") < 0.3).to(torch.uint8)
        bm.fill_diagonal_(1)
        if sync:
            torch.cuda.synchronize()
        out = _chain(sets, B, H, N, d, True, sync, api.fa_forward_masked, api.fa_backward_masked,
                     window=(700, -1), block_mask=bm)
        return out

    _compare(run(False), run(True))


def test_fp32_back_to_back_calls_match_one_at_a_time():
    B, H, N, d = 1, 2, 384, 64
    sets = [_inputs(B, H, N, d, seed, torch.float32) for seed in (31, 32)]
    queued = _chain(sets, B, H, N, d, True, False, api.fa_forward_f32, api.fa_backward_f32,
                    dtype=torch.float32)
    single = _chain(sets, B, H, N, d, True, True, api.fa_forward_f32, api.fa_backward_f32,
                    dtype=torch.float32)
    # the fp32 backward is deterministic throughout, dQ included
    Oa, La, ga = queued
    Ob, Lb, gb = single
    assert torch.equal(Oa, Ob) and torch.equal(La, Lb)
    for x, y in zip(ga, gb):
        for a, b in zip(x, y):
            assert torch.equal(a, b)
