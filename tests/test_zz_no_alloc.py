"""fa_backward_noalloc: the backward for callers that cannot allocate device memory
(code that must not call cudaMalloc because it may synchronise the device, plugins
whose host application owns all allocations, programs whose memory is reserved by
their own pool). Its workspace is a fixed 32 MiB array inside the library.

Checked through the C ABI against fa_backward (caller-provided workspace) on the
same inputs, for two calls in a row with different shapes, so that the second
call runs on whatever the first left in the shared array: dK and dV must match bit
for bit, dQ (fp32 atomic adds) within two bf16 ulps. The array holds no room for
split key tiles' partial sums, so where fa_backward splits tiles the two agree to
rounding only. This file is collected
last and also passes when run alone in a fresh process (the first call on the GPU
does the one-time address look-up).
"""
import math

import numpy as np
import pytest
import torch

from io_aware_attention_flashattention_b200 import api
from io_aware_attention_flashattention_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

FA_ERR_UNSUPPORTED = 2


def _ptr(t):
    return t.data_ptr()


def _forward(q, k, v, scale, causal):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    api.fa_forward(q, k, v, o, lse, scale, causal)
    return o, lse


def _backward_with_workspace(q, k, v, o, do, lse, scale, causal):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    ws = torch.empty(api.fa_backward_workspace_size(B, H, N, d), dtype=torch.uint8,
                     device=q.device)
    s = torch.cuda.current_stream().cuda_stream
    st = api.lib().fa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, scale, int(causal),
                               _ptr(ws), ws.numel(), s)
    assert st == 0
    return dq, dk, dv


def _backward_noalloc(q, k, v, o, do, lse, scale, causal):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    s = torch.cuda.current_stream().cuda_stream
    st = api.lib().fa_backward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                       _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, scale,
                                       int(causal), s)
    return st, (dq, dk, dv)


@pytest.mark.parametrize("first,second", [
    ((1, 4, 1000, 128, True), (1, 8, 4096, 64, False)),
])
def test_noalloc_matches_workspace_backward_twice(first, second):
    for call, (B, H, N, d, causal) in enumerate((first, second)):
        q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, torch.bfloat16, seed=500 + call))
        scale = 1.0 / math.sqrt(d)
        o, lse = _forward(q, k, v, scale, causal)
        want = _backward_with_workspace(q, k, v, o, do, lse, scale, causal)
        st, got = _backward_noalloc(q, k, v, o, do, lse, scale, causal)
        assert st == 0, api.lib().fa_status_string(st)
        torch.cuda.synchronize()
        assert api.fa_get_status() == 0
        # Same kernels, same inputs: dK and dV are deterministic, so they must be
        # identical bit for bit. dQ is summed with fp32 atomic adds in whatever order
        # the key tiles finish, which moves the fp32 sum by about 1e-6 of its size;
        # after rounding to bf16 an element may land one ulp away. Allowed: 2 bf16
        # ulps at the element's magnitude plus 1e-5 of the largest |dQ|.
        for name, g, w in zip(("dK", "dV"), got[1:], want[1:]):
            assert torch.equal(g, w), f"call {call}: {name} differs from fa_backward's"
        _assert_within_two_ulps(got[0], want[0], f"call {call}: dQ")


def _assert_within_two_ulps(got, want, what):
    g = got.double().cpu().numpy()
    w = want.double().cpu().numpy()
    assert np.all(np.isfinite(g)), f"{what} not fully written"
    mag = np.maximum(np.abs(g), np.abs(w))
    ulp = np.exp2(np.floor(np.log2(np.where(mag > 0, mag, 1.0))) - 7)
    excess = np.abs(g - w) - (2 * ulp + 1e-5 * float(np.abs(w).max()))
    worst = int(np.argmax(excess))
    assert excess.flat[worst] <= 0, (
        f"{what} differs by {abs(g.flat[worst] - w.flat[worst]):.3e} at "
        f"|value| = {abs(w.flat[worst]):.3e}")


def test_noalloc_runs_split_key_tiles_whole():
    """B1 H2 N4096 d128 has 64 key tiles: fa_backward runs each as two CTAs with fp32
    partials in its workspace; the built-in array has no room for those, so
    fa_backward_noalloc runs every tile whole. The two differ only in the order of
    fp32 additions: every gradient within two bf16 ulps."""
    B, H, N, d = 1, 2, 4096, 128
    q, k, v, do = (t.cuda() for t in make_inputs(B, H, N, d, torch.bfloat16, seed=520))
    scale = 1.0 / math.sqrt(d)
    o, lse = _forward(q, k, v, scale, False)
    want = _backward_with_workspace(q, k, v, o, do, lse, scale, False)
    st, got = _backward_noalloc(q, k, v, o, do, lse, scale, False)
    assert st == 0, api.lib().fa_status_string(st)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    for name, g, w in zip(("dQ", "dK", "dV"), got, want):
        _assert_within_two_ulps(g, w, name)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    B, H, N, d = 1, 8, 16384, 128  # needs 68 MB of workspace, more than the 32 MiB built in
    assert api.fa_backward_workspace_size(B, H, N, d) > 32 << 20
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    dq = torch.full_like(q, float("nan"))
    s = torch.cuda.current_stream().cuda_stream
    st = api.lib().fa_backward_noalloc(_ptr(q), _ptr(q), _ptr(q), _ptr(q), _ptr(q), _ptr(lse),
                                       _ptr(dq), _ptr(dq), _ptr(dq), B, H, N, d, 0.088, 0, s)
    assert st == FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.isnan(dq).all(), "a rejected call must launch nothing"
