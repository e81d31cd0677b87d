"""The seeded input generator shared by the oracle tests and the CUDA tests (CPU only):
same seed, same bits; the documented recipe; the workload table."""
import math

import torch

from io_aware_attention_flashattention_b200.inputs import WORKLOADS, make_inputs, workload_inputs


def test_same_seed_same_bits_and_different_seeds_differ():
    a = make_inputs(1, 2, 33, 64, torch.bfloat16, seed=7)
    b = make_inputs(1, 2, 33, 64, torch.bfloat16, seed=7)
    c = make_inputs(1, 2, 33, 64, torch.bfloat16, seed=8)
    for x, y, z in zip(a, b, c):
        assert x.dtype == torch.bfloat16 and tuple(x.shape) == (1, 2, 33, 64)
        assert torch.equal(x, y)
        assert not torch.equal(x, z)


def test_recipe_draw_order_gain_and_rounding():
    """Q, K, V, dO are four fp32 randn draws in that order from one CPU generator; Q and
    K are scaled by the gain before the cast, which rounds to nearest even."""
    shape = (2, 1, 5, 64)
    g = torch.Generator().manual_seed(1234)
    raw = [torch.randn(shape, generator=g, dtype=torch.float32) for _ in range(4)]
    q, k, v, do = make_inputs(*shape, torch.float16, seed=1234, qk_gain=8.0)
    assert torch.equal(q, (raw[0] * 8.0).to(torch.float16))
    assert torch.equal(k, (raw[1] * 8.0).to(torch.float16))
    assert torch.equal(v, raw[2].to(torch.float16))
    assert torch.equal(do, raw[3].to(torch.float16))
    q32, *_ = make_inputs(*shape, torch.float32, seed=1234)
    assert torch.equal(q32, raw[0])


def test_workload_table():
    for k, (name, w) in enumerate(WORKLOADS.items(), start=1):
        assert w.name == name
        assert w.seed == 1000 + k
        assert w.fwd_flops() == 4.0 * w.B * w.H * w.N ** 2 * w.d / (2 if w.causal else 1)
        assert w.bwd_flops() == 2.5 * w.fwd_flops()
    assert WORKLOADS["gpt2_causal_b8h12_n1024_d64"].scale == 1.0 / 8.0
    assert WORKLOADS["long_b1h8_n16384_d128"].scale == 1.0 / math.sqrt(128)
    assert WORKLOADS["stress_causal_b2h16_n8192_d128_qk8"].qk_gain == 8.0
    assert not WORKLOADS["stress_causal_b2h16_n8192_d128_qk8"].backward
    w = WORKLOADS["oracle_f32_n256_d64"]
    q, k, v, do = workload_inputs(w)
    assert q.dtype == torch.float32 and tuple(q.shape) == w.shape
