"""Whole-tensor parity on the five named workloads at their full sizes: every element
of O and LSE (and of dQ, dK and dV for the workloads with a backward) from the CUDA
library, through its C ABI and in the launch configuration the benchmark times,
against the fp64 oracle on the same seeded inputs.

The oracle materialises S and P of one head at a time (2 GB per head at N = 16384),
so the long workload costs about a minute of host time on 16 cores; the sampled
checks in test_gpu_parity.py remain as fast pre-checks of the same launches.
Tolerances are those of test_gpu_parity.py (the stated bf16 limits; fp32 1e-5).
"""
import dataclasses

import pytest
import torch

from io_aware_attention_flashattention_b200.inputs import WORKLOADS, workload_inputs
from test_gpu_parity import TOL, check_full

pytestmark = pytest.mark.gpu


def _full(w):
    q, k, v, do = workload_inputs(w)
    check_full(q, k, v, do, w.scale, w.causal, TOL[w.dtype], backward=w.backward)


def test_full_oracle_f32_n256_d64():
    _full(WORKLOADS["oracle_f32_n256_d64"])


def test_full_gpt2_causal_b8h12_n1024_d64():
    """All 96 heads: O, LSE, dQ, dK, dV."""
    _full(WORKLOADS["gpt2_causal_b8h12_n1024_d64"])


def test_full_mid_b1h8_n4096_d128():
    _full(WORKLOADS["mid_b1h8_n4096_d128"])


def test_full_mid_b1h8_n4096_d128_in_f16():
    _full(dataclasses.replace(WORKLOADS["mid_b1h8_n4096_d128"], dtype=torch.float16))


def test_full_stress_causal_b2h16_n8192_d128_qk8():
    """Forward only (the workload has no backward): all 32 heads of O and LSE."""
    _full(WORKLOADS["stress_causal_b2h16_n8192_d128_qk8"])


@pytest.mark.slow
def test_full_long_b1h8_n16384_d128():
    """All 8 heads of O, LSE, dQ, dK and dV at N = 16384 (the benchmark's workload)."""
    _full(WORKLOADS["long_b1h8_n16384_d128"])
