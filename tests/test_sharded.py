"""Head-sharded attention: the partition of B*H into contiguous head ranges, the
gather of per-rank outputs (two gloo ranks on the CPU, with the fp64 oracle standing
in for the GPU kernels), and, on a GPU, the sharded calls against the unsharded
ones and the oracle (several shards placed on one GPU when only one is present)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_attention_flashattention_b200.inputs import make_inputs
from io_aware_attention_flashattention_b200.sharded import rank_heads, shard_ranges


def test_shard_ranges_cover_and_balance():
    for total in (0, 1, 5, 8, 96, 97):
        for parts in (1, 2, 3, 8, 100):
            r = shard_ranges(total, parts)
            assert len(r) == parts
            assert r[0][0] == 0 and r[-1][1] == total
            assert all(r[i][1] == r[i + 1][0] for i in range(parts - 1))  # contiguous
            sizes = [b - a for a, b in r]
            assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    assert rank_heads(2, 3, 1, 4) == (2, 4)  # 6 heads over 4 ranks: 2, 2, 1, 1
    with pytest.raises(ValueError):
        rank_heads(1, 8, 2, 2)
    with pytest.raises(ValueError):
        shard_ranges(4, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import oracle
    from io_aware_attention_flashattention_b200.sharded import gather_heads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        B, H, N, d = 1, 5, 64, 64  # 5 heads over 2 ranks: 3 + 2
        q, k, v, _ = make_inputs(B, H, N, d, torch.float32, seed=77)
        a, b = rank_heads(B, H, rank, world)
        sl = lambda t: t.reshape(B * H, N, d)[a:b].unsqueeze(0)  # noqa: E731
        # this rank's heads (the oracle stands in for the kernels on the CPU)
        O, L = oracle.forward(sl(q), sl(k), sl(v), 0.125, True)
        O_full = gather_heads(torch.from_numpy(O[0]), B, H)
        L_full = gather_heads(torch.from_numpy(L[0]), B, H)
        O_ref, L_ref = oracle.forward(q, k, v, 0.125, True)
        out[rank] = (float(np.max(np.abs(O_full.numpy() - O_ref))),
                     float(np.max(np.abs(L_full.numpy() - L_ref))), (a, b))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_partition_and_gather_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][2] == (0, 3) and res[1][2] == (3, 5)
    for r in (0, 1):
        # each head is computed once, by its owner, with the same definition
        assert res[r][0] == 0.0 and res[r][1] == 0.0


# ------------------------------------------------------------------ on the GPU


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal,nshards", [(1, 5, 640, 128, True, 2),
                                                     (2, 3, 300, 64, False, 4)])
def test_sharded_equals_unsharded_and_oracle(B, H, N, d, causal, nshards):
    import oracle
    from io_aware_attention_flashattention_b200 import api
    from io_aware_attention_flashattention_b200.sharded import (attention_sharded,
                                                                backward_sharded,
                                                                forward_sharded)
    from test_gpu_parity import TOL_BF16, _np, assert_close, assert_close_o, grad_tol

    n_gpu = torch.cuda.device_count()
    devices = [f"cuda:{i % n_gpu}" for i in range(nshards)]
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=600 + N)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    o, lse = forward_sharded(qc, kc, vc, devices, causal)
    dq, dk, dv = backward_sharded(qc, kc, vc, o, lse, doc, devices, causal)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    # per head the sharded call runs the same kernels on the same data: O, LSE, dK and
    # dV are bit-identical to the unsharded call; dQ (fp32 atomic adds) within 2 ulps
    o1, lse1 = api.forward(qc, kc, vc, causal)
    dq1, dk1, dv1 = api.backward(qc, kc, vc, o1, lse1, doc, causal)
    for a, b in ((o, o1), (lse, lse1), (dk, dk1), (dv, dv1)):
        assert torch.equal(a, b)
    g, w = _np(dq), _np(dq1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(g), np.abs(w)), 1e-30))) - 7)
    assert np.all(np.abs(g - w) <= 2 * ulp + 1e-5 * np.abs(w).max())
    # and against the oracle
    O_ref, L_ref = oracle.forward(q, k, v, scale, causal)
    dQ, dK, dV, _ = oracle.backward(q, k, v, do, scale, causal)
    assert_close_o("O", _np(o), O_ref, TOL_BF16["O"])
    assert_close("LSE", _np(lse), L_ref, TOL_BF16["L"])
    for name, got, want in (("dQ", dq, dQ), ("dK", dk, dK), ("dV", dv, dV)):
        assert_close(name, _np(got), want, grad_tol(TOL_BF16, want))
    # the autograd form
    qa, ka, va = (t.clone().requires_grad_() for t in (qc, kc, vc))
    out = attention_sharded(qa, ka, va, devices, causal)
    out.backward(doc)
    assert torch.equal(out.detach(), o)
    assert torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal,nshards", [(1, 5, 640, 128, True, 2),
                                                     (2, 3, 300, 64, False, 3)])
def test_sharded_dropout_draws_the_unsharded_masks(B, H, N, d, causal, nshards):
    """Each shard passes its first flattened head as head_base, so the sharded call
    draws the unsharded call's keep masks: O, LSE, dK and dV bit for bit, dQ within 2
    ulps (fp32 atomic adds); and a different head_base draws other masks."""
    from io_aware_attention_flashattention_b200 import api
    from io_aware_attention_flashattention_b200.sharded import (attention_sharded,
                                                                backward_sharded,
                                                                forward_sharded)
    from test_gpu_parity import _np

    n_gpu = torch.cuda.device_count()
    devices = [f"cuda:{i % n_gpu}" for i in range(nshards)]
    q, k, v, do = make_inputs(B, H, N, d, torch.bfloat16, seed=700 + N)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    drop = (0.2, 4321, 9)
    o, lse = forward_sharded(qc, kc, vc, devices, causal, dropout=drop)
    dq, dk, dv = backward_sharded(qc, kc, vc, o, lse, doc, devices, causal, dropout=drop)
    o1, lse1 = api.forward(qc, kc, vc, causal, dropout=drop)
    dq1, dk1, dv1 = api.backward(qc, kc, vc, o1, lse1, doc, causal, dropout=drop)
    torch.cuda.synchronize()
    assert api.fa_get_status() == 0
    for a, b in ((o, o1), (lse, lse1), (dk, dk1), (dv, dv1)):
        assert torch.equal(a, b)
    g, w = _np(dq), _np(dq1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(g), np.abs(w)), 1e-30))) - 7)
    assert np.all(np.abs(g - w) <= 2 * ulp + 1e-5 * np.abs(w).max())
    # the last head alone, as its own call with head_base = its flattened index
    last = B * H - 1
    qs, ks, vs = (t.reshape(B * H, N, d)[last:].unsqueeze(0).contiguous() for t in (qc, kc, vc))
    os_, _ = api.forward(qs, ks, vs, causal, dropout=drop + (last,))
    assert torch.equal(os_[0, 0], o.reshape(B * H, N, d)[last])
    # with head_base 0 that head draws head 0's mask instead: a different output
    o0, _ = api.forward(qs, ks, vs, causal, dropout=drop)
    assert not torch.equal(o0[0, 0], os_[0, 0])
    # the autograd form
    qa, ka, va = (t.clone().requires_grad_() for t in (qc, kc, vc))
    out = attention_sharded(qa, ka, va, devices, causal, dropout=drop)
    out.backward(doc)
    assert torch.equal(out.detach(), o)
    assert torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)


def test_dropout_tuple_takes_an_optional_head_base():
    from io_aware_attention_flashattention_b200 import api
    from io_aware_attention_flashattention_b200.sharded import _shard_dropout

    assert api._dropout(None) == (0.0, 0, 0, 0)
    assert api._dropout((0.1, 5, 6)) == (0.1, 5, 6, 0)
    assert api._dropout((0.1, 5, 6, 40)) == (0.1, 5, 6, 40)
    with pytest.raises(ValueError):
        api._dropout((0.1, 5, 6, 1, 2))
    assert _shard_dropout(None, 3) is None
    assert _shard_dropout((0.1, 5, 6), 3) == (0.1, 5, 6, 3)
    assert _shard_dropout((0.1, 5, 6, 10), 3) == (0.1, 5, 6, 13)
