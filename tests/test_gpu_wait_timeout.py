"""The bounded-wait error paths of the fused decode step and of the tensor-core prefill attention, driven
without a fault.

infllmv2_test_set_first_wait_limit makes the first kernel-cache wait of every CTA poll a barrier that nothing
arrives on, so it gives up after a few polls while that stage's copy is still in flight -- what a wait whose
copy never lands does after its normal limit.  The step must then end (no hang), report
INFLLMV2_ERR_TIMEOUT through infllmv2_device_status, and leave the device usable: the next call with the
normal wait gives exactly the results of a call made before, and the status is clean again.
"""
import numpy as np
import pytest
import torch

from gpu_util import bparams, dev, dev_i32
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import decode_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

TIMEOUT = 5  # INFLLMV2_ERR_TIMEOUT


def test_fused_decode_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    from trainable_block_sparse_v2_b200.build import build
    build()
    lib = binding.load()
    lens = [40000, 9000, 70000]  # sparse rows: every CTA scans kernels before it attends
    w = decode_case(lens, 32, 2, 128, topk=64, dense_len=8192, seed=1700, n_needles=8)
    p = bparams(w.params)
    B = len(lens)
    K, V, q = dev(w.k), dev(w.v), dev(w.q)
    L = dev_i32(lens)
    nk_cap = binding.num_kernels(max(lens))
    kern = torch.zeros((B, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(B)), L, max(lens), p, kern)

    def step():
        idx = torch.full((B, 1, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B, 1, 2), -7, dtype=torch.int32, device="cuda")
        out = torch.full((B, 1, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 1, 32), float("nan"), dtype=torch.float32, device="cuda")
        binding.infllmv2_sparse_decode_step(q, kern, K, V, L, max(lens), p, idx, cnt, out, lse)
        torch.cuda.synchronize()
        return idx, cnt, out, lse

    assert binding.infllmv2_device_status() == 0
    ref = step()
    assert binding.infllmv2_device_status() == 0
    assert lib.infllmv2_test_set_first_wait_limit(64) == 0
    try:
        step()  # must return: every wait is bounded
        assert binding.infllmv2_device_status() == TIMEOUT
        assert binding.infllmv2_device_status() == 0  # reading clears the record
    finally:
        assert lib.infllmv2_test_set_first_wait_limit(0) == 0
    again = step()
    assert binding.infllmv2_device_status() == 0
    for a, b in zip(ref, again):
        assert torch.equal(a, b) or (a.dtype.is_floating_point and torch.equal(a.nan_to_num(), b.nan_to_num()))


def test_prefill_attention_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    """The same limit on the tensor-core prefill attention: the first wait of every CTA's score-MMA issuer runs
    out, the CTA's roles stop, its producers wait for their copies and its issuers for their MMAs, and the
    next call with the normal waits gives exactly the earlier results."""
    from trainable_block_sparse_v2_b200.build import build
    from trainable_block_sparse_v2_b200.workloads import prefill_case
    build()
    lib = binding.load()
    T = 1500
    w = prefill_case(T, 32, 2, 128, topk=5, dense_len=300, seed=1716, n_needles=2)  # 16 heads per group
    p = bparams(w.params)
    q, K, V = dev(w.q), dev(w.k), dev(w.v)
    L = dev_i32(w.ctx_lens)
    nk_cap = binding.num_kernels(T)
    kern = torch.zeros((1, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(1)), L, T, p, kern)
    idx = torch.empty((1, T, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, T, 2), dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, 1, T, T, 32, 2, 128)
    binding.infllmv2_block_score_topk(q, None, L, T, kern, p, idx, cnt, ws)
    torch.cuda.synchronize()

    def attend():
        out = torch.full((1, T, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((1, T, 32), float("nan"), dtype=torch.float32, device="cuda")
        binding.infllmv2_sparse_attn_prefill(q, K, V, None, L, T, idx, cnt, p, out, lse)
        torch.cuda.synchronize()
        return out, lse

    assert binding.infllmv2_device_status() == 0
    ref = attend()
    assert binding.infllmv2_device_status() == 0
    assert not torch.isnan(ref[0]).any()
    assert lib.infllmv2_test_set_first_wait_limit(64) == 0
    try:
        attend()  # must return: every wait is bounded
        assert binding.infllmv2_device_status() == TIMEOUT
        assert binding.infllmv2_device_status() == 0
    finally:
        assert lib.infllmv2_test_set_first_wait_limit(0) == 0
    again = attend()
    assert binding.infllmv2_device_status() == 0
    for a, b in zip(ref, again):
        assert torch.equal(a, b)


def test_prefill_scoring_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    """The same limit on the tensor-core prefill scoring (16 heads per group, d 128): its MMA issuer's first wait
    runs out, the readers stop and still meet at their named barriers, the producer waits for its copies, and
    the next call selects exactly the earlier blocks."""
    from trainable_block_sparse_v2_b200.build import build
    from trainable_block_sparse_v2_b200.workloads import prefill_case
    build()
    lib = binding.load()
    T = 1500
    w = prefill_case(T, 32, 2, 128, topk=5, dense_len=300, seed=1717, n_needles=2)
    p = bparams(w.params)
    q, K = dev(w.q), dev(w.k)
    L = dev_i32(w.ctx_lens)
    nk_cap = binding.num_kernels(T)
    kern = torch.zeros((1, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(1)), L, T, p, kern)
    ws = binding.workspace(p, 1, T, T, 32, 2, 128)

    def select():
        idx = torch.full((1, T, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1, T, 2), -7, dtype=torch.int32, device="cuda")
        binding.infllmv2_block_score_topk(q, None, L, T, kern, p, idx, cnt, ws)
        torch.cuda.synchronize()
        return idx, cnt

    assert binding.infllmv2_device_status() == 0
    ref = select()
    assert binding.infllmv2_device_status() == 0
    assert bool((ref[1] > 0).all())
    assert lib.infllmv2_test_set_first_wait_limit(64) == 0
    try:
        select()  # must return: every wait is bounded
        assert binding.infllmv2_device_status() == TIMEOUT
        assert binding.infllmv2_device_status() == 0
    finally:
        assert lib.infllmv2_test_set_first_wait_limit(0) == 0
    again = select()
    assert binding.infllmv2_device_status() == 0
    for a, b in zip(ref, again):
        assert torch.equal(a, b)
