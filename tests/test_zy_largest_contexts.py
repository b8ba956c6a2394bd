"""The largest contexts the library takes, against the oracle (run last: the suite's largest caches).

* the fused decode step at its limit, 3072 blocks (196,608 keys), next to a shorter row of the same batch;
* the two-call decode (block scoring + top-k on the scan path, then the split attention) at the library's
  limit of 4096 blocks (262,144 keys);
* prefill rows at 262,144 keys: 16 queries ending the context (explicit q_ctx), scored on the scan path and
  attended by the tensor-core attention.
"""
import numpy as np
import pytest
import torch

from gpu_util import bparams, check_attention, check_selection, dev, dev_i32, host_u16, oparams
from pool_midpoints import rne_bf16_of_exact_mean
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import decode_case, f32_to_bf16_bits

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

FUSED_MAX = 3072 * 64    # blocks per CTA (192) x 16 CTAs
LIBRARY_MAX = 4096 * 64  # the library's context limit


def _pool(w, lens, nk_cap):
    B = len(lens)
    kern = torch.zeros((B, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(dev(w.k), dev_i32(np.zeros(B)), dev_i32(lens), max(lens), bparams(w.params), kern)
    return kern


def test_fused_decode_step_at_its_largest_context(oracle):
    lens = [FUSED_MAX, 131073]
    w = decode_case(lens, 32, 2, 128, topk=64, dense_len=8192, seed=1800, n_needles=16)
    B = len(lens)
    p, P = bparams(w.params), oparams(w.params)
    nk_cap = binding.num_kernels(max(lens))
    kern = _pool(w, lens, nk_cap)
    idx = torch.full((B, 1, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, 1, 2), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((B, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, 32), dtype=torch.float32, device="cuda")
    binding.infllmv2_sparse_decode_step(dev(w.q), kern, dev(w.k), dev(w.v), dev_i32(lens), max(lens), p, idx, cnt,
                                        out, lse)
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0
    kern_o = oracle.kernel_pool(w.k, [0] * B, lens, 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern), kern_o)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    check_selection(gi, gc, r)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P)
    check_attention(out, out_o, lse, lse_o, what="fused decode step at 196,608 keys")


def test_two_call_decode_at_the_library_limit(oracle):
    lens = [LIBRARY_MAX]
    w = decode_case(lens, 32, 2, 128, topk=64, dense_len=8192, seed=1810, n_needles=16)
    p, P = bparams(w.params), oparams(w.params)
    nk_cap = binding.num_kernels(LIBRARY_MAX)
    kern = _pool(w, lens, nk_cap)
    idx = torch.full((1, 1, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1, 1, 2), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 1, 1, LIBRARY_MAX, 32, 2, 128)
    L = dev_i32(lens)
    binding.infllmv2_block_score_topk(dev(w.q), None, L, LIBRARY_MAX, kern, p, idx, cnt, ws)
    binding.infllmv2_sparse_attn_decode(dev(w.q), dev(w.k), dev(w.v), L, LIBRARY_MAX, idx, cnt, p, out, lse, ws)
    torch.cuda.synchronize()
    kern_o = oracle.kernel_pool(w.k, [0], lens, 32, 16, nk_cap=nk_cap)
    kern_g = host_u16(kern)
    # the one window of this cache whose fp32 sum double-rounds: its exact mean rounds to 0x3d0d
    win = (w.k[0, 4016 * 16:4016 * 16 + 32, 1, 34].astype(np.uint32) << 16).view(np.float32)
    assert rne_bf16_of_exact_mean(win) == 0x3D0D == kern_o[0, 1, 4016, 34]
    assert kern_g[0, 1, 4016, 34] == 0x3D0D
    assert np.array_equal(kern_g, kern_o)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    check_selection(gi, gc, r)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P)
    check_attention(out, out_o, lse, lse_o, what="two-call decode at 262,144 keys")


def test_prefill_rows_at_the_library_limit(oracle):
    T = 16
    lens = [LIBRARY_MAX]
    w = decode_case(lens, 32, 2, 128, topk=64, dense_len=8192, seed=1820, n_needles=16)
    rng = np.random.default_rng(1821)
    q = f32_to_bf16_bits(rng.standard_normal((1, T, 32, 128)).astype(np.float32))
    q_ctx = np.arange(LIBRARY_MAX - T + 1, LIBRARY_MAX + 1, dtype=np.int32)[None]  # the context's last 16 rows
    p, P = bparams(w.params), oparams(w.params)
    nk_cap = binding.num_kernels(LIBRARY_MAX)
    kern = _pool(w, lens, nk_cap)
    idx = torch.full((1, T, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1, T, 2), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((1, T, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, T, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 1, T, LIBRARY_MAX, 32, 2, 128)
    qc = dev_i32(q_ctx)
    binding.infllmv2_block_score_topk(dev(q), qc, None, LIBRARY_MAX, kern, p, idx, cnt, ws)
    binding.infllmv2_sparse_attn_prefill(dev(q), dev(w.k), dev(w.v), qc, None, LIBRARY_MAX, idx, cnt, p, out, lse)
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0
    kern_o = oracle.kernel_pool(w.k, [0], lens, 32, 16, nk_cap=nk_cap)
    r = oracle.block_score_topk(q, kern_o, q_ctx, P)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_selection(gidx, gcnt, r)
    # attention on the GPU's own selection: every row is compared
    out_o, lse_o = oracle.sparse_attention(q, w.k, w.v, q_ctx, gidx, gcnt, P)
    check_attention(out, out_o, lse, lse_o, what="prefill rows at 262,144 keys")
    assert same.shape == (1, T, 2)
