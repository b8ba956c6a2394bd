"""The allocation-free decode entry point (infllmv2_sparse_attn_decode_noalloc).

It serves callers that cannot allocate device memory when they call, by keeping the split partials in a
static 4 MiB device array inside the library.  Checked here through the C ABI against the workspace entry
point (infllmv2_sparse_attn_decode) on the same inputs, two calls in a row with different data, within
the attention tolerance of the parity tests; and a call too large for the array is refused."""
import numpy as np
import pytest
import torch

from gpu_util import ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, dev, dev_i32
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import decode_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _decode_inputs(seed):
    lens = [20000, 9000, 70000, 8192]
    w = decode_case(lens, 32, 2, 128, topk=64, dense_len=8192, seed=seed, n_needles=8)
    p = binding.Params(**w.params)
    B = len(lens)
    K, V, q = dev(w.k), dev(w.v), dev(w.q)
    L = dev_i32(w.ctx_lens)
    max_ctx = max(lens)
    nk_cap = binding.num_kernels(max_ctx)
    kern = torch.zeros((B, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(B)), L, max_ctx, p, kern)
    idx = torch.empty((B, 1, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, 1, 2), dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, B, 1, max_ctx, 32, 2, 128)
    binding.infllmv2_block_score_topk(q, None, L, max_ctx, kern, p, idx, cnt, ws)
    return p, q, K, V, L, max_ctx, idx, cnt, ws


def test_decode_noalloc_matches_workspace_entry_point():
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()
    for seed in (1501, 1502):  # two calls in a row, different data
        p, q, K, V, L, max_ctx, idx, cnt, ws = _decode_inputs(seed)
        B = q.shape[0]
        out_ws = torch.empty((B, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
        lse_ws = torch.empty((B, 1, 32), dtype=torch.float32, device="cuda")
        binding.infllmv2_sparse_attn_decode(q, K, V, L, max_ctx, idx, cnt, p, out_ws, lse_ws, ws)
        out_na = torch.full_like(out_ws, float("nan"))
        lse_na = torch.full_like(lse_ws, float("nan"))
        binding.infllmv2_sparse_attn_decode_noalloc(q, K, V, L, max_ctx, idx, cnt, p, out_na, lse_na)
        torch.cuda.synchronize()
        diff = (out_na.float() - out_ws.float()).abs()
        assert torch.isfinite(out_na.float()).all()
        assert diff.max().item() <= ATTN_MAX_ABS and diff.mean().item() <= ATTN_MEAN_ABS
        assert (lse_na - lse_ws).abs().max().item() <= LSE_ABS


def test_decode_noalloc_refuses_calls_larger_than_its_array():
    binding.load()
    p = binding.Params(topk=64, dense_len=8192)
    B = 64  # 64 sequences x 2 groups x 32 splits x 8320 B > 4 MiB
    q = torch.zeros((B, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((B, 8192, 2, 128), dtype=torch.bfloat16, device="cuda")
    L = torch.full((B,), 8192, dtype=torch.int32, device="cuda")
    idx = torch.zeros((B, 1, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.ones((B, 1, 2), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(binding.Infllmv2Error) as err:
        binding.infllmv2_sparse_attn_decode_noalloc(q, K, K, L, 8192, idx, cnt, p, out)
    assert err.value.status == 3
