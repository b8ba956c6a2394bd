"""The allocation-free decode entry point (infllmv2_sparse_attn_decode_noalloc).

It serves callers that cannot allocate device memory when they call, by keeping the split partials in a
static 4 MiB device array inside the library.  Checked here through the C ABI against the workspace entry
point (infllmv2_sparse_attn_decode) and against the fp64 oracle on the same inputs, within the attention
tolerance of the parity tests, over consecutive calls: two large calls with different data, then a smaller
call (fewer rows, fewer splits, head_dim 64, no lse) that must not read the larger calls' leftovers in the
shared array; and a call too large for the array is refused."""
import numpy as np
import pytest
import torch

from gpu_util import ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, check_attention, dev, dev_i32, oparams
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import decode_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

# (seed, context lengths, query heads, KV heads, head_dim, with lse)
CALLS = [
    (1501, [20000, 9000, 70000, 8192], 32, 2, 128, True),
    (1502, [20000, 9000, 70000, 8192], 32, 2, 128, True),
    (1503, [3000, 12000], 8, 2, 64, False),
]


def _decode_inputs(seed, lens, Hq, Hkv, d):
    w = decode_case(lens, Hq, Hkv, d, topk=64, dense_len=8192, seed=seed, n_needles=8)
    p = binding.Params(**w.params)
    B = len(lens)
    K, V, q = dev(w.k), dev(w.v), dev(w.q)
    L = dev_i32(w.ctx_lens)
    max_ctx = max(lens)
    nk_cap = binding.num_kernels(max_ctx)
    kern = torch.zeros((B, Hkv, nk_cap, d), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(B)), L, max_ctx, p, kern)
    idx = torch.empty((B, 1, Hkv, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, 1, Hkv), dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, B, 1, max_ctx, Hq, Hkv, d)
    binding.infllmv2_block_score_topk(q, None, L, max_ctx, kern, p, idx, cnt, ws)
    return w, p, q, K, V, L, max_ctx, idx, cnt, ws


def test_decode_noalloc_matches_workspace_entry_point_and_oracle(oracle):
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()
    for seed, lens, Hq, Hkv, d, with_lse in CALLS:  # consecutive calls, different data and shapes
        w, p, q, K, V, L, max_ctx, idx, cnt, ws = _decode_inputs(seed, lens, Hq, Hkv, d)
        B = q.shape[0]
        out_ws = torch.empty((B, 1, Hq, d), dtype=torch.bfloat16, device="cuda")
        lse_ws = torch.empty((B, 1, Hq), dtype=torch.float32, device="cuda")
        binding.infllmv2_sparse_attn_decode(q, K, V, L, max_ctx, idx, cnt, p, out_ws, lse_ws, ws)
        out_na = torch.full_like(out_ws, float("nan"))
        lse_na = torch.full_like(lse_ws, float("nan")) if with_lse else None
        binding.infllmv2_sparse_attn_decode_noalloc(q, K, V, L, max_ctx, idx, cnt, p, out_na, lse_na)
        torch.cuda.synchronize()
        assert binding.infllmv2_device_status() == 0
        assert torch.isfinite(out_na.float()).all()
        diff = (out_na.float() - out_ws.float()).abs()
        assert diff.max().item() <= ATTN_MAX_ABS and diff.mean().item() <= ATTN_MEAN_ABS
        if with_lse:
            assert (lse_na - lse_ws).abs().max().item() <= LSE_ABS
        # the fp64 oracle's attention over the same selection
        out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, idx.cpu().numpy(), cnt.cpu().numpy(),
                                               oparams(w.params))
        check_attention(out_na, out_o, lse_na, lse_o if with_lse else None, what=f"no-alloc decode, seed {seed}")


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
