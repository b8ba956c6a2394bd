"""GPU parity at the workloads' full sizes, in the same call sequence the benchmark times, on outputs the
oracle computes one by one (sampled query rows and decode steps)."""
import numpy as np
import pytest
import torch

from gpu_util import bparams, check_attention, check_selection, dev, dev_i32, host_u16, oparams
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()


def nk(n):
    return binding.num_kernels(n)


def test_decode_32k(oracle):
    """batch 1, 32K context; kernels pooled up to the previous token, then the step's incremental pool."""
    w = W.decode_32k()
    L = int(w.ctx_lens[0])
    p, P = bparams(w.params), oparams(w.params)
    K, V, q = dev(w.k), dev(w.v), dev(w.q)
    nk_cap = nk(L)
    kern = torch.zeros((1, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32([0]), dev_i32([L - 1]), L, p, kern)
    binding.infllmv2_kernel_pool(K, dev_i32([L - 1]), dev_i32([L]), 1, p, kern)
    idx = torch.empty((1, 1, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, 1, 2), dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 1, 1, L, 32, 2, 128)
    lens = dev_i32(w.ctx_lens)
    binding.infllmv2_block_score_topk(q, None, lens, L, kern, p, idx, cnt, ws)
    binding.infllmv2_sparse_attn_decode(q, K, V, lens, L, idx, cnt, p, out, lse, ws)
    torch.cuda.synchronize()
    kern_o = oracle.kernel_pool(w.k, [0], [L], 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern), kern_o)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    check_selection(gi, gc, r)
    # attention on the GPU's own selection (the oracle's wherever the two agree): no row is excused
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P)
    check_attention(out, out_o, lse, lse_o, what="decode 32K")
    # needles planted toward this query are selected (sanity)
    for g in range(2):
        assert np.isin(w.extras["needles"][0], idx[0, 0, g].cpu().numpy()).mean() >= 0.75


def test_decode_32k_and_128k_fused_step(oracle):
    """The fused decode step at full size: 32K (batch 1) and the 128K ragged batch at its first step."""
    for w in (W.decode_32k(), W.decode_128k_ragged(steps=1)):
        B = w.q.shape[0]
        L = w.ctx_lens.astype(np.int64)
        p, P = bparams(w.params), oparams(w.params)
        K, V, q = dev(w.k), dev(w.v), dev(w.q)
        max_ctx = int(L.max())
        nk_cap = nk(max_ctx)
        kern = torch.zeros((B, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
        binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(B)), dev_i32(L), max_ctx, p, kern)
        idx = torch.empty((B, 1, 2, p.kmax), dtype=torch.int32, device="cuda")
        cnt = torch.empty((B, 1, 2), dtype=torch.int32, device="cuda")
        out = torch.empty((B, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, 1, 32), dtype=torch.float32, device="cuda")
        binding.infllmv2_sparse_decode_step(q, kern, K, V, dev_i32(L), max_ctx, p, idx, cnt, out, lse)
        torch.cuda.synchronize()
        kern_o = oracle.kernel_pool(w.k, np.zeros(B), L, 32, 16, nk_cap=nk_cap)
        r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
        gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
        check_selection(gi, gc, r)
        out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P)
        check_attention(out, out_o, lse, lse_o, what=f"fused decode {w.name}")


def test_prefill_32k_sampled_rows(oracle):
    """32K prefill, dense below 8192; rows sampled across the dense part, the switch and the sparse part."""
    w = W.prefill_32k()
    T = w.q.shape[1]
    p, P = bparams(w.params), oparams(w.params)
    q, K, V = dev(w.q), dev(w.k), dev(w.v)
    lens = dev_i32(w.ctx_lens)
    nk_cap = nk(T)
    kern = torch.zeros((1, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((1, T, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, T, 2), dtype=torch.int32, device="cuda")
    out = torch.empty((1, T, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, T, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 1, T, T, 32, 2, 128)
    binding.infllmv2_kernel_pool(K, dev_i32([0]), lens, T, p, kern)
    binding.infllmv2_block_score_topk(q, None, lens, T, kern, p, idx, cnt, ws)
    binding.infllmv2_sparse_attn_prefill(q, K, V, None, lens, T, idx, cnt, p, out, lse)
    torch.cuda.synchronize()
    kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern), kern_o)
    rng = np.random.default_rng(3)
    # whole 8-token tiles: the first 64 rows, every tile from 8184 to 8207 (both sides of the dense switch),
    # tiles around 16K, the last 64 rows; then random rows up to 1,088
    fixed = np.concatenate([np.arange(0, 64), np.arange(8184, 8208), np.arange(16376, 16392),
                            np.arange(T - 64, T), [4095, 4096, 24575, 24576]])
    rest = rng.choice(np.setdiff1d(np.arange(T), fixed), 1088 - len(np.unique(fixed)), replace=False)
    rows = np.unique(np.concatenate([fixed, rest]))
    assert len(rows) >= 1024
    r = oracle.block_score_topk(w.q[:, rows], kern_o, w.q_ctx[:, rows], P)
    gidx = idx.cpu().numpy()[:, rows]
    gcnt = cnt.cpu().numpy()[:, rows]
    check_selection(gidx, gcnt, r)
    # attention on the GPU's own selection: every sampled row is compared
    out_g, lse_g = oracle.sparse_attention(w.q[:, rows], w.k, w.v, w.q_ctx[:, rows], gidx, gcnt, P)
    check_attention(out[:, rows], out_g, lse[:, rows], lse_g, what="prefill 32K (own selection)")
    # attention on exactly the oracle's sets for the sampled rows
    out_o, lse_o = oracle.sparse_attention(w.q[:, rows], w.k, w.v, w.q_ctx[:, rows], r["idx"], r["cnt"], P)
    idx2, cnt2 = idx.clone(), cnt.clone()
    idx2[:, rows] = dev_i32(r["idx"])
    cnt2[:, rows] = dev_i32(r["cnt"])
    binding.infllmv2_sparse_attn_prefill(q, K, V, None, lens, T, idx2, cnt2, p, out, lse)
    torch.cuda.synchronize()
    check_attention(out[:, rows], out_o, lse[:, rows], lse_o, what="prefill 32K (oracle selection)")


def test_decode_128k_ragged_steps(oracle):
    """batch 4 ragged 128K, 256 decode steps of incremental pooling; steps 0, 1, 100 and 255 checked."""
    w = W.decode_128k_ragged(steps=256)
    p, P = bparams(w.params), oparams(w.params)
    L0 = w.ctx_lens.astype(np.int64)
    B = 4
    Lcap = w.k.shape[1]
    K, V = dev(w.k), dev(w.v)
    qs = w.extras["q_steps"]
    max_ctx = int(L0.max()) + 255
    nk_cap = nk(max_ctx)
    kern = torch.zeros((B, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(np.zeros(B)), dev_i32(L0 - 1), int(L0.max()), p, kern)
    idx = torch.empty((B, 1, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, 1, 2), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, B, 1, max_ctx, 32, 2, 128)
    check_steps = {0, 1, 100, 255}
    for s in range(256):
        L = L0 + s
        lens, old = dev_i32(L), dev_i32(L - 1)
        q = dev(qs[s])
        binding.infllmv2_kernel_pool(K, old, lens, 1, p, kern)
        binding.infllmv2_block_score_topk(q, None, lens, max_ctx, kern, p, idx, cnt, ws)
        binding.infllmv2_sparse_attn_decode(q, K, V, lens, max_ctx, idx, cnt, p, out, lse, ws)
        if s not in check_steps:
            continue
        torch.cuda.synchronize()
        kern_o = oracle.kernel_pool(w.k, np.zeros(B), L, 32, 16, nk_cap=nk_cap)
        gk = host_u16(kern)
        for b in range(B):
            n_b = nk(int(L[b]))
            assert np.array_equal(gk[b, :, :n_b], kern_o[b, :, :n_b]), f"kernel cache differs at step {s}, seq {b}"
        qctx = L[:, None].astype(np.int32)
        r = oracle.block_score_topk(qs[s], kern_o, qctx, P)
        gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
        check_selection(gi, gc, r)
        out_o, lse_o = oracle.sparse_attention(qs[s], w.k, w.v, qctx, gi, gc, P)
        check_attention(out, out_o, lse, lse_o, what=f"decode 128K step {s}")
    assert Lcap >= max_ctx


def test_tree_verify_64k(oracle):
    w = W.tree_verify_64k()
    P_ = int(w.ctx_lens[0])
    N = w.q.shape[1]
    p, P = bparams(w.params), oparams(w.params)
    K, V = dev(w.k), dev(w.v)
    nk_cap = nk(P_)
    kern = torch.zeros((1, 2, nk_cap, 128), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32([0]), dev_i32([P_]), P_, p, kern)
    idx = torch.empty((1, N, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, N, 2), dtype=torch.int32, device="cuda")
    out = torch.empty((1, N, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, N, 32), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 1, N, P_, 32, 2, 128)
    q = dev(w.q)
    binding.infllmv2_block_score_topk(q, dev_i32(w.q_ctx), None, P_, kern, p, idx, cnt, ws)
    binding.infllmv2_sparse_attn_tree_verify(q, K, V, dev_i32(w.ctx_lens), P_, dev(w.extras["k_draft"]),
                                             dev(w.extras["v_draft"]), dev_i32(w.extras["tree_mask"].view(np.int32)),
                                             idx, cnt, p, out, lse, ws)
    torch.cuda.synchronize()
    kern_o = oracle.kernel_pool(w.k, [0], [P_], 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern), kern_o)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    check_selection(gi, gc, r)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P, w.extras["k_draft"],
                                           w.extras["v_draft"], w.extras["tree_mask"])
    check_attention(out, out_o, lse, lse_o, what="tree 64K")
    # depth <= 6 and every node sees itself
    m = w.extras["tree_mask"][0]
    assert all((int(m[i]) >> i) & 1 for i in range(N)) and max(bin(int(x)).count("1") for x in m) <= 7
