"""GPU parity: every step of the CUDA path, called through the C ABI, against the fp64 CPU oracle on the
same seeded inputs, at sizes that span several tiles and ragged tails, plus the edge cases (contexts
shorter than one kernel window, lengths off the 16/64 grid, queries in the first blocks, the dense
threshold and one past it, mixed lengths, head_dim 64/128, GQA groups 1/2/8/16)."""
import numpy as np
import pytest
import torch

from gpu_util import (bparams, check_attention, check_selection, dev, dev_i32, f64, host_u16, oparams)
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import (decode_case, f32_to_bf16_bits, prefill_case, tree_case)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()


def gpu_pool(k_u16, old, new, max_new, nk_cap, kern=None):
    K = dev(k_u16)
    B, Lcap, Hkv, d = k_u16.shape
    if kern is None:
        kern = torch.zeros((B, Hkv, nk_cap, d), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32(old), dev_i32(new), max_new, binding.Params(), kern)
    return kern


def gpu_select(w, kern, q_ctx=None, max_ctx=None, params=None):
    p = bparams(params or w.params)
    B, T, Hq, d = w.q.shape
    Hkv = w.k.shape[2]
    max_ctx = max_ctx or int(w.q_ctx.max())
    idx = torch.full((B, T, Hkv, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, T, Hkv), -7, dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, B, T, max_ctx, Hq, Hkv, d)
    qc = dev_i32(w.q_ctx if q_ctx is None else q_ctx)
    binding.infllmv2_block_score_topk(dev(w.q), qc, None, max_ctx, kern, p, idx, cnt, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy()


# ---------------------------------------------------------------------------------------------------
# step 1: kernel pool
# ---------------------------------------------------------------------------------------------------

@pytest.mark.gpu
def test_kv_append_writes_exactly_the_new_rows():
    """infllmv2_kv_append against plain PyTorch indexing: bit-exact, other rows untouched, a position outside
    the cache writes nothing"""
    torch.manual_seed(3)
    B, L, H, d = 5, 300, 2, 128
    K = torch.randn(B, L, H, d, device="cuda").to(torch.bfloat16)
    V = torch.randn(B, L, H, d, device="cuda").to(torch.bfloat16)
    kn = torch.randn(B, H, d, device="cuda").to(torch.bfloat16)
    vn = torch.randn(B, H, d, device="cuda").to(torch.bfloat16)
    pos = torch.tensor([0, 17, 299, -1, 300], dtype=torch.int32, device="cuda")
    Kw, Vw = K.clone(), V.clone()
    for b in range(B):
        p = int(pos[b])
        if 0 <= p < L:
            Kw[b, p] = kn[b]
            Vw[b, p] = vn[b]
    binding.infllmv2_kv_append(kn, vn, pos, K, V)
    torch.cuda.synchronize()
    assert torch.equal(K, Kw) and torch.equal(V, Vw)


@pytest.mark.parametrize("d", [64, 128])
def test_kernel_pool_bulk_and_incremental(oracle, d):
    rng = np.random.default_rng(100 + d)
    lens = np.array([1000, 777, 31, 32], np.int32)
    Lcap = 1008
    K = f32_to_bf16_bits(rng.standard_normal((4, Lcap, 2, d)).astype(np.float32))
    nk_cap = oracle.num_kernels(1000)
    want = oracle.kernel_pool(K, [0] * 4, lens, 32, 16, nk_cap=nk_cap)
    got = host_u16(gpu_pool(K, np.zeros(4), lens, 1000, nk_cap))
    assert np.array_equal(got, want)
    # incremental: grow by 1, then by 13, then by 200 keys
    kern = gpu_pool(K, np.zeros(4), np.array([500, 400, 0, 1]), 500, nk_cap)
    cur = np.array([500, 400, 0, 1])
    for step in (1, 13, 200, 1000):
        new = np.minimum(cur + step, lens)
        gpu_pool(K, cur, new, step, nk_cap, kern=kern)
        cur = new
    assert np.array_equal(host_u16(kern), want)


@pytest.mark.parametrize("d", [64, 128])
def test_kernel_pool_rounds_the_exact_mean_once(oracle, d):
    """Windows whose exact sum sits a hair beside a bf16 midpoint, or exactly on one: the kernel must be the
    exact mean rounded once (bits worked out by hand in tests/pool_midpoints.py), in bulk and one key at a
    time."""
    from pool_midpoints import midpoint_case
    K, want = midpoint_case(d)
    L = K.shape[1]
    assert np.array_equal(oracle.kernel_pool(K, [0], [L], 32, 16), want)
    got = host_u16(gpu_pool(K, np.zeros(1), np.array([L]), L, want.shape[2]))
    assert np.array_equal(got, want)
    kern = gpu_pool(K, np.zeros(1), np.zeros(1), 1, want.shape[2])
    for n in range(1, L + 1):
        gpu_pool(K, np.array([n - 1]), np.array([n]), 1, want.shape[2], kern=kern)
    assert np.array_equal(host_u16(kern), want)


# ---------------------------------------------------------------------------------------------------
# step 2: scoring + selection
# ---------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("membership", [0, 1])
def test_selection_tiny_prefill_tile_path(oracle, membership):
    """2048-token prefill, 4/2 heads, d 64, top-8 (token-tile path, many tiles, G = 2)."""
    w = prefill_case(2048, 4, 2, 64, topk=8, dense_len=0, seed=1001, n_needles=3, membership=membership)
    nk_cap = oracle.num_kernels(2048)
    kern_o = oracle.kernel_pool(w.k, [0], [2048], 32, 16, nk_cap=nk_cap)
    kern = gpu_pool(w.k, [0], [2048], 2048, nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, oparams(w.params))
    gidx, gcnt = gpu_select(w, kern)
    same = check_selection(gidx, gcnt, r)
    assert same.mean() > 0.99


@pytest.mark.parametrize("G,d", [(16, 128), (8, 64), (1, 128), (2, 64)])
def test_selection_tile_path_groups(oracle, G, d):
    """Ragged prefill length, dense rows at the start (dense_len 300), other group sizes."""
    T = 1337
    w = prefill_case(T, 2 * G, 2, d, topk=6, dense_len=300, seed=200 + G, n_needles=2)
    nk_cap = oracle.num_kernels(T)
    kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
    kern = gpu_pool(w.k, [0], [T], T, nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, oparams(w.params))
    gidx, gcnt = gpu_select(w, kern)
    check_selection(gidx, gcnt, r)


@pytest.mark.parametrize("stride", [2, 4, 8])
def test_selection_lse_estimate_tile_path(oracle, stride):
    """lse_stride = s on the tensor-core prefill scoring against the oracle's same reading of the pages'
    LogSumExp estimation (the LSE from every s-th visible kernel, times s; the pages do not define it, so this
    pins the implementation to the reading, not to the pages): bit-exact selection except at the oracle's near
    ties.  1,500 tokens (ragged last tile, 24 blocks) and 8,500 (133 blocks: three pass-1 stages at s = 2, one
    at s = 8)"""
    for T, seed in ((1500, 980 + stride), (8500, 990 + stride)):
        w = prefill_case(T, 32, 2, 128, topk=6, dense_len=300, seed=seed, n_needles=3)
        nk_cap = oracle.num_kernels(T)
        kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
        rows = slice(T - 256, T)  # the longest rows: the most pass-1 stages
        q_ctx = w.q_ctx[:, rows]
        r = oracle.block_score_topk(w.q[:, rows], kern_o, q_ctx, oparams(dict(w.params, lse_stride=stride)))
        kern = gpu_pool(w.k, [0], [T], T, nk_cap)
        gidx, gcnt = gpu_select(w, kern, params=dict(w.params, lse_stride=stride))
        check_selection(gidx[:, rows], gcnt[:, rows], r)
        # the exact path on the same inputs differs from the estimate somewhere (the estimate is not a no-op)
        e_idx, _ = gpu_select(w, kern)
        assert not np.array_equal(e_idx, gidx)


@pytest.mark.parametrize("G,d", [(16, 128), (2, 64), (8, 128)])
def test_selection_decode_scan_path(oracle, G, d):
    """Decode rows (scan path): ragged lengths, one at the dense threshold, one just past it, one
    shorter than a kernel window, lengths off the 16/64 grid."""
    lens = [20000, 8192, 8193, 30, 4500, 65]
    w = decode_case(lens, 2 * G, 2, d, topk=16, dense_len=8192, seed=300 + G, n_needles=8)
    nk_cap = oracle.num_kernels(max(lens))
    kern_o = oracle.kernel_pool(w.k, [0] * 6, lens, 32, 16, nk_cap=nk_cap)
    kern = gpu_pool(w.k, [0] * 6, lens, max(lens), nk_cap)
    assert np.array_equal(host_u16(kern), kern_o)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, oparams(w.params))
    gidx, gcnt = gpu_select(w, kern)
    check_selection(gidx, gcnt, r)
    # needles are found (sanity; sequence 0 is the only sparse row long enough to hold 8 needles)
    for b in (0,):
        for g in range(2):
            assert np.isin(w.extras["needles"][b], gidx[b, 0, g]).mean() >= 0.5


def test_selection_explicit_q_ctx_and_early_blocks(oracle):
    """Queries in block 0 and 1, contexts below one window, explicit per-query context lengths."""
    rng = np.random.default_rng(400)
    T = 100
    w = prefill_case(T, 32, 2, 128, topk=2, dense_len=0, seed=400, n_needles=0)
    q_ctx = np.sort(rng.integers(1, T + 1, size=(1, T))).astype(np.int32)
    q_ctx[0, :5] = [1, 2, 31, 32, 33]
    nk_cap = oracle.num_kernels(T)
    kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
    kern = gpu_pool(w.k, [0], [T], T, nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, q_ctx, oparams(w.params))
    gidx, gcnt = gpu_select(w, kern, q_ctx=q_ctx, max_ctx=T)
    check_selection(gidx, gcnt, r)


# ---------------------------------------------------------------------------------------------------
# step 3: attention (fed the oracle's selection, so it is compared on identical block sets)
# ---------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("G,d,dense_len", [(2, 64, 0), (16, 128, 700), (1, 128, 0), (8, 64, 2000), (16, 64, 300),
                                         (4, 128, 0), (8, 128, 500), (4, 64, 0)])
def test_sparse_prefill_attention(oracle, G, d, dense_len):
    """Every tile shape of the tensor-core kernel (128 / G tokens x G heads; G = 1 runs on mma.sync), a ragged
    last tile, dense rows before dense_len."""
    T = 1500
    w = prefill_case(T, 2 * G, 2, d, topk=5, dense_len=dense_len, seed=500 + G, n_needles=2)
    nk_cap = oracle.num_kernels(T)
    kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
    P = oparams(w.params)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], P)
    out = torch.empty((1, T, 2 * G, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, T, 2 * G), dtype=torch.float32, device="cuda")
    binding.infllmv2_sparse_attn_prefill(dev(w.q), dev(w.k), dev(w.v), None, dev_i32(w.ctx_lens), T,
                                         dev_i32(r["idx"]), dev_i32(r["cnt"]), bparams(w.params), out, lse)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what="prefill")


@pytest.mark.parametrize("G,d", [(16, 128), (2, 64)])
def test_sparse_decode_attention(oracle, G, d):
    lens = [20000, 8192, 8193, 30, 4500, 65]
    w = decode_case(lens, 2 * G, 2, d, topk=16, dense_len=8192, seed=600 + G, n_needles=8)
    nk_cap = oracle.num_kernels(max(lens))
    kern_o = oracle.kernel_pool(w.k, [0] * 6, lens, 32, 16, nk_cap=nk_cap)
    P = oparams(w.params)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], P)
    p = bparams(w.params)
    B, _, Hq, _ = w.q.shape
    out = torch.empty((B, 1, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, Hq), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, B, 1, max(lens), Hq, 2, d)
    binding.infllmv2_sparse_attn_decode(dev(w.q), dev(w.k), dev(w.v), dev_i32(w.ctx_lens), max(lens),
                                        dev_i32(r["idx"]), dev_i32(r["cnt"]), p, out, lse, ws)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what="decode")


@pytest.mark.parametrize("d", [64, 128])
def test_dense_paths(oracle, d):
    T = 700
    w = prefill_case(T, 32, 2, d, topk=1, dense_len=0, seed=700 + d, n_needles=0)
    out_o, lse_o = oracle.dense_attention(w.q, w.k, w.v, w.q_ctx)
    out = torch.empty((1, T, 32, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, T, 32), dtype=torch.float32, device="cuda")
    binding.infllmv2_dense_attn_prefill(dev(w.q), dev(w.k), dev(w.v), None, dev_i32(w.ctx_lens), T, 0.0, out, lse)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what="dense prefill")
    lens = [5000, 1, 64, 777]
    wd = decode_case(lens, 32, 2, d, topk=1, dense_len=0, seed=710 + d, n_needles=0)
    out_o, lse_o = oracle.dense_attention(wd.q, wd.k, wd.v, wd.q_ctx)
    out = torch.empty((4, 1, 32, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 1, 32), dtype=torch.float32, device="cuda")
    p = binding.Params()
    ws = binding.workspace(p, 4, 1, max(lens), 32, 2, d)
    binding.infllmv2_dense_attn_decode(dev(wd.q), dev(wd.k), dev(wd.v), dev_i32(wd.ctx_lens), max(lens), 0.0, out,
                                       lse, ws)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what="dense decode")


@pytest.mark.parametrize("d,G", [(128, 16), (64, 2)])
@pytest.mark.parametrize("window", [1, 37, 64, 100, 2048, 10000])
def test_window_attention_decode(oracle, d, G, window):
    """infllmv2_window_attn_decode (the draft model's sliding window) against the oracle: ragged contexts,
    windows shorter than a block, block-aligned, longer than some contexts"""
    lens = [5000, 1, 64, 777, 130]
    w = decode_case(lens, 2 * G, 2, d, topk=1, dense_len=0, seed=760 + d + window, n_needles=0)
    out_o, lse_o = oracle.window_attention(w.q, w.k, w.v, w.q_ctx, window)
    B = len(lens)
    out = torch.empty((B, 1, 2 * G, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, 2 * G), dtype=torch.float32, device="cuda")
    ws = binding.workspace(binding.Params(), B, 1, max(lens), 2 * G, 2, d)
    binding.infllmv2_window_attn_decode(dev(w.q), dev(w.k), dev(w.v), dev_i32(w.ctx_lens), max(lens), window, 0.0,
                                        out, lse, ws)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what=f"window {window} decode")


@pytest.mark.parametrize("parents", ["random", "chain", "star"])
def test_tree_verify(oracle, parents):
    P_, N = 3000, 16
    par = None
    if parents == "chain":
        par = np.arange(-1, N - 1)
    elif parents == "star":
        par = np.array([-1] + [0] * (N - 1))
    w = tree_case(P_, N, 32, 2, 128, topk=8, dense_len=1024, seed=800, B=2, parents=par)
    nk_cap = oracle.num_kernels(P_)
    kern_o = oracle.kernel_pool(w.k, [0, 0], [P_, P_], 32, 16, nk_cap=nk_cap)
    Pm = oparams(w.params)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, Pm)
    gidx, gcnt = gpu_select(w, gpu_pool(w.k, [0, 0], [P_, P_], P_, nk_cap))
    check_selection(gidx, gcnt, r)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], Pm, w.extras["k_draft"],
                                           w.extras["v_draft"], w.extras["tree_mask"])
    p = bparams(w.params)
    out = torch.empty(w.q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(w.q.shape[:3], dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, 2, N, P_, 32, 2, 128)
    binding.infllmv2_sparse_attn_tree_verify(dev(w.q), dev(w.k), dev(w.v), dev_i32(w.ctx_lens), P_,
                                             dev(w.extras["k_draft"]), dev(w.extras["v_draft"]),
                                             dev_i32(w.extras["tree_mask"].view(np.int32)), dev_i32(r["idx"]),
                                             dev_i32(r["cnt"]), p, out, lse, ws)
    torch.cuda.synchronize()
    check_attention(out, out_o, lse, lse_o, what="tree")


# ---------------------------------------------------------------------------------------------------
# the whole path on the GPU (its own kernels, its own selection) against the oracle
# ---------------------------------------------------------------------------------------------------

def test_end_to_end_tiny_prefill(oracle):
    w = prefill_case(2048, 4, 2, 64, topk=8, dense_len=0, seed=1001, n_needles=3)
    T = 2048
    nk_cap = oracle.num_kernels(T)
    P = oparams(w.params)
    kern_o = oracle.kernel_pool(w.k, [0], [T], 32, 16, nk_cap=nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], P)
    kern = gpu_pool(w.k, [0], [T], T, nk_cap)
    gidx, gcnt = gpu_select(w, kern)
    same = check_selection(gidx, gcnt, r)
    out = torch.empty((1, T, 4, 64), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_sparse_attn_prefill(dev(w.q), dev(w.k), dev(w.v), None, dev_i32(w.ctx_lens), T,
                                         dev_i32(gidx), dev_i32(gcnt), bparams(w.params), out)
    torch.cuda.synchronize()
    row_same = same.all(axis=-1)  # [B, T]: both groups match
    check_attention(out, out_o, mask=row_same, what="end-to-end")
    # rows whose selection differs at a near tie: the oracle's attention on the GPU's own selection
    if not row_same.all():
        out_g, _ = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gidx, gcnt, P)
        check_attention(out, out_g, what="end-to-end (own selection)")


@pytest.mark.parametrize("path", ["scan_few_members", "scan_degenerate", "tile"])
def test_selection_ties_go_to_lower_block(oracle, path):
    """A zero query scores every block identically: the top-k must be the lowest candidate ids, exactly
    (no near-tie excuse here)."""
    if path == "tile":
        w = prefill_case(2000, 32, 2, 128, topk=16, dense_len=0, seed=900, n_needles=0)
    else:
        L = 131000 if path == "scan_degenerate" else 3000
        w = decode_case([L, 2000], 32, 2, 128, topk=64, dense_len=0, seed=901, n_needles=0)
    w.q[:] = 0
    n_all = w.q_ctx.reshape(-1)
    nk_cap = oracle.num_kernels(int(n_all.max()))
    B = w.k.shape[0]
    kern = gpu_pool(w.k, [0] * B, list(w.ctx_lens), int(w.ctx_lens.max()), nk_cap)
    gidx, gcnt = gpu_select(w, kern)
    k = w.params["topk"]
    for b in range(B):
        for t in range(0, w.q.shape[1], 97):
            n = int(w.q_ctx[b, t])
            c = (n - 1) // 64
            cand = [x for x in range(1, c - 1)]
            want = sorted({0, c - 1, c} | set(cand[:k])) if c >= 1 else [0]
            for g in range(2):
                assert list(gidx[b, t, g, :gcnt[b, t, g]]) == want, (b, t, g)
    kern_o = oracle.kernel_pool(w.k, [0] * B, list(w.ctx_lens), 32, 16, nk_cap=nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, oparams(w.params))
    assert np.array_equal(r["idx"], gidx) and np.array_equal(r["cnt"], gcnt)


FUSED_LENS_14 = [20000, 8192, 8193, 30, 4500, 65, 70000]
# 26 rows: more than one wave of 16-CTA clusters, so the launch takes 8-CTA clusters
FUSED_LENS_26 = [20000, 8192, 8193, 30, 4500, 65, 70000, 9000, 12345, 64 * 130 + 1, 40000, 8300, 98304]


# lengths whose last key completes a kernel window ((n - 32) % 16 == 0: 20000, 8192, 70000, 32, 48, 9008, 98304) and
# lengths whose last key completes none
POOL_LENS = FUSED_LENS_14 + [32, 48, 9008, 31, 98304]


@pytest.mark.parametrize("G,d,lens", [(16, 128, POOL_LENS), (2, 64, POOL_LENS), (8, 128, FUSED_LENS_26)])
def test_fused_decode_step_pool_equals_pool_then_step(oracle, G, d, lens):
    """infllmv2_sparse_decode_step_pool against infllmv2_kernel_pool (old = n - 1, new = n) followed by
    infllmv2_sparse_decode_step on the same cache: the kernel cache and idx, cnt, out, lse bit for bit; the pooled
    cache also bit for bit against the oracle's pool over all n keys.  Dense and sparse rows, windows completed
    by the last key or not, 16- and 8-CTA clusters."""
    w = decode_case(lens, 2 * G, 2, d, topk=16, dense_len=8192, seed=670 + G + len(lens), n_needles=8)
    B = len(lens)
    nk_cap = oracle.num_kernels(max(lens))
    p = bparams(w.params)
    K, V, q = dev(w.k), dev(w.v), dev(w.q)
    prev = [n - 1 for n in lens]
    kern_a = gpu_pool(w.k, [0] * B, prev, max(prev), nk_cap)
    kern_b = kern_a.clone()
    L = dev_i32(lens)
    binding.infllmv2_kernel_pool(K, dev_i32(prev), L, 1, p, kern_a)

    def outputs():
        return (torch.full((B, 1, 2, p.kmax), -7, dtype=torch.int32, device="cuda"),
                torch.full((B, 1, 2), -7, dtype=torch.int32, device="cuda"),
                torch.empty((B, 1, 2 * G, d), dtype=torch.bfloat16, device="cuda"),
                torch.empty((B, 1, 2 * G), dtype=torch.float32, device="cuda"))
    a, bb = outputs(), outputs()
    binding.infllmv2_sparse_decode_step(q, kern_a, K, V, L, max(lens), p, *a)
    binding.infllmv2_sparse_decode_step_pool(q, kern_b, K, V, L, max(lens), p, *bb)
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0
    assert torch.equal(kern_a, kern_b), "kernel cache"
    for x, y, name in zip(a, bb, ("idx", "cnt", "out", "lse")):
        assert torch.equal(x, y) or (x.dtype.is_floating_point and torch.equal(x.nan_to_num(), y.nan_to_num())), name
    kern_o = oracle.kernel_pool(w.k, [0] * B, lens, 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern_b), kern_o)


@pytest.mark.parametrize("G,d,lens,membership,topk", [(16, 128, FUSED_LENS_14, 0, 16), (2, 64, FUSED_LENS_14, 0, 16),
                                                      (8, 128, FUSED_LENS_14, 1, 16), (16, 128, FUSED_LENS_26, 0, 16),
                                                      (4, 64, FUSED_LENS_26, 1, 16), (16, 128, FUSED_LENS_14, 0, 1200)])
def test_fused_decode_step(oracle, G, d, lens, membership, topk):
    """infllmv2_sparse_decode_step (scoring + top-k + attention in one cluster kernel) against the oracle:
    ragged lengths, a row at the dense threshold and one past it, rows shorter than one kernel window,
    both block-membership rules, 16-CTA and 8-CTA clusters; k = 1200 gives block lists of over a thousand
    entries (about 70 per CTA) next to rows that select every block."""
    w = decode_case(lens, 2 * G, 2, d, topk=topk, dense_len=8192, seed=650 + G + len(lens), n_needles=8,
                    membership=membership)
    B = len(lens)
    nk_cap = oracle.num_kernels(max(lens))
    P = oparams(w.params)
    kern_o = oracle.kernel_pool(w.k, [0] * B, lens, 32, 16, nk_cap=nk_cap)
    r = oracle.block_score_topk(w.q, kern_o, w.q_ctx, P)
    out_o, lse_o = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], P)
    p = bparams(w.params)
    kern = gpu_pool(w.k, [0] * B, lens, max(lens), nk_cap)
    idx = torch.full((B, 1, 2, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, 1, 2), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((B, 1, 2 * G, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, 2 * G), dtype=torch.float32, device="cuda")
    K, V = dev(w.k), dev(w.v)
    for b, n in enumerate(lens):  # cache rows past a sequence's context must not leak in, even as NaN
        K[b, n:] = float("nan")
        V[b, n:] = float("nan")
    binding.infllmv2_sparse_decode_step(dev(w.q), kern, K, V, dev_i32(w.ctx_lens), max(lens), p, idx, cnt, out, lse)
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_selection(gi, gc, r)
    check_attention(out, out_o, lse, lse_o, mask=same.all(axis=-1), what="fused decode step")
    if not same.all():  # near-tie rows: the oracle's attention on the GPU's own selection
        out_g, lse_g = oracle.sparse_attention(w.q, w.k, w.v, w.q_ctx, gi, gc, P)
        check_attention(out, out_g, lse, lse_g, what="fused decode step (own selection)")
