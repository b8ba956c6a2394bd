"""GPU parity of the attention backward (gradients for a fixed selection) against the fp64 oracle.

The GPU forward (infllmv2_sparse_attn_prefill) writes out and lse; the backward takes them, with dout, and
returns fp32 dq, dk, dv; the oracle differentiates its own fp64 forward on the same selection.  Error
budget: P and dS enter the tensor-core products rounded to bf16 (relative 2^-9 each) and Dsum = dout . out
uses the bf16 forward output, so per-element errors are a few 1e-3 of the gradient's scale.  Bar, per
tensor: max |gpu - oracle| <= 2e-2 * max |oracle| and mean |gpu - oracle| <= 1e-2 * mean |oracle|.
Cases: sparse and dense rows mixed, GQA groups 1/2/8/16, head_dim 64/128, a cache length off the 64-key
grid, chunked prefill (queries at the end of a longer cache), two sequences, the dense entry (no selection),
and the 32K prefill workload at full size (sampled dq rows against the oracle one by one, and the sum rules
of the softmax Jacobian over all of dk / dv)."""
import numpy as np
import pytest
import torch

from gpu_util import bparams, dev, dev_i32, f64, host_u16, oparams
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import f32_to_bf16_bits, prefill_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

GRAD_MAX_REL = 2e-2
GRAD_MEAN_REL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()


def check_grad(g, ref, what):
    g = g.detach().double().cpu().numpy() if isinstance(g, torch.Tensor) else g
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    scale_max, scale_mean = float(np.abs(ref).max()), float(np.abs(ref).mean())
    if scale_max == 0:  # dq of a query that sees one key: exactly 0 in the oracle, rounding-sized on the GPU
        assert mx <= 1e-4, f"{what}: {mx:.3e} where the oracle is exactly 0"
        return 0.0, 0.0
    print(f"{what}: max-abs / max {mx / scale_max:.2e}, mean-abs / mean {mean / scale_mean:.2e}")
    assert mx <= GRAD_MAX_REL * scale_max and mean <= GRAD_MEAN_REL * scale_mean, \
        f"{what}: max-abs {mx:.3e} (scale {scale_max:.3e}), mean-abs {mean:.3e} (scale {scale_mean:.3e})"
    return mx / scale_max, mean / scale_mean


def gpu_forward_backward(q, k, v, q_ctx, ctx_lens, max_ctx, idx, cnt, params, dout):
    """q, k, v, dout: numpy bf16 bits; idx / cnt numpy int32 or None (dense).  Returns torch tensors."""
    B, T, Hq, d = q.shape
    Lcap, Hkv = k.shape[1], k.shape[2]
    Q, K, V, DO = dev(q), dev(k), dev(v), dev(dout)
    qc = dev_i32(q_ctx) if q_ctx is not None else None
    cl = dev_i32(ctx_lens) if ctx_lens is not None else None
    out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device="cuda")
    p = bparams(params)
    if idx is None:
        binding.infllmv2_dense_attn_prefill(Q, K, V, qc, cl, max_ctx, 0.0, out, lse)
        gi = gc = None
    else:
        gi, gc = dev_i32(idx), dev_i32(cnt)
        binding.infllmv2_sparse_attn_prefill(Q, K, V, qc, cl, max_ctx, gi, gc, p, out, lse)
    dq = torch.full((B, T, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.full((B, Lcap, Hkv, d), float("nan"), dtype=torch.float32, device="cuda")
    dv = torch.full((B, Lcap, Hkv, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = binding.backward_workspace(p, B, T, max_ctx, Hq, Hkv, d)
    ws.fill_(0xAB)  # the workspace needs no initialisation
    binding.infllmv2_sparse_attn_backward(Q, K, V, qc, cl, max_ctx, gi, gc, p, out, lse, DO, dq, dk, dv, ws)
    torch.cuda.synchronize()
    return out, lse, dq, dk, dv


def selection(oracle, w, P):
    B, T = w.q.shape[:2]
    Lcap = w.k.shape[1]
    nk_cap = oracle.num_kernels(Lcap)
    kern = oracle.kernel_pool(w.k, [0] * B, [Lcap] * B, 32, 16, nk_cap=nk_cap)
    return oracle.block_score_topk(w.q, kern, w.q_ctx, P)


@pytest.mark.parametrize("G,d,dense_len,T", [(16, 128, 300, 777), (2, 64, 0, 1000), (8, 128, 1100, 1300),
                                             (1, 64, 100, 450)])
def test_backward_sparse_prefill(oracle, G, d, dense_len, T):
    w = prefill_case(T, 2 * G, 2, d, topk=5, dense_len=dense_len, seed=900 + G + d, n_needles=2)
    P = oparams(w.params)
    r = selection(oracle, w, P)
    rng = np.random.default_rng(901 + G)
    dout = f32_to_bf16_bits(rng.standard_normal(w.q.shape).astype(np.float32))
    _, _, dq, dk, dv = gpu_forward_backward(w.q, w.k, w.v, None, w.ctx_lens, T, r["idx"], r["cnt"], w.params, dout)
    dq_o, dk_o, dv_o = oracle.sparse_attention_backward(w.q, w.k, w.v, w.q_ctx, r["idx"], r["cnt"], P, dout)
    check_grad(dq, dq_o, "dq")
    check_grad(dk, dk_o, "dk")
    check_grad(dv, dv_o, "dv")


def test_backward_dense_entry(oracle):
    """idx = cnt = NULL: the dense attention's backward (every key before n)."""
    T, d = 530, 128
    w = prefill_case(T, 16, 2, d, topk=1, dense_len=0, seed=910, n_needles=0)
    rng = np.random.default_rng(911)
    dout = f32_to_bf16_bits(rng.standard_normal(w.q.shape).astype(np.float32))
    _, _, dq, dk, dv = gpu_forward_backward(w.q, w.k, w.v, None, w.ctx_lens, T, None, None, w.params, dout)
    P = oparams(dict(w.params, dense_len=T))
    nb = (T + 63) // 64
    idx = np.full((1, T, 2, P.kmax), -1, np.int32)
    cnt = np.zeros((1, T, 2), np.int32)
    dq_o, dk_o, dv_o = oracle.sparse_attention_backward(w.q, w.k, w.v, w.q_ctx, idx, cnt, P, dout)
    assert nb > 1
    check_grad(dq, dq_o, "dq")
    check_grad(dk, dk_o, "dk")
    check_grad(dv, dv_o, "dv")


def test_backward_chunked_prefill_two_sequences(oracle):
    """T queries ending two caches of different lengths (ctx_lens path, n = ctx - T + t + 1), rows past the
    dense threshold sparse; cache rows no query reads get exactly zero gradient."""
    rng = np.random.default_rng(920)
    B, T, Lcap, Hq, Hkv, d = 2, 200, 1500, 16, 2, 64
    q = f32_to_bf16_bits(rng.standard_normal((B, T, Hq, d)).astype(np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((B, Lcap, Hkv, d)).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((B, Lcap, Hkv, d)).astype(np.float32))
    dout = f32_to_bf16_bits(rng.standard_normal((B, T, Hq, d)).astype(np.float32))
    ctx = np.array([1500, 1100], np.int32)
    q_ctx = (ctx[:, None] - T + np.arange(T)[None, :] + 1).astype(np.int32)
    params = dict(topk=3, init_blocks=1, local_blocks=2, dense_len=1000, membership=0)
    P = oparams(params)
    kern = oracle.kernel_pool(k, [0, 0], ctx, 32, 16, nk_cap=oracle.num_kernels(Lcap))
    r = oracle.block_score_topk(q, kern, q_ctx, P)
    _, _, dq, dk, dv = gpu_forward_backward(q, k, v, None, ctx, int(ctx.max()), r["idx"], r["cnt"], params, dout)
    dq_o, dk_o, dv_o = oracle.sparse_attention_backward(q, k, v, q_ctx, r["idx"], r["cnt"], P, dout)
    check_grad(dq, dq_o, "dq")
    check_grad(dk, dk_o, "dk")
    check_grad(dv, dv_o, "dv")
    unread = dk_o == 0
    assert unread[1, 1100:].all()
    assert torch.all(dk[1, 1100:] == 0) and torch.all(dv[1, 1100:] == 0)


@pytest.mark.parametrize("G,d", [(16, 128), (4, 64)])
def test_backward_explicit_q_ctx_and_short_rows(oracle, G, d):
    """q_ctx given per query: contexts of 1 key, shorter than a block, on the 64 grid and one past it."""
    rng = np.random.default_rng(930 + G)
    T, Lcap, Hkv = 9, 400, 2
    Hq = G * Hkv
    q = f32_to_bf16_bits(rng.standard_normal((1, T, Hq, d)).astype(np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((1, Lcap, Hkv, d)).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((1, Lcap, Hkv, d)).astype(np.float32))
    dout = f32_to_bf16_bits(rng.standard_normal((1, T, Hq, d)).astype(np.float32))
    q_ctx = np.array([[1, 5, 63, 64, 65, 128, 129, 400, 257]], np.int32)
    params = dict(topk=2, init_blocks=1, local_blocks=1, dense_len=64, membership=0)
    P = oparams(params)
    kern = oracle.kernel_pool(k, [0], [Lcap], 32, 16, nk_cap=oracle.num_kernels(Lcap))
    r = oracle.block_score_topk(q, kern, q_ctx, P)
    _, _, dq, dk, dv = gpu_forward_backward(q, k, v, q_ctx, None, Lcap, r["idx"], r["cnt"], params, dout)
    dq_o, dk_o, dv_o = oracle.sparse_attention_backward(q, k, v, q_ctx, r["idx"], r["cnt"], P, dout)
    # a one-key row has dq = 0 exactly in the oracle; the GPU's is tiny
    check_grad(dq, dq_o, "dq")
    check_grad(dk, dk_o, "dk")
    check_grad(dv, dv_o, "dv")


def test_backward_32k_prefill_full_size(oracle):
    """The 32K prefill workload (32 / 2 heads, d 128, dense below 8192, k = 64) at full size, as the bench
    runs it: dq of sampled rows against the oracle row by row; over all of dk / dv, the identities
    sum_j dk_j = 0, sum_j dv_j = sum of dout over the group's rows, and sum dv . V = sum dout . out."""
    from trainable_block_sparse_v2_b200.workloads import prefill_32k
    w = prefill_32k()
    T = w.q.shape[1]
    Hq, Hkv, d = w.q.shape[2], w.k.shape[2], w.q.shape[3]
    G = Hq // Hkv
    p = bparams(w.params)
    Q, K, V = dev(w.q), dev(w.k), dev(w.v)
    cl = dev_i32(w.ctx_lens)
    kern = torch.zeros((1, Hkv, binding.num_kernels(T), d), dtype=torch.bfloat16, device="cuda")
    binding.infllmv2_kernel_pool(K, dev_i32([0]), cl, T, p, kern)
    idx = torch.empty((1, T, Hkv, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, T, Hkv), dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, 1, T, T, Hq, Hkv, d)
    binding.infllmv2_block_score_topk(Q, None, cl, T, kern, p, idx, cnt, ws)
    out = torch.empty((1, T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, T, Hq), dtype=torch.float32, device="cuda")
    binding.infllmv2_sparse_attn_prefill(Q, K, V, None, cl, T, idx, cnt, p, out, lse)
    gen = torch.Generator(device="cuda").manual_seed(940)
    DO = torch.randn((1, T, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    dq = torch.empty((1, T, Hq, d), dtype=torch.float32, device="cuda")
    dk = torch.empty((1, T, Hkv, d), dtype=torch.float32, device="cuda")
    dv = torch.empty((1, T, Hkv, d), dtype=torch.float32, device="cuda")
    bws = binding.backward_workspace(p, 1, T, T, Hq, Hkv, d)
    binding.infllmv2_sparse_attn_backward(Q, K, V, None, cl, T, idx, cnt, p, out, lse, DO, dq, dk, dv, bws)
    torch.cuda.synchronize()
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    # sampled rows: first, dense, last dense, first sparse, middle, last
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    dout_h = host_u16(DO)
    P = oparams(w.params)
    for t in (0, 100, 8191, 8192, 20000, T - 1):
        qc = np.array([[t + 1]], np.int32)
        dq_o, _, _ = oracle.sparse_attention_backward(w.q[:, t:t + 1], w.k[:, :t + 1], w.v[:, :t + 1], qc,
                                                      idx_h[:, t:t + 1], cnt_h[:, t:t + 1], P,
                                                      dout_h[:, t:t + 1])
        check_grad(dq[:, t:t + 1], dq_o, f"dq row {t}")
    # identities over the whole of dk / dv (fp64 sums of the fp32 results)
    dk64, dv64 = dk.double(), dv.double()
    for g in range(Hkv):
        s_dk = dk64[0, :, g].sum(0)
        assert float(s_dk.abs().max()) <= 1e-3 * float(dk64[0, :, g].abs().sum(0).max())
        want = DO[0, :, g * G:(g + 1) * G].double().sum((0, 1))
        s_dv = dv64[0, :, g].sum(0)
        assert float((s_dv - want).abs().max()) <= 1e-3 * float(want.abs().max() + 1.0)
    lhs = float((dv64 * V.double()).sum())
    rhs = float((DO.double() * out.double()).sum())
    assert abs(lhs - rhs) <= 2e-3 * abs(rhs) + 1.0


# ------------------------------------------------------------------------------------------------
# gradient of the semantic kernels with respect to K (the transpose of the window mean)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
def test_kernel_pool_backward_matches_oracle(oracle, d):
    """Ragged lengths (below one window, off the 16-key grid, at the cache capacity, 0), two KV heads.
    Overwrite: bit-exact with the oracle's fp64 value rounded to fp32 (one fp32 sum of two terms, an exact
    power-of-two scale); rows past each length keep their bytes.  Accumulate: within one fp32 rounding of
    dk0 + oracle."""
    rng = np.random.default_rng(800 + d)
    lens = np.array([5000, 31, 1043, 6000, 0], np.int32)
    B, Lcap, Hkv = len(lens), 6000, 2
    nk_cap = binding.num_kernels(Lcap)
    dkern = rng.standard_normal((B, Hkv, nk_cap, d)).astype(np.float32)
    ref = oracle.kernel_pool_backward(dkern, lens, Lcap)
    dk0 = rng.standard_normal((B, Lcap, Hkv, d)).astype(np.float32)
    p = binding.Params()
    dkern_d, lens_d = torch.from_numpy(dkern).cuda(), dev_i32(lens)
    dk = torch.from_numpy(dk0).cuda()
    binding.infllmv2_kernel_pool_backward(dkern_d, lens_d, int(lens.max()), p, dk, accumulate=False)
    got = dk.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        assert np.array_equal(got[b, :n], ref[b, :n].astype(np.float32)), f"sequence {b}: rows [0, {n})"
        assert np.array_equal(got[b, n:], dk0[b, n:]), f"sequence {b}: rows past the length were written"
    dk = torch.from_numpy(dk0).cuda()
    binding.infllmv2_kernel_pool_backward(dkern_d, lens_d, int(lens.max()), p, dk, accumulate=True)
    got = dk.cpu().numpy().astype(np.float64)
    want = dk0.astype(np.float64) + ref
    for b in range(B):
        n = int(lens[b])
        tol = 2.0 ** -23 * (np.abs(dk0[b, :n]).astype(np.float64) + np.abs(ref[b, :n])) * 2
        assert np.all(np.abs(got[b, :n] - want[b, :n]) <= tol + 1e-30), f"sequence {b} (accumulate)"
        assert np.array_equal(got[b, n:], dk0[b, n:].astype(np.float64))


def test_kernel_pool_backward_full_128k(oracle):
    """One 128K sequence (2 KV heads, d 128), the size of the decode workload's longest rows: every row
    bit-exact with the oracle rounded to fp32."""
    rng = np.random.default_rng(810)
    L, Hkv, d = 131072, 2, 128
    nk_cap = binding.num_kernels(L)
    dkern = rng.standard_normal((1, Hkv, nk_cap, d)).astype(np.float32)
    ref = oracle.kernel_pool_backward(dkern, [L], L).astype(np.float32)
    dk = torch.empty((1, L, Hkv, d), dtype=torch.float32, device="cuda")
    binding.infllmv2_kernel_pool_backward(torch.from_numpy(dkern).cuda(), dev_i32([L]), L, binding.Params(), dk)
    assert np.array_equal(dk.cpu().numpy(), ref)
