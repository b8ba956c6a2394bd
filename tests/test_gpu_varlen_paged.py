"""Packed variable-length prefill and the paged key/value cache, through the C ABI, against the fp64 oracle.

* Packed prefill (infllmv2_sparse_prefill_varlen): every sequence of the packed batch is checked against the
  oracle run on that sequence alone -- kernels bit-exact, selection bit-exact except at the oracle's near
  ties, attention (on the GPU's own selection) within the parity bar.  Lengths are ragged (one query, queries
  fewer than keys, a sequence with no query, one shorter than a kernel window), on the tensor-core path
  (16 heads per group, d 128), the mma.sync path (2 heads per group, d 64) and the few-rows scan path.
* Paged cache: the keys and values of each sequence are scattered over a shuffled page pool.  Appending
  through the page table writes exactly the expected rows; the kernel pool, the fused decode step and the
  prefill attention on the pages equal the same calls on the contiguous cache bit for bit, and the oracle.
"""
import numpy as np
import pytest
import torch

from gpu_util import bparams, check_attention, check_selection, dev, dev_i32, host_u16, oparams
from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.workloads import f32_to_bf16_bits, method_params

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from trainable_block_sparse_v2_b200.build import build
    build()
    binding.load()


def _bf16(rng, shape):
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


# ---------------------------------------------------------------------------------------------------
# packed variable-length prefill
# ---------------------------------------------------------------------------------------------------

VARLEN_CASES = {
    # name: (Hq, Hkv, d, [(T_b, L_b)], topk, dense_len)
    "tensor_core": (32, 2, 128, [(1500, 1500), (700, 2100), (1, 900), (0, 300), (64, 64), (20, 31)], 8, 300),
    "tensor_core_d64": (4, 2, 64, [(1100, 1100), (333, 1800), (1, 64)], 6, 0),
    "mma_sync": (2, 2, 128, [(1100, 1100), (333, 1800), (1, 64)], 6, 0),
    "scan_rows": (32, 2, 128, [(5, 4000), (16, 2500), (1, 70)], 8, 0),
}


@pytest.mark.parametrize("case", list(VARLEN_CASES))
def test_sparse_prefill_varlen_matches_each_sequence_alone(oracle, case):
    Hq, Hkv, d, seqs, topk, dense_len = VARLEN_CASES[case]
    rng = np.random.default_rng(2400 + len(case))
    params = method_params(topk, dense_len, 0)
    p, P = bparams(params), oparams(params)
    qs = [_bf16(rng, (T, Hq, d)) for T, _ in seqs]
    ks = [_bf16(rng, (L, Hkv, d)) for _, L in seqs]
    vs = [_bf16(rng, (L, Hkv, d)) for _, L in seqs]
    cu_q = np.concatenate([[0], np.cumsum([T for T, _ in seqs])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([L for _, L in seqs])]).astype(np.int32)
    max_t, max_l = max(T for T, _ in seqs), max(L for _, L in seqs)
    B = len(seqs)
    q, k, v = dev(np.concatenate(qs)), dev(np.concatenate(ks)), dev(np.concatenate(vs))
    nk_cap = max(1, binding.num_kernels(max_l))
    kern = torch.zeros((B, Hkv, nk_cap, d), dtype=torch.bfloat16, device="cuda")
    total_q = int(cu_q[-1])
    idx = torch.full((total_q, Hkv, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((total_q, Hkv), -7, dtype=torch.int32, device="cuda")
    out = torch.full((total_q, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((total_q, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ws = binding.workspace(p, B, max_t, max_l, Hq, Hkv, d)
    binding.infllmv2_sparse_prefill_varlen(q, k, v, dev_i32(cu_q), dev_i32(cu_k), max_t, max_l, p, kern, idx, cnt,
                                           out, lse, ws)
    torch.cuda.synchronize()
    assert binding.infllmv2_device_status() == 0
    gk = host_u16(kern)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for b, (T, L) in enumerate(seqs):
        nk = binding.num_kernels(L)
        kern_o = oracle.kernel_pool(ks[b][None], [0], [L], 32, 16, nk_cap=nk_cap)
        assert np.array_equal(gk[b, :, :nk], kern_o[0, :, :nk]), f"kernels of sequence {b}"
        if T == 0:
            continue
        rows = slice(int(cu_q[b]), int(cu_q[b + 1]))
        q_ctx = np.arange(L - T + 1, L + 1, dtype=np.int32)[None]
        r = oracle.block_score_topk(qs[b][None], kern_o, q_ctx, P)
        check_selection(gi[rows][None], gc[rows][None], r)
        out_o, lse_o = oracle.sparse_attention(qs[b][None], ks[b][None], vs[b][None], q_ctx, gi[rows][None],
                                               gc[rows][None], P)
        check_attention(out[rows][None], out_o, lse[rows][None], lse_o, what=f"{case} sequence {b}")


def test_sparse_prefill_varlen_refuses_bad_sizes():
    p = binding.Params(topk=8)
    q = torch.zeros((10, 32, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((10, 2, 128), dtype=torch.bfloat16, device="cuda")
    kern = torch.zeros((1, 2, 1, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((10, 2, p.kmax), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((10, 2), dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 10], dtype=torch.int32, device="cuda")
    with pytest.raises(binding.Infllmv2Error) as e:  # more queries than keys in the longest sequence
        binding.infllmv2_sparse_prefill_varlen(q, k, k, cu, cu, 11, 10, p, kern, idx, cnt, torch.empty_like(q))
    assert e.value.status == 1


# ---------------------------------------------------------------------------------------------------
# paged key/value cache
# ---------------------------------------------------------------------------------------------------

def _paged(rng, K, V, lens, num_pages, max_pages):
    """Scatter the first lens[b] positions of each sequence over a shuffled page pool, with a page mapped for
    one more position (an append).  Returns (k_pages, v_pages, table) as host arrays; unused table entries are
    -1, and pool rows past each context hold random values that no call may read."""
    B, Lcap, Hkv, d = K.shape
    perm = rng.permutation(num_pages)
    table = np.full((B, max_pages), -1, np.int32)
    kp = _bf16(rng, (num_pages * 64, Hkv, d))  # garbage in unused rows: it must never be read
    vp = _bf16(rng, (num_pages * 64, Hkv, d))
    nxt = 0
    for b in range(B):
        for blk in range((int(lens[b]) + 64) // 64):  # room for one appended position
            pg = int(perm[nxt])
            nxt += 1
            table[b, blk] = pg
            lo, hi = blk * 64, min(blk * 64 + 64, int(lens[b]))  # rows past the context keep the garbage
            if hi > lo:
                kp[pg * 64:pg * 64 + hi - lo] = K[b, lo:hi]
                vp[pg * 64:pg * 64 + hi - lo] = V[b, lo:hi]
    return kp, vp, table


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 2, 128), (4, 2, 64), (2, 2, 128)])
def test_paged_cache_equals_contiguous_cache(oracle, Hq, Hkv, d):
    rng = np.random.default_rng(2500 + d)
    lens = np.array([5000, 130, 9000], np.int32)  # context lengths after the append below
    B = len(lens)
    Lcap = int(lens.max()) + 64
    K, V = _bf16(rng, (B, Lcap, Hkv, d)), _bf16(rng, (B, Lcap, Hkv, d))
    num_pages, max_pages = 300, Lcap // 64 + 2
    kp_h, vp_h, table_h = _paged(rng, K, V, lens - 1, num_pages, max_pages)
    params = method_params(16, 2000, 0)
    p, P = bparams(params), oparams(params)
    kp, vp, table = dev(kp_h), dev(vp_h), dev_i32(table_h)
    Kc, Vc = dev(K), dev(V)

    # 1. append the last position of each sequence through the page table
    pos = lens - 1
    k_new = dev(np.ascontiguousarray(K[np.arange(B), pos]))
    v_new = dev(np.ascontiguousarray(V[np.arange(B), pos]))
    pre = host_u16(kp)
    binding.infllmv2_kv_append_paged(k_new, v_new, dev_i32(pos), kp, vp, table)
    torch.cuda.synchronize()
    want = pre.copy()
    for b in range(B):
        r = table_h[b, pos[b] // 64] * 64 + pos[b] % 64
        want[r] = K[b, pos[b]]
    assert np.array_equal(host_u16(kp), want)

    # 2. kernel pool on the pages: bulk up to lens - 1, then the appended key; equal to the contiguous pool
    nk_cap = binding.num_kernels(int(lens.max()))
    kern_p = torch.zeros((B, Hkv, nk_cap, d), dtype=torch.bfloat16, device="cuda")
    kern_c = torch.zeros_like(kern_p)
    binding.infllmv2_kernel_pool_paged(kp, table, dev_i32(np.zeros(B)), dev_i32(lens - 1), int(lens.max()), p, kern_p)
    binding.infllmv2_kernel_pool_paged(kp, table, dev_i32(lens - 1), dev_i32(lens), 1, p, kern_p)
    binding.infllmv2_kernel_pool(Kc, dev_i32(np.zeros(B)), dev_i32(lens), int(lens.max()), p, kern_c)
    torch.cuda.synchronize()
    kern_o = oracle.kernel_pool(K, np.zeros(B), lens, 32, 16, nk_cap=nk_cap)
    assert np.array_equal(host_u16(kern_p), kern_o) and np.array_equal(host_u16(kern_c), kern_o)

    # 3. the fused decode step on the pages and on the contiguous cache: identical, and the oracle's
    qd = _bf16(rng, (B, 1, Hq, d))
    res = {}
    for name in ("paged", "contiguous"):
        idx = torch.full((B, 1, Hkv, p.kmax), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B, 1, Hkv), -7, dtype=torch.int32, device="cuda")
        out = torch.empty((B, 1, Hq, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, 1, Hq), dtype=torch.float32, device="cuda")
        if name == "paged":
            binding.infllmv2_sparse_decode_step_paged(dev(qd), kern_p, kp, vp, table, dev_i32(lens), int(lens.max()),
                                                      p, idx, cnt, out, lse)
        else:
            binding.infllmv2_sparse_decode_step(dev(qd), kern_c, Kc, Vc, dev_i32(lens), int(lens.max()), p, idx, cnt,
                                                out, lse)
        torch.cuda.synchronize()
        res[name] = (idx.cpu().numpy(), cnt.cpu().numpy(), host_u16(out), lse.cpu().numpy())
    for a, b_ in zip(res["paged"], res["contiguous"]):
        assert np.array_equal(a, b_)
    assert binding.infllmv2_device_status() == 0
    q_ctx = lens[:, None].astype(np.int32)
    r = oracle.block_score_topk(qd, kern_o, q_ctx, P)
    gi, gc = res["paged"][0], res["paged"][1]
    check_selection(gi, gc, r)
    out_o, lse_o = oracle.sparse_attention(qd, K, V, q_ctx, gi, gc, P)
    check_attention(torch.from_numpy(res["paged"][2].view(np.int16)).view(torch.bfloat16), out_o,
                    torch.from_numpy(res["paged"][3]), lse_o, what="paged decode step")

    # 4. prefill attention of the last 70 positions (a chunked prefill) on the pages and contiguously
    T = 70
    qp = _bf16(rng, (B, T, Hq, d))
    idx = torch.full((B, T, Hkv, p.kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, T, Hkv), -7, dtype=torch.int32, device="cuda")
    ws = binding.workspace(p, B, T, int(lens.max()), Hq, Hkv, d)
    binding.infllmv2_block_score_topk(dev(qp), None, dev_i32(lens), int(lens.max()), kern_p, p, idx, cnt, ws)
    outs = {}
    for name in ("paged", "contiguous"):
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device="cuda")
        if name == "paged":
            binding.infllmv2_sparse_attn_prefill_paged(dev(qp), kp, vp, table, None, dev_i32(lens), int(lens.max()),
                                                       idx, cnt, p, out, lse)
        else:
            binding.infllmv2_sparse_attn_prefill(dev(qp), Kc, Vc, None, dev_i32(lens), int(lens.max()), idx, cnt, p,
                                                 out, lse)
        torch.cuda.synchronize()
        outs[name] = (out, lse)
    assert torch.equal(outs["paged"][0], outs["contiguous"][0]) and torch.equal(outs["paged"][1], outs["contiguous"][1])
    q_ctx = (lens[:, None] - T + 1 + np.arange(T)[None]).astype(np.int32)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    check_selection(gi, gc, oracle.block_score_topk(qp, kern_o, q_ctx, P))
    out_o, lse_o = oracle.sparse_attention(qp, K, V, q_ctx, gi, gc, P)
    check_attention(outs["paged"][0], out_o, outs["paged"][1], lse_o, what="paged prefill attention")
