"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against a value fixed by the mathematics, not by re-typing its code:
a hand-worked example (closed forms), special cases that reduce to library routines (torch softmax
attention, average / max pooling), and invariants of the definition (GQA-shared sets, forced blocks,
top-k order, shift and permutation invariance).  A dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from trainable_block_sparse_v2_b200.workloads import (decode_case, f32_to_bf16_bits, prefill_case,
                                                      tree_mask_from_parents)

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    """exact bf16 bits of a float array (values must be bf16-representable)"""
    x = np.asarray(x, np.float32)
    b = f32_to_bf16_bits(x)
    assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), x), "value not representable in bf16"
    return b


def f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sdpa_fp64(q, K, V, mask, scale):
    """torch softmax attention in fp64.  q [Hq, Tq, d], K/V [Hq, Tk, d], mask [Hq or 1, Tq, Tk] bool."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(K), torch.from_numpy(V), attn_mask=torch.from_numpy(mask),
        scale=scale)
    return out.numpy()


def rand_case(rng, B, T, L, Hq, Hkv, d, scale_q=1.0):
    q = f32_to_bf16_bits(scale_q * rng.standard_normal((B, T, Hq, d)).astype(np.float32))
    K = f32_to_bf16_bits(rng.standard_normal((B, L, Hkv, d)).astype(np.float32))
    V = f32_to_bf16_bits(rng.standard_normal((B, L, Hkv, d)).astype(np.float32))
    return q, K, V


# ------------------------------------------------------------------------------------------------
# hand-worked example
# ------------------------------------------------------------------------------------------------

def _gold():
    with open(os.path.join(GOLD, "two_block_example.json")) as f:
        return json.load(f)


def test_two_block_example(oracle):
    g = _gold()
    e2, e3 = math.exp(2), math.exp(3)
    # the stored numbers are the closed forms they claim to be
    assert g["S"]["value"] == pytest.approx([e2 / (e2 + 3) + 1 / (e3 + 3), 1 / (e2 + 3) + e3 / (e3 + 3)], rel=1e-15)
    P = oracle.Params(**g["params"])
    K = bits(np.array(g["K"], np.float32))[None, :, None, :]
    V = bits(np.array(g["V"], np.float32))[None, :, None, :]
    q = bits(np.array(g["q"], np.float32))[None, None]
    n = g["n"]
    kern = oracle.kernel_pool(K, [0], [n], P.kernel_size, P.kernel_stride)
    assert np.array_equal(f64(kern[0, 0]), np.array(g["kernels"], np.float64))
    r = oracle.block_score_topk(q, kern, np.array([[n]]), P)
    assert r["S"][0, 0, 0] == pytest.approx(g["S"]["value"], abs=1e-14)
    assert r["lse"][0, 0] == pytest.approx(g["lse_heads"]["value"], abs=1e-14)
    assert r["cnt"][0, 0, 0] == 1 and list(r["idx"][0, 0, 0]) == g["idx"]
    out, lse = oracle.sparse_attention(q, K, V, np.array([[n]]), r["idx"], r["cnt"], P)
    assert out[0, 0] == pytest.approx(np.array(g["out"]["value"]), abs=1e-14)
    assert lse[0, 0] == pytest.approx(g["out_lse"]["value"], abs=1e-14)


def test_exact_tie_goes_to_lower_block(oracle):
    """Two blocks with identical kernels score identically; the tie goes to the lower block index."""
    g = _gold()
    P = oracle.Params(**g["params"])
    Kf = np.array([[1, 0], [1, 0], [0, 1], [0, 1], [1, 0], [1, 0], [0, 1], [0, 1]], np.float32)
    K = bits(Kf)[None, :, None, :]
    q = bits(np.array([[2, 0], [0, 1.5]], np.float32))[None, None]
    kern = oracle.kernel_pool(K, [0], [8], 2, 2)
    r = oracle.block_score_topk(q, kern, np.array([[8]]), P)
    assert r["S"][0, 0, 0, 0] == r["S"][0, 0, 0, 1]
    assert list(r["idx"][0, 0, 0]) == [0]
    assert r["gap"][0, 0, 0, 0] == r["gap"][0, 0, 0, 1]


# ------------------------------------------------------------------------------------------------
# semantic kernels
# ------------------------------------------------------------------------------------------------

def test_kernel_pool_closed_forms(oracle):
    # constant keys: every kernel equals the key
    K = np.broadcast_to(bits(np.array([0.75, -1.5, 3.0, 0.0], np.float32)), (1, 200, 1, 4)).copy()
    kern = oracle.kernel_pool(K, [0], [200], 32, 16)
    assert kern.shape[2] == (200 - 32) // 16 + 1
    assert np.array_equal(f64(kern[0, 0]), np.broadcast_to(f64(K[0, 0]), kern.shape[2:]))
    # ramp K[i] = 2i: the window mean is the midpoint 2*(16 j + 15.5) = 32 j + 31 (exact in bf16 for j <= 6)
    ramp = bits((2 * np.arange(128, dtype=np.float32))[None, :, None, None])
    kern = oracle.kernel_pool(ramp, [0], [128], 32, 16)
    assert np.array_equal(f64(kern[0, 0, :, 0]), 32 * np.arange(7) + 31.0)
    # no complete window below 32 keys
    assert oracle.num_kernels(31) == 0 and oracle.num_kernels(32) == 1 and oracle.num_kernels(47) == 1


def test_kernel_pool_matches_avg_pool_and_bf16_rounding(oracle):
    """Window mean = torch avg_pool1d (fp64); storage = torch's fp32 -> bf16 round-to-nearest-even."""
    rng = np.random.default_rng(7)
    L, Hkv, d = 300, 2, 8
    K = f32_to_bf16_bits(rng.standard_normal((1, L, Hkv, d)).astype(np.float32))
    kern = oracle.kernel_pool(K, [0], [L], 32, 16)
    x = torch.from_numpy(f64(K[0])).permute(1, 2, 0)  # [Hkv, d, L]
    mean = torch.nn.functional.avg_pool1d(x, kernel_size=32, stride=16).permute(0, 2, 1)  # [Hkv, NK, d]
    m32 = mean.to(torch.float32)
    assert torch.equal(m32.to(torch.float64), mean), "test data: means must be exact in fp32"
    want = m32.to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(f64(kern[0]), want)


def test_kernel_pool_incremental_equals_bulk(oracle):
    rng = np.random.default_rng(8)
    L = 333
    K = f32_to_bf16_bits(rng.standard_normal((2, L, 2, 16)).astype(np.float32))
    bulk = oracle.kernel_pool(K, [0, 0], [L, L - 40], 32, 16)
    inc = np.zeros_like(bulk)
    for a, b in [(0, 50), (50, 51), (51, 200), (200, L)]:
        oracle.kernel_pool(K, [a, min(a, L - 40)], [b, min(b, L - 40)], 32, 16, kern=inc, nk_cap=bulk.shape[2])
    assert np.array_equal(inc, bulk)


def test_kernel_pool_rounds_the_exact_mean_once(oracle):
    """Hand-worked windows whose exact sum sits a hair beside a bf16 midpoint (an fp32 sum would drop the
    2^-30 key and tie the other way) or exactly on one (ties to even): the expected bits are worked out by
    hand in tests/pool_midpoints.py."""
    from pool_midpoints import midpoint_case
    for d in (16, 64):
        K, want = midpoint_case(d)
        got = oracle.kernel_pool(K, [0], [K.shape[1]], 32, 16)
        assert np.array_equal(got, want)


def test_round_bf16_single_rounding(oracle):
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(2000) * np.exp(rng.uniform(-20, 20, 2000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.round_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)
    # halfway cases round to even
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 0x3F80 and oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82


# ------------------------------------------------------------------------------------------------
# scoring: special cases that reduce to softmax attention
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("bs", [1, 2])
def test_scores_reduce_to_attention_probabilities(oracle, bs):
    """With one-key kernels (window 1, stride 1) the normalised kernel scores are the softmax attention
    probabilities; a block's head score is their max over the block's keys (max_pool1d) and the group
    score sums the group's heads."""
    rng = np.random.default_rng(10 + bs)
    T, Hq, Hkv, d = 6, 4, 2, 8
    L = 24
    q, K, _ = rand_case(rng, 1, T, L, Hq, Hkv, d)
    n = np.array([[5, 9, 12, 17, 23, 24]], np.int32)
    P = oracle.Params(block_size=bs, kernel_size=1, kernel_stride=1, topk=100, init_blocks=0, local_blocks=0,
                      scale=0.3)
    kern = oracle.kernel_pool(K, [0], [L], 1, 1)
    r = oracle.block_score_topk(q, kern, n, P, nb_max=L)
    G = Hq // Hkv
    qt = torch.from_numpy(f64(q[0]))
    Kt = torch.from_numpy(f64(K[0]))
    for t in range(T):
        nn = int(n[0, t])
        for g in range(Hkv):
            logits = 0.3 * qt[t, g * G:(g + 1) * G] @ Kt[:nn, g].T  # [G, nn]
            probs = torch.softmax(logits, dim=-1)
            assert r["lse"][0, t, g * G:(g + 1) * G] == pytest.approx(torch.logsumexp(logits, -1).numpy(), abs=1e-12)
            pooled = torch.nn.functional.max_pool1d(probs[None], kernel_size=bs, stride=bs, ceil_mode=True)[0]
            want = pooled.sum(0).numpy()
            c = (nn - 1) // bs
            assert r["S"][0, t, g, :c + 1] == pytest.approx(want[:c + 1], abs=1e-12)
            assert np.all(np.isneginf(r["S"][0, t, g, c + 1:]))


def test_overlap_contains_contained(oracle):
    """OVERLAP membership is a superset of CONTAINED, so its block score is never smaller; with windows
    that tile the block exactly (stride = window, block a multiple of it) the two rules agree."""
    rng = np.random.default_rng(12)
    w = prefill_case(640, 4, 2, 16, topk=3, dense_len=0, seed=12, n_needles=0)
    kern = oracle.kernel_pool(w.k, [0], [640], 32, 16)
    qc = w.q_ctx[:, 600:]
    q = w.q[:, 600:]
    ov = oracle.block_score_topk(q, kern, qc, oracle.Params(topk=3, membership=0))
    ct = oracle.block_score_topk(q, kern, qc, oracle.Params(topk=3, membership=1))
    fin = np.isfinite(ct["S"])
    assert np.all(ov["S"][fin] >= ct["S"][fin] - 1e-15)
    kern16 = oracle.kernel_pool(w.k, [0], [640], 16, 16)
    a = oracle.block_score_topk(q, kern16, qc, oracle.Params(kernel_size=16, kernel_stride=16, membership=0))
    b = oracle.block_score_topk(q, kern16, qc, oracle.Params(kernel_size=16, kernel_stride=16, membership=1))
    assert np.array_equal(a["S"], b["S"]) and np.array_equal(a["idx"], b["idx"])
    del rng


def test_score_invariant_to_per_head_logit_shift(oracle):
    """Keys whose last coordinate is 1 make every kernel's last coordinate 1; moving q_h's last coordinate
    shifts all of head h's kernel scores by one constant, which the LSE normalisation cancels."""
    rng = np.random.default_rng(13)
    L, Hq, Hkv, d = 700, 4, 2, 16
    Kf = rng.standard_normal((1, L, Hkv, d)).astype(np.float32)
    Kf[..., -1] = 1.0
    K = f32_to_bf16_bits(Kf)
    q = f32_to_bf16_bits(rng.standard_normal((1, 3, Hq, d)).astype(np.float32))
    n = np.array([[650, 690, 700]], np.int32)
    kern = oracle.kernel_pool(K, [0], [L], 32, 16)
    P = oracle.Params(topk=4)
    a = oracle.block_score_topk(q, kern, n, P)
    q2 = q.copy()
    q2[..., 1, -1] = f32_to_bf16_bits(f64(q[..., 1, -1]).astype(np.float32) + 4.0)
    q2[..., 2, -1] = f32_to_bf16_bits(f64(q[..., 2, -1]).astype(np.float32) - 2.0)
    b = oracle.block_score_topk(q2, kern, n, P)
    fin = np.isfinite(a["S"])
    assert np.allclose(a["S"][fin], b["S"][fin], rtol=1e-12, atol=1e-14)
    assert not np.allclose(a["lse"], b["lse"])
    assert np.array_equal(a["idx"], b["idx"])


def test_selection_shared_and_invariant_to_head_order(oracle):
    rng = np.random.default_rng(14)
    w = prefill_case(1024, 8, 2, 16, topk=4, dense_len=0, seed=14, n_needles=2)
    kern = oracle.kernel_pool(w.k, [0], [1024], 32, 16)
    sel = slice(700, 760)
    a = oracle.block_score_topk(w.q[:, sel], kern, w.q_ctx[:, sel], oracle.Params(topk=4))
    perm = np.concatenate([rng.permutation(4), 4 + rng.permutation(4)])
    b = oracle.block_score_topk(w.q[:, sel][:, :, perm], kern, w.q_ctx[:, sel], oracle.Params(topk=4))
    assert np.array_equal(a["idx"], b["idx"])
    assert np.allclose(a["S"][np.isfinite(a["S"])], b["S"][np.isfinite(b["S"])], rtol=1e-13)
    # swapping the two KV groups' heads swaps the groups' selections
    swap = np.concatenate([np.arange(4, 8), np.arange(0, 4)])
    kern_sw = kern[:, ::-1].copy()
    c = oracle.block_score_topk(w.q[:, sel][:, :, swap], kern_sw, w.q_ctx[:, sel], oracle.Params(topk=4))
    assert np.array_equal(c["idx"][:, :, ::-1], a["idx"])


def test_selection_invariants(oracle):
    """Forced blocks present, at most k + init + local entries, ascending and unique, no block past the
    query's own, and every chosen candidate outranks every rejected one (ties to the lower index)."""
    w = prefill_case(1500, 4, 2, 32, topk=5, dense_len=200, seed=15, n_needles=3)
    kern = oracle.kernel_pool(w.k, [0], [1500], 32, 16)
    P = oracle.Params(topk=5, dense_len=200)
    r = oracle.block_score_topk(w.q, kern, w.q_ctx, P)
    for t in range(0, 1500, 7):
        n = t + 1
        c = (n - 1) // 64
        for g in range(2):
            cnt = r["cnt"][0, t, g]
            idx = r["idx"][0, t, g]
            chosen = list(idx[:min(cnt, P.kmax)])
            if n <= P.dense_len:
                assert cnt == c + 1 and chosen == list(range(min(c + 1, P.kmax)))
                continue
            assert cnt <= P.kmax and np.all(idx[cnt:] == -1)
            assert chosen == sorted(set(chosen)) and chosen[-1] <= c
            forced = {0} | {b for b in (c - 1, c) if b >= 0}
            assert forced <= set(chosen)
            S = r["S"][0, t, g]
            cand = [b for b in range(c + 1) if b not in forced and np.isfinite(S[b])]
            picked = [b for b in cand if b in chosen]
            rejected = [b for b in cand if b not in chosen]
            assert len(picked) == min(P.topk, len(cand))
            for a_ in picked:
                for b_ in rejected:
                    assert S[a_] > S[b_] or (S[a_] == S[b_] and a_ < b_)


def test_k_covering_all_blocks_selects_everything(oracle):
    w = prefill_case(900, 4, 2, 16, topk=100, dense_len=0, seed=16, n_needles=0)
    kern = oracle.kernel_pool(w.k, [0], [900], 32, 16)
    r = oracle.block_score_topk(w.q, kern, w.q_ctx, oracle.Params(topk=100))
    for t in range(0, 900, 11):
        c = t // 64
        assert list(r["idx"][0, t, 0, :r["cnt"][0, t, 0]]) == list(range(c + 1))


def test_needle_blocks_are_selected(oracle):
    """Sanity (not a parity pin): blocks whose keys are shifted toward the query's group mean are chosen."""
    w = decode_case([2048, 1500], 4, 2, 64, topk=8, dense_len=0, seed=17, n_needles=3)
    kern = oracle.kernel_pool(w.k, [0, 0], list(w.ctx_lens), 32, 16)
    r = oracle.block_score_topk(w.q, kern, w.q_ctx, oracle.Params(topk=8))
    for b in range(2):
        for g in range(2):
            assert np.all(np.isin(w.extras["needles"][b], r["idx"][b, 0, g]))


# ------------------------------------------------------------------------------------------------
# attention: special cases that reduce to softmax attention
# ------------------------------------------------------------------------------------------------

def _sdpa_rows(oracle_q, K, V, keysets, scale, Hq, Hkv):
    """reference via torch sdpa: per (t, h) attention over the explicit key list"""
    G = Hq // Hkv
    T = oracle_q.shape[1]
    d = oracle_q.shape[-1]
    out = np.zeros((T, Hq, d))
    for t in range(T):
        for h in range(Hq):
            ks = keysets[t][h // G]
            qq = f64(oracle_q[0, t, h])[None, None, None]
            kk = f64(K[0, ks, h // G])[None, None]
            vv = f64(V[0, ks, h // G])[None, None]
            out[t, h] = sdpa_fp64(qq, kk, vv, np.ones((1, 1, 1, len(ks)), bool), scale)[0, 0, 0]
    return out


def test_sparse_attention_with_all_blocks_is_causal_attention(oracle):
    rng = np.random.default_rng(20)
    T = L = 200
    Hq, Hkv, d = 4, 2, 16
    q, K, V = rand_case(rng, 1, T, L, Hq, Hkv, d)
    qc = np.arange(1, T + 1, dtype=np.int32)[None]
    P = oracle.Params(topk=100)
    kern = oracle.kernel_pool(K, [0], [L], 32, 16)
    r = oracle.block_score_topk(q, kern, qc, P)
    out, lse = oracle.sparse_attention(q, K, V, qc, r["idx"], r["cnt"], P)
    dense, dlse = oracle.dense_attention(q, K, V, qc)
    # torch causal attention, GQA expanded
    G = Hq // Hkv
    qq = f64(q[0]).transpose(1, 0, 2)
    kk = np.repeat(f64(K[0]).transpose(1, 0, 2), G, axis=0)
    vv = np.repeat(f64(V[0]).transpose(1, 0, 2), G, axis=0)
    causal = np.tril(np.ones((T, L), bool))[None]
    want = sdpa_fp64(qq, kk, vv, causal, 1 / math.sqrt(d)).transpose(1, 0, 2)
    assert np.max(np.abs(out[0] - want)) < 1e-12
    assert np.max(np.abs(dense[0] - want)) < 1e-12
    logits = np.einsum("htd,hsd->hts", qq, kk) / math.sqrt(d)
    logits[~np.broadcast_to(causal, logits.shape)] = -np.inf
    want_lse = torch.logsumexp(torch.from_numpy(logits), -1).numpy().T
    assert np.max(np.abs(lse[0] - want_lse)) < 1e-12 and np.max(np.abs(dlse[0] - want_lse)) < 1e-12


def test_sparse_attention_explicit_sets(oracle):
    """Attention over hand-chosen block sets (single block, gaps, partial last block) = sdpa over those keys."""
    rng = np.random.default_rng(21)
    L = 300
    Hq, Hkv, d = 4, 2, 8
    q, K, V = rand_case(rng, 1, 3, L, Hq, Hkv, d)
    qc = np.array([[300, 130, 64]], np.int32)
    P = oracle.Params(topk=2, init_blocks=0, local_blocks=0)
    idx = np.full((1, 3, 2, 2), -1, np.int32)
    cnt = np.zeros((1, 3, 2), np.int32)
    sets = [[[4], [0, 2]], [[1, 2], [2]], [[0], [0]]]
    for t in range(3):
        for g in range(2):
            idx[0, t, g, :len(sets[t][g])] = sets[t][g]
            cnt[0, t, g] = len(sets[t][g])
    out, _ = oracle.sparse_attention(q, K, V, qc, idx, cnt, P)
    keysets = [[[i for b in sets[t][g] for i in range(b * 64, min(b * 64 + 64, qc[0, t]))] for g in range(2)]
               for t in range(3)]
    want = _sdpa_rows(q, K, V, keysets, 1 / math.sqrt(d), Hq, Hkv)
    assert np.max(np.abs(out[0] - want)) < 1e-12


def test_dense_rows_ignore_selection(oracle):
    rng = np.random.default_rng(22)
    L = 260
    q, K, V = rand_case(rng, 1, 2, L, 4, 2, 8)
    qc = np.array([[100, 260]], np.int32)
    P = oracle.Params(topk=1, dense_len=150)
    idx = np.full((1, 2, 2, 4), -1, np.int32)
    idx[..., 0] = 0
    cnt = np.ones((1, 2, 2), np.int32)
    out, _ = oracle.sparse_attention(q, K, V, qc, idx, cnt, P)
    dense, _ = oracle.dense_attention(q, K, V, qc)
    assert np.max(np.abs(out[0, 0] - dense[0, 0])) < 1e-13      # n = 100 <= 150: dense
    assert np.max(np.abs(out[0, 1] - dense[0, 1])) > 1e-3       # n = 260 > 150: block 0 only


@pytest.mark.parametrize("shape", ["chain", "star"])
def test_tree_attention_special_shapes(oracle, shape):
    """Chain tree: node i sees drafts 0..i (causal over the draft); star tree: the root and itself."""
    rng = np.random.default_rng(23)
    P_, N = 200, 6
    Hq, Hkv, d = 4, 2, 8
    q, K, V = rand_case(rng, 1, N, P_, Hq, Hkv, d)
    KD = f32_to_bf16_bits(rng.standard_normal((1, N, Hkv, d)).astype(np.float32))
    VD = f32_to_bf16_bits(rng.standard_normal((1, N, Hkv, d)).astype(np.float32))
    parent = np.arange(-1, N - 1) if shape == "chain" else np.array([-1] + [0] * (N - 1))
    mask = tree_mask_from_parents(parent)[None]
    if shape == "chain":
        assert list(mask[0]) == [(1 << (i + 1)) - 1 for i in range(N)]
    else:
        assert list(mask[0]) == [1] + [1 | (1 << i) for i in range(1, N)]
    qc = np.full((1, N), P_, np.int32)
    Pm = oracle.Params(topk=1)
    kern = oracle.kernel_pool(K, [0], [P_], 32, 16)
    r = oracle.block_score_topk(q, kern, qc, Pm)
    out, _ = oracle.sparse_attention(q, K, V, qc, r["idx"], r["cnt"], Pm, KD, VD, mask)
    G = Hq // Hkv
    for i in range(N):
        for h in range(Hq):
            g = h // G
            blocks = r["idx"][0, i, g, :r["cnt"][0, i, g]]
            pre = [k for b in blocks for k in range(b * 64, min(b * 64 + 64, P_))]
            drafts = [j for j in range(N) if (j <= i if shape == "chain" else j in (0, i))]
            kk = np.concatenate([f64(K[0, pre, g]), f64(KD[0, drafts, g])])[None, None]
            vv = np.concatenate([f64(V[0, pre, g]), f64(VD[0, drafts, g])])[None, None]
            qq = f64(q[0, i, h])[None, None, None]
            want = sdpa_fp64(qq, kk, vv, np.ones((1, 1, 1, kk.shape[2]), bool), 1 / math.sqrt(d))[0, 0, 0]
            assert np.max(np.abs(out[0, i, h] - want)) < 1e-12


# ------------------------------------------------------------------------------------------------
# the draft model's sliding-window attention
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("window", [1, 37, 64, 150, 1000])
def test_window_attention_is_banded_softmax_attention(oracle, window):
    """Keys [max(0, n - W), n) per query = torch softmax attention under a banded causal mask (GQA expanded);
    a window past the context is plain causal attention."""
    rng = np.random.default_rng(40 + window)
    T = L = 200
    Hq, Hkv, d = 4, 2, 16
    q, K, V = rand_case(rng, 1, T, L, Hq, Hkv, d)
    qc = np.arange(1, T + 1, dtype=np.int32)[None]
    out, lse = oracle.window_attention(q, K, V, qc, window)
    G = Hq // Hkv
    qq = f64(q[0]).transpose(1, 0, 2)
    kk = np.repeat(f64(K[0]).transpose(1, 0, 2), G, axis=0)
    vv = np.repeat(f64(V[0]).transpose(1, 0, 2), G, axis=0)
    tq = np.arange(T)[:, None]
    ik = np.arange(L)[None, :]
    band = ((ik <= tq) & (ik > tq - window))[None]
    want = sdpa_fp64(qq, kk, vv, band, 1 / math.sqrt(d)).transpose(1, 0, 2)
    assert np.max(np.abs(out[0] - want)) < 1e-12
    logits = np.einsum("htd,hsd->hts", qq, kk) / math.sqrt(d)
    logits[~np.broadcast_to(band, logits.shape)] = -np.inf
    want_lse = torch.logsumexp(torch.from_numpy(logits), -1).numpy().T
    assert np.max(np.abs(lse[0] - want_lse)) < 1e-12
    if window >= L:
        dense, _ = oracle.dense_attention(q, K, V, qc)
        assert np.max(np.abs(out - dense)) < 1e-12


def test_window_of_one_key_returns_that_value(oracle):
    """W = 1: the softmax has one term, so the output is the newest value row and lse its logit"""
    rng = np.random.default_rng(41)
    q, K, V = rand_case(rng, 2, 1, 90, 8, 2, 32)
    qc = np.array([[90], [53]], np.int32)
    out, lse = oracle.window_attention(q, K, V, qc, 1)
    for b in range(2):
        n = int(qc[b, 0])
        for h in range(8):
            assert np.array_equal(out[b, 0, h], f64(V[b, n - 1, h // 4]))
            assert lse[b, 0, h] == pytest.approx(f64(q[b, 0, h]) @ f64(K[b, n - 1, h // 4]) / math.sqrt(32), abs=1e-12)


# ------------------------------------------------------------------------------------------------
# backward of the sparse attention (fixed selection)
# ------------------------------------------------------------------------------------------------

def _grid_case(rng, B, T, L, Hq, Hkv, d):
    """inputs on the grid k/8, |k| <= 8, so that x +- 1/64 and x +- 1/32 are exact bf16 values"""
    def g(shape):
        return bits(rng.integers(-8, 9, size=shape).astype(np.float32) / 8.0)
    return g((B, T, Hq, d)), g((B, L, Hkv, d)), g((B, L, Hkv, d))


def test_backward_matches_central_differences(oracle):
    """Each gradient entry = Richardson-extrapolated central difference of the oracle's own forward loss
    sum(dout * out), stepping the bf16 input by exactly 1/64 and 1/32 (error O(h^4) ~ 1e-8)."""
    rng = np.random.default_rng(50)
    B, T, L, Hq, Hkv, d = 1, 5, 10, 4, 2, 4
    q, K, V = _grid_case(rng, B, T, L, Hq, Hkv, d)
    dout = bits(rng.integers(-8, 9, size=(B, T, Hq, d)).astype(np.float32) / 8.0)
    # block size 2: explicit sets with gaps, a partial last block, and one dense row (n <= dense_len)
    P = oracle.Params(block_size=2, topk=2, init_blocks=0, local_blocks=0, dense_len=3)
    qc = np.array([[10, 7, 3, 9, 5]], np.int32)
    sets = [[[0, 3], [4]], [[1, 3], [0, 2]], [[0], [0]], [[4], [1, 3]], [[2], [0, 1]]]
    idx = np.full((B, T, Hkv, 2), -1, np.int32)
    cnt = np.zeros((B, T, Hkv), np.int32)
    for t in range(T):
        for g in range(Hkv):
            idx[0, t, g, :len(sets[t][g])] = sets[t][g]
            cnt[0, t, g] = len(sets[t][g])
    dq, dk, dv = oracle.sparse_attention_backward(q, K, V, qc, idx, cnt, P, dout)
    w = f64(dout)

    def loss(qb, Kb, Vb):
        out, _ = oracle.sparse_attention(qb, Kb, Vb, qc, idx, cnt, P)
        return float(np.sum(w * out))

    def fd(arr, which, pos):
        vals = []
        for h in (1 / 64, 1 / 32):
            plus, minus = arr.copy(), arr.copy()
            x = f64(arr[pos])
            plus[pos] = bits(np.array([x + h], np.float32))[0]
            minus[pos] = bits(np.array([x - h], np.float32))[0]
            args_p = [q, K, V]
            args_m = [q, K, V]
            args_p[which] = plus
            args_m[which] = minus
            vals.append((loss(*args_p) - loss(*args_m)) / (2 * h))
        return (4 * vals[0] - vals[1]) / 3

    for which, arr, grad in ((0, q, dq), (1, K, dk), (2, V, dv)):
        for pos in np.ndindex(arr.shape):
            assert grad[pos] == pytest.approx(fd(arr, which, pos), abs=2e-6), (which, pos)
    # keys 8, 9 lie past every sparse row's blocks except row 0 (block 4) and row 3: nonzero there
    assert np.any(dv[0, 8:] != 0)


@pytest.mark.parametrize("Hq,Hkv,d", [(4, 2, 16), (16, 1, 8)])
def test_backward_dense_matches_torch_autograd(oracle, Hq, Hkv, d):
    """Every block selected: the gradients are those of torch causal softmax attention (fp64 autograd,
    GQA by repeating K/V over the group, whose backward sums the group's heads)."""
    rng = np.random.default_rng(51 + Hq)
    T = L = 150
    q, K, V = rand_case(rng, 1, T, L, Hq, Hkv, d)
    dout = f32_to_bf16_bits(rng.standard_normal((1, T, Hq, d)).astype(np.float32))
    qc = np.arange(1, T + 1, dtype=np.int32)[None]
    P = oracle.Params(topk=100)
    kern = oracle.kernel_pool(K, [0], [L], 32, 16)
    r = oracle.block_score_topk(q, kern, qc, P)
    dq, dk, dv = oracle.sparse_attention_backward(q, K, V, qc, r["idx"], r["cnt"], P, dout)
    G = Hq // Hkv
    qt = torch.from_numpy(f64(q[0]).transpose(1, 0, 2).copy()).requires_grad_()
    kt = torch.from_numpy(f64(K[0]).transpose(1, 0, 2).copy()).requires_grad_()
    vt = torch.from_numpy(f64(V[0]).transpose(1, 0, 2).copy()).requires_grad_()
    causal = torch.from_numpy(np.tril(np.ones((T, L), bool)))[None]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, 0), vt.repeat_interleave(G, 0), attn_mask=causal, scale=1 / math.sqrt(d))
    out.backward(torch.from_numpy(f64(dout[0]).transpose(1, 0, 2).copy()))
    assert np.max(np.abs(dq[0] - qt.grad.numpy().transpose(1, 0, 2))) < 1e-11
    assert np.max(np.abs(dk[0] - kt.grad.numpy().transpose(1, 0, 2))) < 1e-11
    assert np.max(np.abs(dv[0] - vt.grad.numpy().transpose(1, 0, 2))) < 1e-11


def test_backward_one_key_closed_form(oracle):
    """A query that sees one key has p = 1: its dq and that key's dk are exactly 0, and dv of the key is
    the sum of dout over the rows that read it."""
    rng = np.random.default_rng(52)
    q, K, V = rand_case(rng, 1, 3, 70, 4, 2, 8)
    dout = f32_to_bf16_bits(rng.standard_normal((1, 3, 4, 8)).astype(np.float32))
    qc = np.array([[1, 1, 1]], np.int32)
    P = oracle.Params(topk=1)
    idx = np.zeros((1, 3, 2, 4), np.int32)
    idx[..., 1:] = -1
    cnt = np.ones((1, 3, 2), np.int32)
    dq, dk, dv = oracle.sparse_attention_backward(q, K, V, qc, idx, cnt, P, dout)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    for g in range(2):
        assert np.max(np.abs(dv[0, 0, g] - f64(dout[0, :, 2 * g:2 * g + 2]).sum(axis=(0, 1)))) < 1e-13
    assert np.array_equal(dv[0, 1:], np.zeros_like(dv[0, 1:]))


def test_backward_sum_rules(oracle):
    """Identities of any softmax attention, on a sparse case with dense rows:
    sum_j dk_j = 0 (a common shift of the keys leaves every softmax unchanged);
    sum_j dv_j = sum over rows of dout (each row's probabilities sum to 1);
    sum dv . V = sum dout . out (out is linear in V);  sum dq . q = sum dk . K (logits are bilinear)."""
    rng = np.random.default_rng(53)
    B, T, L, Hq, Hkv, d = 2, 40, 400, 8, 2, 16
    q, K, V = rand_case(rng, B, T, L, Hq, Hkv, d)
    dout = f32_to_bf16_bits(rng.standard_normal((B, T, Hq, d)).astype(np.float32))
    qc = np.stack([np.linspace(20, 400, T).astype(np.int32), np.linspace(5, 300, T).astype(np.int32)])
    P = oracle.Params(topk=2, dense_len=100)
    kern = oracle.kernel_pool(K, [0, 0], [L, L], 32, 16)
    r = oracle.block_score_topk(q, kern, qc, P)
    dq, dk, dv = oracle.sparse_attention_backward(q, K, V, qc, r["idx"], r["cnt"], P, dout)
    out, _ = oracle.sparse_attention(q, K, V, qc, r["idx"], r["cnt"], P)
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            assert np.max(np.abs(dk[b, :, g].sum(axis=0))) < 1e-10
            want = f64(dout[b, :, g * G:(g + 1) * G]).sum(axis=(0, 1))
            assert np.max(np.abs(dv[b, :, g].sum(axis=0) - want)) < 1e-10
    assert np.sum(dv * f64(V)) == pytest.approx(np.sum(f64(dout) * out), rel=1e-12)
    assert np.sum(dq * f64(q)) == pytest.approx(np.sum(dk * f64(K)), rel=1e-10, abs=1e-10)
    assert np.max(np.abs(dq)) > 0.01 and np.max(np.abs(dk)) > 0.01


# ------------------------------------------------------------------------------------------------
# LSE estimate from every s-th kernel (a reading of the pages' undefined "LogSumExp estimation")
# ------------------------------------------------------------------------------------------------

def test_lse_estimate_stride_one_is_exact(oracle):
    rng = np.random.default_rng(60)
    q, K, V = rand_case(rng, 1, 20, 900, 4, 2, 16)
    qc = np.linspace(100, 900, 20).astype(np.int32)[None]
    kern = oracle.kernel_pool(K, [0], [900], 32, 16)
    a = oracle.block_score_topk(q, kern, qc, oracle.Params(topk=3))
    b = oracle.block_score_topk(q, kern, qc, oracle.Params(topk=3, lse_stride=1))
    assert np.array_equal(a["lse"], b["lse"]) and np.array_equal(a["idx"], b["idx"])


@pytest.mark.parametrize("stride", [2, 3, 4])
def test_lse_estimate_closed_form_on_equal_scores(oracle, stride):
    """q = 0: every kernel scores 0, so the exact LSE is log(nk) and the estimate log(s * ceil(nk / s))."""
    rng = np.random.default_rng(61)
    _, K, _ = rand_case(rng, 1, 1, 700, 4, 2, 16)
    q = np.zeros((1, 3, 4, 16), np.uint16)
    qc = np.array([[700, 333, 130]], np.int32)
    kern = oracle.kernel_pool(K, [0], [700], 32, 16)
    r = oracle.block_score_topk(q, kern, qc, oracle.Params(topk=2, lse_stride=stride))
    for t in range(3):
        nk = oracle.num_kernels(int(qc[0, t]))
        assert np.allclose(r["lse"][0, t], math.log(stride * math.ceil(nk / stride)), rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------------
# gradient of the semantic kernels with respect to K (the transpose of the window mean)
# ------------------------------------------------------------------------------------------------

def test_kernel_pool_backward_is_the_adjoint_of_the_forward(oracle):
    """<backward(dkern), K> = <dkern, kernel_pool(K)> for every K and dkern: with K in {0, 1}, every window
    mean s / 32 (s <= 32) is exact in bf16, so the forward oracle's rounding drops out.  Ragged lengths, one
    below a window, one not on the 16-key grid; the gradient of kernels past nk(lens) must not reach K."""
    rng = np.random.default_rng(70)
    B, Lcap, Hkv, d = 3, 300, 2, 8
    lens = np.array([300, 151, 20], np.int32)
    Kf = rng.integers(0, 2, (B, Lcap, Hkv, d)).astype(np.float32)
    K = bits(Kf)
    nk_cap = oracle.num_kernels(Lcap)
    kern = oracle.kernel_pool(K, [0] * B, lens, 32, 16, nk_cap=nk_cap)
    dkern = rng.standard_normal((B, Hkv, nk_cap, d)).astype(np.float32)
    dk = oracle.kernel_pool_backward(dkern, lens, Lcap)
    for b in range(B):
        nk = oracle.num_kernels(int(lens[b]))
        lhs = np.sum(dk[b] * Kf[b].astype(np.float64))
        rhs = np.sum(dkern[b, :, :nk].astype(np.float64) * f64(kern[b, :, :nk]))
        assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)
        assert not dk[b, int(lens[b]):].any()  # keys past the context get nothing
    assert not dk[2].any()  # 20 keys: no complete window


def test_kernel_pool_backward_one_window_and_mass(oracle):
    """One kernel with gradient 1 spreads 1/32 over exactly its 32 keys; in general each kernel's gradient mass
    reaches K whole (the column sums of the mean are 1)."""
    B, Lcap, Hkv, d = 1, 128, 1, 4
    nk_cap = oracle.num_kernels(Lcap)
    dkern = np.zeros((B, Hkv, nk_cap, d), np.float32)
    dkern[0, 0, 3, :] = 1.0
    dk = oracle.kernel_pool_backward(dkern, [Lcap], Lcap)
    want = np.zeros(Lcap)
    want[48:80] = 1.0 / 32
    assert np.array_equal(dk[0, :, 0, 2], want)
    rng = np.random.default_rng(71)
    dkern = rng.standard_normal((2, 2, nk_cap, 6)).astype(np.float32)
    dk = oracle.kernel_pool_backward(dkern, [Lcap, 100], Lcap)
    assert np.allclose(dk[0].sum(axis=0), dkern[0].astype(np.float64).sum(axis=1), rtol=0, atol=1e-12)
    nk = oracle.num_kernels(100)
    assert np.allclose(dk[1].sum(axis=0), dkern[1, :, :nk].astype(np.float64).sum(axis=1), rtol=0, atol=1e-12)
