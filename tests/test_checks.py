"""The host-side input checks (INFLLMV2_CHECK=1): they accept what the oracle's own selection and the workloads
produce, and reject each kind of bad device-side input with an error naming the row (CPU only)."""
import numpy as np
import pytest
import torch

from trainable_block_sparse_v2_b200 import binding, checks
from trainable_block_sparse_v2_b200.workloads import prefill_case


def test_query_contexts_three_forms():
    qc = np.array([[5, 9, 2]], np.int32)
    assert checks.query_contexts(1, 3, q_ctx=qc).tolist() == [[5, 9, 2]]
    lens = np.array([10, 4], np.int32)
    assert checks.query_contexts(2, 3, ctx_lens=lens).tolist() == [[8, 9, 10], [2, 3, 4]]  # causal tail
    assert checks.query_contexts(2, 3, ctx_lens=lens, same_ctx=True).tolist() == [[10, 10, 10], [4, 4, 4]]
    with pytest.raises(checks.InputCheckError):
        checks.query_contexts(1, 1)


def test_contexts_in_range():
    ctx = np.array([[1, 64, 100]])
    checks.check_contexts(ctx, lcap=128, max_ctx=100)
    for bad, lcap, mx in ((np.array([[0, 5]]), 128, 100), (np.array([[5, 101]]), 128, 100),
                          (np.array([[5, 6]]), 90, 100)):
        with pytest.raises(checks.InputCheckError):
            checks.check_contexts(bad, lcap, mx)


def _selection(oracle):
    w = prefill_case(700, 8, 2, 64, topk=3, dense_len=200, seed=77, n_needles=2)
    P = oracle.Params(**w.params)
    kern = oracle.kernel_pool(w.k, [0], [700], 32, 16, nk_cap=oracle.num_kernels(700))
    r = oracle.block_score_topk(w.q, kern, w.q_ctx, P)
    return w, P, r["idx"].copy(), r["cnt"].copy()


def test_oracle_selection_passes_and_mutations_fail(oracle):
    w, P, idx, cnt = _selection(oracle)
    ctx = w.q_ctx.astype(np.int64)
    checks.check_block_lists(idx, cnt, ctx, P.kmax, P.dense_len)
    t = 600  # a sparse row (n = 601 > 200) with k + 3 = 6 blocks
    assert cnt[0, t, 0] == P.kmax
    mutations = {
        "descending": lambda a, c: a.__setitem__((0, t, 0, slice(0, 2)), a[0, t, 0, 1::-1].copy()),
        "duplicate": lambda a, c: a.__setitem__((0, t, 0, 1), a[0, t, 0, 0]),
        "past the context": lambda a, c: a.__setitem__((0, t, 0, P.kmax - 1), 601 // 64 + 1),
        "negative": lambda a, c: a.__setitem__((0, t, 0, 0), -1),
        "cnt above kmax": lambda a, c: c.__setitem__((0, t, 0), P.kmax + 1),
        "negative cnt": lambda a, c: c.__setitem__((0, t, 0), -2),
    }
    for name, mutate in mutations.items():
        a, c = idx.copy(), cnt.copy()
        mutate(a, c)
        with pytest.raises(checks.InputCheckError, match=r"\(0, 600, 0\)"):
            checks.check_block_lists(a, c, ctx, P.kmax, P.dense_len)
    # a dense row's list is not read: anything goes there
    a = idx.copy()
    a[0, 10, 1, :] = 9999
    checks.check_block_lists(a, cnt, ctx, P.kmax, P.dense_len)


def test_pool_lengths():
    checks.check_pool_lengths([0, 100], [1000, 101], lcap=1024, max_new_keys=1000, nk_cap=61)
    for old, new, lcap, mx, cap in (([5], [4], 64, 10, 10), ([0], [70], 64, 100, 10), ([0], [60], 64, 50, 10),
                                    ([0], [64], 64, 64, 2)):
        with pytest.raises(checks.InputCheckError):
            checks.check_pool_lengths(old, new, lcap, mx, cap)


def test_binding_hook_reads_the_environment_and_checks_tensors(oracle, monkeypatch):
    monkeypatch.delenv("INFLLMV2_CHECK", raising=False)
    assert not binding._checking()
    monkeypatch.setenv("INFLLMV2_CHECK", "1")
    assert binding._checking()
    w, P, idx, cnt = _selection(oracle)
    p = binding.Params(**w.params)
    lens = torch.tensor([700], dtype=torch.int32)
    binding._check_rows("prefill", 1, 700, None, lens, False, 700, 700, torch.from_numpy(idx), torch.from_numpy(cnt),
                        p)
    with pytest.raises(checks.InputCheckError, match="context"):
        binding._check_rows("prefill", 1, 700, None, torch.tensor([800], dtype=torch.int32), False, 1024, 700)
    bad = idx.copy()
    bad[0, 650, 1, 2] = bad[0, 650, 1, 1]
    with pytest.raises(checks.InputCheckError, match=r"\(0, 650, 1\)"):
        binding._check_rows("prefill", 1, 700, None, lens, False, 700, 700, torch.from_numpy(bad),
                            torch.from_numpy(cnt), p)


def test_tree_mask():
    from trainable_block_sparse_v2_b200.workloads import tree_mask_from_parents
    rng = np.random.default_rng(5)
    for _ in range(20):  # masks built from random trees pass
        n = int(rng.integers(1, 33))
        parent = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, n)])
        checks.check_tree_mask(tree_mask_from_parents(parent)[None], 1, n)
    good = tree_mask_from_parents(np.array([-1, 0, 1, 1]))  # 0 <- 1 <- {2, 3}
    for i, bad, msg in ((2, int(good[2]) & ~(1 << 2), "own bit"), (1, int(good[1]) | (1 << 4), "past n_draft"),
                        (3, (1 << 3) | (1 << 1), "ancestors")):
        m = good.astype(np.int64).copy()
        m[i] = bad
        with pytest.raises(checks.InputCheckError, match=msg):
            checks.check_tree_mask(m.astype(np.uint32)[None], 1, 4)


def test_page_table_check():
    table = np.array([[3, 0, -1], [1, 2, -1]], np.int32)
    checks.check_page_table(table, [128, 70], num_pages=4)              # 2 pages each, all in range
    with pytest.raises(checks.InputCheckError, match="outside"):
        checks.check_page_table(table, [129, 70], num_pages=4)          # a third page, mapped to -1
    with pytest.raises(checks.InputCheckError, match="outside"):
        checks.check_page_table(table, [128, 70], num_pages=3)          # page 3 past the pool
    with pytest.raises(checks.InputCheckError, match="serves both"):
        checks.check_page_table(np.array([[0, 1], [1, 2]], np.int32), [128, 64], num_pages=4)
    with pytest.raises(checks.InputCheckError, match="needs"):
        checks.check_page_table(table, [64 * 3 + 1, 1], num_pages=4)    # more pages than the table holds


def test_cu_seqlens_check():
    cq, ck = np.array([0, 5, 5, 9], np.int32), np.array([0, 7, 20, 29], np.int32)
    checks.check_cu_seqlens(cq, ck, 9, 29, 5, 13)
    with pytest.raises(checks.InputCheckError, match="never decrease"):
        checks.check_cu_seqlens(np.array([0, 5, 4, 9]), ck, 9, 29, 5, 13)
    with pytest.raises(checks.InputCheckError, match="queries but"):
        checks.check_cu_seqlens(np.array([0, 8, 8, 9]), ck, 9, 29, 8, 13)
    with pytest.raises(checks.InputCheckError, match="max_seqlen"):
        checks.check_cu_seqlens(cq, ck, 9, 29, 4, 13)
    with pytest.raises(checks.InputCheckError, match="end at"):
        checks.check_cu_seqlens(cq, ck, 10, 29, 5, 13)
