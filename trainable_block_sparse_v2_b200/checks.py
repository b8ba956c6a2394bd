"""Host-side checks of the device-side inputs of the C-ABI calls, for debugging.

The library validates every size and pointer on the host before it launches anything, but it trusts the
values that live in device memory: the per-query contexts (``q_ctx`` or ``ctx_lens``) and the block lists
(``idx`` / ``cnt``).  The kernels skip a block id that is negative or lies past the query's context, but a
context past ``max_ctx`` or the cache, or a list that repeats a block, gives results that are not the
method's (a repeated block counts its keys twice).  With ``INFLLMV2_CHECK=1`` in the environment the binding
copies those inputs to the host before every call and checks them here; a violation raises
``InputCheckError`` naming the first offending row.  The checks synchronise with the device, so they are a
debugging aid, not part of the timed path.
"""
from __future__ import annotations

import numpy as np


class InputCheckError(ValueError):
    pass


def _np(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (any device)
        return a.detach().cpu().numpy()
    return np.asarray(a)


def query_contexts(B: int, T: int, q_ctx=None, ctx_lens=None, same_ctx: bool = False) -> np.ndarray:
    """Context length n of every query [B, T]: q_ctx when given; otherwise ctx_lens[b] for every query
    (tree drafts, decode) when same_ctx, else the causal tail n = ctx_lens[b] - T + t + 1."""
    if q_ctx is not None:
        return _np(q_ctx).reshape(B, T).astype(np.int64)
    if ctx_lens is None:
        raise InputCheckError("neither q_ctx nor ctx_lens given")
    lens = _np(ctx_lens).reshape(B).astype(np.int64)
    if same_ctx:
        return np.repeat(lens[:, None], T, axis=1)
    return lens[:, None] - T + np.arange(T)[None, :] + 1


def check_contexts(ctx: np.ndarray, lcap: int, max_ctx: int, what: str = "") -> None:
    """1 <= n <= max_ctx <= lcap for every query."""
    if max_ctx > lcap:
        raise InputCheckError(f"{what}: max_ctx {max_ctx} > cache length {lcap}")
    bad = np.argwhere((ctx < 1) | (ctx > max_ctx))
    if bad.size:
        pos = tuple(int(i) for i in bad[0])
        raise InputCheckError(f"{what}: query {pos} has context {int(ctx[pos])}, outside [1, {max_ctx}]")


def check_block_lists(idx, cnt, ctx: np.ndarray, kmax: int, dense_len: int, block: int = 64,
                      what: str = "") -> None:
    """Every sparse query's list (n > dense_len): 0 <= cnt <= kmax, and its first cnt ids ascending,
    unique, >= 0 and starting before the context (block * id < n).  Dense queries' lists are not read."""
    idx = _np(idx)
    cnt = _np(cnt)
    B, T, Hkv, km = idx.shape
    if km != kmax:
        raise InputCheckError(f"{what}: idx rows hold {km} entries, kmax is {kmax}")
    if cnt.shape != (B, T, Hkv):
        raise InputCheckError(f"{what}: cnt has shape {cnt.shape}, expected {(B, T, Hkv)}")
    for b in range(B):
        for t in range(T):
            n = int(ctx[b, t])
            if n <= dense_len:
                continue
            for g in range(Hkv):
                c = int(cnt[b, t, g])
                if c < 0 or c > kmax:
                    raise InputCheckError(f"{what}: row {(b, t, g)} has cnt {c}, outside [0, {kmax}]")
                ids = idx[b, t, g, :c].astype(np.int64)
                if c and (ids[0] < 0 or ids[-1] * block >= n):
                    raise InputCheckError(f"{what}: row {(b, t, g)} has a block id outside [0, {(n - 1) // block}]: "
                                          f"{ids.tolist()}")
                if c > 1 and np.any(np.diff(ids) <= 0):
                    raise InputCheckError(f"{what}: row {(b, t, g)} block ids are not ascending and unique: "
                                          f"{ids.tolist()}")


def check_pool_lengths(old_lens, new_lens, lcap: int, max_new_keys: int, nk_cap: int, kernel_size: int = 32,
                       kernel_stride: int = 16, what: str = "") -> None:
    """0 <= old <= new <= lcap, new - old <= max_new_keys, and the kernels of new keys fit in nk_cap."""
    old = _np(old_lens).astype(np.int64).ravel()
    new = _np(new_lens).astype(np.int64).ravel()
    for b, (o, n) in enumerate(zip(old, new)):
        if not (0 <= o <= n <= lcap):
            raise InputCheckError(f"{what}: sequence {b} has old {o}, new {n} (cache {lcap})")
        if n - o > max_new_keys:
            raise InputCheckError(f"{what}: sequence {b} adds {n - o} keys, max_new_keys is {max_new_keys}")
        nk = (n - kernel_size) // kernel_stride + 1 if n >= kernel_size else 0
        if nk > nk_cap:
            raise InputCheckError(f"{what}: sequence {b} needs {nk} kernels, nk_cap is {nk_cap}")


def check_tree_mask(tree_mask, B: int, n_draft: int, what: str = "") -> None:
    """Every draft node's mask is an ancestor mask: it has its own bit, no bit at or past n_draft, and it holds
    every node its nodes see (node i seeing node j sees all of j's ancestors)."""
    m = _np(tree_mask).astype(np.int64).reshape(B, n_draft) & 0xFFFFFFFF
    for b in range(B):
        for i in range(n_draft):
            mi = int(m[b, i])
            if not (mi >> i) & 1:
                raise InputCheckError(f"{what}: tree_mask[{b}, {i}] lacks the node's own bit")
            if mi >> n_draft:
                raise InputCheckError(f"{what}: tree_mask[{b}, {i}] has bits at or past n_draft = {n_draft}")
            for j in range(n_draft):
                if (mi >> j) & 1 and int(m[b, j]) & ~mi:
                    raise InputCheckError(f"{what}: node {i} of sequence {b} sees node {j} but not all of node "
                                          f"{j}'s ancestors")


def check_page_table(page_table, lens, num_pages: int, what: str = "") -> None:
    """Every page a sequence's first lens[b] positions use (entries [0, ceil(lens[b] / 64))) is in
    [0, num_pages), the table has room for them, and no page serves two (sequence, block) slots."""
    table = _np(page_table).astype(np.int64)
    lens = _np(lens).astype(np.int64).ravel()
    B, max_pages = table.shape
    seen = {}
    for b in range(B):
        used = (int(lens[b]) + 63) // 64
        if used > max_pages:
            raise InputCheckError(f"{what}: sequence {b} needs {used} pages, the table has {max_pages}")
        for i in range(used):
            p = int(table[b, i])
            if p < 0 or p >= num_pages:
                raise InputCheckError(f"{what}: page_table[{b}, {i}] = {p}, outside [0, {num_pages})")
            if p in seen:
                raise InputCheckError(f"{what}: page {p} serves both {seen[p]} and {(b, i)}")
            seen[p] = (b, i)


def check_cu_seqlens(cu_q, cu_k, total_q: int, total_k: int, max_q: int, max_k: int, what: str = "") -> None:
    """Packed batch offsets: both start at 0, never decrease and end at the totals; every sequence has at most
    as many queries as keys, and the maxima bound the lengths."""
    cq = _np(cu_q).astype(np.int64).ravel()
    ck = _np(cu_k).astype(np.int64).ravel()
    if len(cq) != len(ck) or len(cq) < 2:
        raise InputCheckError(f"{what}: cu_seqlens_q / cu_seqlens_k must both hold B + 1 >= 2 offsets")
    for name, cu, total in (("cu_seqlens_q", cq, total_q), ("cu_seqlens_k", ck, total_k)):
        if cu[0] != 0 or cu[-1] != total or np.any(np.diff(cu) < 0):
            raise InputCheckError(f"{what}: {name} must start at 0, never decrease and end at {total}")
    tq, tk = np.diff(cq), np.diff(ck)
    bad = np.nonzero(tq > tk)[0]
    if len(bad):
        raise InputCheckError(f"{what}: sequence {int(bad[0])} has {int(tq[bad[0]])} queries but {int(tk[bad[0]])} keys")
    if tq.max() > max_q or tk.max() > max_k:
        raise InputCheckError(f"{what}: max_seqlen_q / max_seqlen_k below the longest sequence "
                              f"({int(tq.max())} / {int(tk.max())})")
