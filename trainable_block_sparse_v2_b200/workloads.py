"""Seeded synthetic inputs for the InfLLM v2 path (shared by the tests, the benchmark and the oracle legs).

This module holds input generation only -- none of the method's arithmetic.  Every tensor is drawn in
fp32 with ``numpy.random.default_rng`` and stored as bf16 bit patterns (round to nearest even) in
``numpy.uint16`` arrays, so the CUDA path and the CPU oracle read identical bytes.

The workloads stand in for the pages' long-context evaluation (RULER needle-in-a-haystack at 128K on
MiniCPM4 with YaRN; QbitAI "MiniCPM4 technical details", long-context evaluation) and for a model's
KV cache, neither of which exists here: values are N(0, 1) with planted "needle" blocks whose keys are
shifted toward the mean query of a group, or with per-block mean offsets.

Layouts: q [B, T, Hq, d]; K/V cache [B, Lcap, Hkv, d]; q_ctx [B, T] = context length n seen by each
query (position + 1 for ordinary queries, the prefix length for tree-draft queries).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# method constants of the five workloads (block 64, window 32 / stride 16, 1 initial + 2 local blocks)
BLOCK, KSIZE, KSTRIDE, INIT, LOCAL = 64, 32, 16, 1, 2


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


@dataclass
class Workload:
    name: str
    q: np.ndarray            # [B, T, Hq, d] bf16 bits
    k: np.ndarray            # [B, Lcap, Hkv, d] bf16 bits
    v: np.ndarray            # [B, Lcap, Hkv, d] bf16 bits
    q_ctx: np.ndarray        # [B, T] int32
    ctx_lens: np.ndarray     # [B] int32: keys present in the cache (the last query's n)
    params: dict             # block_size, kernel_size, kernel_stride, topk, init_blocks, local_blocks, dense_len
    extras: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, T, Hq, d = self.q.shape
        return dict(B=B, T=T, Hq=Hq, Hkv=self.k.shape[2], d=d, Lcap=self.k.shape[1])


def method_params(topk: int, dense_len: int, membership: int = 0) -> dict:
    return dict(block_size=BLOCK, kernel_size=KSIZE, kernel_stride=KSTRIDE, topk=topk, init_blocks=INIT,
                local_blocks=LOCAL, dense_len=dense_len, membership=membership)


def _plant_needles(rng, K, L, qbar, n_needles, shift=0.5):
    """Add shift*qbar[g] to the keys of n_needles blocks drawn without replacement from 1 .. c-3.

    K: fp32 [Lcap, Hkv, d] for one sequence; qbar: [Hkv, d]; L: context length.  Returns block ids.
    """
    c = (L - 1) // BLOCK
    hi = max(2, c - 2)  # blocks 1 .. c-3 are ordinary candidates
    n = min(n_needles, hi - 1)
    blocks = np.sort(rng.choice(np.arange(1, hi), size=n, replace=False)) if n > 0 else np.zeros(0, np.int64)
    for blk in blocks:
        K[blk * BLOCK:(blk + 1) * BLOCK] += shift * qbar[None, :, :]
    return blocks


def prefill_case(T, Hq, Hkv, d, topk, dense_len, seed, n_needles=3, block_offset_std=0.0, membership=0,
                 name="prefill"):
    """Causal prefill of one sequence of T tokens (q_ctx = t + 1).

    n_needles > 0: keys of that many blocks are shifted by 0.5 * (mean of Q over all tokens and the
    group's heads).  block_offset_std > 0: every (64-token block, head) of Q, K and V gets its own
    N(0, std^2 I) mean offset (query heads for Q, KV heads for K/V).
    """
    rng = np.random.default_rng(seed)
    G = Hq // Hkv
    q = _normal(rng, (T, Hq, d))
    k = _normal(rng, (T, Hkv, d))
    v = _normal(rng, (T, Hkv, d))
    if block_offset_std > 0:
        nb = (T + BLOCK - 1) // BLOCK
        for arr, H in ((q, Hq), (k, Hkv), (v, Hkv)):
            mu = block_offset_std * _normal(rng, (nb, H, d))
            arr += np.repeat(mu, BLOCK, axis=0)[:T]
    needles = np.zeros(0, np.int64)
    if n_needles > 0:
        qbar = q.reshape(T, Hkv, G, d).mean(axis=(0, 2))
        needles = _plant_needles(rng, k, T, qbar, n_needles)
    return Workload(
        name=name,
        q=f32_to_bf16_bits(q)[None], k=f32_to_bf16_bits(k)[None], v=f32_to_bf16_bits(v)[None],
        q_ctx=np.arange(1, T + 1, dtype=np.int32)[None], ctx_lens=np.array([T], np.int32),
        params=method_params(topk, dense_len, membership), extras=dict(needles=needles))


def decode_case(lens, Hq, Hkv, d, topk, dense_len, seed, n_needles=16, steps=1, membership=0, name="decode"):
    """Decode of B sequences with contexts ``lens`` at step 0 (the step's new token included), ``steps``
    consecutive steps (each step appends one token, so step s sees lens + s keys).

    q: [steps, B, 1, Hq, d] in extras['q_steps'] (q = step 0's).  The cache holds every step's token from
    the start (capacity max(lens) + steps - 1); callers append nothing, they advance the lengths.  Each
    sequence b draws from its own generator (seed + 100 * b).  Needles: keys of n_needles blocks of each
    sequence shifted by 0.5 * (mean of step 0's query over the group's heads).
    """
    lens = np.asarray(lens, np.int64)
    B = len(lens)
    G = Hq // Hkv
    Lcap = int(lens.max()) + steps - 1
    Lcap = (Lcap + 15) // 16 * 16
    K = np.empty((B, Lcap, Hkv, d), np.uint16)
    V = np.empty((B, Lcap, Hkv, d), np.uint16)
    Q = np.empty((steps, B, 1, Hq, d), np.uint16)
    needles = []
    for b in range(B):
        rng = np.random.default_rng(seed + 100 * b)
        qs = _normal(rng, (steps, Hq, d))
        kb = _normal(rng, (Lcap, Hkv, d))
        vb = _normal(rng, (Lcap, Hkv, d))
        qbar = qs[0].reshape(Hkv, G, d).mean(axis=1)
        needles.append(_plant_needles(rng, kb, int(lens[b]), qbar, n_needles))
        K[b] = f32_to_bf16_bits(kb)
        V[b] = f32_to_bf16_bits(vb)
        Q[:, b, 0] = f32_to_bf16_bits(qs)
    return Workload(
        name=name, q=Q[0], k=K, v=V, q_ctx=lens.astype(np.int32)[:, None], ctx_lens=lens.astype(np.int32),
        params=method_params(topk, dense_len, membership),
        extras=dict(q_steps=Q, steps=steps, needles=needles))


def tree_parents(rng, n_nodes, max_depth=6):
    """Random draft tree: parent[0] = -1 (root, depth 0); node i >= 1 picks a parent uniformly among the
    earlier nodes of depth < max_depth, so every depth is <= max_depth."""
    parent = np.full(n_nodes, -1, np.int64)
    depth = np.zeros(n_nodes, np.int64)
    for i in range(1, n_nodes):
        ok = np.nonzero(depth[:i] < max_depth)[0]
        parent[i] = int(rng.choice(ok))
        depth[i] = depth[parent[i]] + 1
    return parent, depth


def tree_mask_from_parents(parent):
    """Bit-packed ancestor mask: bit j of mask[i] is set when node j is node i or one of its ancestors."""
    n = len(parent)
    mask = np.zeros(n, np.uint32)
    for i in range(n):
        j = i
        while j >= 0:
            mask[i] |= np.uint32(1) << np.uint32(j)
            j = parent[j]
    return mask


def tree_case(P, n_draft, Hq, Hkv, d, topk, dense_len, seed, max_depth=6, B=1, parents=None, name="tree"):
    """Tree verification: B sequences with a P-token prefix in the cache and n_draft draft nodes each.

    Draft q/K/V ~ N(0,1) in q [B, n_draft, Hq, d] and extras['k_draft'/'v_draft'] [B, n_draft, Hkv, d];
    every draft query sees the whole prefix (q_ctx = P); extras['tree_mask'] [B, n_draft] uint32.
    """
    Lcap = (P + 15) // 16 * 16
    Q = np.empty((B, n_draft, Hq, d), np.uint16)
    K = np.empty((B, Lcap, Hkv, d), np.uint16)
    V = np.empty((B, Lcap, Hkv, d), np.uint16)
    KD = np.empty((B, n_draft, Hkv, d), np.uint16)
    VD = np.empty((B, n_draft, Hkv, d), np.uint16)
    masks = np.empty((B, n_draft), np.uint32)
    par_all = []
    for b in range(B):
        rng = np.random.default_rng(seed + 100 * b)
        K[b] = f32_to_bf16_bits(_normal(rng, (Lcap, Hkv, d)))
        V[b] = f32_to_bf16_bits(_normal(rng, (Lcap, Hkv, d)))
        Q[b] = f32_to_bf16_bits(_normal(rng, (n_draft, Hq, d)))
        KD[b] = f32_to_bf16_bits(_normal(rng, (n_draft, Hkv, d)))
        VD[b] = f32_to_bf16_bits(_normal(rng, (n_draft, Hkv, d)))
        par = parents if parents is not None else tree_parents(rng, n_draft, max_depth)[0]
        masks[b] = tree_mask_from_parents(par)
        par_all.append(par)
    return Workload(
        name=name, q=Q, k=K, v=V, q_ctx=np.full((B, n_draft), P, np.int32), ctx_lens=np.full(B, P, np.int32),
        params=method_params(topk, dense_len),
        extras=dict(k_draft=KD, v_draft=VD, tree_mask=masks, parents=par_all))


# ---- the five named workloads (seed 1000 + i) ------------------------------------------------------

def tiny_prefill(seed=1001):
    """batch 1, 2048 tokens, 4 query / 2 KV heads, d 64, top-k 8, 3 needle blocks, no dense rows."""
    return prefill_case(2048, 4, 2, 64, topk=8, dense_len=0, seed=seed, n_needles=3, name="tiny_prefill_2k")


def decode_32k(seed=1002):
    """batch 1, 32K context (new token included), 32 / 2 heads, d 128, top-k 64, 16 needles."""
    return decode_case([32768], 32, 2, 128, topk=64, dense_len=8192, seed=seed, n_needles=16,
                       name="decode_32k")


def prefill_32k(seed=1003, T=32768):
    """batch 1, 32K tokens, 32 / 2 heads, d 128, top-k 64, per-block offsets N(0, 0.3^2), dense below 8192."""
    return prefill_case(T, 32, 2, 128, topk=64, dense_len=8192, seed=seed, n_needles=0, block_offset_std=0.3,
                        name="prefill_32k")


def decode_128k_ragged(seed=1004, steps=256, lens=(131072, 98304, 65536, 131072)):
    """batch 4 ragged (128K, 96K, 64K, 128K at step 0), 32 / 2 heads, d 128, top-k 64, 64 needles each."""
    return decode_case(list(lens), 32, 2, 128, topk=64, dense_len=8192, seed=seed, n_needles=64, steps=steps,
                       name="decode_128k_ragged")


def tree_verify_64k(seed=1005, P=65536):
    """batch 1, 64K prefix, 16 draft nodes (depth <= 6), 32 / 2 heads, d 128, top-k 64."""
    return tree_case(P, 16, 32, 2, 128, topk=64, dense_len=8192, seed=seed, name="tree_verify_64k")
