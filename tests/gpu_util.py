"""Helpers for the GPU parity tests: device transfer of bf16 bit patterns, parameter conversion, and the
comparison rules (selection bit-exact except at the oracle's near ties; attention within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle)."""
import numpy as np
import torch

import oracle
from trainable_block_sparse_v2_b200 import binding

ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
TIE_REL = 1e-3


def dev(a_u16):
    """numpy uint16 bf16 bits -> CUDA bf16 tensor (same bytes)"""
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).cuda().view(torch.bfloat16)


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host_u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(u16):
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bparams(p: dict) -> binding.Params:
    return binding.Params(**p)


def oparams(p: dict) -> oracle.Params:
    return oracle.Params(**p)


def check_selection(gidx, gcnt, r, c_of_row=None):
    """Compare GPU selection with the oracle's.  Returns the boolean mask of rows that match exactly.

    A row may differ only when the oracle's k-th and (k+1)-th ranked candidate scores are within 1e-3
    relative; such a row must still be a valid selection: the same count, and every block in which the two
    sets differ scores inside that tie band."""
    oidx, ocnt, S, gap = r["idx"], r["cnt"], r["S"], r["gap"]
    same = (gcnt == ocnt) & np.all(gidx == oidx, axis=-1)
    bad = np.argwhere(~same)
    for pos in bad:
        pos = tuple(pos)
        g0, g1 = gap[pos]
        assert np.isfinite(g1) and abs(g0 - g1) < TIE_REL * abs(g0), \
            f"selection differs at row {pos} without a near tie: gpu {gidx[pos][:gcnt[pos]]} oracle " \
            f"{oidx[pos][:ocnt[pos]]} gap {g0} {g1}"
        assert gcnt[pos] == ocnt[pos]
        a = set(gidx[pos][:gcnt[pos]].tolist())
        b = set(oidx[pos][:ocnt[pos]].tolist())
        for blk in a ^ b:
            assert abs(S[pos][blk] - g0) <= 2 * TIE_REL * abs(g0), (pos, blk, S[pos][blk], g0)
    return same


def check_attention(out_gpu, out_ref, lse_gpu=None, lse_ref=None, mask=None, what=""):
    """out_gpu: bf16 tensor [.., Hq, d]; out_ref: fp64 array; mask selects rows [..] (leading dims)."""
    g = out_gpu.float().cpu().numpy().astype(np.float64)
    diff = np.abs(g - out_ref)
    if mask is not None:
        diff = diff[mask]
    assert diff.size > 0
    mx, mean = float(diff.max()), float(diff.mean())
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    if lse_gpu is not None:
        ld = np.abs(lse_gpu.cpu().numpy().astype(np.float64) - lse_ref)
        if mask is not None:
            ld = ld[mask]
        assert float(ld.max()) <= LSE_ABS, f"{what}: lse max-abs {float(ld.max()):.3e}"
    return mx, mean
