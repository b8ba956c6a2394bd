"""fp64 CPU oracle of the InfLLM v2 sparse-attention path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of ``bench.py``
may import this package.  The product library (``trainable_block_sparse_v2_b200``) never imports it,
and this package imports nothing from the product: the two share no code.  The arithmetic lives in
``infllmv2_oracle.c`` (plain C, fp64); this module only compiles it with gcc and marshals numpy
arrays through ctypes.

Inputs are bf16 bit patterns held in ``numpy.uint16`` arrays (the same bytes the CUDA path reads).

Functions and the steps they follow (sources: the MiniCPM4 pages):
  * ``kernel_pool``        -- semantic kernels = window means of K, rounded to bf16
                              (QbitAI "MiniCPM4 technical details", "Model architecture: InfLLM v2", item 1)
  * ``block_score_topk``   -- max-over-kernels relevance, LSE-normalised per head, summed over the GQA
                              group, top-k plus initial and local blocks (same section, items 1-3)
  * ``sparse_attention``   -- attention over the selected blocks, optional bit-packed tree-draft mask
                              (same article, "speculative sampling ... long text", long-context bullet)
  * ``sparse_attention_backward`` -- gradients of that attention for a fixed selection (training; same
                              section, item 3: operators for training and inference; the derivative of
                              the forward's definition)
  * ``kernel_pool_backward`` -- the gradient of the semantic kernels with respect to K: the transpose of the
                              window mean (same section, item 3; the derivative of step 1's definition)
  * ``dense_attention``    -- plain causal GQA attention, written separately
  * ``window_attention``   -- the draft model's sliding-window attention (same bullet as the tree drafts)
The pages' "efficient LogSumExp estimation" is not defined there (parity unpinned); ``Params.lse_stride`` selects
one reading of it (the LSE from every s-th visible kernel, times s), pinned only to its special cases.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "infllmv2_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liborc.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no FP contraction, OpenMP).  Returns the library path."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-shared", "-fPIC",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [
        ("block_size", ctypes.c_int),
        ("kernel_size", ctypes.c_int),
        ("kernel_stride", ctypes.c_int),
        ("topk", ctypes.c_int),
        ("init_blocks", ctypes.c_int),
        ("local_blocks", ctypes.c_int),
        ("dense_len", ctypes.c_int),
        ("membership", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("lse_stride", ctypes.c_int),
    ]


@dataclass
class Params:
    """Method constants.  ``scale`` None means 1/sqrt(head_dim).  membership: 0 OVERLAP, 1 CONTAINED."""
    block_size: int = 64
    kernel_size: int = 32
    kernel_stride: int = 16
    topk: int = 64
    init_blocks: int = 1
    local_blocks: int = 2
    dense_len: int = 0
    membership: int = 0
    scale: float | None = None
    lse_stride: int = 0  # 0 / 1: exact LSE; s > 1: estimated from every s-th visible kernel (times s)

    @property
    def kmax(self) -> int:
        return self.topk + self.init_blocks + self.local_blocks

    def c_struct(self, head_dim: int) -> _Params:
        s = self.scale if self.scale is not None else 1.0 / math.sqrt(head_dim)
        return _Params(self.block_size, self.kernel_size, self.kernel_stride, self.topk, self.init_blocks,
                       self.local_blocks, self.dense_len, self.membership, float(s), int(self.lse_stride))


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.orc_kernel_pool.argtypes = [P, i, i, i, i, P, P, i, i, P, i]
        lib.orc_kernel_pool.restype = i
        lib.orc_block_score_topk.argtypes = [P, i, i, i, i, i, P, i, P, ctypes.POINTER(_Params), i, i,
                                             P, P, P, P, P]
        lib.orc_block_score_topk.restype = i
        lib.orc_sparse_attention.argtypes = [P, i, i, i, i, i, P, P, i, P, P, P, i, ctypes.POINTER(_Params),
                                             P, P, P, P, P]
        lib.orc_sparse_attention.restype = i
        lib.orc_sparse_attention_backward.argtypes = [P, i, i, i, i, i, P, P, i, P, P, P, i,
                                                      ctypes.POINTER(_Params), P, P, P, P]
        lib.orc_sparse_attention_backward.restype = i
        lib.orc_dense_attention.argtypes = [P, i, i, i, i, i, P, P, i, P, ctypes.c_double, P, P]
        lib.orc_dense_attention.restype = i
        lib.orc_window_attention.argtypes = [P, i, i, i, i, i, P, P, i, P, i, ctypes.c_double, P, P]
        lib.orc_window_attention.restype = i
        lib.orc_kernel_pool_backward.argtypes = [P, i, i, i, i, P, i, i, i, P]
        lib.orc_kernel_pool_backward.restype = i
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_round_bf16.restype = ctypes.c_uint16
        lib.orc_num_threads.restype = i
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().orc_num_threads())


def num_kernels(n: int, kernel_size: int = 32, kernel_stride: int = 16) -> int:
    """Complete kernel windows over the first n keys."""
    return 0 if n < kernel_size else (n - kernel_size) // kernel_stride + 1


def round_bf16(x: float) -> int:
    """bf16 bits of fp64 x, round to nearest even (one rounding step)."""
    return int(_load().orc_round_bf16(float(x)))


def kernel_pool(K, old_len, new_len, kernel_size, kernel_stride, kern=None, nk_cap=None):
    """Semantic kernels of K ([B, Lcap, Hkv, d] bf16 bits) for windows completed between old_len and new_len.

    Returns kern [B, Hkv, nk_cap, d] bf16 bits (updated in place when given).
    """
    lib = _load()
    K = _c(K, np.uint16)
    B, Lcap, Hkv, d = K.shape
    old_len = _c(old_len, np.int32)
    new_len = _c(new_len, np.int32)
    if nk_cap is None:
        nk_cap = max(1, num_kernels(int(new_len.max()), kernel_size, kernel_stride))
    if kern is None:
        kern = np.zeros((B, Hkv, nk_cap, d), np.uint16)
    assert kern.dtype == np.uint16 and kern.flags.c_contiguous and kern.shape == (B, Hkv, nk_cap, d)
    rc = lib.orc_kernel_pool(_ptr(K), B, Lcap, Hkv, d, _ptr(old_len), _ptr(new_len), kernel_size,
                             kernel_stride, _ptr(kern), nk_cap)
    if rc != 0:
        raise ValueError(f"orc_kernel_pool: bad arguments (rc={rc})")
    return kern


def kernel_pool_backward(dkern, lens, Lcap, kernel_size=32, kernel_stride=16):
    """dK ([B, Lcap, Hkv, d] fp64) for the kernel gradients dkern ([B, Hkv, nk_cap, d] fp32) of the kernels
    j < nk(lens[b]): each kernel gives 1/kernel_size of its gradient to each key of its window."""
    lib = _load()
    dkern = _c(dkern, np.float32)
    B, Hkv, nk_cap, d = dkern.shape
    lens = _c(lens, np.int32)
    dk = np.zeros((B, Lcap, Hkv, d), np.float64)
    rc = lib.orc_kernel_pool_backward(_ptr(dkern), B, Lcap, Hkv, d, _ptr(lens), kernel_size, kernel_stride, nk_cap,
                                      _ptr(dk))
    if rc != 0:
        raise ValueError(f"orc_kernel_pool_backward: bad arguments (rc={rc})")
    return dk


def block_score_topk(q, kern, q_ctx, params: Params, nb_max=None):
    """Group block scores and selection.

    q: [B, T, Hq, d] bf16 bits; kern: [B, Hkv, nk_cap, d] bf16 bits; q_ctx: [B, T] int context lengths.
    Returns dict(S [B,T,Hkv,nb_max] f64, lse [B,T,Hq] f64, idx [B,T,Hkv,kmax] i32, cnt [B,T,Hkv] i32,
    gap [B,T,Hkv,2] f64).
    """
    lib = _load()
    q = _c(q, np.uint16)
    kern = _c(kern, np.uint16)
    q_ctx = _c(q_ctx, np.int32)
    B, T, Hq, d = q.shape
    _, Hkv, nk_cap, _ = kern.shape
    if nb_max is None:
        nb_max = int((q_ctx.max() - 1) // params.block_size) + 1
    kmax = params.kmax
    S = np.empty((B, T, Hkv, nb_max), np.float64)
    lse = np.empty((B, T, Hq), np.float64)
    idx = np.empty((B, T, Hkv, kmax), np.int32)
    cnt = np.empty((B, T, Hkv), np.int32)
    gap = np.empty((B, T, Hkv, 2), np.float64)
    cp = params.c_struct(d)
    rc = lib.orc_block_score_topk(_ptr(q), B, T, Hq, Hkv, d, _ptr(kern), nk_cap, _ptr(q_ctx), ctypes.byref(cp),
                                  nb_max, kmax, _ptr(S), _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(gap))
    if rc != 0:
        raise ValueError(f"orc_block_score_topk: bad arguments (rc={rc})")
    return dict(S=S, lse=lse, idx=idx, cnt=cnt, gap=gap)


def sparse_attention(q, K, V, q_ctx, idx, cnt, params: Params, k_draft=None, v_draft=None, tree_mask=None):
    """Attention over the selected blocks (dense for rows with n <= dense_len), optional tree drafts.

    q: [B,T,Hq,d]; K, V: [B,Lcap,Hkv,d]; q_ctx: [B,T]; idx: [B,T,Hkv,kmax]; cnt: [B,T,Hkv];
    k_draft/v_draft: [B,T,Hkv,d]; tree_mask: [B,T] uint32.  Returns (out [B,T,Hq,d] f64, lse [B,T,Hq] f64).
    """
    lib = _load()
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    q_ctx = _c(q_ctx, np.int32)
    idx = _c(idx, np.int32)
    cnt = _c(cnt, np.int32)
    B, T, Hq, d = q.shape
    _, Lcap, Hkv, _ = K.shape
    kmax = idx.shape[-1]
    out = np.empty((B, T, Hq, d), np.float64)
    lse = np.empty((B, T, Hq), np.float64)
    if tree_mask is not None:
        k_draft = _c(k_draft, np.uint16)
        v_draft = _c(v_draft, np.uint16)
        tree_mask = _c(tree_mask, np.uint32)
    cp = params.c_struct(d)
    rc = lib.orc_sparse_attention(_ptr(q), B, T, Hq, Hkv, d, _ptr(K), _ptr(V), Lcap, _ptr(q_ctx), _ptr(idx),
                                  _ptr(cnt), kmax, ctypes.byref(cp), _ptr(k_draft), _ptr(v_draft),
                                  _ptr(tree_mask), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"orc_sparse_attention: bad arguments (rc={rc})")
    return out, lse


def sparse_attention_backward(q, K, V, q_ctx, idx, cnt, params: Params, dout):
    """Gradients of sum(dout * out) for the sparse attention with a fixed selection (no tree drafts).

    Same inputs as sparse_attention plus dout [B,T,Hq,d] (bf16 bits).  Returns (dq [B,T,Hq,d],
    dk [B,Lcap,Hkv,d], dv [B,Lcap,Hkv,d]), all f64.
    """
    lib = _load()
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    dout = _c(dout, np.uint16)
    q_ctx = _c(q_ctx, np.int32)
    idx = _c(idx, np.int32)
    cnt = _c(cnt, np.int32)
    B, T, Hq, d = q.shape
    _, Lcap, Hkv, _ = K.shape
    kmax = idx.shape[-1]
    dq = np.empty((B, T, Hq, d), np.float64)
    dk = np.empty((B, Lcap, Hkv, d), np.float64)
    dv = np.empty((B, Lcap, Hkv, d), np.float64)
    cp = params.c_struct(d)
    rc = lib.orc_sparse_attention_backward(_ptr(q), B, T, Hq, Hkv, d, _ptr(K), _ptr(V), Lcap, _ptr(q_ctx),
                                           _ptr(idx), _ptr(cnt), kmax, ctypes.byref(cp), _ptr(dout), _ptr(dq),
                                           _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError(f"orc_sparse_attention_backward: bad arguments (rc={rc})")
    return dq, dk, dv


def dense_attention(q, K, V, q_ctx, scale=None):
    """Plain causal GQA attention over keys [0, n) for every query.  Returns (out f64, lse f64)."""
    lib = _load()
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    q_ctx = _c(q_ctx, np.int32)
    B, T, Hq, d = q.shape
    _, Lcap, Hkv, _ = K.shape
    s = scale if scale is not None else 1.0 / math.sqrt(d)
    out = np.empty((B, T, Hq, d), np.float64)
    lse = np.empty((B, T, Hq), np.float64)
    rc = lib.orc_dense_attention(_ptr(q), B, T, Hq, Hkv, d, _ptr(K), _ptr(V), Lcap, _ptr(q_ctx), float(s),
                                 _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"orc_dense_attention: bad arguments (rc={rc})")
    return out, lse


def window_attention(q, K, V, q_ctx, window, scale=None):
    """The draft model's sliding-window attention: keys [max(0, n - window), n) for every query.
    Returns (out f64, lse f64)."""
    lib = _load()
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    q_ctx = _c(q_ctx, np.int32)
    B, T, Hq, d = q.shape
    _, Lcap, Hkv, _ = K.shape
    s = scale if scale is not None else 1.0 / math.sqrt(d)
    out = np.empty((B, T, Hq, d), np.float64)
    lse = np.empty((B, T, Hq), np.float64)
    rc = lib.orc_window_attention(_ptr(q), B, T, Hq, Hkv, d, _ptr(K), _ptr(V), Lcap, _ptr(q_ctx), int(window),
                                  float(s), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"orc_window_attention: bad arguments (rc={rc})")
    return out, lse


def bf16_bits_to_f64(a) -> np.ndarray:
    """Widen bf16 bit patterns exactly to fp64 (a data-type conversion, not part of the method)."""
    a = np.asarray(a, np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
