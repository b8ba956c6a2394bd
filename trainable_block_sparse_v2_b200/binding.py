"""ctypes binding of libinfllmv2.so -- argument marshalling only.

Every function has the name of the C entry point it calls (include/infllmv2.h), takes torch CUDA tensors
(or plain ints), checks dtype / device / contiguity, passes raw device pointers and sizes, and raises
``Infllmv2Error`` when the library returns a non-zero status.  All computation happens in the library's
CUDA kernels; there is no CPU fallback: if the library is missing, ``load()`` raises.

Layouts (bf16 unless stated): q [B, T, Hq, d]; k / v cache [B, Lcap, Hkv, d]; kern [B, Hkv, nk_cap, d];
idx [B, T, Hkv, kmax] int32; cnt [B, T, Hkv] int32; out [B, T, Hq, d]; lse [B, T, Hq] float32.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libinfllmv2.so")
_lib = None

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace", 4: "cuda", 5: "timeout"}


class Infllmv2Error(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class CParams(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int), ("kernel_size", ctypes.c_int), ("kernel_stride", ctypes.c_int),
                ("topk", ctypes.c_int), ("init_blocks", ctypes.c_int), ("local_blocks", ctypes.c_int),
                ("dense_len", ctypes.c_int), ("membership", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("lse_stride", ctypes.c_int)]


@dataclass
class Params:
    """Method constants (infllmv2_params).  softmax_scale <= 0 selects 1/sqrt(d)."""
    block_size: int = 64
    kernel_size: int = 32
    kernel_stride: int = 16
    topk: int = 64
    init_blocks: int = 1
    local_blocks: int = 2
    dense_len: int = 0
    membership: int = 0
    softmax_scale: float = 0.0
    lse_stride: int = 0  # 0 / 1: exact LSE; 2, 4, 8: estimated from every s-th kernel (prefill scoring, tensor cores)

    @property
    def kmax(self) -> int:
        return self.topk + self.init_blocks + self.local_blocks

    def c(self) -> CParams:
        return CParams(self.block_size, self.kernel_size, self.kernel_stride, self.topk, self.init_blocks,
                       self.local_blocks, self.dense_len, self.membership, float(self.softmax_scale),
                       int(self.lse_stride))


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_PP = ctypes.POINTER(CParams)
_F = ctypes.c_float

_SIGS = {
    "infllmv2_status_string": ([_I], ctypes.c_char_p),
    "infllmv2_version": ([], _I),
    "infllmv2_device_status": ([], _I),
    "infllmv2_test_set_first_wait_limit": ([ctypes.c_uint], _I),
    "infllmv2_workspace_size": ([_PP, _I, _I, _I, _I, _I, _I], _SZ),
    "infllmv2_kernel_pool": ([_P, _I, _I, _I, _I, _P, _P, _I, _PP, _P, _I, _P], _I),
    "infllmv2_kv_append": ([_P, _P, _I, _I, _I, _P, _P, _P, _I, _P], _I),
    "infllmv2_kernel_pool_backward": ([_P, _I, _I, _I, _I, _P, _I, _PP, _I, _P, _I, _P], _I),
    "infllmv2_block_score_topk": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _PP, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_sparse_attn_prefill": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _P, _PP, _P, _P, _P,
                                      _SZ, _P], _I),
    "infllmv2_sparse_attn_decode": ([_P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _P, _P, _PP, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_sparse_attn_decode_noalloc": ([_P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _P, _P, _PP, _P, _P, _P], _I),
    "infllmv2_sparse_decode_step": ([_P, _I, _I, _I, _I, _P, _I, _P, _P, _I, _P, _I, _PP, _P, _P, _P, _P, _P], _I),
    "infllmv2_sparse_decode_step_pool": ([_P, _I, _I, _I, _I, _P, _I, _P, _P, _I, _P, _I, _PP, _P, _P, _P, _P, _P], _I),
    "infllmv2_sparse_attn_tree_verify": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _P, _P, _P, _P, _P, _PP, _P,
                                          _P, _P, _SZ, _P], _I),
    "infllmv2_dense_attn_prefill": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _I, _F, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_dense_attn_decode": ([_P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _F, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_backward_workspace_size": ([_PP, _I, _I, _I, _I, _I, _I], _SZ),
    "infllmv2_sparse_attn_backward": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _P, _PP, _P, _P, _P,
                                       _P, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_window_attn_decode": ([_P, _I, _I, _I, _I, _P, _P, _I, _P, _I, _I, _F, _P, _P, _P, _SZ, _P], _I),
    "infllmv2_kv_append_paged": ([_P, _P, _I, _I, _I, _P, _P, _P, _I, _P, _I, _P], _I),
    "infllmv2_kernel_pool_paged": ([_P, _I, _P, _I, _I, _I, _I, _P, _P, _I, _PP, _P, _I, _P], _I),
    "infllmv2_sparse_decode_step_paged": ([_P, _I, _I, _I, _I, _P, _I, _P, _P, _I, _P, _I, _P, _I, _PP, _P, _P, _P,
                                           _P, _P], _I),
    "infllmv2_sparse_attn_prefill_paged": ([_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _P, _P, _I, _P, _P, _PP,
                                            _P, _P, _P], _I),
    "infllmv2_sparse_prefill_varlen": ([_P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _I, _I, _I, _PP, _P, _I, _P, _P,
                                        _P, _P, _P, _SZ, _P], _I),
}

EXPORTED = tuple(_SIGS)


def load(path: str = LIB_PATH):
    """Load libinfllmv2.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} not found: build it with `python -m trainable_block_sparse_v2_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, dtype, name, ndim=None, numel=None, shape=None):
    """Type, dtype, contiguity and size of one argument.  The library reads and writes every buffer by the
    sizes it is given, so a buffer smaller than its layout needs would be accessed out of bounds on the
    device: each wrapper checks every tensor's element count (or exact shape) against the sizes it passes.
    The device is checked last, for all arguments at once (_devices)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()} (shape {tuple(t.shape)})")
    return t


def _opt(t, dtype, name, numel):
    """An optional argument (None, or as _need)."""
    return None if t is None else _need(t, dtype, name, numel=numel)


def _devices(fn, *ts):
    """Every tensor argument on one CUDA device."""
    ts = [t for t in ts if isinstance(t, torch.Tensor)]  # None, or a raw device address given as an int
    if not all(t.is_cuda for t in ts):
        raise ValueError(f"{fn}: every tensor argument must be a CUDA tensor")
    if len({t.device for t in ts}) > 1:
        raise ValueError(f"{fn}: tensor arguments are on different devices")


def _int32(t, name, numel):
    """An int32 device array of numel entries (lengths, contexts, positions)."""
    return _need(t, torch.int32, name, numel=numel)


def _qkv(q, k, v, q_ndim=None):
    """q [B, T, Hq, d] (or, for decode, [B, Hq, d] / [B, 1, Hq, d]); k and v [B, Lcap, Hkv, d] of one shape.
    Returns (B, T, Hq, d, Lcap, Hkv)."""
    _need(q, torch.bfloat16, "q", q_ndim)
    if q_ndim is None:  # decode: one query per sequence
        if q.dim() < 3:
            raise ValueError(f"q: expected [B, Hq, d] or [B, 1, Hq, d], got {tuple(q.shape)}")
        B, T, Hq, d = q.shape[0], 1, q.shape[-2], q.shape[-1]
        _need(q, torch.bfloat16, "q", numel=B * Hq * d)
    else:
        B, T, Hq, d = q.shape
    _need(k, torch.bfloat16, "k", 4)
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError(f"k: expected shape ({B}, Lcap, Hkv, {d}), got {tuple(k.shape)}")
    _need(v, torch.bfloat16, "v", shape=tuple(k.shape))
    return B, T, Hq, d, k.shape[1], k.shape[2]


def _checking() -> bool:
    """INFLLMV2_CHECK=1: check the device-side inputs (contexts, block lists) on the host before each call
    (checks.py); off by default, since it copies them to the host and synchronises."""
    return os.environ.get("INFLLMV2_CHECK", "") == "1"


def _check_rows(what, B, T, q_ctx, ctx_lens, same_ctx, lcap, max_ctx, idx=None, cnt=None, params=None):
    from . import checks
    ctx = checks.query_contexts(B, T, q_ctx, ctx_lens, same_ctx)
    checks.check_contexts(ctx, lcap, int(max_ctx), what)
    if idx is not None:
        checks.check_block_lists(idx, cnt, ctx, params.kmax, params.dense_len, params.block_size, what)


def _check(fn, status):
    if status != 0:
        msg = load().infllmv2_status_string(status).decode()
        raise Infllmv2Error(fn, status, msg)


def infllmv2_version() -> int:
    return load().infllmv2_version()


def infllmv2_device_status() -> int:
    """0 when no bounded device-side wait ran out since the last call (reading clears the record)."""
    return int(load().infllmv2_device_status())


def infllmv2_status_string(status: int) -> str:
    return load().infllmv2_status_string(status).decode()


def infllmv2_workspace_size(params: Params, batch, max_q, max_ctx, hq, hkv, head_dim) -> int:
    cp = params.c()
    return int(load().infllmv2_workspace_size(ctypes.byref(cp), batch, max_q, max_ctx, hq, hkv, head_dim))


def infllmv2_kernel_pool(k, old_lens, new_lens, max_new_keys, params: Params, kern, stream=None):
    _need(k, torch.bfloat16, "k", 4)
    B, Lcap, Hkv, d = k.shape
    _need(kern, torch.bfloat16, "kern", 4)
    if (kern.shape[0], kern.shape[1], kern.shape[3]) != (B, Hkv, d):
        raise ValueError(f"kern: expected shape ({B}, {Hkv}, nk_cap, {d}), got {tuple(kern.shape)}")
    _int32(old_lens, "old_lens", B)
    _int32(new_lens, "new_lens", B)
    _devices("infllmv2_kernel_pool", k, kern, old_lens, new_lens)
    if _checking():
        from . import checks
        checks.check_pool_lengths(old_lens, new_lens, Lcap, int(max_new_keys), kern.shape[2], params.kernel_size,
                                  params.kernel_stride, "infllmv2_kernel_pool")
    cp = params.c()
    st = load().infllmv2_kernel_pool(_ptr(k), B, Lcap, Hkv, d, _ptr(old_lens), _ptr(new_lens), int(max_new_keys),
                                     ctypes.byref(cp), _ptr(kern), kern.shape[2], _stream(stream))
    _check("infllmv2_kernel_pool", st)


def infllmv2_kernel_pool_backward(dkern, lens, max_len, params: Params, dk, accumulate=False, stream=None):
    """dk[b, i, g] (+)= sum over the complete windows j that contain key i of dkern[b, g, j] / 32, for
    i < lens[b] (the gradient of the semantic kernels with respect to K)"""
    _need(dkern, torch.float32, "dkern", 4)
    B, Hkv, nk_cap, d = dkern.shape
    _need(dk, torch.float32, "dk", 4)
    if (dk.shape[0], dk.shape[2], dk.shape[3]) != (B, Hkv, d):
        raise ValueError(f"dk: expected shape ({B}, Lcap, {Hkv}, {d}), got {tuple(dk.shape)}")
    _int32(lens, "lens", B)
    _devices("infllmv2_kernel_pool_backward", dkern, dk, lens)
    cp = params.c()
    st = load().infllmv2_kernel_pool_backward(_ptr(dkern), B, dk.shape[1], Hkv, d, _ptr(lens), int(max_len),
                                              ctypes.byref(cp), nk_cap, _ptr(dk), 1 if accumulate else 0,
                                              _stream(stream))
    _check("infllmv2_kernel_pool_backward", st)


def infllmv2_kv_append(k_new, v_new, pos, k_cache, v_cache, stream=None):
    """k_cache[b, pos[b]] = k_new[b] and v_cache[b, pos[b]] = v_new[b] (cache maintenance of a decode step)"""
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    B, Lcap, Hkv, d = k_cache.shape
    _need(v_cache, torch.bfloat16, "v_cache", shape=(B, Lcap, Hkv, d))
    _need(k_new, torch.bfloat16, "k_new", shape=(B, Hkv, d))
    _need(v_new, torch.bfloat16, "v_new", shape=(B, Hkv, d))
    _int32(pos, "pos", B)
    _devices("infllmv2_kv_append", k_new, v_new, pos, k_cache, v_cache)
    st = load().infllmv2_kv_append(_ptr(k_new), _ptr(v_new), B, Hkv, d, _ptr(pos), _ptr(k_cache), _ptr(v_cache), Lcap,
                                   _stream(stream))
    _check("infllmv2_kv_append", st)


def infllmv2_block_score_topk(q, q_ctx, ctx_lens, max_ctx, kern, params: Params, idx, cnt, ws, stream=None):
    _need(q, torch.bfloat16, "q", 4)
    B, T, Hq, d = q.shape
    _need(kern, torch.bfloat16, "kern", 4)
    Hkv = kern.shape[1]
    if (kern.shape[0], kern.shape[3]) != (B, d):
        raise ValueError(f"kern: expected shape ({B}, Hkv, nk_cap, {d}), got {tuple(kern.shape)}")
    _need(idx, torch.int32, "idx", numel=B * T * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=B * T * Hkv)
    _opt(q_ctx, torch.int32, "q_ctx", B * T)
    _opt(ctx_lens, torch.int32, "ctx_lens", B)
    _devices("infllmv2_block_score_topk", q, kern, idx, cnt, q_ctx, ctx_lens, ws)
    if _checking():
        _check_rows("infllmv2_block_score_topk", B, T, q_ctx, ctx_lens, False, int(max_ctx), max_ctx)
    cp = params.c()
    st = load().infllmv2_block_score_topk(_ptr(q), B, T, Hq, Hkv, d, _ptr(q_ctx), _ptr(ctx_lens), int(max_ctx),
                                          _ptr(kern), kern.shape[2], ctypes.byref(cp), _ptr(idx), _ptr(cnt),
                                          _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                          _stream(stream))
    _check("infllmv2_block_score_topk", st)


def infllmv2_sparse_attn_prefill(q, k, v, q_ctx, ctx_lens, max_ctx, idx, cnt, params: Params, out, lse=None,
                                 ws=None, stream=None):
    B, T, Hq, d, Lcap, Hkv = _qkv(q, k, v, 4)
    _need(out, torch.bfloat16, "out", numel=B * T * Hq * d)
    _need(idx, torch.int32, "idx", numel=B * T * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=B * T * Hkv)
    _opt(lse, torch.float32, "lse", B * T * Hq)
    _opt(q_ctx, torch.int32, "q_ctx", B * T)
    _opt(ctx_lens, torch.int32, "ctx_lens", B)
    _devices("infllmv2_sparse_attn_prefill", q, k, v, out, idx, cnt, lse, q_ctx, ctx_lens, ws)
    if _checking():
        _check_rows("infllmv2_sparse_attn_prefill", B, T, q_ctx, ctx_lens, False, Lcap, max_ctx, idx, cnt, params)
    cp = params.c()
    st = load().infllmv2_sparse_attn_prefill(_ptr(q), B, T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(q_ctx),
                                             _ptr(ctx_lens), int(max_ctx), _ptr(idx), _ptr(cnt), ctypes.byref(cp),
                                             _ptr(out), _ptr(lse), _ptr(ws),
                                             0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("infllmv2_sparse_attn_prefill", st)


def _decode_args(fn, q, k, v, ctx_lens, out, lse, idx=None, cnt=None, params=None, kern=None, ws=None):
    """The arguments of the decode entry points: q [B, (1,) Hq, d], k / v [B, Lcap, Hkv, d], ctx_lens [B],
    out like q, lse [B, (1,) Hq], idx [B, (1,) Hkv, kmax], cnt [B, (1,) Hkv], kern [B, Hkv, nk_cap, d]."""
    B, _, Hq, d, Lcap, Hkv = _qkv(q, k, v)
    _need(out, torch.bfloat16, "out", numel=B * Hq * d)
    _int32(ctx_lens, "ctx_lens", B)
    _opt(lse, torch.float32, "lse", B * Hq)
    if idx is not None or cnt is not None:
        _need(idx, torch.int32, "idx", numel=B * Hkv * params.kmax)
        _need(cnt, torch.int32, "cnt", numel=B * Hkv)
    if kern is not None:
        _need(kern, torch.bfloat16, "kern", 4)
        if (kern.shape[0], kern.shape[1], kern.shape[3]) != (B, Hkv, d):
            raise ValueError(f"kern: expected shape ({B}, {Hkv}, nk_cap, {d}), got {tuple(kern.shape)}")
    _devices(fn, q, k, v, ctx_lens, out, lse, idx, cnt, kern, ws)
    return B, Hq, d, Lcap, Hkv


def infllmv2_sparse_attn_decode(q, k, v, ctx_lens, max_ctx, idx, cnt, params: Params, out, lse, ws, stream=None):
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_sparse_attn_decode", q, k, v, ctx_lens, out, lse, idx, cnt, params,
                                       ws=ws)
    if _checking():
        _check_rows("infllmv2_sparse_attn_decode", B, 1, None, ctx_lens, True, Lcap, max_ctx,
                    idx.reshape(B, 1, Hkv, -1), cnt.reshape(B, 1, Hkv), params)
    cp = params.c()
    st = load().infllmv2_sparse_attn_decode(_ptr(q), B, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(ctx_lens),
                                            int(max_ctx), _ptr(idx), _ptr(cnt), ctypes.byref(cp), _ptr(out), _ptr(lse),
                                            _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                            _stream(stream))
    _check("infllmv2_sparse_attn_decode", st)


def infllmv2_sparse_decode_step(q, kern, k, v, ctx_lens, max_ctx, params: Params, idx, cnt, out, lse=None,
                                stream=None):
    """Scoring, top-k and sparse attention of one decode step in one launch (no workspace)."""
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_sparse_decode_step", q, k, v, ctx_lens, out, lse, idx, cnt, params,
                                       kern=kern)
    if _checking():
        _check_rows("infllmv2_sparse_decode_step", B, 1, None, ctx_lens, True, Lcap, max_ctx)
    cp = params.c()
    st = load().infllmv2_sparse_decode_step(_ptr(q), B, Hq, Hkv, d, _ptr(kern), kern.shape[2], _ptr(k), _ptr(v), Lcap,
                                            _ptr(ctx_lens), int(max_ctx), ctypes.byref(cp), _ptr(idx), _ptr(cnt),
                                            _ptr(out), _ptr(lse), _stream(stream))
    _check("infllmv2_sparse_decode_step", st)


def infllmv2_sparse_decode_step_pool(q, kern, k, v, ctx_lens, max_ctx, params: Params, idx, cnt, out, lse=None,
                                     stream=None):
    """The kernel pool of each sequence's last key, then scoring, top-k and sparse attention, in one launch
    (infllmv2_kernel_pool of old = n - 1, new = n followed by infllmv2_sparse_decode_step)"""
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_sparse_decode_step_pool", q, k, v, ctx_lens, out, lse, idx, cnt,
                                       params, kern=kern)
    if _checking():
        _check_rows("infllmv2_sparse_decode_step_pool", B, 1, None, ctx_lens, True, Lcap, max_ctx)
    cp = params.c()
    st = load().infllmv2_sparse_decode_step_pool(_ptr(q), B, Hq, Hkv, d, _ptr(kern), kern.shape[2], _ptr(k), _ptr(v),
                                                 Lcap, _ptr(ctx_lens), int(max_ctx), ctypes.byref(cp), _ptr(idx),
                                                 _ptr(cnt), _ptr(out), _ptr(lse), _stream(stream))
    _check("infllmv2_sparse_decode_step_pool", st)


def infllmv2_sparse_attn_decode_noalloc(q, k, v, ctx_lens, max_ctx, idx, cnt, params: Params, out, lse=None,
                                        stream=None):
    """infllmv2_sparse_attn_decode without a workspace: the library keeps the scratch in its own static
    device array (4 MiB per GPU), for callers that cannot allocate device memory when they call."""
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_sparse_attn_decode_noalloc", q, k, v, ctx_lens, out, lse, idx, cnt,
                                       params)
    cp = params.c()
    st = load().infllmv2_sparse_attn_decode_noalloc(_ptr(q), B, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(ctx_lens),
                                                    int(max_ctx), _ptr(idx), _ptr(cnt), ctypes.byref(cp), _ptr(out),
                                                    _ptr(lse), _stream(stream))
    _check("infllmv2_sparse_attn_decode_noalloc", st)


def infllmv2_sparse_attn_tree_verify(q, k, v, prefix_lens, max_ctx, k_draft, v_draft, tree_mask, idx, cnt,
                                     params: Params, out, lse, ws, stream=None):
    B, N, Hq, d, Lcap, Hkv = _qkv(q, k, v, 4)
    _need(k_draft, torch.bfloat16, "k_draft", numel=B * N * Hkv * d)
    _need(v_draft, torch.bfloat16, "v_draft", numel=B * N * Hkv * d)
    _need(tree_mask, None, "tree_mask", numel=B * N)
    if tree_mask.element_size() != 4:
        raise TypeError(f"tree_mask: expected 32-bit words, got {tree_mask.dtype}")
    _need(out, torch.bfloat16, "out", numel=B * N * Hq * d)
    _int32(prefix_lens, "prefix_lens", B)
    _need(idx, torch.int32, "idx", numel=B * N * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=B * N * Hkv)
    _opt(lse, torch.float32, "lse", B * N * Hq)
    _devices("infllmv2_sparse_attn_tree_verify", q, k, v, prefix_lens, k_draft, v_draft, tree_mask, idx, cnt, out, lse,
             ws)
    if _checking():
        _check_rows("infllmv2_sparse_attn_tree_verify", B, N, None, prefix_lens, True, Lcap, max_ctx, idx, cnt,
                    params)
        from . import checks
        checks.check_tree_mask(tree_mask, B, N, "infllmv2_sparse_attn_tree_verify")
    cp = params.c()
    st = load().infllmv2_sparse_attn_tree_verify(_ptr(q), B, N, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(prefix_lens),
                                                 int(max_ctx), _ptr(k_draft), _ptr(v_draft), _ptr(tree_mask), _ptr(idx),
                                                 _ptr(cnt), ctypes.byref(cp), _ptr(out), _ptr(lse), _ptr(ws),
                                                 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("infllmv2_sparse_attn_tree_verify", st)


def infllmv2_dense_attn_prefill(q, k, v, q_ctx, ctx_lens, max_ctx, softmax_scale, out, lse=None, ws=None,
                                stream=None):
    B, T, Hq, d, Lcap, Hkv = _qkv(q, k, v, 4)
    _need(out, torch.bfloat16, "out", numel=B * T * Hq * d)
    _opt(lse, torch.float32, "lse", B * T * Hq)
    _opt(q_ctx, torch.int32, "q_ctx", B * T)
    _opt(ctx_lens, torch.int32, "ctx_lens", B)
    _devices("infllmv2_dense_attn_prefill", q, k, v, out, lse, q_ctx, ctx_lens, ws)
    if _checking():
        _check_rows("infllmv2_dense_attn_prefill", B, T, q_ctx, ctx_lens, False, Lcap, max_ctx)
    st = load().infllmv2_dense_attn_prefill(_ptr(q), B, T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(q_ctx),
                                            _ptr(ctx_lens), int(max_ctx), float(softmax_scale), _ptr(out), _ptr(lse),
                                            _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                            _stream(stream))
    _check("infllmv2_dense_attn_prefill", st)


def infllmv2_dense_attn_decode(q, k, v, ctx_lens, max_ctx, softmax_scale, out, lse, ws, stream=None):
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_dense_attn_decode", q, k, v, ctx_lens, out, lse, ws=ws)
    if _checking():
        _check_rows("infllmv2_dense_attn_decode", B, 1, None, ctx_lens, True, Lcap, max_ctx)
    st = load().infllmv2_dense_attn_decode(_ptr(q), B, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(ctx_lens), int(max_ctx),
                                           float(softmax_scale), _ptr(out), _ptr(lse), _ptr(ws),
                                           0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("infllmv2_dense_attn_decode", st)


def infllmv2_window_attn_decode(q, k, v, ctx_lens, max_ctx, window, softmax_scale, out, lse, ws, stream=None):
    B, Hq, d, Lcap, Hkv = _decode_args("infllmv2_window_attn_decode", q, k, v, ctx_lens, out, lse, ws=ws)
    if _checking():
        _check_rows("infllmv2_window_attn_decode", B, 1, None, ctx_lens, True, Lcap, max_ctx)
    st = load().infllmv2_window_attn_decode(_ptr(q), B, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(ctx_lens),
                                            int(max_ctx), int(window), float(softmax_scale), _ptr(out), _ptr(lse),
                                            _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                            _stream(stream))
    _check("infllmv2_window_attn_decode", st)


# ---- paged key/value cache: pools [num_pages * 64, Hkv, d], page_table [B, max_pages] int32 ----
def _pages(fn, k_pages, v_pages, page_table, B):
    """The page pools (one shape, [num_pages * 64, Hkv, d]) and the page table ([B, max_pages]).
    Returns (num_pages, max_pages, Hkv, d)."""
    _need(k_pages, torch.bfloat16, "k_pages", 3)
    if k_pages.shape[0] % 64 != 0 or k_pages.shape[0] == 0:
        raise ValueError(f"{fn}: k_pages: expected [num_pages * 64, Hkv, d], got {tuple(k_pages.shape)}")
    if v_pages is not None:
        _need(v_pages, torch.bfloat16, "v_pages", shape=tuple(k_pages.shape))
    _need(page_table, torch.int32, "page_table", 2)
    if page_table.shape[0] != B:
        raise ValueError(f"{fn}: page_table: expected [{B}, max_pages], got {tuple(page_table.shape)}")
    return k_pages.shape[0] // 64, page_table.shape[1], k_pages.shape[1], k_pages.shape[2]


def _check_pages(what, page_table, lens, num_pages):
    from . import checks
    checks.check_page_table(page_table, lens, num_pages, what)


def infllmv2_kv_append_paged(k_new, v_new, pos, k_pages, v_pages, page_table, stream=None):
    """The row of position pos[b] through the page table: k_pages[page * 64 + pos % 64] = k_new[b] (v likewise)"""
    _need(k_new, torch.bfloat16, "k_new", 3)
    B = k_new.shape[0]
    num_pages, max_pages, Hkv, d = _pages("infllmv2_kv_append_paged", k_pages, v_pages, page_table, B)
    _need(k_new, torch.bfloat16, "k_new", shape=(B, Hkv, d))
    _need(v_new, torch.bfloat16, "v_new", shape=(B, Hkv, d))
    _int32(pos, "pos", B)
    _devices("infllmv2_kv_append_paged", k_new, v_new, pos, k_pages, v_pages, page_table)
    if _checking():
        _check_pages("infllmv2_kv_append_paged", page_table, pos.detach().cpu().numpy().astype("int64") + 1,
                     num_pages)
    st = load().infllmv2_kv_append_paged(_ptr(k_new), _ptr(v_new), B, Hkv, d, _ptr(pos), _ptr(k_pages), _ptr(v_pages),
                                         num_pages, _ptr(page_table), max_pages, _stream(stream))
    _check("infllmv2_kv_append_paged", st)


def infllmv2_kernel_pool_paged(k_pages, page_table, old_lens, new_lens, max_new_keys, params: Params, kern,
                               stream=None):
    """infllmv2_kernel_pool over a paged key cache"""
    B = page_table.shape[0] if isinstance(page_table, torch.Tensor) and page_table.dim() == 2 else -1
    num_pages, max_pages, Hkv, d = _pages("infllmv2_kernel_pool_paged", k_pages, None, page_table, B)
    _need(kern, torch.bfloat16, "kern", 4)
    if (kern.shape[0], kern.shape[1], kern.shape[3]) != (B, Hkv, d):
        raise ValueError(f"kern: expected shape ({B}, {Hkv}, nk_cap, {d}), got {tuple(kern.shape)}")
    _int32(old_lens, "old_lens", B)
    _int32(new_lens, "new_lens", B)
    _devices("infllmv2_kernel_pool_paged", k_pages, page_table, kern, old_lens, new_lens)
    if _checking():
        from . import checks
        checks.check_pool_lengths(old_lens, new_lens, max_pages * 64, int(max_new_keys), kern.shape[2],
                                  params.kernel_size, params.kernel_stride, "infllmv2_kernel_pool_paged")
        _check_pages("infllmv2_kernel_pool_paged", page_table, new_lens, num_pages)
    cp = params.c()
    st = load().infllmv2_kernel_pool_paged(_ptr(k_pages), num_pages, _ptr(page_table), max_pages, B, Hkv, d,
                                           _ptr(old_lens), _ptr(new_lens), int(max_new_keys), ctypes.byref(cp),
                                           _ptr(kern), kern.shape[2], _stream(stream))
    _check("infllmv2_kernel_pool_paged", st)


def infllmv2_sparse_decode_step_paged(q, kern, k_pages, v_pages, page_table, ctx_lens, max_ctx, params: Params, idx,
                                      cnt, out, lse=None, stream=None):
    """infllmv2_sparse_decode_step over a paged key/value cache"""
    _need(q, torch.bfloat16, "q")
    if q.dim() < 3:
        raise ValueError(f"q: expected [B, Hq, d] or [B, 1, Hq, d], got {tuple(q.shape)}")
    B, Hq = q.shape[0], q.shape[-2]
    num_pages, max_pages, Hkv, d = _pages("infllmv2_sparse_decode_step_paged", k_pages, v_pages, page_table, B)
    _need(q, torch.bfloat16, "q", numel=B * Hq * d)
    _need(out, torch.bfloat16, "out", numel=B * Hq * d)
    _int32(ctx_lens, "ctx_lens", B)
    _opt(lse, torch.float32, "lse", B * Hq)
    _need(idx, torch.int32, "idx", numel=B * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=B * Hkv)
    _need(kern, torch.bfloat16, "kern", 4)
    if (kern.shape[0], kern.shape[1], kern.shape[3]) != (B, Hkv, d):
        raise ValueError(f"kern: expected shape ({B}, {Hkv}, nk_cap, {d}), got {tuple(kern.shape)}")
    _devices("infllmv2_sparse_decode_step_paged", q, kern, k_pages, v_pages, page_table, ctx_lens, idx, cnt, out, lse)
    if _checking():
        _check_rows("infllmv2_sparse_decode_step_paged", B, 1, None, ctx_lens, True, max_pages * 64, max_ctx)
        _check_pages("infllmv2_sparse_decode_step_paged", page_table, ctx_lens, num_pages)
    cp = params.c()
    st = load().infllmv2_sparse_decode_step_paged(_ptr(q), B, Hq, Hkv, d, _ptr(kern), kern.shape[2], _ptr(k_pages),
                                                  _ptr(v_pages), num_pages, _ptr(page_table), max_pages,
                                                  _ptr(ctx_lens), int(max_ctx), ctypes.byref(cp), _ptr(idx),
                                                  _ptr(cnt), _ptr(out), _ptr(lse), _stream(stream))
    _check("infllmv2_sparse_decode_step_paged", st)


def infllmv2_sparse_attn_prefill_paged(q, k_pages, v_pages, page_table, q_ctx, ctx_lens, max_ctx, idx, cnt,
                                       params: Params, out, lse=None, stream=None):
    """infllmv2_sparse_attn_prefill over a paged key/value cache (q [B, T, Hq, d]: the last T positions of each
    context unless q_ctx gives every query's context)"""
    _need(q, torch.bfloat16, "q", 4)
    B, T, Hq = q.shape[0], q.shape[1], q.shape[2]
    num_pages, max_pages, Hkv, d = _pages("infllmv2_sparse_attn_prefill_paged", k_pages, v_pages, page_table, B)
    _need(q, torch.bfloat16, "q", shape=(B, T, Hq, d))
    _need(out, torch.bfloat16, "out", numel=B * T * Hq * d)
    _need(idx, torch.int32, "idx", numel=B * T * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=B * T * Hkv)
    _opt(lse, torch.float32, "lse", B * T * Hq)
    _opt(q_ctx, torch.int32, "q_ctx", B * T)
    _opt(ctx_lens, torch.int32, "ctx_lens", B)
    _devices("infllmv2_sparse_attn_prefill_paged", q, k_pages, v_pages, page_table, out, idx, cnt, lse, q_ctx,
             ctx_lens)
    if _checking():
        from . import checks
        _check_rows("infllmv2_sparse_attn_prefill_paged", B, T, q_ctx, ctx_lens, False, max_pages * 64, max_ctx, idx,
                    cnt, params)
        ctx = checks.query_contexts(B, T, q_ctx, ctx_lens, False)
        _check_pages("infllmv2_sparse_attn_prefill_paged", page_table, ctx.max(axis=1), num_pages)
    cp = params.c()
    st = load().infllmv2_sparse_attn_prefill_paged(_ptr(q), B, T, Hq, Hkv, d, _ptr(k_pages), _ptr(v_pages),
                                                   num_pages, _ptr(page_table), max_pages, _ptr(q_ctx),
                                                   _ptr(ctx_lens), int(max_ctx), _ptr(idx), _ptr(cnt),
                                                   ctypes.byref(cp), _ptr(out), _ptr(lse), _stream(stream))
    _check("infllmv2_sparse_attn_prefill_paged", st)


# ---- packed variable-length prefill: q [total_q, Hq, d], k / v [total_k, Hkv, d], cu_seqlens [B + 1] ----
def infllmv2_sparse_prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, params: Params,
                                   kern, idx, cnt, out, lse=None, ws=None, stream=None):
    """Kernel pool, scoring + top-k and sparse attention of a packed batch (three launches for the batch)"""
    _need(q, torch.bfloat16, "q", 3)
    _need(k, torch.bfloat16, "k", 3)
    _need(v, torch.bfloat16, "v", shape=tuple(k.shape))
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if k.shape[2] != d:
        raise ValueError(f"k: head_dim {k.shape[2]} differs from q's {d}")
    _need(cu_seqlens_q, torch.int32, "cu_seqlens_q", 1)
    B = cu_seqlens_q.numel() - 1
    _int32(cu_seqlens_k, "cu_seqlens_k", B + 1)
    _need(out, torch.bfloat16, "out", shape=(total_q, Hq, d))
    _need(idx, torch.int32, "idx", numel=total_q * Hkv * params.kmax)
    _need(cnt, torch.int32, "cnt", numel=total_q * Hkv)
    _opt(lse, torch.float32, "lse", total_q * Hq)
    _need(kern, torch.bfloat16, "kern", 4)
    if (kern.shape[0], kern.shape[1], kern.shape[3]) != (B, Hkv, d):
        raise ValueError(f"kern: expected shape ({B}, {Hkv}, nk_cap, {d}), got {tuple(kern.shape)}")
    _devices("infllmv2_sparse_prefill_varlen", q, k, v, cu_seqlens_q, cu_seqlens_k, kern, idx, cnt, out, lse, ws)
    if _checking():
        from . import checks
        checks.check_cu_seqlens(cu_seqlens_q, cu_seqlens_k, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k),
                                "infllmv2_sparse_prefill_varlen")
    cp = params.c()
    st = load().infllmv2_sparse_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, d, _ptr(cu_seqlens_q),
                                               _ptr(cu_seqlens_k), total_q, total_k, int(max_seqlen_q),
                                               int(max_seqlen_k), ctypes.byref(cp), _ptr(kern), kern.shape[2],
                                               _ptr(idx), _ptr(cnt), _ptr(out), _ptr(lse), _ptr(ws),
                                               0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("infllmv2_sparse_prefill_varlen", st)


def infllmv2_backward_workspace_size(params: Params, batch, max_q, max_ctx, hq, hkv, head_dim) -> int:
    cp = params.c()
    return int(load().infllmv2_backward_workspace_size(ctypes.byref(cp), batch, max_q, max_ctx, hq, hkv, head_dim))


def infllmv2_sparse_attn_backward(q, k, v, q_ctx, ctx_lens, max_ctx, idx, cnt, params: Params, out, lse, dout,
                                  dq, dk, dv, ws, stream=None):
    """Gradients (dq, dk, dv; fp32, overwritten) of the sparse attention for a fixed selection; idx and cnt
    both None means dense attention over [0, n)."""
    B, T, Hq, d, Lcap, Hkv = _qkv(q, k, v, 4)
    _need(out, torch.bfloat16, "out", shape=tuple(q.shape))
    _need(dout, torch.bfloat16, "dout", shape=tuple(q.shape))
    _need(dq, torch.float32, "dq", shape=tuple(q.shape))
    _need(dk, torch.float32, "dk", shape=tuple(k.shape))
    _need(dv, torch.float32, "dv", shape=tuple(k.shape))
    _need(lse, torch.float32, "lse", numel=B * T * Hq)
    if (idx is None) != (cnt is None):
        raise ValueError("idx and cnt: give both (sparse) or neither (dense)")
    if idx is not None:
        _need(idx, torch.int32, "idx", numel=B * T * Hkv * params.kmax)
        _need(cnt, torch.int32, "cnt", numel=B * T * Hkv)
    _opt(q_ctx, torch.int32, "q_ctx", B * T)
    _opt(ctx_lens, torch.int32, "ctx_lens", B)
    _devices("infllmv2_sparse_attn_backward", q, k, v, out, dout, dq, dk, dv, lse, idx, cnt, q_ctx, ctx_lens, ws)
    if _checking():
        _check_rows("infllmv2_sparse_attn_backward", B, T, q_ctx, ctx_lens, False, Lcap, max_ctx, idx, cnt, params)
    cp = params.c()
    st = load().infllmv2_sparse_attn_backward(_ptr(q), B, T, Hq, Hkv, d, _ptr(k), _ptr(v), Lcap, _ptr(q_ctx),
                                              _ptr(ctx_lens), int(max_ctx), _ptr(idx), _ptr(cnt), ctypes.byref(cp),
                                              _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                              _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                              _stream(stream))
    _check("infllmv2_sparse_attn_backward", st)


def backward_workspace(params: Params, batch, max_q, max_ctx, hq, hkv, head_dim, device="cuda"):
    """Allocate (with torch) a workspace of infllmv2_backward_workspace_size bytes, 256-byte aligned."""
    n = infllmv2_backward_workspace_size(params, batch, max_q, max_ctx, hq, hkv, head_dim)
    if n == 0:
        raise Infllmv2Error("infllmv2_backward_workspace_size", 1, "invalid sizes")
    return torch.empty(math.ceil(n / 256) * 256, dtype=torch.uint8, device=device)


def num_kernels(n: int, kernel_size: int = 32, kernel_stride: int = 16) -> int:
    return 0 if n < kernel_size else (n - kernel_size) // kernel_stride + 1


def workspace(params: Params, batch, max_q, max_ctx, hq, hkv, head_dim, device="cuda"):
    """Allocate (with torch) a zero-filled workspace of infllmv2_workspace_size bytes, 256-byte aligned."""
    n = infllmv2_workspace_size(params, batch, max_q, max_ctx, hq, hkv, head_dim)
    if n == 0:
        raise Infllmv2Error("infllmv2_workspace_size", 1, "invalid sizes")
    return torch.zeros(math.ceil(n / 256) * 256, dtype=torch.uint8, device=device)
