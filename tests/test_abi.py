"""The C-ABI library: it loads, exports every symbol include/infllmv2.h declares, and rejects bad
arguments on the host with the documented status before launching anything (no GPU needed: every call
here fails validation, so no CUDA work is enqueued)."""
import ctypes
import os
import re

import pytest

from trainable_block_sparse_v2_b200 import binding
from trainable_block_sparse_v2_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "infllmv2.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(infllmv2_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["infllmv2_kernel_pool", "infllmv2_block_score_topk", "infllmv2_sparse_attn_prefill",
              "infllmv2_sparse_attn_decode", "infllmv2_sparse_attn_tree_verify", "infllmv2_dense_attn_prefill",
              "infllmv2_dense_attn_decode", "infllmv2_workspace_size", "infllmv2_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(binding.EXPORTED) >= set(declared_functions())


def test_status_strings_and_version(lib):
    assert binding.infllmv2_status_string(0) == "ok"
    assert "workspace" in binding.infllmv2_status_string(3)
    assert binding.infllmv2_version() >= 100


def test_workspace_size_host_only(lib):
    p = binding.Params(topk=64, dense_len=8192)
    n = binding.infllmv2_workspace_size(p, 4, 1, 131072 + 256, 32, 2, 128)
    assert n > 0 and n % 256 == 0
    assert binding.infllmv2_workspace_size(p, 4, 1, 131072, 32, 2, 128) <= n
    assert binding.infllmv2_workspace_size(p, 4, 1, 131072, 32, 3, 128) == 0      # Hq % Hkv != 0
    assert binding.infllmv2_workspace_size(p, 4, 1, 131072, 32, 2, 96) == 0       # unsupported d
    assert binding.infllmv2_workspace_size(p, 4, 1, 0, 32, 2, 128) == 0           # empty context
    bad = binding.Params(block_size=32)
    assert binding.infllmv2_workspace_size(bad, 1, 1, 1000, 32, 2, 128) == 0


# fake device pointers: aligned, never dereferenced because validation fails first
A16 = 0x10000
A16B = 0x20000
A4 = 0x30000
WS = 0x40000


def _score(lib, p, **kw):
    args = dict(q=A16, batch=1, num_q=1, hq=32, hkv=2, d=128, q_ctx=None, ctx_lens=A4, max_ctx=4096, kern=A16B,
                nk_cap=255, idx=A4, cnt=A4, ws=WS, ws_bytes=1 << 30)
    args.update(kw)
    cp = p.c()
    return lib.infllmv2_block_score_topk(args["q"], args["batch"], args["num_q"], args["hq"], args["hkv"], args["d"],
                                         args["q_ctx"], args["ctx_lens"], args["max_ctx"], args["kern"],
                                         args["nk_cap"], ctypes.byref(cp), args["idx"], args["cnt"], args["ws"],
                                         args["ws_bytes"], None)


def test_block_score_topk_rejects_bad_arguments(lib):
    p = binding.Params(topk=8)
    assert _score(lib, p, q=None) == INVALID
    assert _score(lib, p, q=A16 + 2) == INVALID                  # misaligned
    assert _score(lib, p, hkv=3) == INVALID                      # Hq % Hkv
    assert _score(lib, p, hq=6, hkv=2) == UNSUPPORTED            # group of 3
    assert _score(lib, p, d=96) == UNSUPPORTED
    assert _score(lib, p, q_ctx=None, ctx_lens=None) == INVALID
    assert _score(lib, p, max_ctx=0) == INVALID
    assert _score(lib, p, nk_cap=10) == INVALID                  # kernel cache too small for max_ctx
    assert _score(lib, p, max_ctx=300000, nk_cap=20000) == UNSUPPORTED
    assert _score(lib, p, ws=None) == WORKSPACE                  # few-row path needs workspace
    assert _score(lib, p, ws_bytes=16) == WORKSPACE
    assert _score(lib, p, ws=WS + 16) == WORKSPACE               # workspace not 256-aligned
    assert _score(lib, binding.Params(block_size=128)) == UNSUPPORTED
    assert _score(lib, binding.Params(topk=-1)) == INVALID
    assert _score(lib, binding.Params(membership=2)) == INVALID
    assert _score(lib, binding.Params(topk=0, init_blocks=0, local_blocks=0)) == INVALID
    # counts whose sum would overflow an int are refused before any use
    assert _score(lib, binding.Params(topk=2**31 - 1)) == INVALID
    assert _score(lib, binding.Params(topk=1, init_blocks=2**30, local_blocks=2**30)) == INVALID
    assert binding.infllmv2_workspace_size(binding.Params(topk=2**31 - 1), 1, 1, 4096, 32, 2, 128) == 0
    assert _score(lib, binding.Params(lse_stride=-1)) == INVALID
    assert _score(lib, binding.Params(lse_stride=3)) == UNSUPPORTED
    assert _score(lib, binding.Params(lse_stride=4)) == UNSUPPORTED  # one query per sequence: the scan path


def test_attention_entry_points_reject_bad_arguments(lib):
    p = binding.Params(topk=64, dense_len=8192)
    cp = p.c()
    # decode: lcap smaller than max_ctx
    assert lib.infllmv2_sparse_attn_decode(A16, 1, 32, 2, 128, A16, A16, 1000, A4, 2000, A4, A4, ctypes.byref(cp),
                                           A16, None, WS, 1 << 30, None) == INVALID
    # decode: workspace too small
    assert lib.infllmv2_sparse_attn_decode(A16, 1, 32, 2, 128, A16, A16, 4096, A4, 4096, A4, A4, ctypes.byref(cp),
                                           A16, None, WS, 64, None) == WORKSPACE
    # tree: more than 32 draft nodes
    assert lib.infllmv2_sparse_attn_tree_verify(A16, 1, 33, 32, 2, 128, A16, A16, 4096, A4, 4096, A16, A16, A4, A4,
                                                A4, ctypes.byref(cp), A16, None, WS, 1 << 30, None) == UNSUPPORTED
    # prefill: null v
    assert lib.infllmv2_sparse_attn_prefill(A16, 1, 16, 32, 2, 128, A16, None, 4096, None, A4, 4096, A4, A4,
                                            ctypes.byref(cp), A16, None, None, 0, None) == INVALID
    # dense: NaN scale
    assert lib.infllmv2_dense_attn_prefill(A16, 1, 16, 32, 2, 128, A16, A16, 4096, None, A4, 4096,
                                           ctypes.c_float(float("nan")), A16, None, None, 0, None) == INVALID
    # kernel pool: unsupported window
    bad = binding.Params(kernel_size=16).c()
    assert lib.infllmv2_kernel_pool(A16, 1, 4096, 2, 128, A4, A4, 4096, ctypes.byref(bad), A16, 255, None) == \
        UNSUPPORTED
    assert lib.infllmv2_kernel_pool(A16, 1, 4096, 2, 128, A4, A4, 4096, ctypes.byref(cp), A16, 10, None) == INVALID
    # kernel pool backward: misaligned gradients, max_len past lcap, kernel cache too small, bad mode, d 96
    nk = binding.num_kernels(4096)
    assert lib.infllmv2_kernel_pool_backward(A16 + 4, 1, 4096, 2, 128, A4, 4096, ctypes.byref(cp), nk, A16, 0,
                                             None) == INVALID
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 128, A4, 4097, ctypes.byref(cp), nk + 1, A16, 0,
                                             None) == INVALID
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 128, A4, 4096, ctypes.byref(cp), nk - 1, A16, 0,
                                             None) == INVALID
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 128, A4, 4096, ctypes.byref(cp), nk, A16, 2,
                                             None) == INVALID
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 96, A4, 4096, ctypes.byref(cp), nk, A16, 0,
                                             None) == UNSUPPORTED
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 128, A4, 4096, ctypes.byref(bad), nk, A16, 0,
                                             None) == UNSUPPORTED
    assert lib.infllmv2_kernel_pool_backward(A16, 1, 4096, 2, 128, A4, 0, ctypes.byref(cp), nk, A16, 0, None) == OK
    # window decode: window 0
    assert lib.infllmv2_window_attn_decode(A16, 1, 32, 2, 128, A16, A16, 4096, A4, 4096, 0, ctypes.c_float(0.0),
                                           A16, None, WS, 1 << 30, None) == INVALID
    # kv append: misaligned new rows, null cache, empty capacity
    assert lib.infllmv2_kv_append(A16 + 2, A16, 4, 2, 128, A4, A16, A16, 4096, None) == INVALID
    assert lib.infllmv2_kv_append(A16, A16, 4, 2, 128, A4, None, A16, 4096, None) == INVALID
    assert lib.infllmv2_kv_append(A16, A16, 4, 2, 128, A4, A16, A16, 0, None) == INVALID


def test_backward_rejects_bad_arguments(lib):
    p = binding.Params(topk=64, dense_len=8192)
    cp = p.c()
    need = binding.infllmv2_backward_workspace_size(p, 1, 4096, 4096, 32, 2, 128)
    assert need > 0 and need % 256 == 0
    assert binding.infllmv2_backward_workspace_size(p, 1, 4096, 4096, 32, 2, 96) == 0

    def call(**kw):
        a = dict(q=A16, k=A16, v=A16, lcap=4096, q_ctx=None, ctx=A4, max_ctx=4096, idx=A4, cnt=A4, out=A16,
                 lse=A4, dout=A16, dq=A16, dk=A16, dv=A16, ws=WS, wsb=need)
        a.update(kw)
        return lib.infllmv2_sparse_attn_backward(a["q"], 1, 4096, 32, 2, 128, a["k"], a["v"], a["lcap"], a["q_ctx"],
                                                 a["ctx"], a["max_ctx"], a["idx"], a["cnt"], ctypes.byref(cp),
                                                 a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"], a["ws"],
                                                 a["wsb"], None)

    assert call(lse=None) == INVALID                 # the forward's lse is required
    assert call(dout=A16 + 2) == INVALID             # misaligned gradient input
    assert call(dk=None) == INVALID
    assert call(idx=None) == INVALID                 # idx without cnt (or the reverse)
    assert call(ctx=None) == INVALID                 # neither q_ctx nor ctx_lens
    assert call(max_ctx=5000) == INVALID             # max_ctx past the cache
    assert call(wsb=need - 256) == WORKSPACE
    assert call(ws=WS + 16) == WORKSPACE


def test_noalloc_decode_refuses_what_the_workspace_decode_refuses(lib):
    """The allocation-free decode shares the workspace entry point's argument checks: oversized block counts
    (whose sum would overflow an int), an infinite scale, a context past the cache or past 4096 blocks, and
    too many rows are refused with the same status, before any launch."""

    def both(params, batch=1, hkv=2, lcap=4096, max_ctx=4096, lse=None):
        cp = params.c()
        a = lib.infllmv2_sparse_attn_decode(A16, batch, 16 * hkv, hkv, 128, A16, A16, lcap, A4, max_ctx, A4, A4,
                                            ctypes.byref(cp), A16, lse, WS, 1 << 40, None)
        b = lib.infllmv2_sparse_attn_decode_noalloc(A16, batch, 16 * hkv, hkv, 128, A16, A16, lcap, A4, max_ctx, A4,
                                                    A4, ctypes.byref(cp), A16, lse, None)
        return a, b

    assert both(binding.Params(topk=2**31 - 1)) == (INVALID, INVALID)
    assert both(binding.Params(topk=1, init_blocks=2**30, local_blocks=2**30)) == (INVALID, INVALID)
    assert both(binding.Params(topk=64, softmax_scale=float("inf"))) == (INVALID, INVALID)
    assert both(binding.Params(topk=64, membership=2)) == (INVALID, INVALID)
    assert both(binding.Params(topk=64), lcap=1000, max_ctx=2000) == (INVALID, INVALID)
    assert both(binding.Params(topk=64), lcap=1 << 20, max_ctx=4096 * 64 + 1) == (UNSUPPORTED, UNSUPPORTED)
    assert both(binding.Params(topk=64), lse=A4 + 2) == (INVALID, INVALID)
    assert both(binding.Params(topk=64), batch=1 << 15, hkv=4) == (UNSUPPORTED, UNSUPPORTED)
    assert both(binding.Params(block_size=32)) == (UNSUPPORTED, UNSUPPORTED)


def test_test_wait_limit_is_set_on_the_host(lib):
    """infllmv2_test_set_first_wait_limit only stores the value that later launches take as an argument: it makes
    no CUDA call, returns INFLLMV2_OK, and 0 restores the normal waits (the GPU side is in
    tests/test_gpu_wait_timeout.py)."""
    assert lib.infllmv2_test_set_first_wait_limit(64) == OK
    assert lib.infllmv2_test_set_first_wait_limit(0) == OK
