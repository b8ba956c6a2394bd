"""The binding's argument checks (CPU only): every tensor's dtype and size is checked against the sizes the
wrapper passes to the library, before the device check and before any call, so a buffer too small for its
layout is refused on the host instead of being read or written out of bounds on the device.

Tensors of the documented shapes on the CPU pass every size check and stop at the device check; each
wrongly sized one is refused with its name."""
import pytest
import torch

from trainable_block_sparse_v2_b200 import binding

B, T, HQ, HKV, D, LCAP, NK = 2, 5, 8, 2, 64, 256, 15
P = binding.Params(topk=3, dense_len=0)
KM = P.kmax


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def prefill_args():
    return dict(q=bf(B, T, HQ, D), k=bf(B, LCAP, HKV, D), v=bf(B, LCAP, HKV, D), q_ctx=None, ctx_lens=i32(B),
                max_ctx=LCAP, idx=i32(B, T, HKV, KM), cnt=i32(B, T, HKV), params=P, out=bf(B, T, HQ, D),
                lse=f32(B, T, HQ), ws=None)


def decode_args():
    return dict(q=bf(B, 1, HQ, D), k=bf(B, LCAP, HKV, D), v=bf(B, LCAP, HKV, D), ctx_lens=i32(B), max_ctx=LCAP,
                idx=i32(B, 1, HKV, KM), cnt=i32(B, 1, HKV), params=P, out=bf(B, 1, HQ, D), lse=f32(B, 1, HQ),
                ws=torch.zeros(256, dtype=torch.uint8))


def noalloc_args():
    a = decode_args()
    del a["ws"]
    return a


def step_args():
    a = decode_args()
    del a["ws"]
    a["kern"] = bf(B, HKV, NK, D)
    return a


def tree_args():
    return dict(q=bf(B, T, HQ, D), k=bf(B, LCAP, HKV, D), v=bf(B, LCAP, HKV, D), prefix_lens=i32(B), max_ctx=LCAP,
                k_draft=bf(B, T, HKV, D), v_draft=bf(B, T, HKV, D), tree_mask=i32(B, T), idx=i32(B, T, HKV, KM),
                cnt=i32(B, T, HKV), params=P, out=bf(B, T, HQ, D), lse=f32(B, T, HQ), ws=None)


def backward_args():
    return dict(q=bf(B, T, HQ, D), k=bf(B, LCAP, HKV, D), v=bf(B, LCAP, HKV, D), q_ctx=None, ctx_lens=i32(B),
                max_ctx=LCAP, idx=i32(B, T, HKV, KM), cnt=i32(B, T, HKV), params=P, out=bf(B, T, HQ, D),
                lse=f32(B, T, HQ), dout=bf(B, T, HQ, D), dq=f32(B, T, HQ, D), dk=f32(B, LCAP, HKV, D),
                dv=f32(B, LCAP, HKV, D), ws=None)


def score_args():
    return dict(q=bf(B, T, HQ, D), q_ctx=i32(B, T), ctx_lens=None, max_ctx=LCAP, kern=bf(B, HKV, NK, D), params=P,
                idx=i32(B, T, HKV, KM), cnt=i32(B, T, HKV), ws=None)


def pool_args():
    return dict(k=bf(B, LCAP, HKV, D), old_lens=i32(B), new_lens=i32(B), max_new_keys=LCAP, params=P,
                kern=bf(B, HKV, NK, D))


def append_args():
    return dict(k_new=bf(B, HKV, D), v_new=bf(B, HKV, D), pos=i32(B), k_cache=bf(B, LCAP, HKV, D),
                v_cache=bf(B, LCAP, HKV, D))


def dense_prefill_args():
    a = prefill_args()
    for n in ("idx", "cnt", "params"):
        del a[n]
    a["softmax_scale"] = 0.0
    return a


def dense_decode_args():
    a = decode_args()
    for n in ("idx", "cnt", "params"):
        del a[n]
    a["softmax_scale"] = 0.0
    return a


def window_args():
    a = dense_decode_args()
    a["window"] = 64
    return a


# (wrapper, argument builder, [(argument, wrong value)])
CASES = [
    (binding.infllmv2_kernel_pool, pool_args,
     [("kern", bf(B, HKV + 1, NK, D)), ("new_lens", i32(B + 1)), ("old_lens", torch.zeros(B, dtype=torch.int64))]),
    (binding.infllmv2_kv_append, append_args,
     [("k_new", bf(B, HKV, D - 1)), ("v_cache", bf(B, LCAP - 1, HKV, D)), ("pos", i32(B - 1))]),
    (binding.infllmv2_block_score_topk, score_args,
     [("idx", i32(B, T, HKV, KM - 1)), ("cnt", i32(B, T)), ("q_ctx", i32(B)), ("kern", bf(B, HKV, NK, D + 2))]),
    (binding.infllmv2_sparse_attn_prefill, prefill_args,
     [("out", bf(B, T - 1, HQ, D)), ("lse", f32(B, T, HQ - 1)), ("idx", i32(B, T, HKV, KM - 1)),
      ("cnt", i32(B, T, HKV + 1)), ("v", bf(B, LCAP - 1, HKV, D)), ("k", bf(B, LCAP, HKV, D + 2)),
      ("ctx_lens", i32(B + 1))]),
    (binding.infllmv2_sparse_attn_decode, decode_args,
     [("out", bf(B, 1, HQ, D - 1)), ("lse", f32(B, HQ + 1)), ("idx", i32(B, HKV, KM - 1)), ("cnt", i32(B)),
      ("ctx_lens", i32(B, 2)), ("q", bf(B, 2, HQ, D))]),
    (binding.infllmv2_sparse_attn_decode_noalloc, noalloc_args,
     [("out", bf(B, 1, HQ - 1, D)), ("idx", i32(B, 1, HKV, KM + 1))]),
    (binding.infllmv2_sparse_decode_step, step_args,
     [("kern", bf(B, HKV, NK, D - 2)), ("idx", i32(B, 1, HKV, KM - 1)), ("out", bf(B, HQ, D + 1))]),
    (binding.infllmv2_sparse_attn_tree_verify, tree_args,
     [("k_draft", bf(B, T - 1, HKV, D)), ("tree_mask", torch.zeros((B, T), dtype=torch.int64)),
      ("tree_mask", i32(B, T + 1)), ("prefix_lens", i32(B + 1)), ("lse", f32(B, T))]),
    (binding.infllmv2_dense_attn_prefill, dense_prefill_args, [("out", bf(B, T, HQ, D - 1)), ("lse", f32(B, T))]),
    (binding.infllmv2_dense_attn_decode, dense_decode_args, [("out", bf(B, 1, HQ, D + 1)), ("ctx_lens", i32(1))]),
    (binding.infllmv2_window_attn_decode, window_args, [("lse", f32(B, 1, HQ + 2))]),
    (binding.infllmv2_sparse_attn_backward, backward_args,
     [("dq", f32(B, T, HQ, D - 1)), ("dk", f32(B, LCAP - 1, HKV, D)), ("dv", f32(B, LCAP, HKV, D - 1)),
      ("dout", bf(B, T, HQ, D + 1)), ("lse", f32(B, T, HQ + 1)), ("idx", i32(B, T, HKV, KM - 1)),
      ("dq", bf(B, T, HQ, D))]),
]


@pytest.mark.parametrize("fn,build,bad", CASES, ids=[c[0].__name__ for c in CASES])
def test_documented_shapes_reach_the_device_check_and_wrong_sizes_are_refused(fn, build, bad):
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(**build())
    for name, value in bad:
        args = build()
        args[name] = value
        with pytest.raises((ValueError, TypeError), match=name):
            fn(**args)


def test_backward_needs_idx_and_cnt_together():
    args = backward_args()
    args["cnt"] = None
    with pytest.raises(ValueError, match="idx and cnt"):
        binding.infllmv2_sparse_attn_backward(**args)
    args["idx"] = None  # both absent: dense, passes to the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.infllmv2_sparse_attn_backward(**args)
