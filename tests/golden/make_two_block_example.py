"""Writes two_block_example.json: a two-block example worked by hand from the method's definition.

The pages print no worked example, so this one is derived here; every stored number is a closed form
in e = exp(1) evaluated with ``math`` (no oracle, no GPU).  Definition followed: a kernel is the mean of
K over its window; a head's block relevance is the max over the block's kernels of the LSE-normalised
query-kernel score; the heads of a GQA group sum those scores and share one top-k set (QbitAI
"Tsinghua & ModelBest: MiniCPM4 technical details", section "Model architecture: InfLLM v2", items 1-3).

Setup: block 4 keys, kernel window 2 / stride 2 (so OVERLAP and CONTAINED agree), d = 2, two query
heads in one KV group, scale 1, no forced blocks, k = 1, the query sees n = 8 keys (blocks 0 and 1).
"""
import json
import math
import os

e2, e3 = math.exp(2), math.exp(3)
# head 0: q = (2, 0)  -> kernel scores z = (2, 0, 0, 0); head 1: q = (0, 1.5) -> z = (0, 0, 3, 0)
S0 = e2 / (e2 + 3) + 1 / (e3 + 3)
S1 = 1 / (e2 + 3) + e3 / (e3 + 3)
gold = {
    "citation": __doc__.split("\n\n")[1].replace("\n", " "),
    "params": {"block_size": 4, "kernel_size": 2, "kernel_stride": 2, "topk": 1, "init_blocks": 0,
               "local_blocks": 0, "dense_len": 0, "membership": 0, "scale": 1.0},
    "K": [[1, 0], [1, 0], [0, 0], [0, 0], [0, 2], [0, 2], [0, 0], [0, 0]],
    "V": [[5, 5], [5, 5], [5, 5], [5, 5], [1, 0], [1, 0], [0, 1], [0, 1]],
    "q": [[2, 0], [0, 1.5]],
    "n": 8,
    "kernels": [[1, 0], [0, 0], [0, 2], [0, 0]],
    "lse_heads": {"expr": ["log(e^2+3)", "log(e^3+3)"], "value": [math.log(e2 + 3), math.log(e3 + 3)]},
    "S": {"expr": ["e^2/(e^2+3) + 1/(e^3+3)", "1/(e^2+3) + e^3/(e^3+3)"], "value": [S0, S1]},
    "idx": [1],
    # block 1 keys: head 0 scores (0,0,0,0) -> uniform; head 1 scores (3,3,0,0)
    "out": {"expr": [["1/2", "1/2"], ["e^3/(e^3+1)", "1/(e^3+1)"]],
            "value": [[0.5, 0.5], [e3 / (e3 + 1), 1 / (e3 + 1)]]},
    "out_lse": {"expr": ["log 4", "log(2e^3+2)"], "value": [math.log(4), math.log(2 * e3 + 2)]},
}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "two_block_example.json"), "w") as f:
    json.dump(gold, f, indent=1)
