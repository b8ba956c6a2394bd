#!/usr/bin/env python
"""Benchmark of the InfLLM v2 sparse-attention path on B200 (libinfllmv2 through its C ABI).

Headline workload: sparse decode at 128K, batch 4 ragged (131072, 98304, 65536, 131072 keys at the first
step, +1 key per step), 32 query / 2 KV heads, d 128, top-64 + 1 initial + 2 local blocks of 64, kernels
of 32 keys / stride 16, dense below 8192.  One bench step = one decode step of one attention layer for the
4 sequences: incremental kernel pooling, block scoring + top-k, sparse attention (5 kernels, replayed as a
CUDA graph).  Eight independent layer caches (4.3 GB of K/V) rotate, so a layer's ~31 MB working set has
left the 126 MB L2 before the layer comes back; each layer walks the 256 decode positions.

Second workload (``prefill`` object): a 32K-token prefill of one layer (kernel pooling, scoring + top-k,
sparse attention with the first 8192 rows dense), 32 / 2 heads, d 128, Q/K/V ~ N(0,1) plus per-block
offsets N(0, 0.3^2).  Third (``backward`` object): the gradients dq, dk, dv of that prefill's sparse
attention for its selection, with a seeded N(0,1) dout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle on the host cores on the
same decode workload, each step a bounded sample of it.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode tokens/s @128K (HBM GB/s %) & prefill tok/s @32K (TC %)"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LENS_128K = (131072, 98304, 65536, 131072)
HQ, HKV, D = 32, 2, 128
# DRAM bytes (read + write) per call of the dominant C-ABI calls, each from one ncu capture of the kernel as
# it stands (profiles/decode_fused_128k.md, profiles/prefill_32k.md); None where the kernels changed after
# their capture (the two-call decode kernels took the paged / packed addressing since)
NCU_TRAFFIC = {
    "sparse_decode_step": None,                         # decode_fused_kernel without pooling: not captured at this build
    "sparse_decode_step_pool": 31_319_552,              # decode_fused_kernel pooling the new key's kernel
    "sparse_attn_decode": None,                         # attn_split_kernel + attn_merge_kernel
    "block_score_topk": None,                           # score_scan_kernel + score_select_kernel
    "sparse_attn_prefill": None,                        # attn_tc_kernel<16, 128>: changed since its capture
}
KERNELS_PER_STEP = {"two_call": 5,    # kernel pool, score scan, select, split attention, merge
                    "fused": 2,       # kernel pool, fused decode step (scoring + top-k + attention)
                    "fused_pool": 1}  # the fused decode step pooling the new key's kernel itself


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled every few ms)
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index):
        self.samples, self.reasons = [], 0
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report no clocks
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# decode @128K
# ------------------------------------------------------------------------------------------------
def nk(n):
    return 0 if n < 32 else (n - 32) // 16 + 1


def decode_step_bytes(lens, kmax=67):
    """Algorithmic HBM bytes of one decode step: kernel-cache scan + selected K/V blocks (+ q, out, new kernel)."""
    scan = sum(nk(n) * HKV * D * 2 for n in lens)
    kv = len(lens) * HKV * kmax * 64 * D * 2 * 2
    small = len(lens) * (HQ * D * 2 * 2 + HKV * D * 2 * 3)
    return scan, kv, scan + kv + small


class DecodeBench:
    def __init__(self, layers=8, steps_cycle=256, two_call=False, pooled=False):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import decode_128k_ragged

        self.torch, self.b = torch, binding
        self.NL, self.S = layers, steps_cycle
        self.two_call = two_call
        self.pooled = pooled and not two_call
        w = decode_128k_ragged(steps=steps_cycle)
        self.w = w
        self.p = binding.Params(**w.params)
        B = len(LENS_128K)
        self.B = B
        dev = torch.device("cuda")
        k0 = torch.from_numpy(w.k.view(np.int16)).to(dev).view(torch.bfloat16)
        v0 = torch.from_numpy(w.v.view(np.int16)).to(dev).view(torch.bfloat16)
        self.q_all = torch.from_numpy(w.extras["q_steps"].view(np.int16)).to(dev).view(torch.bfloat16)  # [S,B,1,Hq,d]
        self.Lcap = w.k.shape[1]
        self.max_ctx = max(LENS_128K) + steps_cycle - 1
        self.nk_cap = nk(self.max_ctx)
        # layer l: the same cache rolled along positions (independent data per layer, same lengths)
        self.k = [k0] + [torch.roll(k0, shifts=4096 * l + 64 * l, dims=1) for l in range(1, layers)]
        self.v = [v0] + [torch.roll(v0, shifts=4096 * l + 64 * l, dims=1) for l in range(1, layers)]
        lens0 = torch.tensor(LENS_128K, dtype=torch.int32)
        self.lens = (lens0[None, :] + torch.arange(steps_cycle, dtype=torch.int32)[:, None]).to(dev).contiguous()
        self.old = (self.lens - 1).contiguous()
        self.kern = []
        for l in range(layers):
            kern = torch.zeros((B, HKV, self.nk_cap, D), dtype=torch.bfloat16, device=dev)
            zero = torch.zeros(B, dtype=torch.int32, device=dev)
            binding.infllmv2_kernel_pool(self.k[l], zero, self.old[0], max(LENS_128K), self.p, kern)
            self.kern.append(kern)
        self.idx = torch.empty((B, 1, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, 1, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, 1, HQ, D), dtype=torch.bfloat16, device=dev)
        self.ws = binding.workspace(self.p, B, 1, self.max_ctx, HQ, HKV, D)
        self.graphs = {}
        torch.cuda.synchronize()

    def _coords(self, s):
        layer = s % self.NL
        pos = (s // self.NL) % self.S
        return layer, pos

    def q_of(self, layer, pos):
        return self.q_all[(pos + 37 * layer) % self.S]

    # the C-ABI calls of one decode step: incremental kernel pooling, then scoring + top-k + sparse attention
    # fused in one launch (infllmv2_sparse_decode_step; the two-call form is block_score_topk + sparse_attn_decode)
    def pool(self, layer, pos, stream=None):
        self.b.infllmv2_kernel_pool(self.k[layer], self.old[pos], self.lens[pos], 1, self.p, self.kern[layer], stream)

    def score(self, layer, pos, stream=None):
        self.b.infllmv2_block_score_topk(self.q_of(layer, pos), None, self.lens[pos], self.max_ctx, self.kern[layer],
                                         self.p, self.idx, self.cnt, self.ws, stream)

    def attend(self, layer, pos, stream=None):
        self.b.infllmv2_sparse_attn_decode(self.q_of(layer, pos), self.k[layer], self.v[layer], self.lens[pos],
                                           self.max_ctx, self.idx, self.cnt, self.p, self.out, None, self.ws, stream)

    def fused(self, layer, pos, stream=None):
        self.b.infllmv2_sparse_decode_step(self.q_of(layer, pos), self.kern[layer], self.k[layer], self.v[layer],
                                           self.lens[pos], self.max_ctx, self.p, self.idx, self.cnt, self.out, None,
                                           stream)

    def fused_pool(self, layer, pos, stream=None):
        self.b.infllmv2_sparse_decode_step_pool(self.q_of(layer, pos), self.kern[layer], self.k[layer], self.v[layer],
                                                self.lens[pos], self.max_ctx, self.p, self.idx, self.cnt, self.out,
                                                None, stream)

    def step_eager(self, s, stream=None):
        layer, pos = self._coords(s)
        if self.pooled:
            self.fused_pool(layer, pos, stream)
            return
        self.pool(layer, pos, stream)
        if self.two_call:
            self.score(layer, pos, stream)
            self.attend(layer, pos, stream)
        else:
            self.fused(layer, pos, stream)

    def decode_calls(self, q, layer, pos, out):
        """the step's C-ABI calls after the new rows are in the caches, for a query and output of the caller's"""
        if self.pooled:
            self.b.infllmv2_sparse_decode_step_pool(q, self.kern[layer], self.k[layer], self.v[layer], self.lens[pos],
                                                    self.max_ctx, self.p, self.idx, self.cnt, out, None)
            return
        self.b.infllmv2_kernel_pool(self.k[layer], self.old[pos], self.lens[pos], 1, self.p, self.kern[layer])
        if self.two_call:
            self.b.infllmv2_block_score_topk(q, None, self.lens[pos], self.max_ctx, self.kern[layer], self.p,
                                             self.idx, self.cnt, self.ws)
            self.b.infllmv2_sparse_attn_decode(q, self.k[layer], self.v[layer], self.lens[pos], self.max_ctx,
                                               self.idx, self.cnt, self.p, out, None, self.ws)
        else:
            self.b.infllmv2_sparse_decode_step(q, self.kern[layer], self.k[layer], self.v[layer], self.lens[pos],
                                               self.max_ctx, self.p, self.idx, self.cnt, out, None)

    def _capture(self, key, steps):
        """one CUDA graph of the given consecutive steps (warmed outside capture first)"""
        torch = self.torch
        g = self.graphs.get(key)
        if g is None:
            g = torch.cuda.CUDAGraph()
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                for s in steps:
                    self.step_eager(s)  # warm the launch path outside capture
            torch.cuda.current_stream().wait_stream(st)
            with torch.cuda.graph(g):
                for s in steps:
                    self.step_eager(s)
            self.graphs[key] = g
        return g

    def graph(self, s):
        """the single-step graph of step s"""
        return self._capture(self._coords(s), [s])

    def position_graph(self, s):
        """steps s .. s + NL - 1 (s a multiple of NL): every layer at one decode position, as a model's decode
        step runs them; one replay per position keeps PyTorch's per-replay generator prologue (two small fill
        kernels) off all but one step in NL"""
        return self._capture(("pos", self._coords(s)[1]), list(range(s, s + self.NL)))

    def _plan(self, lo, hi):
        """graphs covering steps [lo, hi): whole positions where they fit, single steps elsewhere"""
        plan, s = [], lo
        while s < hi:
            if s % self.NL == 0 and s + self.NL <= hi:
                plan.append(self.position_graph(s))
                s += self.NL
            else:
                plan.append(self.graph(s))
                s += 1
        return plan

    def timed(self, warmup, steps):
        torch = self.torch
        warm = self._plan(0, warmup)
        run = self._plan(warmup, warmup + steps)
        torch.cuda.synchronize()
        for g in warm:
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for g in run:
            g.replay()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3

    def per_call_times(self, warmup, steps):
        """average device time of each C-ABI call: `steps` consecutive calls of it (each on another layer cache
        and position) captured in one CUDA graph, replayed between two CUDA events on the current stream, so
        that neither host launch overhead nor the graph prologue is counted"""
        torch = self.torch
        names = ["kernel_pool", "block_score_topk", "sparse_attn_decode", "sparse_decode_step", "sparse_decode_step_pool"]
        fns = [self.pool, self.score, self.attend, self.fused, self.fused_pool]
        for s in range(warmup):
            self.step_eager(s)
        torch.cuda.synchronize()
        out = {}
        for name, fn in zip(names, fns):
            calls = [self._coords(s) for s in range(warmup, warmup + steps)]
            g = torch.cuda.CUDAGraph()
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                for layer, pos in calls:
                    fn(layer, pos)
            torch.cuda.current_stream().wait_stream(st)
            with torch.cuda.graph(g):
                for layer, pos in calls:
                    fn(layer, pos)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 4
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            e1.synchronize()
            out[name] = e0.elapsed_time(e1) / 1e3 / (reps * steps)
            del g
        return out

    def window_time(self, window, steps):
        """device time of one sliding-window decode call (the draft model's attention: the last `window` keys of
        each sequence), from `steps` consecutive calls over the rotating layer caches captured in one graph"""
        torch = self.torch
        p = self.b.Params(**self.w.params)
        ws = self.b.workspace(p, self.B, 1, self.max_ctx, HQ, HKV, D)
        out = torch.empty((self.B, 1, HQ, D), dtype=torch.bfloat16, device="cuda")
        calls = [self._coords(s) for s in range(steps)]

        def run():
            for layer, pos in calls:
                self.b.infllmv2_window_attn_decode(self.q_of(layer, pos), self.k[layer], self.v[layer], self.lens[pos],
                                                   self.max_ctx, window, 0.0, out, None, ws)
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            run()
        torch.cuda.current_stream().wait_stream(st)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 4
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3 / (reps * steps)

    def e2e(self, warmup, steps, graphs=True):
        """Same step through the C ABI with host buffers: every step copies that step's query and the new key
        and value rows from pinned host memory to the device in one copy, appends the rows to the caches
        (infllmv2_kv_append), pools, runs the step and reads the attention output back.  graphs: the calls of
        every layer at one decode position (copies included) are captured once as a CUDA graph and replayed
        per position, the way a serving loop issues a decode step; otherwise each call is issued eagerly from
        Python."""
        torch = self.torch
        B = self.B
        nq, nkv = B * HQ * D, B * HKV * D
        # per position: [query | new key rows | new value rows], bf16
        host = torch.empty((self.S, nq + 2 * nkv), dtype=torch.bfloat16).pin_memory()
        host[:, :nq].copy_(self.q_all.reshape(self.S, nq).cpu())
        lens_np = self.lens.cpu().numpy()
        k0c = self.k[0].cpu()
        v0c = self.v[0].cpu()
        for pos in range(self.S):
            for b in range(B):
                row = lens_np[pos, b] - 1
                host[pos, nq + b * HKV * D: nq + (b + 1) * HKV * D] = k0c[b, row].reshape(-1)
                host[pos, nq + nkv + b * HKV * D: nq + nkv + (b + 1) * HKV * D] = v0c[b, row].reshape(-1)
        out_host = torch.empty((B, 1, HQ, D), dtype=torch.bfloat16).pin_memory()
        stage = torch.empty(nq + 2 * nkv, dtype=torch.bfloat16, device="cuda")
        q_dev = stage[:nq].view(B, 1, HQ, D)
        k_new = stage[nq:nq + nkv].view(B, HKV, D)
        v_new = stage[nq + nkv:].view(B, HKV, D)
        h2d = stage.numel() * 2
        d2h = out_host.numel() * 2

        def one(s):
            layer, pos = self._coords(s)
            stage.copy_(host[pos], non_blocking=True)
            self.b.infllmv2_kv_append(k_new, v_new, self.old[pos], self.k[layer], self.v[layer])
            self.decode_calls(q_dev, layer, pos, self.out)
            out_host.copy_(self.out, non_blocking=True)

        # double-buffered staging for the overlapped form: step i's input copy and step i-1's read-back run on a
        # copy stream while step i-1's kernels run
        stage2 = [torch.empty_like(stage), torch.empty_like(stage)]
        out2 = [torch.empty_like(self.out), torch.empty_like(self.out)]
        out_host2 = [torch.empty_like(out_host).pin_memory(), torch.empty_like(out_host).pin_memory()]
        copy_stream = torch.cuda.Stream()

        def kernels(layer, pos, buf):
            st = stage2[buf]
            q2 = st[:nq].view(B, 1, HQ, D)
            kn, vn = st[nq:nq + nkv].view(B, HKV, D), st[nq + nkv:].view(B, HKV, D)
            self.b.infllmv2_kv_append(kn, vn, self.old[pos], self.k[layer], self.v[layer])
            self.decode_calls(q2, layer, pos, out2[buf])

        def overlapped(s0):
            """the NL steps of one position (captured): copies on copy_stream, kernels on the capture stream"""
            cap = torch.cuda.current_stream()
            ev = lambda: torch.cuda.Event()  # noqa: E731
            e_in = [ev() for _ in range(self.NL)]
            e_done = [ev() for _ in range(self.NL)]
            e_out = [ev() for _ in range(self.NL)]
            copy_stream.wait_stream(cap)
            with torch.cuda.stream(copy_stream):
                for i in range(min(2, self.NL)):
                    stage2[i].copy_(host[self._coords(s0 + i)[1]], non_blocking=True)
                    e_in[i].record()
            for i in range(self.NL):
                layer, pos = self._coords(s0 + i)
                buf = i % 2
                cap.wait_event(e_in[i])
                if i >= 2:
                    cap.wait_event(e_out[i - 2])  # out2[buf] read back
                kernels(layer, pos, buf)
                e_done[i].record()
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(e_done[i])
                    out_host2[buf].copy_(out2[buf], non_blocking=True)
                    e_out[i].record()
                    if i + 2 < self.NL:  # stage2[buf] is free once step i's kernels are done
                        stage2[buf].copy_(host[self._coords(s0 + i + 2)[1]], non_blocking=True)
                        e_in[i + 2].record()
            cap.wait_stream(copy_stream)

        for s in range(warmup):
            one(s)
        torch.cuda.synchronize()
        mode = "eager"
        if graphs:
            # whole positions only: warm-up and timed steps start on a position boundary
            lo = (warmup + self.NL - 1) // self.NL * self.NL
            steps = steps // self.NL * self.NL
            plan = []
            try:
                for s0 in range(lo, lo + steps, self.NL):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        overlapped(s0)
                    plan.append(g)
                mode = "overlapped"
            except RuntimeError:
                torch.cuda.synchronize()
                plan = []
                for s0 in range(lo, lo + steps, self.NL):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        for s in range(s0, s0 + self.NL):
                            one(s)
                    plan.append(g)
                mode = "serial"
            for g in plan[:2]:
                g.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if graphs:
            for g in plan:
                g.replay()
        else:
            for s in range(warmup, warmup + steps):
                one(s)
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3, h2d, d2h, steps, mode

    def e2e_batched(self, warmup, steps):
        """The same end-to-end step, with the copies gathered per decode position: one host-to-device copy of
        the position's inputs for all layers (each layer's query and new key / value rows, the same bytes per
        step as e2e), the layers' C-ABI calls, and one read-back of all the layers' outputs, in stream order in
        one CUDA graph per position (no cross-stream dependency inside it)."""
        torch = self.torch
        B, NL = self.B, self.NL
        nq, nkv = B * HQ * D, B * HKV * D
        w = nq + 2 * nkv
        host = torch.empty((self.S, NL, w), dtype=torch.bfloat16).pin_memory()
        q_host = self.q_all.reshape(self.S, nq).cpu()
        lens_np = self.lens.cpu().numpy()
        k0c, v0c = self.k[0].cpu(), self.v[0].cpu()
        for pos in range(self.S):
            row = torch.empty(w, dtype=torch.bfloat16)
            row[:nq] = q_host[pos]
            for b in range(B):
                r = lens_np[pos, b] - 1
                row[nq + b * HKV * D: nq + (b + 1) * HKV * D] = k0c[b, r].reshape(-1)
                row[nq + nkv + b * HKV * D: nq + nkv + (b + 1) * HKV * D] = v0c[b, r].reshape(-1)
            host[pos] = row[None, :].expand(NL, w)
        stage = torch.empty((NL, w), dtype=torch.bfloat16, device="cuda")
        out = torch.empty((NL,) + tuple(self.out.shape), dtype=torch.bfloat16, device="cuda")
        out_host = torch.empty(tuple(out.shape), dtype=torch.bfloat16).pin_memory()

        def position(s0):
            pos = self._coords(s0)[1]
            stage.copy_(host[pos], non_blocking=True)
            for i in range(NL):
                layer, _ = self._coords(s0 + i)
                st = stage[i]
                q2 = st[:nq].view(B, 1, HQ, D)
                kn, vn = st[nq:nq + nkv].view(B, HKV, D), st[nq + nkv:].view(B, HKV, D)
                self.b.infllmv2_kv_append(kn, vn, self.old[pos], self.k[layer], self.v[layer])
                self.decode_calls(q2, layer, pos, out[i])
            out_host.copy_(out, non_blocking=True)

        lo = (warmup + NL - 1) // NL * NL
        steps = steps // NL * NL
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            position(0)
        torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        plan = []
        for s0 in range(lo, lo + steps, NL):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                position(s0)
            plan.append(g)
        for g in plan[:2]:
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for g in plan:
            g.replay()
        e1.record()
        e1.synchronize()
        del plan
        return e0.elapsed_time(e1) / 1e3, w * 2, out_host[0].numel() * 2, steps, "batched"


# ------------------------------------------------------------------------------------------------
# prefill @32K
# ------------------------------------------------------------------------------------------------
def prefill_flops(T=32768, dense_len=8192, kmax=67):
    hq_d = HQ * D
    score = 2 * hq_d * sum(nk(t + 1) for t in range(dense_len, T))
    dense = 4 * hq_d * sum(t + 1 for t in range(dense_len))
    # a sparse row attends to kmax blocks: kmax-1 full ones and its own block up to itself
    attn = 4 * hq_d * sum((kmax - 1) * 64 + (t % 64) + 1 for t in range(dense_len, T))
    return score, attn, dense


def attn_tc_executed_flops(idx, cnt, T, dense_len, tok=8, step_keys=128):
    """MMA flops the tensor-core prefill attention issues for this selection: each 8-token tile walks the union of
    its tokens' block sets (every block 0..c for a dense row), two 64-key blocks per step (an odd last block is
    paired with a masked copy), and every step runs S = Q K^T and O += P V on 128 rows x 128 keys x d."""
    idx = np.asarray(idx)[0]  # [T, Hkv, kmax]
    cnt = np.asarray(cnt)[0]  # [T, Hkv]
    nb = (T - 1) // 64 + 1
    total = 0
    for g in range(idx.shape[1]):
        sel = np.zeros((T, nb), bool)
        k = idx[:, g, :]
        valid = (np.arange(k.shape[1])[None, :] < cnt[:, g][:, None]) & (k >= 0)
        rows = np.nonzero(valid)
        sel[rows[0], k[valid]] = True
        t = np.arange(T)
        dense = (t + 1) <= dense_len
        c = t // 64
        sel[dense] = np.arange(nb)[None, :] <= c[dense][:, None]
        ntile = (T + tok - 1) // tok
        pad = ntile * tok - T
        un = np.concatenate([sel, np.zeros((pad, nb), bool)]).reshape(ntile, tok, nb).any(axis=1).sum(axis=1)
        total += int(((un + 1) // 2).sum())
    return total * 2 * (2 * 128 * step_keys * D)


class PrefillBench:
    def __init__(self):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import prefill_32k

        self.torch, self.b = torch, binding
        w = prefill_32k()
        self.T = w.q.shape[1]
        dev = torch.device("cuda")
        to = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        self.q, self.k, self.v = to(w.q), to(w.k), to(w.v)
        self.p = binding.Params(**w.params)
        self.lens = torch.tensor([self.T], dtype=torch.int32, device=dev)
        self.zero = torch.zeros(1, dtype=torch.int32, device=dev)
        self.nk_cap = nk(self.T)
        self.kern = torch.zeros((1, HKV, self.nk_cap, D), dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty((1, self.T, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((1, self.T, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((1, self.T, HQ, D), dtype=torch.bfloat16, device=dev)
        self.ws = binding.workspace(self.p, 1, self.T, self.T, HQ, HKV, D)

    def pool(self):
        self.b.infllmv2_kernel_pool(self.k, self.zero, self.lens, self.T, self.p, self.kern)

    def score(self):
        self.b.infllmv2_block_score_topk(self.q, None, self.lens, self.T, self.kern, self.p, self.idx, self.cnt, self.ws)

    def attend(self):
        self.b.infllmv2_sparse_attn_prefill(self.q, self.k, self.v, None, self.lens, self.T, self.idx, self.cnt,
                                            self.p, self.out)

    def backward_setup(self):
        """The forward's out / lse for the current selection and a seeded dout, for the gradient pass."""
        torch, b = self.torch, self.b
        dev = torch.device("cuda")
        self.lse = torch.empty((1, self.T, HQ), dtype=torch.float32, device=dev)
        self.pool()
        self.score()
        b.infllmv2_sparse_attn_prefill(self.q, self.k, self.v, None, self.lens, self.T, self.idx, self.cnt, self.p,
                                       self.out, self.lse)
        gen = torch.Generator(device=dev).manual_seed(1103)
        self.dout = torch.randn((1, self.T, HQ, D), generator=gen, device=dev).to(torch.bfloat16)
        self.dq = torch.empty((1, self.T, HQ, D), dtype=torch.float32, device=dev)
        self.dk = torch.empty((1, self.T, HKV, D), dtype=torch.float32, device=dev)
        self.dv = torch.empty((1, self.T, HKV, D), dtype=torch.float32, device=dev)
        self.bws = b.backward_workspace(self.p, 1, self.T, self.T, HQ, HKV, D)

    def backward(self):
        self.b.infllmv2_sparse_attn_backward(self.q, self.k, self.v, None, self.lens, self.T, self.idx, self.cnt,
                                             self.p, self.out, self.lse, self.dout, self.dq, self.dk, self.dv,
                                             self.bws)

    def lse_estimate_leg(self, strides=(2, 4), reps=5):
        """Scoring + top-k with the LSE estimated from every s-th visible kernel (lse_stride = s) against the
        exact scoring of the same kernel cache: the time of one call (mean of `reps`, after two untimed) and the
        share of sparse (token, group) rows whose selection is unchanged.  The pages name a LogSumExp estimation
        for fast top-k but do not define it, so this reading's parity with the pages is unpinned."""
        import dataclasses
        torch, b = self.torch, self.b
        self.pool()

        def timed(p, idx, cnt):
            for _ in range(2):
                b.infllmv2_block_score_topk(self.q, None, self.lens, self.T, self.kern, p, idx, cnt, self.ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                b.infllmv2_block_score_topk(self.q, None, self.lens, self.T, self.kern, p, idx, cnt, self.ws)
            e1.record()
            e1.synchronize()
            return e0.elapsed_time(e1) / reps

        exact_ms = timed(self.p, self.idx, self.cnt)
        ref_idx, ref_cnt = self.idx.clone(), self.cnt.clone()
        idx2, cnt2 = torch.empty_like(self.idx), torch.empty_like(self.cnt)
        t0 = self.p.dense_len  # rows below the dense switch take no selection
        res = {"exact_ms": exact_ms, "rows": f"tokens {t0}..{self.T - 1} x {HKV} groups",
               "parity": "unpinned by the pages (the estimate is this library's reading)"}
        for s in strides:
            ms = timed(dataclasses.replace(self.p, lse_stride=s), idx2, cnt2)
            same = ((cnt2 == ref_cnt) & (idx2 == ref_idx).all(-1))[0, t0:]
            res[f"s{s}"] = {"ms": ms, "time_saved_frac": 1.0 - ms / exact_ms,
                            "rows_unchanged": float(same.float().mean().item())}
        return res

    def run_backward(self, warmup, steps):
        torch = self.torch
        for _ in range(warmup):
            self.backward()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            self.backward()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3

    def run(self, warmup, steps):
        torch = self.torch
        fns = {"kernel_pool": self.pool, "block_score_topk": self.score, "sparse_attn_prefill": self.attend}
        for _ in range(warmup):
            for f in fns.values():
                f()
        torch.cuda.synchronize()
        ev = {n: [] for n in fns}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            for n, f in fns.items():
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                f()
                b.record()
                ev[n].append((a, b))
        e1.record()
        e1.synchronize()
        total = e0.elapsed_time(e1) / 1e3
        per = {n: float(np.mean([a.elapsed_time(b) for a, b in v])) / 1e3 for n, v in ev.items()}
        return total, per


def kernel_pool_backward_leg(peaks, peak_kind, reps=20):
    """The gradient of the semantic kernels with respect to K over the 128K decode batch's shapes (4 sequences
    of 131072 keys, 2 KV heads, d 128): dk (fp32, 537 MB) overwritten from the kernel gradients (fp32, 34 MB).
    HBM-bound; the algorithmic bytes are that write and that read.  The 537 MB written per call exceeds L2, so
    consecutive calls do not hit it; the time is the mean of `reps` calls between two CUDA events."""
    import torch
    from trainable_block_sparse_v2_b200 import binding
    B, L = len(LENS_128K), max(LENS_128K)
    nk_cap = nk(L)
    dkern = torch.randn((B, HKV, nk_cap, D), dtype=torch.float32, device="cuda")
    dk = torch.empty((B, L, HKV, D), dtype=torch.float32, device="cuda")
    lens = torch.tensor([L] * B, dtype=torch.int32, device="cuda")
    p = binding.Params()
    for _ in range(3):
        binding.infllmv2_kernel_pool_backward(dkern, lens, L, p, dk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        binding.infllmv2_kernel_pool_backward(dkern, lens, L, p, dk)
    e1.record()
    e1.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    nbytes = dk.numel() * 4 + B * HKV * nk(L) * D * 4
    del dkern, dk
    torch.cuda.empty_cache()
    return {"workload": "dk of 4 x 131072 keys, 2 KV heads, d 128 (fp32) from their kernel gradients",
            "us_per_call": t * 1e6, "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / t / 1e9,
            "frac_of_" + peak_kind: nbytes / t / 1e9 / peaks["hbm_gbs"], "timing": f"mean of {reps} calls"}


class Decode32kBench:
    """Decode at a 32K context, batch 1 (32 / 2 heads, d 128, top-k 64): one step = the fused decode step that
    pools the new key's kernel, scores, selects and attends in one launch, on a cache restored every step (the pool of the
    step's window rewrites the same kernel).  Its working set (~5.4 MB) fits in L2, so L2 is flushed before
    every timed step; the time is the median of the steps."""

    def __init__(self):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import decode_32k

        self.torch, self.b = torch, binding
        w = decode_32k()
        dev = torch.device("cuda")
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)  # noqa: E731
        self.L = int(w.ctx_lens[0])
        self.q, self.k, self.v = to(w.q), to(w.k), to(w.v)
        self.p = binding.Params(**w.params)
        self.lens, self.old = i32([self.L]), i32([self.L - 1])
        self.kern = torch.zeros((1, HKV, nk(self.L), D), dtype=torch.bfloat16, device=dev)
        binding.infllmv2_kernel_pool(self.k, i32([0]), self.old, self.L - 1, self.p, self.kern)
        self.idx = torch.empty((1, 1, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((1, 1, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((1, 1, HQ, D), dtype=torch.bfloat16, device=dev)
        self.l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(self):
        self.b.infllmv2_sparse_decode_step_pool(self.q, self.kern, self.k, self.v, self.lens, self.L, self.p, self.idx,
                                                self.cnt, self.out, None)

    def run(self, warmup, steps):
        """median seconds per step, each step timed alone after an L2 flush"""
        torch = self.torch
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        evs = []
        for _ in range(steps):
            self.l2_flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            self.step()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in evs])) / 1e3


class PagedDecodeBench:
    """The 128K ragged decode batch (step 0) on a paged cache: the keys and values of the 4 sequences scattered
    over a shuffled pool of 64-position pages.  One step = the paged kernel pool of the new key + the paged fused
    decode step; the same step on the contiguous cache is timed the same way beside it.  L2 is flushed before
    every timed step; the time is the median of the steps."""

    def __init__(self):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import decode_128k_ragged

        self.torch, self.b = torch, binding
        w = decode_128k_ragged(steps=1)
        dev = torch.device("cuda")
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)  # noqa: E731
        self.lens_h = w.ctx_lens.astype(np.int64)
        B = len(self.lens_h)
        self.L = int(self.lens_h.max())
        self.q, self.k, self.v = to(w.q), to(w.k), to(w.v)
        self.p = binding.Params(**w.params)
        # pages: every sequence's blocks on a shuffled set of pages
        need = [int((n + 63) // 64) for n in self.lens_h]
        max_pages = max(need)
        rng = np.random.default_rng(77)
        perm = rng.permutation(sum(need)).astype(np.int32)
        table = np.full((B, max_pages), -1, np.int32)
        off = 0
        for b, m in enumerate(need):
            table[b, :m] = perm[off:off + m]
            off += m
        self.table = i32(table)
        num_pages = sum(need)
        Hkv, Dd = self.k.shape[2], self.k.shape[3]
        self.kp = torch.empty((num_pages * 64, Hkv, Dd), dtype=torch.bfloat16, device=dev)
        self.vp = torch.empty_like(self.kp)
        for b, m in enumerate(need):
            rows = (torch.from_numpy(table[b, :m].astype(np.int64)).to(dev)[:, None] * 64 +
                    torch.arange(64, device=dev)[None]).reshape(-1)
            n = min(m * 64, self.k.shape[1])
            self.kp[rows[:n]] = self.k[b, :n]
            self.vp[rows[:n]] = self.v[b, :n]
        self.lens, self.old = i32(self.lens_h), i32(self.lens_h - 1)
        self.kern_p = torch.zeros((B, HKV, nk(self.L), D), dtype=torch.bfloat16, device=dev)
        self.kern_c = torch.zeros_like(self.kern_p)
        binding.infllmv2_kernel_pool_paged(self.kp, self.table, i32(np.zeros(B)), self.old, self.L, self.p,
                                           self.kern_p)
        binding.infllmv2_kernel_pool(self.k, i32(np.zeros(B)), self.old, self.L, self.p, self.kern_c)
        self.idx = torch.empty((B, 1, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, 1, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, 1, HQ, D), dtype=torch.bfloat16, device=dev)
        self.l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step_paged(self):
        self.b.infllmv2_kernel_pool_paged(self.kp, self.table, self.old, self.lens, 1, self.p, self.kern_p)
        self.b.infllmv2_sparse_decode_step_paged(self.q, self.kern_p, self.kp, self.vp, self.table, self.lens, self.L,
                                                 self.p, self.idx, self.cnt, self.out, None)

    def step_contiguous(self):
        self.b.infllmv2_kernel_pool(self.k, self.old, self.lens, 1, self.p, self.kern_c)
        self.b.infllmv2_sparse_decode_step(self.q, self.kern_c, self.k, self.v, self.lens, self.L, self.p, self.idx,
                                           self.cnt, self.out, None)

    def run(self, fn, warmup, steps):
        """median seconds per step, each step timed alone after an L2 flush"""
        torch = self.torch
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        evs = []
        for _ in range(steps):
            self.l2_flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in evs])) / 1e3


class VarlenPrefillBench:
    """A packed batch of 4 prefill sequences (T = L = 32768, 16384, 8192, 4096 tokens; 32 / 2 heads, d 128,
    top-k 64, dense below 8192, N(0,1) with per-block offsets like the 32K prefill): one call of the packed
    prefill (kernel pool, scoring + top-k, attention: three launches for the batch) against the same sequences
    one at a time through the per-sequence calls (three launches each).  Mean of `steps` passes."""

    LENS = (32768, 16384, 8192, 4096)

    def __init__(self):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import prefill_case

        self.torch, self.b = torch, binding
        dev = torch.device("cuda")
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        self.seqs = []
        for i, T in enumerate(self.LENS):
            w = prefill_case(T, HQ, HKV, D, topk=64, dense_len=8192, seed=1300 + i, n_needles=0,
                             block_offset_std=0.3)
            self.seqs.append((to(w.q[0]), to(w.k[0]), to(w.v[0])))
        self.p = binding.Params(**w.params)
        B = len(self.LENS)
        cu = np.concatenate([[0], np.cumsum(self.LENS)]).astype(np.int32)
        self.cu = torch.from_numpy(cu).to(dev)
        self.q = torch.cat([s[0] for s in self.seqs])
        self.k = torch.cat([s[1] for s in self.seqs])
        self.v = torch.cat([s[2] for s in self.seqs])
        self.T = int(cu[-1])
        self.Lmax = max(self.LENS)
        self.kern = torch.zeros((B, HKV, nk(self.Lmax), D), dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty((self.T, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((self.T, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((self.T, HQ, D), dtype=torch.bfloat16, device=dev)
        # the packed scoring of long prompts runs on the token tiles, which need no workspace (a workspace sized
        # for every entry point at B x 32K rows would be the split attention's, hundreds of GB)
        self.ws = None
        self.lens = [torch.tensor([T], dtype=torch.int32, device=dev) for T in self.LENS]
        self.kerns = [torch.zeros((1, HKV, nk(T), D), dtype=torch.bfloat16, device=dev) for T in self.LENS]
        self.zero = torch.zeros(1, dtype=torch.int32, device=dev)

    def packed(self):
        self.b.infllmv2_sparse_prefill_varlen(self.q, self.k, self.v, self.cu, self.cu, self.Lmax, self.Lmax, self.p,
                                              self.kern, self.idx, self.cnt, self.out, None, self.ws)

    def one_by_one(self):
        b, off = self.b, 0
        for i, T in enumerate(self.LENS):
            q, k, v = self.seqs[i]
            idx, cnt, out = self.idx[off:off + T][None], self.cnt[off:off + T][None], self.out[off:off + T][None]
            b.infllmv2_kernel_pool(k[None], self.zero, self.lens[i], T, self.p, self.kerns[i])
            b.infllmv2_block_score_topk(q[None], None, self.lens[i], T, self.kerns[i], self.p, idx, cnt, self.ws)
            b.infllmv2_sparse_attn_prefill(q[None], k[None], v[None], None, self.lens[i], T, idx, cnt, self.p, out)
            off += T

    def run(self, fn, warmup, steps):
        torch = self.torch
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3 / steps


class TreeBench:
    """Tree-draft verification at a 64K prefix (one sequence, 16 draft nodes of depth <= 6, 32 / 2 heads,
    d 128, top-k 64).  One pass: the draft queries' block scoring + top-k over the whole prefix, then the tree
    attention over each draft's selected prefix blocks and its ancestor drafts.  The prefix's kernel cache is
    pooled once, untimed; L2 is flushed before every timed pass."""

    def __init__(self):
        import torch
        from trainable_block_sparse_v2_b200 import binding
        from trainable_block_sparse_v2_b200.workloads import tree_verify_64k

        self.torch, self.b = torch, binding
        w = tree_verify_64k()
        dev = torch.device("cuda")
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)  # noqa: E731
        self.P = int(w.ctx_lens[0])
        self.N = w.q.shape[1]
        self.q, self.k, self.v = to(w.q), to(w.k), to(w.v)
        self.k_draft, self.v_draft = to(w.extras["k_draft"]), to(w.extras["v_draft"])
        self.mask = i32(w.extras["tree_mask"].view(np.int32))
        self.p = binding.Params(**w.params)
        self.lens = i32(w.ctx_lens)
        self.q_ctx = i32(w.q_ctx)
        self.kern = torch.zeros((1, HKV, nk(self.P), D), dtype=torch.bfloat16, device=dev)
        binding.infllmv2_kernel_pool(self.k, i32([0]), self.lens, self.P, self.p, self.kern)
        self.idx = torch.empty((1, self.N, HKV, self.p.kmax), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((1, self.N, HKV), dtype=torch.int32, device=dev)
        self.out = torch.empty((1, self.N, HQ, D), dtype=torch.bfloat16, device=dev)
        self.ws = binding.workspace(self.p, 1, self.N, self.P, HQ, HKV, D)
        self.l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def verify(self):
        self.b.infllmv2_block_score_topk(self.q, self.q_ctx, None, self.P, self.kern, self.p, self.idx, self.cnt,
                                         self.ws)
        self.b.infllmv2_sparse_attn_tree_verify(self.q, self.k, self.v, self.lens, self.P, self.k_draft, self.v_draft,
                                                self.mask, self.idx, self.cnt, self.p, self.out, None, self.ws)

    def run(self, warmup, passes):
        """median seconds per pass, each pass timed alone after an L2 flush"""
        torch = self.torch
        for _ in range(warmup):
            self.verify()
        torch.cuda.synchronize()
        evs = []
        for _ in range(passes):
            self.l2_flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            self.verify()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in evs])) / 1e3

    def bytes_per_pass(self):
        """Algorithmic bytes: the kernel cache once, each group's union of selected prefix blocks once (keys
        and values; a partial last block counts its keys), the draft keys / values, queries and outputs."""
        idx, cnt = self.idx.cpu().numpy(), self.cnt.cpu().numpy()
        keys = 0
        for g in range(HKV):
            blocks = {int(x) for i in range(self.N) for x in idx[0, i, g, :max(0, min(int(cnt[0, i, g]), self.p.kmax))]
                      if 0 <= x and 64 * int(x) < self.P}
            keys += sum(min(64, self.P - 64 * b) for b in blocks)
        return (nk(self.P) * HKV * D * 2 + keys * D * 2 * 2 + self.N * HKV * D * 2 * 2 + self.N * HQ * D * 2 * 2,
                keys)


# ------------------------------------------------------------------------------------------------
# oracle (CPU) timing on a bounded sample of the decode workload
# ------------------------------------------------------------------------------------------------
class OracleDecode:
    """The fp64 oracle doing decode steps of the 128K workload on the host cores, restricted to a subset of
    the (sequence, KV group) rows; a token is credited per sequence once both of its groups are done."""

    def __init__(self, seqs, groups=(0, 1)):
        import oracle
        from trainable_block_sparse_v2_b200.workloads import decode_128k_ragged

        self.o = oracle
        w = decode_128k_ragged(steps=4)
        self.seqs, self.groups = list(seqs), list(groups)
        self.P = oracle.Params(**w.params)
        G = HQ // HKV
        heads = [h for g in self.groups for h in range(g * G, (g + 1) * G)]
        self.K = np.ascontiguousarray(w.k[self.seqs][:, :, self.groups])
        self.V = np.ascontiguousarray(w.v[self.seqs][:, :, self.groups])
        self.L0 = np.array([LENS_128K[i] for i in self.seqs], np.int32)
        self.nk_cap = nk(int(self.L0.max()) + 4)
        self.kern = oracle.kernel_pool(self.K, np.zeros_like(self.L0), self.L0 - 1, 32, 16, nk_cap=self.nk_cap)
        self.q_steps = np.ascontiguousarray(w.extras["q_steps"][:, self.seqs][:, :, :, heads])
        self.tokens_per_step = len(self.seqs) * len(self.groups) / HKV

    def step(self, s):
        L = self.L0 + (s % 4)
        self.o.kernel_pool(self.K, L - 1, L, 32, 16, kern=self.kern, nk_cap=self.nk_cap)
        q = self.q_steps[s % 4]
        r = self.o.block_score_topk(q, self.kern, L[:, None], self.P)
        self.o.sparse_attention(q, self.K, self.V, L[:, None], r["idx"], r["cnt"], self.P)
        return self.tokens_per_step


def cpu_baseline(budget_s=15.0):
    import oracle
    od = OracleDecode(range(len(LENS_128K)))
    od.step(0)  # warm
    t0 = time.perf_counter()
    n_tok, s = 0.0, 0
    while time.perf_counter() - t0 < budget_s or s < 1:
        n_tok += od.step(s)
        s += 1
    dt = time.perf_counter() - t0
    return {"value": n_tok / dt, "unit": UNIT, "cores": min(oracle.num_threads(), len(LENS_128K) * HKV),
            "kind": "oracle",
            "sample": f"{s} decode steps of the 4-sequence 128K batch (kernel pool of the new window, scoring + "
                      f"top-k, sparse attention), fp64, {dt:.1f} s; rows (sequence, group) run in parallel"}


# ------------------------------------------------------------------------------------------------
def dist_setup(n, backend="nccl"):
    """one process per GPU: RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the launcher's environment.
    backend "gloo" (CPU, no device binding) serves the multi-process tests."""
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier_max(x, ws, device="cuda"):
    """the max over ranks of a per-rank duration (every rank gets it)"""
    import torch
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws, cuda=True):
    import torch
    if cuda:
        torch.cuda.synchronize()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_rate(units_per_rank, ws, t_max):
    """whole-job throughput: the units every rank processed (weak scaling: the same count on each) over the
    slowest rank's device time"""
    return units_per_rank * ws / t_max


def run_ours(args):
    import torch
    from trainable_block_sparse_v2_b200.build import build
    from trainable_block_sparse_v2_b200 import binding

    ws, rank, local = dist_setup(args.gpus)
    if rank == 0:
        build()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    binding.load()
    peaks, peak_kind = load_peaks()

    if not args.no_decode:
        two_call = args.decode_path == "two_call"
        pooled = args.decode_path == "fused_pool"
        db = DecodeBench(layers=args.layers, two_call=two_call, pooled=pooled)
        # timed region: exactly K decode steps (graph replays), barrier + synchronize on both sides
        barrier(ws)
        with ClockSampler(torch.cuda.current_device()) as clk:
            t = db.timed(args.warmup, args.steps)
        barrier(ws)
        t = barrier_max(t, ws)
        value = whole_job_rate(len(LENS_128K) * args.steps, ws, t)

        per = db.per_call_times(8, min(args.steps, 256)) if args.per_call else {
            "kernel_pool": float("nan"), "block_score_topk": float("nan"), "sparse_attn_decode": float("nan"),
            "sparse_decode_step": float("nan"), "sparse_decode_step_pool": float("nan")}
        lens_mid = [n + 128 for n in LENS_128K]
        scan_b, kv_b, step_b = decode_step_bytes(lens_mid)
        if two_call:
            # dominant call of the two-call step: the larger of block scoring + top-k and sparse attention
            dom = max(("block_score_topk", "sparse_attn_decode"), key=lambda k: per[k] if per[k] == per[k] else -1.0)
            dom_bytes = {"block_score_topk": scan_b, "sparse_attn_decode": kv_b}[dom]
        else:
            # the fused scoring + top-k + attention launch carries the whole step's traffic (with pooling: plus the
            # new key's 32-key window once per 16 steps, ~4 KB per sequence and step on average, not counted)
            dom = "sparse_decode_step_pool" if pooled else "sparse_decode_step"
            dom_bytes = scan_b + kv_b
        achieved = dom_bytes / per[dom] / 1e9
        # the draft model's sliding-window attention on the same caches (next-row measurement)
        win = 2048
        t_win = db.window_time(win, min(args.steps, 256))
        win_bytes = len(LENS_128K) * HKV * win * D * 2 * 2
        e2e_steps = min(args.steps, 512)
        e2e_t, h2d, d2h, e2e_steps, e2e_mode = db.e2e(8, e2e_steps) if args.e2e else \
            (float("nan"), 0, 0, e2e_steps, "skipped")
        e2e_eager_t, _, _, e2e_eager_steps, _ = db.e2e(8, e2e_steps, graphs=False) if args.e2e else \
            (float("nan"), 0, 0, e2e_steps, "skipped")
        e2e_modes = {}
        if args.e2e:
            # both graph forms; the line reports the faster, and both
            e2e_modes[e2e_mode] = len(LENS_128K) * e2e_steps / e2e_t
            bt_, bh2d, bd2h, bsteps, bmode = db.e2e_batched(8, e2e_steps)
            e2e_modes[bmode] = len(LENS_128K) * bsteps / bt_
            if bsteps / bt_ > e2e_steps / e2e_t:
                e2e_t, h2d, d2h, e2e_steps, e2e_mode = bt_, bh2d, bd2h, bsteps, bmode

        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "decode_128k_ragged", "batch": 4, "ctx_lens_step0": list(LENS_128K),
                       "heads_q_kv": [HQ, HKV], "head_dim": D, "block": 64, "kernel_window_stride": [32, 16],
                       "topk": 64, "init_local": [1, 2], "dense_len": 8192, "decode_positions": 256,
                       "layers_rotating": args.layers, "parallelism": f"replicas{ws}",
                       "l2": "inputs larger than L2: 8 rotating layer caches, each step's 31 MB working set is evicted "
                             "before its layer returns",
                       "step": ("one decode step of one layer for 4 sequences: kernel_pool + block_score_topk + "
                                "sparse_attn_decode, replayed as a CUDA graph" if two_call else
                                "one decode step of one layer for 4 sequences: sparse_decode_step_pool (the new key's "
                                "kernel pooled, scoring, top-k and sparse attention in one cluster kernel), replayed "
                                "as a CUDA graph" if pooled else
                                "one decode step of one layer for 4 sequences: kernel_pool + sparse_decode_step "
                                "(scoring, top-k and sparse attention in one cluster kernel), replayed as a CUDA graph")},
            "hbm": {"algorithmic_bytes_per_step": step_b, "achieved_gbs_per_gpu": step_b / (t / args.steps) / 1e9,
                    "frac_of_" + peak_kind: step_b / (t / args.steps) / 1e9 / peaks["hbm_gbs"]},
            "per_call_ms": {k: v * 1e3 for k, v in per.items()},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "peak_kind": peak_kind + " (burst copy)",
                         "algorithmic_bytes": dom_bytes, "traffic": NCU_TRAFFIC.get(dom)},
            "clocks": clk.summary(),
            "e2e": {"value": len(LENS_128K) * e2e_steps / e2e_t, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "mode": {"overlapped": "per decode position, one CUDA graph of the 8 layers' C-ABI calls; each "
                                           "step's input copy and read-back on a copy stream, double-buffered, "
                                           "overlapping the neighbouring steps' kernels",
                             "serial": "per decode position, one CUDA graph of the 8 layers' C-ABI calls with "
                                       "their copies in stream order",
                             "batched": "per decode position, one CUDA graph: one copy of the 8 layers' inputs, "
                                        "their C-ABI calls, one read-back of their outputs, in stream order"
                             }.get(e2e_mode, e2e_mode),
                    "modes": e2e_modes,
                    "eager_value": len(LENS_128K) * e2e_eager_steps / e2e_eager_t},
            "gpu_launches": KERNELS_PER_STEP[args.decode_path] * args.steps,
            "window_decode": {"window": win, "value": len(LENS_128K) / t_win, "unit": UNIT, "us_per_call": t_win * 1e6,
                              "algorithmic_bytes": win_bytes, "achieved_gbs": win_bytes / t_win / 1e9,
                              "frac_of_" + peak_kind: win_bytes / t_win / 1e9 / peaks["hbm_gbs"],
                              "note": "the draft model's sliding-window decode attention (last 2048 keys), "
                                      "4 sequences per call, in the decode step's cluster kernel"},
        }
        del db
        torch.cuda.empty_cache()
    else:
        # profiling runs of the prefill kernels alone: no decode line
        line = {"metric": METRIC, "unit": UNIT, "n_gpus": ws, "note": "decode skipped (--no-decode)",
                "gpu_launches": 0}

    if not args.no_prefill:
        pb = PrefillBench()
        pt, pper = pb.run(3, args.prefill_steps)
        pt = barrier_max(pt, ws)
        sf, af, df = prefill_flops()
        flops = sf + af + df
        pdom = max(pper, key=pper.get)
        dom_flops = {"sparse_attn_prefill": af + df, "block_score_topk": 2 * sf, "kernel_pool": 0}[pdom]
        pach = dom_flops / pper[pdom] / 1e12
        exec_tf = attn_tc_executed_flops(pb.idx.cpu().numpy(), pb.cnt.cpu().numpy(), pb.T, pb.p.dense_len) / 1e12
        line["prefill"] = {
            "workload": "prefill_32k", "value": whole_job_rate(pb.T * args.prefill_steps, ws, pt), "unit": UNIT,
            "ms_per_step": pt / args.prefill_steps * 1e3, "steps": args.prefill_steps,
            "algorithmic_tflop_per_step": flops / 1e12,
            "executed_tflop": {"sparse_attn_prefill": exec_tf,
                               "achieved_tflops": exec_tf / pper["sparse_attn_prefill"] if pper.get("sparse_attn_prefill") else None,
                               "frac_of_" + peak_kind: (exec_tf / pper["sparse_attn_prefill"] / peaks["bf16_tflops"]
                                                        if pper.get("sparse_attn_prefill") else None),
                               "note": "MMA flops issued by the tensor-core attention (8-token tiles over the union "
                                       "of their block sets), against af + df algorithmic; achieved_tflops is that "
                                       "issued work over the attention call's time"},
            "tc_frac_of_" + peak_kind: flops / (pt / args.prefill_steps) / 1e12 / peaks["bf16_tflops"],
            "per_call_ms": {k: v * 1e3 for k, v in pper.items()},
            "roofline": {"bound": "tensor", "kernel": pdom, "achieved": pach, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": pach / peaks["bf16_tflops"], "peak_kind": peak_kind + " (burst)",
                         "traffic": NCU_TRAFFIC.get(pdom)},
        }
        line["gpu_launches"] += args.prefill_steps * 3  # kernel pool, scoring + top-k, attention
        if not args.no_lse_estimate:
            # untimed for the headline: the scoring call alone at lse_stride 2 and 4, against the exact call
            line["lse_estimate"] = pb.lse_estimate_leg()
        if not args.no_backward:
            pb.backward_setup()
            bt = barrier_max(pb.run_backward(3, args.prefill_steps), ws)
            bflops = 2.5 * (af + df)  # 10 d flops per attended (row, key): S, dP, dV, dQ, dK
            bach = bflops / (bt / args.prefill_steps) / 1e12
            line["backward"] = {
                "workload": "prefill_32k gradients (dq, dk, dv) for the forward's selection",
                "value": whole_job_rate(pb.T * args.prefill_steps, ws, bt), "unit": UNIT,
                "ms_per_step": bt / args.prefill_steps * 1e3, "steps": args.prefill_steps,
                "algorithmic_tflop_per_step": bflops / 1e12, "achieved_tflops": bach,
                "tc_frac_of_" + peak_kind: bach / peaks["bf16_tflops"],
                "kernels": "zero, prep, scan, fill (block lists), order (work items by token), bwd_dq_tc and "
                           "bwd_dkdv_tc (tcgen05/TMEM, TMA)",
            }
            line["gpu_launches"] += args.prefill_steps * 7
        del pb
        torch.cuda.empty_cache()
        if not args.no_backward:
            line["kernel_pool_backward"] = kernel_pool_backward_leg(peaks, peak_kind)

    if not args.no_decode32k:
        # batch-1 decode at 32K: launch-latency bound by nature (5.4 MB per step); reported, like the tree leg,
        # without raising, and with the same collective steps on every rank
        d32, t32, err = None, float("nan"), None
        try:
            d32 = Decode32kBench()
            t32 = d32.run(10, 1000)
        except Exception as e:  # noqa: BLE001
            err = f"{type(e).__name__}: {e}"[:300]
        t32 = barrier_max(t32, ws)
        if err is None and t32 == t32:
            _, _, b32 = decode_step_bytes([d32.L])
            line["decode_32k"] = {
                "workload": "decode_32k", "value": whole_job_rate(1, ws, t32), "unit": UNIT, "us_per_step": t32 * 1e6,
                "steps": 1000, "timing": "median of 1000 steps, L2 flushed before each",
                "algorithmic_bytes": b32, "achieved_gbs": b32 / t32 / 1e9,
                "frac_of_" + peak_kind: b32 / t32 / 1e9 / peaks["hbm_gbs"],
                "note": "one step = sparse_decode_step_pool (the new key's kernel pooled in the same launch), batch 1",
            }
        else:
            line["decode_32k"] = {"workload": "decode_32k", "error": err or "no time"}
        del d32
        torch.cuda.empty_cache()

    if not args.no_tree:
        # tree-draft verification at a 64K prefix; a failure here is reported in the line, not raised, and every
        # rank takes the same collective step either way
        tree, t_tree, err = None, float("nan"), None
        try:
            tree = TreeBench()
            t_tree = tree.run(10, 1000)
        except Exception as e:  # noqa: BLE001
            err = f"{type(e).__name__}: {e}"[:300]
        t_tree = barrier_max(t_tree, ws)
        if err is None and t_tree == t_tree:
            tb, tkeys = tree.bytes_per_pass()
            line["tree_verify"] = {
                "workload": "tree_verify_64k", "value": whole_job_rate(tree.N, ws, t_tree), "unit": UNIT,
                "us_per_pass": t_tree * 1e6, "passes": 1000, "timing": "median of 1000 passes, L2 flushed before each",
                "algorithmic_bytes": tb, "attended_prefix_keys": tkeys, "achieved_gbs": tb / t_tree / 1e9,
                "frac_of_" + peak_kind: tb / t_tree / 1e9 / peaks["hbm_gbs"],
                "note": "one pass = block_score_topk of the 16 draft queries + sparse_attn_tree_verify",
            }
        else:
            line["tree_verify"] = {"workload": "tree_verify_64k", "error": err or "no time"}
        del tree
        torch.cuda.empty_cache()

    if not args.no_paged:
        # the 128K decode step on a paged cache (reported, not raised; same collective steps on every rank)
        pg, tp, tc, err = None, float("nan"), float("nan"), None
        try:
            pg = PagedDecodeBench()
            tp = pg.run(pg.step_paged, 10, 300)
            tc = pg.run(pg.step_contiguous, 10, 300)
        except Exception as e:  # noqa: BLE001
            err = f"{type(e).__name__}: {e}"[:300]
        tp, tc = barrier_max(tp, ws), barrier_max(tc, ws)
        if err is None and tp == tp:
            _, _, bp = decode_step_bytes([int(n) for n in pg.lens_h])
            line["paged_decode"] = {
                "workload": "decode_128k_ragged step 0 on 64-position pages (shuffled page table)",
                "value": whole_job_rate(len(pg.lens_h), ws, tp), "unit": UNIT, "us_per_step": tp * 1e6,
                "seq_lens": [int(n) for n in pg.lens_h],
                "contiguous_us_per_step": tc * 1e6, "timing": "median of 300 steps, L2 flushed before each",
                "algorithmic_bytes": bp, "frac_of_" + peak_kind: bp / tp / 1e9 / peaks["hbm_gbs"],
                "note": "one step = kernel_pool_paged of the new key + sparse_decode_step_paged",
            }
        else:
            line["paged_decode"] = {"workload": "decode_128k_ragged paged", "error": err or "no time"}
        del pg
        torch.cuda.empty_cache()
        vb, tv, t1, err = None, float("nan"), float("nan"), None
        try:
            vb = VarlenPrefillBench()
            tv = vb.run(vb.packed, 1, 3)
            t1 = vb.run(vb.one_by_one, 1, 3)
        except Exception as e:  # noqa: BLE001
            err = f"{type(e).__name__}: {e}"[:300]
        tv, t1 = barrier_max(tv, ws), barrier_max(t1, ws)
        if err is None and tv == tv:
            line["varlen_prefill"] = {
                "workload": "packed prefill of 4 sequences, T = L = 32768 + 16384 + 8192 + 4096",
                "value": whole_job_rate(vb.T, ws, tv), "unit": UNIT, "ms_per_pass": tv * 1e3,
                "one_sequence_at_a_time_ms": t1 * 1e3, "timing": "mean of 3 passes",
                "note": "one pass = infllmv2_sparse_prefill_varlen (3 launches for the batch)",
            }
        else:
            line["varlen_prefill"] = {"workload": "packed prefill", "error": err or "no time"}
        del vb
        torch.cuda.empty_cache()

    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 oracle on the host cores: each step a bounded sample of the decode workload (sequences
    processed per step chosen so the whole run stays within a few minutes)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    # granularity: one (sequence, group) row per step, or more when the step count leaves time for it
    probe = OracleDecode([0], [0])
    probe.step(0)
    t0 = time.perf_counter()
    probe.step(1)
    t_row = time.perf_counter() - t0
    budget = 150.0
    rows = int(max(1, min(len(LENS_128K) * HKV, budget / max(1, args.steps + args.warmup) / max(t_row, 1e-3))))
    if rows >= HKV:
        od = OracleDecode(range(rows // HKV))
    else:
        od = probe
    nrows = len(od.seqs) * len(od.groups)
    for s in range(args.warmup):
        od.step(s)
    t0 = time.perf_counter()
    tok = 0.0
    for s in range(args.steps):
        tok += od.step(s)
    dt = time.perf_counter() - t0
    value = tok / dt
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": "decode_128k_ragged", "batch": 4, "ctx_lens_step0": list(LENS_128K),
                   "heads_q_kv": [HQ, HKV], "head_dim": D, "topk": 64, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(oracle.num_threads(), nrows), "kind": "oracle",
                         "sample": f"each step: one decode step of {nrows} (sequence, KV group) row(s) of the 4 x 2 "
                                   f"rows of the 128K batch; a token counts once both groups of its sequence are done"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--decode-path", choices=["two_call", "fused", "fused_pool"], default="fused_pool",
                    help="decode step as kernel_pool + block_score_topk + sparse_attn_decode, kernel_pool + "
                         "sparse_decode_step, or the one-launch sparse_decode_step_pool")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the prefill gradient pass")
    ap.add_argument("--no-lse-estimate", action="store_true", help="skip the LSE-estimate scoring leg")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged-decode and packed-prefill legs")
    ap.add_argument("--no-tree", action="store_true", help="skip the tree-verification leg")
    ap.add_argument("--no-decode32k", action="store_true", help="skip the batch-1 32K decode leg")
    ap.add_argument("--no-decode", action="store_true", help="prefill only (for profiling its kernels)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-e2e", dest="e2e", action="store_false", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-per-call", dest="per_call", action="store_false", help="skip per-call event timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
