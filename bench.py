#!/usr/bin/env python
"""Benchmark of the paged KV-cache hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:

* decode: the ragged batch (64 sequences, lengths U[1, 8192], 32/8 heads,
  head_dim 128, bf16, block 16, 40000-block pool, sliding window 4096 on even
  sequences): append one token per sequence, then paged decode (main kernel +
  log-sum-exp combine). Lengths grow by one per step; a sequence takes a new
  block from the shuffled free list when it crosses a block edge.
* prefill: 4 sequences with 30720 cached tokens plus a 2048-token chunk,
  causal: append the chunk through its slot mapping, then paged prefill.

``value`` is decode KV bytes per second (the metric's first part); the
prefill half is reported in the ``prefill`` object. Inputs are resident in
HBM when the device-timed region starts; ``e2e`` repeats the same interleaved
steps through the public API with pinned host buffers: every step copies its
inputs in and its results out inside the timed region, on side streams, so
that a step's copies overlap the kernels next to it.

``--impl reference`` times the float64 CPU oracle (the only reference this
method has) on a bounded sample of the same workload.
"""

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode KV GB/s (frac of HBM peak); paged prefill TFLOP/s (frac of bf16 peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ profiled traffic

# DRAM bytes (read + write) per unit of work, from one ncu capture of each
# kernel (decode: one launch on the full ragged batch; prefill: one launch on
# one of the four long-context sequences; the committed ncu summaries); a full
# launch scales it by its units. Valid only for the kernel code it was taken on: after
# any change to that code (comments aside) the bench reports null until the
# kernels are profiled again.
PROFILED_TRAFFIC = {
    "decode": {"sources": ['csrc/decode.cu', 'csrc/pkv_common.cuh'],
               "code_sha256": "359451da6cfdd4e078767c6a8414b2d2c85eed5e4fb0176a917bda3e068e1b80",
               # per algorithmic byte: one launch of the fused decode step on the full
               # ragged batch (862692096 B read + 4321792 B written for 860911968 B)
               "per_unit": (862692096 + 4321792) / 860911968,
               },
    "prefill": {"sources": ['csrc/prefill.cu', 'csrc/prefill_common.cuh', 'csrc/pkv_common.cuh',
                            'csrc/tc_sm100.cuh'],
                "code_sha256": "cc231aef4686aba1481fecaf71ca60bc396ce4bf41b59ad77a25f4d4fe2bcc5f",
                # per causal FLOP: one launch on one long-context sequence
                "per_unit": (165521152 + 13004032) / 1065168666624,
                },
}


def code_hash(sources):
    """sha256 of the kernel sources with comments and blank lines removed, so
    that an edit of a comment keeps the recorded counters while any change of
    code drops them (the sources hold no comment markers inside strings)."""
    import hashlib
    import re

    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "paged_kv_cache_gather_b200", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()


def profiled_traffic(kind, units):
    rec = PROFILED_TRAFFIC[kind]
    if code_hash(rec["sources"]) != rec["code_sha256"]:
        return None
    return int(rec["per_unit"] * units)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ workloads

def decode_plan(case, steps):
    """Per-step lengths and append slots for `steps` decode steps; the table
    gets the blocks the growth will need (entries past a sequence's length
    are ignored by the kernels)."""
    bs = case.block_size
    tab = case.block_tables.numpy().copy()
    free = case.extra["free_list"]
    nxt = case.extra["blocks_used"]
    lens0 = case.seq_lens.numpy().astype(np.int64)
    nalloc = [(int(L) + bs - 1) // bs for L in lens0]
    lens = np.zeros((steps, case.batch), dtype=np.int32)
    slots = np.zeros((steps, case.batch), dtype=np.int64)
    for s in range(steps):
        for b in range(case.batch):
            L = int(lens0[b]) + s
            p = L - 1
            j = p // bs
            if j >= nalloc[b]:
                tab[b, j] = free[nxt]
                nxt += 1
                nalloc[b] = j + 1
            lens[s, b] = L
            slots[s, b] = int(tab[b, j]) * bs + p % bs
    return torch.from_numpy(tab), torch.from_numpy(lens), torch.from_numpy(slots)


def causal_pairs(ctx_lens, q_lens):
    """(query, key) pairs a causal chunked prefill computes: chunk row i of a
    sequence with C cached tokens sees C + i + 1 keys."""
    C = np.asarray(ctx_lens, dtype=np.int64)
    Q = np.asarray(q_lens, dtype=np.int64)
    return int((Q * C + Q * (Q + 1) // 2).sum())


def document_pairs(ctx_lens, q_lens, doc_offsets, doc_starts):
    """Pairs a chunked prefill computes under the document mask: chunk row at
    position p sees the keys from the start of its document to p (every
    sequence's first document starts at 0)."""
    pairs = 0
    for b, (c, q) in enumerate(zip(ctx_lens, q_lens)):
        starts = np.sort(np.asarray(doc_starts)[doc_offsets[b]:doc_offsets[b + 1]])
        qpos = int(c) + np.arange(int(q))
        ds = starts[np.searchsorted(starts, qpos, side="right") - 1]
        pairs += int((qpos - ds + 1).sum())
    return pairs


def prefix_lm_pairs(ctx_lens, q_lens, prefix_len):
    """Pairs under the prefix-LM mask (prefix_len <= C + Q): chunk row at
    position p sees max(p + 1, prefix_len) keys."""
    return int(sum(np.maximum(int(c) + np.arange(int(q)) + 1, int(pl)).sum()
                   for c, q, pl in zip(ctx_lens, q_lens, prefix_len)))


def visible_tokens(lens, wps):
    lens = np.asarray(lens, dtype=np.int64)
    w = np.asarray(wps, dtype=np.int64)
    return np.where(w > 0, np.minimum(lens, w), lens)


class DecodeWork:
    """The ragged decode batch, resident on the device."""

    def __init__(self, dev, steps, seed, batch=64, num_blocks=40000):
        from paged_kv_cache_gather_b200 import inputs as I

        self.case = I.config3(batch=batch, num_blocks=num_blocks, seed=seed,
                              growth_steps=steps + 1)
        c = self.case
        tab, lens, slots = decode_plan(c, steps)
        gen = torch.Generator().manual_seed(seed + 100)
        B, Hq, Hkv, D = c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim
        self.q_h = I.randn((steps, B, Hq, D), gen).pin_memory()
        self.kn_h = I.randn((steps, B, Hkv, D), gen).pin_memory()
        self.vn_h = I.randn((steps, B, Hkv, D), gen).pin_memory()
        self.lens_h = lens.pin_memory()
        self.slots_h = slots.pin_memory()
        self.tab_h = tab.pin_memory()
        self.k_cache = c.k_cache.to(dev)
        self.v_cache = c.v_cache.to(dev)
        self.tab = tab.to(dev)
        self.lens = lens.to(dev)
        self.slots = slots.to(dev)
        self.q = self.q_h.to(dev)
        self.kn = self.kn_h.to(dev)
        self.vn = self.vn_h.to(dev)
        self.wps = c.window_per_seq.to(dev)
        self.out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
        import paged_kv_cache_gather_b200 as pkv

        self.pkv = pkv
        self.ws = pkv.decode_workspace(B, Hq, self.k_cache)
        self.mask = pkv.sliding_window(self.wps)
        vis = visible_tokens(lens.numpy(), c.window_per_seq.numpy())  # [steps, B]
        self.kv_bytes = vis.sum(axis=1) * Hkv * D * 2 * 2  # K and V, bf16
        self.io_bytes = B * Hq * D * 2 * 2 + B * Hq * 4 + ((vis + 15) // 16).sum(1) * Hkv * 4
        self.append_bytes = B * Hkv * D * 2 * 2 * 2  # new K and V rows read and written
        # end-to-end steps: one host->device copy of every input of a step (packed
        # into one pinned buffer per step) and one device->host copy of out + lse
        # (the fused call finds each new token's slot from the table: no slots)
        parts = [("q", self.q_h[0]), ("kn", self.kn_h[0]), ("vn", self.vn_h[0]),
                 ("lens", self.lens_h[0]), ("tab", self.tab_h)]
        self.layout, off = {}, 0
        for name, t in parts:
            nbytes = t.numel() * t.element_size()
            self.layout[name] = (off, nbytes, t.dtype, tuple(t.shape))
            off += (nbytes + 255) // 256 * 256
        self.pack_h = torch.empty(steps, off, dtype=torch.uint8).pin_memory()
        for st in range(steps):
            for name, t in (("q", self.q_h[st]), ("kn", self.kn_h[st]), ("vn", self.vn_h[st]),
                            ("lens", self.lens_h[st]), ("tab", self.tab_h)):
                o, nb, _, _ = self.layout[name]
                self.pack_h[st, o:o + nb] = t.contiguous().view(torch.uint8).view(-1)
        # two device copies of the packed inputs and of the packed results, so
        # that one step's copies overlap the neighbouring steps' kernels
        self.pack_d = [torch.empty(off, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.views = [{name: pd[o:o + nb].view(dt).view(shape)
                       for name, (o, nb, dt, shape) in self.layout.items()}
                      for pd in self.pack_d]
        ob = self.out.numel() * 2
        lo = (ob + 255) // 256 * 256
        rb = lo + self.lse.numel() * 4
        self.res_d = [torch.empty(rb, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.res_h = [torch.empty(rb, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.out_e = [r[:ob].view(torch.bfloat16).view(B, Hq, D) for r in self.res_d]
        self.lse_e = [r[lo:rb].view(torch.float32).view(B, Hq) for r in self.res_d]
        self.h2d = self.pack_h.shape[1]   # bytes actually copied per step (with alignment pads)
        self.d2h = rb

    def step(self, s):
        """One decode step in one call: append each sequence's new token at its
        next position and decode (the fused entry point)."""
        self.pkv.paged_attention_decode_append(self.q[s], self.kn[s], self.vn[s], self.k_cache,
                                               self.v_cache, self.tab, self.lens[s],
                                               self.case.scale, self.mask, out=self.out,
                                               lse=self.lse, workspace=self.ws)

    def append(self, s):
        self.pkv.paged_kv_append(self.kn[s], self.vn[s], self.slots[s], self.k_cache, self.v_cache)

    def decode(self, s):
        self.pkv.paged_attention_decode(self.q[s], self.k_cache, self.v_cache, self.tab,
                                        self.lens[s], self.case.scale, self.mask, out=self.out,
                                        lse=self.lse, workspace=self.ws)

    # end-to-end step s through device buffer b: inputs in, kernels, results out
    def e2e_in(self, s, b):
        self.pack_d[b].copy_(self.pack_h[s], non_blocking=True)

    def e2e_run(self, s, b):
        v = self.views[b]
        self.pkv.paged_attention_decode_append(v["q"], v["kn"], v["vn"], self.k_cache,
                                               self.v_cache, v["tab"], v["lens"], self.case.scale,
                                               self.mask, out=self.out_e[b], lse=self.lse_e[b],
                                               workspace=self.ws)

    def e2e_out(self, b):
        self.res_h[b].copy_(self.res_d[b], non_blocking=True)


def two_call_steps(dw, pw, step_ids, stream):
    """The same decode steps as two calls (paged_kv_append, then
    paged_attention_decode), for comparison with the fused call, interleaved
    with the prefill steps as in the timed region (so L2 starts each decode
    step in the same state); rewrites the same slots with the same values, so
    the caches end as before."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    a, b, c = [ev() for _ in step_ids], [ev() for _ in step_ids], [ev() for _ in step_ids]
    torch.cuda.synchronize()
    for i, s in enumerate(step_ids):
        a[i].record(stream)
        dw.append(s)
        b[i].record(stream)
        dw.decode(s)
        c[i].record(stream)
        if pw:
            pw.append()
            pw.prefill()
    torch.cuda.synchronize()
    n = len(step_ids)
    app = sum(a[i].elapsed_time(b[i]) for i in range(n)) / n
    dec = sum(b[i].elapsed_time(c[i]) for i in range(n)) / n
    kv = float(sum(dw.kv_bytes[s] for s in step_ids)) / n
    return {"append_ms": round(app, 4), "decode_ms": round(dec, 4),
            "ms_per_step": round(app + dec, 4),
            "kv_GBps": round(kv / ((app + dec) * 1e-3) / 1e9, 1)}


class PrefillWork:
    """The long-context chunked prefill batch, resident on the device."""

    def __init__(self, dev, seed, batch=4):
        import paged_kv_cache_gather_b200 as pkv
        from paged_kv_cache_gather_b200 import inputs as I

        self.pkv = pkv
        self.case = c = I.config5(batch=batch, seed=seed)
        self.k_cache = c.k_cache.to(dev)
        self.v_cache = c.v_cache.to(dev)
        self.tab = c.block_tables.to(dev)
        self.ctx = c.ctx_lens.to(dev)
        self.ql = c.q_lens.to(dev)
        self.q = c.q.to(dev)
        self.kn = c.k_new.to(dev)
        self.vn = c.v_new.to(dev)
        self.slots = c.slot_mapping.to(dev)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[0], self.q.shape[1], dtype=torch.float32, device=dev)
        self.mask = pkv.causal()
        # end-to-end steps: the inputs packed in one pinned host buffer (one
        # host->device copy per step) and out + lse in one device->host copy;
        # two device copies of each so that copies overlap the neighbouring steps
        parts = [("q", c.q), ("kn", c.k_new), ("vn", c.v_new), ("slots", c.slot_mapping)]
        layout, off = {}, 0
        for name, t in parts:
            nbytes = t.numel() * t.element_size()
            layout[name] = (off, nbytes, t.dtype, tuple(t.shape))
            off += (nbytes + 255) // 256 * 256
        self.pack_h = torch.empty(off, dtype=torch.uint8).pin_memory()
        for name, t in parts:
            o, nb, _, _ = layout[name]
            self.pack_h[o:o + nb] = t.contiguous().view(torch.uint8).view(-1)
        self.pack_d = [torch.empty(off, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.views = [{name: pd[o:o + nb].view(dt).view(shape)
                       for name, (o, nb, dt, shape) in layout.items()} for pd in self.pack_d]
        ob = self.out.numel() * 2
        lo = (ob + 255) // 256 * 256
        rb = lo + self.lse.numel() * 4
        self.res_d = [torch.empty(rb, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.res_h = [torch.empty(rb, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.out_e = [r[:ob].view(torch.bfloat16).view(self.out.shape) for r in self.res_d]
        self.lse_e = [r[lo:rb].view(torch.float32).view(self.lse.shape) for r in self.res_d]
        C = c.ctx_lens.numpy().astype(np.int64)
        Q = c.q_lens.numpy().astype(np.int64)
        self.flops = float(4 * c.head_dim * causal_pairs(C, Q) * c.num_q_heads)
        self.h2d = off   # bytes actually copied per step (with alignment pads)
        self.d2h = rb

    def append(self):
        self.pkv.paged_kv_append(self.kn, self.vn, self.slots, self.k_cache, self.v_cache)

    def prefill(self):
        self.pkv.paged_attention_prefill(self.q, self.kn, self.vn, self.k_cache, self.v_cache,
                                         self.tab, self.ctx, self.ql, self.mask,
                                         out=self.out, lse=self.lse)

    def e2e_in(self, s, b):
        self.pack_d[b].copy_(self.pack_h, non_blocking=True)

    def e2e_run(self, s, b):
        v = self.views[b]
        self.pkv.paged_kv_append(v["kn"], v["vn"], v["slots"], self.k_cache, self.v_cache)
        self.pkv.paged_attention_prefill(v["q"], v["kn"], v["vn"], self.k_cache, self.v_cache,
                                         self.tab, self.ctx, self.ql, self.mask,
                                         out=self.out_e[b], lse=self.lse_e[b])

    def e2e_out(self, b):
        self.res_h[b].copy_(self.res_d[b], non_blocking=True)


def run_e2e(works, step_ids, stream):
    """End-to-end steps through the public API, interleaved like the
    device-timed steps (each step runs every work in `works` in turn). Every
    work's step copies its inputs from pinned host memory to the device (one
    copy), runs its kernels, and copies its results back (one copy). Copies run
    on two side streams and step i uses device buffer i % 2, so the next
    inputs arrive and the previous results leave while kernels run; events
    order each buffer's reuse. Returns each work's device time in ms (CUDA
    events on `stream`): from the point where the compute stream starts
    waiting for that work's inputs to the end of its kernels, so a copy that
    is not hidden is charged to its own work; the final copies out are charged
    to the last work."""
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    tev = lambda: torch.cuda.Event(enable_timing=True)
    K = len(works)
    marks = []
    h2d.wait_stream(stream)
    d2h.wait_stream(stream)
    ran = [[None, None] for _ in range(K)]
    copied_in = [[None, None] for _ in range(K)]
    copied_out = [[None, None] for _ in range(K)]
    for i, s in enumerate(step_ids):
        b = i % 2
        for k, work in enumerate(works):
            with torch.cuda.stream(h2d):
                if ran[k][b] is not None:
                    h2d.wait_event(ran[k][b])          # step i-2 no longer reads buffer b
                work.e2e_in(s, b)
                copied_in[k][b] = ev()
                copied_in[k][b].record(h2d)
            m = tev()
            m.record(stream)
            marks.append((k, m))
            stream.wait_event(copied_in[k][b])
            if copied_out[k][b] is not None:
                stream.wait_event(copied_out[k][b])    # step i-2's results have left buffer b
            with torch.cuda.stream(stream):
                work.e2e_run(s, b)
            ran[k][b] = ev()
            ran[k][b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ran[k][b])
                work.e2e_out(b)
                copied_out[k][b] = ev()
                copied_out[k][b].record(d2h)
    stream.wait_stream(h2d)
    stream.wait_stream(d2h)
    end = tev()
    end.record(stream)
    torch.cuda.synchronize()
    ms = [0.0] * K
    for j, (k, m) in enumerate(marks):
        nxt = marks[j + 1][1] if j + 1 < len(marks) else end
        ms[k] += m.elapsed_time(nxt)
    return ms


# ------------------------------------------------------------------ side measurements

def l2_flush_buffer(dev):
    return torch.empty(256 << 20, dtype=torch.uint8, device=dev)


def time_calls(fn, n, flush=None, stream=None):
    """Mean device time of fn() over n calls (CUDA events on the launching
    stream); when `flush` is given it is overwritten before every call, outside
    the event pair, so each call starts with a cold L2."""
    stream = stream or torch.cuda.current_stream()
    ts = []
    for _ in range(n):
        if flush is not None:
            flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return sum(ts) / len(ts)


def decode_sweep(dev, flush):
    """Batch-1 decode over 128..4096 tokens (32/8 heads, d 128, causal), the
    shape of the pages' sequence-length sweep: microseconds per call with a cold
    L2, eagerly and as a replayed CUDA graph, and the 2048/128 latency ratio."""
    import paged_kv_cache_gather_b200 as pkv
    from paged_kv_cache_gather_b200 import inputs as I

    base = I.config2(4096)
    kc, vc = base.k_cache.to(dev), base.v_cache.to(dev)
    q = base.q.to(dev)
    res = {}
    for L in I.CONFIG2_LENGTHS:
        tab = base.block_tables[:, : L // 16].contiguous().to(dev)
        lens = torch.tensor([L], dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        lse = torch.empty(1, 32, dtype=torch.float32, device=dev)
        ws = pkv.decode_workspace(1, 32, kc)
        mask = pkv.causal()
        call = lambda: pkv.paged_attention_decode(q, kc, vc, tab, lens, base.scale, mask,
                                                  out=out, lse=lse, workspace=ws)
        for _ in range(3):
            call()
        eager = time_calls(call, 20, flush)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            call()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        graph = time_calls(g.replay, 20, flush)
        kv = L * 8 * 128 * 2 * 2
        res[str(L)] = {"us_eager": round(eager * 1e3, 2), "us_graph": round(graph * 1e3, 2),
                       "kv_GBps_graph": round(kv / (graph * 1e-3) / 1e9, 1)}
    res["latency_ratio_2048_over_128"] = round(res["2048"]["us_graph"] / res["128"]["us_graph"], 2)
    res["pages_ratio_on_L4"] = "about 2x, end to end in a model (context only)"
    return res


def shared_prefix(dev, flush):
    """8 groups x 8 beams, 4096-token prefix shared by block id + 256 own tokens:
    plain decode time with shared blocks and with copied ones, and the grouped
    (shared-prefix) call on the shared layout; logical bytes are what the beams
    attend over, unique bytes what is stored."""
    import paged_kv_cache_gather_b200 as pkv
    from paged_kv_cache_gather_b200 import inputs as I

    out = {}
    for shared in (True, False):
        c = I.config4(shared=shared)
        kc, vc = c.k_cache.to(dev), c.v_cache.to(dev)
        q, tab, lens = c.q.to(dev), c.block_tables.to(dev), c.seq_lens.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=dev)
        ws = pkv.decode_workspace(q.shape[0], q.shape[1], kc)
        call = lambda: pkv.paged_attention_decode(q, kc, vc, tab, lens, c.scale, pkv.causal(),
                                                  out=o, lse=lse, workspace=ws)
        for _ in range(3):
            call()
        ms = time_calls(call, 20, flush)
        logical = 64 * 4352 * 8 * 128 * 2 * 2
        unique = c.extra["unique_blocks"] * 8 * 16 * 128 * 2 * 2
        out["shared" if shared else "copied"] = {
            "us": round(ms * 1e3, 2), "logical_GBps": round(logical / (ms * 1e-3) / 1e9, 1),
            "unique_bytes": unique, "unique_GBps": round(unique / (ms * 1e-3) / 1e9, 1)}
        if shared:
            # the grouped call: prefix once per (group, KV head), own keys, merge
            gs = c.extra["group_start"].to(dev)
            sl = c.extra["shared_len"].to(dev)
            wsg = pkv.shared_prefix_workspace(q.shape[0], q.shape[1], kc)
            grouped = lambda: pkv.paged_attention_decode_shared_prefix(
                q, kc, vc, tab, lens, gs, sl, c.extra["max_group_size"], c.scale, pkv.causal(),
                out=o, lse=lse, workspace=wsg)
            for _ in range(3):
                grouped()
            ms_g = time_calls(grouped, 20, flush)
            out["grouped"] = {
                "us": round(ms_g * 1e3, 2),
                "logical_GBps": round(logical / (ms_g * 1e-3) / 1e9, 1),
                "unique_GBps": round(unique / (ms_g * 1e-3) / 1e9, 1),
                "launches": 2}
        del kc, vc
        torch.cuda.empty_cache()
    out["grouped_speedup_vs_shared"] = round(out["shared"]["us"] / out["grouped"]["us"], 2)
    return out


def shared_prefix_only(args, dev, rank):
    """The grouped (shared-prefix) decode of the beams workload alone, cold L2
    before every call: warm-up calls, then timed calls; prints one JSON line."""
    import paged_kv_cache_gather_b200 as pkv
    from paged_kv_cache_gather_b200 import inputs as I

    c = I.config4(shared=True)
    kc, vc = c.k_cache.to(dev), c.v_cache.to(dev)
    q, tab, lens = c.q.to(dev), c.block_tables.to(dev), c.seq_lens.to(dev)
    gs, sl = c.extra["group_start"].to(dev), c.extra["shared_len"].to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=dev)
    ws = pkv.shared_prefix_workspace(q.shape[0], q.shape[1], kc)
    call = lambda: pkv.paged_attention_decode_shared_prefix(
        q, kc, vc, tab, lens, gs, sl, c.extra["max_group_size"], c.scale, pkv.causal(),
        out=o, lse=lse, workspace=ws)
    for _ in range(args.warmup):
        call()
    flush = l2_flush_buffer(dev)
    ms = time_calls(call, args.steps, flush)
    unique = c.extra["unique_blocks"] * 8 * 16 * 128 * 2 * 2
    if rank == 0:
        print(json.dumps({"workload": "shared-prefix beams (8 groups x 8 beams, 4096 shared + "
                                      "256 own tokens, 32/8 heads, d128, bf16)",
                          "us_per_call": round(ms * 1e3, 2), "unique_bytes": unique,
                          "unique_GBps": round(unique / (ms * 1e-3) / 1e9, 1),
                          "steps": args.steps, "warmup": args.warmup}))


def mask_modifiers(dev, d=None):
    """Throughput under the further mask modifiers: the long-context prefill with
    packed documents (mean 4096 tokens) and with a prefix-LM prefix covering half
    the chunk (FLOPs of visible pairs only), and the ragged decode batch with
    per-head windows (4096 on even heads, none on odd; bytes of the keys read)."""
    import paged_kv_cache_gather_b200 as pkv
    from paged_kv_cache_gather_b200 import inputs as I

    res = {}
    pw = PrefillWork(dev, 1239)
    c = pw.case
    C = c.ctx_lens.numpy().astype(np.int64)
    Q = c.q_lens.numpy().astype(np.int64)
    off, st = I.document_starts((C + Q).tolist(), 77, mean_doc=4096)
    pairs = document_pairs(C, Q, off.numpy(), st.numpy())
    pw.mask = pkv.document(off.to(dev), st.to(dev))
    pw.prefill()
    ms = time_calls(pw.prefill, 5)
    fl = 4.0 * c.head_dim * pairs * c.num_q_heads
    res["prefill_documents"] = {"ms": round(ms, 3), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                                "visible_pairs_per_head": pairs,
                                "documents": int(off[-1].item())}
    plen = C + Q // 2
    pairs = prefix_lm_pairs(C, Q, plen)
    pw.mask = pkv.prefix_lm(torch.from_numpy(plen.astype(np.int32)).to(dev))
    pw.prefill()
    ms = time_calls(pw.prefill, 5)
    fl = 4.0 * c.head_dim * pairs * c.num_q_heads
    res["prefill_prefix_lm"] = {"ms": round(ms, 3), "tflops": round(fl / (ms * 1e-3) / 1e12, 1)}
    del pw
    torch.cuda.empty_cache()
    d = d if d is not None else I.config3()
    kc, vc = d.k_cache.to(dev), d.v_cache.to(dev)
    q, tab, lens = d.q.to(dev), d.block_tables.to(dev), d.seq_lens.to(dev)
    wph = torch.tensor([4096 if h % 2 == 0 else 0 for h in range(d.num_q_heads)],
                       dtype=torch.int32, device=dev)
    ws = pkv.decode_workspace(q.shape[0], q.shape[1], kc)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=dev)
    mm = pkv.sliding_window(0, per_head=wph)
    call = lambda: pkv.paged_attention_decode(q, kc, vc, tab, lens, d.scale, mm, out=o, lse=lse,
                                              workspace=ws)
    call()
    ms = time_calls(call, 20)
    nbytes = int(d.seq_lens.numpy().astype(np.int64).sum()) * d.num_kv_heads * d.head_dim * 4
    res["decode_per_head_windows"] = {"us": round(ms * 1e3, 1),
                                      "GBps": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    return res


def fp8_decode(dev, d, n=20, warm=1):
    """The ragged decode batch on E4M3 pools: pools written by the quantising
    append from the bf16 pools, then decode timed (20 calls, inputs > L2).
    Reports the bytes read (codes + row scales) and the bf16-equivalent rate."""
    import paged_kv_cache_gather_b200 as pkv

    NB, Hkv, bs, D = d.k_cache.shape
    kc = torch.empty(NB, Hkv, bs, D, dtype=torch.uint8, device=dev)
    vc = torch.empty_like(kc)
    ks = torch.empty(NB, Hkv, bs, dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)
    step = 4096  # blocks per append call
    for b0 in range(0, NB, step):
        b1 = min(NB, b0 + step)
        rows_k = d.k_cache[b0:b1].to(dev).permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        rows_v = d.v_cache[b0:b1].to(dev).permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        slots = torch.arange(b0 * bs, b1 * bs, dtype=torch.int64, device=dev)
        pkv.paged_kv_append_fp8(rows_k, rows_v, slots, kc, vc, ks, vs)
    q, tab, lens = d.q.to(dev), d.block_tables.to(dev), d.seq_lens.to(dev)
    wps = d.window_per_seq.to(dev)
    mm = pkv.sliding_window(wps)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=dev)
    ws = pkv.decode_workspace(q.shape[0], q.shape[1], kc)
    call = lambda: pkv.paged_attention_decode_fp8(q, kc, vc, ks, vs, tab, lens, d.scale, mm,
                                                  out=o, lse=lse, workspace=ws)
    for _ in range(warm):
        call()
    ms = time_calls(call, n)
    vis = int(visible_tokens(d.seq_lens.numpy(), d.window_per_seq.numpy()).sum())
    fp8_bytes = vis * Hkv * 2 * (D + 4)
    bf16_bytes = vis * Hkv * 2 * D * 2
    return {"us": round(ms * 1e3, 1), "bytes_read": fp8_bytes,
            "GBps_read": round(fp8_bytes / (ms * 1e-3) / 1e9, 1),
            "bf16_equivalent_GBps": round(bf16_bytes / (ms * 1e-3) / 1e9, 1),
            "workload": "ragged decode batch (64 seqs, window 4096 on even), E4M3 pools"}


def device_growth(dev, d=None):
    """Device-side growth of the ragged decode batch (64 sequences, one token each):
    the reserve call alone, and a whole step (reserve + append + decode) eager and
    replayed from one CUDA graph."""
    import paged_kv_cache_gather_b200 as pkv
    from paged_kv_cache_gather_b200 import BlockManager
    from paged_kv_cache_gather_b200 import inputs as I

    d = d if d is not None else I.config3()
    mgr = BlockManager(d.num_blocks, d.block_size, seed=3)
    ids = list(range(d.batch))
    for b, L in enumerate(d.seq_lens.tolist()):
        mgr.add_sequence(b, L - 1)
    width = d.block_tables.shape[1] + 8  # room for the ~70 steps taken here
    tab = mgr.block_table_tensor(ids, width).to(dev)
    lens = mgr.seq_lens_tensor(ids).to(dev)
    pool = pkv.DevicePool.from_manager(mgr, dev)
    kc, vc = d.k_cache.to(dev), d.v_cache.to(dev)
    B = d.batch
    one = torch.ones(B, dtype=torch.int32, device=dev)
    kn, vn = d.k_new.to(dev), d.v_new.to(dev)
    q = d.q.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, q.shape[1], dtype=torch.float32, device=dev)
    ws = pkv.decode_workspace(B, q.shape[1], kc)

    def reserve():
        return pkv.paged_kv_reserve_slots(kc, vc, tab, lens, one, pool, B)[0]

    def step():
        slots = reserve()
        pkv.paged_kv_append(kn, vn, slots, kc, vc)
        pkv.paged_attention_decode(q, kc, vc, tab, lens, d.scale, pkv.causal(), out=o,
                                   lse=lse, workspace=ws)

    step()
    us_res = time_calls(reserve, 20) * 1e3
    us_eager = time_calls(step, 20) * 1e3
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    us_graph = time_calls(g.replay, 20) * 1e3
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g2, stream=s):
            reserve()
    torch.cuda.current_stream().wait_stream(s)
    us_res_graph = time_calls(g2.replay, 20) * 1e3
    del g, g2
    return {"reserve_eager_us": round(us_res, 2), "reserve_graph_us": round(us_res_graph, 2),
            "step_eager_us": round(us_eager, 1), "step_graph_us": round(us_graph, 1),
            "batch": B, "free_blocks_left": int(pool.free_top.item()),
            "note": "eager times include the Python binding's launch overhead"}


# ------------------------------------------------------------------ CPU baseline

def oracle_decode_sample(budget_s=12.0, seed=None):
    """Times the float64 oracle on whole decode steps of the ragged batch
    (all 64 sequences, 32 heads) until `budget_s` has passed."""
    import oracle
    from paged_kv_cache_gather_b200 import inputs as I

    c = I.config3(seed=seed)
    vis = visible_tokens(c.seq_lens.numpy(), c.window_per_seq.numpy())
    kv_bytes = float(vis.sum() * c.num_kv_heads * c.head_dim * 2 * 2)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.paged_decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale,
                            c.mask_kind, c.window, c.window_per_seq)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": kv_bytes * n / el / 1e9, "unit": "GB/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{n} full decode step(s) of the ragged batch (64 seqs, 32 heads), "
                      f"{el:.1f} s wall, float64 NumPy"}


def oracle_prefill_sample(budget_s=10.0):
    """Times the oracle on (sequence, head) slices of the prefill batch, scaled."""
    import oracle
    from paged_kv_cache_gather_b200 import inputs as I

    c = I.config5(batch=1)
    C, Q = int(c.ctx_lens[0]), int(c.q_lens[0])
    rows_per_slice = 64
    n, t0 = 0, time.perf_counter()
    while True:
        h = n % c.num_q_heads
        oracle.paged_prefill_rows(c.q, c.k_new, c.v_new, c.k_cache, c.v_cache, c.block_tables,
                                  c.ctx_lens, c.q_lens, c.scale, c.mask_kind,
                                  rows=[(0, h, i) for i in range(Q - rows_per_slice, Q)])
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    pairs = sum(C + i + 1 for i in range(Q - rows_per_slice, Q))
    flops = 4.0 * c.head_dim * pairs * n
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{n} slices of {rows_per_slice} query rows x ~32.7k keys (one head each) "
                      f"of the prefill batch, {el:.1f} s wall, float64 NumPy"}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas = 1
    return int(max(blas, 1))


# ------------------------------------------------------------------ main

def dist_setup(backend="nccl"):
    """One process per GPU (torchrun env vars); returns (world size, rank, local rank)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist

        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, ws, dev):
    if ws == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(with_prefill, ws):
    return {
        "workload": ("ragged batched decode (64 seqs, lengths U[1,8192] growing 1/step, 32/8 "
                     "heads, d128, bf16, block 16, 40000-block shuffled pool, window 4096 on even "
                     "seqs)" + (" + chunked prefill (4 x (30720 ctx + 2048 chunk), causal)"
                                if with_prefill else "")),
        "l2": "inputs larger than L2: 0.86 GB of KV per decode step, 537 MB per prefill step "
              "(126 MB L2), no flush",
        "parallelism": f"replicas x{ws} (independent batches, no collective)"}


def run_reference(args, ws, rank):
    """The float64 CPU oracle as it stands, on whole decode steps of the same
    ragged batch (one step = all 64 sequences x 32 heads)."""
    if rank != 0:
        return
    import oracle
    from paged_kv_cache_gather_b200 import inputs as I

    c = I.config3()
    vis = visible_tokens(c.seq_lens.numpy(), c.window_per_seq.numpy())
    per_step = 8  # sequences per reference step: a bounded sample, cycling through the batch
    done = {"bytes": 0.0}

    def step(k):
        seqs = [(8 * k + i) % c.batch for i in range(per_step)]
        rows = [(b, h) for b in seqs for h in range(c.num_q_heads)]
        oracle.paged_decode_rows(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale,
                                 c.mask_kind, c.window, c.window_per_seq, rows=rows)
        return float(vis[seqs].sum() * c.num_kv_heads * c.head_dim * 2 * 2)

    for k in range(args.warmup):
        step(k)
    t0 = time.perf_counter()
    total = 0.0
    for k in range(args.steps):
        total += step(args.warmup + k)
    el = time.perf_counter() - t0
    val = total / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3 / max(args.steps, 1), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.workload in ("all", "prefill"), 1),
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cpu_threads(),
                             "kind": "oracle",
                             "sample": "8 sequences x 32 heads of the ragged batch per step, "
                                       "cycling through the batch; float64 NumPy, inputs "
                                       "generated once"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all",
                    choices=["all", "decode", "prefill", "shared_prefix", "fp8_decode"],
                    help="shared_prefix / fp8_decode: only the grouped decode of the beams "
                         "workload / the ragged decode on E4M3 pools (side measurements, not "
                         "the bench line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the batch-1 sweep and the shared-prefix measurement")
    ap.add_argument("--small", action="store_true",
                    help="profiling size: 16 decode sequences in a 12000-block pool, one "
                         "prefill sequence (both still larger than L2); not a bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    ws, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, ws, rank)
        barrier(ws)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.workload == "shared_prefix":
        shared_prefix_only(args, dev, rank)
        barrier(ws)
        return
    if args.workload == "fp8_decode":
        from paged_kv_cache_gather_b200 import inputs as I
        res = fp8_decode(dev, I.config3(), n=args.steps, warm=args.warmup)
        if rank == 0:
            print(json.dumps(res))
        barrier(ws)
        return
    pk, pk_kind = peaks()
    total_steps = args.warmup + args.steps
    seed = 1237 + rank
    want_decode = args.workload in ("all", "decode")
    want_prefill = args.workload in ("all", "prefill")
    if args.small:
        dw = DecodeWork(dev, total_steps, seed, batch=16, num_blocks=12000) if want_decode else None
    else:
        dw = DecodeWork(dev, total_steps, seed) if want_decode else None
    pw = None
    prefill_reason = None
    if want_prefill:
        pw = PrefillWork(dev, 1239 + rank, batch=1 if args.small else 4)
        try:
            pw.append()
            pw.prefill()
            torch.cuda.synchronize()
        except Exception as e:  # the prefill kernel may not be built for this config
            prefill_reason = str(e).splitlines()[0]
            pw = None
    stream = torch.cuda.current_stream()

    # ---------------- device-timed region
    for s in range(args.warmup):
        if dw:
            dw.step(s)
        if pw:
            pw.append()
            pw.prefill()
    torch.cuda.synchronize()
    n = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)
    d0, d1, d2 = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
    p0, p1, p2 = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for i in range(n):
        s = args.warmup + i
        if dw:
            d0[i].record(stream)
            dw.step(s)
            d1[i].record(stream)
        if pw:
            p0[i].record(stream)
            pw.append()
            p1[i].record(stream)
            pw.prefill()
            p2[i].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), ws, dev)

    # ---------------- end-to-end region (host buffers, copies inside)
    step_ids = list(range(args.warmup, args.warmup + n))
    torch.cuda.synchronize()
    barrier(ws)
    works = [w for w in (dw, pw) if w is not None]
    e2e_ms_list = run_e2e(works, step_ids, stream)
    e2e_dec_ms = e2e_ms_list[0] if dw else None
    e2e_pre_ms = e2e_ms_list[-1] if pw else None
    barrier(ws)
    clk = clocks.stop()

    line = {"metric": METRIC, "n_gpus": ws, "steps": n, "warmup": args.warmup,
            "ms_per_step": round(ms_total / n, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    launches = 0
    if dw:
        step_ms = [d0[i].elapsed_time(d1[i]) for i in range(n)]
        steps_idx = range(args.warmup, args.warmup + n)
        kv = float(sum(dw.kv_bytes[s] for s in steps_idx))
        io = float(sum(dw.io_bytes[s] for s in steps_idx)) + n * dw.append_bytes
        dec_total_ms = max_over_ranks(sum(step_ms), ws, dev)
        # whole-job KV throughput of the decode steps (append fused into the
        # decode launch), all ranks
        value = kv * ws / (dec_total_ms * 1e-3) / 1e9
        achieved = (kv + io) / n / (dec_total_ms / n * 1e-3) / 1e9
        e2e_ms = max_over_ranks(e2e_dec_ms, ws, dev)
        line.update({
            "value": round(value, 2), "unit": "GB/s",
            "decode": {"ms_per_step": round(dec_total_ms / n, 4),
                       "call": "paged_attention_decode_append (append fused in the decode launch)",
                       "kv_bytes_per_step": int(kv / n),
                       "tokens_visible_per_step": int(kv / n / (8 * 128 * 4))},
            "roofline": {"kernel": "paged_attention_decode_append (main + merge)", "bound": "hbm",
                         "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / pk["hbm_gbs"], 4),
                         "peak_kind": pk_kind,
                         "traffic": profiled_traffic("decode", (kv + io) / n),
                         "bytes_per_launch": int((kv + io) / n)},
            "e2e": {"value": round(kv * ws / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": int(dw.h2d), "d2h_bytes_per_step": int(dw.d2h)},
        })
        launches += 2 * n
    if pw:
        pre_ms = [p1[i].elapsed_time(p2[i]) for i in range(n)]
        papp_ms = [p0[i].elapsed_time(p1[i]) for i in range(n)]
        pre_ms_t = max_over_ranks(sum(pre_ms), ws, dev)
        pstep_ms = max_over_ranks(sum(pre_ms) + sum(papp_ms), ws, dev)
        tf = pw.flops * n / (pre_ms_t * 1e-3) / 1e12
        pe2e = max_over_ranks(e2e_pre_ms, ws, dev)
        peak_tf = pk["bf16_tflops"]
        line["prefill"] = {
            "value": round(pw.flops * n * ws / (pstep_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(pstep_ms / n, 4), "prefill_ms": round(pre_ms_t / n, 4),
            "flops_per_step": pw.flops,
            "roofline": {"kernel": "paged_attention_prefill", "bound": "tensor",
                         "achieved": round(tf, 1), "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": round(tf / peak_tf, 4),
                         "frac_of_sustained": round(tf / pk.get("bf16_tflops_sustained", peak_tf), 4),
                         "peak_kind": pk_kind,
                         "traffic": profiled_traffic("prefill", pw.flops)},
            "e2e": {"value": round(pw.flops * n * ws / (pe2e * 1e-3) / 1e12, 2),
                    "unit": "TFLOP/s", "h2d_bytes_per_step": int(pw.h2d),
                    "d2h_bytes_per_step": int(pw.d2h)}}
        launches += 2 * n  # append + prefill (prefill launch count added below)
    elif want_prefill:
        line["prefill"] = {"value": None, "unavailable": prefill_reason}
    if not dw and pw:
        line.update({"value": line["prefill"]["value"], "unit": "TFLOP/s",
                     "roofline": line["prefill"]["roofline"], "e2e": line["prefill"]["e2e"]})
    line["gpu_launches"] = launches
    line["config"] = workload_config(pw is not None, ws)
    line["clocks"] = clk
    if rank == 0 and not args.no_extras and want_decode:
        line["decode"]["two_calls"] = two_call_steps(dw, pw, step_ids, stream)
    if rank == 0 and not args.no_extras and not args.small and want_decode:
        flush = l2_flush_buffer(dev)
        line["decode_sweep_batch1"] = decode_sweep(dev, flush)
        line["shared_prefix_beams"] = shared_prefix(dev, flush)
        line["mask_modifiers"] = mask_modifiers(dev, dw.case)
        line["device_growth"] = device_growth(dev, dw.case)
        line["fp8_decode"] = fp8_decode(dev, dw.case)
        del flush
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_decode_sample()
        if pw:
            line["prefill"]["cpu_baseline"] = oracle_prefill_sample()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
