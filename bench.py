"""Benchmark of the DSA hot path: one step = one pass of the whole path over one batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode_b64] [--extra prefill_16384]
                    [--impl ours|reference]

A decode step runs, through the C ABI: dsa_index_qk (the dsa_index_keys transform of the new keys,
written into the resident FP8 K-cache, and of the queries, in one launch), dsa_index_scores,
dsa_topk and dsa_sparse_mla. A prefill step runs the same calls over all T queries and S keys. Inputs are seeded synthetic
tensors of the workload's shapes (dsa_inputs); the caches are resident device state.

Timing: W untimed warm-up steps, then K steps, each a replay of a CUDA graph of the step bracketed
by CUDA events on the launching stream, with a 256 MiB L2-flush write between steps (outside the
events) when the inputs fit in L2; the K step times are summed, ranks barrier + synchronise before
and after, and rank 0 reports the max over ranks. After each timed step a second graph of the same
step, with an event pair around each ABI call, is replayed for the per-kernel durations (the
roofline's kernel time); its event nodes would lengthen the step, so it is not part of the step time.
The end-to-end figure (`e2e`) goes through the public API with host buffers: each step copies its
inputs host -> device from pinned memory and reads its results back, and the steps rotate over
independent slots on their own streams so that copies overlap kernels and each other. The steps
are timed twice: with each slot's copies and calls captured once as a CUDA graph and replayed
(`e2e.graph`), and issued from Python every step (`e2e.eager`); `e2e.value` is the faster.
With --gpus N each of N ranks (one process per GPU; started here under torch.distributed.run when
the script is not already a rank) runs its own replica of the workload (independent sequences, no
collective on the data path): weak scaling. The default line also times the 16384-token prefill
(--extra) on the same GPU, for the FP8 index scores and the long-row top-k.

The reference arm (--impl reference) times the CPU oracle on the host cores on a bounded sample
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_inputs as DI  # noqa: E402

METRIC = "indexer scores/s (query·key pairs) + sparse-MLA decode tok/s; % FP8 or HBM roofline"
UNIT = "query·key pairs/s"
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20            # B200 L2


# ------------------------------------------------------------------------------ work accounting
def work_units(inp):
    """Algorithmic units of one step: causal (query, key) pairs scored, queries decoded, and the
    per-kernel algorithmic bytes / flops (the roofline numerators)."""
    from math import prod
    nv = np.clip(np.minimum(inp.q_pos.astype(np.int64) + 1, inp.kv_len[:, None]), 0, None)
    pairs = int(nv.sum())
    k = inp.workload.topk
    sel = int(np.minimum(nv, k).sum())
    BT = int(prod(inp.q_pos.shape))
    new_keys = BT if inp.workload.decode else inp.idx_k.shape[0] * inp.idx_k.shape[1]
    return {
        "pairs": pairs,
        "queries": BT,
        "selected": sel,
        # per kernel, the algorithmic unit of the measurement rules times the units of one launch:
        # index scores 132 B of K-cache per (query, key) pair; top-k 4 B read per visible score and
        # 4 B written per index; sparse MLA 1152 B gathered per (query, selected key)
        "index_keys_bytes": (BT * 64 + new_keys) * (512 + 132) + (BT + new_keys) * 4,
        "index_scores_bytes": pairs * 132,
        "index_scores_flops": pairs * 64 * 128 * 2,
        "topk_bytes": pairs * 4 + BT * k * 4,
        "sparse_mla_bytes": sel * 1152,
        "sparse_mla_flops": sel * 128 * (576 + 512) * 2,
        # further bytes each launch moves beyond those units (reported beside, not in `achieved`):
        # the scores written and the queries/weights read by the index scores; the queries, outputs
        # and indices of the sparse MLA
        "index_scores_other_bytes": pairs * 4 + BT * 64 * (128 + 4 + 4),
        "sparse_mla_other_bytes": BT * 128 * (576 + 512) * 2 + BT * k * 4,
    }


def producer_units(rows):
    """Algorithmic bytes (read + written) and flops of the MLA producers for `rows` tokens: the
    activations in and out once, the 16.8 MB per-head weight matrix once, the RoPE table row."""
    w = 128 * 128 * 512 * 2
    return {
        "q_absorb": {"bytes": rows * 128 * (128 + 64 + 576) * 2 + w + rows * (4 + 256),
                     "flops": rows * 128 * 128 * 512 * 2},
        "kv_entry": {"bytes": rows * ((512 + 64) * 2 + 8 + 4 + 256 + 576 * 2), "flops": 0},
        "out_absorb": {"bytes": rows * 128 * (512 + 128) * 2 + w, "flops": rows * 128 * 512 * 128 * 2},
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------------------ multi-rank plumbing
def max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as tdist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_value(units_per_rank_step, steps, world, t_max_seconds):
    """Whole-job throughput: every rank processes its own replica, so the units add up."""
    return units_per_rank_step * steps * world / t_max_seconds


# ------------------------------------------------------------------------------ clocks sampling
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------ our arm
class Step:
    """Device-resident state and the ABI calls of one step."""

    def __init__(self, inp, device, flush_buffers=True):
        import torch
        import sparse_attention_keys_b200 as dsa
        self.dsa, self.torch, self.inp = dsa, torch, inp
        self.dev_index = device.index if device.index is not None else torch.cuda.current_device()
        wl = inp.workload
        B, T = inp.q_pos.shape
        S = wl.s_max
        self.B, self.T, self.S, self.k = B, T, S, wl.topk
        dev = device
        self.table = dsa.dsa_rope_table(16384).to(dev)
        # resident caches
        self.kcache = torch.zeros((B, S, 128), dtype=torch.uint8, device=dev)
        self.kscale = torch.zeros((B, S), dtype=torch.float32, device=dev)
        self.kv = torch.from_numpy(inp.mla_kv).view(torch.bfloat16).to(dev) if inp.mla_kv is not None else None
        # step inputs (device copies) and their pinned host sources
        if wl.decode:
            # the new token of each sequence is the key at its query position
            new_k = np.stack([inp.idx_k[b, inp.q_pos[b, 0]] for b in range(B)])
            new_pos = inp.q_pos[:, 0].astype(np.int32)
            new_dst = (np.arange(B) * S + new_pos).astype(np.int64)
            # pre-fill the cache for every earlier position (state from previous steps)
            kx = torch.from_numpy(inp.idx_k.reshape(B * S, 128)).to(dev)
            kp = torch.from_numpy(np.tile(np.arange(S, dtype=np.int32), B)).to(dev)
            dsa.dsa_index_keys(kx, kp, self.table, out_fp8=self.kcache, out_scale=self.kscale,
                               dst_row=torch.arange(B * S, dtype=torch.int64, device=dev))
            del kx, kp
        else:
            new_k = inp.idx_k.reshape(B * S, 128)
            new_pos = np.tile(np.arange(S, dtype=np.int32), B)
            new_dst = np.arange(B * S, dtype=np.int64)
        host = {
            "qx": inp.idx_q.reshape(B * T, 64, 128), "qpos_flat": inp.q_pos.reshape(-1).astype(np.int32),
            "w": inp.idx_w, "q_pos": inp.q_pos, "kv_len": inp.kv_len,
            "kx": new_k.astype(np.float32), "kpos": new_pos, "kdst": new_dst,
        }
        if inp.mla_q is not None:
            host["mq"] = inp.mla_q
        self.h = {n: torch.from_numpy(np.ascontiguousarray(a)).pin_memory() for n, a in host.items()}
        self.d = {n: t.to(dev) for n, t in self.h.items()}
        if "mq" in self.d:
            self.d["mq"] = self.d["mq"].view(torch.bfloat16)
        # outputs
        self.q8 = torch.empty((B * T, 64, 128), dtype=torch.uint8, device=dev)
        self.qs = torch.empty((B * T, 64), dtype=torch.float32, device=dev)
        self.ld = (S + 3) // 4 * 4
        self.scores = torch.empty((B, T, self.ld), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, T, self.k), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, T, 128, 512), dtype=torch.bfloat16, device=dev) if self.kv is not None else None
        self.lse = torch.empty((B, T, 128), dtype=torch.float32, device=dev) if self.kv is not None else None
        ws = dsa.dsa_sparse_mla_workspace_size(B, T, self.k) if self.kv is not None else 0
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        # Between timed steps the L2 must not hold this step's data: when the device-resident inputs
        # of a step exceed twice the L2 they evict one another anyway; otherwise a buffer larger than
        # the L2 is written before every step.
        self.input_bytes = sum(t.numel() * t.element_size() for t in
                               [self.kcache, self.kscale] + ([self.kv] if self.kv is not None else []) +
                               list(self.d.values()))
        self.flush_writes = self.input_bytes <= 2 * L2_BYTES
        fb = L2_FLUSH_BYTES // 4 if flush_buffers else 1
        self.flush = torch.empty(fb, dtype=torch.float32, device=dev)
        self.flush_src = torch.ones(fb, dtype=torch.float32, device=dev)
        self.h_idx = torch.empty((B, T, self.k), dtype=torch.int32).pin_memory()
        self.h_out = torch.empty((B, T, 128, 512), dtype=torch.bfloat16).pin_memory() if self.out is not None else None
        self.h_lse = torch.empty((B, T, 128), dtype=torch.float32).pin_memory() if self.out is not None else None
        self.launches_per_step = 3 + (1 if self.kv is not None else 0) + (
            1 if ws > 0 else 0)

    def h2d(self):
        for n, t in self.h.items():
            dst = self.d[n]
            if dst.dtype != t.dtype:
                dst = dst.view(t.dtype)
            dst.copy_(t, non_blocking=True)

    def d2h(self):
        self.h_idx.copy_(self.idx, non_blocking=True)
        if self.out is not None:
            self.h_out.copy_(self.out, non_blocking=True)
            self.h_lse.copy_(self.lse, non_blocking=True)

    def bytes_h2d(self):
        return sum(t.numel() * t.element_size() for t in self.h.values())

    def bytes_d2h(self):
        n = self.h_idx.numel() * 4
        if self.out is not None:
            n += self.h_out.numel() * 2 + self.h_lse.numel() * 4
        return n

    def run(self, ev=None):
        """One step. ev: optional dict name -> list of (start, end) event pairs to record."""
        dsa, d = self.dsa, self.d

        def rec(name, fn):
            if ev is None:
                fn()
                return
            # external: inside a graph capture the records become event nodes of the graph
            s = self.torch.cuda.Event(enable_timing=True, external=True)
            e = self.torch.cuda.Event(enable_timing=True, external=True)
            s.record()
            fn()
            e.record()
            ev.setdefault(name, []).append((s, e))

        B, T = self.B, self.T
        rec("index_keys", lambda: dsa.dsa_index_qk(
            d["kx"], d["kpos"], d["qx"], d["qpos_flat"], self.table, self.kcache, self.kscale, k_dst_row=d["kdst"],
            q_out_fp8=self.q8, q_out_scale=self.qs))
        rec("index_scores", lambda: dsa.dsa_index_scores(
            self.q8.view(B, T, 64, 128), self.qs.view(B, T, 64), d["w"], self.kcache, self.kscale, d["q_pos"],
            d["kv_len"], scores=self.scores, ld=self.ld))
        rec("topk", lambda: dsa.dsa_topk(self.scores, d["q_pos"], d["kv_len"], self.k, idx=self.idx))
        if self.kv is not None:
            # the MLA query is a step input (resident, or copied in from the host), never written by
            # a kernel of the step: the sparse MLA may stage it while the top-k finishes
            rec("sparse_mla", lambda: dsa.dsa_sparse_mla(d["mq"], self.kv, self.idx, out=self.out, lse=self.lse,
                                                         workspace=self.ws, flags=dsa.DSA_Q_READY))

    def l2_flush(self, force=False):
        """Evict the step's data from the L2 (when the step's inputs fit in it, or `force`): write a
        buffer larger than the L2, then read another one, so that the write-back of the dirty flush
        lines happens here, outside the timed events, and the step starts on a cold, clean L2."""
        if self.flush_writes or force:
            self.flush.zero_()
            self.flush_sum = self.flush_src.sum()

    def l2_policy(self):
        if self.flush_writes:
            return f"{L2_FLUSH_BYTES >> 20} MiB flush write, then a {L2_FLUSH_BYTES >> 20} MiB read, between timed steps"
        return f"inputs larger than L2: {self.input_bytes / 2**20:.0f} MiB resident per step, no flush"


def check_status(dsa, stage):
    """Raise if a kernel recorded an error during `stage` (with the wait site for a timeout)."""
    status = dsa.dsa_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after {stage}: {dsa.dsa_status_string(status)} "
                           f"{dsa.dsa_get_error_detail()}")


def time_device(st, args, barrier, sample_clocks=True):
    """Device time of `args.steps` steps of `st` with inputs resident in HBM. The step is captured
    as a CUDA graph and replayed, so no host launch gaps are timed. A second graph of the same
    step holds an event pair around each ABI call and is replayed after every timed step for the
    per-kernel durations: event nodes lengthen a replay by a few microseconds each, so they stay
    out of the step time. Returns (seconds for all steps, {call: seconds per step}, clocks)."""
    import torch

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        cap_stream = torch.cuda.Stream()
        cap_stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap_stream):
            st.run()                              # warm the capture stream (records no events)
        torch.cuda.current_stream().wait_stream(cap_stream)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=cap_stream):
            fn()
        torch.cuda.synchronize()
        return g

    kev = {}
    graph = capture(st.run)
    graph_k = capture(lambda: st.run(kev))
    steps = []
    clk = ClockSampler(st.dev_index) if sample_clocks else None
    if clk is not None:
        clk.__enter__()
    try:
        # the sampler polls every 20 ms: keep the GPU under the same load for ~0.5 s before the
        # timed steps so that the samples taken while they run see steady-state clocks
        t_end = time.perf_counter() + (0.5 if sample_clocks else 0.05)
        while time.perf_counter() < t_end:
            st.l2_flush()
            graph.replay()
            st.l2_flush()
            graph_k.replay()
            torch.cuda.synchronize()
        barrier()
        per_kernel_sum = {n: 0.0 for n in kev}
        for _ in range(args.steps):
            st.l2_flush()
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record()
            graph.replay()
            e.record()
            steps.append((s, e))
            st.l2_flush()
            graph_k.replay()                       # the same step with per-call event nodes
            torch.cuda.synchronize()               # read this replay's kernel events before the next
            for n, v in kev.items():
                per_kernel_sum[n] += sum(a.elapsed_time(b) for a, b in v)
        barrier()
    finally:
        if clk is not None:
            clk.__exit__(None, None, None)
    clocks = clk.summary() if clk is not None else None
    t_dev = sum(s.elapsed_time(e) for s, e in steps) / 1e3          # seconds
    per_kernel = {n: v / args.steps / 1e3 for n, v in per_kernel_sum.items()}
    del graph, graph_k
    return t_dev, per_kernel, clocks


def extra_workload(name, args, dev, peaks):
    """A second workload timed in the same run (device time only, one GPU): the step's throughput
    and the roofline of each of its kernels. The default decode line adds the 16384-token prefill
    here, whose index scores are the FP8 tensor-core half of the metric."""
    import torch
    import sparse_attention_keys_b200 as dsa
    inp = DI.make_inputs(name, seed=0)
    units = work_units(inp)
    st = Step(inp, dev)
    for _ in range(args.warmup):
        st.l2_flush()
        st.run()
    torch.cuda.synchronize()
    check_status(dsa, f"{name} warm-up")
    t_dev, per_kernel, _ = time_device(st, args, torch.cuda.synchronize, sample_clocks=False)
    check_status(dsa, f"{name} graph replays")
    out = {"workload": name, "desc": inp.workload.note, "steps": args.steps,
           "ms_per_step": t_dev / args.steps * 1e3, "value": units["pairs"] * args.steps / t_dev, "unit": UNIT,
           "pairs_per_step": units["pairs"], "l2": st.l2_policy(),
           "kernel_ms": {n: v * 1e3 for n, v in per_kernel.items()},
           "roofline": {n: roofline_entry(n, v, units, peaks, args, workload=name) for n, v in per_kernel.items()
                        if f"{n}_bytes" in units}}
    del st
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as tdist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inp = DI.make_inputs(args.workload, seed=rank)
    units = work_units(inp)
    st = Step(inp, dev)
    import sparse_attention_keys_b200 as dsa

    for _ in range(args.warmup):
        st.l2_flush()
        st.run()
    torch.cuda.synchronize()
    check_status(dsa, "warm-up")

    def barrier():
        if world > 1:
            tdist.barrier()
        torch.cuda.synchronize()

    # ---- device-timed region (inputs resident in HBM)
    t_dev, per_kernel, clocks = time_device(st, args, barrier, sample_clocks=True)
    check_status(dsa, "graph replays")

    # ---- end to end through the public API with host buffers: every step copies its inputs host ->
    # device from pinned memory, runs the calls and reads its results back. Steps rotate over
    # independent slots (device state, pinned buffers, a stream each), so one step's copies overlap
    # another's kernels and the other direction's copies, as a serving loop would run them. When
    # the step's inputs fit in the L2, up to 16 slots rotate (enough that their data exceeds twice
    # the L2 where 16 suffice); e2e.slots_data_exceeds_2x_l2 records whether it did.
    n_slots = 3
    if st.flush_writes:
        n_slots = min(16, max(3, math.ceil(2 * L2_BYTES / max(1, st.input_bytes)) + 1))
    slots_exceed_l2 = n_slots * st.input_bytes > 2 * L2_BYTES
    slots = [st] + [Step(inp, dev, flush_buffers=False) for _ in range(n_slots - 1)]
    streams = [torch.cuda.Stream() for _ in slots]

    def e2e_step(i):
        j = i % n_slots
        with torch.cuda.stream(streams[j]):
            slots[j].h2d()
            slots[j].run()
            slots[j].d2h()

    def timed_rotation(step_fn):
        cur = torch.cuda.current_stream()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(cur)
        for sj in streams:
            sj.wait_event(s)
        for i in range(args.steps):
            step_fn(i)
        for sj in streams:
            cur.wait_stream(sj)
        e.record(cur)
        torch.cuda.synchronize()
        barrier()
        return s.elapsed_time(e) / 1e3

    for i in range(max(1, args.warmup) * n_slots):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    t_e2e_eager = timed_rotation(e2e_step)      # each call issued from Python every step
    check_status(dsa, "end-to-end steps")
    # The same steps with each slot's copies and API calls captured once as a CUDA graph on its
    # stream and replayed: every replay still copies the inputs in and the results out.
    graphs = []
    for j, sl in enumerate(slots):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=streams[j]):
            sl.h2d()
            sl.run()
            sl.d2h()
        graphs.append(g)
    torch.cuda.synchronize()

    def graph_step(i):
        j = i % n_slots
        with torch.cuda.stream(streams[j]):
            graphs[j].replay()

    for i in range(max(1, args.warmup) * n_slots):
        graph_step(i)
    torch.cuda.synchronize()
    barrier()
    t_e2e = timed_rotation(graph_step)
    check_status(dsa, "end-to-end graph steps")
    del graphs
    link = time_link(slots, streams, args.steps)
    del slots[1:]

    producers = None if (args.no_producers or st.kv is None) else time_producers(st, args, dev)
    paged = None if (args.no_producers or st.kv is None) else time_paged(st, args, dev)

    # ---- max over ranks
    t_dev, t_e2e, t_e2e_eager = max_over_ranks([t_dev, t_e2e, t_e2e_eager], world, dev)
    if rank != 0:
        return None

    peaks = load_peaks()
    value = weak_scaling_value(units["pairs"], args.steps, world, t_dev)
    tok_s = weak_scaling_value(units["queries"], args.steps, world, t_dev)
    # dominant kernel and its roofline
    dom = max(per_kernel, key=per_kernel.get)
    roof = roofline_entry(dom, per_kernel[dom], units, peaks, args)
    wl = inp.workload
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_dev / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 scores / bf16 attention, fp32 accumulate",
        "data": "synthetic (seeded N(0,1) of the workload shapes; resident caches)",
        "config": {"workload": wl.name, "desc": wl.note, "batch": int(inp.q_pos.shape[0]),
                   "queries_per_seq": int(inp.q_pos.shape[1]), "s_max": wl.s_max, "topk": wl.topk,
                   "pairs_per_step": units["pairs"], "parallelism": f"replicas x{world}",
                   "l2": st.l2_policy()},
        "mla_decode_tok_s": tok_s if wl.decode else None,
        "kernel_ms": {n: v * 1e3 for n, v in per_kernel.items()},
        "roofline": roof,
        # the faster of the two ways of issuing the same calls (both timed, both reported)
        "e2e": {"value": weak_scaling_value(units["pairs"], args.steps, world, min(t_e2e, t_e2e_eager)), "unit": UNIT,
                "h2d_bytes_per_step": st.bytes_h2d(), "d2h_bytes_per_step": st.bytes_d2h(),
                "ms_per_step": min(t_e2e, t_e2e_eager) / args.steps * 1e3,
                "mode": "graph" if t_e2e <= t_e2e_eager else "eager",
                "pipelined_slots": n_slots,
                "slots_data_exceeds_2x_l2": slots_exceed_l2,
                "graph": {"value": weak_scaling_value(units["pairs"], args.steps, world, t_e2e),
                          "ms_per_step": t_e2e / args.steps * 1e3},
                "eager": {"value": weak_scaling_value(units["pairs"], args.steps, world, t_e2e_eager),
                          "ms_per_step": t_e2e_eager / args.steps * 1e3},
                "link": link},
        "gpu_launches": st.launches_per_step * args.steps,
        "timing": ("device: CUDA-graph replay of the step, CUDA events around each replay; kernel_ms and "
                   "roofline: a replay of the same step with CUDA events around each call, after each "
                   "timed step; e2e: the API calls with host copies in and out every step, steps rotating "
                   "over independent slots on their own streams, timed both as per-slot CUDA graphs "
                   "(e2e.graph) and as calls issued from Python every step (e2e.eager); e2e.value is "
                   "the faster, named by e2e.mode"),
        "clocks": clocks,
    }
    if producers is not None:
        line["mla_producers"] = producer_rooflines(producers, peaks, args.workload)
    if paged is not None:
        line["paged_caches"] = paged_rooflines(paged, units, peaks, args)
    extras = [w for w in (args.extra or "").split(",") if w and w not in (args.workload, "none")]
    if world == 1 and extras:
        del st, slots
        torch.cuda.empty_cache()
        for name in extras:
            line[name] = extra_workload(name, args, dev, peaks)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    return line


def time_producers(st, args, dev):
    """Device time of each MLA producer call for this workload's tokens (B*T rows): each call is
    captured alone as a CUDA graph and replayed `steps` times after warm-up, each replay after an
    L2 flush and bracketed by CUDA events. Outside the step: the step is the indexer + sparse
    MLA path the metric names."""
    import torch
    import sparse_attention_keys_b200 as dsa
    rows = st.B * st.T
    pin = DI.make_mla_producer_inputs(rows, seed=1)
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    bf = lambda a: dv(a).view(torch.bfloat16)
    wkv_b = bf(pin.wkv_b)
    q_nope, q_pe, kv, k_pe, o = bf(pin.q_nope), bf(pin.q_pe), bf(pin.kv), bf(pin.k_pe), bf(pin.o)
    pos = dv(pin.pos)
    q_out = torch.empty((rows, 128, 576), dtype=torch.bfloat16, device=dev)
    x = torch.empty((rows, 128, 128), dtype=torch.bfloat16, device=dev)
    cache = torch.empty((rows, 576), dtype=torch.bfloat16, device=dev)
    dst = torch.arange(rows, dtype=torch.int64, device=dev)
    calls = {
        "q_absorb": lambda: dsa.dsa_mla_q_absorb(q_nope, q_pe, pos, st.table, wkv_b[:, :128], q_out=q_out),
        "kv_entry": lambda: dsa.dsa_mla_kv_entry(kv, k_pe, pos, st.table, dst, cache),
        "out_absorb": lambda: dsa.dsa_mla_out_absorb(o, wkv_b[:, 128:], out=x),
    }
    out = {"rows": rows}
    for name, fn in calls.items():
        out[name] = _graph_time(st, fn, args)
    check_status(dsa, "MLA producers")
    return out


def time_link(slots, streams, steps):
    """The host link alone, per step: the step's host -> device copies with nothing else running,
    its device -> host copies alone, and both directions at once (two slots, two streams). The
    last is the floor under the end-to-end step time when kernels hide behind the copies."""
    import torch
    a, b = streams[0], streams[1 % len(streams)]
    sa, sb = slots[0], slots[1 % len(slots)]

    def timed(jobs):
        cur = torch.cuda.current_stream()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(cur)
        a.wait_event(s)
        b.wait_event(s)
        for _ in range(steps):
            for stream, fn in jobs:
                with torch.cuda.stream(stream):
                    fn()
        cur.wait_stream(a)
        cur.wait_stream(b)
        e.record(cur)
        torch.cuda.synchronize()
        return s.elapsed_time(e) / 1e3 / steps

    timed([(a, sa.h2d), (b, sb.d2h)])                   # warm-up
    t_h, t_d = timed([(a, sa.h2d)]), timed([(b, sb.d2h)])
    t_both = timed([(a, sa.h2d), (b, sb.d2h)])
    return {"h2d_ms": t_h * 1e3, "d2h_ms": t_d * 1e3, "both_ms": t_both * 1e3,
            "h2d_gbs": sa.bytes_h2d() / t_h / 1e9, "d2h_gbs": sb.bytes_d2h() / t_d / 1e9}


def _graph_time(st, fn, args):
    """Mean device time of `fn` captured alone as a CUDA graph: warm-up replays, then `steps`
    replays, each after an L2 flush (whatever the step's own policy) and bracketed by CUDA events."""
    import torch
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        fn()
    torch.cuda.current_stream().wait_stream(cs)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=cs):
        fn()
    for _ in range(max(3, args.warmup)):
        st.l2_flush(force=True)
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(max(5, args.steps)):
        st.l2_flush(force=True)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize()
        ts.append(s.elapsed_time(e) / 1e3)
    del g
    return sum(ts) / len(ts)


def time_paged(st, args, dev, page_size=64):
    """The step's index scores and sparse MLA over paged copies of its caches (pages of 64 rows laid
    out in a seeded random order), each timed alone beside the same call on the dense caches; the
    paged outputs are checked bit for bit against the dense ones."""
    import torch
    import sparse_attention_keys_b200 as dsa
    B, T, S = st.B, st.T, st.S
    max_pages = S // page_size
    num_pages = B * max_pages
    gen = torch.Generator().manual_seed(5)
    perm = torch.randperm(num_pages, generator=gen).to(dev)
    table = perm.view(B, max_pages).to(torch.int32).contiguous()

    def to_pool(dense, row_shape):
        pool = torch.empty((num_pages, page_size) + row_shape, dtype=dense.dtype, device=dev)
        pool[perm.long()] = dense.reshape((num_pages, page_size) + row_shape)
        return pool.view((num_pages * page_size,) + row_shape)

    k8p, ksp, kvp = to_pool(st.kcache, (128,)), to_pool(st.kscale, ()), to_pool(st.kv, (576,))
    d = st.d
    q8, qs = st.q8.view(B, T, 64, 128), st.qs.view(B, T, 64)
    sp = torch.empty_like(st.scores)
    outp, lsep = torch.empty_like(st.out), torch.empty_like(st.lse)
    calls = {
        "index_scores": lambda: dsa.dsa_index_scores(q8, qs, d["w"], st.kcache, st.kscale, d["q_pos"], d["kv_len"],
                                                     scores=st.scores, ld=st.ld),
        "index_scores_paged": lambda: dsa.dsa_index_scores_paged(q8, qs, d["w"], k8p, ksp, table, page_size, d["q_pos"],
                                                                 d["kv_len"], scores=sp, ld=st.ld),
        "sparse_mla": lambda: dsa.dsa_sparse_mla(d["mq"], st.kv, st.idx, out=st.out, lse=st.lse, workspace=st.ws),
        "sparse_mla_paged": lambda: dsa.dsa_sparse_mla_paged(d["mq"], kvp, table, page_size, st.idx, out=outp,
                                                             lse=lsep, workspace=st.ws),
    }
    t = {n: _graph_time(st, fn, args) for n, fn in calls.items()}
    check_status(dsa, "paged caches")
    if not (torch.equal(outp, st.out) and torch.equal(lsep, st.lse)):
        raise RuntimeError("paged sparse MLA differs from the dense call")
    nv = np.clip(np.minimum(st.inp.q_pos.astype(np.int64) + 1, st.inp.kv_len[:, None]), 0, None)
    a, b = st.scores.cpu().numpy(), sp.cpu().numpy()
    for bb in range(B):
        for tt in range(T):
            if not np.array_equal(a[bb, tt, :nv[bb, tt]], b[bb, tt, :nv[bb, tt]]):
                raise RuntimeError("paged index scores differ from the dense call")
    t["page_size"] = page_size
    return t


def paged_rooflines(t, units, peaks, args):
    res = {"page_size": t["page_size"], "layout": "seeded random page order", "timing": "graph of the call alone, L2 flushed before each replay",
           "check": "paged outputs equal the dense ones bit for bit"}
    for name in ("index_scores", "sparse_mla"):
        r = roofline_entry(name, t[f"{name}_paged"], units, peaks, args)
        res[name] = {"dense_us": t[name] * 1e6, "paged_us": t[f"{name}_paged"] * 1e6, "bound": r["bound"],
                     "achieved": r["achieved"], "peak": r["peak"], "unit": r["unit"], "frac": r["frac"]}
    return res


def producer_rooflines(t, peaks, workload=None):
    """Per producer: device time, algorithmic bytes / flops and the HBM roofline (all three are
    below the bf16 ridge: bound by memory), with the ncu DRAM traffic where a current capture of
    that producer on this workload is committed."""
    units = producer_units(t["rows"])
    res = {"rows": t["rows"], "timing": "graph of the call alone, L2 flushed before each replay"}
    for name in ("q_absorb", "kv_entry", "out_absorb"):
        sec = t[name]
        u = units[name]
        ach = u["bytes"] / sec / 1e9
        res[name] = {"us": sec * 1e6, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": u["bytes"],
                     "tflops": u["flops"] / sec / 1e12 if u["flops"] else None,
                     "traffic": load_traffic(name, workload) if workload else None}
    return res


def roofline_entry(name, seconds, units, peaks, args, workload=None):
    """Roofline of one kernel. Prefill shares one cache among all queries, so its index scores
    (e4m3) and sparse MLA (bf16) are bound by the tensor cores; decode kernels stream their own
    cache rows and are bound by HBM."""
    workload = workload or args.workload
    traffic = load_traffic(name, workload)
    prefill = not DI.WORKLOADS[workload].decode
    if prefill and name in ("index_scores", "sparse_mla"):
        flops = units[f"{name}_flops"]
        if name == "index_scores":
            peak = 2.0 * peaks["bf16_tflops"]        # e4m3 dense = 2 x measured bf16 (nominal ratio)
            src = f"{peaks['source']} bf16_tflops x2 (e4m3 nominal ratio)"
        else:
            peak = peaks["bf16_tflops"]
            src = f"{peaks['source']} bf16_tflops"
        ach = flops / seconds / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": traffic, "peak_source": src, "algorithmic_flops": flops,
                "kernel_us": seconds * 1e6}
    nbytes = units[f"{name}_bytes"]
    ach = nbytes / seconds / 1e9
    entry = {"kernel": name, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "peak_source": f"{peaks['source']} hbm_gbs",
             "algorithmic_bytes": nbytes, "kernel_us": seconds * 1e6}
    if f"{name}_other_bytes" in units:
        entry["other_bytes"] = units[f"{name}_other_bytes"]
    return entry


def load_traffic(kernel, workload):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the committed ncu
    summary for this kernel and workload; null when none exists or the kernel's sources changed
    since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(f"{kernel}/{workload}")
    if not e:
        return None
    if sources_digest(e["sources"]) != e["sources_sha256_16"]:
        return None
    return e.get("dram_bytes_per_launch")


def sources_digest(paths):
    """First 16 hex digits of the SHA-256 of the named source files, concatenated in order."""
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------ oracle timing
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def oracle_step(inp, seqs, table, caches):
    """The oracle's pass over sequences `seqs` of one step (new keys and queries quantised,
    scores, top-k, sparse MLA). Returns the (query, key) pairs processed."""
    from oracle import dsa_oracle as O
    k8_all, ks_all = caches
    pairs = 0
    for b in seqs:
        sl = slice(b, b + 1)
        q8, qs = O.index_keys(inp.idx_q[sl], inp.q_pos[sl][..., None], table)
        if inp.workload.decode:
            p = int(inp.q_pos[b, 0])
            k8_all[b, p], ks_all[b, p] = O.index_keys(inp.idx_k[b, p], p, table)
        sc = O.index_scores(q8, qs, inp.idx_w[sl], k8_all[sl], ks_all[sl], inp.q_pos[sl], inp.kv_len[sl])
        idx = O.topk_indices(sc, inp.q_pos[sl], inp.kv_len[sl], inp.workload.topk)
        if inp.mla_q is not None:
            O.sparse_mla(inp.mla_q[sl], inp.mla_kv[sl], idx)
        pairs += int(O.valid_len(inp.q_pos[sl], inp.kv_len[sl]).sum())
    return pairs


def _oracle_setup(workload):
    """Inputs, RoPE table and the K-cache state: empty for decode (each step quantises its new key),
    the whole prefill K-cache quantised once for prefill (cache state, outside the timing)."""
    from oracle import dsa_oracle as O
    inp = DI.make_inputs(workload)
    table = O.rope_table(16384)
    B, S = inp.idx_k.shape[:2]
    if inp.workload.decode:
        return inp, table, (np.zeros((B, S, 128), np.uint8), np.zeros((B, S), np.float32))
    k8, ks = O.index_keys(inp.idx_k, np.arange(S)[None, :], table)
    return inp, table, (k8, ks)


PREFILL_CHUNK = 16       # query rows per oracle unit of a prefill workload


def _oracle_units(inp):
    """The oracle's units of work for a bounded sample: whole sequences for decode; for prefill,
    chunks of PREFILL_CHUNK query rows taken evenly across the causal triangle."""
    if inp.workload.decode:
        return [("seq", b) for b in range(inp.q_pos.shape[0])]
    T = inp.q_pos.shape[1]
    starts = np.linspace(0, T - PREFILL_CHUNK, num=min(64, T // PREFILL_CHUNK)).astype(int)
    return [("rows", int(t0)) for t0 in starts]


def oracle_prefill_rows(inp, t0, table, caches):
    """The oracle's pass over query rows t0 .. t0+PREFILL_CHUNK-1 of sequence 0 of a prefill step
    (queries quantised, scores against the cache, top-k, sparse MLA). Returns the pairs processed."""
    from oracle import dsa_oracle as O
    k8_all, ks_all = caches
    rows = slice(t0, t0 + PREFILL_CHUNK)
    q_pos = inp.q_pos[:1, rows]
    q8, qs = O.index_keys(inp.idx_q[:1, rows], q_pos[..., None], table)
    sc = O.index_scores(q8, qs, inp.idx_w[:1, rows], k8_all[:1], ks_all[:1], q_pos, inp.kv_len[:1])
    idx = O.topk_indices(sc, q_pos, inp.kv_len[:1], inp.workload.topk)
    if inp.mla_q is not None:
        O.sparse_mla(inp.mla_q[:1, rows], inp.mla_kv[:1], idx)
    return int(O.valid_len(q_pos, inp.kv_len[:1]).sum())


def _oracle_unit(inp, unit, table, caches):
    kind, i = unit
    return oracle_step(inp, [i], table, caches) if kind == "seq" else oracle_prefill_rows(inp, i, table, caches)


def cpu_baseline(workload, budget_s=15.0):
    """Time the oracle as it stands on this host, on whole sequences of the workload until about
    `budget_s` seconds of CPU work are done; value in the metric's unit."""
    inp, table, caches = _oracle_setup(workload)
    units = _oracle_units(inp)
    pairs = 0
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        pairs += _oracle_unit(inp, units[done % len(units)], table, caches)
        done += 1
    dt = time.perf_counter() - t0
    if inp.workload.decode:
        what = (f"{done} sequences of {workload} (full path per sequence: new key and query quantised, "
                f"scores, top-{inp.workload.topk}, sparse MLA)")
    else:
        what = (f"{done} chunks of {PREFILL_CHUNK} query rows spread over {workload} (queries quantised, "
                f"scores, top-{inp.workload.topk}{', sparse MLA' if inp.mla_q is not None else ''}; "
                f"the K-cache quantised once, outside the timing)")
    return {"value": pairs / dt, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{what} in {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    inp, table, caches = _oracle_setup(args.workload)
    B = inp.q_pos.shape[0]
    # one step = a bounded sample: two units of the workload (two sequences for decode, two chunks
    # of query rows for prefill)
    units = _oracle_units(inp)
    sample = units[:2] if inp.workload.decode else [units[len(units) // 3], units[-1]]
    for _ in range(args.warmup):
        for u in sample:
            _oracle_unit(inp, u, table, caches)
    t0 = time.perf_counter()
    pairs = 0
    for _ in range(args.steps):
        for u in sample:
            pairs += _oracle_unit(inp, u, table, caches)
    dt = time.perf_counter() - t0
    value = pairs / dt
    wl = inp.workload
    cores = _blas_threads()
    sample_desc = (f"{len(sample)} of {B} sequences of {wl.name} per step (full path per sequence)" if wl.decode else
                   f"2 chunks of {PREFILL_CHUNK} query rows of {wl.name} per step (queries quantised, scores, "
                   f"top-k, sparse MLA; the K-cache quantised once, outside the timing)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded N(0,1) of the workload shapes)",
        "config": {"workload": wl.name, "desc": wl.note, "batch": B, "s_max": wl.s_max, "topk": wl.topk,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample_desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def launch_command(n_gpus, argv):
    """The command that runs this script as `n_gpus` ranks on this node (rendezvous on 127.0.0.1)."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_gpus}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_b64", choices=sorted(DI.WORKLOADS))
    ap.add_argument("--extra", default="prefill_16384",
                    help="comma-separated workloads also timed (device time, one GPU) in the same run; '' or 'none' for none")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-producers", action="store_true", help="skip timing the MLA producer calls")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the ranks here (torch.distributed.run on this node)
        os.execv(sys.executable, launch_command(args.gpus, sys.argv[1:]))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU", file=sys.stderr)
        sys.exit(2)
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            import torch
            import torch.distributed as tdist
            torch.cuda.set_device(local_rank)
            tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                     device_id=torch.device("cuda", local_rank))
        try:
            line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as tdist
                tdist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
