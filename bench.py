#!/usr/bin/env python
"""Benchmark of the CSA/HCA hybrid-attention decode layer on B200.

Metric: decode-layer query-tokens/s (one new query token per sequence per
step) and the achieved fraction of the HBM roofline.  A step is one pass of
the whole hot path over one batch:
  CSA: compress the block the new token completes (KV + indexer streams),
       Lightning-Indexer scores, top-k, sparse shared-KV MQA (+ combine);
  HCA: compress the newest block, dense shared-KV MQA (+ combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (the fp64 CPU oracle, same metric)

Timing: W untimed warm-up steps (plus one untimed replay of every CUDA graph
the timed steps replay), then exactly K steps replayed as CUDA graphs of the
public step call (csa_decode_step / hca_decode_step), bracketed by a barrier
and torch.cuda.synchronize() on both sides, CUDA events on the launching
stream, max over ranks.  Inputs rotate over R independent device-resident
sets whose combined per-step traffic exceeds four times the 126 MB L2, so
every step reads its data from HBM.  A second pass over the same sets runs
each step as separate stage calls with CUDA events between them; it gives
each kernel's average launch time, from which the dominant kernel's
roofline fraction is computed.  The e2e figure runs the same steps as
direct public calls (no graph) with the step's new inputs copied from
pinned host memory and the output copied back, inside the timed region.
A default run then times the other decode workloads (1M-token HCA and CSA)
and the CSA prefill chunk the same way and reports them under "workloads".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from compressed_sparse_kv_04_b200 import configs  # noqa: E402

L2_BYTES = 126 * 2 ** 20
METRIC = "CSA/HCA decode layer query-tokens/s at 128K and 1M ctx; % of HBM roofline"
DEFAULT_WORKLOAD = configs.CSA_128K.name


# ----------------------------------------------------------- byte accounting --
def algorithmic_bytes(w) -> dict:
    """Algorithmic HBM bytes per step (whole batch) of each kernel.

    Only bytes the method must move are counted: inputs read once, outputs
    written once.  Intermediates the library materialises (indexer scores,
    split partials) are implementation overhead and are not counted, except
    as the input of the kernel whose job is to read them: the top-k stage's
    own figure counts the scores it ranks, the step total does not."""
    B, d, m, W, H = w.B, w.d, w.m, w.W, w.H
    out = {}
    blk_in = B * m * d * 2 + (B * m * w.D_I * 2 if w.csa else 0)
    blk_out = B * d * 2 + (B * (w.D_I + 4) if w.csa else 0)
    out["compress"] = blk_in + blk_out + (d + m) * 4 * (2 if w.csa else 1)
    q_bytes = B * H * d * 2
    o_bytes = B * H * d * 2
    if w.csa:
        n = w.N_c
        out["index_scores"] = B * n * (w.D_I + 4) + B * w.H_I * (w.D_I + 8)
        out["topk"] = B * n * 4 + B * w.k * 4 + B * 4
        kv = B * (w.k + W) * d * 2
        out["mqa"] = kv + q_bytes + B * w.k * 4 + H * 4
    else:
        kv = B * (w.N_c + W) * d * 2
        out["mqa"] = kv + q_bytes + H * 4
    out["combine"] = o_bytes
    out["step"] = sum(out.values()) - (B * w.N_c * 4 if w.csa else 0)
    return out


def step_flops(w) -> dict:
    f = {}
    if w.csa:
        f["index_scores"] = 2.0 * w.B * w.N_c * w.H_I * w.D_I
        f["mqa"] = 4.0 * w.B * w.H * (w.k + w.W) * w.d
    else:
        f["mqa"] = 4.0 * w.B * w.H * (w.N_c + w.W) * w.d
    return f


# ------------------------------------------------------------ peak figures --
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


def kernel_source_sha(kernel: str) -> str:
    src = {"index_scores": "indexer.cu", "topk": "topk.cu", "mqa": "mqa.cu",
           "combine": "mqa.cu", "compress": "compress.cu"}[kernel]
    h = hashlib.sha256()
    for f in (src, "common.cuh"):
        with open(os.path.join(ROOT, "compressed_sparse_kv_04_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if it is still current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return e.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz = float(f[1])
                smax = float(f[2])
            except ValueError:
                continue
            sm.append(mhz)
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- aggregation --
def aggregate(units_per_rank: float, elapsed_ms: float, world: int, reduce_max, reduce_sum):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    t = reduce_max(elapsed_ms)
    u = reduce_sum(units_per_rank)
    return u / (t / 1e3), t


def l2_note(R: int, step_bytes: int) -> str:
    total = R * step_bytes
    rel = "more than 4x" if total > 4 * L2_BYTES else "NOT more than 4x (timings partly L2-warm)"
    return (f"rotating {R} resident input sets (~{total / 1e6:.0f} MB of step traffic per "
            f"rotation, {rel} the 126 MB L2)")


def make_reducers(world: int, device):
    """(barrier, max, sum) over the ranks of the default process group, on
    `device` (cuda for NCCL, cpu for gloo); identity functions for one rank.
    Every rank must call them in the same order."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()
        if device.type == "cuda":
            torch.cuda.synchronize(device)

    def _reduce(x, op):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=op)
        return t.item()

    def rmax(x):
        return _reduce(x, dist.ReduceOp.MAX)

    def rsum(x):
        return _reduce(x, dist.ReduceOp.SUM)

    return barrier, rmax, rsum


def workload_for_rank(w, rank: int):
    """Replicas: every rank decodes its own independent sequences (same
    shapes, its own seed); no data crosses between ranks."""
    return configs.scaled(w, seed=w.seed + 1000 * rank) if rank else w


# ------------------------------------------------------------- GPU workload --
class Decode:
    """Device state for R rotating input sets of one decode workload."""

    def __init__(self, w, R, device):
        import torch

        from compressed_sparse_kv_04_b200 import binding, synth
        self.torch, self.binding = torch, binding
        self.w, self.R, self.dev = w, R, device
        B, L, d, N = w.B, w.L, w.d, w.N_c
        self.p = binding.params_for(w)
        self.w_s, self.b_pos = synth.pool_params(w, device)
        if w.csa:
            self.w_si, self.b_pi = synth.pool_params(w, device, indexer=True)
        qi = synth.queries(w, Q=1, device=device)
        self.sink = qi["sink"]
        self.ctx = torch.full((B,), L, dtype=torch.int64, device=device)
        self.pos = self.ctx - 1
        self.pos2 = self.pos.view(B, 1)
        # One source stream and its whole-context compression (setup, untimed).
        kv_src, idx_src = synth.token_streams(w, device=device)
        kv_c_src = torch.empty(B, N, d, dtype=torch.bfloat16, device=device)
        if w.csa:
            key_src = torch.empty(B, N, w.D_I, dtype=torch.uint8, device=device)
            ksc_src = torch.empty(B, N, dtype=torch.float32, device=device)
            binding.csa_compress(self.p, kv_src, self.ctx, self.w_s, self.b_pos, None, 0, N,
                                 kv_c_src, idx_src, self.w_si, self.b_pi, key_src, ksc_src)
        else:
            binding.hca_compress(self.p, kv_src, self.ctx, self.w_s, self.b_pos, None, 0, N,
                                 kv_c_src)
        tail = max(w.W, w.m)
        self.tail = tail
        op_step = binding.OP_CSA_DECODE_STEP if w.csa else binding.OP_HCA_DECODE_STEP
        self.sets = []
        for r in range(R):
            s = {}
            # Full-size token buffers; only the tail the step reads is filled.
            s["kv_tok"] = torch.empty(B, L, d, dtype=torch.bfloat16, device=device)
            s["kv_tok"][:, L - tail:] = kv_src[:, L - tail:]
            s["kv_c"] = kv_c_src.clone()
            q = synth.normal_bf16((B, w.H, d), w.seed + 1000 + r, "q", device)
            s["out"] = torch.empty(B, w.H, d, dtype=torch.bfloat16, device=device)
            s["ws_step"] = binding.workspace(self.p, op_step, 1, N, device)
            if w.csa:
                s["idx_tok"] = torch.empty(B, L, w.D_I, dtype=torch.bfloat16, device=device)
                s["idx_tok"][:, L - tail:] = idx_src[:, L - tail:]
                s["key"] = key_src.clone()
                s["ksc"] = ksc_src.clone()
                qr = synth.queries(configs.scaled(w, seed=w.seed + 1000 + r), Q=1, device=device)
                # The step's query-side inputs in one buffer (one copy per
                # step on the end-to-end path).
                parts = [q, qr["q_idx"], qr["q_scale"], qr["w"]]
                offs, o = [], 0
                for t in parts:
                    offs.append(o)
                    o += (t.numel() * t.element_size() + 255) // 256 * 256
                s["qin"] = torch.empty(o, dtype=torch.uint8, device=device)
                views = []
                for t, o0 in zip(parts, offs):
                    nb = t.numel() * t.element_size()
                    v = s["qin"][o0:o0 + nb].view(t.dtype).view(t.shape)
                    v.copy_(t)
                    views.append(v)
                s["q"], s["q_idx"], s["q_scale"], s["w"] = views
                s["q_idx3"] = s["q_idx"].view(B, w.H_I, w.D_I)
                s["q_scale2"] = s["q_scale"].view(B, w.H_I)
                s["w2"] = s["w"].view(B, w.H_I)
                s["scores"] = torch.empty(B, 1, N, dtype=torch.float32, device=device)
                s["tidx"] = torch.empty(B, 1, w.k, dtype=torch.int32, device=device)
                s["tcnt"] = torch.empty(B, 1, dtype=torch.int32, device=device)
                s["ws"] = binding.workspace(self.p, binding.OP_SPARSE_MQA, 1, N, device)
            else:
                s["q"] = q
                s["ws"] = binding.workspace(self.p, binding.OP_DENSE_MQA, 1, N, device)
            self.sets.append(s)
        del kv_src, idx_src
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        torch.cuda.synchronize()

    def step(self, s):
        """One decode step of the whole batch: ONE public call (newest-block
        compression, then indexer, top-k and sparse attention for CSA, or
        dense attention for HCA)."""
        b, w, p = self.binding, self.w, self.p
        if w.csa:
            b.csa_decode_step(p, self.pos, s["kv_tok"], s["idx_tok"], self.w_s, self.b_pos, None,
                              self.w_si, self.b_pi, s["kv_c"], s["key"], s["ksc"], s["q"],
                              s["q_idx3"], s["q_scale2"], s["w2"], self.sink,
                              s["tidx"].view(w.B, w.k), s["tcnt"].view(w.B), s["out"],
                              ws=s["ws_step"], dev_status=self.status)
        else:
            b.hca_decode_step(p, self.pos, s["kv_tok"], self.w_s, self.b_pos, None, s["kv_c"],
                              s["q"], self.sink, s["out"], ws=s["ws_step"], dev_status=self.status)

    # The same step as separate calls, one per stage (for the per-stage
    # timing pass: events between the calls).
    def stages(self, s):
        b, w, p, N = self.binding, self.w, self.p, self.w.N_c
        st = self.status
        if w.csa:
            return [
                ("compress", lambda: b.csa_compress(p, s["kv_tok"], self.ctx, self.w_s, self.b_pos,
                                                    None, N - 1, 1, s["kv_c"], s["idx_tok"],
                                                    self.w_si, self.b_pi, s["key"], s["ksc"],
                                                    dev_status=st)),
                ("index_scores", lambda: b.lightning_index_scores(p, 1, s["q_idx"], s["q_scale"],
                                                                  s["w"], s["key"], s["ksc"],
                                                                  self.pos2, s["scores"],
                                                                  dev_status=st)),
                ("topk", lambda: b.topk_select(p, 1, s["scores"], self.pos2, s["tidx"], s["tcnt"],
                                               dev_status=st)),
                ("mqa", lambda: b.sparse_mqa_decode(p, s["q"], self.pos, s["kv_c"],
                                                    s["tidx"].view(w.B, w.k),
                                                    s["tcnt"].view(w.B), s["kv_tok"], self.sink,
                                                    s["out"], ws=s["ws"], dev_status=st)),
            ]
        return [
            ("compress", lambda: b.hca_compress(p, s["kv_tok"], self.ctx, self.w_s, self.b_pos,
                                                None, N - 1, 1, s["kv_c"], dev_status=st)),
            ("mqa", lambda: b.dense_mqa_decode(p, s["q"], self.pos, s["kv_c"], s["kv_tok"],
                                               self.sink, s["out"], ws=s["ws"], dev_status=st)),
        ]

    def prepared_step(self, s, stream):
        """The step of input set s as a prepared public call bound to its
        buffers (binding CsaDecodeStep / HcaDecodeStep .bind: arguments
        converted once); returns f() that runs one step on `stream`."""
        b, w, p = self.binding, self.w, self.p
        if w.csa:
            f = b.CsaDecodeStep(p, s["kv_tok"], s["idx_tok"], self.w_s, self.b_pos, None, self.w_si,
                                self.b_pi, s["kv_c"], s["key"], s["ksc"], self.sink,
                                s["tidx"].view(w.B, w.k), s["tcnt"].view(w.B), s["ws_step"],
                                dev_status=self.status)
            return f.bind(self.pos, s["q"], s["q_idx3"], s["q_scale2"], s["w2"], s["out"],
                          stream=stream)
        f = b.HcaDecodeStep(p, s["kv_tok"], self.w_s, self.b_pos, None, s["kv_c"], self.sink,
                            s["ws_step"], dev_status=self.status)
        return f.bind(self.pos, s["q"], s["out"], stream=stream)

    def launches_per_step(self):
        """Kernel launches of one step, counted from the kernel nodes of a
        captured step graph (a separate capture kept as a cudaGraph_t);
        falls back to the call's known sequence (compress, (indexer, top-k,)
        attention, split merge) where the runtime does not expose nodes."""
        torch = self.torch
        try:
            from cuda.bindings import runtime as rt
            stream = torch.cuda.Stream()
            stream.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g, stream=stream):
                self.step(self.sets[0])
            torch.cuda.synchronize()
            raw = g.raw_cuda_graph()
            _, _, n = rt.cudaGraphGetNodes(raw, numNodes=0)
            _, nodes, n = rt.cudaGraphGetNodes(raw, numNodes=n)
            kernels = sum(1 for nd in nodes[:n]
                          if rt.cudaGraphNodeGetType(nd)[1] ==
                          rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
            del g
            if kernels > 0:
                return kernels
        except Exception:  # noqa: BLE001 - the count then falls back
            pass
        return 5 if self.w.csa else 3

    def _warm(self):
        torch = self.torch
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):  # warm the launch path outside capture
            for s in self.sets:
                self.step(s)
                for _, fn in self.stages(s):
                    fn()
        torch.cuda.current_stream().wait_stream(stream)
        torch.cuda.synchronize()
        return stream

    def capture_steps(self):
        """One CUDA graph per input set holding one step (one public call)."""
        torch = self.torch
        stream = self._warm()
        graphs = []
        for s in self.sets:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                self.step(s)
            graphs.append(g)
        return graphs

    def capture_cycle(self):
        """One CUDA graph holding a step of every input set in turn (R
        consecutive steps), so that consecutive steps meet at a kernel
        boundary, as consecutive attention layers of a model step do,
        rather than at a graph launch."""
        torch = self.torch
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in self.sets:
                self.step(s)
        return g

    def capture_instrumented(self):
        """One graph per input set: the step as separate stage calls with an
        event between consecutive stages."""
        torch = self.torch
        stream = self._warm()
        graphs, events = [], []
        for s in self.sets:
            g = torch.cuda.CUDAGraph()
            ev = []
            with torch.cuda.graph(g, stream=stream):
                e = torch.cuda.Event(enable_timing=True, external=True)
                e.record()
                ev.append(e)
                for _, fn in self.stages(s):
                    fn()
                    e = torch.cuda.Event(enable_timing=True, external=True)
                    e.record()
                    ev.append(e)
            graphs.append(g)
            events.append(ev)
        return graphs, events


def measure_decode(w, K, W, dev, barrier, rmax, rsum, world, rotate=0, e2e=True):
    """Times K decode steps of workload w (after W warm-up steps); returns
    the per-workload record (throughput, step and dominant-kernel rooflines,
    per-stage times, e2e)."""
    import torch
    ab = algorithmic_bytes(w)
    R = rotate or max(2, math.ceil(4 * L2_BYTES / ab["step"]) + 1)
    st = Decode(w, R, dev)
    graphs = st.capture_steps()
    cycle = st.capture_cycle()
    torch.cuda.synchronize()
    launches_step = st.launches_per_step()

    def plan(n):
        """The graphs that n consecutive steps replay: whole R-step cycles,
        then single-step graphs."""
        return [cycle] * (n // R) + [graphs[i] for i in range(n % R)]

    # Warm-up: W steps, then one untimed replay of every graph the timed
    # region replays and the W steps did not (so no first replay, with its
    # one-time upload, falls inside the timed region).
    warm = plan(W)
    for g in warm:
        g.replay()
    timed = plan(K)
    for g in timed:
        if not any(g is x for x in warm):
            g.replay()
            warm.append(g)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for g in timed:
        g.replay()
    e1.record()
    barrier()
    elapsed = e0.elapsed_time(e1)
    value, t_max = aggregate(w.B * K, elapsed, world, rmax, rsum)
    status = int(st.status.item())
    del graphs, cycle

    # Per-stage pass: K steps as separate stage calls with events between
    # them (the events break the overlap between kernels, so the stage times
    # add up to more than a step).
    igraphs, ievents = st.capture_instrumented()
    names = [n for n, _ in st.stages(st.sets[0])]
    sums = {n: 0.0 for n in names}
    for _ in range(max(1, W)):  # warm the instrumented graphs too
        for g in igraphs:
            g.replay()
    torch.cuda.synchronize()
    done = 0
    while done < K:
        batch = min(R, K - done)
        for j in range(batch):
            igraphs[j].replay()
        torch.cuda.synchronize()
        for j in range(batch):
            ev = ievents[j]
            for n, a, b in zip(names, ev[:-1], ev[1:]):
                sums[n] += a.elapsed_time(b)
        done += batch
    stage_ms = {n: sums[n] / K for n in names}
    del igraphs, ievents

    e2e_rec = run_e2e(st, K, W, barrier, rmax, rsum, world) if e2e else None

    peaks = measured_peaks()
    dom = max(stage_ms, key=stage_ms.get)
    dom_ms = stage_ms[dom]
    # the attention call is the attention kernel + the split merge
    bytes_dom = ab["mqa"] + ab["combine"] if dom == "mqa" else ab[dom]
    achieved = bytes_dom / (dom_ms * 1e-3) / 1e9
    ms_per_step = t_max / K
    rec = {
        "value": round(value, 1), "unit": "query-tokens/s", "ms_per_step": round(ms_per_step, 6),
        "config": {"workload": w.name, "batch": w.B, "context": w.L, "compressed_entries": w.N_c,
                   "m": w.m, "heads": w.H, "head_dim": w.d, "window": w.W,
                   "top_k": w.k if w.csa else None,
                   "indexer": [w.H_I, w.D_I] if w.csa else None,
                   "call": "csa_decode_step" if w.csa else "hca_decode_step",
                   "l2": l2_note(R, ab["step"]),
                   "warmup": "W steps plus one untimed replay of every graph the timed steps "
                             "replay"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"], "traffic": stored_traffic(dom, w.name),
                     "algorithmic_bytes_per_launch": bytes_dom, "avg_launch_ms": round(dom_ms, 6)},
        "step_roofline": {"algorithmic_bytes": ab["step"],
                          "achieved_GBps": round(ab["step"] / (ms_per_step * 1e-3) / 1e9, 1),
                          "frac": round(ab["step"] / (ms_per_step * 1e-3) / 1e9 /
                                        peaks["hbm_gbs"], 4),
                          "peak": peaks["hbm_gbs"], "peak_source": peaks["source"]},
        "kernels_ms": {k: round(v, 6) for k, v in stage_ms.items()},
        "gpu_launches": launches_step * K,
        "device_status": status,
    }
    if e2e_rec is not None:
        rec["e2e"] = e2e_rec
    return rec, st


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    barrier, rmax, rsum = make_reducers(world, dev)

    w = workload_for_rank(configs.BY_NAME[args.workload], rank)
    K, W = args.steps, args.warmup
    extras = {}
    with ClockSampler(local) as clocks:
        rec, st = measure_decode(w, K, W, dev, barrier, rmax, rsum, world, args.rotate,
                                 e2e=not args.no_e2e)
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(w, st, args.cpu_seconds)
        del st
        torch.cuda.empty_cache()
        # The other decode workloads (and the prefill chunk) in the same run,
        # each with its own time and rooflines.
        if not args.no_extra:
            for name in EXTRA_WORKLOADS:
                if name == w.name:
                    continue
                if name in PROJ_TOKENS:
                    extras[name] = measure_proj(name, K, W, dev)
                    torch.cuda.empty_cache()
                    continue
                wx = workload_for_rank(configs.BY_NAME[name], rank)
                if wx.kind == "csa_prefill":
                    extras[name] = measure_prefill(wx, K, W, dev)
                else:
                    r, sx = measure_decode(wx, K, W, dev, barrier, rmax, rsum, world, 0,
                                           e2e=False)
                    extras[name] = r
                    del sx
                torch.cuda.empty_cache()
    clk = clocks.summary()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    line = {
        "metric": METRIC,
        "value": rec["value"],
        "unit": "query-tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16+e4m3",
        "data": "synthetic (seeded N(0,1) token streams, random query/indexer inputs)",
        "config": dict(rec["config"],
                       parallelism=f"replicas x{world} (independent sequences per GPU)"),
        "roofline": rec["roofline"],
        "step_roofline": rec["step_roofline"],
        "kernels_ms": rec["kernels_ms"],
        "e2e": rec.get("e2e"),
        "gpu_launches": rec["gpu_launches"],
        "clocks": clk,
        "device_status": rec["device_status"],
    }
    if extras:
        line["workloads"] = extras
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# The workloads timed after the primary one in a default run.
EXTRA_WORKLOADS = ["hca_decode_1m_b8", "csa_decode_1m_b4", "csa_prefill_4096_after_65536",
                   "grouped_out_proj_decode_t8", "grouped_out_proj_prefill_t4096"]

# Grouped output projection ("DeepSeek V4-Pro" (llm-arch-kb), "1. Hybrid
# attention": g = 16 groups, d_g = 1024) of the 128-head x 512 attention
# output; d = 7168 (the pages give no model dim).  T = 8 is one decode step of
# the 128K batch, T = 4096 the prefill chunk.
PROJ_SHAPE = dict(H=128, D=512, g=16, d_g=1024, d_model=7168)
PROJ_TOKENS = {"grouped_out_proj_decode_t8": 8, "grouped_out_proj_prefill_t4096": 4096}


def measure_proj(name, K, W, dev):
    """K calls of grouped_out_proj on one fixed input (the weights, 352 MiB,
    exceed the L2, so every call streams them from HBM)."""
    import torch

    from compressed_sparse_kv_04_b200 import binding, synth
    T = PROJ_TOKENS[name]
    H, D, g, d_g, dm = (PROJ_SHAPE[k] for k in ("H", "D", "g", "d_g", "d_model"))
    gen = torch.Generator(device=dev).manual_seed(20260008)
    k1 = H // g * D
    w_g = (torch.randn(g, d_g, k1, generator=gen, device=dev) / math.sqrt(k1)).to(torch.bfloat16)
    w_o = (torch.randn(dm, g * d_g, generator=gen, device=dev) / math.sqrt(g * d_g)).to(
        torch.bfloat16)
    o = synth.normal_bf16((T, H, D), 20260008, "q", dev)
    z = torch.empty(T, dm, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(binding.grouped_out_proj_workspace_bytes(T, H, D, g, d_g, dm),
                     dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        binding.grouped_out_proj(o, w_g, w_o, z, ws=ws, dev_status=status)

    for _ in range(W):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    peaks = measured_peaks()
    flops = 2.0 * T * (g * d_g * k1 + dm * g * d_g)
    wbytes = (g * d_g * k1 + dm * g * d_g) * 2
    abytes = wbytes + T * H * D * 2 + T * g * d_g * 2 * 2 + T * dm * 2
    launches = 2 + sum(1 for sp in _proj_splits(T, H, D, g, d_g, dm) if sp > 1)
    rec = {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 6),
           "config": {"workload": name, "tokens": T, **PROJ_SHAPE, "call": "grouped_out_proj",
                      "l2": "no rotation: the weights (352 MiB) exceed the L2"},
           "gpu_launches": launches * K, "device_status": int(status.item())}
    tf = flops / (ms * 1e-3) / 1e12
    gbs = abytes / (ms * 1e-3) / 1e9
    if T <= 64:  # weight streaming: HBM-bound
        rec["roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                           "peak_source": peaks["source"], "algorithmic_bytes": abytes,
                           "avg_launch_ms": round(ms, 6), "traffic": None}
    else:
        rec["roofline"] = {"bound": "tensor", "achieved": round(tf, 1),
                           "peak": round(peaks["bf16_tflops"], 1), "unit": "TFLOP/s",
                           "frac": round(tf / peaks["bf16_tflops"], 4),
                           "peak_source": peaks["source"], "algorithmic_flops": flops,
                           "avg_launch_ms": round(ms, 6), "traffic": None}
    return rec


def _proj_splits(T, H, D, g, d_g, dm):
    """The split-K factors the library picks (mirrors its planning, for the
    launch count: a split projection adds one reduce launch)."""
    import torch
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    bn = 16 if T <= 16 else 32 if T <= 32 else 64 if T <= 64 else 128 if T <= 128 else 256

    def choose(N, groups, Kin):
        tiles = (N // 128) * -(-T // bn) * groups
        chunks = Kin // 64
        s = 1
        while tiles * s * 2 <= sms and chunks % (s * 2) == 0 and chunks // (s * 2) >= 8:
            s *= 2
        return s
    return choose(d_g, g, H // g * D), choose(dm, 1, g * d_g)


def run_e2e(st, K, W, barrier, rmax, rsum, world):
    """The same K steps through the public call (csa_decode_step /
    hca_decode_step, each step a direct call: argument checks and launches
    included, no graph), with the step's new query and token rows copied
    from pinned host memory and its output copied back to pinned host
    memory, all inside the timed region."""
    torch = st.torch
    w, R = st.w, st.R
    L = w.L
    # CSA: the query-side inputs are one buffer (qin); HCA: the query.
    qkey = "qin" if w.csa else "q"
    hq = [s[qkey].cpu().pin_memory() for s in st.sets]
    # The step's new token: one KV (and indexer) row per sequence at the
    # step's position L - 1 (the block's earlier rows came with earlier steps).
    hkv = [s["kv_tok"][:, L - 1:].cpu().pin_memory() for s in st.sets]
    hout = [torch.empty_like(s["out"], device="cpu").pin_memory() for s in st.sets]
    hidx = [s["idx_tok"][:, L - 1:].cpu().pin_memory() for s in st.sets] if w.csa else []

    # Copies run on their own streams: the inputs of step i+1 travel while
    # step i computes, and the output of step i returns while step i+1
    # computes (each step has its own input set and its own host output
    # buffer, so nothing is overwritten while in use).  Copies and steps are
    # the binding's prepared calls (csa_copy_async / csa_copy_rows_async and
    # the bound decode step): one library call each, arguments converted once.
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    PC = st.binding.PreparedCopy
    ups = []
    for r, s in enumerate(st.sets):
        c = [PC(s[qkey], hq[r], up), PC(s["kv_tok"][:, L - 1:], hkv[r], up)]
        if w.csa:
            c.append(PC(s["idx_tok"][:, L - 1:], hidx[r], up))
        ups.append(c)
    downs = [PC(hout[r], s["out"], down) for r, s in enumerate(st.sets)]
    h2d = sum(c.bytes for c in ups[0])
    d2h = downs[0].bytes
    steps = [st.prepared_step(s, comp) for s in st.sets]
    copied = [torch.cuda.Event() for _ in range(R)]
    done = [torch.cuda.Event() for _ in range(R)]
    fetched = [torch.cuda.Event() for _ in range(R)]
    used = [False] * R

    def upload(i):
        r = i % R
        if used[r]:
            up.wait_event(done[r])  # the set's previous step has finished
        for c in ups[r]:
            c()
        copied[r].record(up)

    def compute(i):
        r = i % R
        comp.wait_event(copied[r])
        if used[r]:
            comp.wait_event(fetched[r])  # the set's previous output has left
        steps[r]()
        done[r].record(comp)
        used[r] = True
        down.wait_event(done[r])
        downs[r]()
        fetched[r].record(down)

    def run(n):
        up.wait_stream(comp)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
        comp.wait_stream(down)

    run(W)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    run(K)
    e1.record()
    barrier()
    val, _ = aggregate(w.B * K, e0.elapsed_time(e1), world, rmax, rsum)
    return {"value": round(val, 1), "unit": "query-tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "path": "direct public calls per step (no graph): the binding's prepared "
                    "CsaDecodeStep / HcaDecodeStep bound to the set's buffers, and prepared "
                    "copies (csa_copy_async / csa_copy_rows_async) of the inputs from pinned "
                    "host memory and of the output to pinned host memory, inside the timed "
                    "region"}


# ---------------------------------------------------------------- prefill --
PREFILL_METRIC = "CSA prefill chunk query-tokens/s; % of FP8 / BF16 tensor roofline"


def prefill_work(w):
    """Causal work of one chunk: FP8 indexer flops, BF16 attention flops."""
    import numpy as np
    t = w.P + np.arange(w.T, dtype=np.int64)
    nv = (t + 1) // w.m
    win = np.minimum(t + 1, w.W)
    fp8 = 2.0 * w.H_I * w.D_I * float(nv.sum())
    bf16 = 4.0 * w.H * w.d * float((np.minimum(nv, w.k) + win).sum())
    return fp8, bf16


def measure_prefill(w, K, W, dev):
    """One CSA prefill chunk per step (csa_prefill_chunk: compression of the
    chunk's blocks, causal indexer, top-k, sparse attention), B = 1.  The
    step's scores alone (T x N_cap fp32) exceed the L2, so no rotation."""
    import torch

    from compressed_sparse_kv_04_b200 import binding, synth
    b = binding
    L_cap = w.P + w.T
    N_cap = -(-L_cap // w.m)
    kv_tok, idx_tok = synth.token_streams(w, L_cap=L_cap, device=dev)
    w_s, b_pos = synth.pool_params(w, dev)
    w_si, b_pi = synth.pool_params(w, dev, indexer=True)
    qi = synth.queries(w, Q=w.T, device=dev)
    q = qi["q"][0].contiguous()
    q_idx, q_scale, wq = qi["q_idx"][0].contiguous(), qi["q_scale"][0].contiguous(), qi["w"][0].contiguous()
    p = b.params_for(w, B=1)
    kv_c = torch.zeros(1, N_cap, w.d, dtype=torch.bfloat16, device=dev)
    key = torch.zeros(1, N_cap, w.D_I, dtype=torch.uint8, device=dev)
    ksc = torch.zeros(1, N_cap, dtype=torch.float32, device=dev)
    ctx = torch.full((1,), w.P, dtype=torch.int64, device=dev)
    b.csa_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, w.P // w.m, kv_c, idx_tok, w_si, b_pi,
                   key, ksc)  # the cached part, before the chunk
    ws = b.workspace(p, b.OP_PREFILL, w.T, N_cap, device=dev)
    out = torch.empty(w.T, w.H, w.d, dtype=torch.bfloat16, device=dev)
    tidx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    tcnt = torch.empty(w.T, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scores = ws[: w.T * N_cap * 4].view(torch.float32).view(1, w.T, N_cap)
    pos = (w.P + torch.arange(w.T, device=dev, dtype=torch.int64)).view(1, w.T)

    def chunk():
        b.csa_prefill_chunk(p, w.P, w.T, kv_tok, idx_tok, w_s, b_pos, None, w_si, b_pi, kv_c,
                            key, ksc, q, q_idx, q_scale, wq, qi["sink"], tidx, tcnt, out, ws=ws,
                            dev_status=status)

    def index_only():
        b.lightning_index_scores(p, w.T, q_idx, q_scale, wq, key, ksc, pos, scores,
                                 dev_status=status)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    for _ in range(W):
        chunk()
        index_only()
    torch.cuda.synchronize()
    ms = timed(chunk, K)
    ms_idx = timed(index_only, K)
    fp8, bf16 = prefill_work(w)
    peaks = measured_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]  # dense FP8 = 2 x dense BF16 (nominal ratio)
    idx_tf = fp8 / (ms_idx * 1e-3) / 1e12
    t_ideal = fp8 / (fp8_peak * 1e12) + bf16 / (peaks["bf16_tflops"] * 1e12)
    return {
        "metric": PREFILL_METRIC, "value": round(w.T / (ms * 1e-3), 1), "unit": "query-tokens/s",
        "ms_per_step": round(ms, 4), "dtype": "e4m3+bf16",
        "config": {"workload": w.name, "prior_tokens": w.P, "chunk_tokens": w.T, "heads": w.H,
                   "head_dim": w.d, "top_k": w.k, "indexer": [w.H_I, w.D_I],
                   "call": "csa_prefill_chunk",
                   "l2": "no rotation: the chunk's scores alone (T x N_cap fp32) exceed the L2"},
        "roofline": {"bound": "tensor", "kernel": "index_scores", "achieved": round(idx_tf, 1),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(idx_tf / fp8_peak, 4),
                     "peak_source": peaks["source"] + " (bf16 x 2, nominal FP8/BF16 ratio)",
                     "avg_launch_ms": round(ms_idx, 4), "algorithmic_flops": fp8},
        "step_roofline": {"fp8_flops": fp8, "bf16_flops": bf16,
                          "ideal_ms": round(t_ideal * 1e3, 4),
                          "frac": round(t_ideal * 1e3 / ms, 4)},
        # per chunk: compress, indexer, top-k, attention (one split per row:
        # no merge)
        "gpu_launches": 4 * K, "device_status": int(status.item()),
    }


def run_prefill(args):
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    with ClockSampler(0) as clocks:
        rec = measure_prefill(configs.CSA_PREFILL, K, W, dev)
    line = dict(rec, n_gpus=1, steps=K, warmup=W, higher_is_better=True, scaling="weak",
                vs_baseline=None,
                data="synthetic (seeded N(0,1) token streams, random query/indexer inputs)",
                clocks=clocks.summary())
    line["gpu_launches"] = rec["gpu_launches"] + K  # plus the separately timed indexer
    print(json.dumps(line), flush=True)


HCA_PREFILL_METRIC = "HCA prefill chunk query-tokens/s; % of BF16 tensor roofline"


def hca_prefill_flops(w):
    """Causal attention flops of one HCA chunk: every query against its
    visible entries and its window (QK^T and PV, 2 flops per MAC)."""
    import numpy as np
    t = w.P + np.arange(w.T, dtype=np.int64)
    nv = (t + 1) // w.m
    win = np.minimum(t + 1, w.W)
    return 4.0 * w.H * w.d * float((nv + win).sum())


def run_hca_prefill(args):
    """One HCA prefill chunk per step (hca_prefill_chunk: compression of the
    chunk's blocks, dense attention per query), B = 1.  The step's output
    (T x H x d x 2 bytes) exceeds the L2, so no rotation."""
    import torch

    from compressed_sparse_kv_04_b200 import binding as b
    from compressed_sparse_kv_04_b200 import synth
    w = configs.HCA_PREFILL
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L_cap = w.P + w.T
    N_cap = -(-L_cap // w.m)
    kv_tok, _ = synth.token_streams(w, L_cap=L_cap, device=dev)
    w_s, b_pos = synth.pool_params(w, dev)
    qi = synth.queries(w, Q=w.T, device=dev)
    q = qi["q"][0].contiguous()
    p = b.params_for(w, B=1)
    kv_c = torch.zeros(1, N_cap, w.d, dtype=torch.bfloat16, device=dev)
    ctx = torch.full((1,), w.P, dtype=torch.int64, device=dev)
    b.hca_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, w.P // w.m, kv_c)  # the cached part
    ws = b.workspace(p, b.OP_HCA_PREFILL, w.T, N_cap, device=dev)
    out = torch.empty(w.T, w.H, w.d, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def chunk():
        b.hca_prefill_chunk(p, w.P, w.T, kv_tok, w_s, b_pos, None, kv_c, q, qi["sink"], out,
                            ws=ws, dev_status=status)

    K, W = args.steps, args.warmup
    with ClockSampler(0) as clocks:
        for _ in range(W):
            chunk()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            chunk()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / K
    flops = hca_prefill_flops(w)
    peaks = measured_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": HCA_PREFILL_METRIC, "value": round(w.T / (ms * 1e-3), 1),
        "unit": "query-tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) token streams and queries)",
        "config": {"workload": w.name, "prior_tokens": w.P, "chunk_tokens": w.T, "heads": w.H,
                   "head_dim": w.d, "m": w.m, "window": w.W,
                   "l2": "no rotation: the chunk's output exceeds the L2"},
        "roofline": {"bound": "tensor", "kernel": "hca_prefill_chunk (compress + attention)",
                     "achieved": round(tf, 1), "peak": round(peaks["bf16_tflops"], 1),
                     "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                     "peak_source": peaks["source"], "avg_launch_ms": round(ms, 4),
                     "algorithmic_flops": flops},
        # per chunk: compress, attention (one split per row: no merge)
        "gpu_launches": 2 * K, "clocks": clocks.summary(), "device_status": int(status.item()),
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ CPU oracle --
class OracleStep:
    """One sequence's decode step through the fp64 oracle, as it stands:
    compress the newest block, then (CSA) indexer scores, top-k and sparse
    MQA, or (HCA) dense MQA.  Inputs are drawn once (or taken from the GPU
    state's first set, for the same cache contents).

    run(n_sub, h_sub) times the three parts separately, optionally on a
    bounded sample: the indexer and top-k over the first n_sub compressed
    entries, attention for the first h_sub heads."""

    def __init__(self, w, state=None):
        import numpy as np

        from oracle import oracle as orc
        self.np, self.orc, self.w = np, orc, w
        rng = np.random.default_rng(w.seed)
        d, N, L, m = w.d, w.N_c, w.L, w.m

        def bf16(shape):
            x = rng.standard_normal(shape).astype(np.float32)
            return (x.view(np.uint32) >> 16).astype(np.uint16)

        self.tail = tail = max(w.W, m)
        if state is not None:
            import torch
            s = state.sets[0]
            self.kv_c = s["kv_c"][0:1].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
            self.tok = (s["kv_tok"][0:1, L - tail:].contiguous().view(torch.int16).cpu().numpy()
                        .view(np.uint16))
        else:
            self.kv_c = bf16((1, N, d))
            self.tok = bf16((1, tail, d))
        self.q = bf16((1, 1, w.H, d))
        self.sink = rng.standard_normal(w.H).astype(np.float32)
        self.w_s = (rng.standard_normal(d) * 0.02).astype(np.float32)
        self.b_pos = (rng.standard_normal(m) * 0.1).astype(np.float32)
        self.pos = np.array([[L - 1]])
        if w.csa:
            self.keys = rng.integers(0, 0x7E, (1, N, w.D_I)).astype(np.uint8)
            self.ksc = rng.uniform(0.005, 0.015, (1, N)).astype(np.float32)
            self.q_idx = rng.integers(0, 0x7E, (1, 1, w.H_I, w.D_I)).astype(np.uint8)
            self.q_scale = rng.uniform(0.005, 0.02, (1, 1, w.H_I)).astype(np.float32)
            self.wh = rng.uniform(0, 1, (1, 1, w.H_I)).astype(np.float32)
            self.itok = bf16((1, tail, w.D_I))
            self.w_si = (rng.standard_normal(w.D_I) * 0.02).astype(np.float32)
        self.threads = os.cpu_count() or 1
        # RoPE frequencies and logit scale: the oracle's own YaRN table for a
        # workload with YaRN settings, else plain RoPE and 1/sqrt(d).
        self.freq, self.scale = None, None
        if w.yarn is not None:
            self.freq = orc.yarn_inv_freq(w.rope_dim, *w.yarn)
            self.scale = orc.yarn_logit_gain(w.yarn[0]) / d ** 0.5

    def run(self, n_sub=None, h_sub=None, a_sub=None):
        """Returns (compress_s, index_s, attention_s).  A sample covers the
        indexer + top-k over the first n_sub entries and attention for the
        first h_sub heads over at most a_sub compressed entries (the first of
        the selection, or of the visible entries for HCA) plus the window."""
        np, orc, w = self.np, self.orc, self.w
        N, m, tail = w.N_c, w.m, self.tail
        n_sub = N if n_sub is None else max(1, min(N, n_sub))
        h_sub = w.H if h_sub is None else max(1, min(w.H, h_sub))
        t0 = time.perf_counter()
        orc.pool(self.tok, [tail], self.w_s, self.b_pos, None, m, tail // m - 1, 1, tail // m,
                 rope_dim=w.rope_dim, rope_freq=self.freq)
        if w.csa:
            orc.pool(self.itok, [tail], self.w_si, self.b_pos, None, m, tail // m - 1, 1,
                     tail // m)
        t1 = time.perf_counter()
        q, sink = self.q[:, :, :h_sub], self.sink[:h_sub]
        if w.csa:
            keys, ksc = self.keys[:, :n_sub], self.ksc[:, :n_sub]
            sc = orc.index_scores(self.q_idx, self.q_scale, self.wh, keys, ksc,
                                  np.array([[n_sub * m - 1]]), m)
            idx, cnt = orc.topk(sc, np.array([[n_sub]]), w.k)
            t2 = time.perf_counter()
            if a_sub is not None:
                cnt = np.minimum(cnt, a_sub).astype(np.int32)
            orc.mqa(q, self.pos, self.kv_c, self.tok, sink, m, w.W, w.rope_dim, idx, cnt,
                    tok_base=w.L - tail, rope_freq=self.freq, scale=self.scale)
        else:
            t2 = t1
            if a_sub is None:
                orc.mqa(q, self.pos, self.kv_c, self.tok, sink, m, w.W, w.rope_dim,
                        tok_base=w.L - tail, rope_freq=self.freq, scale=self.scale)
            else:
                sel = np.arange(min(a_sub, N), dtype=np.int32).reshape(1, 1, -1)
                orc.mqa(q, self.pos, self.kv_c, self.tok, sink, m, w.W, w.rope_dim, sel,
                        np.full((1, 1), sel.shape[-1], np.int32), tok_base=w.L - tail,
                        rope_freq=self.freq, scale=self.scale)
        t3 = time.perf_counter()
        return t1 - t0, t2 - t1, t3 - t2


def cpu_baseline(w, state, seconds):
    """The oracle on whole decode steps of one sequence for about `seconds`."""
    o = OracleStep(w, state)
    steps, t0 = 0, time.perf_counter()
    while True:
        o.run()
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(steps / el, 4), "unit": "query-tokens/s", "cores": o.threads,
            "kind": "oracle",
            "sample": f"{steps} whole decode step(s) of one sequence ({w.name}: {w.N_c} "
                      f"compressed entries), {el:.1f} s wall on {o.threads} host threads"}


REFERENCE_BUDGET_S = 150.0


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores.

    Each step is one sequence's decode step (one query token).  When W + K
    whole steps would take longer than REFERENCE_BUDGET_S, every step after
    the first two warm-ups runs a bounded sample instead (indexer + top-k
    over the first 2k entries, attention for one head) and is charged its
    own measured time plus the time of the part it leaves out, measured in
    warm-up as (whole step) - (sample) part by part."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = configs.BY_NAME[args.workload]
    from oracle import oracle as orc
    orc.lib()
    o = OracleStep(w)
    full = o.run()  # warm-up 1: a whole step
    t_full = sum(full)
    per_step = 0.8 * REFERENCE_BUDGET_S / (args.steps + args.warmup)
    sampled = t_full > per_step
    sub = {}
    extra = 0.0
    n_cal = 1
    if sampled:
        # Size the sample to the per-step budget (the oracle's threads split
        # its work in fixed chunks, so time is not proportional to size).
        r = per_step / t_full
        for _ in range(8):
            sub = dict(n_sub=min(w.N_c, max(64, math.ceil(w.N_c * r))),
                       h_sub=max(1, math.ceil(w.H * r)),
                       a_sub=max(16, math.ceil((w.k if w.csa else w.N_c) * r)))
            part = o.run(**sub)
            n_cal += 1
            if sum(part) <= per_step:
                break
            r *= 0.7 * per_step / sum(part)
        # time of the part the sample leaves out, from warm-up
        extra = max(0.0, full[1] - part[1]) + max(0.0, full[2] - part[2])
    for _ in range(args.warmup - n_cal):
        o.run(**sub)
    total, wall0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        total += sum(o.run(**sub)) + extra
    wall = time.perf_counter() - wall0
    value = args.steps / total
    if sampled:
        what = (f"indexer + top-k over {sub['n_sub']} of {w.N_c} entries, " if w.csa else "")
        sample = (f"each step = one sequence's decode step of {w.name}, run on a sample "
                  f"({what}attention for {sub['h_sub']} of {w.H} heads over at most "
                  f"{sub['a_sub']} compressed entries + the window) plus {extra * 1e3:.1f} ms "
                  f"for the rest, measured once in warm-up as whole step minus sample; "
                  f"{wall:.1f} s wall for {args.steps} steps")
    else:
        sample = f"each step = one sequence's whole decode step of {w.name}"
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 4),
        "unit": "query-tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name},
        "cpu_baseline": {"value": round(value, 4), "unit": "query-tokens/s",
                         "cores": o.threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(configs.BY_NAME))
    ap.add_argument("--rotate", type=int, default=0, help="input sets (default: from L2 size)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the primary workload (not the other decode workloads and "
                         "the prefill chunk)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        if configs.BY_NAME[args.workload].kind.endswith("prefill"):
            ap.error("the reference arm times decode workloads")
        return run_reference(args)
    if args.workload == configs.TINY_CSA.name:
        ap.error("the tiny case is a parity-test case")
    if args.workload == configs.CSA_PREFILL.name:  # explicit request only; not the default line
        return run_prefill(args)
    if args.workload == configs.HCA_PREFILL.name:
        return run_hca_prefill(args)
    run_gpu(args)


if __name__ == "__main__":
    main()
