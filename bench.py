#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

One step = one decode iteration of one attention layer over a batch of
sequences: paged_kv_append of each sequence's new token, then
paged_attention_decode (a memset of its split counters and one kernel, which
also merges split sequences by log-sum-exp). Inputs are seeded synthetic
tensors already resident in HBM. The timed steps replay a CUDA graph of one
step; the decode kernel's own time per launch is measured with CUDA events
around eager launches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gqa70b]
    python bench.py --impl reference ...    # the fp64 CPU oracle on host cores

Under torchrun every rank runs its own replica of the workload (weak scaling;
decode has no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import paged_kv_cache_367_b200 as pkv  # noqa: E402
from paged_kv_cache_367_b200 import roofline  # noqa: E402
from paged_kv_cache_367_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention HBM GB/s (% of B200 peak) and decode tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20

WORKLOAD_TEXT = {
    "gqa70b": "70B-class GQA decode: 128 seqs, 64 q / 8 KV heads, head_dim 128, bf16 N(0,1), "
              "block 16, lognormal lengths (median 1024, sigma 0.8) clipped to [16, 8192], "
              "shuffled pool, one appended token per sequence",
    "llama2_13b_mha": "Llama-2-13B-shaped decode: 64 seqs, 40 q = 40 KV heads, head_dim 128, fp16, "
                      "block 16, lengths U[128, 2048], shuffled pool, append of 1 token per seq",
    "long_splitk": "long-context split-K decode: 8 seqs, 32 q / 8 KV heads, head_dim 128, bf16, "
                   "block 32, lengths U[32768, 131072], partitions of 512 merged by LSE",
    "fp8_prefix": "FP8 E4M3 KV with per-tensor scales and a shared 1024-token prefix: 64 seqs, "
                  "32 q / 8 KV heads, head_dim 128, bf16 Q, private suffix U[16, 512], block 16",
    "tiny": "tiny fp32 decode: 4 seqs, 8 heads, head_dim 64, block 16, lengths U[1, 100]",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gqa70b", choices=sorted(W.CONFIGS))
    ap.add_argument("--partition-size", type=int, default=None)
    ap.add_argument("--max-ctas", type=int, default=0)
    ap.add_argument("--flags", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-graph", action="store_true", help="time eager launches")
    ap.add_argument("--plain-launch", action="store_true",
                    help="decode without PKV_DECODE_ZEROED_WORKSPACE | PKV_DECODE_EARLY_START "
                         "(zero the counters every call; no programmatic dependent launch)")
    ap.add_argument("--op", default="decode",
                    choices=["decode", "blocks", "blocksize", "prefill", "kernels"],
                    help="blocks: time the block copies (copy-on-write, swap) and the host "
                         "block manager; blocksize: decode time and pool fragmentation for "
                         "block sizes 8/16/32; prefill: causal multi-token queries over the "
                         "paged cache; kernels: the tensor-core decode kernel against the "
                         "CUDA-core one on the MHA and GQA workloads (one JSON line each) "
                         "instead of the decode step")
    return ap.parse_args()


DECODE_SOURCES = ("common.cuh", "schedule.cuh", "tc_common.cuh", "decode_tc.cu", "decode_simt.cu",
                  "pkv_api.cu")


def _code_only(text: str) -> str:
    """C/C++ source without its comments and with white space collapsed, so that
    an edit of a comment or of the layout does not count as a kernel change."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_sha() -> str:
    """Hash of the code (comments aside) the decode kernels and their launch are
    built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_367_b200", "csrc")
    paths = [os.path.join(csrc, name) for name in DECODE_SOURCES]
    paths.append(os.path.join(ROOT, "include", "pagedkv.h"))
    for path in paths:
        with open(path, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:12]


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken
    on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", f"ncu_decode_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"^source_sha:\s*(\w+)", text, re.M)
    m_b = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not (m_sha and m_b) or m_sha.group(1) != source_sha():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """SM clock and clock-event reasons through NVML: one sample when entered,
    one every `period` seconds while running, one when left."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, index: int, period: float = 0.0005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            p = torch.cuda.get_device_properties(index)
            try:
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def sample(self):
        if self._nv is None:
            return
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.wait(self.period):
            self.sample()

    def __enter__(self):
        self.sample()
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join()
        self.sample()

    def summary(self):
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "sm_mhz_min": float(np.min(self.samples)) if self.samples else None,
                "reasons": sorted(self.reasons)}


def workload_config(wl, partition_size):
    c = wl.cfg
    kv_bytes = 2 * int(wl.seq_lens.sum()) * c.num_kv_heads * c.head_dim * W.ELEM_BYTES[c.cache_dtype]
    return {"workload": WORKLOAD_TEXT.get(c.name, c.name), "name": c.name,
            "num_seqs": c.num_seqs, "num_heads": c.num_heads, "num_kv_heads": c.num_kv_heads,
            "head_dim": c.head_dim, "block_size": c.block_size, "q_dtype": c.q_dtype,
            "cache_dtype": c.cache_dtype, "total_tokens": int(wl.seq_lens.sum()),
            "max_seq_len": wl.max_seq_len, "partition_size": partition_size,
            "l2": (f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of K/V read per step vs "
                   f"126 MB L2" if kv_bytes > L2_BYTES else
                   "K/V fit in L2: timing reuses L2-resident data (no flush)"),
            "parallelism": "replicas: one independent workload per GPU, no collective"}


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (all ranks call it)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s replica of a workload (distinct per rank)."""
    return base_seed + 7919 * rank


def step_bytes(wl):
    c = wl.cfg
    eq, ekv = W.ELEM_BYTES[c.q_dtype], W.ELEM_BYTES[c.cache_dtype]
    dec = roofline.decode_bytes(wl.seq_lens, c.num_heads, c.num_kv_heads, c.head_dim,
                                c.block_size, eq, ekv, shared_prefix_tokens=c.prefix_len)
    app = roofline.append_bytes(c.num_seqs, c.num_kv_heads, c.head_dim, eq, ekv)
    return dec, app


# ------------------------------------------------------------------ our arm ----

def kernel_time_ms(pre, call, n=16, reps=5):
    """Mean device time of call() per launch: a CUDA graph of n x (pre(), event,
    call(), event) is replayed `reps` times and the events' spans averaged. The
    events are graph nodes (recorded as external events), so the span is the
    launch's own time with no host gap. Falls back to events around eager
    launches if the graph cannot be built. Returns (ms, how)."""
    stream = torch.cuda.current_stream()
    try:
        evs = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n)]
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for _ in range(3):
                pre()
                call()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for a, b in evs:
                pre()
                a.record()
                call()
                b.record()
        g.replay()
        torch.cuda.synchronize()
        spans = []
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            spans += [a.elapsed_time(b) for a, b in evs]
        del g
        return float(np.mean(spans)), (f"CUDA events as graph nodes around each of {n} launches "
                                        f"per graph replay, {reps} replays")
    except Exception as e:  # noqa: BLE001 - report how it was timed instead
        torch.cuda.synchronize()
        reason = f"{type(e).__name__}"
    m = max(n * reps, 20)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(m)]
    for a, b in ev:
        pre()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return (float(np.mean([a.elapsed_time(b) for a, b in ev])),
            f"CUDA events around {m} eager launches (graph events unavailable: {reason})")


_CUDART = None


def _cudart():
    """The CUDA runtime (the copy torch ships with, else the system one), for the
    copies and events of the end-to-end loop: issued directly they cost about
    1 us of host time each, against 5-10 us through torch's stream context
    managers, so the loop stays ahead of the GPU on slower hosts."""
    global _CUDART
    if _CUDART is None:
        import ctypes
        import glob
        cands = sorted(glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia",
                                              "cuda_runtime", "lib", "libcudart.so*")))
        cands += ["libcudart.so.12", "/usr/local/cuda/lib64/libcudart.so"]
        lib = None
        for c in cands:
            try:
                lib = ctypes.CDLL(c)
                break
            except OSError:
                continue
        if lib is None:
            raise RuntimeError("libcudart not found")
        V, S = ctypes.c_void_p, ctypes.c_size_t
        lib.cudaMemcpyAsync.argtypes = [V, V, S, ctypes.c_int, V]
        lib.cudaMemcpyAsync.restype = ctypes.c_int
        lib.cudaEventRecord.argtypes = [V, V]
        lib.cudaEventRecord.restype = ctypes.c_int
        lib.cudaStreamWaitEvent.argtypes = [V, V, ctypes.c_uint]
        lib.cudaStreamWaitEvent.restype = ctypes.c_int
        _CUDART = lib
    return _CUDART


def e2e_time_ms(args, wl, c_calls, out, world):
    """Per-step time of the step through the public API with host buffers.

    Every step copies its inputs (query, new K/V, slot mapping, block table,
    lengths), packed in one pinned host buffer, to the device in one copy, calls
    paged_kv_append and paged_attention_decode through the C ABI (their
    arguments marshalled once per buffer by `c_calls`), and copies the output
    back to pinned host memory. Inputs and outputs are double
    buffered and the copies run on their own streams, so step k+1's inputs and
    step k-1's output move while step k computes; the timed region spans the
    first input copy to the last output copy. The copies and the events that
    order them are issued through the CUDA runtime directly. The loop is
    timed twice: eagerly, and as `graph_steps` steps captured once in a CUDA
    graph and replayed, as a serving loop would, so the host issues one launch
    per `graph_steps` steps (every replay still copies each step's inputs from,
    and its output to, pinned host memory); the faster form is reported, both
    times are returned."""
    cr = _cudart()
    K = args.steps
    KE = args.e2e_steps or max(min(K, 200), 100)
    parts = [wl.query, wl.new_key, wl.new_value, torch.from_numpy(wl.slot_mapping),
             torch.from_numpy(wl.block_table), torch.from_numpy(wl.seq_lens)]
    offs, total = [], 0
    for t in parts:
        total = (total + 255) // 256 * 256
        offs.append(total)
        total += t.numel() * t.element_size()
    h_in = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(2)]
    d_in = [torch.empty(total, dtype=torch.uint8, device=out.device) for _ in range(2)]
    views = []
    for b in range(2):
        v = []
        for t, o in zip(parts, offs):
            nb = t.numel() * t.element_size()
            h_in[b][o:o + nb].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
            v.append(d_in[b][o:o + nb].view(t.dtype).view(t.shape))
        views.append(v)
    outs = [out, torch.empty_like(out)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d, d2h = total, out.numel() * out.element_size()
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    cs, si, so = compute.cuda_stream, s_in.cuda_stream, s_out.cuda_stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]     # step done: inputs free, output ready
    ev_read = [torch.cuda.Event() for _ in range(2)]     # output copied to the host
    for evs in (ev_in, ev_done, ev_read):                # create the events
        for e in evs:
            e.record(compute)
    torch.cuda.synchronize()
    hin = [h.data_ptr() for h in h_in]
    din = [d.data_ptr() for d in d_in]
    hout = [h.data_ptr() for h in h_out]
    dout = [o.data_ptr() for o in outs]
    H2D, D2H = 1, 2
    calls = [c_calls(*views[b], outs[b], cs) for b in range(2)]
    evi = [e.cuda_event for e in ev_in]
    evd = [e.cuda_event for e in ev_done]
    evr = [e.cuda_event for e in ev_read]

    def ck(rc):
        if rc != 0:
            raise RuntimeError(f"CUDA runtime error {rc} in the end-to-end loop")

    def body(k, cs, calls):  # step k on buffer k % 2, compute on stream cs
        b = k & 1
        if k >= 2:
            ck(cr.cudaStreamWaitEvent(si, evd[b], 0))
        ck(cr.cudaMemcpyAsync(din[b], hin[b], h2d, H2D, si))
        ck(cr.cudaEventRecord(evi[b], si))
        ck(cr.cudaStreamWaitEvent(cs, evi[b], 0))
        if k >= 2:
            ck(cr.cudaStreamWaitEvent(cs, evr[b], 0))
        for fn, a in calls[b]:
            st = fn(*a)
            if st != 0:
                raise pkv.PagedKVError(fn.__name__, st)
        ck(cr.cudaEventRecord(evd[b], cs))
        ck(cr.cudaStreamWaitEvent(so, evd[b], 0))
        ck(cr.cudaMemcpyAsync(hout[b], dout[b], d2h, D2H, so))
        ck(cr.cudaEventRecord(evr[b], so))

    def run(steps):
        for k in range(steps):
            body(k, cs, calls)

    run(4)
    torch.cuda.synchronize()
    GS = min(25, KE)
    graph = None
    if not args.no_graph:
        ev_fork, ev_ji, ev_jo = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        for e in (ev_fork, ev_ji, ev_jo):
            e.record(compute)
        torch.cuda.synchronize()
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                cap = torch.cuda.current_stream().cuda_stream
                gcalls = [c_calls(*views[b], outs[b], cap) for b in range(2)]
                ck(cr.cudaEventRecord(ev_fork.cuda_event, cap))   # the copy streams join
                ck(cr.cudaStreamWaitEvent(si, ev_fork.cuda_event, 0))
                ck(cr.cudaStreamWaitEvent(so, ev_fork.cuda_event, 0))
                for k in range(GS):
                    body(k, cap, gcalls)
                ck(cr.cudaEventRecord(ev_ji.cuda_event, si))       # and leave
                ck(cr.cudaStreamWaitEvent(cap, ev_ji.cuda_event, 0))
                ck(cr.cudaEventRecord(ev_jo.cuda_event, so))
                ck(cr.cudaStreamWaitEvent(cap, ev_jo.cuda_event, 0))
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize()
            graph = g
        except Exception:
            torch.cuda.synchronize()
            graph = None
    # Both loop forms are timed, the same steps through the same calls; the
    # faster is reported (the graph saves host time per step, the eager loop
    # the graph's cross-stream edges: which wins depends on the host).
    reps = max(1, KE // GS)
    KG = reps * GS
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    s_in.wait_stream(compute)
    run(KE)
    compute.wait_stream(s_out)
    e1.record(compute)
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1) / KE
    graph_ms = None
    if graph is not None:
        if world > 1:
            torch.distributed.barrier()
        e0.record(compute)
        for _ in range(reps):
            graph.replay()
        e1.record(compute)
        torch.cuda.synchronize()
        graph_ms = e0.elapsed_time(e1) / KG
    if world > 1:  # every rank reports the same form
        both = torch.tensor([eager_ms, graph_ms if graph_ms is not None else float("inf")],
                            device=out.device)
        torch.distributed.all_reduce(both, op=torch.distributed.ReduceOp.MAX)
        eager_ms, g = both.tolist()
        graph_ms = None if g == float("inf") else g
    use_graph = graph_ms is not None and graph_ms < eager_ms
    ms, steps = (graph_ms, KG) if use_graph else (eager_ms, KE)
    last = ((GS if use_graph else KE) - 1) & 1
    return (ms, steps, h2d, d2h, h_out[last], GS if use_graph else 0,
            {"eager_ms_per_step": round(eager_ms, 5),
             "graph_ms_per_step": None if graph_ms is None else round(graph_ms, 5)})



def run_ours(args, rank, world, dev):
    cfg = W.CONFIGS[args.workload]
    cfg = cfg.replace(seed=replica_seed(cfg.seed, rank))
    P = cfg.partition_size if args.partition_size is None else args.partition_size
    wl = W.make_workload(cfg, device=dev)
    c = wl.cfg
    bt = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    slots = torch.from_numpy(wl.slot_mapping).to(dev)
    ks = vs = None
    if c.cache_dtype == "e4m3":
        ks = torch.tensor([wl.k_scale], dtype=torch.float32, device=dev)
        vs = torch.tensor([wl.v_scale], dtype=torch.float32, device=dev)
    msl = wl.max_seq_len
    ws_bytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                  c.head_dim, msl, P)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev) if ws_bytes else None
    out = torch.empty_like(wl.query)
    launches_per_step = 2  # append kernel + decode kernel (plus a memset when split)

    def append(key, value, slot_t):
        pkv.paged_kv_append(key, value, wl.k_cache, wl.v_cache, slot_t, k_scale=ks, v_scale=vs)

    # After the first call has zeroed the workspace's counters (every call
    # leaves them zero), the step runs the decode with the serving flags: no
    # zeroing memset, and an early start behind the append of this step.
    serving = 0 if args.plain_launch else (pkv.PKV_DECODE_ZEROED_WORKSPACE |
                                           pkv.PKV_DECODE_EARLY_START)
    first = [True]

    def decode(q, bt_t, lens_t, out_t, early=True):
        flags = args.flags | (0 if first[0] else serving)
        if not early:
            flags &= ~pkv.PKV_DECODE_EARLY_START
        first[0] = False
        pkv.paged_attention_decode(out_t, q, wl.k_cache, wl.v_cache, bt_t, lens_t, max_seq_len=msl,
                                   scale=c.scale, partition_size=P, workspace=ws, k_scale=ks,
                                   v_scale=vs, max_ctas=args.max_ctas, flags=flags)

    def step():
        append(wl.new_key, wl.new_value, slots)
        decode(wl.query, bt, lens, out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(max(args.warmup, 3)):
            step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        for _ in range(K):
            if graph is not None:
                graph.replay()
            else:
                step()
        t1.record(stream)
        torch.cuda.synchronize()
    step_ms = t0.elapsed_time(t1) / K
    if world > 1:
        torch.distributed.barrier()
    # The decode kernel alone: CUDA events recorded around each decode launch
    # inside a CUDA graph of several steps (append, event, decode, event), so no
    # host launch gap is timed; eager launches if the graph cannot hold events.
    decode_ms, decode_timing = kernel_time_ms(
        lambda: append(wl.new_key, wl.new_value, slots),
        lambda: decode(wl.query, bt, lens, out, early=False), reps=max(1, min(K // 20, 10)))
    status = pkv.pkv_device_status(clear=True)
    assert status == 0, f"device wait expired (status {status})"

    lib = pkv.load_library()
    e2e_flags = args.flags | serving

    def c_calls(q, nk, nv, sl, bt_t, ln, out_t, stream):
        """The step's two C-ABI calls on these buffers, each argument converted
        to its C type once."""
        def prebuilt(fn, a):
            return fn, tuple(t(x) for t, x in zip(fn.argtypes, a))
        return (prebuilt(lib.paged_kv_append,
                         pkv.append_args(nk, nv, wl.k_cache, wl.v_cache, sl, k_scale=ks,
                                         v_scale=vs, stream=stream)),
                prebuilt(lib.paged_attention_decode,
                         pkv.decode_args(out_t, q, wl.k_cache, wl.v_cache, bt_t, ln,
                                         max_seq_len=msl, scale=c.scale, partition_size=P,
                                         workspace=ws, k_scale=ks, v_scale=vs,
                                         max_ctas=args.max_ctas, flags=e2e_flags,
                                         stream=stream)))

    e2e_ms, KE, h2d, d2h, h_out, e2e_graph, e2e_forms = e2e_time_ms(args, wl, c_calls, out, world)
    assert torch.isfinite(h_out.float()).all(), "non-finite decode output"

    if world > 1:
        step_ms, decode_ms, e2e_ms = max_over_ranks([step_ms, decode_ms, e2e_ms], dev)

    dec_b, app_b = step_bytes(wl)
    peak, peak_src = measured_hbm_peak()
    value = world * (dec_b + app_b) / (step_ms * 1e-3) / 1e9
    achieved = dec_b / (decode_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": c.q_dtype if c.cache_dtype == c.q_dtype else f"{c.q_dtype}+{c.cache_dtype}",
        "data": "synthetic (seeded N(0,1) tensors, shuffled block pool)",
        "config": workload_config(wl, P),
        "tokens_per_s": round(world * c.num_seqs / (step_ms * 1e-3), 1),
        "pct_of_8TBs_nominal": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "decode_ms": round(decode_ms, 5),
        "decode_timing": decode_timing,
        "bytes_per_step": {"decode": dec_b, "append": app_b},
        "roofline": {"bound": "hbm", "kernel": "paged_attention_decode (decode kernel" +
                     (", counter memset)" if args.plain_launch else ", counters left zero by the previous call)"),
                     "achieved": round(achieved, 2), "peak": peak, "peak_source": peak_src,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(c.name)},
        "e2e": {"value": round(world * (dec_b + app_b) / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "steps": KE, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "each step: one H2D copy of the step's packed inputs (query, new K/V, "
                       "slot mapping, block table, lengths) from pinned host memory, "
                       "paged_kv_append and paged_attention_decode through the C ABI "
                       "(arguments marshalled once per double buffer), "
                       "one D2H copy of the output to pinned host memory; copies run on two "
                       "copy streams, double-buffered, so step k+1's inputs and step k-1's "
                       "output move while step k computes; copies and events issued through "
                       "the CUDA runtime; timed both eagerly and as a loop of graph_steps steps "
                       "captured in one CUDA graph and replayed, the faster reported "
                       "(graph_steps 0: eager)",
                "graph_steps": e2e_graph, **e2e_forms},
        "gpu_launches": K * launches_per_step,
        "timing": "CUDA graph replay of one step" if graph is not None else "eager launches",
        "decode_flags": "plain" if args.plain_launch else
                        "PKV_DECODE_ZEROED_WORKSPACE | PKV_DECODE_EARLY_START (no counter memset; "
                        "programmatic dependent launch behind the append)",
        "clocks": clk.summary(),
        "source_sha": source_sha(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return res


# -------------------------------------------------------- oracle on the host ----

def _oracle_rate(wl, kc, vc, items, threads=0):
    import oracle
    c = wl.cfg
    t = time.perf_counter()
    _, used = oracle.decode(W.host(wl.query), kc, vc, wl.block_table, wl.seq_lens,
                            num_heads=c.num_heads, num_kv_heads=c.num_kv_heads, head_dim=c.head_dim,
                            block_size=c.block_size, scale=c.scale, q_dtype=c.q_dtype,
                            cache_dtype=c.cache_dtype, k_scale=wl.k_scale, v_scale=wl.v_scale,
                            items=items, threads=threads)
    return time.perf_counter() - t, used


def _item_bytes(wl, items):
    c = wl.cfg
    eq, ekv = W.ELEM_BYTES[c.q_dtype], W.ELEM_BYTES[c.cache_dtype]
    per_seq = [roofline.decode_bytes([L], c.num_heads, c.num_kv_heads, c.head_dim, c.block_size,
                                     eq, ekv) for L in wl.seq_lens]
    return sum(per_seq[i] for i, _ in items) / c.num_heads


def cpu_baseline(wl, seconds):
    """The fp64 oracle, as it stands, on a bounded sample of the same workload."""
    c = wl.cfg
    kc, vc = W.host(wl.k_cache), W.host(wl.v_cache)
    all_items = [(i, j) for i in range(c.num_seqs) for j in range(c.num_heads)]
    probe = all_items[:c.num_heads]
    dt, _ = _oracle_rate(wl, kc, vc, probe)
    per_seq = max(dt, 1e-4)
    n_seq = int(max(1, min(c.num_seqs, seconds / per_seq)))
    items = all_items[:n_seq * c.num_heads]
    dt, used = _oracle_rate(wl, kc, vc, items)
    b = _item_bytes(wl, items)
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"first {n_seq} of {c.num_seqs} sequences, all {c.num_heads} query heads "
                      f"({sum(int(wl.seq_lens[i]) for i in range(n_seq))} tokens), fp64 C "
                      f"oracle with OpenMP over (sequence, head)"}


def run_reference(args):
    cfg = W.CONFIGS[args.workload]
    wl = W.make_workload(cfg, device="cpu")
    c = wl.cfg
    kc, vc = W.host(wl.k_cache), W.host(wl.v_cache)
    # Fill each sequence's newest slot as the append of a step would.
    import oracle
    oracle.append(W.host(wl.new_key), W.host(wl.new_value), kc, vc, wl.slot_mapping,
                  num_kv_heads=c.num_kv_heads, head_dim=c.head_dim, block_size=c.block_size,
                  num_blocks=wl.num_blocks, src_dtype=c.q_dtype, cache_dtype=c.cache_dtype,
                  k_scale=wl.k_scale, v_scale=wl.v_scale)
    all_items = [(i, j) for i in range(c.num_seqs) for j in range(c.num_heads)]
    dt, _ = _oracle_rate(wl, kc, vc, all_items[:c.num_heads])
    rate = c.num_heads / max(dt, 1e-6)                        # items per second, all threads
    budget = 90.0 / max(1, args.steps + args.warmup)          # seconds per step
    n = int(max(1, min(len(all_items), budget * rate)))
    pos = 0
    total_b, total_t, used = 0.0, 0.0, 1
    for k in range(args.warmup + args.steps):
        items = [all_items[(pos + m) % len(all_items)] for m in range(n)]
        pos += n
        dt, used = _oracle_rate(wl, kc, vc, items)
        if k >= args.warmup:
            total_t += dt
            total_b += _item_bytes(wl, items)
    value = total_b / total_t / 1e9
    ms = total_t / args.steps * 1e3
    sample = (f"{n} (sequence, query head) items per step, cycling through the workload; "
              f"fp64 C oracle, OpenMP over items")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) tensors)",
            "config": workload_config(wl, c.partition_size),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": used,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _event_time_ms(fn, steps, warmup, flush=None):
    """Mean device time of fn() over `steps` calls (CUDA events on the current
    stream), after `warmup` calls; `flush` runs untimed before each call."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(steps):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        total += a.elapsed_time(b)
    return total / steps


def run_block_ops(args, dev):
    """Block copies and the host block manager, each as one JSON line."""
    from paged_kv_cache_367_b200.blocks import BlockManager
    peak, peak_src = measured_hbm_peak()
    steps, warmup = max(args.steps // 50, 10), max(args.warmup, 3)
    bs, Hkv, D = 16, 8, 128                      # the 70B-class GQA pool: 32 KB per K block
    nb = 16384                                   # 1 GiB of K+V
    gen = torch.Generator(device=dev).manual_seed(1)
    kc = torch.randn((nb, bs, Hkv, D), generator=gen, device=dev).to(torch.bfloat16)
    vc = torch.randn((nb, bs, Hkv, D), generator=gen, device=dev).to(torch.bfloat16)
    bb = bs * Hkv * D * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    lines = []
    for n in (64, 4096):
        perm = torch.randperm(nb, generator=torch.Generator().manual_seed(n))[:2 * n]
        pairs = perm.view(n, 2).to(torch.int64).to(dev)
        ms = _event_time_ms(lambda: pkv.paged_kv_copy_blocks(kc, vc, pairs), steps, warmup,
                            flush=flush.zero_)
        byt = 2 * 2 * n * bb                     # K and V, read and write
        gbs = byt / ms / 1e6
        lines.append({"metric": "paged_kv_copy_blocks (copy-on-write) HBM GB/s", "value": round(gbs, 1),
                      "unit": "GB/s", "higher_is_better": True, "us_per_call": round(ms * 1e3, 2),
                      "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": f"{n} random block pairs of a [{nb}, {bs}, {Hkv}, {D}] "
                                             "bf16 pool (K and V)", "l2": "flushed before each call"},
                      "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                                   "peak_source": peak_src, "unit": "GB/s",
                                   "frac": round(gbs / peak, 4), "traffic": None,
                                   "bytes": byt}})
    # Swap: n blocks device -> pinned host and back, against one contiguous copy
    # of the same bytes through the copy engine.
    n = 2048
    hk = torch.empty((n, bs, Hkv, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    src = torch.randperm(nb, generator=torch.Generator().manual_seed(3))[:n].to(torch.int64)
    out_pairs = torch.stack([src, torch.arange(n)], 1).to(dev)
    in_pairs = torch.stack([torch.arange(n), src.flip(0)], 1).to(dev)
    byt = 2 * n * bb
    ms_out = _event_time_ms(lambda: pkv.paged_kv_swap_blocks(kc, vc, hk, hv, out_pairs), steps,
                            warmup)
    ms_in = _event_time_ms(lambda: pkv.paged_kv_swap_blocks(hk, hv, kc, vc, in_pairs), steps,
                           warmup)
    big = torch.empty(2 * n * bb, dtype=torch.uint8).pin_memory()
    dbig = torch.empty(2 * n * bb, dtype=torch.uint8, device=dev)
    ms_d2h = _event_time_ms(lambda: big.copy_(dbig, non_blocking=True), steps, warmup)
    ms_h2d = _event_time_ms(lambda: dbig.copy_(big, non_blocking=True), steps, warmup)
    for name, ms, ref in (("swap-out (device -> pinned host)", ms_out, ms_d2h),
                          ("swap-in (pinned host -> device)", ms_in, ms_h2d)):
        gbs, ref_gbs = byt / ms / 1e6, byt / ref / 1e6
        lines.append({"metric": f"paged_kv_swap_blocks {name} GB/s", "value": round(gbs, 2),
                      "unit": "GB/s", "higher_is_better": True, "ms_per_call": round(ms, 3),
                      "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": f"{n} scattered blocks of 32 KB, K and V "
                                             f"({byt / 2**20:.0f} MiB)"},
                      "roofline": {"bound": "host link", "achieved": round(gbs, 2),
                                   "peak": round(ref_gbs, 2),
                                   "peak_source": "one contiguous pinned cudaMemcpyAsync of the "
                                                  "same bytes, measured in this run",
                                   "unit": "GB/s", "frac": round(gbs / ref_gbs, 4),
                                   "traffic": None}})
    # Host block manager: a decode-serving trace of 128 sequences.
    S, steps_bm = 128, 2000
    rng = np.random.default_rng(0)
    bm = BlockManager(S * ((8192 + steps_bm) // 16 + 2), 16, prefix_caching=True)
    system = rng.integers(0, 32000, size=1024).astype(np.int32)
    prompts = [np.concatenate([system, rng.integers(0, 32000, size=int(rng.integers(16, 4096)))
                               .astype(np.int32)]) for _ in range(S)]
    t0 = time.perf_counter()
    for s in range(S):
        bm.allocate(s, prompts[s])
    t1 = time.perf_counter()
    toks = rng.integers(0, 32000, size=(2 * steps_bm, S)).astype(np.int32)
    ids = np.arange(S, dtype=np.int64)
    for k in range(steps_bm):                    # one append_slots call per decode step
        bm.append_slots(ids, toks[k])
    t2 = time.perf_counter()
    for k in range(steps_bm, 2 * steps_bm):      # one append_slot call per sequence
        for s in range(S):
            bm.append_slot(s, int(toks[k, s]))
    t3 = time.perf_counter()
    lines.append({"metric": "host block manager: sequence appends per second (batched step call)",
                  "value": round(S * steps_bm / (t2 - t1), 0), "unit": "appends/s",
                  "higher_is_better": True,
                  "us_per_decode_step": round((t2 - t1) / steps_bm * 1e6, 2),
                  "us_per_decode_step_one_call_per_sequence":
                      round((t3 - t2) / steps_bm * 1e6, 2),
                  "allocate_ms_per_prompt": round((t1 - t0) / S * 1e3, 4),
                  "config": {"workload": f"{S} sequences with a shared 1024-token prompt plus "
                                         "U[16, 4096] own tokens (prefix caching on), "
                                         f"{steps_bm} decode steps, through the Python binding; "
                                         "prompts built as int32 arrays before the timed admission"},
                  "data": "synthetic"})
    return lines


def run_block_sizes(args, dev):
    """Decode time of the workload at block sizes 8, 16 and 32 (same lengths),
    and the pool fragmentation of its lengths and of a short-request mix under
    fixed blocks, the dynamic page-size policy and whole-length reservation."""
    from paged_kv_cache_367_b200 import fragmentation as FR
    peak, peak_src = measured_hbm_peak()
    base = W.CONFIGS[args.workload]
    lines = []
    reps, warmup = max(args.steps // 20, 20), max(args.warmup, 3)
    for bs in (8, 16, 32):
        wl = W.make_workload(base.replace(block_size=bs), device=dev)
        c = wl.cfg
        P = c.partition_size
        bt = torch.from_numpy(wl.block_table).to(dev)
        sl = torch.from_numpy(wl.seq_lens).to(dev)
        nbytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                    c.head_dim, wl.max_seq_len, P)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
        out = torch.empty_like(wl.query)
        ks = vs = None
        if c.cache_dtype == "e4m3":
            ks = torch.tensor([wl.k_scale], device=dev)
            vs = torch.tensor([wl.v_scale], device=dev)

        def call(flags=pkv.PKV_DECODE_ZEROED_WORKSPACE):
            pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, sl,
                                       max_seq_len=wl.max_seq_len, scale=c.scale,
                                       partition_size=P, workspace=ws, k_scale=ks, v_scale=vs,
                                       flags=flags)
        call(0)  # zeroes the split counters; every call leaves them zero
        ms, how = kernel_time_ms(lambda: None, call, reps=max(3, reps // 4))
        dec, _ = step_bytes(wl)
        gbs = dec / ms / 1e6
        lines.append({"metric": "paged decode attention HBM GB/s by block size", "value": round(gbs, 1),
                      "unit": "GB/s", "higher_is_better": True, "block_size": bs,
                      "us_per_launch": round(ms * 1e3, 2), "timing": how, "dtype": c.q_dtype,
                      "data": "synthetic", "config": {"workload": WORKLOAD_TEXT.get(
                          args.workload, args.workload).replace("block 16", f"block {bs}")},
                      "fragmentation": round(FR.fixed_block_fragmentation(wl.seq_lens, bs), 5),
                      "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                                   "peak_source": peak_src, "unit": "GB/s",
                                   "frac": round(gbs / peak, 4), "traffic": None}})
        del wl, out, ws
        torch.cuda.empty_cache()
    lens = W.draw_seq_lens(base, np.random.default_rng(base.seed))
    short = np.random.default_rng(7).integers(16, 161, size=128)
    for name, L in ((args.workload + " lengths", lens), ("128 short requests U[16, 160]", short)):
        lines.append({"metric": "KV pool fragmentation (allocated - used) / allocated",
                      "unit": "fraction", "higher_is_better": False, "lengths": name,
                      "value": round(FR.fixed_block_fragmentation(L, 16), 5),
                      "fixed": {str(b): round(FR.fixed_block_fragmentation(L, b), 5)
                                for b in (8, 16, 32)},
                      "dynamic_page_size": round(FR.dynamic_fragmentation(L), 5),
                      "reservation_to_max_len": round(
                          FR.reservation_fragmentation(L, int(max(L))), 5),
                      "data": "synthetic"})
    return lines


def run_decode_kernels(args, dev):
    """Where the decode's products run: the TMA-fed kernel with Q K^T and P V on
    the tensor cores (mma.sync) or on the CUDA cores (fp32 FMA), and the plain
    CUDA-core kernel without TMA staging (PKV_DECODE_FORCE_SIMT), on the MHA
    workload (one query head per KV head), the 70B-class shape with 4 query heads
    per KV head, and the 70B-class GQA workload (8). Each timed alone per launch
    (events inside a CUDA graph), same inputs and split."""
    peak, peak_src = measured_hbm_peak()
    lines = []
    cases = [("llama2_13b_mha", W.CONFIGS["llama2_13b_mha"]),
             ("gqa70b_g4", W.CONFIGS["gqa70b"].replace(num_heads=32)),
             ("gqa70b", W.CONFIGS["gqa70b"])]
    kernels = [(pkv.PKV_DECODE_TENSOR_CORES, "decode_tc_kernel, products on the tensor cores "
                                             "(mma.sync m16n8k16, S^T = K Q^T)"),
               (pkv.PKV_DECODE_CUDA_CORES, "decode_tc_kernel, products on the CUDA cores "
                                           "(fp32 FMA, lanes over head_dim)"),
               (pkv.PKV_DECODE_FORCE_SIMT, "decode_simt_kernel: CUDA cores, plain loads (no TMA)")]
    for name, cfg in cases:
        wl = W.make_workload(cfg, device=dev)
        c = wl.cfg
        g = c.num_heads // c.num_kv_heads
        bt = torch.from_numpy(wl.block_table).to(dev)
        sl = torch.from_numpy(wl.seq_lens).to(dev)
        slots = torch.from_numpy(wl.slot_mapping).to(dev)
        pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots)
        P = c.partition_size
        nbytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                    c.head_dim, wl.max_seq_len, P)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
        out = torch.empty_like(wl.query)
        dec, _ = step_bytes(wl)
        for flags, kname in kernels:
            if flags == pkv.PKV_DECODE_CUDA_CORES and g > 4:
                continue  # the CUDA-core products serve groups of up to 4 heads
            def call(f=flags):
                pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, sl,
                                           max_seq_len=wl.max_seq_len, scale=c.scale,
                                           partition_size=P, workspace=ws,
                                           flags=f | pkv.PKV_DECODE_ZEROED_WORKSPACE)
            pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, sl,
                                       max_seq_len=wl.max_seq_len, scale=c.scale,
                                       partition_size=P, workspace=ws, flags=flags)
            if args.no_graph:  # eager launches (e.g. under a profiler): warmup, then steps
                ms, how = _event_time_ms(call, args.steps, args.warmup), "CUDA events, eager launches"
            else:
                ms, how = kernel_time_ms(lambda: None, call, reps=max(3, args.steps // 50))
            assert pkv.pkv_device_status(clear=True) == 0, "device wait expired"
            gbs = dec / ms / 1e6
            text = WORKLOAD_TEXT.get(name, WORKLOAD_TEXT["gqa70b"].replace("64 q / 8 KV", "32 q / 8 KV"))
            lines.append({"metric": "paged decode attention HBM GB/s by kernel", "value": round(gbs, 1),
                          "unit": "GB/s", "higher_is_better": True, "kernel": kname,
                          "us_per_launch": round(ms * 1e3, 2), "timing": how,
                          "group_size": g, "dtype": c.q_dtype, "data": "synthetic",
                          "config": {"workload": text, "partition_size": P},
                          "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                                       "peak_source": peak_src, "unit": "GB/s",
                                       "frac": round(gbs / peak, 4), "traffic": None,
                                       "bytes": dec}})
        del wl, out, ws
        torch.cuda.empty_cache()
    return lines


def measured_bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured burst (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:
        return 1590.0, "fallback 1.59 PFLOP/s"


def run_prefill(args, dev):
    """Causal multi-token queries over the paged cache: a chunked-prefill step
    (chunks of 1024 tokens continuing cached contexts) and full prefills, in the
    70B-class GQA shape. TFLOP/s counts 4 * head_dim flops per (query head, row,
    attended token): the two contractions of the causal range, nothing masked."""
    peak, peak_src = measured_bf16_peak()
    Hq, Hkv, D, bs = 64, 8, 128, 16
    lines = []
    reps, warmup = max(args.steps // 20, 20), max(args.warmup, 3)
    for name, ctx, qlen in (("chunked prefill: 8 sequences, 1024-token chunks after 2048 "
                             "cached tokens", [3072] * 8, [1024] * 8),
                            ("full prefill: 4 prompts of 4096 tokens", [4096] * 4, [4096] * 4),
                            ("full prefill: 16 prompts of 512 tokens", [512] * 16, [512] * 16)):
        S = len(ctx)
        nbs = [-(-L // bs) for L in ctx]
        nb = sum(nbs)
        g = torch.Generator(device=dev).manual_seed(5)
        kc = torch.randn((nb, bs, Hkv, D), generator=g, device=dev).to(torch.bfloat16)
        vc = torch.randn((nb, bs, Hkv, D), generator=g, device=dev).to(torch.bfloat16)
        perm = torch.randperm(nb, generator=torch.Generator().manual_seed(6)).to(torch.int32)
        bt = torch.full((S, max(nbs)), -1, dtype=torch.int32)
        o = 0
        for i, k in enumerate(nbs):
            bt[i, :k] = perm[o:o + k]
            o += k
        qs = torch.tensor(np.concatenate([[0], np.cumsum(qlen)]), dtype=torch.int32)
        T = int(qs[-1])
        q = torch.randn((T, Hq, D), generator=g, device=dev).to(torch.bfloat16)
        out = torch.empty_like(q)
        btd, lensd, qsd = bt.to(dev), torch.tensor(ctx, dtype=torch.int32, device=dev), qs.to(dev)

        attended = sum(sum(L - n + r + 1 for r in range(n)) for L, n in zip(ctx, qlen))
        flops = 4.0 * D * Hq * attended
        for flags, kname in ((0, "tcgen05.mma, accumulators in tensor memory"),
                             (pkv.PKV_PREFILL_MMA_SYNC, "mma.sync m16n8k16 (legacy tensor path)")):
            def call():
                pkv.paged_attention_prefill(out, q, kc, vc, btd, lensd, qsd, max_q_len=max(qlen),
                                            scale=D ** -0.5, flags=flags)
            ms, how = kernel_time_ms(lambda: None, call, n=8, reps=max(3, reps // 8))
            assert pkv.pkv_device_status(clear=True) == 0, "device wait expired"
            tflops = flops / ms / 1e9
            lines.append({"metric": "paged causal multi-token attention TFLOP/s",
                          "value": round(tflops, 1), "unit": "TFLOP/s", "higher_is_better": True,
                          "us_per_launch": round(ms * 1e3, 1), "timing": how,
                          "tokens_per_s": round(T / ms * 1e3, 0), "dtype": "bf16",
                          "data": "synthetic",
                          "config": {"workload": name + f"; {Hq} q / {Hkv} KV heads, head_dim {D}, "
                                                        f"block {bs}, shuffled pool"},
                          "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                                       "peak_source": peak_src, "unit": "TFLOP/s",
                                       "frac": round(tflops / peak, 4), "traffic": None,
                                       "flops": flops, "kernel": kname}})
        # The same queries over an E4M3 cache (codes as in the workload generator,
        # per-tensor scales), on the tcgen05 kernel.
        kc8 = (kc.float() * (448.0 / 4.0)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        vc8 = (vc.float() * (448.0 / 4.0)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        sc = torch.tensor([4.0 / 448.0], dtype=torch.float32, device=dev)

        def call8():
            pkv.paged_attention_prefill(out, q, kc8, vc8, btd, lensd, qsd, max_q_len=max(qlen),
                                        scale=D ** -0.5, k_scale=sc, v_scale=sc)
        ms, how = kernel_time_ms(lambda: None, call8, n=8, reps=max(3, reps // 8))
        assert pkv.pkv_device_status(clear=True) == 0, "device wait expired"
        tflops = flops / ms / 1e9
        lines.append({"metric": "paged causal multi-token attention TFLOP/s",
                      "value": round(tflops, 1), "unit": "TFLOP/s", "higher_is_better": True,
                      "us_per_launch": round(ms * 1e3, 1), "timing": how,
                      "tokens_per_s": round(T / ms * 1e3, 0),
                      "dtype": "f16 MMAs over an e4m3 cache (bf16 query and output)",
                      "data": "synthetic",
                      "config": {"workload": name + f"; {Hq} q / {Hkv} KV heads, head_dim {D}, "
                                                    f"block {bs}, shuffled pool, FP8-E4M3 cache"},
                      "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                                   "peak_source": peak_src, "unit": "TFLOP/s",
                                   "frac": round(tflops / peak, 4), "traffic": None,
                                   "flops": flops,
                                   "kernel": "tcgen05.mma over codes widened to f16 in shared memory"}})
        del kc, vc, kc8, vc8, q, out
        torch.cuda.empty_cache()
    return lines


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        if args.op in ("blocks", "blocksize", "prefill", "kernels"):
            if rank == 0:
                fn = {"blocks": run_block_ops, "blocksize": run_block_sizes,
                      "prefill": run_prefill, "kernels": run_decode_kernels}[args.op]
                for line in fn(args, dev):
                    print(json.dumps(line), flush=True)
            return
        res = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
