#!/usr/bin/env python
"""Decode benchmark for QK-Normed MLA on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole decode hot path over one batch: append the
step's new tokens (latent, RoPE key, a_k), absorb the step's queries, split-KV
decode and combine.  Inputs are seeded synthetic tensors shaped like the
named workload (default: large_mla_bf16, 32 sequences of 1,024 to 32,768
tokens in a paged cache, 128 heads, r = 512, d_R = 64, bf16: the largest
workload that fits one GPU).  Each rank runs its own replica (its own sequences;
weak scaling, no collective on the data path); the step time is the max over
ranks of CUDA-event time.  Every step is a CUDA graph replay; consecutive
steps read different copies of the cache so that the working set of the timed
steps is larger than L2.

One JSON line on rank 0 carries the whole-job decode tokens/s, the decode
kernel's roofline fraction, the overhead against the same kernel with a_k
fixed to 1 (plain MLA), an end-to-end figure through the public API with
host buffers, SM clocks sampled while the GPU was under this load, and the
fp64 oracle's throughput on this host's cores.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and us/step at 1 B200; % of HBM/tensor roofline; overhead vs MLA"
# kernels of libqkn launched per step: append + absorb (one launch), split-KV decode, merge
LAUNCHES_PER_STEP = 3              # preparation (one launch up to 256 new tokens, else two), split-KV, merge
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="large_mla_bf16")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--kernel", choices=["auto", "simt", "tcgen05"], default="auto")
    p.add_argument("--head-tile", type=int, default=0, choices=[0, 16, 32, 64, 128],
                   help="query rows per tcgen05 tile (128: the CTA-pair kernel); 0 = automatic")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--soak-seconds", type=float, default=1.0, help="load window around the timed steps for clocks")
    p.add_argument("--overhead-rounds", type=int, default=5)
    p.add_argument("--route", choices=["absorbed", "gqa"], default="absorbed",
                   help="decode route: the absorbed latent decode, or GQLA's GQA route over keys and values "
                        "expanded per group (workloads with one key and one value head per group)")
    p.add_argument("--cp-emulate", type=int, default=0,
                   help="also time a context-parallel decode over this many ranks, emulated on one GPU "
                        "(every rank's slice decode and the merge of the partials; one GPU only)")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    if a.steps < 1:
        p.error("--steps must be >= 1")
    return a


# ----------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_workload(name: str, rank: int):
    """The workload replica of one rank: same shapes, its own sequences (seed offset by rank)."""
    from qkn_inputs import WORKLOADS
    wl = WORKLOADS[name]
    return wl.with_(seed=wl.seed + rank)


def job_throughput(tokens_per_rank: int, world: int, local_ms_total: float, steps: int, device=None):
    """Whole-job tokens/s and ms per step: every rank's tokens over the slowest rank's time."""
    step_ms = reduce_max(local_ms_total, device) / steps
    return world * tokens_per_rank / (step_ms * 1e-3), step_ms


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- CUDA events that survive capture
def load_traffic(workload: str):
    """DRAM bytes per launch of the split-KV kernel from the committed ncu capture, if that capture
    was taken on this workload with the kernel source as it is now; else None."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "profiles", "decode_tc_traffic.json")) as f:
            rec = json.load(f)
        with open(os.path.join(here, rec["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("workload") != workload or rec.get("source_sha256") != sha:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


class Events:
    """Raw cudaEvent_t handles recorded with cudaEventRecordExternal, so that a
    record inside stream capture becomes an event node of the graph."""

    def __init__(self):
        import torch
        lib = None
        for cand in ("libcudart.so.12", "libcudart.so"):
            try:
                lib = ctypes.CDLL(cand)
                break
            except OSError:
                continue
        if lib is None:
            base = os.path.join(os.path.dirname(os.path.dirname(torch.__file__)), "nvidia", "cuda_runtime", "lib")
            lib = ctypes.CDLL(os.path.join(base, "libcudart.so.12"))
        self.lib = lib
        lib.cudaEventCreate.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
        lib.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        lib.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p, ctypes.c_void_p]
        lib.cudaEventDestroy.argtypes = [ctypes.c_void_p]

    def create(self) -> int:
        h = ctypes.c_void_p()
        assert self.lib.cudaEventCreate(ctypes.byref(h)) == 0
        return h.value

    def record(self, ev: int, stream: int) -> None:
        assert self.lib.cudaEventRecordWithFlags(ctypes.c_void_p(ev), ctypes.c_void_p(stream), 1) == 0

    def ms(self, a: int, b: int) -> float:
        out = ctypes.c_float()
        rc = self.lib.cudaEventElapsedTime(ctypes.byref(out), ctypes.c_void_p(a), ctypes.c_void_p(b))
        assert rc == 0, rc
        return float(out.value)


# ----------------------------------------------------------------- clocks
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the GPU is loaded."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.period = [], set(), period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            self.h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    h = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(h)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.nvml, self.error = None, str(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for b, name in REASON_BITS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml:
            self.t.join()

    def summary(self, window_s: float):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "window_s": round(window_s, 2), "source": "nvml"}


# ----------------------------------------------------------------- oracle CPU baseline
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_throughput(inp, budget_s: float, max_seqs=None):
    """Decode tokens/s of the fp64 oracle: whole sequences of the workload until the budget is spent."""
    import oracle
    wl = inp.wl
    done, t0 = 0, time.perf_counter()
    order = list(range(wl.batch)) if max_seqs is None else list(range(min(wl.batch, max_seqs)))
    for b in order:
        oracle.decode_sequence(inp, b)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return done * wl.s_q / el, done, el


# ----------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import torch
    import qk_normed_latent_qkn_b200 as qkn
    from qk_normed_latent_qkn_b200.roofline import decode_step_cost, merge_cost, split_counts
    from qk_normed_latent_qkn_b200.session import DecodeSession, session_from_inputs
    from qkn_inputs import WORKLOADS, make_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = rank_workload(args.workload, rank)
    kernel = {"auto": qkn.KERNEL_AUTO, "simt": qkn.KERNEL_SIMT, "tcgen05": qkn.KERNEL_TCGEN05}[args.kernel]
    inp = make_inputs(wl)
    B, s_q, H = wl.batch, wl.s_q, wl.heads
    n_q = B * s_q

    # per-step inputs: the step's new tokens (the last s_q of every sequence) and its queries
    last = np.concatenate([np.arange(inp.tok_off[b + 1] - s_q, inp.tok_off[b + 1]) for b in range(B)])
    slots, poss = inp.token_slots()[last], inp.token_positions()[last]
    host = {
        "c": inp.c[last], "kr": inp.k_rope[last], "slot": slots, "pos": poss,
        "q": inp.q.reshape(n_q, H, wl.d_h), "qr": inp.q_rope.reshape(n_q, H, wl.d_rope),
        "qpos": inp.query_positions().reshape(-1), "bt": inp.block_table, "sl": inp.seq_lens,
    }
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    types = {"c": dt, "kr": dt, "slot": torch.int32, "pos": torch.int32, "q": dt, "qr": dt,
             "qpos": torch.int32, "bt": torch.int32, "sl": torch.int32}

    base = session_from_inputs(inp, device=device)
    cache_bytes = sum(t.numel() * t.element_size() for t in (base.cache.latent, base.cache.k_rope, base.cache.a_k))
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    n_copies = max(1, min(16, math.ceil(3 * l2 / cache_bytes))) if cache_bytes < 2 * l2 else 1
    sessions = [base]
    for _ in range(n_copies - 1):
        s = DecodeSession(base.dims, inp.num_blocks, device=device)
        s.cache.latent.copy_(base.cache.latent)
        s.cache.k_rope.copy_(base.cache.k_rope)
        s.cache.a_k.copy_(base.cache.a_k)
        s.load_weights(base.w_k, base.gamma_q, base.gamma_k, base.gamma_qr, base.gamma_kr)
        s.w_uv = base.w_uv.clone()             # its own W^UV, so that no copy finds it in L2
        sessions.append(s)
    dev_in = [{k: torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=types[k]) for k, v in
               host.items()} for _ in sessions]
    outs = [(torch.empty((B, s_q, H, wl.r_kv), dtype=dt, device=device),
             torch.empty((B, s_q, H), dtype=torch.float32, device=device)) for _ in sessions]
    outs_v = [(torch.empty((B, s_q, H, wl.d_v), dtype=dt, device=device),
               torch.empty((B, s_q, H), dtype=torch.float32, device=device)) for _ in sessions]

    evs = torch.cuda.Stream(device=device)

    def step(i, split_event=None, ak_mode=qkn.AK_CACHE, start_event=None, end_event=None):
        """Append and absorb in one launch, then the split-KV decode and its merge, all on one stream.
        The start event is recorded on a branch that joins only at the end of the step, so that no
        graph node sits between the preparation and the decode."""
        s, d, (o, l) = sessions[i], dev_in[i], outs[i]
        main = torch.cuda.current_stream(device)
        s.prepare(d["c"], d["kr"], d["slot"], d["pos"], d["q"], d["qr"], d["qpos"])
        if start_event is not None:
            evs.wait_stream(main)
            ev.record(start_event, evs.cuda_stream)
        s.decode(d["bt"], d["sl"], s_q, out=o, lse=l, ak_mode=ak_mode, kernel=kernel, split_event=split_event,
                 step_writes_only=True, head_tile=args.head_tile)
        if end_event is not None:
            ev.record(end_event, main.cuda_stream)
        if start_event is not None:
            main.wait_stream(evs)

    def decode_only(i, split_event=None, ak_mode=qkn.AK_CACHE):
        s, d, (o, l) = sessions[i], dev_in[i], outs[i]
        s.decode(d["bt"], d["sl"], s_q, out=o, lse=l, ak_mode=ak_mode, kernel=kernel, split_event=split_event,
                 head_tile=args.head_tile)

    def decode_up_only(i, split_event=None):
        s, d, (ov, l) = sessions[i], dev_in[i], outs_v[i]
        s.decode_up(d["bt"], d["sl"], s_q, out_v=ov, lse=l, kernel=kernel, split_event=split_event,
                    head_tile=args.head_tile)

    ev = Events()
    stream = torch.cuda.Stream(device=device)

    # eager warm-up: first-call attributes, workspaces, absorbed queries
    for i in range(len(sessions)):
        step(i)
        step(i, ak_mode=qkn.AK_ONE)
        decode_up_only(i)
    torch.cuda.synchronize(device)
    status = [s.device_status() for s in sessions]
    assert all(v == qkn.OK for v in status), f"device status {status}"
    kernel_used = qkn.decode_kernel_for(base.dims, s_q, kernel=kernel, head_tile=args.head_tile)

    total = args.warmup + args.steps
    graphs, marks = [], []
    with torch.cuda.stream(stream):
        for k in range(total):
            i = k % n_copies
            # two event nodes per step, around the decode op (split-KV kernel + merge kernel, chained
            # by programmatic launch with no node between them): reported as decode_op_in_step
            e = [ev.create() for _ in range(2)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                step(i, start_event=e[0], end_event=e[1])
            graphs.append(g)
            marks.append(e)
        # decode-only graphs, QK-Normed and plain MLA: events before the split-KV kernel, between it
        # and the merge, and after the merge.  Nothing runs before the split-KV kernel, so its
        # duration holds every page read it makes (the roofline's figure) and the overhead figure
        # compares the two modes' split-KV kernels alone.
        over = {}
        for mode in (qkn.AK_CACHE, qkn.AK_ONE):
            lst = []
            for i in range(n_copies):
                e = [ev.create() for _ in range(3)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                    ev.record(e[0], stream.cuda_stream)
                    decode_only(i, split_event=e[1], ak_mode=mode)
                    ev.record(e[2], stream.cuda_stream)
                lst.append((g, e))
            over[mode] = lst
        # decode-only graphs with the value up-projection fused into the merge: events before the
        # split-KV kernel, between it and the fused merge, and after
        up_graphs = []
        for i in range(n_copies):
            e = [ev.create() for _ in range(3)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                ev.record(e[0], stream.cuda_stream)
                decode_up_only(i, split_event=e[1])
                ev.record(e[2], stream.cuda_stream)
            up_graphs.append((g, e))
    torch.cuda.synchronize(device)

    soak_graphs = graphs[:n_copies] if len(graphs) >= n_copies else graphs

    def soak(seconds):
        t_end = time.perf_counter() + seconds
        with torch.cuda.stream(stream):
            while time.perf_counter() < t_end:
                for g in soak_graphs:
                    g.replay()
                stream.synchronize()

    t_start_ev = torch.cuda.Event(enable_timing=True)
    t_end_ev = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    w0 = time.perf_counter()
    with sampler:
        soak(args.soak_seconds)
        with torch.cuda.stream(stream):
            for k in range(args.warmup):
                graphs[k].replay()
        barrier(device)
        torch.cuda.synchronize(device)
        with torch.cuda.stream(stream):
            t_start_ev.record(stream)
            for k in range(args.warmup, total):
                graphs[k].replay()
            t_end_ev.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        soak(args.soak_seconds)
    window = time.perf_counter() - w0
    local_ms = t_start_ev.elapsed_time(t_end_ev)
    value, step_ms = job_throughput(B * s_q, world, local_ms, args.steps, device)

    op_ms = [ev.ms(marks[k][0], marks[k][1]) for k in range(args.warmup, total)]

    # breakdown of one step (separate graphs with an event node between every stage; not the timed region)
    bd_graphs = []
    with torch.cuda.stream(stream):
        for i in range(n_copies):
            e = [ev.create() for _ in range(4)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                sid = stream.cuda_stream
                ev.record(e[0], sid)
                step(i, split_event=e[2], start_event=e[1])
                ev.record(e[3], sid)
            bd_graphs.append((g, e))
    prep_ms, split_ms, combine_ms = [], [], []
    with torch.cuda.stream(stream):
        for _ in range(3):
            for g, e in bd_graphs:
                g.replay()
                stream.synchronize()
                prep_ms.append(ev.ms(e[0], e[1]))
                split_ms.append(ev.ms(e[1], e[2]))
                combine_ms.append(ev.ms(e[2], e[3]))

    # overhead vs plain MLA: interleaved rounds of decode-only graphs; the same replays give the
    # split-KV kernel's launch duration for the roofline and the split + merge op
    per_mode = {qkn.AK_CACHE: [], qkn.AK_ONE: []}
    op_only, merge_only, up_merge, up_op = [], [], [], []
    with torch.cuda.stream(stream):
        for _ in range(args.overhead_rounds):
            for mode in (qkn.AK_CACHE, qkn.AK_ONE):
                for g, _e in over[mode]:
                    g.replay()
                stream.synchronize()
                per_mode[mode] += [ev.ms(e[0], e[1]) for _g, e in over[mode]]
                if mode == qkn.AK_CACHE:
                    op_only += [ev.ms(e[0], e[2]) for _g, e in over[mode]]
                    merge_only += [ev.ms(e[1], e[2]) for _g, e in over[mode]]
            for g, _e in up_graphs:
                g.replay()
            stream.synchronize()
            up_merge += [ev.ms(e[1], e[2]) for _g, e in up_graphs]
            up_op += [ev.ms(e[0], e[2]) for _g, e in up_graphs]
    t_qkn = statistics.median(per_mode[qkn.AK_CACHE])
    t_mla = statistics.median(per_mode[qkn.AK_ONE])
    t_split_avg = statistics.mean(per_mode[qkn.AK_CACHE])

    # end to end through the public API: DecodeStep replays copy-in, append + absorb (one launch), decode and
    # copy-out as one graph per step, from and to pinned host buffers, with a synchronize per step
    from qk_normed_latent_qkn_b200.step import DecodeStep
    names = {"c": "c", "kr": "k_rope", "slot": "slot", "pos": "pos", "q": "q", "qr": "q_rope", "qpos": "qpos",
             "bt": "block_table", "sl": "seq_lens"}
    steps = []
    for i in range(n_copies):
        st = DecodeStep(sessions[i], B, s_q, inp.block_table.shape[1], len(last), kernel=kernel,
                        head_tile=args.head_tile)
        for key, name in names.items():
            st.host_in[name].copy_(torch.from_numpy(np.ascontiguousarray(host[key])).to(st.host_in[name].dtype))
        st.capture()
        steps.append(st)
    h2d, d2h = steps[0].h2d_bytes, steps[0].d2h_bytes

    for k in range(args.warmup):
        steps[k % n_copies].run()
    barrier(device)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(args.steps):
        steps[k % n_copies].run()
    e1.record()
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1), device) / args.steps
    assert all(s.device_status() == qkn.OK for s in sessions)

    # roofline of the dominant kernel (the split-KV decode kernel)
    cost = decode_step_cost(inp.seq_lens, s_q, H, wl.groups, wl.r_kv, wl.d_rope,
                            elem=2 if wl.dtype == "bf16" else 4)
    peaks, peak_src = load_peaks()
    op_avg = statistics.mean(op_ms)
    # the dominant kernel is the split-KV kernel: its average launch duration with nothing started early
    achieved_gbs = cost.bytes / (t_split_avg * 1e-3) / 1e9
    tflops = cost.flops / (t_split_avg * 1e-3) / 1e12
    op_only_avg = statistics.mean(op_only)
    tokens = world * B * s_q
    traffic = load_traffic(wl.name) if kernel_used == qkn.KERNEL_TCGEN05 else None
    # the merge kernels' rooflines: partial rows read per the split schedule of this launch
    rows_t, ncta_t, item_cost_t = schedule_shape(kernel_used, args.head_tile, s_q, H,
                                                 torch.cuda.get_device_properties(device).multi_processor_count)
    splits = split_counts(inp.seq_lens, s_q, inp.block_table.shape[1], -(-s_q * H // rows_t), ncta_t, item_cost_t)
    elem = 2 if wl.dtype == "bf16" else 4
    m_plain = merge_cost(splits, s_q, H, wl.r_kv, elem)
    m_up = merge_cost(splits, s_q, H, wl.r_kv, elem, d_v=wl.d_v)
    t_merge, t_up = statistics.mean(merge_only), statistics.mean(up_merge)

    line = None
    tensor_bound = cost.flops / cost.bytes > peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tps, nseq, el = oracle_throughput(inp, args.cpu_seconds)
            cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{nseq} of {B} sequences of the workload ({nseq * s_q} query tokens, "
                             f"{int(inp.seq_lens[:nseq].sum())} cached tokens) in {el:.1f} s, fp64 numpy"}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "us_per_step": step_ms * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(workload_config(wl, inp, world),
                           kernel={qkn.KERNEL_TCGEN05: "tcgen05", qkn.KERNEL_SIMT: "simt"}.get(kernel_used),
                           head_tile=args.head_tile or "auto",
                           l2=f"{n_copies} rotating cache copies, {n_copies * cache_bytes / 2**20:.0f} MiB "
                              f"(L2 {l2 / 2**20:.0f} MiB)", step_launch="CUDA graph per step"),
            "breakdown_us": {"append_absorb": statistics.median(prep_ms) * 1e3,
                             "decode_split": statistics.median(split_ms) * 1e3,
                             "combine": statistics.median(combine_ms) * 1e3,
                             "decode_op_in_step": op_avg * 1e3, "decode_op_alone": op_only_avg * 1e3,
                             "what": "append + absorb (one launch) / split-KV kernel / merge kernel, from "
                                     "separate graphs with an event between every stage; decode_op_in_step is the "
                                     "split-KV + merge pair inside the timed steps, from the end of the preparation "
                                     "kernel (its CTAs may have streamed early pages before that point); "
                                     "decode_op_alone is the same pair replayed alone"},
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                         "intensity_flop_per_byte": cost.flops / cost.bytes,
                         "ridge_flop_per_byte": peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9),
                         "traffic_what": ("DRAM read + write bytes of one split-KV kernel launch from the "
                                          "committed ncu capture (profiles/); null when the kernel source "
                                          "or the workload differs from the capture's"),
                         "algorithmic_bytes": cost.bytes, "peak_source": f"{peak_src} HBM copy bandwidth",
                         "kernel": ("split-KV kernel (%s): mean launch duration over %d replays of decode-only "
                                    "graphs (CUDA events on the launching stream before and after it; nothing "
                                    "starts before it, so the window holds every page read it makes)"
                                    % ("tcgen05" if kernel_used == qkn.KERNEL_TCGEN05 else "simt",
                                       len(per_mode[qkn.AK_CACHE]))),
                         "duration_us": t_split_avg * 1e3,
                         "decode_op_frac": cost.bytes / (op_only_avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "tensor": {"achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                    "frac": tflops / peaks["bf16_tflops"], "flops": cost.flops}},
            "value_up": {
                "d_v": wl.d_v, "op_us": statistics.mean(up_op) * 1e3, "merge_up_us": t_up * 1e3,
                "merge_us": t_merge * 1e3,
                "roofline": {"bound": "hbm", "achieved": m_up.bytes / (t_up * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": m_up.bytes / (t_up * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "algorithmic_bytes": m_up.bytes, "partial_bytes": m_up.partial_bytes,
                             "weight_bytes": m_up.weight_bytes, "flops": m_up.flops},
                "merge_roofline": {"bound": "hbm", "achieved": m_plain.bytes / (t_merge * 1e-3) / 1e9,
                                   "frac": m_plain.bytes / (t_merge * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                   "algorithmic_bytes": m_plain.bytes},
                "what": ("qkn_decode_up replayed alone in decode-only graphs (same rounds as the overhead "
                         "figure): op_us = split-KV kernel + merge fused with the W^UV up-projection; "
                         "merge_up_us = the fused merge kernel alone (event after the split-KV kernel); "
                         "merge_us = qkn_decode's plain merge kernel, measured the same way; bytes = fp32 "
                         "partial rows read per the split schedule + W^UV once + outputs written once"),
            },
            "overhead_vs_mla": {"qkn_us": t_qkn * 1e3, "mla_us": t_mla * 1e3, "frac": t_qkn / t_mla - 1.0,
                                "what": "decode split kernel, a_k cache vs a_k = 1, median of interleaved rounds"},
            "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "DecodeStep.run(): one graph per step with copy-in from pinned host buffers, "
                            "append + absorb (one launch), decode, copy-out to pinned host buffers; synchronize per step"},
            "gpu_launches": (LAUNCHES_PER_STEP + (1 if len(last) > 256 else 0)) * args.steps,
            "clocks": sampler.summary(window),
            "cpu_baseline": cpu,
        }
        if args.cp_emulate > 1 and world == 1:
            line["context_parallel_emulated"] = cp_emulate(args.cp_emulate, base, inp, device, ev, stream)
        if tensor_bound:
            # the step's intensity is above the ridge (every query row sees most of its sequence): the
            # binding roof is the bf16 tensor peak; algorithmic FLOPs count the causal (query, key) pairs
            r = line["roofline"]
            t = r.pop("tensor")
            r["hbm"] = {"achieved": r["achieved"], "peak": r["peak"], "unit": "GB/s", "frac": r["frac"]}
            r.update(bound="tensor", achieved=t["achieved"], peak=t["peak"], unit="TFLOP/s", frac=t["frac"],
                     flops=t["flops"], peak_source=f"{peak_src} bf16 dense GEMM (burst)")
    return line


def run_gqa(args, world, rank, local):
    """GQLA's GQA route: per step, the step's new tokens expanded into the per-group cache
    (qkn_gqa_append) and the dense decode (qkn_gqa_decode: split-KV kernel, then the merge)."""
    import torch
    import qk_normed_latent_qkn_b200 as qkn
    from qk_normed_latent_qkn_b200.roofline import gqa_step_cost
    from qk_normed_latent_qkn_b200.session import GqaSession, gqa_session_from_inputs
    from qkn_inputs import make_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = rank_workload(args.workload, rank)
    if not wl.tied_groups or wl.dtype != "bf16":
        raise SystemExit("--route gqa needs a bf16 workload with one key and one value head per group")
    inp = make_inputs(wl)
    B, s_q, H = wl.batch, wl.s_q, wl.heads
    last = np.concatenate([np.arange(inp.tok_off[b + 1] - s_q, inp.tok_off[b + 1]) for b in range(B)])
    host = {"c": inp.c[last], "kr": inp.k_rope[last], "slot": inp.token_slots()[last],
            "pos": inp.token_positions()[last], "q": inp.q, "qr": inp.q_rope, "bt": inp.block_table,
            "sl": inp.seq_lens}
    types = {"c": torch.bfloat16, "kr": torch.bfloat16, "slot": torch.int32, "pos": torch.int32,
             "q": torch.bfloat16, "qr": torch.bfloat16, "bt": torch.int32, "sl": torch.int32}

    base = gqa_session_from_inputs(inp, device=device)
    cache_bytes = sum(t.numel() * t.element_size() for t in (base.cache.k, base.cache.v, base.cache.k_rope))
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    n_copies = max(1, min(16, math.ceil(3 * l2 / cache_bytes))) if cache_bytes < 2 * l2 else 1
    sessions = [base]
    for _ in range(n_copies - 1):
        s = GqaSession(base.dims, inp.num_blocks, wl.d_v, device=device)
        for dst, src in ((s.cache.k, base.cache.k), (s.cache.v, base.cache.v), (s.cache.k_rope, base.cache.k_rope)):
            dst.copy_(src)
        s.load_weights(base.w_uk, base.gamma_k, base.w_uv.clone(), base.gamma_q, base.gamma_qr, base.gamma_kr)
        sessions.append(s)
    dev_in = [{k: torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=types[k]) for k, v in
               host.items()} for _ in sessions]
    outs = [(torch.empty((B, s_q, H, wl.d_v), dtype=torch.bfloat16, device=device),
             torch.empty((B, s_q, H), dtype=torch.float32, device=device)) for _ in sessions]
    wss = [s.ensure_workspace(B, s_q) for s in sessions]
    ev = Events()
    stream = torch.cuda.Stream(device=device)

    def append(i):
        s, d = sessions[i], dev_in[i]
        qkn.gqa_append(s.dims, s.cache, d["c"], d["kr"], d["slot"], d["pos"], s.w_uk, s.gamma_k, s.w_uv, s.gamma_kr)

    def decode(i):
        s, d, (o, l) = sessions[i], dev_in[i], outs[i]
        qkn.gqa_decode(s.dims, s.cache, d["q"], d["qr"], s.gamma_q, s.gamma_qr, d["bt"], d["sl"], s_q, wss[i], o, l)

    for i in range(n_copies):
        append(i)
        decode(i)
    torch.cuda.synchronize(device)
    assert all(s.device_status() == qkn.OK for s in sessions)

    total = args.warmup + args.steps
    graphs, op_graphs, bd_graphs = [], [], []
    with torch.cuda.stream(stream):
        for k in range(total):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                append(k % n_copies)
                decode(k % n_copies)
            graphs.append(g)
        for i in range(n_copies):
            e = [ev.create() for _ in range(2)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                ev.record(e[0], stream.cuda_stream)
                decode(i)
                ev.record(e[1], stream.cuda_stream)
            op_graphs.append((g, e))
            e = [ev.create() for _ in range(3)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                ev.record(e[0], stream.cuda_stream)
                append(i)
                ev.record(e[1], stream.cuda_stream)
                decode(i)
                ev.record(e[2], stream.cuda_stream)
            bd_graphs.append((g, e))
    torch.cuda.synchronize(device)

    def soak(seconds):
        t_end = time.perf_counter() + seconds
        with torch.cuda.stream(stream):
            while time.perf_counter() < t_end:
                for g in graphs[:n_copies]:
                    g.replay()
                stream.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    w0 = time.perf_counter()
    with sampler:
        soak(args.soak_seconds)
        with torch.cuda.stream(stream):
            for k in range(args.warmup):
                graphs[k].replay()
        barrier(device)
        torch.cuda.synchronize(device)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for k in range(args.warmup, total):
                graphs[k].replay()
            t1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        soak(args.soak_seconds)
    window = time.perf_counter() - w0
    value, step_ms = job_throughput(B * s_q, world, t0.elapsed_time(t1), args.steps, device)

    op_ms, app_ms, dec_ms = [], [], []
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.overhead_rounds)):
            for g, e in op_graphs:
                g.replay()
                stream.synchronize()
                op_ms.append(ev.ms(e[0], e[1]))
            for g, e in bd_graphs:
                g.replay()
                stream.synchronize()
                app_ms.append(ev.ms(e[0], e[1]))
                dec_ms.append(ev.ms(e[1], e[2]))

    # end to end through the public API from pinned host buffers: copy-in, append, decode, copy-out of
    # o_v and lse, synchronize, every step
    pinned = {k: torch.from_numpy(np.ascontiguousarray(v)).to(types[k]).pin_memory() for k, v in host.items()}
    o_host = torch.empty(outs[0][0].shape, dtype=torch.bfloat16).pin_memory()
    l_host = torch.empty(outs[0][1].shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = o_host.numel() * 2 + l_host.numel() * 4

    def e2e_step(k):
        i = k % n_copies
        for key, t in pinned.items():
            dev_in[i][key].copy_(t, non_blocking=True)
        append(i)
        decode(i)
        o_host.copy_(outs[i][0], non_blocking=True)
        l_host.copy_(outs[i][1], non_blocking=True)
        torch.cuda.synchronize(device)

    for k in range(args.warmup):
        e2e_step(k)
    barrier(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(args.steps):
        e2e_step(k)
    e1.record()
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1), device) / args.steps
    assert all(s.device_status() == qkn.OK for s in sessions)

    cost = gqa_step_cost(inp.seq_lens, s_q, H, wl.groups, wl.d_h, wl.d_rope, wl.d_v)
    peaks, peak_src = load_peaks()
    t_op = statistics.mean(op_ms)
    achieved = cost.bytes / (t_op * 1e-3) / 1e9
    tflops = cost.flops / (t_op * 1e-3) / 1e12
    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        wts = inp.group_weights()
        done, c0 = 0, time.perf_counter()
        for b in range(B):
            oracle.gqa_decode_sequence(inp, b, *wts)
            done += 1
            if time.perf_counter() - c0 >= args.cpu_seconds:
                break
        el = time.perf_counter() - c0
        cpu = {"value": done * s_q / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{done} of {B} sequences of the workload ({done * s_q} query tokens, "
                         f"{int(inp.seq_lens[:done].sum())} cached tokens) in {el:.1f} s, fp64 numpy, GQA route"}
    tokens = world * B * s_q
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "us_per_step": step_ms * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl, inp, world), route="gqa", d_v=wl.d_v,
                       l2=f"{n_copies} rotating cache copies, {n_copies * cache_bytes / 2**20:.0f} MiB "
                          f"(L2 {l2 / 2**20:.0f} MiB)", step_launch="CUDA graph per step"),
        "breakdown_us": {"gqa_append": statistics.median(app_ms) * 1e3,
                         "gqa_decode_op": statistics.median(dec_ms) * 1e3,
                         "what": "expansion of the step's new tokens / split-KV decode + merge, from separate "
                                 "graphs with an event between the stages"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "intensity_flop_per_byte": cost.flops / cost.bytes,
                     "algorithmic_bytes": cost.bytes, "peak_source": f"{peak_src} HBM copy bandwidth",
                     "kernel": ("GQA decode op (split-KV kernel + merge of its partials): mean duration over "
                                "%d replays of decode-only graphs, CUDA events on the launching stream" % len(op_ms)),
                     "duration_us": t_op * 1e3,
                     "tensor": {"achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": tflops / peaks["bf16_tflops"], "flops": cost.flops}},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": "per step: copy-in from pinned host buffers, qkn_gqa_append, qkn_gqa_decode, copy-out of "
                        "o_v and lse to pinned host buffers, synchronize"},
        "gpu_launches": 3 * args.steps,
        "clocks": sampler.summary(window),
        "cpu_baseline": cpu,
    }


def schedule_shape(kernel_used: int, head_tile: int, s_q: int, heads: int, sms: int):
    """Row tile, schedule CTAs and item cost of the decode's split schedule for this launch (the C-ABI
    layer's choice restated for cost accounting; 128-row tiles on CTA pairs count sms / 2 pairs)."""
    import qk_normed_latent_qkn_b200 as qkn
    if kernel_used != qkn.KERNEL_TCGEN05:
        return 8, sms, 1
    qrows = s_q * heads
    rows = head_tile or (16 if qrows <= 16 else 32 if qrows <= 32 else 64)
    ncta = sms // 2 if rows == 128 else sms
    return rows, ncta, 3 if rows >= 64 else rows // 16


# ----------------------------------------------------------------- reference arm (the oracle)
def cp_emulate(world: int, base, inp, device, ev, stream, rounds: int = 10) -> dict:
    """Context-parallel decode over `world` ranks, timed on one GPU: each rank's slice decode (its
    page slices of every sequence, qkn_decode with vis_end) replayed alone, and the merge of the
    stacked partials (qkn_merge_partials).  The step on `world` GPUs is estimated as the slowest
    rank's slice + an all-gather of the partials at the pool's measured NVLink peer-copy bandwidth
    + the merge; the all-gather is not run here."""
    import torch
    import qk_normed_latent_qkn_b200 as qkn
    from qk_normed_latent_qkn_b200 import context_parallel as cp
    wl = inp.wl
    B, s_q, H, r = wl.batch, wl.s_q, wl.heads, wl.r_kv
    dt = base.dims.torch_dtype
    ws = base.ensure_workspace(B, s_q)
    outs = torch.empty((world, B, s_q, H, r), dtype=dt, device=device)
    lses = torch.empty((world, B, s_q, H), dtype=torch.float32, device=device)
    out = torch.empty((B, s_q, H, r), dtype=dt, device=device)
    lse = torch.empty((B, s_q, H), dtype=torch.float32, device=device)
    views = []
    for k in range(world):
        bt, lens, ve = cp.rank_view(inp.block_table, inp.seq_lens, k, world, s_q)
        views.append([torch.from_numpy(x).to(device) for x in (bt, lens, ve)])
    graphs = []
    with torch.cuda.stream(stream):
        for k in range(world):
            bt, lens, ve = views[k]
            e = [ev.create() for _ in range(2)]
            g = torch.cuda.CUDAGraph()
            # eager first (first-call set-up), then captured
            qkn.decode(base.dims, base.cache, base.q_tilde, base.a_q, base.q_rope_hat, bt, lens, s_q, ws, outs[k],
                       lses[k], vis_end=ve)
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                ev.record(e[0], stream.cuda_stream)
                qkn.decode(base.dims, base.cache, base.q_tilde, base.a_q, base.q_rope_hat, bt, lens, s_q, ws,
                           outs[k], lses[k], vis_end=ve)
                ev.record(e[1], stream.cuda_stream)
            graphs.append((g, e))
        qkn.merge_partials(base.dims, outs, lses, out, lse)
        em = [ev.create() for _ in range(2)]
        gm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gm, stream=stream, capture_error_mode="relaxed"):
            ev.record(em[0], stream.cuda_stream)
            qkn.merge_partials(base.dims, outs, lses, out, lse)
            ev.record(em[1], stream.cuda_stream)
    torch.cuda.synchronize(device)
    slice_ms = [[] for _ in range(world)]
    merge_ms = []
    with torch.cuda.stream(stream):
        for _ in range(rounds):
            for k, (g, e) in enumerate(graphs):
                g.replay()
                stream.synchronize()
                slice_ms[k].append(ev.ms(e[0], e[1]))
            gm.replay()
            stream.synchronize()
            merge_ms.append(ev.ms(em[0], em[1]))
    assert base.device_status() == qkn.OK
    part_bytes = B * s_q * H * (r * outs.element_size() + 4)
    peer_gbs = 770.0                                  # measured NVLink peer copy, GB/s per direction
    gather_us = part_bytes * (world - 1) / (peer_gbs * 1e9) * 1e6
    slices = [statistics.median(v) * 1e3 for v in slice_ms]
    merge_us = statistics.median(merge_ms) * 1e3
    return {"world": world, "slice_us": slices, "merge_us": merge_us, "gather_bytes_per_rank": part_bytes,
            "gather_us_estimate": gather_us, "step_us_estimate": max(slices) + gather_us + merge_us,
            "what": ("each rank's slice decode (split-KV + merge of its own slices) and the merge of the "
                     "ranks' partials, timed on one GPU (CUDA events, decode-only graphs); the all-gather "
                     "is estimated at the measured 770 GB/s NVLink peer copy, not run")}


def workload_config(wl, inp, world: int) -> dict:
    """The workload part of the JSON line's config, the same for both arms."""
    return {"workload": wl.name, "batch_per_gpu": wl.batch, "s_q": wl.s_q, "heads": wl.heads, "groups": wl.groups,
            "r_kv": wl.r_kv, "d_h": wl.d_h, "d_rope": wl.d_rope,
            "context": list(wl.context) if isinstance(wl.context, tuple) else wl.context,
            "cached_tokens_per_gpu": int(inp.seq_lens.sum()), "paged": wl.paged,
            "parallelism": f"replicas x{world}"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    from qkn_inputs import WORKLOADS, make_inputs
    import oracle
    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl)
    # each step: one whole sequence of the workload through the explicit-key oracle
    times = []
    for k in range(args.warmup + args.steps):
        b = k % wl.batch
        t0 = time.perf_counter()
        if args.route == "gqa":
            oracle.gqa_decode_sequence(inp, b, *inp.group_weights())
        else:
            oracle.decode_sequence(inp, b)
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_tok = statistics.mean(times) / wl.s_q
    v = 1.0 / per_tok
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl, inp, world), sample="one whole sequence per step",
                       **({"route": "gqa", "d_v": wl.d_v} if args.route == "gqa" else {})),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one sequence of {wl.name} per step (explicit keys, fp64 numpy)"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        line = (run_gqa if args.route == "gqa" else run_ours)(args, world, rank, local)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
