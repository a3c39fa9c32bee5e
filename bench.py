#!/usr/bin/env python
"""Benchmark of the streaming KV-cache Compressor on B200.

One step = one Compressor call over one batch: the C128A 128K prefill (one
sequence of 131072 tokens, H=4096, D=512, ratio 128, block_size 128), which is
the workload of the headline metric (128K-prefill tokens/s). Inputs are seeded
synthetic tensors of that shape, resident in HBM; x alone (1 GiB) is larger
than the 126 MB L2, so no flush is needed between prefill steps.

Also reported on the same line:
  * e2e: the same metric through the public call with host buffers: every step
    copies x, cu_seqlens, start_pos, the block tables and sin/cos from pinned
    host memory and reads the output back;
  * decode: the C4A 32-request decode step (one token each), microseconds per
    call, with L2 flushed before every timed call;
  * roofline: the projection kernel's tensor throughput against the measured
    bf16 peak (with the pooling epilogue's HBM throughput beside it when it is
    a separate launch), and the decode call's HBM throughput against measured
    bandwidth;
  * nsa: the NsaCompressWithCache decode step (128 batches), microseconds per
    call with L2 flushed before every timed call, against HBM bandwidth;
  * configs: the other workloads (c4li_tiny, c4a_varlen, c4li_chunked),
    microseconds per step and projection TFLOP/s;
  * cpu_baseline: the CPU oracle on a bounded sample of the same workload.

Multi-GPU (torchrun): every rank runs its own replica on its own GPU (requests
are independent; no data-path collective), the time is the max over ranks and
value counts the tokens of all ranks ("scaling": "weak").

--impl reference times the CPU oracle (the only reference implementation this
method has) on the same workload; rank 0 alone prints its line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "128K-prefill tokens/s"
PREFILL = dict(name="c128a_128k", B=1, T=131072, H=4096, D=512, ratio=128, block_size=128)
DECODE_ALG_BYTES = None  # computed from the decode workload


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    """The max of v over all ranks (the job's time is its slowest rank's)."""
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ws: int, ms_this_rank: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank in the timed
    region (weak scaling), the region lasts as long as the slowest rank."""
    ms = max_over_ranks(ms_this_rank, ws)
    return units_per_rank * ws / (ms / 1e3)


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """SM clock, max clock and clock-event reasons sampled every 5 ms while the
    timed region runs, read through NVML (read-only queries), or through
    `nvidia-smi -lms 50` when NVML cannot be loaded."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []   # (sm_mhz, max_mhz, set of active reason names)
        self.proc = None
        self.nvml = None
        self.dev = device_index
        self.stop = threading.Event()

    def _uuid(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:  # noqa: BLE001
            return None

    def __enter__(self):
        uuid = self._uuid()
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(0)
            self.nvml = (pynvml, h)
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return self
        except Exception:  # noqa: BLE001 - fall back to nvidia-smi
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *(["-i", uuid] if uuid else []), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _poll_nvml(self):
        nv, h = self.nvml
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), {n for n, b in self.REASONS if bits & b}))
            except Exception:  # noqa: BLE001
                pass
            self.stop.wait(0.005)

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            num = lambda v: float(v) if v.replace(".", "", 1).isdigit() else None
            self.samples.append((num(parts[0]), num(parts[1]),
                                 {names[i] for i in range(4) if parts[3 + i].lower() == "active"}))

    def __exit__(self, *a):
        self.stop.set()
        if self.nvml:
            self.thread.join(timeout=2)
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm = [s[0] for s in self.samples if s[0] is not None]
        mx = [s[1] for s in self.samples if s[1] is not None]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        reasons = sorted(set().union(*[s[2] for s in self.samples]))
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples),
                "source": "nvml" if self.nvml else "nvidia-smi"}


# ----------------------------------------------------------------------------
# workloads on the device
# ----------------------------------------------------------------------------

def prefill_inputs(device, seed: int):
    """The C128A 128K prefill, drawn on the device with a seeded generator:
    x ~ N(0,1); wkv, wgate ~ N(0, 1/H); ape ~ N(0, 0.1); norm_weight ~ 1 + N(0, 0.05);
    states ~ N(0,1); block table = a random permutation of the 1024 pool rows."""
    import numpy as np
    import torch

    import streaming_kv_cache_varlen_b200 as cmp
    from workloads import rope_tables

    c = PREFILL
    T, H, D, r, bs = c["T"], c["H"], c["D"], c["ratio"], c["block_size"]
    C = D
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(T, H, generator=g, device=device).to(bf)
    wkv = (torch.randn(C, H, generator=g, device=device) / H ** 0.5).to(bf)
    wgate = (torch.randn(C, H, generator=g, device=device) / H ** 0.5).to(bf)
    ape = torch.randn(r, C, generator=g, device=device) * 0.1 ** 0.5
    norm_w = (1 + torch.randn(D, generator=g, device=device) * 0.05 ** 0.5).to(bf)
    nblk = T // bs
    kv_state = torch.randn(nblk, bs, C, generator=g, device=device)
    score_state = torch.randn(nblk, bs, C, generator=g, device=device)
    perm = torch.randperm(nblk, generator=g, device=device).to(torch.int32).view(1, nblk)
    cu = torch.tensor([0, T], dtype=torch.int32, device=device)
    sp = torch.zeros(1, dtype=torch.int32, device=device)
    # sin / cos per output row from the library's own row layout (window w at w*ratio)
    rs, rw = cmp.out_row_layout(np.array([0, T], np.int32), np.array([0], np.int32), r)
    cos, sin = rope_tables(np.where(rw >= 0, rw * r, 0), 64)
    cos_t = torch.from_numpy(cos.view(np.int16)).to(device).view(bf)
    sin_t = torch.from_numpy(sin.view(np.int16)).to(device).view(bf)
    return dict(x=x, kv_state=kv_state, score_state=score_state, kv_block_table=perm,
                state_block_table=perm.clone(), sin=sin_t, cos=cos_t, wkv=wkv, wgate=wgate,
                ape=ape, norm_weight=norm_w, hadamard=None, start_pos=sp, cu_seqlens=cu,
                ratio=r, rope_head_dim=64, rotate=False)


def with_library_rope(inp):
    """sin/cos rows for the output rows the library's layout gives (positions w*ratio)."""
    import numpy as np

    import streaming_kv_cache_varlen_b200 as cmp
    from workloads import rope_tables

    rs, rw = cmp.out_row_layout(inp.cu_seqlens, inp.start_pos, inp.ratio)
    cos, sin = rope_tables(np.where(rw >= 0, rw * inp.ratio, 0), 64)
    return inp.__class__(**{**inp.__dict__, "cos": cos, "sin": sin})


def device_args(inp, device, kv_state=None, score_state=None):
    """The compressor's arguments for ``inp`` as device tensors (states optional:
    pass device buffers to carry state across calls)."""
    import numpy as np
    import torch

    def bfd(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    return dict(x=bfd(inp.x), kv_state=d(inp.kv_state) if kv_state is None else kv_state,
                score_state=d(inp.score_state) if score_state is None else score_state,
                kv_block_table=d(inp.kv_block_table), state_block_table=d(inp.state_block_table),
                sin=bfd(inp.sin), cos=bfd(inp.cos), wkv=bfd(inp.wkv), wgate=bfd(inp.wgate),
                ape=d(inp.ape), norm_weight=bfd(inp.norm_weight), hadamard=bfd(inp.hadamard),
                start_pos=d(inp.start_pos), cu_seqlens=d(inp.cu_seqlens), ratio=inp.ratio,
                rope_head_dim=64, rotate=inp.hadamard is not None)


def bench_configs(args, ws, local, peaks, peak_src):
    """The other workloads, reported beside the headline: c4li_tiny and
    c4a_varlen (one call each) and c4li_chunked (its 4 calls, state carried from
    call to call). Device time per step: a CUDA graph of 20 back-to-back steps
    after 3 warm-ups, the best of 3 replays / 20 (a repeated step recomputes the
    same values: a call reads only positions before its start and writes only
    its tail), no L2 flush; achieved = the projection's 2*T*H*2C flop over
    that time."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp
    from workloads import make_chunked, make_config

    device = torch.device("cuda", local)
    res = {}
    for name in ("c4li_tiny", "c4a_varlen", "c4li_chunked"):
        if name == "c4li_chunked":
            ch = make_chunked()
            calls = [with_library_rope(c) for c in ch.calls]
            first = device_args(calls[0], device)
            steps_args = [first] + [device_args(c, device, first["kv_state"], first["score_state"])
                                    for c in calls[1:]]
        else:
            calls = [with_library_rope(make_config(name))]
            steps_args = [device_args(calls[0], device)]
        outs = [torch.empty((cmp.out_rows(c.B, c.T, c.ratio), c.D), dtype=torch.bfloat16, device=device)
                for c in calls]
        flops = sum(2.0 * c.T * c.H * 2 * c.C for c in calls)

        def step():
            for a, o in zip(steps_args, outs):
                cmp.compressor(**a, out=o)

        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))  # inputs were made on the current stream
        with torch.cuda.stream(side):
            for _ in range(3):
                step()
        torch.cuda.synchronize()
        assert cmp.get_error(side) == 0
        n = 20
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for _ in range(n):
                step()
        torch.cuda.synchronize()
        best = None
        barrier(ws)
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(side):
                e0.record(side)
                g.replay()
                e1.record(side)
            torch.cuda.synchronize()
            best = e0.elapsed_time(e1) if best is None else min(best, e0.elapsed_time(e1))
        us = max_over_ranks(best, ws) * 1e3 / n
        assert cmp.get_error(side) == 0
        del g
        tf = flops / (us / 1e6) / 1e12
        res[name] = {"calls_per_step": len(calls), "tokens_per_step": int(sum(c.T for c in calls)),
                     "us_per_step": us, "tflops": tf, "frac_of_bf16_burst": tf / peaks["bf16_tflops"],
                     "kernel_us": kernel_times(step, side, steps=5)}
        del steps_args, outs
        torch.cuda.empty_cache()
    return res


def kernel_times(step, stream, steps: int):
    """Per-kernel device time of `step`: the library's CUDA events around each of
    its launches (cmp_profile_start/stop) over `steps` eager steps. The steps are
    queued behind a ~10 ms sleep kernel so that the host has enqueued them all
    before the first one runs (launch overhead does not show up between a
    kernel's events). Returns {kernel: {"us": mean per launch, "launches_per_step": n}}."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp

    with torch.cuda.stream(stream):
        torch.cuda._sleep(20_000_000)
        cmp.profile_start()
        for _ in range(steps):
            step()
        prof = cmp.profile_stop()
    return {k: {"us": ms / n * 1e3, "launches_per_step": n / steps} for k, (ms, n) in prof.items() if n}


def decode_inputs(device):
    from workloads import make_config

    inp = with_library_rope(make_config("c4a_decode"))
    args = device_args(inp, device)
    # algorithmic bytes of one decode call: both weight matrices, x, the earlier
    # state rows the completed windows pool (coff*ratio - 1 half rows of D floats,
    # kv and score), the state rows written (every token, kv and score), the ape
    # rows, the output rows and the sin/cos rows of the windows, norm_weight
    C, H, D = inp.C, inp.H, inp.D
    n_win = int((((inp.start_pos + 1) % inp.ratio) == 0).sum())
    hist_half_rows = n_win * (inp.coff * inp.ratio - 1)
    alg = (2 * C * H * 2 + inp.T * H * 2 + hist_half_rows * D * 4 * 2 + inp.T * C * 4 * 2
           + inp.ratio * C * 4 + inp.B * D * 2 + n_win * 64 * 2 * 2 + D * 2)
    return args, alg, inp


# ----------------------------------------------------------------------------
# measurement
# ----------------------------------------------------------------------------

def read_peaks():
    try:
        p = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def traffic_for(kernel_file: str, kernel: str, units_scale: float = 1.0):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel source as it is now (else None)."""
    try:
        t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    except OSError:
        return None
    e = t.get(kernel)
    if not e:
        return None
    src = os.path.join(ROOT, "streaming_kv_cache_varlen_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if e.get("source_sha") != sha:
        return None
    return e["bytes_per_launch"] * units_scale


def bench_prefill(args, ws, local, stream, peaks, peak_src):
    """Device-resident prefill steps: value, per-kernel times and the roofline."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp

    device = torch.device("cuda", local)
    rank = int(os.environ.get("RANK", "0"))
    pf = prefill_inputs(device, seed=1234 + rank)
    out = torch.empty((cmp.out_rows(1, PREFILL["T"], PREFILL["ratio"]), PREFILL["D"]),
                      dtype=torch.bfloat16, device=device)
    for _ in range(args.warmup):
        cmp.compressor(**pf, out=out)
    torch.cuda.synchronize()
    assert cmp.get_error() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = cmp.launch_count()
    with ClockSampler(local) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        cmp.profile_start()
        e0.record(stream)
        for _ in range(args.steps):
            cmp.compressor(**pf, out=out)
        e1.record(stream)
        torch.cuda.synchronize()
        prof = cmp.profile_stop()
        barrier(ws)
    launches = cmp.launch_count() - launches0
    assert cmp.get_error() == 0
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    value = PREFILL["T"] * ws * args.steps / (ms / 1e3)

    # dominant kernel: the projection (a dense bf16 contraction)
    proj_name = max(("proj_tcgen05", "proj_mma_sync", "proj_decode", "fused_tcgen05"),
                    key=lambda k: prof[k][0])
    p_ms, p_n = prof[proj_name]
    T, H, C = PREFILL["T"], PREFILL["H"], PREFILL["D"]
    flops = 2.0 * T * H * 2 * C
    achieved = flops / (p_ms / p_n / 1e3) / 1e12 if p_n else None
    clocks = clk.summary()
    # burst peak for a short timed region; the sustained (power-capped) one when
    # the clocks show the power cap during it
    sustained = "sw_power_cap" in clocks.get("reasons", []) and "bf16_tflops_sustained" in peaks
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    kfile = {"proj_tcgen05": "cmp_proj_tc.cu", "proj_mma_sync": "cmp_proj_mma.cu",
             "proj_decode": "cmp_proj_decode.cu", "fused_tcgen05": "cmp_fused_tc.cu"}[proj_name]
    roofline = {"kernel": proj_name, "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak if achieved else None,
                "traffic": traffic_for(kfile, proj_name, T / 131072.0),
                "peak_source": peak_src + (" (sustained: sw_power_cap during the timed region)"
                                           if sustained else " (burst)"),
                "frac_of_burst": achieved / peaks["bf16_tflops"] if achieved else None,
                "algorithmic_flops_per_launch": flops,
                "kernel_ms": {k: (v[0] / v[1] if v[1] else None) for k, v in prof.items()}}
    # the pooling epilogue that follows the fused projection when it is a separate
    # launch (merge, RMSNorm, RoPE, bf16 store): HBM, its algorithmic bytes over its
    # launch time (calls without rotation finish their rows inside the fused kernel)
    f_ms, f_n = prof["finish"]
    if f_n:
        n_out, coff, D = out.shape[0], (2 if PREFILL["ratio"] == 4 else 1), PREFILL["D"]
        fb = (n_out * coff * D * 4 * (2 if coff == 2 else 1)  # pooled halves (+ their lse)
              + n_out * 64 * 2 * 2 + D * 2                   # sin, cos rows, norm_weight
              + n_out * D * 2)                               # bf16 rows out
        f_gbs = fb / (f_ms / f_n / 1e3) / 1e9
        roofline["epilogue"] = {"kernel": "finish", "bound": "hbm", "us": f_ms / f_n * 1e3,
                                "algorithmic_bytes": fb, "achieved": f_gbs, "unit": "GB/s",
                                "frac": f_gbs / peaks["hbm_gbs"]}
    return dict(value=value, ms_step=ms / args.steps, launches=launches, roofline=roofline,
                clocks=clocks, inputs=pf, out=out)


def bench_e2e(args, ws, stream, pf, out):
    """The same metric through the public call with host buffers: per step, H2D of
    the step's inputs from pinned memory, the call, D2H of the output."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp

    host_names = ("x", "cu_seqlens", "start_pos", "kv_block_table", "state_block_table", "sin", "cos")
    host = {k: pf[k].cpu().pin_memory() for k in host_names}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dev_in = {k: torch.empty_like(pf[k]) for k in host_names}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out.numel() * out.element_size()
    steps = max(1, min(args.steps, 20))
    call = dict(pf)

    def step():
        for k in host_names:
            dev_in[k].copy_(host[k], non_blocking=True)
            call[k] = dev_in[k]
        cmp.compressor(**call, out=out)
        out_host.copy_(out, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    return {"value": PREFILL["T"] * ws * steps / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


def bench_decode(args, ws, local, stream, peaks, peak_src):
    """C4A 32-request decode, microseconds of device time per call.

    Device time comes from CUDA-graph replays: a graph of N x (256 MB L2 flush,
    call) minus a graph of N flushes alone, divided by N, so host and binding
    overhead is excluded and every call starts with a cold L2. The eager time
    (events around each call from Python, host overhead included) is reported
    beside it."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp

    device = torch.device("cuda", local)
    dec, dec_bytes, dec_inp = decode_inputs(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    dout = torch.empty((cmp.out_rows(dec_inp.B, dec_inp.T, dec_inp.ratio), dec_inp.D),
                       dtype=torch.bfloat16, device=device)
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))  # the inputs were made on the current stream
    with torch.cuda.stream(side):
        for _ in range(max(3, args.warmup)):
            cmp.compressor(**dec, out=dout)
            flush.fill_(1)
    torch.cuda.synchronize()
    n = 50
    g_call, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g_call, stream=side):
            for _ in range(n):
                flush.fill_(1)
                cmp.compressor(**dec, out=dout)
        with torch.cuda.graph(g_flush, stream=side):
            for _ in range(n):
                flush.fill_(1)
        torch.cuda.synchronize()
        graphs = True
    except Exception as exc:  # noqa: BLE001 - report eager timing instead
        torch.cuda.synchronize()
        graphs = False
        graph_error = str(exc).splitlines()[0][:200]

    def replay(g):
        best = None
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(side):  # replay() launches on the current stream
                a.record(side)
                g.replay()
                b.record(side)
            torch.cuda.synchronize()
            t = a.elapsed_time(b)
            best = t if best is None else min(best, t)
        return best

    barrier(ws)
    if graphs:
        t_call, t_flush = replay(g_call), replay(g_flush)
        assert cmp.get_error(side) == 0
        dec_us = max_over_ranks((t_call - t_flush) * 1e3 / n, ws)
    del g_call, g_flush

    # eager: events around each call from Python (host overhead included)
    times = []
    cmp.profile_start()
    for _ in range(20):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cmp.compressor(**dec, out=dout)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    dprof = cmp.profile_stop()
    eager = statistics.median(a.elapsed_time(b) * 1e3 for a, b in times)
    if graphs:
        timing = "CUDA-graph replay of 50 x (L2 flush + call) minus 50 flushes, / 50"
    else:
        dec_us = max_over_ranks(eager, ws)
        timing = f"eager events around each call (graph capture failed: {graph_error})"
    ach = dec_bytes / (dec_us / 1e6) / 1e9
    return {"workload": "c4a_decode: 32 requests x 1 token, H=4096, D=512, ratio 4",
            "us_per_call": dec_us, "us_per_call_eager": eager, "calls": n,
            "timing": timing,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes_per_call": dec_bytes,
                         "peak_source": peak_src},
            "kernel_us_eager": {k: (v[0] / v[1] * 1e3 if v[1] else None) for k, v in dprof.items()}}


NSA = dict(B=128, N=24, D=192, page=128, cbs=32, stride=16, max_seq=512)


def bench_nsa(args, ws, local, peaks, peak_src):
    """NsaCompressWithCache, one decode step in which all 128 batches reach a
    compression step: N=24 heads of D=192 (the shapes of its page's example), bf16,
    paged cache (page 128), window 32, stride 16. Device time per call from graph
    replays of 50 x (256 MB L2 flush + call) minus 50 flushes; the algorithmic bytes
    are the windows read once plus the slots written."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp

    c = NSA
    device = torch.device("cuda", local)
    g = torch.Generator(device=device).manual_seed(4)
    per = c["max_seq"] // c["page"]
    block_num = c["B"] * per
    bf = torch.bfloat16
    inp = torch.randn((block_num, c["page"], c["N"], c["D"]), generator=g, device=device).to(bf)
    weight = (torch.randn((c["cbs"], c["N"]), generator=g, device=device) / c["cbs"] ** 0.5).to(bf)
    table = torch.randperm(block_num, generator=g, device=device).to(torch.int32).view(c["B"], per)
    steps = (c["max_seq"] - c["cbs"]) // c["stride"] + 1
    lens = (c["cbs"] + c["stride"] * torch.randint(0, steps, (c["B"],), generator=g, device=device)).to(torch.int64)
    result_len = 4 * c["B"]
    slots = torch.randperm(result_len, generator=g, device=device)[:c["B"]].to(torch.int32)
    out = torch.zeros((result_len, c["N"], c["D"]), dtype=bf, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def call():
        cmp.nsa_compress(inp, weight, slots, lens, out, compress_block_size=c["cbs"],
                         compress_stride=c["stride"], block_table=table, page_block_size=c["page"])

    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))  # the inputs were made on the current stream
    with torch.cuda.stream(side):
        for _ in range(max(3, args.warmup)):
            call()
            flush.fill_(1)
    torch.cuda.synchronize()
    n = 50
    g_call, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_call, stream=side):
        for _ in range(n):
            flush.fill_(1)
            call()
    with torch.cuda.graph(g_flush, stream=side):
        for _ in range(n):
            flush.fill_(1)
    torch.cuda.synchronize()

    def replay(gr):
        best = None
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(side):
                a.record(side)
                gr.replay()
                b.record(side)
            torch.cuda.synchronize()
            best = a.elapsed_time(b) if best is None else min(best, a.elapsed_time(b))
        return best

    barrier(ws)
    us = max_over_ranks((replay(g_call) - replay(g_flush)) * 1e3 / n, ws)
    assert cmp.get_error(side) == 0
    del g_call, g_flush
    plane = c["N"] * c["D"] * 2
    nbytes = c["B"] * (c["cbs"] + 1) * plane + c["cbs"] * c["N"] * 2
    ach = nbytes / (us / 1e6) / 1e9
    return {"workload": f"nsa_decode_step: {c['B']} batches on a compression step, N={c['N']}, "
                        f"D={c['D']}, bf16, paged (page {c['page']}), window {c['cbs']}, stride {c['stride']}",
            "us_per_call": us, "timing": "CUDA-graph replay of 50 x (L2 flush + call) minus 50 flushes, / 50",
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
                         "traffic": traffic_for("cmp_nsa.cu", "nsa_compress"), "peak_source": peak_src}}


PHASE_NAMES = ("entry", "setup_done", "first_stage", "last_mma", "metadata", "partials_sent",
               "partials_received", "pooled_arrived", "-", "exchange_done", "rows_stored",
               "all_arrived", "-", "-", "tails_written", "end",
               "meta_wave1", "meta_windows", "meta_wave2", "meta_wave3")


def run_decode_phases(args):
    """--only decode-phases: the C4A 32-request decode call run through the
    phase-stamp build of the library (built beside the normal one if missing),
    cold (256 MB L2 flush before the call) and warm (the same call again). Per
    phase, min / median / max over the CTAs of the time since the earliest
    CTA's entry, in microseconds, medians over `steps` calls of each kind."""
    import numpy as np

    sys.path.insert(0, os.path.join(ROOT, "streaming_kv_cache_varlen_b200"))
    import _build
    os.environ["CMP_LIBRARY"] = _build.build(phases=True)
    import torch

    import streaming_kv_cache_varlen_b200 as cmp
    assert cmp.LIB_PATH == os.environ["CMP_LIBRARY"]

    device = torch.device("cuda", 0)
    dec, _, inp = decode_inputs(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    dout = torch.empty((cmp.out_rows(inp.B, inp.T, inp.ratio), inp.D), dtype=torch.bfloat16, device=device)
    n_ctas = (inp.D // 16) * 4
    res = {}
    for kind in ("cold", "warm"):
        runs = []
        for i in range(args.warmup + args.steps):
            if kind == "cold":
                flush.fill_(1)
            torch.cuda.synchronize()
            cmp.compressor(**dec, out=dout)
            st = cmp.debug_phase_stamps(n_ctas).astype(np.int64)
            assert cmp.get_error() == 0
            if i >= args.warmup:
                runs.append((st - st[:, 0].min()) / 1e3)
        a = np.stack(runs)   # [runs, ctas, 16]
        res[kind] = {name: {"min": float(np.median(a[:, :, k].min(axis=1))),
                            "median": float(np.median(np.median(a[:, :, k], axis=1))),
                            "max": float(np.median(a[:, :, k].max(axis=1)))}
                     for k, name in enumerate(PHASE_NAMES) if name != "-"}
    print(json.dumps({"decode_phases_us": res, "ctas": n_ctas, "calls_per_kind": args.steps,
                      "workload": "c4a_decode: 32 requests x 1 token, H=4096, D=512, ratio 4"}), flush=True)


def run_chunked_calls(args):
    """--only chunked-calls: the c4li_chunked workload's 4 calls (state carried),
    run eagerly `warmup` then `steps` times, with the library's per-kernel times
    (for profiler captures of the projection and pooling kernels on that path;
    the configs section times the same calls as graph replays)."""
    import torch

    import streaming_kv_cache_varlen_b200 as cmp
    from workloads import make_chunked

    device = torch.device("cuda", 0)
    ch = make_chunked()
    calls = [with_library_rope(c) for c in ch.calls]
    first = device_args(calls[0], device)
    steps_args = [first] + [device_args(c, device, first["kv_state"], first["score_state"]) for c in calls[1:]]
    outs = [torch.empty((cmp.out_rows(c.B, c.T, c.ratio), c.D), dtype=torch.bfloat16, device=device)
            for c in calls]

    def step():
        for a, o in zip(steps_args, outs):
            cmp.compressor(**a, out=o)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    cmp.profile_start()
    for _ in range(args.steps):
        step()
    prof = cmp.profile_stop()
    assert cmp.get_error() == 0
    print(json.dumps({"workload": "c4li_chunked: 8 requests x 4 calls of U[1, 2048] tokens, H=7168, D=128, "
                                  "ratio 4, rotate", "steps": args.steps,
                      "tokens_per_step": int(sum(c.T for c in calls)),
                      "kernel_us": {k: ms / n * 1e3 for k, (ms, n) in prof.items() if n},
                      "launches": {k: n for k, (ms, n) in prof.items() if n}}), flush=True)


def run_ours(args):
    import torch

    ws, rank, local = dist_setup()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peaks, peak_src = read_peaks()

    pre = e2e = decode = None
    if args.only in ("all", "prefill"):
        pre = bench_prefill(args, ws, local, stream, peaks, peak_src)
        if args.only == "all":
            e2e = bench_e2e(args, ws, stream, pre["inputs"], pre["out"])
        pre.pop("inputs")
        pre.pop("out")
        torch.cuda.empty_cache()
    if args.only in ("all", "decode"):
        decode = bench_decode(args, ws, local, stream, peaks, peak_src)
    nsa = None
    if args.only in ("all", "nsa"):
        nsa = bench_nsa(args, ws, local, peaks, peak_src)
        torch.cuda.empty_cache()
    configs = None
    if args.only in ("all", "configs"):
        configs = bench_configs(args, ws, local, peaks, peak_src)
    cpu = None
    if rank == 0 and ws == 1 and args.only == "all" and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_tokens or cpu_sample_tokens(args.cpu_seconds))

    if rank == 0:
        line = {"metric": METRIC, "value": pre["value"] if pre else None, "unit": "tokens/s",
                "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": pre["ms_step"] if pre else None,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 in, fp32 accumulate / state, bf16 out", "data": "synthetic",
                "config": {"workload": f"c128a_128k: C128A prefill, 1 sequence x {PREFILL['T']} "
                                       "tokens, H=4096, D=512, ratio=128, coff=1, block_size=128",
                           "global_batch": ws, "seq_len": PREFILL["T"],
                           "parallelism": f"dp{ws} (independent replicas)",
                           "l2": "inputs larger than L2 (x is 1 GiB per step)"},
                "e2e": e2e, "gpu_launches": pre["launches"] if pre else None,
                "roofline": pre["roofline"] if pre else None, "decode": decode, "nsa": nsa, "configs": configs,
                "clocks": pre["clocks"] if pre else None, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


class _Marks:
    """Time stamps on the device (CUDA events on the current stream) or, on CPU,
    host clock readings; spans_ms() gives the times between consecutive marks."""

    def __init__(self, cuda: bool):
        self.cuda = cuda
        self.m = []

    def mark(self):
        if self.cuda:
            import torch
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            self.m.append(e)
        else:
            self.m.append(time.perf_counter())

    def spans_ms(self):
        if self.cuda:
            import torch
            torch.cuda.synchronize()
            return [a.elapsed_time(b) for a, b in zip(self.m, self.m[1:])]
        return [(b - a) * 1e3 for a, b in zip(self.m, self.m[1:])]


def sharded_inputs(device, T: int, H: int, D: int, ratio: int, seed: int):
    """One sequence of T tokens from position 0, drawn with a seeded torch
    generator on `device` (identical on every rank): x ~ N(0,1), weights
    N(0, 1/H), ape N(0, 0.1), norm_weight 1 + N(0, 0.05), and the sin/cos rows of
    its windows (position w * ratio)."""
    import numpy as np
    import torch

    from streaming_kv_cache_varlen_b200 import sharded
    from workloads import rope_tables

    coff = 2 if ratio == 4 else 1
    C = coff * D
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(T, H, generator=g, device=device).to(bf)
    wkv = (torch.randn(C, H, generator=g, device=device) / H ** 0.5).to(bf)
    wgate = (torch.randn(C, H, generator=g, device=device) / H ** 0.5).to(bf)
    ape = torch.randn(ratio, C, generator=g, device=device) * 0.1 ** 0.5
    norm_w = (1 + torch.randn(D, generator=g, device=device) * 0.05 ** 0.5).to(bf)
    n_out = sharded.n_out_rows(T, ratio)
    pos = np.where(np.arange(n_out) < T // ratio, np.arange(n_out) * ratio, 0)
    cos, sin = rope_tables(pos, 64)
    to = lambda a: torch.from_numpy(a.view(np.int16)).to(device).view(bf)
    return dict(x=x, wkv=wkv, wgate=wgate, ape=ape, norm_weight=norm_w, hadamard=None, sin=to(sin),
                cos=to(cos))


def bench_sharded(args, ws: int, rank: int, device, *, T: int, H: int, D: int, ratio: int,
                  block_size: int = 128, run_call=None):
    """One long prefill split across the ranks by tokens (the library's sharded
    prefill: per-rank calls on window-aligned slices with a halo, then one
    all-gather of the output rows). Per step: this rank's call (with its scratch
    state) and the all-gather, timed separately; the step time is the max over
    ranks. Returns (the JSON line's fields, the assembled output of the last step)."""
    import torch

    from streaming_kv_cache_varlen_b200 import sharded

    cuda = device.type == "cuda"
    inp = sharded_inputs(device, T, H, D, ratio, seed=1234)
    shards = sharded.plan(T, ratio, ws)
    me = shards[rank]
    C = inp["wkv"].shape[0]
    if run_call is None:
        from streaming_kv_cache_varlen_b200 import compressor as run_call

    def step(marks):
        marks.mark()
        loc = sharded.local_inputs(me, inp["x"], inp["sin"], inp["cos"], ratio, block_size, C)
        out_loc = run_call(wkv=inp["wkv"], wgate=inp["wgate"], ape=inp["ape"],
                           norm_weight=inp["norm_weight"], hadamard=None, ratio=ratio, rope_head_dim=64,
                           rotate=False, **loc)
        mine = sharded.own_rows(me, out_loc)
        marks.mark()
        rows = sharded.all_gather_rows(shards, mine) if ws > 1 else [mine]
        out = sharded.assemble(shards, rows, T, ratio, mine)
        marks.mark()
        return out

    for _ in range(args.warmup):
        step(_Marks(cuda))
    if cuda:
        torch.cuda.synchronize()
    barrier(ws)
    if cuda:
        torch.cuda.synchronize()
    marks = _Marks(cuda)
    for _ in range(args.steps):
        out = step(marks)
    spans = marks.spans_ms()
    barrier(ws)
    compute = sum(spans[0::3])     # call spans; spans[1::3] all-gather; spans[2::3] between steps
    gather = sum(spans[1::3])
    total = sum(spans)
    total_max = max_over_ranks(total, ws)
    line = {"metric": METRIC, "value": T * args.steps / (total_max / 1e3), "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_max / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate / state, bf16 out",
            "data": "synthetic",
            "config": {"workload": f"one sequence x {T} tokens, H={H}, D={D}, ratio={ratio}, "
                                   f"block_size={block_size}",
                       "global_batch": 1, "seq_len": T,
                       "parallelism": f"cp{ws} (token-sharded prefill, one all-gather of the output rows)"},
            "sharded": {"compute_ms_per_step_max": max_over_ranks(compute, ws) / args.steps,
                        "gather_ms_per_step_max": max_over_ranks(gather, ws) / args.steps,
                        "windows_per_rank": [s.n_windows for s in shards],
                        "backend": "nccl" if cuda else "gloo"}}
    return line, out


def run_sharded(args):
    """--mode sharded: the token-sharded 128K prefill under torchrun (NCCL)."""
    import torch

    ws, rank, local = dist_setup()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    line, _ = bench_sharded(args, ws, rank, device, T=args.prefill_tokens, H=PREFILL["H"],
                            D=PREFILL["D"], ratio=PREFILL["ratio"], block_size=PREFILL["block_size"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline(tokens: int):
    """The oracle, as it is, on the first ``tokens`` tokens of the prefill workload
    (drawn on the host with the workload generator), on this host's cores."""
    import numpy as np

    from oracle import run_inputs, window_row_positions
    from workloads import make_inputs

    c = PREFILL
    inp = make_inputs(name="cpu_sample", seed=2, lengths=[tokens], start_pos=[0], H=c["H"],
                      D=c["D"], coff=1, ratio=c["ratio"], block_size=c["block_size"], rotate=False)
    inp = inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, c["ratio"]))
    t0 = time.perf_counter()
    run_inputs(inp)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info())
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {tokens} tokens ({tokens // c['ratio']} windows) of the 128K "
                      f"prefill workload, float64 numpy oracle, {dt:.2f} s"}


def cpu_sample_tokens(seconds: float) -> int:
    """Tokens of the prefill workload the oracle processes in about ``seconds`` on
    this host (a 2048-token probe sets the rate), whole windows, at most the
    workload."""
    rate = cpu_baseline(2048)["value"]
    r = PREFILL["ratio"]
    return int(max(4096, min(PREFILL["T"], rate * seconds)) // r * r)


def run_reference(args):
    """The CPU oracle as the reference arm: each step is the oracle on a bounded
    sample of the prefill workload, sized so warm-up plus all steps take about
    two minutes on this host."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    probe = cpu_baseline(512)
    rate = probe["value"]  # tokens/s of the oracle on this host
    per_step = int(rate * 120.0 / (args.steps + args.warmup))
    per_step = max(PREFILL["ratio"], min(16384, per_step // PREFILL["ratio"] * PREFILL["ratio"]))
    for _ in range(args.warmup):
        cpu_baseline(per_step)
    dts = []
    for _ in range(args.steps):
        r = cpu_baseline(per_step)
        dts.append(per_step / r["value"])
    total = sum(dts)
    value = per_step * len(dts) / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / len(dts) * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "c128a_128k: C128A prefill, 1 sequence x 131072 tokens, "
                                   "H=4096, D=512, ratio=128, coff=1, block_size=128",
                       "global_batch": 1, "seq_len": PREFILL["T"], "parallelism": "cpu",
                       "sample_tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--mode", choices=("replicas", "sharded"), default="replicas",
                    help="replicas: every rank runs its own copy of the workload (the default); "
                         "sharded: one 128K prefill split across the ranks by tokens")
    ap.add_argument("--cpu-tokens", type=int, default=None,
                    help="tokens of the CPU-baseline sample (default: about --cpu-seconds of oracle work)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=("all", "prefill", "decode", "nsa", "configs", "decode-phases",
                                       "chunked-calls"),
                    default="all",
                    help="run only one part (for profiler captures); decode-phases: the decode "
                         "kernel's timeline from the phase-stamp build of the library")
    ap.add_argument("--prefill-tokens", type=int, default=PREFILL["T"],
                    help="tokens of the prefill sequence (smaller cases for profiler captures)")
    ap.add_argument("--path", type=int, default=0,
                    help="the library's path knob (cmp_set_proj_kernel) for every call: 0 = automatic "
                         "(the default); others force one path, for comparisons and captures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    PREFILL["T"] = args.prefill_tokens
    if args.path and args.impl == "ours":
        import streaming_kv_cache_varlen_b200 as cmp
        if cmp.set_proj_kernel(args.path) < 0:
            raise SystemExit(f"--path {args.path}: not a path of the library")
    if args.impl == "reference":
        run_reference(args)
    elif args.only == "decode-phases":
        run_decode_phases(args)
    elif args.only == "chunked-calls":
        run_chunked_calls(args)
    elif args.mode == "sharded":
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
