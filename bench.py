#!/usr/bin/env python
"""Benchmark of the ReLU linear-attention forward on B200.

One step = one whole-sequence forward (ReLU + 3D RoPE prologue, state build,
reduction, apply) of the 480p-shaped workload: B=1, H=32, N=32760 (21 x 30 x 52
latent grid), D=64, bf16 I/O, fp32 state, RoPE split 16/24/24, theta 1e4.
Inputs (537 MB per step) are larger than the 126 MB L2, so no flush is needed
between steps. Timing: W warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream,
max over ranks. With --gpus N every rank runs its own replica (weak scaling,
no collective on the data path).

Prints one JSON line (rank 0). ``--impl reference`` times the fp64 CPU oracle
on the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "linear-attn fwd tokens/s & HBM GB/s (% of peak), N=32760 H=32 D=64 bf16"
MAIN = "480p_bidir"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=MAIN, choices=sorted(workloads.WORKLOADS),
                    help="workload of the timed line (another one than the default is for "
                         "profiling runs)")
    ap.add_argument("--mode", default="bidirectional",
                    choices=["bidirectional", "block_causal", "token_causal"])
    ap.add_argument("--settle", type=int, default=50,
                    help="untimed forwards before the timed region (clock settling)")
    ap.add_argument("--only", default=None,
                    help="run one secondary measurement alone (for profiling runs) and print "
                         "its line, e.g. 480p_bidir_x_text300/cross, 480p_hidden_tconv, "
                         "480p_2b_d112/bidirectional, 480p_bidir/token_causal")
    return ap.parse_args()


def launches_per_forward(w, mode) -> int:
    """Kernels one forward launches: state build (+ reduction when a head has
    more than one segment) + apply."""
    if mode == "token_causal":
        # tensor cores (bf16, D = 64): state partials + causal apply; CUDA
        # cores: state partials, scan, chunked apply
        return 2 if (w.dtype == "bf16" and w.D == 64) else 3
    one_segment = mode == "bidirectional" or w.block_tokens in (0, w.N)
    return 2 if one_segment else 3


# ---------------------------------------------------------------- dist ----

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def reduce_max(value: float, pg, device=None) -> float:
    """Max of a float over ranks (identity without a process group)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device=None):
    if pg is not None:
        if device is not None:
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# ------------------------------------------------------------- helpers ----

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# CUDA-core attention kernels and the temporal convolution: not part of the
# profiled tensor-core kernels' sources
_NOT_TC_SOURCES = ("simt.cuh", "tconv.cu")


def _source_selected(name: str, kind: str) -> bool:
    if kind == "tconv":
        return name == "tconv.cu"
    return name not in _NOT_TC_SOURCES


def kernel_source_hash(kind: str = "tc") -> str:
    """Hash of a kernel family's sources with comments and whitespace removed,
    so that a committed traffic figure stays tied to the code it was measured
    on, not to its comments or to other kernels. kind "tc": the attention
    kernels (every CUDA source but the CUDA-core kernels and the temporal
    convolution, host launch code included); "tconv": the temporal
    convolution's translation unit."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_video_relu_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")) and _source_selected(name, kind):
            with open(os.path.join(csrc, name)) as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            text = " ".join(text.split())
            h.update(name.encode() + b"\0" + text.encode())
    return h.hexdigest()[:12]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (a line '# bench-traffic <kernel> <workload>
    <bytes> <source-hash>' in profiles/*.txt); else None."""
    pdir = os.path.join(ROOT, "profiles")
    want = kernel_source_hash("tconv" if kernel == "temporal_conv" else "tc")
    if not os.path.isdir(pdir):
        return None
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".txt", ".md")):
            continue
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 6 and parts[0] == "#" and parts[1] == "bench-traffic":
                    if parts[2] == kernel and parts[3] == workload and parts[5] == want:
                        return int(parts[4])
    return None


class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self.period = period_s

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def device_inputs(w: workloads.Workload, device, seed: int):
    """Seeded synthetic inputs drawn on the device (same shapes and value
    distributions as workloads.make_inputs; a torch CUDA generator here)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (w.B, w.H, w.N, w.D)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = {}
    for name in ["q", "k", "v"] + (["g"] if w.gate else []):
        if w.qk_dist == "student_t3" and name in ("q", "k"):
            # t_3 = Z / sqrt(chi2_3 / 3), scaled to unit variance
            z = torch.randn(shape, generator=g, device=device)
            chi = torch.randn((3,) + shape, generator=g, device=device).pow_(2).sum(0)
            x = z / torch.sqrt(chi / 3.0) / math.sqrt(3.0)
            del z, chi
        else:
            x = torch.randn(shape, generator=g, device=device)
        out[name] = x.to(dt)
        del x
    return out


# ---------------------------------------------------------- GPU timing ----

def time_forward(w, mode, t, steps, warmup, pg, device, record_kernels=True):
    """Time `steps` forwards; returns (max-over-ranks ms, per-kernel ms lists)."""
    import torch
    import linear_attention_video_relu_b200 as la
    C = la._native
    p = la.make_params(w.B, w.H, w.N, w.D, t["q"].dtype, mode,
                       w.block_tokens if mode == "block_causal" else 0, w.grid, w.rope_split,
                       w.rope_theta, w.eps)
    ws = la.workspace_for(p, device)
    out = torch.empty_like(t["q"])
    stream = torch.cuda.current_stream(device)
    sp = stream.cuda_stream
    args = (p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
            t["g"].data_ptr() if "g" in t else None, out.data_ptr(), ws.ptr, ws.nbytes, sp)
    for _ in range(warmup):
        C.check(C.lin_attn_forward(*args), "lin_attn_forward")
    evs = []
    if record_kernels:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for row in evs:
            for e in row:
                e.record(stream)          # materialise the event handles
    torch.cuda.synchronize(device)
    barrier(pg, device)
    torch.cuda.synchronize(device)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        if record_kernels:
            C.check(C.lin_attn_forward_timed(*args, [e.cuda_event for e in evs[i]]),
                    "lin_attn_forward_timed")
        else:
            C.check(C.lin_attn_forward(*args), "lin_attn_forward")
    stop.record(stream)
    torch.cuda.synchronize(device)
    barrier(pg, device)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(stop)
    st = C.lin_attn_device_status(ws.ptr, sp)
    if st != C.LA_OK:
        raise RuntimeError("device status after timing: %s" % C.status_string(st))
    kern = None
    if record_kernels:
        kern = [[r[j].elapsed_time(r[j + 1]) for r in evs] for j in range(3)]
    ms_max = reduce_max(ms, pg, device)
    return ms_max, kern, out


def roofline_entry(name, bytes_per_launch, ms_list, peak, peak_kind, workload):
    avg_ms = sum(ms_list) / len(ms_list)
    gbs = bytes_per_launch / (avg_ms * 1e-3) / 1e9
    traffic = ncu_traffic(name, workload)
    return {"kernel": name, "bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
            "unit": "GB/s", "frac": round(gbs / peak, 4), "traffic": traffic,
            "algorithmic_bytes": bytes_per_launch, "avg_us": round(avg_ms * 1e3, 2),
            "peak_source": peak_kind}


def traffic_note(line: dict):
    """One short reason, for the whole line, when the roofline's traffic is
    null: no committed ncu capture was taken on the current kernel sources."""
    rf = line.get("roofline") or {}
    if rf.get("traffic") is None and "kernel" in rf:
        return "no ncu capture on kernel sources %s" % kernel_source_hash("tc")
    return None


def measure_workload(w, mode, steps, warmup, pg, device, peak, peak_kind, seed):
    import torch
    t = device_inputs(w, device, seed)
    ms, _, out = time_forward(w, mode, t, steps, warmup, pg, device, record_kernels=False)
    _, kern, out = time_forward(w, mode, t, steps, 2, pg, device, record_kernels=True)
    elt = 2 if w.dtype == "bf16" else 4
    tensor_bytes = w.B * w.H * w.N * w.D * elt
    state_bytes = 2 * tensor_bytes
    apply_bytes = (3 if w.gate else 2) * tensor_bytes
    total_bytes = w.algorithmic_bytes()
    if mode == "token_causal":
        # the two-pass causal form reads k and v twice: 12 D bytes per
        # token-head (bf16), the apply kernel reading q, k, v and writing out
        apply_bytes += 2 * tensor_bytes
        total_bytes += 2 * tensor_bytes
    step_ms = ms / steps
    key = w.name if mode == "bidirectional" else "%s/%s" % (w.name, mode)
    k_state = roofline_entry("state_build", state_bytes, kern[0], peak, peak_kind, key)
    k_reduce_us = round(sum(kern[1]) / len(kern[1]) * 1e3, 2)
    k_apply = roofline_entry("apply", apply_bytes, kern[2], peak, peak_kind, key)
    res = {
        "workload": w.name, "mode": mode, "ms_per_step": step_ms,
        "tokens_per_s": w.B * w.N / (step_ms * 1e-3),
        "hbm_gbs": total_bytes / (step_ms * 1e-3) / 1e9,
        "hbm_frac": total_bytes / (step_ms * 1e-3) / 1e9 / peak,
        "kernels": {"state_build": k_state, "reduce_us": k_reduce_us, "apply": k_apply},
    }
    del t, out
    torch.cuda.empty_cache()
    return res


def measure_block_steps(w, steps, warmup, device, peak, peak_kind, seed):
    """Algorithm 1's per-block call: lin_attn_block_step with commit on every
    block of the 720p workload, one call per block through BlockState.step.
    Also the host time to issue one step (issue_us): below us_per_block the
    GPU bounds the rate, near it the host does."""
    import torch
    import linear_attention_video_relu_b200 as la
    t = device_inputs(w, device, seed)
    bt = w.block_tokens
    T, Hg, Wg = w.grid
    fpb = bt // (Hg * Wg)
    nblk = w.N // bt
    blocks = [{n: t[n][:, :, b * bt:(b + 1) * bt].contiguous() for n in t} for b in range(nblk)]
    del t
    st = la.BlockState(w.B, w.H, w.D, device=device)
    outs = [torch.empty_like(blocks[0]["q"]) for _ in range(2)]

    def run_all():
        for b in range(nblk):
            st.step(blocks[b]["q"], blocks[b]["k"], blocks[b]["v"], t_offset=b * fpb, commit=True,
                    grid=(fpb, Hg, Wg), rope_split=w.rope_split, eps=w.eps, out=outs[b % 2])

    reps = max(1, steps // nblk)
    for _ in range(max(1, warmup // nblk)):
        st.reset()
        run_all()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h0 = time.perf_counter()
    for _ in range(reps):
        run_all()
    h1 = time.perf_counter()
    b_.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b_) / (reps * nblk)
    bytes_blk = 4 * w.B * w.H * bt * w.D * 2
    return {"workload": w.name + "_block_step", "block_tokens": bt, "us_per_block": ms * 1e3,
            "issue_us": (h1 - h0) / (reps * nblk) * 1e6,
            "tokens_per_s": w.B * bt / (ms * 1e-3),
            "hbm_frac": bytes_blk / (ms * 1e-3) / 1e9 / peak}


def measure_cross(w, n_kv, steps, warmup, device, peak, seed):
    """Linear cross-attention: the workload's video tokens as queries reading
    n_kv text tokens per head as keys and values (no RoPE), one C-ABI call per
    forward, CUDA events around `steps` calls."""
    import torch
    import linear_attention_video_relu_b200 as la
    C = la._native
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    q = torch.randn((w.B, w.H, w.N, w.D), generator=g, device=device).to(bf)
    k = torch.randn((w.B, w.H, n_kv, w.D), generator=g, device=device).to(bf)
    v = torch.randn((w.B, w.H, n_kv, w.D), generator=g, device=device).to(bf)
    out = torch.empty_like(q)
    p = la.make_params(w.B, w.H, w.N, w.D, bf, eps=w.eps)
    ws = la.Workspace(C.lin_attn_cross_workspace_size(p, n_kv), device)
    stream = torch.cuda.current_stream(device)
    args = (p, n_kv, q.data_ptr(), k.data_ptr(), v.data_ptr(), None, out.data_ptr(), ws.ptr,
            ws.nbytes, stream.cuda_stream)
    for _ in range(warmup):
        C.check(C.lin_attn_cross_forward(*args), "lin_attn_cross_forward")
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        C.check(C.lin_attn_cross_forward(*args), "lin_attn_cross_forward")
    b.record(stream)
    torch.cuda.synchronize(device)
    st = C.lin_attn_device_status(ws.ptr, stream.cuda_stream)
    if st != C.LA_OK:
        raise RuntimeError("device status after timing: %s" % C.status_string(st))
    ms = a.elapsed_time(b) / steps
    nbytes = 2 * 2 * w.B * w.H * (w.N + n_kv) * w.D     # read q, k, v; write out (bf16)
    del q, k, v, out
    name = "%s_x_text%d" % (w.name, n_kv)
    t_sb, t_ap = ncu_traffic("state_build", name), ncu_traffic("apply", name)
    return {"workload": name, "mode": "cross", "n_kv": n_kv,
            "us_per_forward": ms * 1e3, "tokens_per_s": w.B * w.N / (ms * 1e-3),
            "algorithmic_bytes": nbytes, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
            "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peak,
            "traffic": (t_sb + t_ap) if (t_sb is not None and t_ap is not None) else None}


def measure_tconv(steps, warmup, device, peak, seed):
    """The Mix-FFN temporal convolution on 480p hidden states (B=1, 21 frames x
    1560 positions x 2240 channels, bf16) with bias, reading and writing the
    last-frame cache: CUDA events around `steps` calls."""
    import torch
    import linear_attention_video_relu_b200 as la
    C = la._native
    sh = workloads.TCONV_480P
    B, T, S, nc = sh["B"], sh["T"], sh["S"], sh["C"]
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn((B, T, S, nc), generator=g, device=device).to(bf)
    w = 0.5 * torch.randn((3, nc), generator=g, device=device)
    b = 0.1 * torch.randn((nc,), generator=g, device=device)
    cache_in = torch.randn((B, S, nc), generator=g, device=device).to(bf)
    cache_out = torch.empty_like(cache_in)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(device)
    args = (B, T, S, nc, C.LA_BF16, x.data_ptr(), w.data_ptr(), b.data_ptr(),
            cache_in.data_ptr(), y.data_ptr(), cache_out.data_ptr(), stream.cuda_stream)
    for _ in range(warmup):
        C.check(C.lin_attn_temporal_conv(*args), "lin_attn_temporal_conv")
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        C.check(C.lin_attn_temporal_conv(*args), "lin_attn_temporal_conv")
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    nbytes = (2 * T + 2) * B * S * nc * 2     # x in, y out, cache frame in and out (bf16)
    del x, y, cache_in, cache_out
    return {"workload": "480p_hidden_tconv", "mode": "temporal_conv_cached",
            "shape": [B, T, S, nc], "us_per_call": ms * 1e3,
            "tokens_per_s": B * T * S / (ms * 1e-3), "algorithmic_bytes": nbytes,
            "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peak,
            "traffic": ncu_traffic("temporal_conv", "480p_hidden_tconv")}


def measure_e2e(w, steps, device, seed):
    """The same forward end to end through the public API: every step copies
    its inputs in from pinned host memory, calls la.forward and copies the
    output back, all inside the timed region. As a serving loop would, the
    loop keeps two sets of device buffers and three streams, so that one
    step's host-to-device copies overlap the previous step's forward and its
    device-to-host copy (the two directions of the link run at once)."""
    import torch
    import linear_attention_video_relu_b200 as la
    td = device_inputs(w, device, seed)
    host = {n: torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for n, x in td.items()}
    for n in td:
        host[n].copy_(td[n])
    bufs = [td, {n: torch.empty_like(x) for n, x in td.items()}]
    outs = [torch.empty_like(td["q"]) for _ in range(2)]
    out_h = torch.empty(td["q"].shape, dtype=td["q"].dtype, pin_memory=True)
    p = la.make_params(w.B, w.H, w.N, w.D, td["q"].dtype, "bidirectional", 0, w.grid,
                       w.rope_split, w.rope_theta, w.eps)
    ws = la.workspace_for(p, device)
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i % 2
        x = bufs[b]
        if used[b]:
            s_in.wait_event(ev_comp[b])      # the forward that read set b has finished
        with torch.cuda.stream(s_in):
            for n in x:
                x[n].copy_(host[n], non_blocking=True)
        ev_in[b].record(s_in)
        s_comp.wait_event(ev_in[b])
        if used[b]:
            s_comp.wait_event(ev_out[b])     # out[b] is back on the host before it is rewritten
        la.forward(x["q"], x["k"], x["v"], x.get("g"), grid=w.grid, rope_split=w.rope_split,
                   theta=w.rope_theta, eps=w.eps, out=outs[b], workspace=ws, stream=s_comp)
        ev_comp[b].record(s_comp)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            out_h.copy_(outs[b], non_blocking=True)
        ev_out[b].record(s_out)
        used[b] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        step(i)
    b.record(s_out)                            # after the last copy back, which follows all
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = out_h.numel() * out_h.element_size()
    return {"value": w.B * w.N / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "pipeline": "2 buffer sets; copy-in, forward and copy-out on 3 streams"}


# ----------------------------------------------------------- CPU oracle ----

def oracle_sample(w, budget_s: float, max_heads=None):
    """Time the fp64 oracle (as it stands) on a bounded sample of workload w:
    the first `heads` heads over the first `frames` latent frames."""
    import numpy as np
    import oracle
    cores = oracle.threads(0)
    heads = min(w.B * w.H, max_heads or w.B * w.H)
    T, Hg, Wg = w.grid
    # about 10 us of one core per token-head at D = 64 (scaled by D^2), as measured on
    # the hosts: size frames to the budget
    frames = T
    est = lambda f: heads * f * Hg * Wg * (w.D * w.D / 4096.0) * 10e-6 / min(cores, heads)
    while frames > 1 and est(frames) > budget_s:
        frames -= 1
    sw = workloads.Workload(name=w.name + "_sample", B=1, H=heads, N=frames * Hg * Wg, D=w.D,
                            dtype=w.dtype, seed=w.seed, grid=(frames, Hg, Wg),
                            rope_split=w.rope_split, gate=w.gate, qk_dist=w.qk_dist)
    x = workloads.make_inputs(sw)
    p = oracle.params_for(sw, "bidirectional")
    return sw, x, p, min(cores, heads)


def run_oracle_once(sw, x, p, cores):
    import oracle
    t0 = time.perf_counter()
    oracle.forward(p, x["q"], x["k"], x["v"], g=x.get("g"), nthreads=cores)
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s=2.0):
    """The oracle on the host cores: repeated over a sample of the workload
    until about budget_s of wall time (tens of seconds of CPU work)."""
    sw, x, p, cores = oracle_sample(w, budget_s=budget_s)
    runs, dt = 0, 0.0
    while runs < 1 or (dt < budget_s and runs < 20):
        dt += run_oracle_once(sw, x, p, cores)
        runs += 1
    # tokens/s of the whole workload: the sample covers sw.H of the w.B*w.H heads
    tok_s = runs * sw.N * (sw.H / (w.B * w.H)) / dt
    return {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d heads x %d tokens (%d frames) of %s, fp64, %d runs in %.1f s "
                      "wall on %d threads" % (sw.H, w.B * w.H, sw.N, sw.grid[0], w.name, runs,
                                              dt, cores)}


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle on the host cores."""
    if rank != 0:
        return
    w = workloads.WORKLOADS[MAIN]
    total_steps = args.steps + args.warmup
    per_step = max(0.05, min(2.0, 120.0 / max(total_steps, 1)))
    sw, x, p, cores = oracle_sample(w, budget_s=per_step)
    for _ in range(args.warmup):
        run_oracle_once(sw, x, p, cores)
    t = 0.0
    for _ in range(args.steps):
        t += run_oracle_once(sw, x, p, cores)
    step_s = t / max(args.steps, 1)
    tok_s = sw.N * (sw.H / (w.B * w.H)) / step_s
    sample = "%d of %d heads x %d tokens (%d frames) of %s per step, fp64" % (
        sw.H, w.B * w.H, sw.N, sw.grid[0], w.name)
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, "bidirectional", world),
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# the SANA-Video 2B model's attention shape: 20 heads of 112 at 480p
W_2B_480P = workloads.Workload("480p_2b_d112", B=1, H=20, N=21 * 30 * 52, D=112, dtype="bf16",
                               seed=2004, grid=(21, 30, 52), rope_split=(16, 48, 48))


def secondary_lines(K, device, peak, peak_kind):
    """The other workloads and rows, each timed on its own; a line that fails
    records its error instead of ending the run."""
    return run_jobs(secondary_jobs(K, device, peak, peak_kind))


def secondary_jobs(K, device, peak, peak_kind, warmup=3):
    """(name, measurement) of every secondary line, K timed steps each."""
    jobs = []
    for name, mode in (("480p_block_causal", "block_causal"), ("720p_long", "bidirectional"),
                       ("720p_long", "block_causal"), ("gated_d128", "bidirectional"),
                       ("480p_bidir", "token_causal")):
        ww = workloads.WORKLOADS[name]
        jobs.append((name + "/" + mode,
                     lambda ww=ww, mode=mode: measure_workload(ww, mode, K, warmup, None, device,
                                                               peak, peak_kind, ww.seed)))
    jobs.append(("480p_2b_d112/bidirectional",
                 lambda: measure_workload(W_2B_480P, "bidirectional", K, warmup, None, device, peak,
                                          peak_kind, W_2B_480P.seed)))
    jobs.append(("480p_bidir_x_text300/cross",
                 lambda: measure_cross(workloads.WORKLOADS["480p_bidir"], 300, K, max(warmup, 1),
                                       device, peak, 2002)))
    jobs.append(("480p_hidden_tconv",
                 lambda: measure_tconv(K, max(warmup, 1), device, peak, 2003)))
    jobs.append(("720p_long_block_step",
                 lambda: measure_block_steps(workloads.WORKLOADS["720p_long"], max(K, 60),
                                             max(warmup, 60), device, peak, peak_kind, 1004)))
    return jobs


def run_jobs(jobs):
    out = []
    for name, job in jobs:
        try:
            out.append(compact(job()))
        except Exception as e:   # reported in the line, not swallowed
            out.append({"w": name, "error": ("%s: %s" % (type(e).__name__, e))[:160]})
    return out


def compact(r: dict) -> dict:
    """A secondary result in a few short keys, so that every one of them fits
    in the tail of the output: w workload, mode, ms (or us) per call, frac =
    algorithmic HBM bytes / time as a fraction of the peak, and per kernel its
    average us and roofline fraction (sb state build, ap apply, red the
    separate reduction)."""
    c = {"w": r["workload"], "mode": r.get("mode")}
    if "ms_per_step" in r:
        c["ms"] = round(r["ms_per_step"], 4)
    for key, short in (("us_per_forward", "us"), ("us_per_call", "us"),
                       ("us_per_block", "us_blk"), ("issue_us", "issue_us")):
        if key in r:
            c[short] = round(r[key], 2)
    if "tokens_per_s" in r:
        c["tok_s"] = float("%.4g" % r["tokens_per_s"])
    if "hbm_frac" in r:
        c["frac"] = round(r["hbm_frac"], 4)
    mb = lambda t: None if t is None else round(t / 1e6, 1)
    k = r.get("kernels")
    if k:
        # [event-timed us, roofline fraction, ncu DRAM MB per launch or null]
        c["sb"] = [k["state_build"]["avg_us"], k["state_build"]["frac"],
                   mb(k["state_build"].get("traffic"))]
        c["ap"] = [k["apply"]["avg_us"], k["apply"]["frac"], mb(k["apply"].get("traffic"))]
        c["red_us"] = k["reduce_us"]
    if "traffic" in r:
        c["traffic_MB"] = mb(r["traffic"])
    return c


def config_of(w, mode, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "mode": mode,
            "grid": list(w.grid) if w.grid else None,
            "rope_split": list(w.rope_split) if w.rope_split else None,
            "gate": w.gate, "global_batch": w.B * world, "seq_len": w.N,
            "parallelism": "replicas x%d" % world,
            "l2": "inputs larger than L2 (%.0f MB per step vs 126 MB), no flush" % (
                w.algorithmic_bytes() / 1e6)}


# ------------------------------------------------------------------ main ----

def main():
    args = parse_args()
    world, rank, local, pg = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if pg is not None:
            pg.destroy_process_group()
        return
    import torch
    import linear_attention_video_relu_b200 as la
    la._native.load()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peak, peak_kind = measured_peaks()
    if args.only:
        # one secondary line alone (profiling runs)
        jobs = [j for j in secondary_jobs(args.steps, device, peak, peak_kind, args.warmup)
                if j[0] == args.only]
        if not jobs:
            raise SystemExit("unknown --only job %r" % args.only)
        if rank == 0:
            print(json.dumps(run_jobs(jobs)[0]), flush=True)
        if pg is not None:
            barrier(pg, device)
            pg.destroy_process_group()
        return
    w = workloads.WORKLOADS[args.workload]
    mode = args.mode

    t = device_inputs(w, device, seed=w.seed + rank)
    # settle clocks with untimed work, then sample clocks across the timed region
    if args.settle > 0:
        _ = time_forward(w, mode, t, args.settle, args.warmup, None, device, record_kernels=False)
    sampler = ClockSampler(local)
    sampler.start()
    # the headline: plain forwards back to back (the launches overlap through
    # programmatic dependent launch)
    ms, _, out = time_forward(w, mode, t, args.steps, args.warmup, pg, device,
                              record_kernels=False)
    sampler.stop()
    # per-kernel breakdown: a second timed pass with events between the kernels
    ms_k, kern, out = time_forward(w, mode, t, min(args.steps, 200), 3, pg, device,
                                   record_kernels=True)
    del t, out
    torch.cuda.empty_cache()

    step_ms = ms / args.steps
    tokens = w.B * w.N * world
    value = tokens / (step_ms * 1e-3)
    elt = 2
    tensor_bytes = w.B * w.H * w.N * w.D * elt
    k_state = roofline_entry("state_build", 2 * tensor_bytes, kern[0], peak, peak_kind, w.name)
    k_apply = roofline_entry("apply", 2 * tensor_bytes, kern[2], peak, peak_kind, w.name)
    dominant = k_state if k_state["avg_us"] >= k_apply["avg_us"] else k_apply
    total_bytes = w.algorithmic_bytes()
    gbs = total_bytes / (step_ms * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded torch CUDA generator, N(0,1) -> bf16)",
        "config": config_of(w, mode, world),
        "hbm_gbs": round(gbs, 1), "hbm_frac_of_peak": round(gbs / peak, 4),
        "peak_hbm_gbs": peak, "peak_source": peak_kind,
        "roofline": dominant,
        "kernels": {"state_build": k_state,
                    "reduce_us": round(sum(kern[1]) / len(kern[1]) * 1e3, 2),
                    "apply": k_apply},
        "ms_per_step_with_kernel_events": ms_k / min(args.steps, 200),
        "gpu_launches": launches_per_forward(w, mode) * args.steps,
        "tensor_core_path": bool(la.uses_tensor_cores(w.B, w.H, w.N, w.D, torch.bfloat16,
                                                      grid=w.grid, rope_split=w.rope_split)),
        "clocks": sampler.summary(),
    }
    if args.workload != MAIN or mode != "bidirectional":
        line["metric"] = "linear-attn fwd tokens/s (profiling run: %s, %s)" % (w.name, mode)
    note = traffic_note(line)
    if note:
        line["traffic_note"] = note
    if rank == 0 and args.e2e_steps > 0:
        line["e2e"] = measure_e2e(w, args.e2e_steps, device, w.seed)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if not args.no_extra and rank == 0:
        # last in the line, in short keys (see compact), so it survives in a tail
        line["also"] = secondary_lines(max(20, args.steps // 5), device, peak, peak_kind)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        barrier(pg, device)
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
