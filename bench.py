"""Benchmark of the KDA hot path on B200: prefill tokens/s (headline) with decode
state GB/s, full-mixer and varlen prefill alongside, each against its roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one process per GPU)

A step is one kda_chunk_fwd call over the model-shape prefill workload (B=1,
T=4096, H=32, d_k=d_v=128, bf16 q/k/v, fp32 log_alpha/beta/state). The path is
independent per (sequence, head), so N GPUs run N replicas of the workload
("weak" scaling, no data-path collective); each GPU's time comes from CUDA
events on the launching stream and the job time is the max over ranks.
Between timed steps the inputs rotate through copies whose total exceeds L2.
`--impl reference` times the fp64 CPU oracle instead (a deliberately slow
reference arm on the host cores).
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s & decode state GB/s at H=32,d=128 (1 B200, % roofline)"
H, D, T1 = 32, 128, 4096
CHUNK = 64
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
# The prefill's MMAs are kind::tf32; its peak is the measured bf16 peak times the nominal
# dense tf32 : bf16 ratio of the B200 (1.1 : 2.25 PFLOP/s).
TF32_PER_BF16 = 1.1 / 2.25


# ----------------------------------------------------------------------------------
# algorithmic work (bytes / flops the method must move or do, per call)
# ----------------------------------------------------------------------------------
def kernels_per_call(workspace_bytes: int) -> int:
    """Kernels one kda_chunk_fwd / kda_mixer_fwd call launches (d = 128): the chunk plan,
    the intra-chunk pass and the recurrence when the workspace query asked for the
    two-pass scratch (more than the 256-byte status word), else the single-pass kernel."""
    return 3 if workspace_bytes > 256 else 1


def prefill_bytes(total_T: int, N: int, Hh: int = H, d: int = D, with_h0: bool = True, mixer: bool = False) -> int:
    """q, k, v, out (bf16) + log_alpha (fp32) + beta (fp32) + states in/out (fp32).
    The full mixer adds the gate (bf16) and conv weights; its q, k, v are the raw ones."""
    tok = total_T * Hh
    b = tok * d * 2 * 4 + tok * d * 4 + tok * 4
    b += N * Hh * d * d * 4 * (2 if with_h0 else 1)
    if mixer:
        b += tok * d * 2 + 3 * Hh * d * 4 * 4
    return b


def prefill_tc_flops(total_T: int, Hh: int = H, d: int = D, chunk: int = CHUNK) -> int:
    """Tensor-core work the chunked form must do per token-head, triangle-aware: three
    d x d state GEMMs (6 d^2) and five C-wide GEMMs whose operands are triangular
    (K Kt^T, Q Kt^T, T K, T V, P U: 5 C d) = 139,264 flops at d = 128, C = 64."""
    return total_T * Hh * (6 * d * d + 5 * chunk * d)


def prefill_tc_flops_issued(total_T: int, Hh: int = H, d: int = D, chunk: int = CHUNK) -> int:
    """The same GEMMs as the kernels issue them, on dense tiles (10 C d for the C-wide
    ones) = 180,224 flops per token-head at d = 128, C = 64."""
    return total_T * Hh * (6 * d * d + 10 * chunk * d)


def decode_bytes(N: int, Hh: int = H, d: int = D) -> int:
    """State read + write (fp32) plus the token's q, k, v, out (bf16), log_alpha, beta."""
    return N * Hh * (2 * d * d * 4 + 4 * d * 2 + d * 4 + 4)


def mixer_decode_bytes(N: int, Hh: int = H, d: int = D) -> int:
    """Serving mixer decode step: the fp32 state and the bf16 three-row conv history of q, k,
    v read and written per (sequence, head), plus the token's raw q, k, v, gate, out (bf16),
    log_alpha (fp32), beta and the slot index."""
    return N * Hh * (2 * d * d * 4 + 2 * 9 * d * 2 + 5 * d * 2 + d * 4 + 4) + N * 4


def mixer_decode_tokens_bytes(N: int, K: int, Hh: int = H, d: int = D) -> int:
    """K tokens per call without checkpoints: the state and conv history read and written
    once, each token's raw q, k, v, gate, out (bf16), log_alpha and beta, the slot index."""
    return N * Hh * (2 * d * d * 4 + 2 * 9 * d * 2 + K * (5 * d * 2 + d * 4 + 4)) + N * 4


def backward_bytes(total_T: int, N: int, Hh: int = H, d: int = D) -> int:
    """Algorithmic HBM bytes of one backward call: q, k, v, d_out (bf16), log_alpha (fp32),
    beta read; dq, dk, dv, d_log_alpha (fp32), d_beta written; initial state and the
    final state's gradient read, the initial state's gradient written."""
    tok = total_T * Hh * (4 * d * 2 + d * 4 + 4 + 4 * d * 4 + 4)
    return tok + 3 * N * Hh * d * d * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def headline_input_sets() -> int:
    """Device copies of the headline inputs the timed calls rotate through: more than
    3x the 126 MB L2 in all, so no call finds its inputs in L2."""
    return max(2, math.ceil(3 * 126e6 / prefill_bytes(T1, 1)) + 1)


def headline_config(world: int) -> dict:
    """The workload of the headline line, the same for both arms (the reference arm
    times the oracle on a bounded sample of it; its `cpu_baseline` says which)."""
    n_sets = headline_input_sets()
    return {"workload": "KDA chunked prefill B=1 T=4096 H=32 d_k=d_v=128 (bf16 q/k/v, fp32 log_alpha/beta/state)",
            "global_batch": world, "seq_len": T1, "heads": H, "head_dim": D, "chunk": CHUNK,
            "parallelism": f"replicas x{world} (independent (sequence, head) chains, no collective)",
            "l2": f"inputs rotate through {n_sets} device copies ({n_sets * prefill_bytes(T1, 1) / 1e6:.0f} MB > L2)"}


# The sources the headline call's kernels (plan, intra-chunk, recurrence) are compiled from.
HEADLINE_KERNEL_SOURCES = ("kda_split.cu", "kda_tile.cuh", "sm100_ptx.cuh")


def kernel_sources_sha256() -> str:
    """Hash of the headline call's kernel sources (HEADLINE_KERNEL_SOURCES, in that order):
    identifies the kernels an ncu traffic figure was captured from."""
    import hashlib
    csrc = os.path.join(ROOT, "gated_delta_rule_137_b200", "csrc")
    h = hashlib.sha256()
    for name in HEADLINE_KERNEL_SOURCES:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


def load_traffic(override=None):
    """DRAM bytes per headline call (read + write of the plan, intra-chunk and recurrence
    kernels) from profiles/traffic.json, if it was captured from these kernel sources;
    None once the sources have changed since."""
    if override is not None:
        return override
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p))
    return float(j["bytes_per_call"]) if j.get("source_sha256") == kernel_sources_sha256() else None


# ----------------------------------------------------------------------------------
# distributed plumbing (replicas): rank info, barrier, max over ranks
# ----------------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_throughput(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Weak scaling: every rank processes `units_per_rank`; the job time is the slowest rank's."""
    return units_per_rank * world / seconds_max


# ----------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------
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
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit()) if rows else None,
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------
# synthetic inputs on the device (timing only; parity runs on the NumPy generator)
# ----------------------------------------------------------------------------------
def device_prefill_inputs(total_T, Hh, d, seed, device, normalise=True, state_N=None, mixer=False):
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    def nrm(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    q, k, v = nrm(total_T, Hh, d), nrm(total_T, Hh, d), nrm(total_T, Hh, d)
    if normalise:
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
    la = -torch.nn.functional.softplus(nrm(total_T, Hh, d)) / 16
    beta = torch.sigmoid(nrm(total_T, Hh))
    out = dict(q=q.bfloat16(), k=k.bfloat16(), v=v.bfloat16(), log_alpha=la.contiguous(), beta=beta.contiguous())
    out["initial_state"] = (0.02 * nrm(state_N, Hh, d, d)) if state_N else None
    if mixer:
        out["conv_w"] = 0.5 * nrm(3, Hh * d, 4)
        out["gate"] = nrm(total_T, Hh, d).bfloat16()
    return out


# ----------------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------------
def time_region(fn, steps, warmup, stream, device):
    """W untimed calls, then K calls between events; returns per-step ms list (events
    per step) and the total ms for the K steps, bracketed by barrier + sync."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        fn(warmup + i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return per, ev[0].elapsed_time(ev[steps])


def run_gpu(args):
    import numpy as np
    import torch

    import gated_delta_rule_137_b200 as kda
    from gated_delta_rule_137_b200 import build as kbuild
    from gated_delta_rule_137_b200 import inputs as I

    rank, local_rank, world = dist_env()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    if rank == 0:
        kbuild.build()
    barrier(device)
    lib = kda.load_library()
    stream = torch.cuda.current_stream(device)
    hbm_peak, tc_peak, tc_peak_sus, peak_src = load_peaks()
    launches = 0

    # ---------------- headline: model-shape prefill, inputs resident in HBM -----------
    w = I.prefill_model_shape()
    host = dict(q=torch.from_numpy(w.q).to(torch.bfloat16), k=torch.from_numpy(w.k).to(torch.bfloat16),
                v=torch.from_numpy(w.v).to(torch.bfloat16), log_alpha=torch.from_numpy(w.log_alpha),
                beta=torch.from_numpy(w.beta), initial_state=torch.from_numpy(w.initial_state))
    bytes_call = prefill_bytes(T1, 1)
    n_sets = headline_input_sets()
    sets = []
    for _ in range(n_sets):
        sets.append({k: t.to(device) for k, t in host.items()})
    outs = [torch.empty(T1, H, D, dtype=torch.bfloat16, device=device) for _ in range(n_sets)]
    fins = [torch.empty(1, H, D, D, dtype=torch.float32, device=device) for _ in range(n_sets)]
    ws_bytes = kda.chunk_fwd_workspace_bytes(T1, 1, H, D, D, kda.KDA_DT_BF16)
    head_kernels = kernels_per_call(ws_bytes)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)

    def step(i):
        s = sets[i % n_sets]
        kda.chunk_fwd(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], s["initial_state"], None, N=1,
                      out=outs[i % n_sets], final_state=fins[i % n_sets], workspace=ws, stream=stream)

    with ClockSampler(device.index) as clk:
        per, total_ms = time_region(step, args.steps, args.warmup, stream, device)
        # The timed region is short next to the 200 ms sampling period: the same calls keep
        # running (untimed) for about a second more, so that the record shows the clocks
        # and power under this load, not only around it.
        soak_end, i = time.time() + 1.0, 0
        while time.time() < soak_end:
            for _ in range(64):
                step(i)
                i += 1
            torch.cuda.synchronize(device)
    launches += head_kernels * args.steps
    kda.workspace_status(ws)
    clocks = clk.summary()
    clocks["window"] = "the timed region, then 1 s more of the same calls (untimed)"
    total_ms_max = max_over_ranks(total_ms, device)
    ms_per_step = total_ms_max / args.steps
    value = job_throughput(T1 * args.steps, world, total_ms_max / 1e3)
    kern_ms = statistics.mean(per)
    achieved_gbs = bytes_call / (kern_ms / 1e3) / 1e9
    tc_tflops = prefill_tc_flops(T1) / (kern_ms / 1e3) / 1e12

    # ---------------- e2e: host buffers through the public API ----------------------
    # Every step copies its inputs from pinned host memory and reads its output and final
    # state back; steps are pipelined as a caller streaming requests would run them: the
    # upload of step i+1 (copy-in stream) overlaps the kernels of step i (compute stream)
    # and the download of step i-1 (copy-out stream), over two device buffer sets.
    pin = {k: t.pin_memory() for k, t in host.items()}
    nbuf = 2
    devs = [{k: torch.empty_like(t, device=device) for k, t in host.items()} for _ in range(nbuf)]
    d_outs = [torch.empty(T1, H, D, dtype=torch.bfloat16, device=device) for _ in range(nbuf)]
    d_fins = [torch.empty(1, H, D, D, dtype=torch.float32, device=device) for _ in range(nbuf)]
    h_out = torch.empty(T1, H, D, dtype=torch.bfloat16).pin_memory()
    h_fin = torch.empty(1, H, D, D, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = h_out.numel() * 2 + h_fin.numel() * 4
    copy_in, copy_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    uploaded, computed, downloaded = [ev() for _ in range(nbuf)], [ev() for _ in range(nbuf)], [ev() for _ in range(nbuf)]
    used = [False] * nbuf

    def e2e_step(i):
        b = i % nbuf
        if used[b]:  # buffer set b: step i - nbuf's kernels and download are done with it
            copy_in.wait_event(computed[b])
            stream.wait_event(downloaded[b])
        used[b] = True
        with torch.cuda.stream(copy_in):
            for k in pin:
                devs[b][k].copy_(pin[k], non_blocking=True)
            uploaded[b].record(copy_in)
        stream.wait_event(uploaded[b])
        x = devs[b]
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], None,
                      N=1, out=d_outs[b], final_state=d_fins[b], workspace=ws, stream=stream)
        computed[b].record(stream)
        copy_out.wait_event(computed[b])
        with torch.cuda.stream(copy_out):
            h_out.copy_(d_outs[b], non_blocking=True)
            h_fin.copy_(d_fins[b], non_blocking=True)
            downloaded[b].record(copy_out)

    def e2e_region(n):
        """n pipelined steps between events on the compute stream, which waits for the
        last download before the closing event."""
        torch.cuda.synchronize(device)
        barrier(device)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_in.wait_stream(stream)
        copy_out.wait_stream(stream)
        for i in range(n):
            e2e_step(i)
        stream.wait_stream(copy_in)
        stream.wait_stream(copy_out)
        e1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        return e0.elapsed_time(e1)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_region(max(3, min(args.warmup, 3)))  # warm-up
    e2e_ms = max_over_ranks(e2e_region(e2e_steps), device)
    e2e_value = job_throughput(T1 * e2e_steps, world, e2e_ms / 1e3)
    launches += head_kernels * e2e_steps

    # ---------------- decode: 256 sequences x 32 heads, 64 in-place steps ----------------
    Nd, dsteps = 256, 64
    gd = torch.Generator(device=device).manual_seed(1370003)
    state = 0.02 * torch.randn(Nd, H, D, D, generator=gd, device=device)
    n_tok_sets = 8
    toks = []
    for _ in range(n_tok_sets):
        q = torch.randn(Nd, H, D, generator=gd, device=device)
        k = torch.randn(Nd, H, D, generator=gd, device=device)
        toks.append(dict(q=(q / q.norm(dim=-1, keepdim=True)).bfloat16(), k=(k / k.norm(dim=-1, keepdim=True)).bfloat16(),
                         v=torch.randn(Nd, H, D, generator=gd, device=device).bfloat16(),
                         la=(-torch.nn.functional.softplus(torch.randn(Nd, H, D, generator=gd, device=device)) / 16).contiguous(),
                         b=torch.sigmoid(torch.randn(Nd, H, generator=gd, device=device)).contiguous()))
    d_outbuf = torch.empty(Nd, H, D, dtype=torch.bfloat16, device=device)

    def dstep(i):
        t = toks[i % n_tok_sets]
        kda.decode_step(t["q"], t["k"], t["v"], t["la"], t["b"], state, out=d_outbuf, stream=stream)

    dper, dtot = time_region(dstep, dsteps, 3, stream, device)
    launches += dsteps
    dtot = max_over_ranks(dtot, device)
    dbytes = decode_bytes(Nd)
    d_us = dtot / dsteps * 1e3
    decode = {"workload": f"decode N={Nd} H={H} d={D} fp32 state in place, {dsteps} consecutive steps",
              "us_per_step": d_us, "state_GBps": 2 * Nd * H * D * D * 4 / (d_us * 1e-6) / 1e9,
              "GBps_all_bytes": dbytes / (d_us * 1e-6) / 1e9,
              "tokens_per_s": job_throughput(Nd * dsteps, world, dtot / 1e3),
              "roofline": {"bound": "hbm", "achieved": dbytes / (statistics.mean(dper) * 1e-3) / 1e9, "peak": hbm_peak,
                           "unit": "GB/s", "frac": dbytes / (statistics.mean(dper) * 1e-3) / 1e9 / hbm_peak,
                           "algorithmic_bytes_per_launch": dbytes}}
    del state, toks

    # ---------------- serving mixer decode: conv history + L2 + KDA + gate, pooled ---------
    mdec = None
    if not args.quick:
        pool = Nd
        gm = torch.Generator(device=device).manual_seed(1370005)
        sp = 0.02 * torch.randn(pool, H, D, D, generator=gm, device=device)
        cp = torch.randn(pool, H, 3, 3, D, generator=gm, device=device).bfloat16()
        idx = torch.randperm(pool, generator=gm, device=device).to(torch.int32)
        cw = (0.5 * torch.randn(3, H * D, 4, generator=gm, device=device)).contiguous()
        mtoks = []
        for _ in range(n_tok_sets):
            mtoks.append(dict(q=torch.randn(Nd, H, D, generator=gm, device=device).bfloat16(),
                              k=torch.randn(Nd, H, D, generator=gm, device=device).bfloat16(),
                              v=torch.randn(Nd, H, D, generator=gm, device=device).bfloat16(),
                              g=torch.randn(Nd, H, D, generator=gm, device=device).bfloat16(),
                              la=(-torch.nn.functional.softplus(torch.randn(Nd, H, D, generator=gm, device=device))
                                  / 16).contiguous(),
                              b=torch.sigmoid(torch.randn(Nd, H, generator=gm, device=device)).contiguous()))
        md_out = torch.empty(Nd, H, D, dtype=torch.bfloat16, device=device)

        def mdstep(i):
            t = mtoks[i % n_tok_sets]
            kda.mixer_decode_step(t["q"], t["k"], t["v"], cw, t["la"], t["b"], t["g"], sp, cp, idx, out=md_out,
                                  stream=stream)

        mper, mtot = time_region(mdstep, dsteps, 3, stream, device)
        launches += dsteps
        mtot = max_over_ranks(mtot, device)
        mbytes_d = mixer_decode_bytes(Nd)
        m_us = mtot / dsteps * 1e3
        mdec = {"workload": f"serving mixer decode N={Nd} H={H} d={D}: conv4 over a 3-row history, L2, KDA, gate; "
                            f"states and histories at permuted slots of a {pool}-slot pool, {dsteps} steps",
                "us_per_step": m_us, "tokens_per_s": job_throughput(Nd * dsteps, world, mtot / 1e3),
                "roofline": {"bound": "hbm", "achieved": mbytes_d / (statistics.mean(mper) * 1e-3) / 1e9,
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": mbytes_d / (statistics.mean(mper) * 1e-3) / 1e9 / hbm_peak,
                             "algorithmic_bytes_per_launch": mbytes_d}}
        # K = 4 draft tokens per call (no checkpoints: the pools get the state after the 4)
        Kt = 4
        ktok = [{k: torch.stack([mtoks[(s + j) % n_tok_sets][k] for j in range(Kt)], dim=1).contiguous()
                 for k in mtoks[0]} for s in range(2)]
        mk_out = torch.empty(Nd, Kt, H, D, dtype=torch.bfloat16, device=device)

        def mkstep(i):
            t = ktok[i % 2]
            kda.mixer_decode_tokens(t["q"], t["k"], t["v"], cw, t["la"], t["b"], t["g"], sp, cp, idx, out=mk_out,
                                    stream=stream)

        ksteps = 16
        kper, ktot = time_region(mkstep, ksteps, 3, stream, device)
        launches += ksteps
        ktot = max_over_ranks(ktot, device)
        kbytes = mixer_decode_tokens_bytes(Nd, Kt)
        mdec["k_tokens"] = {
            "workload": f"{Kt} tokens per sequence per call (N={Nd} H={H}), state kept on chip across them",
            "us_per_call": ktot / ksteps * 1e3, "tokens_per_s": job_throughput(Nd * Kt * ksteps, world, ktot / 1e3),
            "roofline": {"bound": "hbm", "achieved": kbytes / (statistics.mean(kper) * 1e-3) / 1e9, "peak": hbm_peak,
                         "unit": "GB/s", "frac": kbytes / (statistics.mean(kper) * 1e-3) / 1e9 / hbm_peak,
                         "algorithmic_bytes_per_launch": kbytes}}
        del sp, cp, mtoks, ktok

    # ---------------- context-parallel prefill, its pieces timed on one GPU ---------------
    cpar = None
    if not args.quick:
        from gated_delta_rule_137_b200 import context_parallel as cpm
        segs, Tc = 4, 4 * T1
        ci = device_prefill_inputs(Tc, H, D, 1370006, device, state_N=1)
        cargs = [ci[k] for k in ("q", "k", "v", "log_alpha", "beta")]
        seg_of = lambda x, i: x[i * T1:(i + 1) * T1].contiguous()
        segs_in = [[seg_of(x, i) for x in cargs] for i in range(segs)]
        maps = [kda.segment_maps(*p, N=1) for p in segs_in]
        last = segs_in[segs - 1]

        def timed(fn, n=5):
            for _ in range(2):
                fn()
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
            return e0.elapsed_time(e1) / n

        MB = torch.stack([torch.stack([m[0], m[1]]) for m in maps])  # the all-gather's layout
        S_last = torch.empty_like(ci["initial_state"])
        fold = lambda: lib.kda_state_fold(MB.data_ptr(), segs - 1, ci["initial_state"].data_ptr(),
                                          S_last.data_ptr(), H, D, stream.cuda_stream)
        kda._check(fold())
        mws = maps[segs - 1][2].workspace
        M_l, B_l = torch.empty_like(maps[0][0]), torch.empty_like(maps[0][1])
        o_l = torch.empty(T1, H, D, dtype=torch.bfloat16, device=device)
        f_l = torch.empty(1, H, D, D, dtype=torch.float32, device=device)
        t_map = timed(lambda: lib.kda_segment_maps(last[0].data_ptr(), last[1].data_ptr(), last[2].data_ptr(),
                                                   kda.KDA_DT_BF16, last[3].data_ptr(), last[4].data_ptr(), None,
                                                   T1, 1, H, D, D, M_l.data_ptr(), B_l.data_ptr(), mws.data_ptr(),
                                                   mws.numel(), stream.cuda_stream))
        t_fold = timed(fold)
        t_final = timed(lambda: lib.kda_segment_prefill(mws.data_ptr(), mws.numel(), kda.KDA_DT_BF16,
                                                        S_last.data_ptr(), None, T1, 1, H, D, D, o_l.data_ptr(),
                                                        f_l.data_ptr(), stream.cuda_stream))
        t_emul = timed(lambda: cpm.context_parallel_emulate(*cargs, ci["initial_state"], N=1, segments=segs), 3)
        t_plain = timed(lambda: kda.chunk_fwd(*cargs, ci["initial_state"], None, N=1), 3)
        # timed calls x kernels: maps 7 x 3, fold 7 x 1, segment prefill 7 x 1,
        # emulation 5 x (4 maps x 3 + 3 folds + 4 prefills x 1), plain prefill 5 x 3
        launches += 7 * 3 + 7 + 7 + 5 * (4 * 3 + 3 + 4) + 5 * 3
        cpar = {"workload": f"context-parallel prefill of one {Tc}-token sequence (H={H} d={D}) in {segs} segments; "
                            "pieces timed on one GPU with CUDA events (the exchange is not part of it); the last "
                            "rank's path: segment maps, fold of the earlier maps, segment prefill",
                "segment_maps_ms": t_map, "fold_ms": t_fold, "segment_prefill_ms": t_final,
                "per_rank_path_ms": t_map + t_fold + t_final,
                "emulated_on_one_gpu_ms": t_emul, "plain_prefill_ms": t_plain,
                "exchange_bytes_per_rank": 2 * H * D * D * 4}
        del ci, cargs, maps, last, segs_in, MB

    # ---------------- full mixer (conv4 + L2 + KDA + gate), B=2 x T=32768 ----------------
    mix = None
    if not args.quick:
        Bm, Tm = 2, 32768
        mi = device_prefill_inputs(Bm * Tm, H, D, 1370002, device, normalise=False, mixer=True)
        mo = torch.empty(Bm * Tm, H, D, dtype=torch.bfloat16, device=device)
        mf = torch.empty(Bm, H, D, D, dtype=torch.float32, device=device)
        mws = torch.empty(lib.kda_mixer_fwd_workspace(Bm * Tm, Bm, H, D, D), dtype=torch.uint8, device=device)

        def mstep(i):
            kda.mixer_fwd(mi["q"], mi["k"], mi["v"], mi["conv_w"], mi["log_alpha"], mi["beta"], mi["gate"], None,
                          None, N=Bm, out=mo, final_state=mf, workspace=mws, stream=stream)

        msteps = max(3, min(args.steps, 10))
        mper, mtot = time_region(mstep, msteps, 2, stream, device)
        launches += kernels_per_call(mws.numel()) * msteps
        mtot = max_over_ranks(mtot, device)
        mbytes = prefill_bytes(Bm * Tm, Bm, with_h0=False, mixer=True)
        mms = statistics.mean(mper)
        mix = {"workload": f"full mixer B={Bm} T={Tm} H={H} d={D} (conv4 + L2 + KDA + sigmoid gate)",
               "ms_per_call": mtot / msteps, "tokens_per_s": job_throughput(Bm * Tm * msteps, world, mtot / 1e3),
               "roofline": {"bound": "hbm", "achieved": mbytes / (mms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                            "frac": mbytes / (mms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes_per_launch": mbytes}}
        # the same mixer with the decay gate made on the device from its bf16 pre-activation
        a_pre = torch.randn(Bm * Tm, H, D, generator=torch.Generator(device=device).manual_seed(1370007),
                            device=device).bfloat16()
        a_scale = torch.full((H,), 1 / 16, device=device)
        gws = torch.empty(lib.kda_mixer_fwd_gate_workspace(Bm * Tm, Bm, H, D, D), dtype=torch.uint8, device=device)

        def gstep(i):
            kda.mixer_fwd_gate(mi["q"], mi["k"], mi["v"], mi["conv_w"], a_pre, a_scale, mi["beta"], mi["gate"], None,
                               None, N=Bm, out=mo, final_state=mf, workspace=gws, stream=stream)

        gper, gtot = time_region(gstep, msteps, 2, stream, device)
        launches += 3 * msteps
        gtot = max_over_ranks(gtot, device)
        gbytes = mbytes - Bm * Tm * H * D * 2  # log_alpha fp32 -> a_pre bf16
        gms = statistics.mean(gper)
        mix["gate_from_preactivation"] = {
            "workload": "same mixer, log_alpha = -scale_h softplus(a) made on the device from bf16 a",
            "ms_per_call": gtot / msteps, "tokens_per_s": job_throughput(Bm * Tm * msteps, world, gtot / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbytes / (gms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbytes / (gms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes_per_launch": gbytes}}
        del mi, mo, mws, a_pre, gws

    # ---------------- varlen packed prefill, 64 sequences U[256, 8192] ------------------
    var = None
    if not args.quick:
        rng = np.random.default_rng(I.SEED_BASE + 4)
        lens = [int(x) for x in rng.integers(256, 8193, 64)]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=device)
        TT = int(sum(lens))
        vi = device_prefill_inputs(TT, H, D, 1370004, device, state_N=len(lens))
        vo = torch.empty(TT, H, D, dtype=torch.bfloat16, device=device)
        vf = torch.empty(len(lens), H, D, D, dtype=torch.float32, device=device)
        vws = torch.empty(kda.chunk_fwd_workspace_bytes(TT, len(lens), H, D, D, kda.KDA_DT_BF16), dtype=torch.uint8,
                          device=device)

        def vstep(i):
            kda.chunk_fwd(vi["q"], vi["k"], vi["v"], vi["log_alpha"], vi["beta"], vi["initial_state"], cu,
                          N=len(lens), out=vo, final_state=vf, workspace=vws, stream=stream)

        vsteps = max(3, min(args.steps, 10))
        vper, vtot = time_region(vstep, vsteps, 2, stream, device)
        launches += kernels_per_call(vws.numel()) * vsteps
        vtot = max_over_ranks(vtot, device)
        vbytes = prefill_bytes(TT, len(lens))
        vms = statistics.mean(vper)
        var = {"workload": f"varlen prefill 64 seqs (U[256,8192], {TT} tokens) H={H} d={D}",
               "ms_per_call": vtot / vsteps, "tokens_per_s": job_throughput(TT * vsteps, world, vtot / 1e3),
               "roofline": {"bound": "hbm", "achieved": vbytes / (vms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                            "frac": vbytes / (vms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes_per_launch": vbytes},
               "tensor_tflops": prefill_tc_flops(TT) / (vms * 1e-3) / 1e12}
        del vi, vo, vf, vws

    # ---------------- backward of the recurrence, the model shape B=1 T=4096 H=32 ---------------
    bwd = None
    if not args.quick:
        bi = device_prefill_inputs(T1, H, D, 1370008, device, state_N=1)
        gen = torch.Generator(device=device).manual_seed(1370009)
        d_out = torch.randn(T1, H, D, generator=gen, device=device).bfloat16()
        d_fin = 0.1 * torch.randn(1, H, D, D, generator=gen, device=device)
        bws = torch.empty(kda.chunk_bwd_workspace_bytes(T1, 1, H), dtype=torch.uint8, device=device)

        def bstep(i):
            kda.chunk_bwd(bi["q"], bi["k"], bi["v"], bi["log_alpha"], bi["beta"], d_out, bi["initial_state"], None,
                          d_fin, N=1, workspace=bws, stream=stream)

        bsteps = max(3, min(args.steps, 5))
        bper, btot = time_region(bstep, bsteps, 3, stream, device)
        launches += 2 * bsteps  # plan + backward kernel
        btot = max_over_ranks(btot, device)
        bbytes = backward_bytes(T1, 1)
        bms = statistics.mean(bper)
        bwd = {"workload": f"backward of the recurrence B=1 T={T1} H={H} d={D} (bf16 q/k/v/d_out, fp32 gradients, "
                           "initial state and final-state gradient)",
               "ms_per_call": btot / bsteps, "tokens_per_s": job_throughput(T1 * bsteps, world, btot / 1e3),
               "roofline": {"bound": "hbm", "achieved": bbytes / (bms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                            "frac": bbytes / (bms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes_per_launch": bbytes}}
        del bi, d_out, d_fin, bws

    cpu = cpu_baseline(args) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded NumPy generator; random inputs, no weights)",
            "config": headline_config(world),
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved_gbs / hbm_peak, "traffic": load_traffic(args.traffic),
                         "kernel": "kda_chunk_fwd (plan + intra-chunk + recurrence kernels, one call)",
                         "algorithmic_bytes_per_launch": bytes_call,
                         "kernel_us": kern_ms * 1e3, "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_src}, burst copy)",
                         "tensor": {"achieved_tflops": tc_tflops, "flops_per_launch": prefill_tc_flops(T1),
                                    "flops_count": "triangle-aware, 6 d^2 + 5 C d per token-head",
                                    "mma_kind": "tf32",
                                    "peak_tflops_tf32": tc_peak * TF32_PER_BF16,
                                    "frac_tf32": tc_tflops / (tc_peak * TF32_PER_BF16),
                                    "peak_tflops_bf16": tc_peak, "frac_bf16": tc_tflops / tc_peak,
                                    "peak_source": f"MEASURED_PEAKS.json bf16_tflops ({peak_src}, burst) x "
                                                   f"{TF32_PER_BF16:.3f} (nominal tf32 : bf16)",
                                    "issued_flops_per_launch": prefill_tc_flops_issued(T1),
                                    "issued_tflops": prefill_tc_flops_issued(T1) / (kern_ms / 1e3) / 1e12}},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "pipelining": "2 device buffer sets; upload, kernels and download of consecutive steps overlap "
                                  "on three streams; every step's copies are inside the timed region"},
            "decode": decode, "mixer_decode": mdec, "context_parallel": cpar, "mixer": mix, "varlen": var,
            "backward": bwd, "clocks": clocks, "gpu_launches": launches, "cpu_baseline": cpu,
        }
        # the figures a reader of the line's tail needs, last (a truncated copy keeps them)
        frac = lambda x: None if x is None else round(x["roofline"]["frac"], 4)
        line["summary"] = {
            "prefill_us": round(kern_ms * 1e3, 1), "prefill_frac": round(achieved_gbs / hbm_peak, 4),
            "decode_us_per_step": round(decode["us_per_step"], 1), "decode_frac": frac(decode),
            "mixer_decode_frac": frac(mdec), "mixer_ms": None if mix is None else round(mix["ms_per_call"], 3),
            "mixer_frac": frac(mix), "varlen_ms": None if var is None else round(var["ms_per_call"], 3),
            "varlen_frac": frac(var), "backward_ms": None if bwd is None else round(bwd["ms_per_call"], 3),
            "backward_frac": frac(bwd), "e2e_tokens_per_s": round(e2e_value),
            "tensor_frac_tf32": round(tc_tflops / (tc_peak * TF32_PER_BF16), 4)}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(device)
        dist.destroy_process_group()


# ----------------------------------------------------------------------------------
# CPU oracle: the reported baseline and the reference arm
# ----------------------------------------------------------------------------------
def oracle_sample(heads: int = 2, T: int = T1):
    """Times the fp64 oracle on `heads` of the 32 heads over T tokens of the
    model-shape prefill; returns (token-equivalents/s at H=32, seconds, description)."""
    from gated_delta_rule_137_b200 import inputs as I
    from oracle import kda_oracle as O
    w = I.prefill_model_shape(T)
    hs = list(range(heads))
    t0 = time.perf_counter()
    O.kda_recurrence(w.q[:, hs], w.k[:, hs], w.v[:, hs], w.log_alpha[:, hs], w.beta[:, hs],
                     w.initial_state[:, hs], w.cu_seqlens)
    dt = time.perf_counter() - t0
    tok_equiv = T * heads / H
    return tok_equiv / dt, dt, f"fp64 NumPy oracle, {heads} of {H} heads x {T} tokens of the B=1 T=4096 workload (scaled to all heads)"


def oracle_threads():
    """The oracle runs single-threaded: its contractions are NumPy einsums without BLAS,
    and any BLAS pool is capped at one thread while it is timed. Returns a context
    manager for that cap and a record of the host (cores, BLAS pools before the cap)."""
    import numpy  # noqa: F401  (loads the BLAS the oracle would see)
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        pools = [{"api": p.get("internal_api"), "threads": p.get("num_threads")} for p in threadpool_info()]
        cap = threadpool_limits(limits=1)
    except ImportError:  # pragma: no cover - threadpoolctl ships with the image
        import contextlib
        pools, cap = [], contextlib.nullcontext()
    return cap, {"host_cpu_count": os.cpu_count(), "blas_pools_default": pools, "blas_threads_used": 1}


def cpu_baseline(args):
    cap, host = oracle_threads()
    with cap:
        v, dt, desc = oracle_sample(heads=args.cpu_heads)
    return {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc, "seconds": dt, **host}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    cap, host = oracle_threads()
    per = []
    with cap:
        for _ in range(args.warmup if args.warmup < 1 else 1):
            oracle_sample(heads=1, T=256)
        for _ in range(args.steps):
            v, dt, desc = oracle_sample(heads=1, T=1024)
            per.append(dt)
    total = sum(per)
    tok_equiv = args.steps * 1024 * 1 / H
    value = tok_equiv / total
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded NumPy generator)",
        "config": headline_config(world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: 1 of 32 heads x the first 1024 tokens (scaled to all heads)", **host},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile_case(args):
    """A mid-size single-pass prefill for kernel captures: 8 packed sequences x 4096
    tokens x 32 heads (256 chains, so the single-pass kernel; 1.6 GB of inputs, above L2),
    W + K calls, then one line with the CUDA-event time per call."""
    import torch
    import gated_delta_rule_137_b200 as kda
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    kda.load_library()
    n, T = 8, 4096
    x = device_prefill_inputs(n * T, H, D, 1370010, device, state_N=n)
    out = torch.empty(n * T, H, D, dtype=torch.bfloat16, device=device)
    fin = torch.empty(n, H, D, D, dtype=torch.float32, device=device)
    ws = torch.empty(max(256, kda.chunk_fwd_workspace_bytes(n * T, n, H, D, D, kda.KDA_DT_BF16)), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    def call(i):
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], None, N=n, out=out,
                      final_state=fin, workspace=ws, stream=stream)

    per, tot = time_region(call, args.steps, args.warmup, stream, device)
    print(json.dumps({"case": f"single-pass prefill {n} x {T} tokens, H={H} d={D}", "ms_per_call": tot / args.steps,
                      "bytes_per_call": prefill_bytes(n * T, n)}), flush=True)


def run_profile_tokens(args):
    """The serving decode with K = 4 draft tokens per call (N = 256 sequences x 32 heads,
    no checkpoints, the block form), W + K calls, then one line with the CUDA-event time
    per call; for kernel captures."""
    import torch
    import gated_delta_rule_137_b200 as kda
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    kda.load_library()
    Nd, Kt = 256, 4
    g = torch.Generator(device=device).manual_seed(1370005)
    sp = 0.02 * torch.randn(Nd, H, D, D, generator=g, device=device)
    cp = torch.randn(Nd, H, 3, 3, D, generator=g, device=device).bfloat16()
    idx = torch.randperm(Nd, generator=g, device=device).to(torch.int32)
    cw = (0.5 * torch.randn(3, H * D, 4, generator=g, device=device)).contiguous()
    t = dict(q=torch.randn(Nd, Kt, H, D, generator=g, device=device).bfloat16(),
             k=torch.randn(Nd, Kt, H, D, generator=g, device=device).bfloat16(),
             v=torch.randn(Nd, Kt, H, D, generator=g, device=device).bfloat16(),
             g=torch.randn(Nd, Kt, H, D, generator=g, device=device).bfloat16(),
             la=(-torch.nn.functional.softplus(torch.randn(Nd, Kt, H, D, generator=g, device=device)) / 16).contiguous(),
             b=torch.sigmoid(torch.randn(Nd, Kt, H, generator=g, device=device)).contiguous())
    out = torch.empty(Nd, Kt, H, D, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def call(i):
        kda.mixer_decode_tokens(t["q"], t["k"], t["v"], cw, t["la"], t["b"], t["g"], sp, cp, idx, out=out,
                                stream=stream)

    per, tot = time_region(call, args.steps, args.warmup, stream, device)
    print(json.dumps({"case": f"serving decode, {Kt} tokens per call, N={Nd} H={H} d={D}",
                      "us_per_call": tot / args.steps * 1e3,
                      "bytes_per_call": mixer_decode_tokens_bytes(Nd, Kt)}), flush=True)


def run_profile_mixer(args):
    """The full mixer (conv4 + L2 + KDA + gate) on 2 x 8192 tokens of 32 heads — the config-2
    shape with a quarter of its tokens (about 2 GB on the device), W + K calls, then one
    line with the CUDA-event time per call; for kernel captures."""
    import torch
    import gated_delta_rule_137_b200 as kda
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    lib = kda.load_library()
    Bm, Tm = 2, 8192
    mi = device_prefill_inputs(Bm * Tm, H, D, 1370002, device, normalise=False, mixer=True)
    mo = torch.empty(Bm * Tm, H, D, dtype=torch.bfloat16, device=device)
    mf = torch.empty(Bm, H, D, D, dtype=torch.float32, device=device)
    mws = torch.empty(lib.kda_mixer_fwd_workspace(Bm * Tm, Bm, H, D, D), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def call(i):
        kda.mixer_fwd(mi["q"], mi["k"], mi["v"], mi["conv_w"], mi["log_alpha"], mi["beta"], mi["gate"], None,
                      None, N=Bm, out=mo, final_state=mf, workspace=mws, stream=stream)

    per, tot = time_region(call, args.steps, args.warmup, stream, device)
    print(json.dumps({"case": f"full mixer {Bm} x {Tm} tokens, H={H} d={D}", "ms_per_call": tot / args.steps,
                      "bytes_per_call": prefill_bytes(Bm * Tm, Bm, with_h0=False, mixer=True)}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="headline and decode only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-heads", type=int, default=32)
    ap.add_argument("--profile-case", action="store_true",
                    help="only a mid-size single-pass prefill (8 x 4096 tokens, 32 heads), for kernel captures")
    ap.add_argument("--profile-tokens", action="store_true",
                    help="only the 4-token serving decode (256 sequences, 32 heads), for kernel captures")
    ap.add_argument("--profile-mixer", action="store_true",
                    help="only the full mixer on 2 x 8192 tokens (32 heads), for kernel captures")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per headline call to report instead of profiles/traffic.json")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.profile_case:
        run_profile_case(args)
    elif args.profile_tokens:
        run_profile_tokens(args)
    elif args.profile_mixer:
        run_profile_mixer(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
