#!/usr/bin/env python
"""Benchmark of the Simple GLA mixer hot path on B200.

One step = one training step of one Laplace-layer mixer at B = 8, T = 2048,
H = 16, dk = 96, dv = 192 in bf16: the chunked forward followed by the
chunked backward (dO ~ N(0,1), zero gradient on the final state), as the
library's training pair gla_chunk_fwd_train (which keeps the state entering
every chunk) and gla_chunk_bwd_saved (which reads them).  The headline value is
chunk fwd+bwd tokens/s over all ranks.  The metric also names decode
tokens/s at 1,280 sequences, so the same run times the 24-layer decode step
(1,280 sequences x 24 layers x 16 heads, fp32 state in place) and reports
it under "decode", and the long-context prefill (T = 65,536: the LayerNorm +
conv + SiLU front end, then the chunked forward with S_0) under
"long_prefill", each call against its HBM roofline.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
cuda synchronize, measured with CUDA events on the launching stream, max
over ranks.  Inputs (about 0.6 GB per rank for the training step, 36 GB of
decode state) are larger than the 126 MB L2, so no flush is needed.
Rooflines, all against MEASURED_PEAKS.json:
  roofline       the dominant kernel: right after the timed region the same K
                 steps run again with libgla's per-launch event tracing
                 (events between launches cost a few percent, so they stay
                 out of the headline region); its method bytes (the inputs
                 and outputs of the computation it reads or writes) per
                 launch over its mean launch time against HBM copy bandwidth,
                 with its design bytes (per-chunk states, partial sums) and
                 its bf16 tensor-core fraction beside it, and under
                 "per_kernel" the same fractions for every kernel of the step;
  roofline_step  the whole step: 3,084 method bytes per token-head (+ the
                 final state) against HBM, 64.5 MF of algorithmic flops per
                 (batch, head, chunk) against the sustained bf16 peak;
  prefill_fwd    the forward alone at the same shape, both rooflines.
The dominant kernel's "traffic" (DRAM bytes per launch) comes from the ncu
capture summarised in profiles/dram_traffic.md, and only while the digest of
the kernel's source files (their code, comments removed) still matches the
one recorded there; otherwise it is null.

--skip-decode / --skip-e2e time only the training step: the command the
profiles' ncu captures run (a few GB on the device instead of the 36 GB of
decode state); --skip-decode also skips the long prefill.
"""
import hashlib
import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import linear_attention_simple_b200 as gla  # noqa: E402
from linear_attention_simple_b200 import inputs  # noqa: E402
from linear_attention_simple_b200.configs import WORKLOADS  # noqa: E402

METRIC = "GLA chunk fwd+bwd tokens/s; decode tokens/s at 1280 seqs; % of roofline"
TRAIN = WORKLOADS["train_fwd_bwd_b8_t2048"]
DECODE = WORKLOADS["decode_n1280_l24"]
LONG = WORKLOADS["long_prefill_t65536"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Byte and flop models per unit = one (batch, head, 128-token chunk).  bf16
# tiles: q, k 24,576 B; v, o, dO 49,152 B; a 512 B; one bf16 plane of a
# per-chunk state 36,864 B; an fp32 state 73,728 B.
QK, VO, A, HS, FS = 24576, 49152, 512, 36864, 73728
# Method bytes: the inputs and outputs of the computation itself (q, k, v, a
# in and o out forward; q, k, v, dO, a in and dq, dk, dv, da out backward),
# counted for the kernel that reads or writes them.  The roofline fraction is
# taken on these.
METHOD_BYTES = {
    "chunk_fwd_fused_kernel": 2 * QK + 2 * VO + A,      # q, k, v, a in; o out   (+ S_T per head)
    "chunk_state_fwd_kernel": QK + VO + A,              # k, v, a in
    "chunk_state_rev_kernel": QK + VO + A,              # q, dO, a in
    "bwd_dqdk_kernel": 2 * QK + 2 * VO + A + 2 * QK,    # q, k, v, dO, a in; dq, dk out
    "chunk_rev_fused_kernel": 2 * QK + VO + A + VO,     # q, k, dO, a in; dv out (reverse sweep + dv)
    "da_finish_kernel": A,                              # da out
}
# Design bytes: intermediates the kernels exchange through HBM (the
# per-chunk states as bf16 hi + lo planes, the per-token halves of the da
# sum), reported beside the method bytes and not counted in the fraction.
DESIGN_BYTES = {
    "chunk_fwd_fused_kernel": 2 * HS,                   # training forward: h_c kept (hi, lo)
    "chunk_state_fwd_kernel": 2 * HS,                   # h_c written (hi, lo)
    "chunk_state_rev_kernel": 2 * HS,                   # D_c written (hi, lo)
    "bwd_dqdk_kernel": 2 * 2 * HS + 2 * A,              # h_c, D_c read (hi, lo); q.dq, k.dk written
    "chunk_rev_fused_kernel": 2 * HS,                   # D_c written (hi, lo)
    "da_finish_kernel": 2 * A,                          # q.dq, k.dk read
}
# Algorithmic flops per unit on dense 128-token tiles (2 m n k per product;
# the hi + lo splits the kernels make for precision are not counted).
MM = lambda m, n, k: 2 * m * n * k  # noqa: E731
CHUNK_FLOPS = {
    # scores Q K^T, Q S_prev, P V, state update K~^T V
    "chunk_fwd_fused_kernel": MM(128, 128, 96) + MM(128, 192, 96) + MM(128, 192, 128) + MM(96, 192, 128),
    "chunk_state_fwd_kernel": MM(96, 192, 128),          # K~^T V
    "chunk_state_rev_kernel": MM(96, 192, 128),          # Q~^T dO
    # dP = dO V^T, dO h^T, dP K, V D^T, dP^T Q
    "bwd_dqdk_kernel": MM(128, 128, 192) + 2 * MM(128, 96, 192) + 2 * MM(128, 96, 128),
    # the reverse sweep with dv fused in: scores^T K Q^T, K D, P~ dO, and Q~^T dO
    "chunk_rev_fused_kernel": MM(128, 128, 96) + MM(128, 192, 96) + MM(128, 192, 128) + MM(96, 192, 128),
}
# The whole training step per unit: forward (q, k, v, a in, o out) and
# backward (q, k, v, dO, a in; dq, dk, dv, da out) method bytes, and the
# forward + backward algorithmic flops (18.9 + 45.6 MF: the backward counted
# with both state scans, whichever kernel runs them).
STEP_BYTES = (2 * QK + 2 * VO + A) + (2 * QK + 2 * VO + A + 2 * QK + VO + A)
STEP_FLOPS = sum(CHUNK_FLOPS[k] for k in ("chunk_fwd_fused_kernel", "chunk_state_fwd_kernel",
                                           "chunk_rev_fused_kernel", "bwd_dqdk_kernel"))


# Source files each kernel is built from (the digest that ties a recorded
# ncu traffic figure to the code it was measured on).
CSRC = os.path.join(ROOT, "linear_attention_simple_b200", "csrc")
KERNEL_SOURCES = {
    "chunk_fwd_fused_kernel": ("chunk_fwd.cu", "chunk_state.cuh", "gla_device.cuh"),
    "chunk_state_fwd_kernel": ("chunk_fwd.cu", "chunk_state.cuh", "gla_device.cuh"),
    "chunk_state_rev_kernel": ("chunk_fwd.cu", "chunk_state.cuh", "gla_device.cuh"),
    "bwd_dqdk_kernel": ("chunk_bwd.cu", "chunk_state.cuh", "gla_device.cuh"),
    "chunk_rev_fused_kernel": ("chunk_fwd.cu", "chunk_state.cuh", "gla_device.cuh"),
    "da_finish_kernel": ("chunk_bwd.cu",),
}


def strip_comments(src):
    """C++ source text without its comments and blank lines (a comment-only
    edit leaves the compiled kernel, and so its digest, unchanged)."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] in "\"'":
            q, j = src[i], i + 1
            while j < n and src[j] != q:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return "\n".join(l.rstrip() for l in "".join(out).splitlines() if l.strip())


def kernel_digest(name):
    """Digest of the code (comments aside) of the files a kernel is built from."""
    files = KERNEL_SOURCES.get(name)
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:12]


def recorded_traffic(name):
    """DRAM bytes per launch of `name` from profiles/dram_traffic.md, if the
    row's source digest matches the current sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    dig = kernel_digest(name)
    if dig is None or not os.path.exists(path):
        return None
    for line in open(path):
        cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[0] == name and cells[1] == dig:
            try:
                return int(cells[4].replace(",", ""))
            except ValueError:
                return None
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------- helpers

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x, ws, device="cuda"):
    """x maximised over all ranks (every rank gets the result)."""
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def train_buffers(seed, device="cuda"):
    w = TRAIN
    d = inputs.chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=seed, device=device, with_dO=True)
    dev = torch.device(device)
    d["o"] = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    d["sf"] = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    d["grads"] = (torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
                  torch.empty_like(d["a"]), None)
    d["ws_f"] = torch.empty(max(1, gla.gla_chunk_workspace_bytes(w.B, w.T, w.H)), dtype=torch.uint8,
                            device=dev)
    d["ws_b"] = torch.empty(gla.gla_chunk_workspace_bytes(w.B, w.T, w.H, for_bwd=True, from_saved=True),
                            dtype=torch.uint8, device=dev)
    d["saved"] = torch.empty(gla.gla_chunk_saved_state_bytes(w.B, w.T, w.H), dtype=torch.uint8, device=dev)
    return d


def train_step(d):
    """One training step of the mixer: the forward that keeps the per-chunk
    states, then the backward that reads them."""
    gla.gla_chunk_fwd_train(d["q"], d["k"], d["v"], d["a"], o=d["o"], s_final=d["sf"], saved=d["saved"],
                            ws=d["ws_f"])
    gla.gla_chunk_bwd_saved(d["q"], d["k"], d["v"], d["a"], d["saved"], d["dO"], grads=d["grads"], ws=d["ws_b"],
                            want_grad_s0=False)


def kernel_roofline(summary, peaks, peak_kind, units_per_launch, B, H):
    """Roofline of the kernel with the largest summed time in the trace:
    HBM on its method bytes (the fraction), with its design bytes and its
    bf16 tensor-core fraction beside it."""
    if not summary:
        return None, None
    name, launches, total_ms = max(summary, key=lambda r: r[2])
    mean_s = total_ms / launches / 1e3
    if name in METHOD_BYTES:
        bytes_per_launch = METHOD_BYTES[name] * units_per_launch
        if name in ("chunk_fwd_fused_kernel",):
            bytes_per_launch += FS * B * H          # final state written per head
        design = DESIGN_BYTES.get(name, 0) * units_per_launch
        achieved = bytes_per_launch / mean_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "bytes_per_launch": bytes_per_launch, "bytes": "method (inputs and outputs of the path)",
                "design_bytes_per_launch": design,
                "frac_incl_design_bytes": round((bytes_per_launch + design) / mean_s / 1e9 / peak, 4),
                "mean_launch_us": round(mean_s * 1e6, 2),
                "traffic": recorded_traffic(name), "source_digest": kernel_digest(name),
                "peak_source": "%s copy bandwidth" % peak_kind}
        if name in CHUNK_FLOPS:
            tf = CHUNK_FLOPS[name] * units_per_launch / mean_s / 1e12
            tpk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
            roof["tensor"] = {"achieved": round(tf, 1), "peak": tpk, "unit": "TFLOP/s",
                              "frac": round(tf / tpk, 4),
                              "flops_per_launch": CHUNK_FLOPS[name] * units_per_launch,
                              "peak_source": "%s bf16 dense, sustained" % peak_kind}
    else:
        roof = {"kernel": name, "bound": None, "achieved": None, "peak": None, "unit": None,
                "frac": None, "traffic": None, "mean_launch_us": round(mean_s * 1e6, 2)}
    shares = {n: round(t / sum(r[2] for r in summary), 4) for n, _, t in summary}
    return roof, shares


def kernel_rooflines(summary, peaks, units_per_launch, B, H):
    """Every traced kernel with a byte model: mean launch time, HBM fraction
    on its method bytes and with its design bytes, and its bf16 tensor
    fraction where it has an algorithmic flop count."""
    out = {}
    tpk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    for name, launches, total_ms in summary:
        if name not in METHOD_BYTES or launches <= 0:
            continue
        mean_s = total_ms / launches / 1e3
        nb = METHOD_BYTES[name] * units_per_launch + (FS * B * H if name == "chunk_fwd_fused_kernel" else 0)
        design = DESIGN_BYTES.get(name, 0) * units_per_launch
        e = {"mean_launch_us": round(mean_s * 1e6, 2),
             "frac": round(nb / mean_s / 1e9 / peaks["hbm_gbs"], 4),
             "frac_incl_design_bytes": round((nb + design) / mean_s / 1e9 / peaks["hbm_gbs"], 4)}
        if name in CHUNK_FLOPS:
            e["tensor_frac"] = round(CHUNK_FLOPS[name] * units_per_launch / mean_s / 1e12 / tpk, 4)
        out[name] = e
    return out


def step_roofline(step_s, units, B, H, peaks, peak_kind):
    """The training step as a whole against both rooflines: its method bytes
    (+ the final state the forward writes) over HBM, its algorithmic flops
    over the sustained bf16 tensor-core peak."""
    nbytes = STEP_BYTES * units + FS * B * H
    flops = STEP_FLOPS * units
    gbs = nbytes / step_s / 1e9
    tfs = flops / step_s / 1e12
    tpk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    return {"hbm": {"achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_step": nbytes,
                    "peak_source": "%s copy bandwidth" % peak_kind},
            "tensor": {"achieved": round(tfs, 1), "peak": tpk, "unit": "TFLOP/s", "frac": round(tfs / tpk, 4),
                       "flops_per_step": flops, "peak_source": "%s bf16 dense, sustained" % peak_kind},
            "ms_per_step": round(step_s * 1e3, 4)}


# ------------------------------------------------------------ oracle arm

def oracle_sample_time(units, seed, with_bwd=True):
    """Run the fp64 oracle (fwd + bwd) on `units` (batch, head) sequences of
    the training workload; returns (seconds, tokens, threads)."""
    from oracle import recurrent
    w = TRAIN
    d = inputs.chunk_inputs(1, w.T, units, w.dk, w.dv, seed=seed, device="cpu", with_dO=True)
    f = lambda t: t.float().numpy().astype("float64")  # noqa: E731
    q, k, v, a, dO = (f(d[n]) for n in ("q", "k", "v", "a", "dO"))
    t0 = time.perf_counter()
    recurrent.fwd(q, k, v, a)
    if with_bwd:
        recurrent.bwd(q, k, v, a, dO)
    dt = time.perf_counter() - t0
    # one token of the workload covers all H heads
    return dt, units * w.T / w.H, recurrent.max_threads()


def run_reference(args, ws, rank):
    if rank != 0:
        return
    units = max(1, int(os.environ.get("GLA_ORACLE_UNITS", "16")))
    for _ in range(args.warmup):
        oracle_sample_time(units, 7)
    times, toks = [], 0.0
    for i in range(args.steps):
        dt, tok, cores = oracle_sample_time(units, 7 + i)
        times.append(dt)
        toks = tok
    t = sum(times) / len(times)
    value = toks / t
    line = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": TRAIN.name, "global_batch": TRAIN.B, "seq_len": TRAIN.T,
                       "heads": TRAIN.H, "dk": TRAIN.dk, "dv": TRAIN.dv,
                       "parallelism": "oracle on host cores"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": "%d of %d (batch, head) sequences of T=%d per step, fwd+bwd"
                                       % (units, TRAIN.B * TRAIN.H, TRAIN.T)},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ours

def run_ours(args, ws, rank, local):
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()
    peaks, peak_kind = load_peaks()
    if args.only:
        leg = {"decode": run_decode, "decode_front": run_decode_front, "long_prefill": run_long_prefill}[args.only]
        rec = leg(args, ws, peaks, peak_kind)
        if rank == 0:
            print(json.dumps({"only": args.only, args.only: rec}), flush=True)
        return
    st = torch.cuda.current_stream()
    w = TRAIN
    d = train_buffers(seed=w.seed + 97 * rank)
    NC = (w.T + 127) // 128
    units_per_launch = w.B * w.H * NC

    for _ in range(max(3, args.warmup)):
        train_step(d)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)                       # let the sampler come up
    launches0 = gla.gla_launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for _ in range(args.steps):
        train_step(d)
    ev1.record(st)
    ev1.synchronize()
    launches = gla.gla_launch_count() - launches0
    torch.cuda.synchronize()
    barrier(ws)
    elapsed = max_over_ranks(ev0.elapsed_time(ev1) / 1e3, ws)
    ms_step = elapsed / args.steps * 1e3
    value = ws * w.B * w.T * args.steps / elapsed
    # per-kernel times: the same steps again with libgla's per-launch events
    # (kept out of the timed region above: the events themselves cost time)
    gla.gla_trace_enable(True)
    for _ in range(args.steps):
        train_step(d)
    summary = gla.gla_trace_summary()
    gla.gla_trace_enable(False)
    torch.cuda.synchronize()
    roof, shares = kernel_roofline([(n, c, t) for n, c, t in summary], peaks, peak_kind,
                                   units_per_launch, w.B, w.H)
    if roof is not None:
        roof["per_kernel"] = kernel_rooflines(summary, peaks, units_per_launch, w.B, w.H)
    roof_step = step_roofline(elapsed / args.steps, units_per_launch, w.B, w.H, peaks, peak_kind)
    # ---- prefill: the forward alone at the same shape
    pre = run_prefill(args, ws, d, st, peaks, peak_kind, units_per_launch)

    # ---- end to end through the public API with host buffers
    e2e = None
    if args.skip_e2e:
        del d
        torch.cuda.empty_cache()
    else:
        e2e = run_e2e(args, ws, d, st)
        torch.cuda.empty_cache()

    # ---- decode step at 1280 sequences x 24 layers
    dec = None if args.skip_decode else run_decode(args, ws, peaks, peak_kind)
    # ---- long-context prefill: front end, then the chunked forward at T = 65,536
    lp = None
    if not args.skip_decode:
        try:
            lp = run_long_prefill(args, ws, peaks, peak_kind)
        except Exception as e:          # reported, never at the cost of the lines above
            lp = {"error": ("%s: %s" % (type(e).__name__, e))[:300]}
    clk = clocks.stop()
    if clk is not None:
        clk["region"] = "fwd+bwd, decode and long-prefill timed regions"
    run_tail(args, ws, rank, value, ms_step, roof, shares, e2e, launches, clk, dec, lp,
             roof_step=roof_step, prefill=pre)


def run_prefill(args, ws, d, st, peaks, peak_kind, units):
    """Prefill forward alone (gla_chunk_fwd at B8 H16 T2048, S_T written),
    K launches between two events on the launching stream: tokens/s and both
    rooflines on its method bytes (q, k, v, a in, o and S_T out) and its
    algorithmic flops."""
    w = TRAIN

    def fwd():
        gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], o=d["o"], s_final=d["sf"], ws=d["ws_f"])

    for _ in range(max(3, args.warmup)):
        fwd()
    torch.cuda.synchronize()
    barrier(ws)
    n = max(1, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(n):
        fwd()
    e1.record(st)
    e1.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / n, ws)
    nbytes = METHOD_BYTES["chunk_fwd_fused_kernel"] * units + FS * w.B * w.H
    flops = CHUNK_FLOPS["chunk_fwd_fused_kernel"] * units
    gbs, tfs = nbytes / t / 1e9, flops / t / 1e12
    tpk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    return {"value": round(ws * w.B * w.T / t, 1), "unit": "tokens/s", "workload": "prefill_fwd_b8_t2048",
            "us_per_launch": round(t * 1e6, 2), "launches": n,
            "roofline": {"kernel": "chunk_fwd_fused_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "bytes_per_launch": nbytes, "peak_source": "%s copy bandwidth" % peak_kind},
            "tensor": {"achieved": round(tfs, 1), "peak": tpk, "unit": "TFLOP/s", "frac": round(tfs / tpk, 4),
                       "flops_per_launch": flops, "peak_source": "%s bf16 dense, sustained" % peak_kind}}


def run_e2e(args, ws, d, st):
    """Training steps through the public API from pinned host buffers: every
    step copies its inputs (q, k, v, a, dO) in and its gradients (dq, dk, dv,
    da) out.  Steps are pipelined on two device buffer sets: step i+1's
    inputs arrive (copy-in stream) and step i-1's gradients leave (copy-out
    stream) while step i computes, as a training loop with prefetch would."""
    w = TRAIN
    names = ("q", "k", "v", "a", "dO")
    pin = {n: torch.empty_like(d[n], device="cpu").pin_memory() for n in names}
    for n in pin:
        pin[n].copy_(d[n])
    outs = [torch.empty_like(g, device="cpu").pin_memory() for g in d["grads"][:4]]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)
    second = dict(d)
    for n in names:
        second[n] = torch.empty_like(d[n])
    second["o"] = torch.empty_like(d["o"])
    second["sf"] = torch.empty_like(d["sf"])
    second["saved"] = torch.empty_like(d["saved"])
    second["grads"] = tuple(None if g is None else torch.empty_like(g) for g in d["grads"])
    sets = (d, second)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    consumed = [None, None]      # compute finished reading the set's inputs
    sent = [None, None]          # the set's gradients are on the host

    def e2e_step(i):
        k = i % 2
        x = sets[k]
        with torch.cuda.stream(s_in):
            if consumed[k] is not None:
                s_in.wait_event(consumed[k])
            for n in names:
                x[n].copy_(pin[n], non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(s_in)
        st.wait_event(arrived)
        if sent[k] is not None:
            st.wait_event(sent[k])
        train_step(x)
        done = torch.cuda.Event()
        done.record(st)
        consumed[k] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for g, o in zip(x["grads"][:4], outs):
                o.copy_(g, non_blocking=True)
            out_ev = torch.cuda.Event()
            out_ev.record(s_out)
            sent[k] = out_ev
        return out_ev

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, min(args.steps, 20))
    e0.record(st)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    last = None
    for i in range(e_steps):
        last = e2e_step(i)
    st.wait_event(last)
    e1.record(st)
    e1.synchronize()
    e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, ws)
    del second, sets
    return {"value": round(ws * w.B * w.T * e_steps / e_elapsed, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": e_steps, "overlap": "copy-in, compute and copy-out of consecutive steps on three streams"}


def run_tail(args, ws, rank, value, ms_step, roof, shares, e2e, launches, clk, dec, lp=None,
             roof_step=None, prefill=None):
    w = TRAIN
    # ---- oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        units = int(os.environ.get("GLA_ORACLE_UNITS", str(w.B * w.H)))
        total_t, total_tok, reps = 0.0, 0.0, 0
        while total_t < 10.0 and reps < 20:
            dt, toks, cores = oracle_sample_time(units, 11 + reps)
            total_t += dt
            total_tok += toks
            reps += 1
        cpu = {"value": round(total_tok / total_t, 3), "unit": "tokens/s", "cores": cores,
               "kind": "oracle",
               "sample": "fwd+bwd of %d of the %d (batch, head) sequences (T=%d), %d repetitions, "
                         "%.1f s" % (units, w.B * w.H, w.T, reps, total_t)}

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
                "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": w.name, "global_batch": w.B * ws, "seq_len": w.T,
                           "heads": w.H, "dk": w.dk, "dv": w.dv, "parallelism": "dp%d" % ws,
                           "l2": "inputs larger than L2 (no flush)"},
                "roofline": roof, "roofline_step": roof_step, "kernel_shares": shares,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
                "prefill_fwd": prefill, "decode": dec, "long_prefill": lp}
        print(json.dumps(line), flush=True)


def run_decode(args, ws, peaks, peak_kind):
    w = DECODE
    layers = inputs.decode_inputs(w.N, w.H, w.dk, w.dv, seed=w.seed, device="cuda", layers=w.layers)
    outs = [torch.empty((w.N, w.H, w.dv), dtype=torch.float32, device="cuda") for _ in layers]
    st = torch.cuda.current_stream()

    def step():
        for L, o in zip(layers, outs):
            gla.gla_decode_step(L["state"], L["q"], L["k"], L["v"], L["a"], o=o)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    steps = max(1, min(args.steps, 30))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        step()
    e1.record(st)
    e1.synchronize()
    el = max_over_ranks(e0.elapsed_time(e1) / 1e3, ws)
    per_step = el / steps
    bytes_step = w.layers * w.N * w.H * (2 * FS + 2 * 96 * 2 + 192 * 2 + 192 * 4 + 4)
    achieved = bytes_step / per_step / 1e9
    out = {"value": round(ws * w.N / per_step, 1), "unit": "tokens/s",
           "workload": w.name, "ms_per_step": round(per_step * 1e3, 4),
           "roofline": {"kernel": "decode_step_kernel", "bound": "hbm", "achieved": round(achieved, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(achieved / peaks["hbm_gbs"], 4),
                        "frac_of_8tbs": round(achieved / 8000.0, 4),
                        "peak_source": "%s copy bandwidth (this kernel streams faster than that copy, "
                                       "so frac_of_8tbs against the nominal 8 TB/s is given beside it)"
                                       % peak_kind}}
    del layers, outs
    torch.cuda.empty_cache()
    out["front_end_layer"] = run_decode_front(args, ws, peaks, peak_kind)
    return out


def run_decode_front(args, ws, peaks, peak_kind):
    """The front end of the decode step, one layer a launch: LayerNorm + one
    conv token + SiLU for 1,280 sequences at D = 3,072, conv histories in a
    slot pool.  Each layer has its own pool, x, y and weights (63 MB); the
    launches walk four layers in turn, 252 MB together, so no launch finds
    its inputs in the 126 MB L2."""
    w = DECODE
    st = torch.cuda.current_stream()
    D = LONG.D
    nl = 4
    lay = [{"x": inputs.randn((w.N, D), w.seed + 5 + 10 * i, "cuda", dtype=torch.bfloat16),
            "w": inputs.randn((D, 4), w.seed + 6 + 10 * i, "cuda", std=0.5),
            "pool": inputs.randn((w.N, 3, D), w.seed + 7 + 10 * i, "cuda")} for i in range(nl)]
    for L in lay:
        L["y"] = torch.empty_like(L["x"])

    def launch(i):
        L = lay[i % nl]
        gla.conv1d_silu_decode_step(L["x"], L["w"], L["pool"], y=L["y"])

    for i in range(max(3, args.warmup) * nl):
        launch(i)
    torch.cuda.synchronize()
    barrier(ws)
    n = max(1, min(args.steps, 50)) * nl
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(n):
        launch(i)
    e1.record(st)
    e1.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / n, ws)
    fb = w.N * D * (2 + 2 + 12 + 12)              # x in, y out (bf16); history read and written (fp32)
    rec = {"us_per_launch": round(t * 1e6, 2), "layers_rotated": nl,
           "roofline": {"kernel": "conv_decode_kernel", "bound": "hbm",
                        "achieved": round(fb / t / 1e9, 1), "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": round(fb / t / 1e9 / peaks["hbm_gbs"], 4),
                        "bytes_per_launch": fb,
                        "peak_source": "%s copy bandwidth" % peak_kind}}
    del lay
    torch.cuda.empty_cache()
    return rec


def run_long_prefill(args, ws, peaks, peak_kind):
    """Long-context prefill at T = 65,536 (B = 1, H = 16, D = 3,072): the
    LayerNorm + conv + SiLU front end over x, then the chunked forward with
    S_0 on independent q, k, v (their projection is not part of the path).
    Each call is timed on its own, K launches between two events."""
    w = LONG
    if getattr(args, "lp_tokens", None):            # a smaller case of the same leg (profiling)
        w = dataclasses.replace(LONG, T=args.lp_tokens, name="long_prefill_t%d" % args.lp_tokens)
    st = torch.cuda.current_stream()
    f = inputs.front_inputs(w.B, w.T, w.D, w.W, seed=w.seed, device="cuda")
    y = torch.empty_like(f["x"])
    d = inputs.chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, device="cuda", s0_std=w.s0_std)
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    wsf = torch.empty(max(1, gla.gla_chunk_workspace_bytes(w.B, w.T, w.H)), dtype=torch.uint8, device="cuda")

    def front():
        gla.conv1d_silu_causal(f["x"], f["w"], y=y)

    dy = inputs.randn((w.B, w.T, w.D), w.seed + 3, "cuda", dtype=torch.bfloat16)
    wsb = torch.empty(max(16, gla.conv1d_silu_causal_bwd_workspace_bytes(w.B, w.T, w.D, w.W)), dtype=torch.uint8,
                      device="cuda")

    def front_bwd():
        gla.conv1d_silu_causal_bwd(f["x"], f["w"], dy, ws=wsb, want=("dx", "dw"))

    def mixer():
        gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"], o=o, s_final=sf, ws=wsf)

    def timed(fn, n):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(n):
            fn()
        e1.record(st)
        e1.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / 1e3 / n, ws)

    n = max(1, min(args.steps, 20))
    t_front, t_mix = timed(front, n), timed(mixer, n)
    t_fbwd = timed(front_bwd, max(1, min(n, 10)))
    front_bytes = w.B * w.T * w.D * 4                       # x in, y out (bf16)
    front_bwd_bytes = w.B * w.T * w.D * 6                   # x, dy in, dx out (bf16)
    units = w.B * w.H * ((w.T + 127) // 128)
    mix_bytes = METHOD_BYTES["chunk_fwd_fused_kernel"] * units + 2 * FS * w.B * w.H   # + S_0 in, S_T out

    def roof(kernel, nbytes, t):
        a = nbytes / t / 1e9
        return {"kernel": kernel, "bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(a / peaks["hbm_gbs"], 4), "bytes_per_launch": nbytes,
                "peak_source": "%s copy bandwidth" % peak_kind}

    out = {"value": round(ws * w.B * w.T / (t_front + t_mix), 1), "unit": "tokens/s", "workload": w.name,
           "ms_per_step": round((t_front + t_mix) * 1e3, 4),
           "front_end": {"us_per_launch": round(t_front * 1e6, 2),
                         "roofline": roof("ln_conv_silu_kernel", front_bytes, t_front)},
           "front_end_bwd": {"us_per_launch": round(t_fbwd * 1e6, 2),
                             "roofline": roof("conv1d_silu_causal_bwd (one row pass by clusters of 2 CTAs, reduction)",
                                              front_bwd_bytes, t_fbwd)},
           "gla_fwd": {"us_per_launch": round(t_mix * 1e6, 2),
                       "roofline": roof("gla_chunk_fwd (segmented: state pre-pass, combine, fused pass)",
                                        mix_bytes, t_mix)}}
    del f, y, d, o, sf, wsf, dy, wsb
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-decode", action="store_true", help="time the training step only (profiling)")
    ap.add_argument("--skip-e2e", action="store_true", help="no host-buffer end-to-end leg (profiling)")
    ap.add_argument("--only", choices=["decode", "decode_front", "long_prefill"],
                    help="run that leg alone and print its record (profiling; no headline line)")
    ap.add_argument("--lp-tokens", type=int, default=None,
                    help="sequence length of the long-prefill leg (default 65,536; profiling)")
    args = ap.parse_args()
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, ws, rank)
        return
    ws, rank, local = dist_setup()
    try:
        run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
