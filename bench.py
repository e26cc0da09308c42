#!/usr/bin/env python
"""Benchmark of the MSA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole prefill hot path over one 128K-token layer:
index branch (scores, block max-pool, top-k with the forced local block) and
main branch (selection inversion, KV-outer sparse attention, combine).  The
timed region holds K steps between a barrier and a device synchronize; the
value is the whole-job throughput (query tokens/s, summed over ranks, each rank
running its own independent layer: weak scaling, no data-path collective).

Also reported on the same JSON line:
  roofline     the dominant kernel's achieved TFLOP/s (or GB/s) against the
               measured peak, from CUDA events the library records on its launch
               stream around every launch during the timed region;
  step_roofline  the whole step against max(FLOPs / tensor peak, bytes / HBM peak);
  decode       decode step time (32 sequences, cache 128K..1M) and its HBM roofline;
  e2e          the same prefill step through the public API with host (pinned)
               buffers: host->device inputs and device->host output inside the
               timed region;
  cpu_baseline the fp64 oracle timed on this host's cores on a bounded sample;
  clocks       nvidia-smi SM clocks and throttle reasons sampled while timing.

--impl reference times the oracle alone (the reference arm of this comparison).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA prefill tokens/s @128K; decode µs/step; % of roofline on 1 B200"
PREFILL = "prefill_n131072_hot2"
DECODE = "decode_b32_l128k_1m_hot2"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


HBM_SPEC_GBS = 7700.0            # B200 HBM3e, nominal (HGX figure)


def tensor_peak(peaks, src, clk):
    """The bf16 tensor peak the sampled clocks support: the burst figure
    (measured at the maximum SM clock) when the median SM clock under load was
    within 5% of the maximum, else the sustained one (measured under the power
    cap).  Returns (peak, source text)."""
    med, mx = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    at_max = bool(med and mx and med >= 0.95 * mx)
    if at_max:
        return peaks["bf16_tflops"], (f"bf16_tflops, burst ({src}): median SM clock {med:.0f} of {mx:.0f} MHz "
                                      f"under load")
    how = f"median SM clock {med:.0f} of {mx:.0f} MHz" if med and mx else "clocks not sampled"
    return peaks["bf16_tflops_sustained"], f"bf16_tflops_sustained ({src}): {how}"


# ------------------------------------------------------------------ clocks ---

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"msa_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        loaded = [s for s, m in zip(sm, mx) if s > 0.5 * m] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- helpers ---

L2_BYTES = 126 * 1024 * 1024     # B200 L2


def pass_rows(q_chunk, T):
    """Query rows per attention pass: q_chunk < 0 picks passes of 131072 rows
    above 128K tokens (the partials of a pass must fit the device), 0 = one pass."""
    if q_chunk < 0:
        return 131072 if T > 131072 else 0
    return q_chunk


def run_config(args, w, T, world):
    """The workload description, printed the same by both arms (T: the
    layer's query tokens)."""
    par = (f"query ranges of one layer x{world}" if getattr(args, "shard", "none") == "queries"
           else f"independent layer per GPU x{world}")
    return {"workload": args.workload, "T": T, "H": w.H, "G": w.G, "d": w.d, "d_idx": w.d_idx,
            "B_k": w.B_k, "k": w.k, "hot_block_frac": w.hot_frac,
            "l2": ("inputs larger than L2 (q alone is %.1f GB)" % (T * w.H * w.d * 2 / 1e9)
                   if T * w.H * w.d * 2 > L2_BYTES else
                   "inputs fit in L2 (q is %.0f MB, L2 not flushed): a profiling size, not a timing one"
                   % (T * w.H * w.d * 2 / 1e6)),
            "parallelism": par,
            "attention_pass_rows": pass_rows(args.q_chunk, T) or T}


def make_ctx(w, inp, torch, msa):
    shape = msa.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
    seqs = msa.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    T = inp["cu_q_host"][-1]
    dev = inp["q"].device
    ctx = dict(shape=shape, seqs=seqs, inp=inp, T=T)
    ctx["sel"] = torch.empty((T, w.G, w.k), dtype=torch.int32, device=dev)
    ctx["out"] = torch.empty((T, w.H, w.d), dtype=torch.bfloat16, device=dev)
    lib = msa.load_library()
    import ctypes
    n_idx = lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))
    # passes of at most q_chunk query rows (the partials of a pass must fit the device)
    ctx["q_chunk"] = pass_rows(getattr(make_ctx, "q_chunk", 0), T)
    n_att = (msa.msa_sparse_attn_workspace_size(shape, seqs, ctx["q_chunk"])
             if not getattr(make_ctx, "index_only", False) else 256)
    ctx["ws_idx"] = torch.empty(n_idx, dtype=torch.uint8, device=dev)
    ctx["ws_att"] = torch.zeros(n_att, dtype=torch.uint8, device=dev) if n_att <= 256 else \
        torch.empty(n_att, dtype=torch.uint8, device=dev)
    return ctx


def step_prefill(ctx, msa, inp=None, index_only=False):
    inp = inp or ctx["inp"]
    msa.msa_index_topk(ctx["shape"], ctx["seqs"], inp["q_idx"], inp["k_idx"], sel=ctx["sel"], ws=ctx["ws_idx"],
                       check=False)
    if index_only:
        return
    msa.msa_sparse_attn_prefill(ctx["shape"], ctx["seqs"], inp["q"], inp["k"], inp["v"], ctx["sel"],
                                q_chunk=ctx.get("q_chunk", 0),
                                out=ctx["out"], want_lse=False, ws=ctx["ws_att"], check=False)


def step_decode(ctx, msa):
    inp = ctx["inp"]
    msa.msa_index_topk(ctx["shape"], ctx["seqs"], inp["q_idx"], inp["k_idx"], sel=ctx["sel"], ws=ctx["ws_idx"],
                       check=False)
    msa.msa_sparse_attn_decode(ctx["shape"], ctx["seqs"], inp["q"], inp["k"], inp["v"], ctx["sel"],
                               out=ctx["out"], want_lse=False, ws=ctx["ws_att"], check=False)


def training_leg(args, w, W, R, msa, torch, device="cuda"):
    """The training-side kernels on one prefill layer of args.training_T tokens
    with the workload's heads and dimensions: the Main Branch backward for a
    seeded upstream gradient, then the KL target (tau = 0.125) and its
    gradient, fed by the forward's selection and log-sum-exps.  Each kernel is
    timed by the library's CUDA events on its launching stream over
    args.training_steps passes after args.training_warmup (inputs larger than
    L2; its own small counts).  The backward runs its products on the tensor
    cores and is held to the measured bf16 peak; the KL target
    computes its scores on the tensor cores and is held to the exponential rate
    of the special-function units; the KL gradient computes the same scores on
    the tensor cores and its dq_idx / dk_idx products on the CUDA cores, which
    are held to the fp32 FMA rate."""
    tinp = W.make_inputs(w, device, T_override=args.training_T)
    shape = msa.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
    seqs = msa.make_varlen(tinp["cu_q"], tinp["cu_k"], tinp["cu_q_host"], tinp["cu_k_host"])
    q, k, v, q_idx, k_idx = (tinp[n] for n in ("q", "k", "v", "q_idx", "k_idx"))
    sel = msa.msa_index_topk(shape, seqs, q_idx, k_idx)
    out, lse = msa.msa_sparse_attn_prefill(shape, seqs, q, k, v, sel)
    gen = torch.Generator(device=q.device).manual_seed(w.seed + 1000)
    dout = torch.randn(tuple(q.shape), generator=gen, device=q.device).to(torch.bfloat16)
    tau = 0.125

    def one(check):
        msa.msa_sparse_attn_backward(shape, seqs, q, k, v, sel, out, lse, dout, check=check)
        _, lse_z = msa.msa_index_kl(shape, seqs, q, k, q_idx, k_idx, sel, lse, tau, want_lse_z=True, check=check)
        msa.msa_index_kl_backward(shape, seqs, q, k, q_idx, k_idx, sel, lse, lse_z, tau, check=check)

    one(True)
    for _ in range(args.training_warmup):
        one(False)
    torch.cuda.synchronize()
    msa.msa_profile_reset()
    msa.msa_profile_enable(True)
    for _ in range(args.training_steps):
        one(False)
    torch.cuda.synchronize()
    msa.msa_profile_enable(False)
    one(True)                                 # device checks after the timed passes
    S_lens = [tinp["cu_k_host"][i + 1] - tinp["cu_k_host"][i] for i in range(len(tinp["cu_k_host"]) - 1)]
    T_lens = [tinp["cu_q_host"][i + 1] - tinp["cu_q_host"][i] for i in range(len(tinp["cu_q_host"]) - 1)]
    tw = R.training_work(S_lens, T_lens, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
    peak = R.alu_fp32_tflops()
    res = {"workload": f"{args.workload} at T = {sum(T_lens)}", "T": sum(T_lens), "tau": tau,
           "steps": args.training_steps, "warmup": args.training_warmup, "peak": peak, "unit": "TFLOP/s",
           "peak_source": "148 SMs x 128 fp32 lanes x 2 FLOPs x 1965 MHz (CUDA cores, nominal)",
           "kernels": {}}
    for name, key in (("attn_bwd", "backward_flops"), ("index_kl", "kl_flops"), ("index_kl_grad", "kl_grad_flops")):
        kms, n = msa.msa_profile_read(name)
        if n:
            per = kms / n
            ach = tw[key] / (per / 1000.0) / 1e12
            res["kernels"][name] = {"ms_per_launch": per, "launches": n, "flops_per_launch": tw[key],
                                    "bound": "alu", "achieved": ach, "frac": ach / peak}
    kr = res["kernels"].get("attn_bwd")
    if kr is not None:
        # the selected support's backward runs its five products on the tensor cores
        peaks, src = load_peaks()
        ach = tw["backward_flops"] / (kr["ms_per_launch"] / 1000.0) / 1e12
        kr.update({"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "frac": ach / peaks["bf16_tflops"],
                   "peak_source": f"bf16_tflops ({src}, burst)"})
    kr = res["kernels"].get("index_kl_grad")
    if kr is not None:
        # the gradient's scores run on the tensor cores; its dq_idx / dk_idx
        # products stay on the CUDA cores and are held to the fp32 FMA rate
        sec = kr["ms_per_launch"] / 1000.0
        peaks, src = load_peaks()
        ach_a = tw["kl_grad_alu_flops"] / sec / 1e12
        ach_t = tw["kl_tensor_flops"] / sec / 1e12
        kr.update({"flops_per_launch": tw["kl_grad_alu_flops"], "achieved": ach_a, "frac": ach_a / peak,
                   "tensor": {"flops_per_launch": tw["kl_tensor_flops"], "achieved": ach_t,
                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": ach_t / peaks["bf16_tflops"], "peak_source": f"bf16_tflops ({src})"}})
    kr = res["kernels"].get("index_kl")
    if kr is not None:
        # the KL target's scores run on the tensor cores; what stays on the
        # CUDA cores is dominated by one exponential per head and pair, so the
        # kernel is held to the exponential rate, the tensor-core figure beside it
        sec = kr["ms_per_launch"] / 1000.0
        peaks, src = load_peaks()
        mufu = R.mufu_gexps()
        ach_e = tw["kl_exps"] / sec / 1e9
        ach_t = tw["kl_tensor_flops"] / sec / 1e12
        kr.update({"bound": "mufu", "unit": "Gexp/s", "exps_per_launch": tw["kl_exps"], "achieved": ach_e,
                   "peak": mufu, "frac": ach_e / mufu,
                   "peak_source": "148 SMs x 16 ex2 per clock x 1965 MHz (special-function units)",
                   "tensor": {"flops_per_launch": tw["kl_tensor_flops"], "achieved": ach_t,
                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": ach_t / peaks["bf16_tflops"], "peak_source": f"bf16_tflops ({src})"}})
    return res


def decode_result(name, d_ms, L, dw, dk, scan_ms, peaks, peak_src):
    """Decode step against its HBM roofline.  Two denominators, each labelled:
    the measured copy bandwidth (hbm_gbs: a read + write stream) and the
    nominal HBM3e bandwidth.  A read-only stream (the index-key scan) can run
    above the copy figure, which pays for read-write turnarounds; part of the
    index keys can also stay in L2 between timed steps."""
    achieved_scan = None if scan_ms is None else dw["index_bytes"] / (scan_ms / 1000.0) / 1e9
    return {"workload": name, "us_per_step": d_ms * 1000.0, "sum_L": sum(L),
            "algorithmic_bytes": dw["bytes"],
            "roofline_us": dw["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6,
            "frac": dw["bytes"] / (peaks["hbm_gbs"] * 1e9) / (d_ms / 1000.0),
            "frac_of_spec_hbm": dw["bytes"] / (HBM_SPEC_GBS * 1e9) / (d_ms / 1000.0),
            "peak_source": f"hbm_gbs {peaks['hbm_gbs']:.0f} GB/s ({peak_src} copy); spec {HBM_SPEC_GBS:.0f} GB/s",
            "scan_kernel": None if scan_ms is None else {
                "bound": "hbm", "achieved": achieved_scan, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_scan / peaks["hbm_gbs"], "frac_of_spec_hbm": achieved_scan / HBM_SPEC_GBS},
            "kernels": dk}


def decode_leg(args, W, R, msa, torch, peaks, peak_src):
    """Decode step of args.decode_workload (one query per sequence against its
    cache), timed by CUDA events over max(5, steps) steps after 3 warm-up ones,
    with the library's per-kernel events."""
    wd = W.WORKLOADS[args.decode_workload]
    dinp = W.make_inputs(wd, "cuda")
    dctx = make_ctx(wd, dinp, torch, msa)
    for _ in range(3):
        step_decode(dctx, msa)
    torch.cuda.synchronize()
    device_errors(dctx, msa)
    msa.msa_profile_reset()
    msa.msa_profile_enable(True)
    d_steps = max(5, args.steps)
    d_ms = time_steps(lambda: step_decode(dctx, msa), d_steps, torch) / d_steps
    msa.msa_profile_enable(False)
    device_errors(dctx, msa)
    L = [dinp["cu_k_host"][i + 1] - dinp["cu_k_host"][i] for i in range(wd.batch)]
    dw = R.decode_work(L, wd.H, wd.G, wd.d, wd.d_idx, wd.B_k, wd.k)
    dk = {}
    for name in ("decode_scan", "decode_select", "rows_attn", "sparse_attn", "combine", "count", "scatter", "plan"):
        kms, n = msa.msa_profile_read(name)
        if n:
            dk[name] = {"ms_per_launch": kms / n, "launches": n}
    scan_ms = dk.get("decode_scan", {}).get("ms_per_launch")
    res = decode_result(args.decode_workload, d_ms, L, dw, dk, scan_ms, peaks, peak_src)
    del dctx, dinp
    torch.cuda.empty_cache()
    return res


def config_leg(args, name, W, R, msa, torch, peaks, peak_t, peak_t_src):
    """One more prefill configuration (the 32K layer, the 1M layer in passes of
    131072 query rows): ms per step, query tokens/s and the step against its
    roofline, timed by CUDA events after 3 warm-up steps (inputs larger than
    L2).  Not the headline line."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, "cuda")
    make_ctx.q_chunk = -1
    ctx = make_ctx(w, inp, torch, msa)
    for _ in range(3):
        step_prefill(ctx, msa)
    torch.cuda.synchronize()
    device_errors(ctx, msa)
    steps = 3 if ctx["T"] > 131072 else max(5, args.steps)
    msa.msa_profile_reset()
    msa.msa_profile_enable(True)
    ms = time_steps(lambda: step_prefill(ctx, msa), steps, torch) / steps
    msa.msa_profile_enable(False)
    device_errors(ctx, msa)
    S_lens = [inp["cu_k_host"][i + 1] - inp["cu_k_host"][i] for i in range(len(inp["cu_k_host"]) - 1)]
    T_lens = [inp["cu_q_host"][i + 1] - inp["cu_q_host"][i] for i in range(len(inp["cu_q_host"]) - 1)]
    work = R.prefill_work(S_lens, T_lens, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
    t_b = max(work["flops"] / (peaks["bf16_tflops"] * 1e12), work["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    t_s = max(work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12), work["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    ks = {}
    for kn in ("index_topk_prefill", "tile_plan", "tile_attn", "sparse_attn", "combine"):
        kms, n = msa.msa_profile_read(kn)
        if n:
            ks[kn] = {"ms_per_step": kms / steps, "launches_per_step": n / steps}
    res = {"workload": name, "T": ctx["T"], "steps": steps, "warmup": 3, "ms_per_step": ms,
           "value": ctx["T"] / (ms / 1000.0), "unit": "tokens/s",
           "attention_pass_rows": ctx["q_chunk"] or ctx["T"],
           "roofline_ms_burst": t_b, "roofline_ms_sustained": t_s,
           "frac_burst": t_b / ms, "frac_sustained": t_s / ms, "kernels": ks}
    del ctx, inp
    return res


def device_errors(ctx, msa):
    for key in ("ws_idx", "ws_att"):
        code, where, i0, i1 = msa.msa_get_device_error(ctx[key])
        if code != 0:
            raise RuntimeError(f"device error {code} at site {where} ({i0}, {i1}) in {key}")


def time_steps(fn, steps, torch, dist=None):
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return s.elapsed_time(e)


def _reduce_device(dist):
    """NCCL reduces device tensors; gloo (the CPU tests) host tensors."""
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x, torch, dist):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device(dist))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, torch, dist):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device(dist))
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_rate(tokens_local, ms_local, torch, dist):
    """Whole-job tokens/s: tokens of all ranks over the slowest rank's time."""
    ms_max = max_over_ranks(ms_local, torch, dist)
    return sum_over_ranks(float(tokens_local), torch, dist) / (ms_max / 1000.0), ms_max


def rank_workload(w, rank, W):
    """Each rank runs an independent layer of the same shape (its own seed)."""
    return W.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def traffic_for(kernel):
    """DRAM bytes per full-size launch from a committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d:
        return None
    sha = kernel_source_sha(d.get("source", ""))
    return d.get("dram_bytes_per_launch") if sha is not None and sha == d.get("source_sha") else None


def code_tokens(text):
    """C/C++/CUDA source with its comments removed (string and character
    literals kept as they are), whitespace runs collapsed and blank lines
    dropped: two sources with equal results differ only in comments or layout."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                                   # literal: copy through its closing quote
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (" ".join(line.split()) for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_source_sha(source):
    """Hash of the code (comments and layout ignored) of a kernel's .cu file
    together with the headers every kernel includes: a change to the code of
    either makes recorded counters stale."""
    csrc = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")
    h = hashlib.sha256()
    for f in (source, "msa_common.cuh", "msa_internal.h"):
        p = os.path.join(csrc, f)
        if not f or not os.path.exists(p):
            return None
        h.update(code_tokens(open(p, encoding="utf-8").read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


# ------------------------------------------------------------- CPU oracle ---

def cpu_oracle_rate(w, inp, budget_s, torch, np, seed=0):
    """Oracle throughput (query rows per second) on a seeded random sample of
    rows, grown in batches until ~budget_s of CPU work."""
    from oracle import msa_oracle as O
    T = inp["cu_q_host"][-1]
    g = torch.Generator().manual_seed(1234 + seed)
    order = torch.randperm(T, generator=g).tolist()
    full = {"q_idx": inp["q_idx"].float().cpu().numpy(), "k_idx": inp["k_idx"].float().cpu().numpy(),
            "k": inp["k"].float().cpu().numpy(), "v": inp["v"].float().cpu().numpy()}
    n_done, t_used, batch = 0, 0.0, 16
    while t_used < budget_s and n_done < T:
        rows = sorted(order[n_done:n_done + batch])
        idx = torch.tensor(rows, dtype=torch.long, device=inp["q"].device)
        host = dict(full, q=inp["q"].index_select(0, idx).float().cpu().numpy())
        t0 = time.perf_counter()
        _oracle_batch(w, host, rows, O, np)
        t_used += time.perf_counter() - t0
        n_done += len(rows)
        batch = min(256, batch * 2)
    return n_done / t_used, n_done, t_used


def _oracle_batch(w, host, rows, O, np):
    pos = np.asarray(rows)
    sel = O.index_topk_rows(host["q_idx"][rows], host["k_idx"], pos, w.k, w.B_k)
    Hg = w.H // w.G
    for r, t in enumerate(rows):
        for g in range(w.G):
            J = O.selected_token_set([int(x) for x in sel[r, g]], int(t), w.B_k)
            O.attend(host["q"][r, g * Hg:(g + 1) * Hg], host["k"][J, g], host["v"][J, g], w.sm_scale)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return None


# ------------------------------------------------------------------- arms ---

def run_reference(args):
    """The oracle as it stands, timed on this host's cores (rank 0 only)."""
    import numpy as np
    import torch
    from block_sparse_long_exp_b200 import workloads as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_inputs(w, dev, T_override=args.T or None)
    T = inp["cu_q_host"][-1]
    from oracle import msa_oracle as O
    gen = torch.Generator().manual_seed(99)
    order = torch.randperm(T, generator=gen).tolist()
    per_step = args.ref_rows
    host_full = {"q_idx": inp["q_idx"].float().cpu().numpy(), "k_idx": inp["k_idx"].float().cpu().numpy(),
                 "k": inp["k"].float().cpu().numpy(), "v": inp["v"].float().cpu().numpy()}
    times = []
    for s in range(args.warmup + args.steps):
        rows = sorted(order[(s * per_step) % T:(s * per_step) % T + per_step])
        idx = torch.tensor(rows, dtype=torch.long, device=inp["q"].device)
        host = dict(host_full, q=inp["q"].index_select(0, idx).float().cpu().numpy())
        t0 = time.perf_counter()
        _oracle_batch(w, host, rows, O, np)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    sec = sum(times)
    rate = per_step * len(times) / sec
    cores = len(os.sched_getaffinity(0))
    sample = f"{per_step} random query rows of {args.workload} per step (of {T}); oracle selection + main branch"
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sec / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": run_config(args, w, T, args.gpus),
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "blas_threads": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import numpy as np
    import torch
    from block_sparse_long_exp_b200 import build as B
    from block_sparse_long_exp_b200 import msa
    from block_sparse_long_exp_b200 import roofline as R
    from block_sparse_long_exp_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    B.build()
    msa.load_library()
    msa.msa_set_tile_threshold(args.theta)
    if args.window:
        msa.msa_set_attn_window(args.window)
    peaks, peak_src = load_peaks()
    if args.decode_only:
        if rank == 0:
            print(json.dumps({"metric": "decode µs/step (decode leg alone: a profiling run, not the headline)",
                              "decode": decode_leg(args, W, R, msa, torch, peaks, peak_src)}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    if args.training_only:
        if rank == 0:
            print(json.dumps({"metric": "training kernel ms (training leg alone: a profiling run, not the headline)",
                              "training": training_leg(args, W.WORKLOADS[args.workload], W, R, msa, torch)}),
                  flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    def tile_theta(w_):
        if args.theta >= 0:
            return args.theta
        uq = 2 * (128 // max(w_.H // w_.G, 8))
        return (5 * uq + 7) // 8
    w = W.WORKLOADS[args.workload]
    shard_q = args.shard == "queries"
    # weak scaling: each rank runs an independent layer (its own seed); with
    # --shard queries every rank holds the same layer and computes one range
    # of its queries as a chunked prefill (strong scaling, no collective)
    wr = w if shard_q else rank_workload(w, rank, W)
    inp = W.make_inputs(wr, "cuda", T_override=args.T or None)
    T_layer = inp["cu_q_host"][-1]
    if shard_q:
        from block_sparse_long_exp_b200 import shard as SH
        if len(inp["cu_q_host"]) != 2 or w.kind != "prefill":
            raise SystemExit("--shard queries takes a single-sequence prefill workload")
        work_q = SH.query_work(T_layer, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
        a_, b_ = SH.split_query_ranges(work_q, world, align=w.B_k)[rank]
        inp = SH.chunk_of(inp, a_, b_)
    torch.cuda.synchronize()
    make_ctx.index_only = args.index_only
    make_ctx.q_chunk = args.q_chunk
    ctx = make_ctx(wr, inp, torch, msa)
    make_ctx.index_only = False
    make_ctx.q_chunk = -1
    S_lens = [inp["cu_k_host"][i + 1] - inp["cu_k_host"][i] for i in range(len(inp["cu_k_host"]) - 1)]
    T_lens = [inp["cu_q_host"][i + 1] - inp["cu_q_host"][i] for i in range(len(inp["cu_q_host"]) - 1)]
    T = ctx["T"]
    work = R.prefill_work(S_lens, T_lens, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)

    for _ in range(args.warmup):
        step_prefill(ctx, msa, index_only=args.index_only)
    torch.cuda.synchronize()
    device_errors(ctx, msa)

    gpu_uuid = str(torch.cuda.get_device_properties(local).uuid)
    gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    clocks = ClockSampler(gpu_uuid)
    clocks.start()
    msa.msa_profile_reset()
    msa.msa_profile_enable(True)
    ms = time_steps(lambda: step_prefill(ctx, msa, index_only=args.index_only), args.steps, torch, dist)
    msa.msa_profile_enable(False)
    clk = clocks.stop()
    device_errors(ctx, msa)
    launches = msa.msa_profile_read(None)[1]
    kernels = {}
    for name in ("index_topk_prefill", "tile_plan", "tile_attn", "sparse_attn", "combine", "count", "scatter",
                 "plan", "block_offsets"):
        kms, n = msa.msa_profile_read(name)
        if n:
            kernels[name] = {"ms_per_launch": kms / n, "launches": n, "share": None}
    tot = sum(v["ms_per_launch"] * v["launches"] for v in kernels.values()) or 1.0
    for v in kernels.values():
        v["share"] = v["ms_per_launch"] * v["launches"] / tot

    value, ms_max = job_rate(T * args.steps, ms, torch, dist)
    ms_step = ms_max / args.steps

    # algorithmic work of each kernel: the main branch split between the query
    # tiles and the KV-outer lists as the library's planner splits it
    split = None if args.index_only else R.tile_split(
        ctx["sel"], inp["cu_q_host"], inp["cu_k_host"], w.H, w.G, w.d, w.B_k, tile_theta(w), 0)
    per_kernel_work = {"index_topk_prefill": ("tensor", work["index_flops"])}
    if split is not None:
        per_kernel_work.update({"tile_attn": ("tensor", split["tile_flops"]),
                                "sparse_attn": ("tensor", split["kv_flops"]),
                                "combine": ("hbm", split["combine_bytes"])})
    peak_t, peak_t_src = tensor_peak(peaks, peak_src, clk)
    for name, v in kernels.items():
        if name in per_kernel_work:
            bound, units = per_kernel_work[name]
            per = units / (v["launches"] / args.steps)
            v["algorithmic_per_launch"] = per
            v["achieved"] = per / (v["ms_per_launch"] / 1000.0) / (1e12 if bound == "tensor" else 1e9)
            if bound == "tensor":
                v["frac"] = v["achieved"] / peak_t
                v["frac_burst"] = v["achieved"] / peaks["bf16_tflops"]
                v["frac_sustained"] = v["achieved"] / peaks["bf16_tflops_sustained"]
            else:
                v["frac"] = v["achieved"] / peaks["hbm_gbs"]
    # roofline of the dominant kernel, against the peak the sampled clocks support
    dom = max((n for n in kernels if n in per_kernel_work),
              key=lambda n: kernels[n]["ms_per_launch"] * kernels[n]["launches"])
    bound = per_kernel_work[dom][0]
    roof = {"kernel": dom, "bound": bound, "achieved": kernels[dom]["achieved"],
            "peak": peak_t if bound == "tensor" else peaks["hbm_gbs"],
            "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": kernels[dom]["frac"],
            "traffic": traffic_for(dom), "algorithmic_per_launch": kernels[dom]["algorithmic_per_launch"],
            "peak_source": peak_t_src if bound == "tensor" else f"hbm_gbs ({peak_src})"}
    if bound == "tensor":
        roof["frac_burst"] = kernels[dom]["frac_burst"]
        roof["frac_sustained"] = kernels[dom]["frac_sustained"]
    t_roof_ms = max(work["flops"] / (peaks["bf16_tflops"] * 1e12), work["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    t_roof_sus = max(work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12),
                     work["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    step_roof = {"flops": work["flops"], "index_flops": work["index_flops"], "main_flops": work["main_flops"],
                 "bytes": work["bytes"], "roofline_ms_burst": t_roof_ms, "roofline_ms_sustained": t_roof_sus,
                 "frac_burst": t_roof_ms / ms_step, "frac_sustained": t_roof_sus / ms_step,
                 "bound": "tensor" if work["flops"] / (peaks["bf16_tflops"] * 1e12) >
                 work["bytes"] / (peaks["hbm_gbs"] * 1e9) else "hbm"}

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        keys = ("q", "k", "v", "q_idx", "k_idx")
        host = {k_: inp[k_].cpu().pin_memory() for k_ in keys}
        dev = {k_: torch.empty_like(inp[k_]) for k_ in keys}
        host_out = torch.empty(ctx["out"].shape, dtype=ctx["out"].dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = host_out.numel() * host_out.element_size()

        def e2e_step():
            for k_ in keys:
                dev[k_].copy_(host[k_], non_blocking=True)
            step_prefill(ctx, msa, inp={**inp, **dev})
            host_out.copy_(ctx["out"], non_blocking=True)

        e2e_step()
        e_steps = max(2, args.steps // 3)
        ms_e = max_over_ranks(time_steps(e2e_step, e_steps, torch, dist), torch, dist)
        e2e = {"value": sum_over_ranks(float(T * e_steps), torch, dist) / (ms_e / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e / e_steps}
        del host, dev, host_out

    # dense causal GQA on the same q / k / v: the denominator of the speedup ratio
    dense = None
    if rank == 0 and not args.no_dense and not args.index_only:
        dws = torch.empty(msa.load_library().msa_dense_attn_workspace_size(
            __import__("ctypes").byref(ctx["shape"]), __import__("ctypes").byref(ctx["seqs"])),
            dtype=torch.uint8, device=inp["q"].device)

        def dense_step():
            msa.msa_dense_attn(ctx["shape"], ctx["seqs"], inp["q"], inp["k"], inp["v"], out=ctx["out"], ws=dws,
                               check=False)

        dense_step()
        torch.cuda.synchronize()
        code = msa.msa_get_device_error(dws)[0]
        if code != 0:
            raise RuntimeError(f"dense attention device error {code}")
        d_steps = 2
        dms = time_steps(dense_step, d_steps, torch) / d_steps
        dfl = R.dense_work(S_lens, T_lens, w.H, w.d)
        main_ms = sum(kernels[n]["ms_per_launch"] * kernels[n]["launches"] for n in kernels
                      if n != "index_topk_prefill") / args.steps
        dense = {"workload": args.workload, "ms": dms, "flops": dfl,
                 "achieved_tflops": dfl / (dms / 1000.0) / 1e12,
                 "frac": dfl / (dms / 1000.0) / 1e12 / peak_t,
                 "frac_burst": dfl / (dms / 1000.0) / 1e12 / peaks["bf16_tflops"],
                 "frac_sustained": dfl / (dms / 1000.0) / 1e12 / peaks["bf16_tflops_sustained"],
                 "speedup_step": dms / ms_step, "speedup_main_branch": dms / main_ms,
                 "flops_ratio": dfl / work["main_flops"]}
        del dws

    # dense GQA done: the prefill context's workspace is no longer needed
    ctx = None
    torch.cuda.empty_cache()
    # decode: 32 sequences with caches of 128K..1M tokens
    decode = None
    cpu = None
    if rank == 0 and not args.no_decode:
        decode = decode_leg(args, W, R, msa, torch, peaks, peak_src)
    # the other prefill configurations, one line each (not the headline)
    configs = None
    if rank == 0 and world == 1 and args.configs:
        configs = {}
        for name in [c for c in args.configs.split(",") if c]:
            configs[name] = config_leg(args, name, W, R, msa, torch, peaks, peak_t, peak_t_src)
            torch.cuda.empty_cache()
    training = None
    if rank == 0 and args.training:
        training = training_leg(args, w, W, R, msa, torch)
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n_rows, secs = cpu_oracle_rate(w, inp, args.cpu_budget, torch, np)
        cores = len(os.sched_getaffinity(0))
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "blas_threads": blas_threads(), "kind": "oracle",
               "sample": f"{n_rows} random query rows of {args.workload} ({secs:.1f} s of fp64 oracle work: "
                         f"selection + main branch per row)"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "strong" if shard_q else "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": run_config(args, w, T_layer, world),
                "roofline": roof, "step_roofline": step_roof, "tile_split": split, "dense_gqa": dense,
                "decode": decode, "configs": configs, "e2e": e2e,
                "cpu_baseline": cpu, "clocks": clk, "gpu_launches": launches, "kernels": kernels}
        if training is not None:
            line["training"] = training
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def build_parser():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL)
    ap.add_argument("--T", type=int, default=0, help="shorter prefill (same heads/dims), for profiling")
    ap.add_argument("--index-only", action="store_true", help="time only the index branch (for profiling)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-workload", default=DECODE, help="decode workload of the decode leg")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode leg and print its line (for profiler captures)")
    ap.add_argument("--configs", default="prefill_n32768,prefill_n1048576_hot2",
                    help="other prefill workloads timed after the headline (comma list; empty: none)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense causal GQA comparison")
    ap.add_argument("--q-chunk", type=int, default=-1,
                    help="query rows per attention pass (-1: 131072 above 128K tokens, else one pass)")
    ap.add_argument("--theta", type=int, default=-1,
                    help="query-tile threshold of the prefill (-1 automatic, 0 off)")
    ap.add_argument("--window", type=int, default=0,
                    help="query rows per planning window of the KV-outer lists (0: the library's default)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--no-training", dest="training", action="store_false",
                    help="skip the training leg (the backward and KL kernels, CUDA cores, on a --training-T layer)")
    ap.add_argument("--training", dest="training", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--training-only", action="store_true",
                    help="run only the training leg (a profiling run; prints no headline line)")
    ap.add_argument("--training-T", type=int, default=32768)
    ap.add_argument("--training-steps", type=int, default=2)
    ap.add_argument("--training-warmup", type=int, default=1)
    ap.set_defaults(training=True)
    ap.add_argument("--shard", choices=["none", "queries"], default="none",
                    help="N > 1: independent layers per rank (none, weak scaling) or the query ranges of one "
                         "layer split across ranks (queries, strong scaling)")
    return ap


def main():
    args = build_parser().parse_args()
    if args.warmup < 3:
        log("note: fewer than 3 warm-up steps")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
