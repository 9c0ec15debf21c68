"""Benchmark: exact attention forward + backward on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one pass of the whole hot path over one batch of synthetic input:
fa_fwd, then the three backward stages (fa_bwd_prep, fa_bwd_dkdv, fa_bwd_dq,
i.e. fa_bwd).  Default workload: the causal training step, B=4, Hq=Hkv=16,
N=4096, d=128, bf16 (the configuration the metric is quoted on).  FLOPs per
step: forward 4*B*Hq*Nq*Nk*d, backward 2.5x that, both halved for causal.

Multi-GPU (torchrun, one process per GPU): attention shards by (batch,
key/value head) with no exchange between shards, so every rank runs an
identical replica of the workload on its own GPU (weak scaling); the time is
the max over ranks and the value is the sum of all ranks' FLOPs over it.

``--impl reference`` times the float64 CPU oracle (the only reference there
is) on a bounded sample of the same workload and prints the same JSON line.

``--workload inference_b1_h8_nq512_nk16384_d128`` (or any forward-only
workload with fewer query rows than keys) times the split-KV forward
(fa_fwd_splitkv: key-range pieces merged by their log-sum-exp, causal
bottom-right aligned) instead; its line reports forward TFLOP/s.
"""
from __future__ import annotations

import argparse
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

METRIC = "attention fwd+bwd TFLOP/s (BF16, d=128, causal) and % of B200 dense BF16 peak"
METRIC_SPLITKV = "attention forward TFLOP/s (BF16, split-KV inference shape)"
METRIC_FP8 = "attention forward TFLOP/s (FP8 e4m3 inputs, bf16 output)"


def metric_for(w):
    """The metric a workload's line reports (the same for both arms)."""
    if w.dtype == "e4m3":
        return METRIC_FP8
    if not w.backward and w.Nq < w.Nk:
        return METRIC_SPLITKV
    return METRIC
NOMINAL_BF16_TFLOPS = 2250.0


def flops(w):
    """Nominal FLOPs: 4*B*Hq*d per visible (query, key) pair, with Nq*Nk/2
    pairs for causal Nq == Nk and Nq*Nk - Nq^2/2 for causal Nq < Nk
    (bottom-right alignment)."""
    pairs = w.Nq * w.Nk - (w.Nq * w.Nq / 2 if w.causal else 0)
    f = 4.0 * w.B * w.Hq * pairs * w.d
    return f, 2.5 * f


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), \
            d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def peak_label(src, what="bf16 dense burst"):
    """Where the roofline denominator came from."""
    if src == "measured":
        return f"measured {what} (MEASURED_PEAKS.json)"
    return f"fallback {what} (no MEASURED_PEAKS.json on this machine)"


def l2_note(w):
    """How the GPU arm keeps the timed inputs out of L2 (126 MB) for this
    workload: inputs larger than L2, or otherwise what stays resident."""
    el = 1 if w.dtype == "e4m3" else 2
    qb = w.B * w.Hq * w.Nq * w.d * el
    kvb = 2 * w.B * w.Hkv * w.Nk * w.d * el
    if not w.backward:
        tot = qb + kvb + w.B * w.Hq * w.Nq * w.d * 2
        what = "q,k,v,o"
    else:
        tot = 3 * qb + kvb     # q, o, dO and k, v
        what = "q,k,v,o,dO"
    mib = tot / 2 ** 20
    if tot > 126e6:
        return f"inputs larger than L2 (no flush): {what} {mib:.0f} MiB"
    return f"inputs {what} {mib:.0f} MiB fit L2 (resident between steps)"


def config_dict(w, n):
    """The workload's configuration; identical in both arms."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "Nq": w.Nq, "d": w.d,
            "causal": w.causal, "scale": "1/sqrt(d)", "global_batch": w.B * n, "seq_len": w.N,
            "parallelism": f"replicas x{n} (no collective: shards by batch/head)",
            "l2": l2_note(w)}


# --------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix=f"fa_clocks_rank{index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        cmd = ["nvidia-smi", f"--id={self.index}",
               "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            try:
                os.remove(self.path)
            except OSError:
                pass
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxs.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------- cross-rank aggregation
def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity alone).
    Every rank must call it at the same point."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_tflops(world, flops_per_rank_step, ms_per_step):
    """All ranks' FLOPs over the slowest rank's time, in TFLOP/s."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ ours
def run_ours(args, rank, world, local_rank):
    import torch
    import attn_inputs
    import exact_io_aware_50_b200 as F

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = attn_inputs.BY_NAME[args.workload]
    fwd_f, bwd_f = flops(w)
    step_flops = fwd_f + bwd_f

    x = attn_inputs.make(w, seed=w.seed + 1000 * rank)
    g = {k: v.to(dev) for k, v in x.items()}
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(g["q"])
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    ws = torch.empty(F.fa_bwd_workspace_size(B, Hq, N, d), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    P = {n: t.data_ptr() for n, t in g.items()}

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {F.fa_strerror(st)}")

    ev = None

    def step(rec=None):
        if rec is not None:
            rec[0].record(stream)
        check(F.fa_fwd(P["q"], P["k"], P["v"], o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                       w.scale, w.causal, sh), "fa_fwd")
        if rec is not None:
            rec[1].record(stream)
        check(F.fa_bwd_prep(P["q"], P["k"], o.data_ptr(), lse.data_ptr(), P["do"], ws.data_ptr(), B,
                            Hq, Hkv, N, N, d, w.scale, sh), "fa_bwd_prep")
        if rec is not None:
            rec[2].record(stream)
        check(F.fa_bwd_dkdv(P["q"], P["k"], P["v"], P["do"], dk.data_ptr(), dv.data_ptr(),
                            ws.data_ptr(), B, Hq, Hkv, N, N, d, w.scale, w.causal, sh),
              "fa_bwd_dkdv")
        if rec is not None:
            rec[3].record(stream)
        check(F.fa_bwd_dq(ws.data_ptr(), dq.data_ptr(), B, Hq, N, d, w.scale, sh), "fa_bwd_dq")
        if rec is not None:
            rec[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if F.fa_device_status(sh) != 0:
        raise RuntimeError("device error word set during warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(events[k])
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    if F.fa_device_status(sh) != 0:
        raise RuntimeError("device error word set during the timed region")
    seg = {"fwd": [], "prep": [], "dkdv": [], "dq": []}
    for e in events:
        seg["fwd"].append(e[0].elapsed_time(e[1]))
        seg["prep"].append(e[1].elapsed_time(e[2]))
        seg["dkdv"].append(e[2].elapsed_time(e[3]))
        seg["dq"].append(e[3].elapsed_time(e[4]))
    mean = {k: sum(v) / len(v) for k, v in seg.items()}

    # ---------------------------------------------------- end to end (host buffers)
    host = {k: v.pin_memory() for k, v in x.items()}
    out_host = {"o": torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                "lse": torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True),
                "dq": torch.empty(dq.shape, dtype=dq.dtype, pin_memory=True),
                "dk": torch.empty(dk.shape, dtype=dk.dtype, pin_memory=True),
                "dv": torch.empty(dv.shape, dtype=dv.dtype, pin_memory=True)}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    e2e_steps = max(2, min(args.steps, 5))

    e2e_ms = time_e2e_pipelined(F, w, g, host, out_host, o, lse, dq, dk, dv, dev, stream,
                                e2e_steps, dist)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(world, step_flops, ms_per_step)
    e2e_value = whole_job_tflops(world, step_flops, e2e_ms)

    burst, sustained, hbm, src = measured_peaks()
    # dominant kernel by measured share of the step
    dom = max(("fwd", "dkdv"), key=lambda k: mean[k])
    dom_flops = fwd_f if dom == "fwd" else bwd_f
    achieved = dom_flops / (mean[dom] * 1e-3) / 1e12
    traffic = load_traffic(w.name, "fa_fwd" if dom == "fwd" else "fa_bwd_dkdv")
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, shapes of the workload)",
        "config": config_dict(w, world),
        "pct_of_nominal_bf16_peak": round(100 * value / world / NOMINAL_BF16_TFLOPS, 2),
        "pct_of_measured_bf16_peak": round(100 * value / world / burst, 2),
        "stage_ms": {k: round(v, 4) for k, v in mean.items()},
        "fwd_tflops": round(fwd_f / (mean["fwd"] * 1e-3) / 1e12, 2),
        "bwd_tflops": round(bwd_f / ((mean["prep"] + mean["dkdv"] + mean["dq"]) * 1e-3) / 1e12, 2),
        "roofline": {"bound": "tensor", "kernel": "fa_fwd" if dom == "fwd" else "fa_bwd_dkdv",
                     "achieved": round(achieved, 2), "peak": burst,
                     "peak_source": peak_label(src),
                     "unit": "TFLOP/s", "frac": round(achieved / burst, 4), "traffic": traffic},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        # per step: forward; prep = centring + preprocess; dkdv (two passes
        # at d = 256); dq conversion
        "gpu_launches": (1 + 2 + (2 if w.d == 256 else 1) + 1) * args.steps,
        "clocks": clk,
    }
    second = SECOND_CONFIG.get(w.name)
    if second and not args.no_second_config:
        # every rank times it (same steps on every rank), max over ranks
        sc = time_training_steps(F, attn_inputs.BY_NAME[second], dev, stream,
                                 max(3, min(args.steps, 10)), 3, rank, world)
        ms = max_over_ranks([sc["ms_per_step"]] + [sc["stage_ms"][k] for k in STAGES], dist, dev)
        sc["ms_per_step"], stage = round(ms[0], 4), dict(zip(STAGES, ms[1:]))
        sc["stage_ms"] = {k: round(v, 4) for k, v in stage.items()}
        sw = attn_inputs.BY_NAME[second]
        f2, b2 = flops(sw)
        sc["value"] = round(whole_job_tflops(world, f2 + b2, ms[0]), 2)
        sc["fwd_tflops"] = round(f2 / (stage["fwd"] * 1e-3) / 1e12, 2)
        sc["bwd_tflops"] = round(b2 / ((stage["prep"] + stage["dkdv"] + stage["dq"]) * 1e-3) / 1e12, 2)
        out["second_config"] = sc
        out["gpu_launches"] += sc["gpu_launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# The metric's headline names d = 128, causal, N >= 4096; the long-context GQA
# configuration is the second one it is quoted on, timed in the same process
# after the first so the driver's run covers both.
SECOND_CONFIG = {"causal_b4_h16_n4096_d128": "long_gqa_b1_hq32_hkv8_n16384_d128_q2x"}
STAGES = ("fwd", "prep", "dkdv", "dq")


def e2e_chunks(w):
    """Chunks of the workload for the end-to-end timing: (first batch element,
    batch elements, first key/value head, key/value heads), each a contiguous
    slice of [B, H, N, d] (several whole batch elements, or one batch element
    and some of its heads).  About eight chunks."""
    if w.B >= 8:
        bn = w.B // 8
        while w.B % bn:
            bn -= 1
        return [(b0, bn, 0, w.Hkv) for b0 in range(0, w.B, bn)]
    kvc = max(1, w.Hkv // max(1, 8 // w.B))
    while w.Hkv % kvc:
        kvc -= 1
    return [(b, 1, h0, kvc) for b in range(w.B) for h0 in range(0, w.Hkv, kvc)]


def time_e2e_pipelined(F, w, g, host, out_host, o, lse, dq, dk, dv, dev, stream, steps, dist):
    """Forward + backward with inputs and results in pinned host memory,
    pipelined over chunks of (batch element, key/value heads): the upload of
    chunk c+1, the kernels of chunk c and the download of chunk c-1 run on
    three streams at once (PCIe copies in both directions overlap each other
    and the kernels).  Every step moves all inputs host -> device and all
    results device -> host; the time runs from the first upload to the last
    download of the timed steps.  Returns ms per step."""
    import torch
    chunks = e2e_chunks(w)
    gq = w.Hq // w.Hkv
    N, d = w.N, w.d
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ws = torch.empty(F.fa_bwd_workspace_size(chunks[0][1], chunks[0][3] * gq, N, d), device=dev,
                     dtype=torch.uint8)

    def sl(t, b, bn, h0, hn):   # batch elements b .. b + bn, heads h0 .. h0 + hn
        return t[b:b + bn, h0:h0 + hn]

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {F.fa_strerror(st)}")

    # per chunk: kernels of the previous step done (inputs free to overwrite),
    # results downloaded (outputs free to overwrite)
    ran = [None] * len(chunks)
    fetched = [None] * len(chunks)

    def one_step():
        for c, (b, bn, k0, kn) in enumerate(chunks):
            q0, qn = k0 * gq, kn * gq
            if ran[c] is not None:
                s_in.wait_event(ran[c])
            with torch.cuda.stream(s_in):
                for name in ("q", "do"):
                    sl(g[name], b, bn, q0, qn).copy_(sl(host[name], b, bn, q0, qn), non_blocking=True)
                for name in ("k", "v"):
                    sl(g[name], b, bn, k0, kn).copy_(sl(host[name], b, bn, k0, kn), non_blocking=True)
                up = torch.cuda.Event()
                up.record(s_in)
            s_run.wait_event(up)
            if fetched[c] is not None:
                s_run.wait_event(fetched[c])
            hs = s_run.cuda_stream
            P = {n: sl(g[n], b, bn, q0, qn).data_ptr() for n in ("q", "do")}
            P.update({n: sl(g[n], b, bn, k0, kn).data_ptr() for n in ("k", "v")})
            po, pl = sl(o, b, bn, q0, qn).data_ptr(), sl(lse, b, bn, q0, qn).data_ptr()
            check(F.fa_fwd(P["q"], P["k"], P["v"], po, pl, bn, qn, kn, N, N, d, w.scale, w.causal, hs),
                  "fa_fwd")
            check(F.fa_bwd(P["q"], P["k"], P["v"], po, pl, P["do"], sl(dq, b, bn, q0, qn).data_ptr(),
                           sl(dk, b, bn, k0, kn).data_ptr(), sl(dv, b, bn, k0, kn).data_ptr(),
                           ws.data_ptr(), bn, qn, kn, N, N, d, w.scale, w.causal, hs), "fa_bwd")
            ran[c] = torch.cuda.Event()
            ran[c].record(s_run)
            s_out.wait_event(ran[c])
            with torch.cuda.stream(s_out):
                for name, t in (("o", o), ("lse", lse), ("dq", dq)):
                    sl(out_host[name], b, bn, q0, qn).copy_(sl(t, b, bn, q0, qn), non_blocking=True)
                for name, t in (("dk", dk), ("dv", dv)):
                    sl(out_host[name], b, bn, k0, kn).copy_(sl(t, b, bn, k0, kn), non_blocking=True)
                fetched[c] = torch.cuda.Event()
                fetched[c].record(s_out)

    one_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for s_ in (s_in, s_run, s_out):
        s_.wait_event(a0)
    for _ in range(steps):
        one_step()
    for s_ in (s_in, s_run, s_out):
        stream.wait_stream(s_)
    a1.record(stream)
    torch.cuda.synchronize()
    return a0.elapsed_time(a1) / steps


def time_e2e_forward_pipelined(F, w, x, g, host, o, lse, o_h, l_h, dev, stream, steps, fp8,
                                dist):
    """Forward only (E4M3 or split-KV) with Q, K, V uploaded from and O, L
    downloaded to pinned host memory every step, pipelined over the same
    chunks as the training step's end-to-end timing.  Returns ms per step."""
    import torch
    chunks = e2e_chunks(w)
    gq = w.Hq // w.Hkv
    Nq, Nk, d = w.Nq, w.Nk, w.d
    b0, bn0, _, kn0 = chunks[0]
    splits = 1 if fp8 else F.fa_fwd_splitkv_num_splits(bn0, kn0 * gq, Nq, Nk, d)
    ws = torch.empty(max(F.fa_fwd_splitkv_workspace_size(bn0, kn0 * gq, Nq, d, splits), 1),
                     device=dev, dtype=torch.uint8)
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def sl(t, b, bn, h0, hn):
        return t[b:b + bn, h0:h0 + hn]

    ran = [None] * len(chunks)
    fetched = [None] * len(chunks)

    def one_step():
        for c, (b, bn, k0, kn) in enumerate(chunks):
            q0, qn = k0 * gq, kn * gq
            if ran[c] is not None:
                s_in.wait_event(ran[c])
            with torch.cuda.stream(s_in):
                sl(g["q"], b, bn, q0, qn).copy_(sl(host["q"], b, bn, q0, qn), non_blocking=True)
                for name in ("k", "v"):
                    sl(g[name], b, bn, k0, kn).copy_(sl(host[name], b, bn, k0, kn), non_blocking=True)
                up = torch.cuda.Event()
                up.record(s_in)
            s_run.wait_event(up)
            if fetched[c] is not None:
                s_run.wait_event(fetched[c])
            hs = s_run.cuda_stream
            pq = sl(g["q"], b, bn, q0, qn).data_ptr()
            pk, pv = (sl(g[n], b, bn, k0, kn).data_ptr() for n in ("k", "v"))
            po, pl = sl(o, b, bn, q0, qn).data_ptr(), sl(lse, b, bn, q0, qn).data_ptr()
            if fp8:
                st = F.fa_fwd_fp8(pq, pk, pv, po, pl, bn, qn, kn, Nq, d, w.scale, x["descale_q"],
                                  x["descale_k"], x["descale_v"], w.causal, hs)
            else:
                st = F.fa_fwd_splitkv(pq, pk, pv, po, pl, ws.data_ptr(), bn, qn, kn, Nq, Nk, d,
                                      w.scale, w.causal, splits, hs)
            if st != 0:
                raise RuntimeError(f"forward: {F.fa_strerror(st)}")
            ran[c] = torch.cuda.Event()
            ran[c].record(s_run)
            s_out.wait_event(ran[c])
            with torch.cuda.stream(s_out):
                sl(o_h, b, bn, q0, qn).copy_(sl(o, b, bn, q0, qn), non_blocking=True)
                sl(l_h, b, bn, q0, qn).copy_(sl(lse, b, bn, q0, qn), non_blocking=True)
                fetched[c] = torch.cuda.Event()
                fetched[c].record(s_out)

    one_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for s_ in (s_in, s_run, s_out):
        s_.wait_event(a0)
    for _ in range(steps):
        one_step()
    for s_ in (s_in, s_run, s_out):
        stream.wait_stream(s_)
    a1.record(stream)
    torch.cuda.synchronize()
    return a0.elapsed_time(a1) / steps


def time_training_steps(F, w, dev, stream, steps, warmup, rank, world):
    """Device time of `steps` training steps (fa_fwd, fa_bwd_prep, fa_bwd_dkdv,
    fa_bwd_dq) on workload `w`, each stage bracketed by CUDA events on the
    launching stream; inputs are created, moved to the device and released
    here (they are larger than L2, so no flush is needed between steps)."""
    import torch
    import attn_inputs
    x = attn_inputs.make(w, seed=w.seed + 1000 * rank)
    g = {k: v.to(dev) for k, v in x.items()}
    del x
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(g["q"])
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    ws = torch.empty(F.fa_bwd_workspace_size(B, Hq, N, d), device=dev, dtype=torch.uint8)
    sh = stream.cuda_stream
    P = {n: t.data_ptr() for n, t in g.items()}

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {F.fa_strerror(st)}")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        check(F.fa_fwd(P["q"], P["k"], P["v"], o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                       w.scale, w.causal, sh), "fa_fwd")
        if ev is not None:
            ev[1].record(stream)
        check(F.fa_bwd_prep(P["q"], P["k"], o.data_ptr(), lse.data_ptr(), P["do"], ws.data_ptr(),
                            B, Hq, Hkv, N, N, d, w.scale, sh), "fa_bwd_prep")
        if ev is not None:
            ev[2].record(stream)
        check(F.fa_bwd_dkdv(P["q"], P["k"], P["v"], P["do"], dk.data_ptr(), dv.data_ptr(),
                            ws.data_ptr(), B, Hq, Hkv, N, N, d, w.scale, w.causal, sh),
              "fa_bwd_dkdv")
        if ev is not None:
            ev[3].record(stream)
        check(F.fa_bwd_dq(ws.data_ptr(), dq.data_ptr(), B, Hq, N, d, w.scale, sh), "fa_bwd_dq")
        if ev is not None:
            ev[4].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(steps):
        step(events[k])
    t1.record(stream)
    torch.cuda.synchronize()
    if F.fa_device_status(sh) != 0:
        raise RuntimeError(f"device error word set while timing {w.name}")
    stage = {k: sum(e[i].elapsed_time(e[i + 1]) for e in events) / steps
             for i, k in enumerate(STAGES)}
    del g, o, lse, dq, dk, dv, ws
    return {"workload": w.name, "config": config_dict(w, world), "steps": steps, "warmup": warmup,
            "ms_per_step": t0.elapsed_time(t1) / steps, "stage_ms": stage,
            "gpu_launches": (1 + 2 + (2 if d == 256 else 1) + 1) * steps}


def run_forward_only(args, rank, world, local_rank):
    """Forward only: the split-KV path on an inference-shaped workload, or the
    E4M3 forward on an e4m3 workload."""
    import torch
    import attn_inputs
    import exact_io_aware_50_b200 as F

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = attn_inputs.BY_NAME[args.workload]
    fwd_f, _ = flops(w)
    fp8 = w.dtype == "e4m3"
    x = (attn_inputs.make_fp8 if fp8 else attn_inputs.make)(w, seed=w.seed + 1000 * rank)
    g = {k: x[k].to(dev) for k in ("q", "k", "v")}
    B, Hq, Hkv, Nq, Nk, d = w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d
    splits = 1 if fp8 else F.fa_fwd_splitkv_num_splits(B, Hq, Nq, Nk, d)
    o = torch.empty(B, Hq, Nq, d, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, Nq, device=dev, dtype=torch.float32)
    ws = torch.empty(max(F.fa_fwd_splitkv_workspace_size(B, Hq, Nq, d, splits), 1), device=dev,
                     dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        if fp8:
            st = F.fa_fwd_fp8(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(),
                              o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, d, w.scale,
                              x["descale_q"], x["descale_k"], x["descale_v"], w.causal,
                              stream.cuda_stream)
        else:
            st = F.fa_fwd_splitkv(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(),
                                  o.data_ptr(), lse.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, Nk,
                                  d, w.scale, w.causal, splits, stream.cuda_stream)
        if st != 0:
            raise RuntimeError(f"{'fa_fwd_fp8' if fp8 else 'fa_fwd_splitkv'}: {F.fa_strerror(st)}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    if F.fa_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device error word set during the timed region")
    total_ms = t0.elapsed_time(t1)
    host = {k: x[k].pin_memory() for k in ("q", "k", "v")}
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + l_h.numel() * l_h.element_size()
    n_e2e = max(2, min(args.steps, 5))
    e2e_ms = time_e2e_forward_pipelined(F, w, x, g, host, o, lse, o_h, l_h, dev, stream, n_e2e,
                                        fp8, dist)
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
    ms = total_ms / args.steps
    burst, _, _, src = measured_peaks()
    value = whole_job_tflops(world, fwd_f, ms)
    achieved = fwd_f / (ms * 1e-3) / 1e12
    if fp8:
        # e4m3 dense peak: the measured bf16 burst times the nominal ratio
        # (4.5 / 2.25 PFLOP/s dense)
        peak, peak_src = 2.0 * burst, peak_label(src, "bf16 dense burst x 2 (nominal e4m3/bf16 ratio)")
        metric = METRIC_FP8
        data = "synthetic (seeded N(0,1) float32 quantised per tensor to e4m3, shapes of the workload)"
        kernel = "fa_fwd_fp8"
    else:
        peak, peak_src = burst, peak_label(src)
        metric = METRIC_SPLITKV
        data = "synthetic (seeded N(0,1) bf16, shapes of the workload)"
        kernel = "fa_fwd_splitkv (pieces + merge)"
    out = {
        "metric": metric,
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16",
        "data": data,
        "config": dict(config_dict(w, world), num_splits=splits),
        "roofline": {"bound": "tensor", "kernel": kernel,
                     "achieved": round(achieved, 2), "peak": round(peak, 2),
                     "peak_source": peak_src,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": load_traffic(w.name, "fa_fwd_fp8") if fp8 else None},
        "e2e": {"value": round(whole_job_tflops(world, fwd_f, e2e_ms), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": (2 if splits > 1 else 1) * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def load_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if
    one exists for this workload and the kernel source has not changed since
    (the summary records the source hash)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as fh:
            d = json.load(fh)
        ent = d.get(workload, {}).get(kernel)
        if not ent:
            return None
        if ent.get("source_sha") != source_sha(KERNEL_SOURCES.get(kernel)):
            return None
        return ent.get("bytes_per_launch")
    except (OSError, ValueError):
        return None


# The sources each recorded kernel is compiled from.
KERNEL_SOURCES = {
    "fa_fwd": ("common.cuh", "cta_pair.cuh", "fa_fwd_sm100.cu", "launch.h"),
    "fa_fwd_fp8": ("common.cuh", "cta_pair.cuh", "fa_fwd_sm100.cu", "launch.h"),
    "fa_bwd_dkdv": ("common.cuh", "fa_bwd_sm100.cu", "launch.h"),
}


def source_sha(files=None):
    """Hash of the given kernel source files (default: all of them) with
    comments and blank lines removed, so a comment edit does not invalidate
    recorded counters but a code edit does."""
    import hashlib
    import re
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "exact_io_aware_50_b200", "csrc")
    for f in sorted(files or os.listdir(cs)):
        with open(os.path.join(cs, f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())
        h.update(f.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


# ------------------------------------------------------------ CPU oracle
def cpu_baseline(w, seconds):
    """Time the float64 oracle (as it stands) on whole (batch, head) units of
    the workload until about `seconds` of CPU work; throughput in the same
    unit (attention fwd+bwd FLOPs per second)."""
    import numpy as np
    import attn_inputs
    import oracle
    import oracle.fp8
    fp8 = w.dtype == "e4m3"
    if fp8:
        x = attn_inputs.make_fp8(w, B=1, Hq=w.Hq // w.Hkv, Hkv=1)
        q, k, v = (x[n].numpy() for n in ("q", "k", "v"))
    else:
        x = attn_inputs.make(w, B=1, Hq=w.Hq // w.Hkv, Hkv=1)  # one key/value group of batch 0
        q, k, v, do = (attn_inputs.as_f64(x[n]) for n in ("q", "k", "v", "do"))
    heads = 0
    t0 = time.perf_counter()
    g = w.Hq // w.Hkv
    off = w.Nk - w.Nq if w.causal else 0     # bottom-right alignment when Nq < Nk
    while True:
        h = heads % g
        if fp8:
            oracle.fp8.fp8_forward(q[:, h:h + 1], k, v, x["descale_q"], x["descale_k"],
                                   x["descale_v"], w.scale, w.causal)
        else:
            oracle.forward(q[:, h:h + 1], k, v, w.scale, w.causal, off)
        if w.backward:
            oracle.backward(q[:, h:h + 1], k, v, do[:, h:h + 1], w.scale, w.causal)
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds or heads >= w.B * w.Hq:
            break
    fwd_f, bwd_f = flops(w)
    per_head = (fwd_f + (bwd_f if w.backward else 0.0)) / (w.B * w.Hq)
    value = heads * per_head / el / 1e12
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        nth = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if nth:
            cores = nth[0]
    except Exception:
        pass
    return {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} whole (batch 0, head) units of {w.name}, "
                      f"{'forward+backward' if w.backward else 'forward'}, "
                      f"{el:.1f} s; full workload has {w.B * w.Hq} heads",
            "units": heads, "seconds": el}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle as it stands, on the host cores.
    Each of the `steps` samples times whole (batch, head) units of the
    workload for about cpu_seconds / steps; the line's value is the median
    throughput and its ms_per_step the time one whole step of the workload
    would take at that rate (extrapolated: the oracle does not run a whole
    step here, and the line says so beside the time it did measure)."""
    if rank != 0:
        return
    import attn_inputs
    w = attn_inputs.BY_NAME[args.workload]
    samples = [cpu_baseline(w, args.cpu_seconds / max(1, args.steps)) for _ in range(args.steps)]
    value = statistics.median(s["value"] for s in samples)
    fwd_f, bwd_f = flops(w)
    ms = (fwd_f + (bwd_f if w.backward else 0.0)) / (value * 1e12) * 1e3
    units = sum(s["units"] for s in samples)
    secs = sum(s["seconds"] for s in samples)
    cb = dict(samples[-1])
    cb["value"] = value
    out = {"impl": "reference", "metric": metric_for(w), "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms, "extrapolated": True,
           "measured": {"units_timed": units, "seconds": round(secs, 3),
                        "ms_per_unit": round(1e3 * secs / max(units, 1), 3),
                        "units_per_step": w.B * w.Hq,
                        "unit": "one (batch, head) of the workload, "
                                + ("forward+backward" if w.backward else "forward")},
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic (seeded N(0,1), shapes of the workload)",
           "config": config_dict(w, world),
           "cpu_baseline": cb,
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="causal_b4_h16_n4096_d128")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-second-config", action="store_true",
                    help="skip the long-context GQA step timed after the default workload")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.warmup < 3:
        args.warmup = 3
    import attn_inputs
    w = attn_inputs.BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif not w.backward and (w.Nq < w.Nk or w.dtype == "e4m3"):
        run_forward_only(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
