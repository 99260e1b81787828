#!/usr/bin/env python
"""Throughput of the exact-attention hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch of synthetic input: attn_fwd and
attn_bwd (D preprocess, main backward, dQ convert) on the gate workload B=4, H=16,
N=4096, d=128, bf16 (the head_dim/seqlen sweep's d=128, N=4096 point), once without and
once with the causal mask.  The metric is attention TFLOP/s (4*B*H*N^2*d for the forward,
2.5x that for the backward, halved for causal) and its fraction of the measured dense
BF16 tensor-core peak; the line also gives the forward and the backward pass separately
(per mask), each with the roofline of its main kernel and the oracle's time for the same
pass.

One process per GPU (torchrun sets RANK / LOCAL_RANK / WORLD_SIZE); each rank runs its own
batch (weak scaling, no collective on the data path); the time is the max over ranks.
Timing: CUDA events on the launching stream around each step and each pass, L2 flushed
(a 256 MiB write) between timed steps, per-kernel times from the library's own launch
events.  ``--impl reference`` times the fp64 CPU oracle (the only reference there is) on
a bounded sample of the same workload, on rank 0 only.
"""
import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import attn_workloads as W  # noqa: E402

METRIC = "attention fwd/bwd TFLOPs/s on 1 B200 (bf16, d=128) and % of dense BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
DATA = "synthetic: Q, K, V, dO iid N(0,1) drawn in fp32 from a seeded torch CPU generator, rounded to bf16"


DEFAULT_WORKLOAD = "sweep_d128_n4096"
WORKLOAD = DEFAULT_WORKLOAD   # set from --workload


def base_workload(name):
    """The named workload (non-causal variant where it has both)."""
    if name == "mha2k":
        return W.mha2k(False)
    if name.startswith("sweep_d"):       # sweep_d<d>_n<N>
        d, n = name[len("sweep_d"):].split("_n")
        return W.sweep(int(d), int(n))
    return {"gqa8k": W.gqa8k(), "varlen16": W.varlen16(), "long32k": W.long32k()}[name]


def workload_variants(rank=0):
    base = base_workload(WORKLOAD)
    import dataclasses
    base = dataclasses.replace(base, seed=base.seed + rank)
    if base.causal:          # configurations that are causal only
        return [base]
    return [base, base.with_causal(True)]


def config_block(n_gpus):
    w = base_workload(WORKLOAD)
    desc = (f"{WORKLOAD}: B={w.batch} Hq={w.hq} Hkv={w.hkv} N={w.seqlen or w.max_seqlen} d={w.d} bf16, fwd+bwd, "
            + ("causal" if w.causal else "non-causal and causal"))
    return {"workload": desc, "global_batch": w.batch * n_gpus, "seq_len": w.seqlen or w.max_seqlen,
            "heads": w.hq, "head_dim": w.d,
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{n_gpus}"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]), "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", 0)),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ---------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], 0, False
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that, keep going
            self.err = str(e)

    def _run(self):
        while not self.stop_flag.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self.stop_flag.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# CPU side: the fp64 oracle as a timed baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------------------
_ORACLE_CACHE = {}


def oracle_sample(heads, budget_s=None):
    """Oracle forward + backward on whole heads of sequence 0 of both variants.  Runs the
    given number of heads, or (budget_s) adds heads until the budget is spent.
    Returns ({"fwd": (flops, s), "bwd": (flops, s)}, heads done, threads)."""
    import oracle
    per = {"fwd": [0.0, 0.0], "bwd": [0.0, 0.0]}
    done = 0
    threads = oracle.default_threads()
    variants = workload_variants()
    base = variants[0]
    if "inputs" not in _ORACLE_CACHE:
        _ORACLE_CACHE["inputs"] = W.make_inputs(base)
    q, k, v, do, cu = _ORACLE_CACHE["inputs"]
    n = int(cu[1] - cu[0])
    G = base.hq // base.hkv
    for h in range(base.hq):
        if heads is not None and done >= heads:
            break
        if budget_s is not None and per["fwd"][1] + per["bwd"][1] >= budget_s:
            break
        qs, dos = (t[:n, h:h + 1].contiguous() for t in (q, do))
        ks, vs = (t[:n, h // G:h // G + 1].contiguous() for t in (k, v))
        for causal in sorted({w.causal for w in variants}):
            f = 4.0 * n * n * base.d * (0.5 if causal else 1.0)
            t0 = time.perf_counter()
            oracle.attn_fwd(qs, ks, vs, scale=base.scale, causal=causal, threads=threads)
            t1 = time.perf_counter()
            oracle.attn_bwd(qs, ks, vs, dos, scale=base.scale, causal=causal, threads=threads)
            t2 = time.perf_counter()
            per["fwd"][0] += f
            per["fwd"][1] += t1 - t0
            per["bwd"][0] += 2.5 * f
            per["bwd"][1] += t2 - t1
        done += 1
    return {k_: tuple(v_) for k_, v_ in per.items()}, done, threads


def oracle_totals(per):
    return per["fwd"][0] + per["bwd"][0], per["fwd"][1] + per["bwd"][1]


def run_reference(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(heads=1)
    flops = secs = 0.0
    threads = 1
    for _ in range(args.steps):
        per, _, threads = oracle_sample(heads=1)
        f, s = oracle_totals(per)
        flops += f
        secs += s
    value = flops / secs / 1e12
    sample = f"fp64 CPU oracle, fwd+bwd of 1 head of sequence 0 of {WORKLOAD} (all its mask variants), per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": config_block(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank contributes its own device-timed milliseconds."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------
# GPU side
# ---------------------------------------------------------------------------------------
def code_hash(path):
    """sha256 (first 16 hex digits) of a C/CUDA source with its comments and all whitespace
    removed: it changes when the code does, not when only a comment is edited."""
    import hashlib
    import re
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    text = re.sub(r"\s+", "", text)
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def traffic_record(kernel, workload=None, path=None):
    """The committed ncu record of `kernel` (DRAM bytes per launch, tensor-pipe and
    special-function-unit activity) if it was taken on the current kernel code and, when
    `workload` is given, on that workload (else None: the figures would not apply).
    Records are keyed "<kernel>@<workload>"."""
    path = path or os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    if workload is not None:
        rec = table.get(f"{kernel}@{workload}")
    else:
        rec = next((r for key, r in table.items() if key.split("@")[0] == kernel), None)
    if not isinstance(rec, dict):
        return None
    src = os.path.join(ROOT, "io_aware_exact_qk_b200", "csrc", rec["source"])
    return rec if code_hash(src) == rec["source_code_sha256_16"] else None


def roofline_block(kernel, flops_per_launch, mean_launch_ms, peaks, workload):
    """Roofline of one tensor-bound kernel: algorithmic FLOPs per launch over its mean
    event-timed launch, against the measured dense bf16 peak; DRAM traffic and ncu's
    tensor-pipe activity from the committed capture of the same code and workload."""
    achieved = flops_per_launch / (mean_launch_ms / 1e3) / 1e12
    rec = traffic_record(kernel, workload)
    return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": UNIT,
            "frac": achieved / peaks["bf16_tflops"],
            "traffic": rec["dram_bytes_per_launch"] if rec else None,
            "ncu_tensor_pipe_active": rec.get("tensor_pipe_active") if rec else None,
            "ncu_sfu_pipe_active": rec.get("xu_pipe_active") if rec else None,
            "peak_source": f"{peaks['source']} dense bf16 (burst)",
            "flops_per_launch": flops_per_launch, "mean_launch_ms": mean_launch_ms}


def run_ours(args, rank, world, local_rank):
    import io_aware_exact_qk_b200 as attn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    attn.load_library()
    variants = workload_variants(rank)
    q, k, v, do, cu = W.make_inputs(variants[0])
    host = {"q": q.pin_memory(), "k": k.pin_memory(), "v": v.pin_memory(), "do": do.pin_memory()}
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    w0 = variants[0]
    shape_kw = (dict(cu_seqlens=cu.to(dev), max_seqlen=w0.max_seqlen) if w0.varlen else dict(batch=w0.batch))
    outs = {}
    for w in variants:
        outs[w.causal] = {"o": torch.empty_like(qd), "lse": torch.empty(w.hq, w.total_tokens, device=dev),
                          "dq": torch.empty_like(qd), "dk": torch.empty_like(kd), "dv": torch.empty_like(vd)}
    ws = torch.empty(attn.workspace_size("bwd", qd, kd, **shape_kw), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(marks=None):
        """One step; with `marks` ({(causal, pass): [start, end] events}) each pass is
        bracketed by events on the launching stream."""
        for w in variants:
            b = outs[w.causal]
            if marks:
                marks[(w.causal, "fwd")][0].record(stream)
            attn.attn_fwd(qd, kd, vd, scale=w.scale, causal=w.causal, o=b["o"], lse=b["lse"], **shape_kw)
            if marks:
                marks[(w.causal, "fwd")][1].record(stream)
            attn.attn_bwd(qd, kd, vd, b["o"], dod, b["lse"], scale=w.scale, causal=w.causal,
                          dq=b["dq"], dk=b["dk"], dv=b["dv"], workspace=ws, **shape_kw)
            if marks:
                marks[(w.causal, "bwd")][1].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    flops_fwd = {w.causal: w.fwd_flops() for w in variants}
    flops_step = sum(w.fwd_flops() + w.bwd_flops() for w in variants)

    for _ in range(args.warmup):
        step()
    attn.attn_get_device_error()
    barrier()

    # ---- timed region (device): per-step and per-pass events, L2 flushed between steps ----
    def new_marks():
        m = {}
        for w in variants:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            m[(w.causal, "fwd")] = (e[0], e[1])
            m[(w.causal, "bwd")] = (e[1], e[2])   # the backward starts where the forward ends
        return m

    attn.attn_profile_collect()
    attn.attn_profile_enable(True)
    launches0 = attn.attn_launch_count()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), new_marks())
              for _ in range(args.steps)]
    with ClockSampler(local_rank) as clocks:
        barrier()
        for s, e, marks in events:
            flush.zero_()
            s.record(stream)
            step(marks)
            e.record(stream)
        barrier()
    attn.attn_profile_enable(False)
    launches = attn.attn_launch_count() - launches0
    per_kernel = attn.attn_profile_collect()
    attn.attn_get_device_error()
    total_ms = sum(s.elapsed_time(e) for s, e, _ in events)
    total_ms = max_over_ranks(total_ms, world, dev)
    value = world * flops_step * args.steps / (total_ms / 1e3) / 1e12
    pass_ms = {key: max_over_ranks(sum(m[key][0].elapsed_time(m[key][1]) for _, _, m in events), world, dev)
               for key in events[0][2]}

    # ---- end to end: host buffers, copies inside the timed region ----
    if args.quick:
        if rank == 0:
            print(json.dumps({"quick": True, "value": value, "unit": UNIT, "ms_per_step": total_ms / args.steps,
                              "passes_ms": {f"{p_}{'+causal' if c else ''}": v_ / args.steps
                                            for (c, p_), v_ in pass_ms.items()},
                              "kernels": {k: list(v) for k, v in per_kernel.items()}, "gpu_launches": launches}))
        return
    e2e_steps = min(args.steps, 20)
    e2e_bufs = {}
    e2e_out = {}
    host_kw = dict(cu_seqlens=cu, max_seqlen=w0.max_seqlen) if w0.varlen else dict(batch=w0.batch)
    for w in variants:
        _, e2e_bufs[w.causal] = attn.attention_host(host["q"], host["k"], host["v"], host["do"], scale=w.scale,
                                                    causal=w.causal, **host_kw)
    torch.cuda.synchronize()
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v", "do")) * len(variants)
    d2h = sum(t.numel() * t.element_size() for b in e2e_bufs.values() for t in b["host"])
    barrier()
    # the two masks are independent problems with their own buffers: each goes on a stream
    # of its own, so that one's uploads can run while the other computes or downloads
    mask_streams = {w.causal: torch.cuda.Stream() for w in variants}
    e2e_start, e2e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_start.record(stream)
    for ms in mask_streams.values():
        ms.wait_event(e2e_start)
    for _ in range(e2e_steps):
        for w in variants:
            e2e_out[w.causal], _ = attn.attention_host(host["q"], host["k"], host["v"], host["do"], scale=w.scale,
                                                       causal=w.causal, out=e2e_bufs[w.causal],
                                                       stream=mask_streams[w.causal], **host_kw)
    for ms in mask_streams.values():
        stream.wait_stream(ms)
    e2e_end.record(stream)
    barrier()
    attn.attn_get_device_error()
    e2e_ms = e2e_start.elapsed_time(e2e_end)
    e2e_value = world * flops_step * e2e_steps / (max_over_ranks(e2e_ms, world, dev) / 1e3) / 1e12

    if rank != 0:
        return
    peaks = load_peaks()
    # per-pass results: TF/s of each (pass, mask) from its events, and the roofline of the
    # pass's main kernel from the library's per-launch events
    cpu = None
    cpu_per = None
    if world == 1:
        cpu_per, heads, threads = oracle_sample(heads=None, budget_s=12.0)
        f, s_ = oracle_totals(cpu_per)
        cpu = {"value": f / s_ / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 CPU oracle, fwd+bwd of {heads} whole head(s) of sequence 0 of {WORKLOAD} "
                         f"(all its mask variants), {s_:.1f} s"}
    passes = {}
    for pname, kname, mult in (("fwd", "fwd_bf16_sm100", 1.0), ("bwd", "bwd_bf16_sm100", 2.5)):
        by_mask = {}
        tot_f = tot_ms = 0.0
        for w in variants:
            f = mult * flops_fwd[w.causal] * args.steps
            ms = pass_ms[(w.causal, pname)]
            by_mask["causal" if w.causal else "non_causal"] = {
                "value": world * f / (ms / 1e3) / 1e12, "frac": world * f / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                "ms": ms / args.steps}
            tot_f += f
            tot_ms += ms
        entry = {"value": world * tot_f / (tot_ms / 1e3) / 1e12, "unit": UNIT,
                 "frac": world * tot_f / (tot_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                 "ms_per_step": tot_ms / args.steps, "by_mask": by_mask,
                 "includes": ("attn_fwd: work-item counter reset + fwd_bf16_sm100" if pname == "fwd" else
                              "attn_bwd: bwd_preprocess + bwd_bf16_sm100 + bwd_dq_convert")}
        if kname in per_kernel:
            k_ms, k_n = per_kernel[kname]
            entry["roofline"] = roofline_block(kname, mult * sum(flops_fwd.values()) * args.steps / k_n,
                                               k_ms / k_n, peaks, WORKLOAD)
        if cpu_per is not None:
            f, s_ = cpu_per[pname]
            entry["cpu_baseline"] = {"value": f / s_ / 1e12, "unit": UNIT, "cores": cpu["cores"], "kind": "oracle",
                                     "sample": f"fp64 CPU oracle, {pname} of {heads} whole head(s) of sequence 0 of "
                                               f"{WORKLOAD} (all its mask variants), {s_:.1f} s"}
        passes[pname] = entry
    # dominant kernel and its roofline (algorithmic FLOPs per launch / mean event duration)
    dom = max(per_kernel, key=lambda n: per_kernel[n][0])
    dom_ms, dom_n = per_kernel[dom]
    if dom.startswith("bwd_bf16"):
        dom_flops = sum(2.5 * f for f in flops_fwd.values()) * args.steps
    elif dom.startswith("fwd_bf16"):
        dom_flops = sum(flops_fwd.values()) * args.steps
    else:
        dom_flops = 0.0
    roofline = roofline_block(dom, dom_flops / dom_n, dom_ms / dom_n, peaks, WORKLOAD)
    breakdown = {}
    for name, (ms, n) in sorted(per_kernel.items()):
        breakdown[name] = {"launches": n, "total_ms": ms, "share": ms / sum(x[0] for x in per_kernel.values())}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA, "config": config_block(world),
            "pct_of_peak": value / peaks["bf16_tflops"], "roofline": roofline, "passes": passes,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gpu_launches": launches, "clocks": clocks.summary(), "kernels": breakdown}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# Decoding workloads (split-KV forward): HBM-bound, reported in GB/s of algorithmic traffic
# ---------------------------------------------------------------------------------------
DECODE_METRIC = "split-KV decode forward: algorithmic HBM GB/s (K, V, Q read once, O, LSE written) on 1 B200"
DECODE_WORKLOADS = {"decode8k": W.decode8k, "decode_var": W.decode_var, "decode_spec4": W.decode_spec4}
DECODE_DATA = ("synthetic: Q, K, V iid N(0,1) drawn in fp32 from a seeded torch CPU generator (decode_var: key "
               "lengths drawn first from the same generator), rounded to bf16")


def decode_config(n_gpus):
    w = DECODE_WORKLOADS[WORKLOAD]()
    return {"workload": f"{WORKLOAD}: {w.batch} sequences, Lq={sorted(set(w.q_lens))}, Lk max {w.max_k} "
                        f"(total {w.total_k}), Hq={w.hq} Hkv={w.hkv} d={w.d} bf16, "
                        + ("causal" if w.causal else "non-causal"),
            "global_batch": w.batch * n_gpus, "kv_bytes": w.kv_bytes(), "hbm_bytes_per_step": w.hbm_bytes(),
            "l2": "inputs larger than L2 (K/V of 268-979 MB against 126 MB), no flush between steps (a 256 MiB "
                  "write would leave dirty lines whose write-back competes with the reads)",
            "parallelism": f"replicas x{n_gpus}"}


def decode_oracle_sample(budget_s):
    """Oracle decode forward on whole sequences (all heads) until the budget is spent.
    Returns (algorithmic bytes of the sequences done, seconds, sequences, threads)."""
    import oracle
    w = DECODE_WORKLOADS[WORKLOAD]()
    if "decode" not in _ORACLE_CACHE:
        _ORACLE_CACHE["decode"] = W.make_decode_inputs(w)
    q, k, v, cu_q, cu_k = _ORACLE_CACHE["decode"]
    threads = oracle.default_threads()
    nbytes, secs, done = 0, 0.0, 0
    for b in range(w.batch):
        if secs >= budget_s and done > 0:
            break
        qs, ks, vs = q[cu_q[b]:cu_q[b + 1]], k[cu_k[b]:cu_k[b + 1]], v[cu_k[b]:cu_k[b + 1]]
        lq, lk = int(cu_q[b + 1] - cu_q[b]), int(cu_k[b + 1] - cu_k[b])
        t0 = time.perf_counter()
        oracle.attn_fwd_cross(qs, ks, vs, [0, lq], [0, lk], scale=w.scale, causal=w.causal, threads=threads)
        secs += time.perf_counter() - t0
        nbytes += 2 * lk * w.hkv * w.d * 2 + 2 * lq * w.hq * w.d * 2 + 4 * lq * w.hq
        done += 1
    return nbytes, secs, done, threads


def run_reference_decode(args, rank, world):
    if rank != 0:
        return
    decode_oracle_sample(0.0)
    nbytes = secs = 0.0
    threads = 1
    for _ in range(args.steps):
        b, s_, _, threads = decode_oracle_sample(0.0)   # one whole sequence per step
        nbytes += b
        secs += s_
    value = nbytes / secs / 1e9
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DECODE_DATA,
            "config": decode_config(world),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"fp64 CPU oracle, sequence 0 of {WORKLOAD} (all heads) per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode(args, rank, world, local_rank):
    import io_aware_exact_qk_b200 as attn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    attn.load_library()
    w = DECODE_WORKLOADS[WORKLOAD]()
    w = dataclasses.replace(w, seed=w.seed + rank)
    q, k, v, cu_q, cu_k = W.make_decode_inputs(w)
    qd, kd, vd, cqd, ckd = (t.to(dev) for t in (q, k, v, cu_q, cu_k))
    mq = max(w.q_lens)
    ws_bytes = attn.decode_workspace_size(qd, kd, cqd, ckd, mq, w.max_k)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    o = torch.empty_like(qd)
    lse = torch.empty(w.hq, w.total_q, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        attn.attn_fwd_decode(qd, kd, vd, cqd, ckd, mq, w.max_k, scale=w.scale, causal=w.causal, o=o, lse=lse,
                             workspace=ws)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    attn.attn_get_device_error()
    barrier()
    attn.attn_profile_collect()
    attn.attn_profile_enable(True)
    launches0 = attn.attn_launch_count()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clocks:
        barrier()
        for s_, e_ in events:
            s_.record(stream)
            step()
            e_.record(stream)
        barrier()
    attn.attn_profile_enable(False)
    launches = attn.attn_launch_count() - launches0
    per_kernel = attn.attn_profile_collect()
    attn.attn_get_device_error()
    total_ms = sum(s_.elapsed_time(e_) for s_, e_ in events)
    total_ms = max_over_ranks(total_ms, world, dev)
    value = world * w.hbm_bytes() * args.steps / (total_ms / 1e3) / 1e9
    if args.quick:
        if rank == 0:
            print(json.dumps({"quick": True, "value": value, "unit": "GB/s", "ms_per_step": total_ms / args.steps,
                              "kernels": {k_: list(v_) for k_, v_ in per_kernel.items()}, "gpu_launches": launches}))
        return
    # end to end: the caller's Q/K/V in pinned host memory, O and LSE back to the host
    hq_, hk_, hv_ = q.pin_memory(), k.pin_memory(), v.pin_memory()
    ho, hl = torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(lse.shape).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        qd.copy_(hq_, non_blocking=True)
        kd.copy_(hk_, non_blocking=True)
        vd.copy_(hv_, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)
    e1.record(stream)
    barrier()
    attn.attn_get_device_error()
    e2e_value = world * w.hbm_bytes() * args.steps / (max_over_ranks(e0.elapsed_time(e1), world, dev) / 1e3) / 1e9
    if rank != 0:
        return
    peaks = load_peaks()
    dom = max(per_kernel, key=lambda n_: per_kernel[n_][0])
    dom_ms, dom_n = per_kernel[dom]
    dom_bytes = w.hbm_bytes() if dom.startswith("decode_bf16") else 0
    achieved = dom_bytes * args.steps / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "peak_source": f"{peaks['source']} HBM copy bandwidth",
                "bytes_per_launch": dom_bytes * args.steps / dom_n, "mean_launch_ms": dom_ms / dom_n}
    breakdown = {k_: {"launches": n_, "total_ms": ms, "share": ms / sum(x[0] for x in per_kernel.values())}
                 for k_, (ms, n_) in sorted(per_kernel.items())}
    cpu = None
    if world == 1:
        b, s_, done, threads = decode_oracle_sample(12.0)
        cpu = {"value": b / s_ / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"fp64 CPU oracle, {done} whole sequence(s) of {WORKLOAD} (all heads), {s_:.1f} s"}
    line = {"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DECODE_DATA, "config": decode_config(world),
            "pct_of_peak": value / peaks["hbm_gbs"], "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches, "clocks": clocks.summary(), "kernels": breakdown}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# FP8 (e4m3) forward: per-head quantised operands, both products on e4m3 tensor cores
# ---------------------------------------------------------------------------------------
FP8_METRIC = "FP8 (e4m3) attention forward TFLOPs/s on 1 B200 (d=128) and % of dense FP8 peak"
FP8_WORKLOADS = {"fp8_mha2k": lambda: W.mha2k(False)}


def fp8_config(n_gpus):
    w = FP8_WORKLOADS[WORKLOAD]()
    return {"workload": f"{WORKLOAD}: B={w.batch} Hq={w.hq} Hkv={w.hkv} N={w.seqlen} d={w.d}, e4m3 Q/K/V with "
                        "per-head scales (quantised once, outside the timed step), forward only, non-causal and "
                        "causal",
            "global_batch": w.batch * n_gpus, "seq_len": w.seqlen, "heads": w.hq, "head_dim": w.d,
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{n_gpus}"}


def fp8_oracle_sample(heads=None, budget_s=None):
    """The oracle's FP8 forward (fp8sim) on whole heads of sequence 0, both masks, on the
    operands dequantised from a per-head e4m3 quantisation done here on the CPU."""
    import oracle
    w = FP8_WORKLOADS[WORKLOAD]()
    if "fp8" not in _ORACLE_CACHE:
        q, k, v, _, _ = W.make_inputs(w, with_grad=False)
        deq = []
        for x in (q, k, v):
            xf = x.float()
            amax = xf.abs().amax(dim=(0, 2))
            ds = torch.where(amax > 0, amax / torch.tensor(448.0), torch.ones_like(amax))
            x8 = (xf / ds[None, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn)
            deq.append(x8.double() * ds.double()[None, :, None])
        _ORACLE_CACHE["fp8"] = deq
    q, k, v = _ORACLE_CACHE["fp8"]
    n, G = w.seqlen, w.hq // w.hkv
    threads = oracle.default_threads()
    flops, secs, done = 0.0, 0.0, 0
    for h in range(w.hq):
        if (heads is not None and done >= heads) or (budget_s is not None and secs >= budget_s):
            break
        qs = q[:n, h:h + 1].numpy().copy()
        ks, vs = (t[:n, h // G:h // G + 1].numpy().copy() for t in (k, v))
        for causal in (False, True):
            t0 = time.perf_counter()
            oracle.attn_fwd_fp8sim(qs, ks, vs, scale=w.scale, causal=causal, threads=threads)
            secs += time.perf_counter() - t0
            flops += 4.0 * n * n * w.d * (0.5 if causal else 1.0)
        done += 1
    return flops, secs, done, threads


def run_reference_fp8(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        fp8_oracle_sample(heads=1)
    flops = secs = 0.0
    threads = 1
    for _ in range(args.steps):
        f, s_, _, threads = fp8_oracle_sample(heads=1)
        flops += f
        secs += s_
    value = flops / secs / 1e12
    line = {"impl": "reference", "metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": fp8_config(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"fp64 CPU oracle (FP8 steps), 1 head of sequence 0 of {WORKLOAD}, both "
                                       "masks, per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fp8(args, rank, world, local_rank):
    import io_aware_exact_qk_b200 as attn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    attn.load_library()
    w = dataclasses.replace(FP8_WORKLOADS[WORKLOAD](), seed=FP8_WORKLOADS[WORKLOAD]().seed + rank)
    q, k, v, _, _ = W.make_inputs(w, with_grad=False)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    ops = attn.attn_fp8_quantize(qd, kd, vd, w.batch)
    outs = {c: (torch.empty_like(qd), torch.empty(w.hq, w.total_tokens, device=dev)) for c in (False, True)}
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    variants = [w, w.with_causal(True)]

    def step():
        for c in (False, True):
            attn.attn_fwd_fp8(*ops, batch=w.batch, scale=w.scale, causal=c, o=outs[c][0], lse=outs[c][1],
                              workspace=ws)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    flops_step = sum(x.fwd_flops() for x in variants)
    for _ in range(args.warmup):
        step()
    attn.attn_get_device_error()
    barrier()
    attn.attn_profile_collect()
    attn.attn_profile_enable(True)
    launches0 = attn.attn_launch_count()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clocks:
        barrier()
        for s_, e_ in events:
            flush.zero_()
            s_.record(stream)
            step()
            e_.record(stream)
        barrier()
    attn.attn_profile_enable(False)
    launches = attn.attn_launch_count() - launches0
    per_kernel = attn.attn_profile_collect()
    attn.attn_get_device_error()
    total_ms = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in events), world, dev)
    value = world * flops_step * args.steps / (total_ms / 1e3) / 1e12
    if args.quick:
        if rank == 0:
            print(json.dumps({"quick": True, "value": value, "unit": UNIT, "ms_per_step": total_ms / args.steps,
                              "kernels": {k_: list(v_) for k_, v_ in per_kernel.items()}, "gpu_launches": launches}))
        return
    # end to end: bf16 Q, K, V from pinned host memory, quantised and attended on the
    # device, O and LSE of both masks back to pinned host memory
    hq_, hk_, hv_ = q.pin_memory(), k.pin_memory(), v.pin_memory()
    ho = {c: (torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory(),
              torch.empty(w.hq, w.total_tokens).pin_memory()) for c in (False, True)}
    h2d = sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_))
    d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b in ho.values())
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        qd.copy_(hq_, non_blocking=True)
        kd.copy_(hk_, non_blocking=True)
        vd.copy_(hv_, non_blocking=True)
        ops = attn.attn_fp8_quantize(qd, kd, vd, w.batch)
        step()
        for c in (False, True):
            ho[c][0].copy_(outs[c][0], non_blocking=True)
            ho[c][1].copy_(outs[c][1], non_blocking=True)
    e1.record(stream)
    barrier()
    attn.attn_get_device_error()
    e2e_value = world * flops_step * args.steps / (max_over_ranks(e0.elapsed_time(e1), world, dev) / 1e3) / 1e12
    if rank != 0:
        return
    peaks = load_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]     # dense e4m3 runs at twice the bf16 rate
    dom = "fwd_fp8_sm100"
    dom_ms, dom_n = per_kernel[dom]
    achieved = flops_step * args.steps / (dom_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": fp8_peak, "unit": UNIT,
                "frac": achieved / fp8_peak, "traffic": traffic_record(dom),
                "peak_source": f"{peaks['source']} dense bf16 (burst) x 2, the nominal e4m3 / bf16 ratio",
                "flops_per_launch": flops_step * args.steps / dom_n, "mean_launch_ms": dom_ms / dom_n}
    breakdown = {k_: {"launches": n_, "total_ms": ms, "share": ms / sum(x[0] for x in per_kernel.values())}
                 for k_, (ms, n_) in sorted(per_kernel.items())}
    cpu = None
    if world == 1:
        f, s_, heads, threads = fp8_oracle_sample(budget_s=12.0)
        cpu = {"value": f / s_ / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 CPU oracle (FP8 steps), {heads} whole head(s) of sequence 0 of {WORKLOAD}, both "
                         f"masks, {s_:.1f} s"}
    line = {"metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate, bf16 O)", "data": DATA,
            "config": fp8_config(world), "pct_of_peak": value / fp8_peak, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches, "clocks": clocks.summary(), "kernels": breakdown}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="sweep_d128_n4096 (default: the gate's d=128, N=4096 point), mha2k, sweep_d<d>_n<N>, "
                         "gqa8k, varlen16, long32k; "
                         "or a split-KV decode workload: decode8k, decode_var, decode_spec4; "
                         "or the FP8 forward: fp8_mha2k")
    ap.add_argument("--quick", action="store_true",
                    help="device timing only: skip the end-to-end loop and the CPU baseline (profiling runs)")
    args = ap.parse_args()
    global WORKLOAD
    WORKLOAD = args.workload
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    decode = WORKLOAD in DECODE_WORKLOADS
    fp8 = WORKLOAD in FP8_WORKLOADS
    if args.impl == "reference":
        (run_reference_decode if decode else run_reference_fp8 if fp8 else run_reference)(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        (run_decode if decode else run_fp8 if fp8 else run_ours)(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
