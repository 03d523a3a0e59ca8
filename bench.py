"""Benchmark: branch-attention forward + backward on B200.

One step = ba_fused_fwd + ba_bwd (fused main-sequence + branch-local
attention with the in-kernel Eq. 2 merge, then dQ/dK/dV through both parts)
over one synthetic packed batch shaped like the 64K-token EAGLE-3
training-time-test workload: S = 65536 packed tokens in 16 log-normal
documents (mean 4096), a depth-3 chain branch at every main position, GQA
32/8, d = 128, bf16, R = 8 virtual zigzag ranks.

Metric: useful TFLOPS = 14 * d * P * Hq / step time, P = exact visible
(row, key) pairs per query head (forward 4 d P Hq, backward 2.5x that).
Inputs (several GB) are far larger than L2, so no flush between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1: launched under torchrun, one process per GPU, each rank runs its own
independent batch (different seed), no collective on the data path; the
reported value is the whole job's useful FLOPs / max-over-ranks time
("scaling": "weak").
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

METRIC = "branch-attn fwd+bwd useful TFLOPS at 64K tokens; % of B200 BF16 dense peak"
WORKLOAD_INDEX = 3  # the 64K-token EAGLE-3 configuration (the headline)
REFERENCE_PREFIX = 640  # tokens per reference-arm step: about 3 s of oracle time
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, nominal


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return 7919 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="ba_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: the upper half of the power draw
        pmed = statistics.median(power)
        load = [s for s, p in zip(sm, power) if p >= pmed] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def cpu_baseline(target_s: float = 15.0, prefix: int = 0):
    """Times the oracle (as it stands) on the host: full forward + backward of
    whole documents of the 64K workload, one KV group (4 query heads), adding
    documents until about ``target_s`` seconds of CPU work (``prefix`` > 0:
    only the first ``prefix`` tokens of the shortest document, a shorter
    document of the same layout).  Returns the same metric (useful TFLOPS)
    over that sample."""
    import numpy as np
    import oracle as orc
    import workloads as wl
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    cfg = wl.CONFIGS[WORKLOAD_INDEX]
    cu_t, anc_t = wl.make_layout(WORKLOAD_INDEX)
    cu = cu_t.numpy()
    anc = anc_t.numpy()
    G = cfg.Hq // cfg.Hkv
    heads = list(range(G))
    lengths = np.diff(cu)
    order = np.argsort(lengths)  # shortest documents first: bounded steps
    dt = 0.0
    done_pairs = 0
    docs = 0
    for di in order:
        s, e = int(cu[di]), int(cu[di + 1])
        if prefix > 0:
            e = min(e, s + prefix)
        a_doc = anc[(anc >= s) & (anc < e)] - s
        # one document of the workload, one KV group (G query heads), same draws' law
        sub = wl.make_custom([e - s], a_doc.tolist(), Hq=G, Hkv=1, d=cfg.d, B=cfg.B, mode=cfg.mode,
                             seed=wl.seed_of(WORKLOAD_INDEX) + int(di))
        scu = sub.cu_seqlens.numpy()
        sanc = sub.anchors.numpy()
        t0 = time.perf_counter()
        orc.forward_rows(sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb, scu, sanc, cfg.B, cfg.mode)
        orc.backward_rows(sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb, sub.do, sub.dob, scu, sanc,
                          cfg.B, cfg.mode)
        dt += time.perf_counter() - t0
        done_pairs += orc.visible_pair_count(scu, sanc, cfg.B, cfg.mode)
        docs += 1
        if dt >= target_s or prefix > 0:
            break
    flops = 14.0 * cfg.d * done_pairs * len(heads)
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle fwd+bwd (row-set form) of {docs} "
                      f"{'document prefix of ' + str(prefix) + ' tokens' if prefix else 'whole document(s)'} "
                      f"of the 64K workload's layout (shortest first), 1 KV group = {len(heads)} query "
                      f"heads, {done_pairs} visible pairs/head, {dt:.1f} s of oracle time",
            "seconds": dt}


# ---------------------------------------------------------------------------
# GPU benchmark
# ---------------------------------------------------------------------------

def workload_config(world: int, index: int = WORKLOAD_INDEX) -> dict:
    import workloads as wl
    cfg = wl.CONFIGS[index]
    return {"workload": cfg.name + ": " + cfg.description, "S": cfg.S, "ndoc": cfg.ndoc,
            "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d, "branches": cfg.n_anchors, "B": cfg.B,
            "mask": "chain" if cfg.mode == wl.CHAIN else "block", "R": cfg.R,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# DRAM traffic of one launch of a kernel on the 64K workload, from an ncu
# capture of the same kernel on the 8K configuration (dram__bytes_read.sum +
# dram__bytes_write.sum, scaled to the 64K launch by its slot count), valid
# for the kernel source it was taken on: reported only while that source file
# is unchanged.
KERNEL_TRAFFIC = {
    "bwd_dkdv": {"bytes_per_launch": 4.969e9, "source": "bwd_dkdv.cu",
                 "sha1": "7bc703feb171c6e70c556c3980a28cd32d7fbacd"},
}


def kernel_traffic(kind: str):
    import hashlib
    t = KERNEL_TRAFFIC.get(kind)
    if t is None:
        return None
    path = os.path.join(ROOT, "branch_attention_speculative_packed_b200", "csrc", t["source"])
    try:
        digest = hashlib.sha1(open(path, "rb").read()).hexdigest()
    except OSError:
        return None
    return t["bytes_per_launch"] if digest == t["sha1"] else None


def kernel_flops(kind: str, d: int, pairs: int, Hq: int) -> float:
    """Algorithmic FLOPs of one launch of a tensor-core kernel over the
    visible pairs: forward 2 GEMMs (QK^T, PV), dQ pass 3 (QK^T, dO V^T, dS K),
    dK/dV pass 4 (K Q^T, V dO^T, P^T dO, dS^T Q); 2 d FLOPs per pair and GEMM."""
    g = {"fused_fwd": 2, "bwd_dq": 3, "bwd_dkdv": 4}[kind]
    return 2.0 * g * d * pairs * Hq


def merge_bandwidth(ba, cfg, rows: int, dev, world: int, hbm_gbs: float, parts: int = 2,
                    d: int = None) -> dict:
    """HBM bandwidth of the k-way Eq. 2 merge (`ba_lse_merge`) over `rows`
    rows of the workload's head layout (head dim `d`, default the
    workload's): k fp32 partials in, bf16 O and fp32 LSE out; inputs far
    larger than L2, timed with CUDA events."""
    import torch
    d = cfg.d if d is None else d
    g = torch.Generator(device=dev).manual_seed(2024)
    o_parts = [torch.randn(rows, cfg.Hq, d, device=dev, generator=g) for _ in range(parts)]
    lse_parts = [torch.randn(cfg.Hq, rows, device=dev, generator=g) * 4.0 for _ in range(parts)]
    o = torch.empty(rows, cfg.Hq, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.Hq, rows, dtype=torch.float32, device=dev)
    for _ in range(2):
        ba.lse_merge(o_parts, lse_parts, out=(o, lse))
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = 5
    e0.record()
    for _ in range(reps):
        ba.lse_merge(o_parts, lse_parts, out=(o, lse))
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / reps, world, dev)
    nbytes = rows * cfg.Hq * (parts * (4 * d + 4) + 2 * d + 4)
    gbs = nbytes / (ms / 1e3) / 1e9
    del o_parts, lse_parts, o, lse
    return {"kernel": "lse_merge", "parts": parts, "rows": rows, "d": d, "bytes_per_launch": nbytes,
            "ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "peak_gbs": hbm_gbs,
            "frac": round(gbs / hbm_gbs, 4)}


def run_gpu(args):
    import torch
    import branch_attention_speculative_packed_b200 as ba
    import workloads as wl

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    widx = args.workload_index
    cfg = wl.CONFIGS[widx]
    # draw on the device (rank-dependent seed for weak scaling)
    cu, anc = wl.make_layout(widx)
    prob = wl._draw(cfg, wl.seed_of(widx) + rank_seed_offset(rank), cu, anc, dev, True)
    a = ba.BranchAttention(cu, anc, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, B=cfg.B, mode=cfg.mode,
                           R=cfg.R, device=dev)
    # host planning cost (cold: the library's plan cache is cleared first); later
    # calls on the same packing reuse the cached plan
    ba.clear_cache()
    host_plan_ms = {cfg.name: round(a.prepare(), 3)}
    big = wl.CONFIGS[4]
    cu_big, anc_big = wl.make_layout(4)
    host_plan_ms[big.name] = round(ba.BranchAttention(
        cu_big, anc_big, Hq=big.Hq, Hkv=big.Hkv, d=big.d, B=big.B, mode=big.mode, R=big.R,
        device="cpu").prepare(), 3)
    stats = a.plan_stats()
    P = stats["visible_pairs"]
    useful = 14.0 * cfg.d * P * cfg.Hq
    S, Nb = prob.S, prob.Nb
    o = torch.empty_like(prob.q)
    ob = torch.empty(Nb, cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.Hq, a.rows, dtype=torch.float32, device=dev)
    grads = (torch.empty_like(prob.q), torch.empty_like(prob.k), torch.empty_like(prob.v),
             torch.empty_like(prob.qb), torch.empty_like(prob.kb), torch.empty_like(prob.vb))
    stream = torch.cuda.current_stream()

    def step():
        a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, out=(o, ob, lse))
        a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse, prob.do, prob.dob,
              out=grads)

    for _ in range(args.warmup):
        step()
    ba.sync_status()
    # ------------------------------------------------------------ timed region
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ba.profile_enable(True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ba.profile_enable(False)
    clocks = sampler.stop()
    ms_local = ev0.elapsed_time(ev1)
    prof = ba.profile_collect()
    ba.sync_status()
    ms_max = max_over_ranks(ms_local, world, dev)
    ms_per_step = ms_max / args.steps
    total_useful = sum_over_ranks(useful, world, dev)
    value = total_useful * args.steps / (ms_max / 1e3) / 1e12

    # ------------------------------------------------------------ roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    per_kernel = {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches": v[1], "share": None}
                  for k, v in prof.items()}
    tot = sum(v[0] for v in prof.values()) or 1.0
    for k, v in prof.items():
        per_kernel[k]["share"] = v[0] / tot
    tensor_kernels = [k for k in ("fused_fwd", "bwd_dq", "bwd_dkdv") if k in prof]
    dom = max(tensor_kernels, key=lambda k: prof[k][0])
    dom_ms = per_kernel[dom]["ms_per_launch"]
    achieved = kernel_flops(dom, cfg.d, P, cfg.Hq) / (dom_ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    launches = sum(v[1] for v in prof.values())

    # ------------------------------------------------------------ end to end (host buffers)
    # Each step copies its inputs from pinned host memory, runs the forward and
    # backward through the public API and reads every output back to pinned
    # host memory.  Steps are pipelined the way a training loop prefetches:
    # host-to-device copies on one stream, compute on another, device-to-host
    # copies on a third, with two device buffer sets so step k+1's inputs and
    # step k-1's outputs move while step k computes.
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 6))
    e2e = None
    if e2e_steps:
        names = ("q", "k", "v", "qb", "kb", "vb", "do", "dob")
        host = {name: getattr(prob, name).cpu().pin_memory() for name in names}
        dev_in = [{name: torch.empty_like(getattr(prob, name)) for name in names} for _ in range(2)]
        dev_out = [(o, ob, lse) + grads,
                   tuple(torch.empty_like(t) for t in (o, ob, lse) + grads)]
        outs_h = [t.new_empty(t.shape, device="cpu").pin_memory() for t in dev_out[0]]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in outs_h)
        s_h2d, s_comp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {kind: [torch.cuda.Event() for _ in range(2)]
              for kind in ("in_ready", "in_free", "out_ready", "out_free")}

        def e2e_step(k: int):
            b = k % 2
            if k >= 2:
                s_h2d.wait_event(ev["in_free"][b])
            with torch.cuda.stream(s_h2d):
                for name, t in host.items():
                    dev_in[b][name].copy_(t, non_blocking=True)
            ev["in_ready"][b].record(s_h2d)
            s_comp.wait_event(ev["in_ready"][b])
            if k >= 2:
                s_comp.wait_event(ev["out_free"][b])
            x = dev_in[b]
            oo, oob, olse = dev_out[b][:3]
            with torch.cuda.stream(s_comp):
                a.fused_fwd(x["q"], x["k"], x["v"], x["qb"], x["kb"], x["vb"], out=(oo, oob, olse))
                a.bwd(x["q"], x["k"], x["v"], x["qb"], x["kb"], x["vb"], oo, oob, olse, x["do"], x["dob"],
                      out=dev_out[b][3:])
            ev["in_free"][b].record(s_comp)
            ev["out_ready"][b].record(s_comp)
            s_d2h.wait_event(ev["out_ready"][b])
            with torch.cuda.stream(s_d2h):
                for dst, src in zip(outs_h, dev_out[b]):
                    dst.copy_(src, non_blocking=True)
            ev["out_free"][b].record(s_d2h)

        for k in range(2):  # warm-up of the pipeline
            e2e_step(k)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_h2d)
        s_comp.wait_event(e0)
        s_d2h.wait_event(e0)
        for k in range(2, 2 + e2e_steps):
            e2e_step(k)
        s_d2h.wait_event(ev["out_ready"][(1 + e2e_steps) % 2])
        e1.record(s_d2h)
        torch.cuda.synchronize()
        ba.sync_status()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e_value = total_useful * e2e_steps / (e2e_ms / 1e3) / 1e12

        e2e = {"value": round(e2e_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "pipelined": "h2d / compute / d2h on three streams, two buffer sets"}
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    merge = merge_bandwidth(ba, cfg, Nb * cfg.B if Nb else S, dev, world, hbm)
    merge_d64 = merge_bandwidth(ba, cfg, Nb * cfg.B if Nb else S, dev, world, hbm, d=64)

    # The literal three-step forward of the decomposition: main component over
    # every row (fp32 partial), branch-local component, Eq. 2 merge of the
    # branch rows (k = 2) and the main rows' conversion (k = 1), against the
    # fused kernel that does all three in one pass.
    def three_step():
        om, lm = a.main_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
        obr, lbr = a.branch_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
        ba.lse_merge([om[S:], obr], [lm[:, S:], lbr],
                     out=(ob.view(-1, cfg.Hq, cfg.d), lse[:, S:]))
        ba.lse_merge([om[:S]], [lm[:, :S]], out=(o, lse[:, :S]))
    three_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(3):
        three_step()
    t1.record(stream)
    torch.cuda.synchronize()
    ba.sync_status()
    three_ms = max_over_ranks(t0.elapsed_time(t1) / 3, world, dev)

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOPS",
        "pct_of_peak": round(100.0 * value / (peak * world), 2),
        "pct_of_peak_basis": f"{peak_src} sustained cuBLAS bf16 rate, {peak} TF/s per GPU",
        "pct_of_burst_peak": round(100.0 * value / (burst * world), 2),
        "pct_of_datasheet_peak": round(100.0 * value / (DATASHEET_BF16_TFLOPS * world), 2),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(workload_config(world, widx), visible_pairs_per_head=P,
                       useful_flop_per_step=useful),
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": kernel_traffic(dom) if widx == WORKLOAD_INDEX else None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained"},
        "kernels": {k: {"ms": round(v["ms_per_launch"], 4), "launches": v["launches"],
                        "share": round(v["share"], 4)} for k, v in per_kernel.items()},
        "e2e": e2e,
        "gpu_launches": launches,
        "host_plan_ms": dict(host_plan_ms, note="cold host planning per packing; every step "
                                                "reuses the cached plan"),
        "merge": merge,
        "merge_d64": merge_d64,
        "three_step_fwd": {"ms": round(three_ms, 3), "fused_fwd_ms": round(per_kernel["fused_fwd"]["ms_per_launch"], 3),
                           "steps": "ba_main_fwd + ba_branch_fwd + ba_lse_merge (branch rows k=2, main rows k=1)"},
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline and widx == WORKLOAD_INDEX:
        try:
            result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        except Exception as e:  # keep the GPU line even if the host leg fails
            result["cpu_baseline"] = {"error": repr(e)}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, same metric and
    workload, each step a bounded sample (whole documents, one KV group)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    vals = []
    for _ in range(args.warmup):
        cpu_baseline(prefix=REFERENCE_PREFIX)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(prefix=REFERENCE_PREFIX))
    dt = time.perf_counter() - t0
    value = statistics.median(v["value"] for v in vals)
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(world),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": vals[0]["cores"],
                         "kind": "oracle", "sample": vals[0]["sample"]},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) leg, for lines of the other workloads")
    ap.add_argument("--workload", default="eagle3_64k",
                    help="configuration name (default: the 64K headline); others are parity-test "
                         "sizes, useful for small profiling captures")
    args = ap.parse_args()
    import workloads as wl
    names = [c.name for c in wl.CONFIGS]
    if args.workload not in names:
        ap.error(f"--workload must be one of {names}")
    args.workload_index = names.index(args.workload)
    if args.impl == "reference" and args.workload_index != WORKLOAD_INDEX:
        ap.error("the reference arm times the 64K headline workload only")
    if args.warmup < 3 and args.impl == "b200":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
