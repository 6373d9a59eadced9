#!/usr/bin/env python
"""Benchmark of the MoE indirect expert matmul on B200.

Workload (one step): a DeepSeek-V3-shaped routed expert layer, moe_ffn =
row-id pass + gate/up grouped GEMM with SwiGLU + down grouped GEMM with the
scatter to dst; 256 experts, top-8, n_embd 7168, expert ffn 2048, Q8_0
weights (~12 GB), 4096 bf16 tokens per GPU, routing = top-8 of N(0,1) logits
plus a per-expert N(0, 0.5) bias.  Synthetic, seeded inputs (workloads/).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own 4096-token batch with replicated
weights (weak scaling, no data-path collective); the step time is the max
over ranks.  Rank 0 prints one JSON line.  Also reported: the decode step
(T = 1, 4, 8 tokens, 256 experts top-8 + a shared expert, n_embd 2048, ffn
512) as HBM bandwidth, an end-to-end number through host buffers, the
roofline of the dominant kernel, and the CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))

# dram__bytes_read.sum + dram__bytes_write.sum of one V3 gate/up launch: an ncu
# capture of the 32-expert, 512-token case (same per-expert load) times 8.  It
# describes only the kernel sources it was measured on; when any of them changes
# the bench reports null.
GATE_UP_TRAFFIC = {
    "bytes_per_launch": 8 * (1103071744 + 16093952),
    "sources_sha256": {
        "gemm.cu": "0f45022495884171e0c42baa41e71df067b38acdd9509998740b830204d1e398",
        "gemm_api.cuh": "dd7bf3b03c707a7676aafa55f8e79562e44196a9042c9cbac6d70b1f1cb10cfb",
        "common.cuh": "79d6480bd268349c0de107f1d8d81c039fdfe2f08bf55125faebb8ecc9e51fcf",
        "ptx.cuh": "d9acdcaedb2ed563aa9944e8157f2b6fc5664b3a6120c45702c1b8dddf90bc22",
    },
}


def gate_up_traffic():
    """The recorded traffic if the GEMM sources still match the capture, else None."""
    import hashlib
    for name, digest in GATE_UP_TRAFFIC["sources_sha256"].items():
        path = os.path.join(ROOT, "indirect_expert_matmul_b200", "csrc", name)
        try:
            with open(path, "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return GATE_UP_TRAFFIC["bytes_per_launch"]
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "mul_mat_id tokens/s at pp4096 (V3 shape)"
WL = workloads.WORKLOADS["v3"]
DEC = workloads.WORKLOADS["decode"]
Q8_BYTES_PER_W = 34.0 / 32.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU while running:
    read-only NVML queries every few milliseconds from a background thread
    (the timed region can be only tens of milliseconds), else nvidia-smi
    writing into a temporary file that is removed afterwards."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                   ("hw_thermal_slowdown", 0x40))

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.nv = None
        self.samples = []  # (sm MHz, reason bits)
        self.smax = None
        self.path = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self):
        nv, h = self.nv, self.h
        while not self.stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                break
            self.stop.wait(0.004)

    def __enter__(self):
        import threading
        try:
            self.nv, self.h = self._nvml_handle()
            self.smax = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.002)
            return self
        except Exception:
            self.nv = None
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"clocks_gpu{self.gpu}_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.nv is not None:
            self.stop.set()
            self.thread.join(timeout=2)
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.nv is not None:
            sm = [float(x) for x, _ in self.samples]
            reasons = sorted({nm for _, bits in self.samples for nm, b in self.REASON_BITS if bits & b})
            smax = float(self.smax) if self.smax else None
            load = [x for x in sm if smax and x > 0.3 * smax] or sm
            return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                    "reasons": reasons, "samples": len(sm), "source": "nvml"}
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()
        try:
            os.unlink(self.path)
        except OSError:
            pass
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        load = [s for s in sm if smax and s > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


# ------------------------------------------------------------ CPU baseline
def cpu_baseline(budget_s: float = 12.0, t0: int = 0):
    """The oracle as it stands on a bounded sample of the V3 layer: routed FFN
    rows of sampled slots (one expert's weights regenerated per sampled slot)."""
    import oracle

    T = WL.n_tokens[0]
    ids = WL.ids(T, t0=t0)
    x = WL.x(T, t0=t0)
    flat = ids.reshape(-1)
    rng = np.random.default_rng(1)
    order = rng.permutation(len(flat))
    # all host cores, whatever a launcher set OMP_NUM_THREADS to; report the threads used
    oracle.set_num_threads(len(os.sched_getaffinity(0)))
    cores = oracle.num_threads()
    done, elapsed, i = 0, 0.0, 0
    while elapsed < budget_s and i < len(order):
        batch = order[i:i + cores]
        i += len(batch)
        es = set(int(flat[s]) for s in batch)
        # the oracle checks k <= n_experts: a small batch may touch fewer than k
        # experts, so pad the set with unused ones (their rows are never computed)
        pad = (e for e in range(WL.n_experts) if e not in es)
        while len(es) < WL.k:
            es.add(next(pad))
        es = sorted(es)
        remap = {e: j for j, e in enumerate(es)}
        Wg = np.concatenate([workloads.q8_0_weights_experts(e, 1, WL.n_out, WL.n_in, WL.seed, workloads.T_WG)
                             for e in es])
        Wu = np.concatenate([workloads.q8_0_weights_experts(e, 1, WL.n_out, WL.n_in, WL.seed, workloads.T_WU)
                             for e in es])
        Wd = np.concatenate([workloads.q8_0_weights_experts(e, 1, WL.n_in, WL.n_out, WL.seed, workloads.T_WD)
                             for e in es])
        sub_ids = np.vectorize(lambda e: remap.get(int(e), 0))(ids).astype(np.int32)
        t = time.perf_counter()
        oracle.ffn(Wg, Wu, Wd, x, "bf16", sub_ids, slots=np.asarray(batch, np.int64))
        elapsed += time.perf_counter() - t
        done += len(batch)
    tok_s = (done / WL.k) / elapsed
    return {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of {T * WL.k} (token, slot) rows of the V3 moe_ffn (fp64 oracle, "
                      f"{elapsed:.1f} s), scaled to tokens/s at k={WL.k}"}


# ------------------------------------------------------------------ GPU arm
def upload_prepared(moe, torch, n_experts, n_out, n_in, tensor, seed=0, chunk=16):
    """Generate a stacked Q8_0 matrix in expert chunks and repack it on the GPU."""
    per_expert = moe.weights_prepared_size(1, n_out, n_in)
    out = torch.empty(per_expert * n_experts, dtype=torch.uint8, device="cuda")
    for e0 in range(0, n_experts, chunk):
        n_e = min(chunk, n_experts - e0)
        q = workloads.q8_0_weights_experts(e0, n_e, n_out, n_in, seed, tensor)
        raw = torch.from_numpy(q).cuda()
        moe.weights_prepare(raw, n_e, n_out, n_in, out=out[e0 * per_expert:(e0 + n_e) * per_expert])
        del raw
    return out


def bf16_dev(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def touched_ffn_bytes(ids, n_experts, n_embd, n_ff):
    used = np.unique(ids.reshape(-1)).size
    return used, used * 3 * n_embd * n_ff * Q8_BYTES_PER_W


def run_ours(args):
    import torch

    import indirect_expert_matmul_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    hbm_peak, tc_peak, tc_sust, peak_src = load_peaks()

    E, k, n_embd, n_ff, T = WL.n_experts, WL.k, WL.n_in, WL.n_out, WL.n_tokens[0]
    small = args.experts is not None or args.tokens is not None
    if args.experts is not None:
        E = args.experts
    if args.tokens is not None:
        T = args.tokens
    S = T * k
    from indirect_expert_matmul_b200.dist import max_over_ranks, token_shard
    t0, _ = token_shard(T * world, rank, world)  # each rank its own batch of T tokens
    Wg = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WG)
    Wu = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WU)
    Wd = upload_prepared(moe, torch, E, n_embd, n_ff, workloads.T_WD)
    ids_np = workloads.routing(WL.routing, T, E, k, WL.seed, t0=t0, bias_sigma=WL.bias_sigma) if small \
        else WL.ids(T, t0=t0)
    x_np = WL.x(T, t0=t0)
    x = bf16_dev(torch, x_np)
    ids = torch.from_numpy(ids_np).cuda()
    ws = moe.workspace(T, k, E, n_embd, n_ff, 0, torch.bfloat16)
    dst = torch.empty((T, k, n_embd), dtype=torch.float32, device="cuda")

    def step():
        moe.ffn(Wg, Wu, Wd, E, n_embd, n_ff, x, ids, ws=ws, out=dst)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = moe.get_status(ws)
    if st != moe.OK:
        raise RuntimeError(f"device status after warm-up: {moe.status_string(st)}")

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- timed region (device, resident inputs)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        moe.profile_enable(True)
        ev0.record()
        for _ in range(args.steps):
            step()
        ev1.record()
        torch.cuda.synchronize()
        moe.profile_enable(False)
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    stages = moe.profile_read()
    st = moe.get_status(ws)
    if st != moe.OK:
        raise RuntimeError(f"device status after timed run: {moe.status_string(st)}")
    ms = max_over_ranks(ms, device="cuda")

    # algorithmic work of one step
    used, w_bytes = touched_ffn_bytes(ids_np, E, n_embd, n_ff)
    x_bytes = T * n_embd * 2
    h_bytes = S * n_ff * 2
    dst_bytes = S * n_embd * 4
    step_bytes = w_bytes + x_bytes + 2 * h_bytes + dst_bytes
    step_flops = 2.0 * S * n_embd * n_ff * 3
    gu_bytes = w_bytes * 2 / 3 + x_bytes + h_bytes
    gu_flops = 2.0 * S * n_embd * n_ff * 2
    n_gu, ms_gu = stages.get("gemm_gate_up", (0, float("nan")))
    t_gu = ms_gu / max(n_gu, 1) * 1e-3
    gu_gbs = gu_bytes / t_gu / 1e9
    gu_tflops = gu_flops / t_gu / 1e12
    bound = "hbm" if gu_bytes / (hbm_peak * 1e9) >= gu_flops / (tc_peak * 1e12) else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": round(gu_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(gu_gbs / hbm_peak, 4)}
    else:
        roof = {"bound": "tensor", "achieved": round(gu_tflops, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "frac": round(gu_tflops / tc_peak, 4)}
    traffic = None if small else gate_up_traffic()
    roof.update({"traffic": traffic, "kernel": "grouped_gemm_kernel<1> (gate/up + SwiGLU)",
                 "peak_source": peak_src, "ms_per_launch": round(t_gu * 1e3, 4),
                 "tensor_tflops": round(gu_tflops, 1), "tensor_frac": round(gu_tflops / tc_peak, 4),
                 "algorithmic_bytes": int(gu_bytes), "flops": gu_flops})
    step_roof_ms = max(step_bytes / (hbm_peak * 1e9), step_flops / (tc_peak * 1e12)) * 1e3
    launches_per_step = sum(n for n, _ in stages.values()) / args.steps

    result = {
        "metric": METRIC, "value": round(T * world / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16+bf16", "data": "synthetic",
        "config": {"workload": ("v3 moe_ffn: 256 experts top-8, n_embd 7168, expert ffn 2048, Q8_0 gate/up/down, "
                                "bf16 x, 4096 tokens per GPU, biased top-8 routing") if not small else
                               f"profiling case (not a bench line): v3 shape with {E} experts, {T} tokens",
                   "arithmetic": "gate/up: fp16 operands (activation rows scaled by exact powers of two), "
                                 "down: bf16 operands; Q8_0 dequantised exactly then rounded once; fp32 accumulation",
                   "tokens_per_gpu": T, "experts_touched": int(used),
                   "l2": "inputs larger than L2 (12 GB of weights per step)", "parallelism": f"dp{world}"},
        "tflops": round(step_flops * world / (ms * 1e-3) / 1e12, 1),
        "step_roofline": {"ms": round(step_roof_ms, 4), "frac": round(step_roof_ms / ms, 4),
                          "bytes": int(step_bytes), "flops": step_flops},
        "stages_ms_per_step": {k_: round(v[1] / args.steps, 4) for k_, v in stages.items()},
        "roofline": roof,
        "gpu_launches": int(round(launches_per_step * args.steps)),
    }
    result["clocks"] = clk.summary()

    # ---- end to end through host buffers (pinned), same metric
    if not args.no_e2e:
        x_pin = torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).pin_memory()
        ids_pin = torch.from_numpy(ids_np).pin_memory()
        dst_pin = torch.empty((T, k, n_embd), dtype=torch.float32).pin_memory()

        def e2e_step():
            x.copy_(x_pin, non_blocking=True)
            ids.copy_(ids_pin, non_blocking=True)
            moe.ffn(Wg, Wu, Wd, E, n_embd, n_ff, x, ids, ws=ws, out=dst)
            dst_pin.copy_(dst, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        ev0.record()
        n_e2e = max(2, min(args.steps, 5))
        for _ in range(n_e2e):
            e2e_step()
        ev1.record()
        torch.cuda.synchronize()
        barrier()
        ms_e2e = ev0.elapsed_time(ev1) / n_e2e
        ms_e2e = max_over_ranks(ms_e2e, device="cuda")
        result["e2e"] = {"value": round(T * world / (ms_e2e * 1e-3), 1), "unit": "tokens/s",
                         "h2d_bytes_per_step": int(x_bytes + ids_np.nbytes), "d2h_bytes_per_step": int(dst_bytes),
                         "ms_per_step": round(ms_e2e, 3)}
        del x_pin, dst_pin

    # ---- the weighted combine that follows the path (its own kernel, timed alone):
    # y[t] = sum_s r[t][s] * dst[t][s] over this step's output, HBM-bound
    if not args.no_combine:
        r_dev = torch.from_numpy(workloads.router_weights(T, k, WL.seed)).cuda()
        y = torch.empty((T, n_embd), dtype=torch.float32, device="cuda")
        for _ in range(3):
            moe.combine(dst, r_dev, out=y)
        torch.cuda.synchronize()
        n_c = 10
        ev0.record()
        for _ in range(n_c):
            moe.combine(dst, r_dev, out=y)
        ev1.record()
        torch.cuda.synchronize()
        ms_c = max_over_ranks(ev0.elapsed_time(ev1) / n_c, device="cuda")
        c_bytes = dst_bytes + S * 4 + T * n_embd * 4
        c_gbs = c_bytes / (ms_c * 1e-3) / 1e9
        result["combine"] = {"ms": round(ms_c, 4), "GB/s": round(c_gbs, 1), "frac_of_hbm": round(c_gbs / hbm_peak, 4),
                             "algorithmic_bytes": int(c_bytes), "kernel": "combine_kernel",
                             "config": f"dst [{T}][{k}][{n_embd}] fp32 of this step, router weights, no shared "
                                       "expert; inputs larger than L2"}
        del y, r_dev

    # ---- the router that precedes the path (its own kernel, timed alone): top-k of
    # logit + bias over the experts and softmax weights, at the V3 routing shape
    if not args.no_combine:
        logits = torch.from_numpy(workloads.activations(T, E, "f32", WL.seed, 51)).cuda()
        bias_e = torch.from_numpy((workloads.activations(1, E, "f32", WL.seed, 52)[0] * 0.5).astype(np.float32)).cuda()
        r_ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
        r_w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        for _ in range(3):
            moe.route(logits, k, bias_e, True, ids=r_ids, weights=r_w)
        torch.cuda.synchronize()
        # one launch is a few microseconds: replay them from a CUDA graph so that host
        # launch overhead is not what is timed
        n_r = 20
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(n_r):
                moe.route(logits, k, bias_e, True, ids=r_ids, weights=r_w)
        graph.replay()
        torch.cuda.synchronize()
        ev0.record()
        graph.replay()
        ev1.record()
        torch.cuda.synchronize()
        us_r = max_over_ranks(ev0.elapsed_time(ev1) / n_r, device="cuda") * 1e3
        del graph
        r_bytes = T * E * 4 + E * 4 + T * k * 8
        result["route"] = {"us": round(us_r, 2), "GB/s": round(r_bytes / (us_r * 1e-6) / 1e9, 1),
                           "frac_of_hbm": round(r_bytes / (us_r * 1e-6) / 1e9 / hbm_peak, 4),
                           "algorithmic_bytes": int(r_bytes), "kernel": "route_kernel",
                           "config": f"logits [{T}][{E}] fp32 + bias, top-{k}, softmax weights renormalised; "
                                     f"{n_r} launches replayed from one CUDA graph"}
        del logits, bias_e, r_ids, r_w

    del Wg, Wu, Wd
    torch.cuda.empty_cache()
    if not args.no_decode:
        result["decode"] = run_decode(moe, torch, args, hbm_peak)
        result["decode_noalloc"] = run_decode(moe, torch, args, hbm_peak, noalloc=True)
    if not args.no_report:
        result["lite"] = run_lite(moe, torch, hbm_peak, tc_peak)
        result["skew"] = run_skew(moe, torch, hbm_peak, tc_peak)

    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def _roof(bytes_, flops, ms, hbm_peak, tc_peak):
    """Roofline of one timed unit: the slower of its algorithmic bytes at the
    HBM peak and its flops at the tensor peak, against the measured time."""
    t_b, t_f = bytes_ / (hbm_peak * 1e9), flops / (tc_peak * 1e12)
    return {"bound": "hbm" if t_b >= t_f else "tensor", "roofline_ms": round(max(t_b, t_f) * 1e3, 4),
            "frac": round(max(t_b, t_f) * 1e3 / ms, 4), "GB/s": round(bytes_ / (ms * 1e-3) / 1e9, 1),
            "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1), "algorithmic_bytes": int(bytes_), "flops": flops}


def _time_calls(torch, fn, reps=20, warm=3):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_lite(moe, torch, hbm_peak, tc_peak):
    """DeepSeek-Lite-shaped expert FFN: one moe_ffn on 512 tokens (64 experts,
    top-6, 2048 -> 1408 -> 2048, uniform routing); weights 588 MB, beyond L2."""
    wl = workloads.WORKLOADS["lite"]
    E, k, n_embd, n_ff, T = wl.n_experts, wl.k, wl.n_in, wl.n_out, wl.n_tokens[0]
    Wg = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WG)
    Wu = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WU)
    Wd = upload_prepared(moe, torch, E, n_embd, n_ff, workloads.T_WD)
    ids_np = wl.ids(T)
    x, ids = bf16_dev(torch, wl.x(T)), torch.from_numpy(ids_np).cuda()
    ws = moe.workspace(T, k, E, n_embd, n_ff, 0, torch.bfloat16)
    dst = torch.empty((T, k, n_embd), dtype=torch.float32, device="cuda")
    ms = _time_calls(torch, lambda: moe.ffn(Wg, Wu, Wd, E, n_embd, n_ff, x, ids, ws=ws, out=dst))
    if moe.get_status(ws) != moe.OK:
        raise RuntimeError("lite: device status")
    used, w_bytes = touched_ffn_bytes(ids_np, E, n_embd, n_ff)
    S = T * k
    b = w_bytes + T * n_embd * 2 + 2 * S * n_ff * 2 + S * n_embd * 4
    out = {"ms": round(ms, 4), "tokens/s": round(T / (ms * 1e-3), 1), "experts_touched": int(used),
           **_roof(b, 2.0 * S * n_embd * n_ff * 3, ms, hbm_peak, tc_peak),
           "config": "moe_ffn, 64 experts top-6, 2048 -> 1408 -> 2048, Q8_0, bf16 x, 512 tokens, uniform routing; "
                     "20 calls between CUDA events after 3 warm-up calls; weights beyond L2"}
    del Wg, Wu, Wd
    torch.cuda.empty_cache()
    return out


def _gemm_balance(counts, n_out, sms, bn=192, tile_m=128):
    """The persistent GEMM's schedule for one mul_mat_id (tiles walked in (expert,
    column tile, row unit) order, tile t on CTA t mod grid): per CTA the tiles and
    the token columns (rounded to 16) it multiplies - where the 0-token and the
    heavy experts of the skewed routing land."""
    cols = []
    for c in counts:
        while c > 0:
            cols.append(min(c, bn))
            c -= bn
    units = ((n_out + 15) // 16 * 16 + tile_m - 1) // tile_m
    units = (units + 1) // 2  # two 128-row tiles per row unit (single matrix)
    work = [int((n + 15) // 16 * 16) for n in cols for _ in range(units)]
    grid = min(sms, len(work)) if work else 1
    per_tiles = [len(work[i::grid]) for i in range(grid)]
    per_cols = [sum(work[i::grid]) for i in range(grid)]
    mean = sum(per_cols) / grid
    return {"tiles": len(work), "grid": grid, "tiles_per_cta": [int(min(per_tiles)), int(max(per_tiles))],
            "columns_per_cta": {"min": int(min(per_cols)), "max": int(max(per_cols)), "mean": round(float(mean), 1)},
            "max_over_mean": round(float(max(per_cols) / mean), 4) if mean else None,
            "experts_empty": int(sum(1 for c in counts if c == 0)), "largest_expert_tokens": int(max(counts))}


def run_skew(moe, torch, hbm_peak, tc_peak):
    """Skewed-load stress: moe_mul_mat_id on 8192 tokens (128 experts, top-4 Zipf
    popularity with 8 empty experts, 2880 x 2880), broadcast and per_slot."""
    wl = workloads.WORKLOADS["skew"]
    E, k, n_in, n_out, T = wl.n_experts, wl.k, wl.n_in, wl.n_out, wl.n_tokens[0]
    W = upload_prepared(moe, torch, E, n_out, n_in, workloads.T_W)
    ids_np = wl.ids(T)
    ids = torch.from_numpy(ids_np).cuda()
    counts = np.bincount(ids_np.reshape(-1), minlength=E)
    used = int((counts > 0).sum())
    S = T * k
    dst = torch.empty((T, k, n_out), dtype=torch.float32, device="cuda")
    ws = moe.workspace(T, k, E, n_in, x_dtype=torch.bfloat16)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = {"balance": _gemm_balance(counts, n_out, sms)}
    for mode in ("broadcast", "per_slot"):
        x = bf16_dev(torch, wl.x(T, mode=mode))
        ms = _time_calls(torch, lambda: moe.mul_mat_id(W, E, n_out, n_in, x, ids, mode, ws=ws, out=dst))
        if moe.get_status(ws) != moe.OK:
            raise RuntimeError("skew: device status")
        b = used * n_out * n_in * Q8_BYTES_PER_W + x.numel() * 2 + S * n_out * 4
        out[mode] = {"ms": round(ms, 4), "tokens/s": round(T / (ms * 1e-3), 1),
                     **_roof(b, 2.0 * S * n_in * n_out, ms, hbm_peak, tc_peak)}
        del x
    out["config"] = ("moe_mul_mat_id, 128 experts top-4, Zipf(1.2) popularity (8 experts empty), 2880 x 2880, "
                     "Q8_0, bf16 x, 8192 tokens; 20 calls between CUDA events after 3 warm-up calls")
    del W
    torch.cuda.empty_cache()
    return out


def run_decode(moe, torch, args, hbm_peak, noalloc=False):
    """Decode step: n_layers distinct layer copies (beyond L2), fresh routing per
    layer, replayed as one CUDA graph per token count; through moe_ffn with a
    workspace per layer, or (noalloc) through the entry point without one."""
    E, k, n_embd, n_ff, n_sh = DEC.n_experts, DEC.k, DEC.n_in, DEC.n_out, DEC.n_ff_shared
    L = args.decode_layers
    base_g = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WG)
    base_u = upload_prepared(moe, torch, E, n_ff, n_embd, workloads.T_WU)
    base_d = upload_prepared(moe, torch, E, n_embd, n_ff, workloads.T_WD)
    sh = [upload_prepared(moe, torch, 1, n_sh, n_embd, workloads.T_SG),
          upload_prepared(moe, torch, 1, n_sh, n_embd, workloads.T_SU),
          upload_prepared(moe, torch, 1, n_embd, n_sh, workloads.T_SD)]
    layers = [(base_g, base_u, base_d)] + [(base_g.clone(), base_u.clone(), base_d.clone()) for _ in range(L - 1)]
    shared = [[t.clone() for t in sh] for _ in range(L)]
    per_expert = 3 * n_embd * n_ff * Q8_BYTES_PER_W
    per_shared = 3 * n_embd * n_sh * Q8_BYTES_PER_W
    out = {}
    for T in (DEC.n_tokens if args.decode_tokens is None else (args.decode_tokens,)):
        x = bf16_dev(torch, DEC.x(T))
        ids = [torch.from_numpy(DEC.ids(T, layer=l)).cuda() for l in range(L)]
        touched = sum(np.unique(i.cpu().numpy()).size for i in ids)
        ws = [moe.workspace(T, k, E, n_embd, n_ff, n_sh, torch.bfloat16) for _ in range(L)]
        dst = [torch.empty((T, k, n_embd), dtype=torch.float32, device="cuda") for _ in range(L)]
        dsh = [torch.empty((T, n_embd), dtype=torch.float32, device="cuda") for _ in range(L)]

        status = torch.zeros(1, dtype=torch.int32, device="cuda")

        def all_layers():
            for l in range(L):
                g, u, d = layers[l]
                if noalloc:
                    moe.ffn_decode_noalloc(g, u, d, E, n_embd, n_ff, x, ids[l], shared=(*shared[l], n_sh),
                                           out=dst[l], out_shared=dsh[l], status=status)
                else:
                    moe.ffn(g, u, d, E, n_embd, n_ff, x, ids[l], shared=(*shared[l], n_sh), ws=ws[l], out=dst[l],
                            out_shared=dsh[l])

        all_layers()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(graph, stream=s):
                all_layers()
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        ev0.record()
        for _ in range(reps):
            graph.replay()
        ev1.record()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / reps
        for w in ws:
            st = moe.get_status(w)
            if st != moe.OK:
                raise RuntimeError(f"decode T={T}: {moe.status_string(st)}")
        if noalloc and int(status.item()) != moe.OK:
            raise RuntimeError(f"decode (no workspace) T={T}: {moe.status_string(int(status.item()))}")
        bytes_step = touched * per_expert + L * per_shared
        gbs = bytes_step / (ms * 1e-3) / 1e9
        out[f"T={T}"] = {"us_per_layer": round(ms * 1e3 / L, 2), "GB/s": round(gbs, 1),
                         "frac_of_hbm": round(gbs / hbm_peak, 4), "layers": L,
                         "experts_touched_per_layer": round(touched / L, 2)}
        del graph
    del layers, shared, base_g, base_u, base_d
    torch.cuda.empty_cache()
    return out


def run_reference(args):
    """The oracle timed on the host cores on a bounded sample of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    per_step = []
    cb = None
    for _ in range(args.warmup + args.steps):
        cb = cpu_baseline(args.cpu_seconds / 4)
        per_step.append(cb["value"])
    vals = per_step[args.warmup:]
    v = statistics.median(vals)
    ms = WL.n_tokens[0] / v * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "v3 moe_ffn: 256 experts top-8, n_embd 7168, expert ffn 2048, Q8_0 gate/up/down, "
                                   "bf16 x, 4096 tokens per GPU, biased top-8 routing", "parallelism": "host"},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-combine", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-report", action="store_true", help="skip the Lite and skewed-load report keys")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--decode-layers", type=int, default=16)
    ap.add_argument("--decode-only", action="store_true", help="profiling only: the decode measurement alone")
    ap.add_argument("--decode-tokens", type=int, default=None, help="profiling only: one decode token count")
    ap.add_argument("--experts", type=int, default=None, help="profiling only: fewer experts than the V3 layer")
    ap.add_argument("--tokens", type=int, default=None, help="profiling only: tokens per GPU")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        import torch

        import indirect_expert_matmul_b200 as moe
        hbm_peak = load_peaks()[0]
        print(json.dumps({"decode": run_decode(moe, torch, args, hbm_peak),
                          "decode_noalloc": run_decode(moe, torch, args, hbm_peak, noalloc=True)}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
