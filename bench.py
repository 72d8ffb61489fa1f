#!/usr/bin/env python
"""Benchmark of the KDA operator on B200 (prints one JSON line on rank 0).

Headline workload (one "step"): one kda_prefill over B=1, H=32, T=131072,
d_k=d_v=128, bf16 q/k/v, fp32 gates and state, chunk 64 -- the long-context
prefill.  Inputs are resident in HBM before timing and are larger than L2
(6.4 GB), so no flush is needed between steps.  The same run also measures:
  * "decode": the batched decode step (256 rows x 32 heads x 128 x 128 fp32
    state, 26 masked rows per step);
  * "prefill_sweep": prefill at T = 4096, 16384, 65536 (L2 flushed between
    iterations);
  * "e2e": the headline metric through the public API with pinned HOST
    buffers, host<->device copies inside the timed region;
  * "cpu_baseline": the fp64 CPU oracle on a bounded sample of the workload.

Multi-GPU (torchrun, one process per GPU): every rank runs the same workload
on its own GPU with no collective on the data path (the operator shards by
sequence and head: replicas, weak scaling); the timed region is bracketed by
barriers and the max time over ranks is reported.

``--impl reference`` times the CPU oracle instead (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA tokens/s (prefill 4k–128k, batched decode) and % of roofline on 1 B200"
PREFILL_BYTES_PER_TOKEN_HEAD = 1540          # q,k,v bf16 + log_alpha fp32 + beta + o bf16
STATE_BYTES = 128 * 128 * 4                  # one (sequence, head) fp32 state
DECODE_ACTIVE_BYTES = 2 * STATE_BYTES + 768 + 512 + 4 + 256
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# kernels one kda_prefill launches on the tensor-core path: pad/cu_seqlens pre-pass, chunk
# index, the intra kernel and the state pass; chunks of 128 / 256 add one chunk index and one
# merge kernel per doubling
LAUNCHES_PER_PREFILL = 2 + 2 * 1


def launches_per_prefill(chunk: int) -> int:
    return LAUNCHES_PER_PREFILL + {64: 0, 128: 2, 256: 4}[chunk]
PREFILL_TRAFFIC_T = 131072   # token count the recorded prefill traffic is for


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--T", type=int, default=131072)
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--no-extras", action="store_true", help="headline prefill line only")
    ap.add_argument("--only", choices=["prefill", "decode", "conv", "backward"], default=None,
                    help="time one workload only (for profiling runs)")
    ap.add_argument("--chunk", type=int, choices=[64, 128, 256], default=64,
                    help="prefill chunk size (128 / 256: 64-row items merged into chunk items)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"],
                    source="fallback")


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's source files are
    unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            e = json.load(f).get(kernel)
        if not e:
            return None
        hs = hashlib.sha256()
        for src in e.get("sources") or [e["source"]]:
            with open(os.path.join(ROOT, src), "rb") as fh:
                hs.update(fh.read())
        if hs.hexdigest()[:16] == e.get("source_hash"):
            return e.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


def prefill_traffic(T: int):
    """Recorded DRAM bytes of one prefill call, scaled from the capture's token count to T
    (inputs, items and outputs all grow in proportion to the tokens)."""
    b = recorded_traffic("prefill")
    return None if b is None else int(round(b * T / PREFILL_TRAFFIC_T))


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling (200 ms) of SM clock and throttle reasons during a region."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or parts[0] != self.uuid:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- helpers
def max_over_ranks(value: float, world: int, device=None) -> float:
    """The max of a per-rank timing over all ranks (NCCL on the GPU, gloo on the CPU)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    on_gpu = device is not None and dist.get_backend() == "nccl"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if on_gpu else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def to_dev(x, dtype, device, pin=True):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    if pin:
        t = t.pin_memory()
    return t, t.to(device, non_blocking=False)


def flush_l2(buf):
    buf.add_(1)


def prefill_setup(T, device):
    import torch
    from gated_delta_rule_148_b200 import inputs as gen
    w = gen.long_prefill(T)
    inp = gen.prefill_inputs(w)
    host, dev = {}, {}
    for key, dt in (("q", torch.bfloat16), ("k", torch.bfloat16), ("v", torch.bfloat16),
                    ("log_alpha", None), ("beta", None), ("cu_seqlens", None)):
        host[key], dev[key] = to_dev(inp[key], dt, device)
    N, H = inp["q"].shape[0], inp["q"].shape[1]
    dev["o"] = torch.empty((N, H, 128), dtype=torch.bfloat16, device=device)
    dev["fs"] = torch.empty((1, H, 128, 128), dtype=torch.float32, device=device)
    return w, inp, host, dev


def run_prefill(kda, dev, chunk=64):
    kda.prefill(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev["cu_seqlens"],
                o=dev["o"], final_state=dev["fs"], chunk=chunk)


def prefill_bytes(T, H):
    return T * H * PREFILL_BYTES_PER_TOKEN_HEAD + H * STATE_BYTES


def prefill_bytes_head_gate(T, H):
    """Same, with one fp32 gate per token and head instead of d_k of them."""
    return T * H * (PREFILL_BYTES_PER_TOKEN_HEAD - 4 * 128 + 4) + H * STATE_BYTES


def time_loop(fn, K, W, flush_buf=None):
    """K timed calls after W warm-ups; returns per-call ms (events on the current stream)."""
    import torch
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    if flush_buf is None:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(K):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / K
    tot = 0.0
    for _ in range(K):
        flush_l2(flush_buf)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        tot += s.elapsed_time(e)
    return tot / K


def cpu_baseline(inp, budget_s=10.0):
    """The fp64 oracle on the first T_s tokens (all heads) of the workload."""
    from oracle import kda_oracle as orc
    H = inp["q"].shape[1]
    cores = orc.max_threads()

    def run(Ts, nthreads=0):
        cu = np.array([0, Ts], np.int32)
        t0 = time.perf_counter()
        orc.prefill(inp["q"][:Ts], inp["k"][:Ts], inp["v"][:Ts], inp["log_alpha"][:Ts],
                    inp["beta"][:Ts], cu, nthreads=nthreads)
        return time.perf_counter() - t0
    probe = 512
    dt = run(probe)
    Ts = int(min(inp["q"].shape[0], max(probe, probe * budget_s / max(dt, 1e-3))))
    Ts = max(probe, (Ts // 512) * 512)
    dt = run(Ts)
    t1 = 256                                   # the same oracle on one core, a short prefix
    dt1 = run(t1, nthreads=1)
    return {"value": Ts / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {Ts} of {inp['q'].shape[0]} tokens, all {H} heads, fp64 "
                      f"token-by-token C oracle, {dt:.1f} s",
            "one_core": {"value": t1 / dt1, "unit": "tokens/s", "cores": 1,
                         "sample": f"first {t1} tokens, all {H} heads, {dt1:.2f} s"}}


# ---------------------------------------------------------------- reference arm
def main_reference(args, rank, world):
    if rank != 0:
        return
    from gated_delta_rule_148_b200 import inputs as gen
    from oracle import kda_oracle as orc
    w = gen.long_prefill(args.T)
    # a bounded sample of the workload per step: its first Ts tokens, all heads
    Ts_max = 8192
    inp = gen.prefill_inputs(gen.long_prefill(Ts_max))   # same seed: a prefix of the workload
    H = inp["q"].shape[1]
    per_step_budget = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    t0 = time.perf_counter()
    orc.prefill(inp["q"][:512], inp["k"][:512], inp["v"][:512], inp["log_alpha"][:512],
                inp["beta"][:512], np.array([0, 512], np.int32))
    dt = time.perf_counter() - t0
    Ts = int(min(Ts_max, max(512, 512 * per_step_budget / max(dt, 1e-3))))
    Ts = max(512, (Ts // 512) * 512)
    cu = np.array([0, Ts], np.int32)

    def step():
        orc.prefill(inp["q"][:Ts], inp["k"][:Ts], inp["v"][:Ts], inp["log_alpha"][:Ts],
                    inp["beta"][:Ts], cu)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = Ts * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": 1, "seq_len": args.T, "heads": 32,
                   "d_k": 128, "d_v": 128, "parallelism": "replicas" if args.gpus > 1 else "none",
                   "l2": "inputs larger than L2"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": orc.max_threads(),
                         "kind": "oracle",
                         "sample": f"each step: first {Ts} of {args.T} tokens, all {H} heads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def main_ours(args, rank, world, device):
    import torch
    import torch.distributed as dist
    from gated_delta_rule_148_b200 import kda
    from gated_delta_rule_148_b200 import inputs as gen

    kda.load()
    pk = peaks()
    props = torch.cuda.get_device_properties(device)
    clocks = ClockSampler("GPU-" + str(props.uuid))

    T = args.T
    C = args.chunk
    w, inp, host, dev = prefill_setup(T, device)
    H = 32
    K, W = args.steps, args.warmup
    for _ in range(W):
        run_prefill(kda, dev, C)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(K):
        run_prefill(kda, dev, C)
    e.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(s.elapsed_time(e), world, device)
    st = kda.get_device_status()
    if st != kda.KDA_OK:
        raise RuntimeError("device status after prefill: " + kda.status_string(st))
    ms_step = ms / K
    value = aggregate_rate(T, world, ms_step)
    algo_bytes = prefill_bytes(T, H)
    achieved = algo_bytes / (ms_step / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": prefill_traffic(T) if C == 64 else None,
                "peak_source": pk["source"] + " (hbm_gbs, copy bandwidth)",
                "kernel": "kda prefill (whole kda_prefill call: pre-pass, chunk index, intra and state kernels"
                          + (")" if C == 64 else ", chunk-item merges)"),
                "algorithmic_bytes_per_launch": algo_bytes,
                "flops_bound_frac": (141013.0 * T * H / (ms_step / 1e3) / 1e12) / pk["bf16_tflops"]}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "global_batch": 1, "seq_len": T, "heads": H,
                       "d_k": 128, "d_v": 128, "chunk": C, "state": "fp32",
                       "parallelism": f"replicas{world}" if world > 1 else "none",
                       "l2": f"inputs larger than L2 ({algo_bytes / 1e9:.2f} GB per step), no flush"},
            "roofline": roofline, "clocks": clk, "gpu_launches": launches_per_prefill(C) * K}

    # ---- e2e through the public API with host buffers
    Ke = max(1, min(K, 3))
    o_host = torch.empty(dev["o"].shape, dtype=dev["o"].dtype).pin_memory()
    fs_host = torch.empty(dev["fs"].shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        for key in ("q", "k", "v", "log_alpha", "beta", "cu_seqlens"):
            dev[key].copy_(host[key], non_blocking=True)
        run_prefill(kda, dev, C)
        o_host.copy_(dev["o"], non_blocking=True)
        fs_host.copy_(dev["fs"], non_blocking=True)
    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(Ke):
        e2e_step()
    e2.record()
    torch.cuda.synchronize()
    ms2 = max_over_ranks(s2.elapsed_time(e2), world, device)
    h2d = sum(host[k].numel() * host[k].element_size()
              for k in ("q", "k", "v", "log_alpha", "beta", "cu_seqlens"))
    d2h = o_host.numel() * o_host.element_size() + fs_host.numel() * 4
    line["e2e"] = {"value": aggregate_rate(T, world, ms2 / Ke), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke}
    line["gpu_launches"] += launches_per_prefill(C) * Ke
    del o_host, fs_host

    if not args.no_extras:
        line["decode"] = bench_decode(args, world, device, pk)
        line["gpu_launches"] += args.decode_steps
        # ---- prefill sweep (smaller T; L2 flushed between iterations)
        sweep = {}
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        for Ts in (4096, 16384, 65536):
            if Ts >= T:
                continue
            _, _, _, dv_ = prefill_setup(Ts, device)
            mss = time_loop(lambda: run_prefill(kda, dv_, C), max(3, K), W,
                            flush_buf=flush if Ts <= 16384 else None)
            ach = prefill_bytes(Ts, H) / (mss / 1e3) / 1e9
            sweep[str(Ts)] = {"tokens_per_s": Ts / (mss / 1e3), "ms": mss,
                              "hbm_frac": ach / pk["hbm_gbs"],
                              "l2": "flushed" if Ts <= 16384 else "inputs larger than L2"}
            line["gpu_launches"] += LAUNCHES_PER_PREFILL * (max(3, K))
            del dv_
        sweep[str(T)] = {"tokens_per_s": T / (ms_step / 1e3), "ms": ms_step,
                         "hbm_frac": roofline["frac"], "l2": "inputs larger than L2"}
        line["prefill_sweep"] = sweep
        del flush
        # ---- head-wise gate (one decay per token and head), same q, k, v, beta
        devh = dict(dev, log_alpha=torch.from_numpy(gen.head_gates(w.seed, T, H)).to(device))
        msh = time_loop(lambda: run_prefill(kda, devh, C), K, W)
        hb = prefill_bytes_head_gate(T, H)
        line["prefill_head_gate"] = {
            "tokens_per_s": aggregate_rate(T, world, msh), "ms": msh,
            "hbm_frac": hb / (msh / 1e3) / 1e9 / pk["hbm_gbs"], "algorithmic_bytes": hb,
            "log_alpha": "[N, H] fp32", "l2": "inputs larger than L2"}
        line["gpu_launches"] += LAUNCHES_PER_PREFILL * K
        del devh
        # ---- chunk 64 / 128 / 256 on the tensor-core path, the headline workload
        line["prefill_chunk_sweep_tc"] = bench_chunk_sweep_tc(kda, dev, T, H, K, W, pk, ms_step, C)
        line["gpu_launches"] += sum(launches_per_prefill(c) * K for c in (64, 128, 256) if c != C)
        # ---- chunk-size sweep on the path that takes every chunk size (CUDA cores, fp32 q/k/v)
        line["prefill_chunk_sweep"] = bench_chunk_sweep(K, W, device)
        line["gpu_launches"] += 2 * 3 * K
        # ---- backward pass at T = 4096 (blockwise, fp32 CUDA cores)
        line["backward"] = bench_backward(K, W, world, device, pk)
        line["gpu_launches"] += 5 * max(1, K // 2)
        # ---- short convolution of q, k and v (D = H * d = 4096 each, W = 4, bf16, carried state)
        line["short_conv"] = bench_conv(K, W, world, device, pk,
                                        [dev[key].view(T, H * 128) for key in ("q", "k", "v")], w.seed)
        line["gpu_launches"] += 2 * 3 * K

    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(inp)
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_chunk_sweep_tc(kda, dev, T, H, K, W, pk, ms_headline, C_headline):
    """The headline prefill (bf16, B=1, H=32, d=128) at chunk 64, 128 and 256 on the
    tensor-core path: 128 / 256 merge the 64-row items into chunk items (one or two extra
    passes over the items) and halve / quarter the serial steps of the state pass."""
    out = {"workload": f"prefill_T{T}_H{H}_d128_bf16", "path": "tensor cores (tcgen05)",
           "l2": "inputs larger than L2"}
    for c in (64, 128, 256):
        ms = ms_headline if c == C_headline else time_loop(lambda: run_prefill(kda, dev, c), K, W)
        ach = prefill_bytes(T, H) / (ms / 1e3) / 1e9
        out[str(c)] = {"ms": ms, "tokens_per_s": T / (ms / 1e3), "hbm_frac": ach / pk["hbm_gbs"],
                       "state_steps_per_sequence": -(-T // c)}
    st = kda.get_device_status()
    if st != kda.KDA_OK:
        raise RuntimeError("device status after the tensor-core chunk sweep: " + kda.status_string(st))
    return out


def bench_chunk_sweep(K, W, device, T=16384):
    """kda_prefill with fp32 q, k, v (the CUDA-core path) at chunk 16, 32 and 64: B=1, H=32,
    d=128, the headline workload's first T tokens.  Per-call ms; the tensor-core path's bf16
    chunk-64 call at the same T is the prefill_sweep entry."""
    import torch
    from gated_delta_rule_148_b200 import kda
    _, _, _, d = prefill_setup(T, device)
    for key in ("q", "k", "v"):
        d[key] = d[key].float()
    d["o"] = torch.empty(d["o"].shape, dtype=torch.float32, device=device)
    out = {"workload": f"prefill_T{T}_H32_d128_f32_simt", "path": "CUDA cores (fp32 FMA)"}
    for c in (16, 32, 64):
        fn = lambda: kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                 d["cu_seqlens"], o=d["o"], final_state=d["fs"], chunk=c)
        ms = time_loop(fn, K, W)
        out[str(c)] = {"ms": ms, "tokens_per_s": T / (ms / 1e3)}
    st = kda.get_device_status()
    if st != kda.KDA_OK:
        raise RuntimeError("device status after the chunk sweep: " + kda.status_string(st))
    return out


def bench_decode(args, world, device, pk):
    """Batched decode: 256 rows x 32 heads, 26 masked rows per step; per-step time."""
    import torch
    import torch.distributed as dist
    from gated_delta_rule_148_b200 import kda
    from gated_delta_rule_148_b200 import inputs as gen
    W = args.warmup
    if True:
        wd = gen.batched_decode()
        state = torch.from_numpy(gen.decode_state(wd)).to(device)
        pool = []
        for t in gen.decode_pool(wd):
            pool.append({k: torch.from_numpy(t[k]).to(device).to(torch.bfloat16)
                         if k in ("q", "k", "v") else torch.from_numpy(t[k]).to(device)
                         for k in ("q", "k", "v", "log_alpha", "beta")})
        Dsteps = args.decode_steps
        masks = torch.from_numpy(np.stack([gen.decode_mask(wd, i) for i in range(Dsteps + W)])
                                 ).to(device)
        o_dec = torch.empty((wd.decode_rows, wd.H, wd.dv), dtype=torch.bfloat16, device=device)
        it = [0]

        def dstep():
            i = it[0]
            d = pool[i % len(pool)]
            kda.decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state, mask=masks[i],
                       o=o_dec)
            it[0] += 1
        dms = max_over_ranks(time_loop(dstep, Dsteps, W), world, device)
        active = wd.decode_rows - wd.decode_masked
        dbytes = (active * wd.H * DECODE_ACTIVE_BYTES + wd.decode_masked * wd.H * 256
                  + wd.decode_rows)
        dach = dbytes / (dms / 1e3) / 1e9
        return {
            "workload": wd.name, "value": aggregate_rate(active, world, dms), "unit": "tokens/s",
            "us_per_step": dms * 1e3, "steps": Dsteps,
            "roofline": {"bound": "hbm", "achieved": dach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": dach / pk["hbm_gbs"], "traffic": recorded_traffic("decode"),
                         "algorithmic_bytes_per_launch": dbytes}}


def bench_backward(K, W, world, device, pk, T=4096):
    """kda_prefill_backward on one sequence of T tokens, H = 32, d = 128, bf16 inputs, fp32
    gradients (all of them, including the initial state's)."""
    import torch
    from gated_delta_rule_148_b200 import inputs as gen
    from gated_delta_rule_148_b200 import kda
    w = gen.prefill(T)
    inp = gen.prefill_inputs(w)
    H = inp["q"].shape[1]
    d = {key: torch.from_numpy(inp[key]).to(device) for key in ("log_alpha", "beta", "cu_seqlens")}
    for key in ("q", "k", "v"):
        d[key] = torch.from_numpy(inp[key]).to(device).to(torch.bfloat16)
    go = torch.from_numpy(gen.grad_outputs(w.seed, T, H, 128)).to(device)
    s0 = torch.zeros((1, H, 128, 128), dtype=torch.float32, device=device)
    ws = torch.empty(kda.prefill_backward_workspace_bytes(T, 1, H, 128, 128), dtype=torch.uint8, device=device)

    def step():
        kda.prefill_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], go,
                             init_state=s0, workspace=ws)
    ms = max_over_ranks(time_loop(step, max(1, K // 2), max(1, W // 2)), world, device)
    if kda.get_device_status() != kda.KDA_OK:
        raise RuntimeError("device status after the backward pass")
    # inputs q, k, v (bf16), log_alpha, beta, grad_o; outputs dq, dk, dv, dlog_alpha, dbeta (fp32)
    per = 3 * 256 + 512 + 4 + 512 + 3 * 512 + 512 + 4
    nb = T * H * per + 2 * H * 128 * 128 * 4
    return {"workload": f"prefill_backward_T{T}_H{H}_d128_bf16_inputs", "tokens_per_s": aggregate_rate(T, world, ms),
            "ms": ms, "algorithmic_bytes": nb,
            "roofline": {"bound": "hbm", "achieved": nb / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": nb / (ms / 1e3) / 1e9 / pk["hbm_gbs"]},
            "note": "blockwise backward (chunks of 64), fp32 accuracy: dense products in 3xTF32 on tensor cores, the rest on CUDA cores; its workspace traffic (chunk "
                    "quantities, states at chunk starts and ends) is not algorithmic bytes"}


def bench_conv(K, W, world, device, pk, xs, seed):
    """One layer's short convolutions: kda_short_conv over each [T, D] input of xs (q, k
    and v), width 4, bf16, the carried state updated in place; K timed steps after W."""
    import torch
    from gated_delta_rule_148_b200 import inputs as gen
    from gated_delta_rule_148_b200 import kda
    T, D = xs[0].shape
    cw = gen.conv_inputs(seed, [0], D, 4)
    cwt, cbias = torch.from_numpy(cw["weight"]).to(device), torch.from_numpy(cw["bias"]).to(device)
    cst = torch.from_numpy(cw["state"]).to(device)
    cu1 = torch.tensor([0, T], dtype=torch.int32, device=device)
    ys = [torch.empty((T, D), dtype=torch.bfloat16, device=device) for _ in xs]

    def conv_step():
        for x, y in zip(xs, ys):
            kda.short_conv(x, cwt, cu1, bias=cbias, state_in=cst, state_out=cst, y=y)
    ms = max_over_ranks(time_loop(conv_step, K, W), world, device)
    if kda.get_device_status() != kda.KDA_OK:
        raise RuntimeError("device status after the short convolution")
    nb = len(xs) * (2 * T * D * 2 + 2 * 3 * D * 4 + D * 5 * 4)
    tr = recorded_traffic("short_conv")     # recorded for 3 calls at T = 131072, D = 4096
    if tr is not None:
        tr = int(round(tr * (len(xs) / 3) * (T / 131072) * (D / 4096)))
    return {"workload": f"short_conv_{len(xs)}x_T{T}_D{D}_W4_bf16",
            "tokens_per_s": aggregate_rate(T, world, ms), "ms": ms,
            "roofline": {"bound": "hbm", "achieved": nb / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": nb / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                         "traffic": tr, "algorithmic_bytes_per_step": nb}}


def main_conv_only(args, rank, world, device):
    import torch
    from gated_delta_rule_148_b200 import inputs as gen
    from gated_delta_rule_148_b200 import kda
    kda.load()
    c = gen.conv_inputs(gen.SEED_BASE + 5, [args.T], 4096, 4)
    x = torch.from_numpy(c["x"]).to(device).to(torch.bfloat16)
    d = bench_conv(args.steps, args.warmup, world, device, peaks(), [x, x, x], gen.SEED_BASE + 5)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "short_conv": d}), flush=True)


def main_decode_only(args, rank, world, device):
    from gated_delta_rule_148_b200 import kda
    kda.load()
    d = bench_decode(args, world, device, peaks())
    if rank == 0:
        print(json.dumps({"metric": METRIC, "decode": d}), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        main_reference(args, rank, world)
        return
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    try:
        if args.only == "decode":
            main_decode_only(args, rank, world, device)
        elif args.only == "conv":
            main_conv_only(args, rank, world, device)
        elif args.only == "backward":
            from gated_delta_rule_148_b200 import kda
            kda.load()
            d = bench_backward(args.steps, args.warmup, world, device, peaks(), T=min(args.T, 4096))
            if rank == 0:
                print(json.dumps({"metric": METRIC, "backward": d}), flush=True)
        else:
            if args.only == "prefill":
                args.no_extras = True
            main_ours(args, rank, world, device)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
