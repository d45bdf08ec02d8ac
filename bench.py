#!/usr/bin/env python
"""Benchmark of the flow-matching action-expert denoise loop on B200.

One "step" of this benchmark is one whole denoise loop (N Euler steps through every DiT layer)
of one batch of synthetic inputs.  The metric is the loop time and the achieved algorithmic
HBM bandwidth: bytes = N x (streamed linear weights + B x prefix K/V); activations (<1 %) and
the input-independent adaLN table are not counted.  The VLA-Perf roofline (section 2.3 of the
VLA-Perf summary page: T = max(FLOPs / peak, bytes / bandwidth)) makes this stage HBM-bound at
batch 1.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload starvla|pi05|pi05_fp8|tiny]
  python bench.py --impl reference ...   # the CPU oracle on the host cores, same metric

Multi-GPU (torchrun, one process per GPU): independent replicas with no collective on the data
path ("scaling": "weak"); timing is per-rank CUDA events with a barrier on both sides and the
max over ranks.
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

METRIC = "action-expert denoise-loop ms and achieved HBM GB/s at batch 1 (1x B200)"
FALLBACK_HBM_GBS = 6650.0
OP_NAMES = ("qkv_rope", "attention", "o_proj_resid", "gate_up_swiglu", "down_resid")
DOMINANT_OP = 3
# the dominant kernel's source and the host code that plans its launch shape (split, ring depth)
KERNEL_SOURCES = ("ptx.cuh", "gemm.cuh", "vla_ae.cu")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200, help="timed denoise loops")
    ap.add_argument("--warmup", type=int, default=20, help="untimed denoise loops (>= 3)")
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--workload", default="starvla", choices=("starvla", "pi05", "pi05_fp8", "pi05_int8", "pi05_int4", "tiny"))
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--euler-steps", type=int, default=None, help="Euler steps per loop (default: workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip e2e / per-kernel timing (profiling runs)")
    ap.add_argument("--engine", choices=("auto", "per_op", "persistent"), default="auto",
                    help="layer engine: auto (the library times both on the first loop and keeps the "
                         "faster), one kernel per op, or one persistent kernel per step")
    return ap.parse_args()


def workload(args):
    from synth import config
    d = config(args.workload).replace(batch=args.batch)
    if args.euler_steps:
        d = d.replace(steps=args.euler_steps)
    return d


def workload_config(d, args):
    return {
        "workload": f"{args.workload}-shaped action expert, batch {d.batch}, {d.steps} Euler steps",
        "model": f"DiT L={d.n_layers} H={d.hidden} heads={d.n_q_heads}/{d.n_kv_heads}x{d.head_dim} "
                 f"I={d.inter} tokens={d.n_action_tokens}+{d.has_state_token} A={d.action_dim}",
        "prefix_tokens": d.n_prefix,
        "batch": d.batch,
        "euler_steps": d.steps,
        "weights": d.wtype,
        "l2": "inputs larger than L2: each loop streams every layer's weights from HBM (no flush)",
        "parallelism": "replicas (no collective on the data path)",
    }


def algorithmic_bytes(d):
    """Bytes one loop must move from HBM: N x (linear weights (+ fp8 scales) + B x prefix K/V)."""
    H, I, qd, kd = d.hidden, d.inter, d.qd, d.kd
    params = H * (qd + 2 * kd) + H * qd + 2 * I * H + H * I
    if d.wtype == "int4_g128":   # half a byte per weight + one fp32 scale per row and 128 inputs
        wb = params // 2 + 4 * ((qd + 2 * kd) * -(-H // 128) + H * -(-qd // 128) + 2 * I * -(-H // 128) + H * -(-I // 128))
    else:
        wb = params * (1 if d.wtype != "bf16" else 2)
        if d.wtype != "bf16":
            wb += 4 * ((qd + 2 * kd) + H + 2 * I + H)
    kv = 2 * d.n_prefix * kd * 2
    return d.steps * d.n_layers * (wb + d.batch * kv)


def replica_seed(rank: int) -> int:
    """Replicas share the weights and take their own inputs: rank r draws sample inputs with seed r."""
    return rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time (the job is done when every replica is done)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(bytes_per_loop: int, world: int, ms_per_loop_max: float) -> float:
    """Whole-job throughput: all replicas' algorithmic bytes over the slowest replica's loop time."""
    return world * bytes_per_loop / (ms_per_loop_max * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "flow_matching_action_euler_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload_name):
    """dram bytes per launch of the dominant kernel from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        ent = t.get(workload_name)
        if ent and ent.get("kernel_source_hash") == kernel_source_hash():
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
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
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s, p in zip(sm, power)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle timing
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample_rate(d, w, x, budget_s=10.0, per_layer=False, n_samples=None, warmup=0):
    """Time the oracle on a bounded sample of the workload; returns (GB/s, seconds, description, ms/sample)."""
    import numpy as np
    import oracle
    W = oracle.OracleWeights(w, d, quantized=d.wtype)
    for l in range(d.n_layers):
        W.layer(l)
    noise = oracle.bf16_to_f64(x["noise"][0])
    st = oracle.bf16_to_f64(x["state"][0]) if d.has_state_token else None
    kp, vp = oracle.bf16_to_f64(x["k"][0]), oracle.bf16_to_f64(x["v"][0])
    bytes_loop = algorithmic_bytes(d.replace(batch=1))
    if per_layer:
        # one DiT layer of one Euler step per sample, cycling over the layers
        ts, _ = oracle.t_schedule(d.steps)
        h = oracle.embed_tokens(noise, st, W, d)
        pos = kp.shape[1] + np.arange(h.shape[0], dtype=np.float64)
        mods = [oracle.adaln_table(W.layer(l)["w_ada"], W.layer(l)["b_ada"], ts[0], d.t_emb_dim)
                for l in range(d.n_layers)]

        def one(i):
            l = i % d.n_layers
            oracle.dit_layer(h, W.layer(l), mods[l], kp[l], vp[l], pos, d)

        for i in range(warmup):
            one(i)
        t0 = time.perf_counter()
        for i in range(n_samples):
            one(i)
        dt = time.perf_counter() - t0
        unit_bytes = bytes_loop / (d.steps * d.n_layers)
        return (unit_bytes * n_samples / dt / 1e9, dt,
                f"{n_samples} samples of one DiT layer at one Euler step (sample 0, layers cycled)",
                dt / n_samples * 1e3)
    loops, t0 = 0, time.perf_counter()
    while True:
        oracle.denoise(noise, st, W, kp, vp, d, d.steps)
        loops += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    return (bytes_loop * loops / dt / 1e9, dt,
            f"{loops} full denoise loop(s) of sample 0 ({d.steps} Euler steps x {d.n_layers} layers)",
            dt / loops * 1e3)


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import generate_inputs, generate_weights
    d = workload(args)
    w = generate_weights(d, 0)
    x = generate_inputs(d.replace(batch=1), 0)
    gbs, dt, sample, ms = oracle_sample_rate(d, w, x, per_layer=True, n_samples=args.steps,
                                             warmup=max(args.warmup, 0))
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(d, args),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- native arm
def run_native(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import __graft_entry__
    __graft_entry__._build_module().build_library()
    import flow_matching_action_euler_b200 as fm
    from synth import abi_dims, generate_inputs, generate_weights

    d = workload(args)
    w = generate_weights(d, 0)
    x = generate_inputs(d, seed=replica_seed(rank))   # each replica its own inputs, same weights
    ae = fm.ActionExpert(abi_dims(d), w)
    stream = torch.cuda.current_stream()
    kdev = torch.from_numpy(x["k"].view(np.int16)).cuda()
    vdev = torch.from_numpy(x["v"].view(np.int16)).cuda()
    sdev = torch.from_numpy(x["state"].view(np.int16)).cuda() if d.has_state_token else None
    ae.set_prefix(kdev, vdev, d.n_prefix, sdev, on_device=True, stream=stream)
    ae.set_engine({"auto": fm.ENGINE_AUTO, "per_op": fm.ENGINE_PER_OP,
                   "persistent": fm.ENGINE_PERSISTENT}[args.engine])
    noise = torch.from_numpy(x["noise"].view(np.int16)).cuda()
    out = torch.empty((d.batch, d.n_action_tokens, d.action_dim), dtype=torch.float32, device="cuda")
    N = d.steps

    def barrier():
        if world > 1:
            dist.barrier()

    ae.denoise(noise, N, out, stream)          # first call: adaLN table + graph capture (auto: both engines timed)
    torch.cuda.synchronize()
    engine = "persistent" if ae.engine == fm.ENGINE_PERSISTENT else "per_op"
    for _ in range(max(args.warmup, 3)):
        ae.denoise(noise, N, out, stream)
    torch.cuda.synchronize()
    if ae.status() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    # keep the GPU loaded for ~1.5 s before the timed region so the clock samples see the load
    t_soak = time.perf_counter()
    while not args.no_extras and time.perf_counter() - t_soak < 1.5:
        for _ in range(20):
            ae.denoise(noise, N, out, stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    # one event between consecutive loops: the total over all K gives the line's time, the
    # per-loop spans its spread (median, p10, p90)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        ae.denoise(noise, N, out, stream)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(evs[0].elapsed_time(evs[-1]) / args.steps, world, "cuda")
    per_loop = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps))
    loop_dist = {q: round(per_loop[min(len(per_loop) - 1, int(f * len(per_loop)))], 5)
                 for q, f in (("p10", 0.1), ("p50", 0.5), ("p90", 0.9))}
    if ae.status() != 0:
        raise RuntimeError("device-side timeout during the timed region")

    bytes_loop = algorithmic_bytes(d)
    value = job_throughput_gbs(bytes_loop, world, ms)
    kernels_per_loop = ae.query(fm.Q_KERNELS_PER_LOOP, N)
    peak, peak_kind = measured_peak()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"bf16": "bf16", "fp8_e4m3": "e4m3 weights x bf16 activations",
                  "int8": "int8 weights x bf16 activations",
                  "int4_g128": "int4 weights (groups of 128) x bf16 activations"}[d.wtype],
        "data": "synthetic", "config": workload_config(d, args), "engine": engine,
        "ms_per_loop": round(ms, 5),
        "ms_per_loop_dist": dict(loop_dist, rank=0),
        "actions_per_s": round(world * d.batch * d.n_action_tokens * 1000.0 / ms, 1),
        "chunks_per_s": round(world * d.batch * 1000.0 / ms, 2),
        "hbm_frac_of_8tbs": round(value / world / 8000.0, 4),
        "hbm_frac_of_measured": round(value / world / peak, 4),
        "gpu_launches": int(kernels_per_loop * args.steps),
        "clocks": clocks,
    }

    if not args.no_extras:
        # both layer engines on the same handle and inputs (context: the line's value is `engine`'s)
        engines = {}
        for name, eid in (("per_op", fm.ENGINE_PER_OP), ("persistent", fm.ENGINE_PERSISTENT)):
            try:
                ae.set_engine(eid)
            except fm.VlaAeError:
                continue
            for _ in range(3):
                ae.denoise(noise, N, out, stream)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(10, min(args.steps, 50))
            a.record(stream)
            for _ in range(reps):
                ae.denoise(noise, N, out, stream)
            b.record(stream)
            torch.cuda.synchronize()
            engines[name] = {"ms_per_loop": round(a.elapsed_time(b) / reps, 4),
                             "kernels_per_loop": int(ae.query(fm.Q_KERNELS_PER_LOOP, N))}
        ae.set_engine({"auto": fm.ENGINE_AUTO, "per_op": fm.ENGINE_PER_OP,
                       "persistent": fm.ENGINE_PERSISTENT}[args.engine])
        line["engines"] = engines
        # prefix K/V producer (backbone RMSNorm + K/V projection + RoPE), synthetic backbone of
        # width 2048: the compute-bound neighbour stage, against the tensor-core peak
        if d.wtype == "bf16":
            Hv = 2048
            rng = np.random.default_rng(11)
            from synth import f32_to_bf16_bits
            mk = lambda shape, sd: f32_to_bf16_bits((rng.standard_normal(shape) * sd).astype(np.float32))
            wk = [mk((d.kd, Hv), 0.02) for _ in range(d.n_layers)]
            wv = [mk((d.kd, Hv), 0.02) for _ in range(d.n_layers)]
            gn = [f32_to_bf16_bits((1.0 + 0.1 * rng.standard_normal(Hv)).astype(np.float32)) for _ in range(d.n_layers)]
            ae.attach_vlm_kv(wk, wv, gn, Hv)
            hid = torch.from_numpy(mk((d.batch, d.n_layers, d.n_prefix, Hv), 1.0).view(np.int16)).cuda()
            for _ in range(3):
                ae.set_prefix_hidden(hid, d.n_prefix, sdev, stream)
            torch.cuda.synchronize()
            reps = 20
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                ae.set_prefix_hidden(hid, d.n_prefix, sdev, stream)
            b.record(stream)
            torch.cuda.synchronize()
            ms_p = a.elapsed_time(b) / reps
            flops = 2.0 * d.batch * d.n_prefix * Hv * 2 * d.kd * d.n_layers
            try:
                with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                    tpk = float(json.load(f)["bf16_tflops"])
            except Exception:
                tpk = 1590.0
            tf = flops / (ms_p * 1e-3) / 1e12
            line["prefix_kv_producer"] = {
                "ms_per_prefix": round(ms_p, 4), "tflops": round(tf, 2), "peak_tflops": tpk,
                "frac": round(tf / tpk, 4), "bound": "tensor",
                "shape": f"{d.n_layers} layers x [{d.batch * d.n_prefix} tokens x {Hv}] x [{Hv} x {2 * d.kd}] (K and V)",
                "note": "operands are hi/lo bf16 pairs (2x the MMA work of plain bf16); FLOPs counted once"}
            ae.set_prefix(kdev, vdev, d.n_prefix, sdev, on_device=True, stream=stream)
        # per-kernel timing through the bench hook: PDL-chained launches over successive layers
        L = d.n_layers
        count = 4 * L
        kern = {}
        for op in range(5):
            ae.bench_op(op, count, N, stream)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ae.bench_op(op, count, N, stream)
            b.record(stream)
            torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / count
            nbytes = ae.query(fm.Q_OP_BYTES, op)
            kern[OP_NAMES[op]] = {"us_per_launch": round(us, 3), "bytes_per_launch": nbytes,
                                  "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)}
        line["kernels"] = kern
        dom = kern[OP_NAMES[DOMINANT_OP]]
        achieved = dom["GB/s"]
        traffic = ncu_traffic(args.workload)
        line["roofline"] = {
            "kernel": "gemm_stream_kernel<SWIGLU> (gate/up GEMM + SwiGLU)", "bound": "hbm",
            "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "algorithmic_bytes_per_launch": dom["bytes_per_launch"],
            "timing": f"{count} PDL-chained launches over successive layers, CUDA events on the launch stream",
        }
        # end to end through the public API: new prefix (device, D2D) + host noise in, host actions out
        noise_h = torch.from_numpy(x["noise"].view(np.int16)).pin_memory()
        out_h = torch.empty((d.batch, d.n_action_tokens, d.action_dim), dtype=torch.float32).pin_memory()
        for _ in range(3):
            ae.set_prefix(kdev, vdev, d.n_prefix, sdev, on_device=True, stream=stream)
            ae.denoise_host(noise_h, N, out_h, stream)
            stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            ae.set_prefix(kdev, vdev, d.n_prefix, sdev, on_device=True, stream=stream)
            ae.denoise_host(noise_h, N, out_h, stream)
            stream.synchronize()               # the caller reads the actions every control cycle
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / args.steps, world, "cuda")
        line["e2e"] = {"value": round(job_throughput_gbs(bytes_loop, world, ms_e2e), 2), "unit": "GB/s",
                       "ms_per_loop": round(ms_e2e, 5),
                       "h2d_bytes_per_step": int(noise_h.numel() * 2),
                       "d2h_bytes_per_step": int(out_h.numel() * 4),
                       "includes": "set_prefix (device prefix, D2D) + H2D noise + loop + D2H actions + host sync"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, sample, _ = oracle_sample_rate(d, w, x, budget_s=10.0)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": sample, "seconds": round(dt, 2)}
    ae.close()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
