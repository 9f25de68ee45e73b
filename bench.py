"""Benchmark of the denoise loop on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A "step" of this benchmark is one full denoise call: the time MLP once, then
`euler_steps` Euler steps of the 36-layer expert over one 50 x 75 chunk per
request (the workload of "LingBot-VLA on Thor (sm_110)", §1 and §5: chunk
[1, 50, 75], 10 denoise steps, CUDA-graph replay).  Weights are synthetic
N(0, 0.02) bf16 (no checkpoint is available), prefix K/V N(0, 1), x0 N(0, 1).

value      = Euler steps per second over the whole job (all ranks), device
             timed with CUDA events, inputs resident in HBM.
e2e        = the same metric through fm_denoise with pinned host buffers, the
             host->device copy of x0 and the device->host copy of the result
             inside the timed region.
roofline   = the denoise-loop kernel: algorithmic bytes (weights + prefix/chunk
             KV per Euler step) / its event-timed duration, against the
             measured HBM copy bandwidth.
The one-request path does not shard: with N GPUs every rank runs its own
replica (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import re
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

from vla_flow_matching_denoise_b200 import synth  # noqa: E402

METRIC = "ms per 10-step 50x75 chunk & denoise steps/s (B=1); % HBM roofline"
UNIT = "denoise steps/s"

# DRAM bytes of one launch of the loop kernel from an ncu capture, keyed by
# workload, with the hash of the kernel sources it was taken on; reported as
# null when the sources changed since.
NCU_TRAFFIC = {
    # step_kernel, bench workload: dram__bytes_read.sum + dram__bytes_write.sum of one
    # `python bench.py --workload lingbot_l4_p256_n10 --once` launch (4 layers x 1 Euler
    # step: 140.582 + 3.483 MB), scaled by the 90x layer-steps of a 36-layer, 10-step
    # launch (weight and KV traffic grow in proportion).
    "lingbot_p256_n10": {"source_hash": "4c8f763fcfd0d301", "dram_bytes": 144.066e6 * 90},
}


def kernel_source_hash() -> str:
    """Hash of the loop kernel's sources with comments and blank space removed
    (a comment edit does not change the kernel the counters were taken on)."""
    h = hashlib.sha256()
    for f in ("fm_step.cu", "fm_ptx.cuh", "fm_internal.h"):
        with open(os.path.join(ROOT, "vla_flow_matching_denoise_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", " ", text).strip().encode())
    return h.hexdigest()[:16]


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def loop_flops(shape: synth.ExpertShape, steps: int, batch: int) -> float:
    """Algorithmic flops of the denoise loop for one call: 2 per weight per
    token row for every linear (per-layer, in- and out-projection) and 4 * hd
    per (query head, token, key) for attention over the P + T keys."""
    s = shape
    ws = s.weight_shapes()
    per_layer = sum(int(np.prod(ws[k])) for k in synth.LAYER_KEYS)
    io = int(np.prod(ws["in_proj"])) + int(np.prod(ws["out_proj"]))
    rows = batch * s.chunk_len
    lin = 2.0 * rows * (s.n_layers * per_layer + io)
    att = 4.0 * rows * s.n_q_heads * (s.prefix_len + s.chunk_len) * s.head_dim * s.n_layers
    return steps * (lin + att)


def loop_bytes(shape: synth.ExpertShape, steps: int, batch: int) -> float:
    """Algorithmic bytes of the denoise-loop kernel for one call.

    Per Euler step: every per-layer weight once (bf16, or E4M3 plus one fp32
    scale per row), the in/out projections, and per request the prefix K/V and
    the chunk K/V of every layer read once."""
    s = shape
    ws = s.weight_shapes()
    per_layer = sum(int(np.prod(ws[k])) for k in synth.LAYER_KEYS)
    rows = sum(ws[k][0] for k in synth.LAYER_KEYS)
    if s.nvfp4_gu:
        # E4M3 + row scales for wq/wk/wv/wo/w_down; NVFP4 (half a byte per code,
        # one E4M3 scale per 16 codes, one fp32 per tensor) for w_gate, w_up
        gu = int(np.prod(ws["w_gate"])) + int(np.prod(ws["w_up"]))
        rows_8 = rows - ws["w_gate"][0] - ws["w_up"][0]
        wbytes = s.n_layers * ((per_layer - gu) * 1.0 + rows_8 * 4.0 + gu * (0.5 + 1.0 / 16) + 8.0)
    else:
        q8 = s.fp8 or s.w8a8
        wbytes = s.n_layers * (per_layer * (1.0 if q8 else 2.0) + (rows * 4.0 if q8 else 0.0))
    io = (int(np.prod(ws["in_proj"])) + int(np.prod(ws["out_proj"]))) * 2.0
    kv = batch * s.n_layers * 2 * (s.prefix_len + s.chunk_len) * s.n_kv_heads * s.head_dim * 2.0
    return steps * (wbytes + io + kv)


def time_mlp_bytes(shape: synth.ExpertShape) -> float:
    ws = shape.weight_shapes()
    return (int(np.prod(ws["time_w1"])) + int(np.prod(ws["time_w2"]))) * 2.0


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


class OracleRunner:
    """The oracle as it stands, on request 0 of the same workload."""

    def __init__(self, shape: synth.ExpertShape, seed: int = 0):
        from oracle import fm_oracle as O
        self.O = O
        self.shape = shape
        raw = synth.make_weights(shape, seed)
        kp, vp = synth.make_prefix(shape, seed, batch=1)
        self.x0 = synth.make_x0(shape, seed, batch=1)[0]
        self.W = O.Weights(raw, fp8=shape.fp8 or shape.w8a8, nvfp4_gu=shape.nvfp4_gu)
        self.kp = [O.decode_bf16(k[0]) for k in kp]
        self.vp = [O.decode_bf16(v[0]) for v in vp]
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
        except Exception:
            self.cores = os.cpu_count()

    def run(self, n_sample: int) -> float:
        """Seconds for `n_sample` Euler steps (whole chunks repeat from x0), each
        chunk with its own time MLP."""
        O, s = self.O, self.shape
        t0 = time.perf_counter()
        done = 0
        while done < n_sample:
            ts, dt = O.time_schedule(s.steps)
            M = O.time_modulation(ts, self.W.time_w1, self.W.time_w2)
            x = self.x0.astype(np.float64)
            for k in range(min(s.steps, n_sample - done)):
                v = O.expert_velocity(x, M[k], self.W, self.kp, self.vp, s.rms_eps, s.rope_base, s.n_q_heads,
                                      s.n_kv_heads, act_fp8=s.w8a8)
                x = x + dt * v
                done += 1
        return time.perf_counter() - t0

    def sample_text(self, n_sample: int, el: float) -> str:
        return (f"{n_sample} Euler steps of request 0 ({self.shape.steps}-step chunks, time MLP per chunk), "
                f"fp64 numpy, {el:.1f} s")


def cpu_baseline(shape: synth.ExpertShape, n_sample: int, seed: int = 0):
    r = OracleRunner(shape, seed)
    el = r.run(n_sample)
    return {"value": n_sample / el, "unit": UNIT, "cores": r.cores, "kind": "oracle",
            "sample": r.sample_text(n_sample, el)}


def dist_setup(gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK /
    MASTER_*).  Returns (world size, rank, local rank, torch.distributed or None)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if ws > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return ws, rank, local, pg


def max_over_ranks(value: float, pg, device) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(shape: synth.ExpertShape, rank: int):
    """Each rank's own requests: prefix K/V and x0 seeded by the rank (the
    weights are the same on every rank)."""
    kp, vp = synth.make_prefix(shape, seed=rank)
    return kp, vp, synth.make_x0(shape, seed=rank)


def job_value(ws: int, batch: int, steps: int, calls: int, ms_total: float) -> float:
    """Euler steps per second of the whole job: every rank's requests count."""
    return ws * batch * steps * calls / (ms_total / 1000.0)


def run_reference(args, shape):
    # Rank 0 alone times the oracle; other ranks exit without work.
    if int(os.environ.get("RANK", "0")) != 0:
        return
    n_sample = 1
    runner = OracleRunner(shape)
    vals, el = [], 0.0
    for i in range(args.warmup + args.steps):
        el = runner.run(n_sample)
        if i >= args.warmup:
            vals.append(n_sample / el)
    r = {"cores": runner.cores, "sample": runner.sample_text(n_sample, el)}
    v = statistics.mean(vals)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            # one bench step is one denoise call of shape.steps Euler steps, as on the GPU arm
            "ms_per_step": 1000.0 * shape.steps / v, "ms_per_chunk": 1000.0 * shape.steps / v,
            "ms_per_euler_step": 1000.0 / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="lingbot_p256_n10", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-steps", type=int, default=30)
    ap.add_argument("--once", action="store_true",
                    help="one fm_velocity call of the workload and exit (profiling driver)")
    args = ap.parse_args()
    shape = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, shape)
        return

    import torch
    ws, rank, local, pg = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    from vla_flow_matching_denoise_b200.binding import Expert

    B, n = shape.batch, shape.steps
    raw = synth.make_weights(shape, seed=0)
    kp, vp, x0 = rank_inputs(shape, rank)
    e = Expert(shape, raw, device=local)
    del raw
    e.set_prefix(kp, vp, B, shape.prefix_len)
    if args.once:
        v = e.velocity(x0, 0, n)
        torch.cuda.synchronize()
        print(json.dumps({"once": args.workload, "mean_abs_v": float(np.abs(v).mean())}), flush=True)
        e.close()
        return
    x_dev = torch.from_numpy(x0).cuda()
    out_dev = torch.empty_like(x_dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        e.denoise(x_dev, n, out=out_dev)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            e.denoise(x_dev, n, out=out_dev)
        ev1.record(stream)
        barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), pg, "cuda")
    ms_call = ms_total / args.steps
    value = job_value(ws, B, n, args.steps, ms_total)

    # end to end through the public API with pinned host buffers
    xh = torch.from_numpy(x0).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    for _ in range(2):
        e.denoise(xh, n, out=oh)
    barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        e.denoise(xh, n, out=oh)
    ev1.record(stream)
    barrier()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), pg, "cuda")
    e2e_value = job_value(ws, B, n, args.steps, ms_e2e)

    # the loop kernel alone (event-timed, outside the graph)
    ms_time_mlp, ms_loop = e.profile(B, n, max(3, min(args.steps, 10)))
    hbm, tflops, tflops_sus, peak_kind = measured_peaks()
    lb = loop_bytes(shape, n, B)
    achieved = lb / (ms_loop / 1000.0) / 1e9
    lf = loop_flops(shape, n, B)
    batched = shape.w8a8 or (B >= 2 and not shape.fp8 and not shape.nvfp4_gu)
    # an E4M3 contraction takes the measured bf16 peak x the nominal fp8 / bf16 ratio (4.5 / 2.25)
    tpeak = tflops_sus * (2.0 if shape.w8a8 else 1.0)
    tpeak_burst = tflops * (2.0 if shape.w8a8 else 1.0)
    per_layer_launches = 9 if shape.w8a8 else 7   # W8A8: two row-quantiser passes per layer
    traffic = None
    rec = NCU_TRAFFIC.get(args.workload)
    if rec and rec.get("source_hash") == kernel_source_hash():
        traffic = rec["dram_bytes"]
    e.close()

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_call, "ms_per_chunk": ms_call,
        "ms_per_euler_step": ms_call / shape.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if shape.w8a8 else "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "layers": shape.n_layers, "d_model": shape.d_model,
                   "heads": f"{shape.n_q_heads}q/{shape.n_kv_heads}kv x {shape.head_dim}",
                   "d_ff": shape.d_ff, "prefix_len": shape.prefix_len,
                   "chunk": f"{shape.chunk_len}x{shape.action_dim}", "euler_steps": n,
                   "requests_per_gpu": B,
                   "weights": ("fp8-e4m3 + nvfp4 gate_up" if shape.nvfp4_gu else "fp8-e4m3" if shape.fp8
                               else "fp8-e4m3, per-token e4m3 activations" if shape.w8a8 else "bf16"),
                   "parallelism": f"replicas x{ws}",
                   "l2": f"inputs larger than L2: {loop_bytes(shape, 1, B) / 1e9:.3f} GB of weights and KV "
                         "stream per Euler step (L2 126 MB)"},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_chunk": ms_e2e / args.steps,
                "h2d_bytes_per_step": int(x0.nbytes), "d2h_bytes_per_step": int(x0.nbytes)},
        # per Euler step: in-proj, layer 0's norm, per layer (QKV, attention, o_proj, norm,
        # gate_up, down, norm but none after the last layer), out-proj; per call the two
        # time-MLP kernels
        "gpu_launches": args.steps * ((2 + n * (per_layer_launches * shape.n_layers + 2)) if batched else (2 + B)),
        "roofline": ({"bound": "tensor", "achieved": lf / (ms_loop / 1000.0) / 1e12, "peak": tpeak,
                      "unit": "TFLOP/s", "frac": lf / (ms_loop / 1000.0) / 1e12 / tpeak,
                      "traffic": traffic,
                      "peak_kind": peak_kind + (" sustained bf16 x 2 (fp8)" if shape.w8a8 else " sustained bf16"),
                      "kernel": "batched loop (bgemm + attention + row kernels)", "flops_per_launch": lf,
                      "ms_per_launch": ms_loop, "frac_of_burst": lf / (ms_loop / 1000.0) / 1e12 / tpeak_burst}
                     if batched else
                     {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                      "frac": achieved / hbm, "traffic": traffic, "peak_kind": peak_kind,
                      "kernel": "step_kernel", "bytes_per_launch": lb, "ms_per_launch": ms_loop,
                      "frac_of_8TBs": achieved / 8000.0}),
        "time_mlp_ms": ms_time_mlp,
        "time_mlp_gbs": time_mlp_bytes(shape) / (ms_time_mlp / 1000.0) / 1e9,
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, args.cpu_sample_steps)
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
