"""Benchmark: nested r-bit GEMM on the Llama-3.1-8B decode layers (M = 1).

One step = the seven linear layers of a Llama-3.1-8B decoder layer (q, k, v,
o, gate, up, down) at batch M = 1, run at r = 4, 3 and 2 (21 GEMV launches),
each r reading its own copy of the packed parent so that one step streams
245 MB of bit planes (about twice the 126 MB L2): every read is cold.

Prints one JSON line (rank 0).  value = algorithmic bytes of the step
(r N K / 8 + 2 N K / 128 + 2 M K + 2 M N per layer, summed) / device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "nested r-bit GEMM µs & effective HBM GB/s vs 8 TB/s, per bit-width r and batch"
R_LIST = (4, 3, 2)
M = 1
FALLBACK_HBM_GBS = 6650.0


def algo_bytes(N: int, K: int, r: int, m: int = M) -> int:
    return r * N * K // 8 + 2 * N * K // 128 + 2 * m * K + 2 * m * N


def step_bytes() -> int:
    return sum(algo_bytes(l.N, l.K, r) for r in R_LIST for l in wl.LLAMA8B)


def config_dict():
    return {"workload": "Llama-3.1-8B decoder-layer linears (q,k,v,o 4096x4096/1024x4096, "
                        "gate/up 14336x4096, down 4096x14336), M=1, r in {4,3,2}, group 128",
            "M": M, "r": list(R_LIST), "layers": [[l.name, l.N, l.K] for l in wl.LLAMA8B],
            "bytes_per_step": step_bytes(),
            "l2": "inputs larger than L2: each r reads its own parent copy, "
                  "245 MB of planes per step vs 126 MB L2",
            "seed": "layer i: 1000*1 + i (workloads.layer_seed)"}


def gen_layers():
    def one(i_l):
        i, l = i_l
        codes, s, _ = wl.gen_weights(l.N, l.K, wl.layer_seed(1, i))
        xbits, _ = wl.gen_x(M, l.K, wl.layer_seed(1, i))
        return codes, s, xbits
    with cf.ThreadPoolExecutor(max_workers=7) as ex:
        return list(ex.map(one, enumerate(wl.LLAMA8B)))


def read_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.path = index, None, None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        mhz = [float(r[1]) for r in rows]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": float(rows[0][2]),
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows),
                "reasons": reasons}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(layers, budget_s: float = 12.0):
    """The plain-C oracle on whole layers of the same step until ~budget_s."""
    import oracle
    done_bytes, t_total, n_layers = 0, 0.0, 0
    order = [(r, i) for r in R_LIST for i in range(len(wl.LLAMA8B))]
    while n_layers == 0 or (t_total < budget_s and n_layers < 4 * len(order)):
        r, i = order[n_layers % len(order)]
        l = wl.LLAMA8B[i]
        codes, s, xbits = layers[i]
        X = wl.bf16_bits_to_f32(xbits)
        t0 = time.perf_counter()
        oracle.gemm(X, codes, s, r)
        t_total += time.perf_counter() - t0
        done_bytes += algo_bytes(l.N, l.K, r)
        n_layers += 1
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"{n_layers} layer GEMVs of the step (M=1, fp64 C oracle, OpenMP), "
                      f"{t_total:.1f} s"}


def run_mq(args, ws_n, rank, local):
    import torch
    import nested_bit_weight_b200 as mq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    layers = gen_layers()
    # one packed parent per layer, plus two device copies: r = 4, 3, 2 each
    # stream their own planes so a step never re-reads from L2
    parents = {}
    for i, (codes, s, _) in enumerate(layers):
        p = mq.pack_parent(torch.from_numpy(codes).to(dev), torch.from_numpy(s).to(dev))
        for j, r in enumerate(R_LIST):
            q = p if j == 0 else mq.NestedWeights(p.planes.clone(), p.scales16.clone(),
                                                  p.N, p.K)
            parents[(r, i)] = q
    X = [torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
         for (_, _, xb) in layers]
    Y = {(r, i): torch.empty((M, l.N), dtype=torch.bfloat16, device=dev)
         for r in R_LIST for i, l in enumerate(wl.LLAMA8B)}
    need = max(mq.mq_gemm_workspace_bytes(M, l.N, l.K, r) for r in R_LIST for l in wl.LLAMA8B)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    views = {k: v.view(k[0]) for k, v in parents.items()}
    calls = [(X[i], views[(r, i)], Y[(r, i)]) for r in R_LIST for i in range(len(wl.LLAMA8B))]

    def step(events=None):
        for c, (x, w, y) in enumerate(calls):
            if events is not None:
                events[c][0].record()
            mq.mq_gemm(x, w, y, ws)
            if events is not None:
                events[c][1].record()

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        step()                                     # first launch outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in calls]
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi, stream=stream):
            step(ev)
    torch.cuda.synchronize()

    # parity spot check of this run's outputs (one layer per r) happens in the
    # tests; here only the timing.
    for _ in range(max(args.warmup, 3)):
        g.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(ws_n)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t_start.record()
        for _ in range(args.steps):
            g.replay()
        t_end.record()
    torch.cuda.synchronize()
    barrier(ws_n)
    ms_local = t_start.elapsed_time(t_end)
    soak = None
    if ms_local < 1500.0:                          # too short for clock samples
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            while time.perf_counter() - t0 < 1.5:
                for _ in range(200):
                    g.replay()
                torch.cuda.synchronize()
        soak = "clocks sampled over the timed region plus a 1.5 s soak of the same graph"
    clk = clocks.stop()
    if soak:
        clk["note"] = soak
    ms = reduce_max(ms_local, ws_n)
    ms_per_step = ms / args.steps

    # per-launch durations: the same step with an event pair around each launch
    per = np.zeros(len(calls))
    reps = max(args.steps, 20)
    for _ in range(reps):
        with torch.cuda.stream(stream):
            gi.replay()
        torch.cuda.synchronize()
        per += np.array([a.elapsed_time(b) for a, b in ev])
    per /= reps

    # end to end through the public Python API: pinned host X in, Y out
    Xh = [torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True) for x in X]
    for xh, x in zip(Xh, X):
        xh.copy_(x.cpu())
    Yh = {k: torch.empty(v.shape, dtype=torch.bfloat16, pin_memory=True) for k, v in Y.items()}
    h2d = sum(x.numel() * 2 for x in Xh)
    d2h = sum(y.numel() * 2 for y in Yh.values())
    Xd = [torch.empty_like(x) for x in X]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def e2e_step():
        for xd, xh in zip(Xd, Xh):
            xd.copy_(xh, non_blocking=True)
        for r in R_LIST:
            for i in range(len(wl.LLAMA8B)):
                mq.gemm(Xd[i], parents[(r, i)], r, Y=Y[(r, i)])
        for k, yh in Yh.items():
            yh.copy_(Y[k], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws_n)
        e0.record()
        for _ in range(args.steps):
            e2e_step()
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), ws_n) / args.steps

    sb = step_bytes()
    peak, peak_kind = read_peaks()
    lay_bytes = np.array([algo_bytes(wl.LLAMA8B[i].N, wl.LLAMA8B[i].K, r)
                          for r in R_LIST for i in range(len(wl.LLAMA8B))], dtype=np.float64)
    achieved = lay_bytes.sum() / (per.sum() * 1e-3) / 1e9
    detail = {}
    for c, (r, i) in enumerate([(r, i) for r in R_LIST for i in range(len(wl.LLAMA8B))]):
        l = wl.LLAMA8B[i]
        detail[f"r{r}/{l.name}"] = {"us": round(per[c] * 1e3, 3),
                                    "GBps": round(lay_bytes[c] / (per[c] * 1e-3) / 1e9, 1),
                                    "frac_8TBps": round(lay_bytes[c] / (per[c] * 1e-3) / 8e12, 3)}
    for r in R_LIST:
        idx = [c for c, (rr, _) in enumerate([(rr, i) for rr in R_LIST
                                              for i in range(len(wl.LLAMA8B))]) if rr == r]
        detail[f"r{r}/decoder_layer"] = {
            "us": round(per[idx].sum() * 1e3, 3),
            "GBps": round(lay_bytes[idx].sum() / (per[idx].sum() * 1e-3) / 1e9, 1),
            "frac_8TBps": round(lay_bytes[idx].sum() / (per[idx].sum() * 1e-3) / 8e12, 3)}

    out = {
        "metric": METRIC, "value": round(ws_n * sb / (ms_per_step * 1e-3) / 1e9, 2),
        "unit": "GB/s", "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; weights, codes and X per the layer recipe)",
        "config": config_dict(),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                                    if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": "mq_gemm M<=8 call: bfrag prep + gemv_mma_kernel, "
                               "all 21 calls of the step",
                     "frac_of_8TBps": round(achieved / 8000.0, 4)},
        "e2e": {"value": round(ws_n * sb / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": len(calls) * args.steps,
        "clocks": clk,
        "per_layer": detail,
    }
    return out, layers


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mq", choices=["mq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    ws_n, rank, local = dist_init()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    out, layers = run_mq(args, ws_n, rank, local)
    if rank == 0:
        if ws_n == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_oracle_sample(layers)
        print(json.dumps(out), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the CPU oracle, timed on the host cores."""
    layers = gen_layers()
    import oracle
    sb = step_bytes()
    cpu_oracle_sample(layers, budget_s=0.0)            # one layer as warm-up
    t0 = time.perf_counter()
    n = 0
    while n < args.steps and (n == 0 or time.perf_counter() - t0 < 60.0):
        for r in R_LIST:
            for i, l in enumerate(wl.LLAMA8B):
                codes, s, xbits = layers[i]
                oracle.gemm(wl.bf16_bits_to_f32(xbits), codes, s, r)
        n += 1
    dt = time.perf_counter() - t0
    val = n * sb / dt / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": n, "warmup": args.warmup,
            "ms_per_step": round(dt / n * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(),
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": oracle.threads(),
                             "kind": "oracle",
                             "sample": f"{n} full steps (21 layer GEMVs each), fp64 C oracle"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


if __name__ == "__main__":
    main()
