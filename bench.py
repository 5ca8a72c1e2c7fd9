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


# DRAM traffic of one step (dram__bytes_read.sum + dram__bytes_write.sum
# summed over the 21 launches) from one ncu capture of this step (its summary
# is kept with the other profiles), valid for the kernel source it was taken
# with (sha256 of csrc/mq_gemv_tc.cu); None once that source changes.
STEP_TRAFFIC = {"bytes": 257207552, "sha256": "41bd2a91ec1688de3deb334ffff1423e930c225992e283b1b9f4b2ec9c043d84"}


def step_traffic():
    if not STEP_TRAFFIC:
        return None
    import hashlib
    src = os.path.join(ROOT, "nested_bit_weight_b200", "csrc", "mq_gemv_tc.cu")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    return STEP_TRAFFIC["bytes"] if digest == STEP_TRAFFIC["sha256"] else None


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


def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun env); replicas only, no data-path collective."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, ws: int) -> float:
    """Max over ranks of a device-timed duration (the slowest replica sets the step)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbps(ws: int, bytes_per_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every replica moves bytes_per_step in the max-over-ranks step."""
    return round(ws * bytes_per_step / (ms_per_step * 1e-3) / 1e9, 2)


def time_point(mq, X, views, Y, ws, n_samples: int = 100):
    """Device time of one mq_gemm shape over rotated weight copies.

    Returns (median, p10, p90) in µs over >= n_samples launches, each timed
    alone by an event pair inside a CUDA graph (the events stop consecutive
    launches from overlapping), and the mean µs per launch of the same
    launches back to back in a graph without events (overlap allowed)."""
    import torch
    n_launch = max(len(views), 25)
    stream = torch.cuda.Stream()
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n_launch)]
    with torch.cuda.stream(stream):
        for v in views:
            mq.mq_gemm(X, v, Y, ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(n_launch):
                mq.mq_gemm(X, views[j % len(views)], Y, ws)
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi, stream=stream):
            for j in range(n_launch):
                ev[j][0].record()
                mq.mq_gemm(X, views[j % len(views)], Y, ws)
                ev[j][1].record()
        for _ in range(3):
            g.replay()
            gi.replay()
        torch.cuda.synchronize()
        samples = []
        while len(samples) < n_samples:
            gi.replay()
            torch.cuda.synchronize()
            samples += [a.elapsed_time(b) * 1e3 for a, b in ev]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = max(1, -(-n_samples // n_launch))
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
    torch.cuda.synchronize()
    b2b = e0.elapsed_time(e1) * 1e3 / (reps * n_launch)
    del g, gi
    q = np.percentile(np.array(samples), [50, 10, 90])
    return float(q[0]), float(q[1]), float(q[2]), float(b2b), len(samples)


def rotated_parents(mq, codes, s, l2: int):
    """A packed parent and enough device copies that cycling through them
    reads more than twice the L2 (every launch streams its planes from HBM)."""
    import torch
    p0 = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    pbytes = p0.planes.numel() * 4 + p0.scales16.numel() * 2
    copies = max(1, -(-2 * l2 // pbytes))
    return [p0] + [mq.NestedWeights(p0.planes.clone(), p0.scales16.clone(), p0.N, p0.K)
                   for _ in range(copies - 1)]


PER_POINTS = [("gate_proj", 14336, 4096), ("q_proj", 4096, 4096)]
PER_POINT_M = (8, 16, 64)
PER_POINT_R = (4, 2)


def run_per_points():
    """Config 2 points (Llama-3.1-8B gate and q at M in {8, 16, 64}, r in
    {4, 2}): each timed in isolation over rotated weights (L2-cold)."""
    import torch
    import nested_bit_weight_b200 as mq
    peak, _ = read_peaks()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    out = {}
    for name, N, K in PER_POINTS:
        li = [l.name for l in wl.LLAMA8B].index(name)
        codes, s, _ = wl.gen_weights(N, K, wl.layer_seed(2, li))
        parents = rotated_parents(mq, codes, s, l2)
        del codes
        for M in PER_POINT_M:
            xbits, _ = wl.gen_x(M, K, wl.layer_seed(2, li))
            X = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            for r in PER_POINT_R:
                ws = torch.zeros(max(mq.mq_gemm_workspace_bytes(M, N, K, r), 256),
                                 dtype=torch.uint8, device="cuda")
                med, p10, p90, b2b, n = time_point(mq, X, [q.view(r) for q in parents], Y, ws)
                b = algo_bytes(N, K, r, M)
                out[f"{name}/M{M}/r{r}"] = {
                    "N": N, "K": K, "M": M, "r": r, "path": "gemv" if mq.uses_gemv(M, N, K, r) else "gemm",
                    "us_median": round(med, 3), "us_p10": round(p10, 3), "us_p90": round(p90, 3),
                    "launches": n, "us_back_to_back": round(b2b, 3),
                    "GBps_median": round(b / (med * 1e-6) / 1e9, 1),
                    "frac_hbm_median": round(b / (med * 1e-6) / 1e9 / peak, 4)}
        del parents
        torch.cuda.empty_cache()
    return out


def run_chain(layers, steps: int):
    """Config 1 as one decoder layer per r: fused q|k|v, o, fused gate|up and
    down (4 launches per r, 12 per step), each r on its own parents (L2-cold),
    enqueued by mq_gemm_chain and timed as a CUDA graph."""
    import torch
    import nested_bit_weight_b200 as mq
    peak, _ = read_peaks()
    idx = {l.name: i for i, l in enumerate(wl.LLAMA8B)}
    dev = lambda a: torch.from_numpy(a).cuda()
    C = {n: dev(layers[idx[n]][0]) for n in idx}
    S = {n: dev(layers[idx[n]][1]) for n in idx}
    X = {n: torch.from_numpy(layers[idx[n]][2].view(np.int16)).cuda().view(torch.bfloat16) for n in idx}
    calls, nbytes = [], 0
    for r in R_LIST:
        qkv = mq.pack_fused([C["q_proj"], C["k_proj"], C["v_proj"]], [S["q_proj"], S["k_proj"], S["v_proj"]])
        gu = mq.pack_fused([C["gate_proj"], C["up_proj"]], [S["gate_proj"], S["up_proj"]])
        o = mq.pack_parent(C["o_proj"], S["o_proj"])
        dn = mq.pack_parent(C["down_proj"], S["down_proj"])
        for w, xn in ((qkv, "q_proj"), (o, "o_proj"), (gu, "gate_proj"), (dn, "down_proj")):
            Y = torch.empty((M, w.N), dtype=torch.bfloat16, device="cuda")
            calls.append((X[xn], w, r, Y))
            nbytes += algo_bytes(w.N, w.K, r, M)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        mq.gemm_chain(calls)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            mq.gemm_chain(calls)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    gbps = nbytes / (ms * 1e-3) / 1e9
    del g
    return {"note": "config 1 as one decoder layer per r: fused q|k|v, o, fused gate|up, "
                    "down (4 launches per r, 12 per step), mq_gemm_chain in a CUDA graph, "
                    "each r on its own parents (L2-cold)",
            "ms_per_step": round(ms, 5), "bytes_per_step": nbytes, "GBps": round(gbps, 1),
            "frac_hbm": round(gbps / peak, 4), "launches_per_step": len(calls)}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


_ONE_CORE = r"""
import sys, time, json
sys.path.insert(0, ROOTDIR)
import numpy as np
import oracle, workloads as wl
out = {}
for name, N, K, ci in (("config0 512x512 M=1 r=4", 512, 512, 0), ("llama q_proj 4096x4096 M=1 r=4", 4096, 4096, 1)):
    codes, s, _ = wl.gen_weights(N, K, wl.layer_seed(ci, 0))
    xbits, X = wl.gen_x(1, K, wl.layer_seed(ci, 0))
    oracle.gemm(X, codes, s, 4)
    n, t0 = 0, time.perf_counter()
    while n == 0 or time.perf_counter() - t0 < 2.0:
        oracle.gemm(X, codes, s, 4)
        n += 1
    dt = (time.perf_counter() - t0) / n
    b = 4 * N * K // 8 + 2 * N * K // 128 + 2 * K + 2 * N
    out[name] = {"ms": round(dt * 1e3, 3), "GBps": round(b / dt / 1e9, 4)}
out["threads"] = oracle.threads()
print(json.dumps(out))
"""


def one_core_oracle():
    """The oracle restricted to one thread (OMP_NUM_THREADS=1, a fresh process)."""
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", _ONE_CORE.replace("ROOTDIR", repr(ROOT))],
                           env=env, capture_output=True, text=True, timeout=120)
        return json.loads(r.stdout.strip().splitlines()[-1])
    except Exception as e:  # reported, not fatal: the baseline is context only
        return {"error": str(e)[:200]}


def cpu_oracle_sample(layers, budget_s: float = 12.0):
    """The plain-C oracle on whole layers of the same step for about budget_s."""
    import oracle
    done_bytes, t_total, n_layers = 0, 0.0, 0
    order = [(r, i) for r in R_LIST for i in range(len(wl.LLAMA8B))]
    xs = [wl.bf16_bits_to_f32(xbits) for (_, _, xbits) in layers]
    while n_layers == 0 or t_total < budget_s:
        r, i = order[n_layers % len(order)]
        l = wl.LLAMA8B[i]
        codes, s, _ = layers[i]
        t0 = time.perf_counter()
        oracle.gemm(xs[i], codes, s, r)
        t_total += time.perf_counter() - t0
        done_bytes += algo_bytes(l.N, l.K, r)
        n_layers += 1
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": oracle.threads(),
            "kind": "oracle", "cpu_model": cpu_model(), "one_core": one_core_oracle(),
            "sample": f"{n_layers} layer products of the step (M=1, r in {{4,3,2}}, in step "
                      f"order), fp64 C oracle with OpenMP, {t_total:.1f} s"}


def run_case(args):
    """One layer, launched eagerly: the small case for ncu captures.

    --case N,K,M,r  runs --warmup + --steps launches of mq_gemm on that shape
    (seeded weights and X) and prints the CUDA-event time per launch."""
    import torch
    import nested_bit_weight_b200 as mq
    N, K, M, r = (int(v) for v in args.case.split(","))
    codes, s, _ = wl.gen_weights(N, K, seed=N + K)
    xbits, _ = wl.gen_x(M, K, seed=N + K)
    p = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    X = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(args.warmup):
        mq.gemm(X, p, r, Y=Y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        mq.gemm(X, p, r, Y=Y)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / max(args.steps, 1) * 1e3
    print(json.dumps({"case": [N, K, M, r], "us_per_launch_eager": round(us, 3),
                      "GBps": round(algo_bytes(N, K, r, M) / (us * 1e-6) / 1e9, 1)}), flush=True)


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

    # end to end through the public Python API: the step's inputs copied in
    # from one pinned host buffer and its outputs read back into another (one
    # copy each way), the 21 products enqueued by one gemm_chain call (the
    # same launches as the timed graph)
    xsz = [x.numel() for x in X]
    ykeys = [(r, i) for r in R_LIST for i in range(len(wl.LLAMA8B))]
    ysz = [Y[k].numel() for k in ykeys]
    Xh = torch.empty(sum(xsz), dtype=torch.bfloat16, pin_memory=True)
    Xh.copy_(torch.cat([x.reshape(-1) for x in X]).cpu())
    Yh = torch.empty(sum(ysz), dtype=torch.bfloat16, pin_memory=True)
    Xall = torch.empty(sum(xsz), dtype=torch.bfloat16, device=dev)
    Yall = torch.empty(sum(ysz), dtype=torch.bfloat16, device=dev)
    Xd = [v.view(x.shape) for v, x in zip(torch.split(Xall, xsz), X)]
    Yd = {k: v.view(Y[k].shape) for k, v in zip(ykeys, torch.split(Yall, ysz))}
    h2d, d2h = Xh.numel() * 2, Yh.numel() * 2
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    chain = [(Xd[i], parents[(r, i)], r, Yd[(r, i)]) for (r, i) in ykeys]

    def e2e_step():
        Xall.copy_(Xh, non_blocking=True)
        mq.gemm_chain(chain)
        Yh.copy_(Yall, non_blocking=True)

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
    # the roofline of the step as timed: algorithmic bytes of the 21 launches
    # over the graph's device time per step on this GPU (launches overlap
    # through programmatic dependent launch, so per-launch times do not add up
    # to the step)
    achieved = sb / (ms_local / args.steps * 1e-3) / 1e9
    detail = {"note": "each launch timed alone (an event pair around it stops the overlap "
                      "with its neighbours): per-launch context, not the step's time"}
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
        "metric": METRIC, "value": aggregate_gbps(ws_n, sb, ms_per_step),
        "unit": "GB/s", "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; weights, codes and X per the layer recipe)",
        "config": config_dict(),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": step_traffic(),
                     "traffic_unit": "bytes per step (dram read + write of the 21 launches)",
                     "algorithmic_bytes": sb,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                                    if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": "nested_gemv_tc_kernel (one launch per mq_gemm call), "
                               "all 21 calls of the step, timed as the step",
                     "frac_of_8TBps": round(achieved / 8000.0, 4)},
        "e2e": {"value": aggregate_gbps(ws_n, sb, e2e_ms), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": len(calls) * args.steps,
        "clocks": clk,
        "per_launch_isolated": detail,
    }
    if ws_n == 1:
        out["decoder_layer_chain"] = run_chain(layers, max(args.steps, 20))
        out["per_point"] = {"note": "config 2 points (Llama-3.1-8B gate and q), each shape "
                                    "alone over rotated weights (L2-cold): median, p10, p90 "
                                    "of >= 100 launches timed one by one, and the mean of the "
                                    "same launches back to back",
                            **run_per_points()}
    return out, layers


def run_sweep(args):
    """Per-(layer, M, r) isolated timings for one workload table (configs of
    workloads.CONFIGS), weights rotated over more than twice the L2 so every
    launch reads its planes from HBM: median, p10 and p90 of >= 100 launches
    timed one by one, and the back-to-back mean.  Prints one JSON line per
    point and a markdown table."""
    import torch
    import nested_bit_weight_b200 as mq
    peak, _ = read_peaks()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    cfgs = sorted(wl.CONFIGS) if args.sweep == "all" else [int(c) for c in args.sweep.split(",")]
    rows = []
    for ci in cfgs:
        cfg = wl.CONFIGS[ci]
        done = {}
        for li, layer in enumerate(cfg["layers"]):
            key = (layer.N, layer.K)
            if key in done:            # same shape as an earlier layer: same numbers
                for r_ in done[key]:
                    rows.append(dict(r_, layer=layer.name))
                continue
            codes, s, _ = wl.gen_weights(layer.N, layer.K, wl.layer_seed(ci, li))
            parents = rotated_parents(mq, codes, s, l2)
            del codes
            rs = cfg["r"] if cfg["r"] is not None else (wl.QWEN3_R[layer.name],)
            out_rows = []
            for M in cfg["M"]:
                xbits, _ = wl.gen_x(M, layer.K, wl.layer_seed(ci, li), outlier_channels=(ci == 3))
                X = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
                Y = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
                for r in rs:
                    need = mq.mq_gemm_workspace_bytes(M, layer.N, layer.K, r)
                    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
                    us, p10, p90, b2b, n = time_point(mq, X, [q.view(r) for q in parents], Y, ws)
                    b = algo_bytes(layer.N, layer.K, r, M)
                    fl = 2.0 * M * layer.N * layer.K
                    row = {"config": ci, "layer": layer.name, "N": layer.N, "K": layer.K, "M": M,
                           "r": r, "us": round(us, 3), "us_p10": round(p10, 3),
                           "us_p90": round(p90, 3), "launches": n,
                           "us_back_to_back": round(b2b, 3),
                           "GBps": round(b / (us * 1e-6) / 1e9, 1),
                           "TFLOPs": round(fl / (us * 1e-6) / 1e12, 2),
                           "frac_hbm_measured": round(b / (us * 1e-6) / 1e9 / peak, 3),
                           "frac_8TBps": round(b / (us * 1e-6) / 8e12, 3),
                           "path": "gemv" if mq.uses_gemv(M, layer.N, layer.K, r) else "tcgen05 gemm"}
                    out_rows.append(row)
                    rows.append(row)
                    print(json.dumps(row), flush=True)
            done[key] = out_rows
            del parents
            torch.cuda.empty_cache()
    print("| config | layer | N | K | M | r | µs median | p10 | p90 | back-to-back µs | GB/s | "
          "TFLOP/s | frac of measured HBM | frac of 8 TB/s | path |")
    print("|---|---|---|---|---|---|---|---|---|---|---|---|---|---|---|")
    for r_ in rows:
        print(f"| {r_['config']} | {r_['layer']} | {r_['N']} | {r_['K']} | {r_['M']} | {r_['r']} | "
              f"{r_['us']} | {r_['us_p10']} | {r_['us_p90']} | {r_['us_back_to_back']} | "
              f"{r_['GBps']} | {r_['TFLOPs']} | {r_['frac_hbm_measured']} | "
              f"{r_['frac_8TBps']} | {r_['path']} |")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mq", choices=["mq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, help="N,K,M,r: one layer, eager launches (for ncu)")
    ap.add_argument("--sweep", default=None, help="config indices (e.g. 0,1,2) or 'all': "
                                                  "per-(layer, M, r) isolated timings")
    ap.add_argument("--quantizer", action="store_true",
                    help="host only: time the one-shot quantizer on the Llama-3.1-8B shapes")
    args = ap.parse_args()
    if args.quantizer:
        run_quantizer()
        return
    if args.case:
        run_case(args)
        return
    if args.sweep:
        run_sweep(args)
        return
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


# The pages' complete MatGPTQ passes over the Llama-3.1-8B shapes (seconds;
# "MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models",
# appendix Table 3; their machine is not stated): context for the host times.
PAGES_MATGPTQ_PASS_S = {"k_proj": 3.59, "q_proj": 3.59, "gate_proj": 6.58, "down_proj": 12.45}


def run_quantizer():
    """One JSON line per shape: the one-shot quantizer (r = 3, 4, 8, lambda =
    1, 1, 1, five scale multipliers) on a synthetic AR(1) Hessian, timed on
    the host around the library calls; total_s is prepare plus the symmetric
    quantize, quantize_asym_s the asymmetric variant on the same U."""
    import nested_bit_weight_b200 as mq
    for i, name in enumerate(("k_proj", "q_proj", "gate_proj", "down_proj")):
        l = next(x for x in wl.LLAMA8B if x.name == name)
        H = wl.gen_hessian(l.K, 7000 + i)
        W = wl.gen_float_weights(l.N, l.K, 7100 + i)
        t0 = time.perf_counter()
        U = mq.matgptq_prepare(H)
        t1 = time.perf_counter()
        mq.matgptq_quantize(W, U)
        t2 = time.perf_counter()
        mq.matgptq_quantize(W, U, asymmetric=True)
        t3 = time.perf_counter()
        print(json.dumps({"metric": "quantizer_pass_s", "layer": name, "N": l.N, "K": l.K,
                          "prepare_s": round(t1 - t0, 2), "quantize_s": round(t2 - t1, 2),
                          "total_s": round(t2 - t0, 2), "quantize_asym_s": round(t3 - t2, 2),
                          "threads": os.cpu_count(),
                          "pages_matgptq_pass_s": PAGES_MATGPTQ_PASS_S[name],
                          "higher_is_better": False, "data": "synthetic"}), flush=True)
        del H, U, W


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
