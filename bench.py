#!/usr/bin/env python3
"""Benchmark of the NVFP4 weight-streaming decode round on B200.

One step = one replay of the full synthetic decode round (64 layers of
q/k/v, o, fused gate/up + SiLU-multiply and down GEMMs, plus the vocabulary
head; about 13.84 GB of NVFP4 weights) at batch width M (default 8), from
its per-width CUDA graph.  The metric is the HBM weight-stream rate in GB/s
(algorithmic weight bytes per round / round time) with the round time in ms
alongside; a per-M sweep of single GEMMs is reported as detail.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--width M] [--impl reference]

For N > 1 it runs under torchrun, one independent replica per GPU (the round
does not shard: replicas only), timed as the max over ranks.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 decode GEMM HBM GB/s and % of B200 peak at M=1..8; full round ms"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the B200's nominal HBM3e bandwidth (~8 TB/s), a second denominator
KERNEL_SOURCES = ["gemm.cu", "dequant.cuh", "layout.cuh", "async.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--width", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--round-mode", default="chain", choices=["chain", "persistent"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="only warm-up and timed replays (for an ncu launch list)")
    ap.add_argument("--gemm-case", default=None, choices=["head", "proj", "qkv", "gateup", "down"],
                    help="only three direct calls of one workload GEMM at --width (for an ncu capture)")
    ap.add_argument("--topk-case", type=int, default=None,
                    help="only three top-k calls with this k over --width rows of 151,936 logits (for an ncu capture)")
    ap.add_argument("--grouped-case", action="store_true",
                    help="only three grouped expert calls (512 experts of 768 x 2,048, --width lanes, 10 picks each; "
                         "for an ncu capture)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_code(text):
    """Source text without comments and blank lines: what the compiler sees of it."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_hash():
    """Hash of the decode GEMM's sources, comments aside (a comment edit does not change the kernel)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "nvfp4_weight_streaming_decode_b200", "csrc", name)) as f:
            h.update(kernel_code(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per round from the committed ncu summary, if its kernel hash is current."""
    path = os.path.join(ROOT, "profiles", "decode_gemm_round_m8_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_hash") != kernel_hash():
            return None
        return float(kv["dram_bytes_per_round"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus, backend=None):
    """One process per GPU (torchrun environment).  NCCL on GPUs; gloo when
    asked for, or when no GPU is present (the CPU tests of this plumbing)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        be = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if be == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(be, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world):
    """The slowest rank's value (device time of the timed region)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbps(weight_bytes, steps, elapsed_s, world):
    """Whole-job weight-stream rate: every replica streams weight_bytes per
    step; the job takes the slowest rank's time."""
    return world * weight_bytes * steps / elapsed_s / 1e9


# ------------------------------------------------------------------ CPU oracle legs

def oracle_sample(device, seconds_budget):
    """Time the float64 oracle on a bounded sample of the round's layer-0 q/k/v
    GEMM (K = 5120, M = 8): blocks of rows, cycling through the matrix, until
    the time budget is spent; returns (GB/s of weights processed, cores,
    description)."""
    import numpy as np
    import torch

    import oracle
    from nvfp4_weight_streaming_decode_b200 import synth
    hidden = synth.WORKLOADS[4]["hidden"]
    q_full, s_full = synth.torch_matrix(4, 0, 3 * hidden, hidden, device)
    q_full, s_full = q_full.cpu().numpy(), s_full.cpu().numpy()
    Xb = synth.torch_activations(4, 0, 8, hidden, device).view(torch.int16).cpu().numpy().view(np.uint16)
    block = 1024
    rows_total, elapsed, lo = 0, 0.0, 0
    while elapsed < seconds_budget:
        q = np.ascontiguousarray(q_full[lo:lo + block])
        s = np.ascontiguousarray(s_full[lo:lo + block])
        t0 = time.perf_counter()
        oracle.gemm(Xb, q, s, synth.GSCALE)
        elapsed += time.perf_counter() - t0
        rows_total += q.shape[0]
        lo = (lo + block) % q_full.shape[0]
    gbs = rows_total * hidden * (0.5 + 1 / 16) / elapsed / 1e9
    return gbs, oracle.threads(), (f"float64 oracle GEMM, M=8, {rows_total} rows (blocks of {block}, cycling) "
                                   f"of the round's layer-0 q/k/v matrix, K={hidden}, {elapsed:.1f} s")


def round_weight_bytes(layers, hidden, ffn, vocab):
    """Weight bytes one round streams: every matrix in 32 x 64 units of 1,024 code bytes and
    128 scale bytes (q/k/v stacked, o, gate, up and down per layer, then the head)."""
    def mat(N, K):
        return -(-N // 32) * -(-K // 64) * (1024 + 128)
    per_layer = mat(3 * hidden, hidden) + mat(hidden, hidden) + 2 * mat(ffn, hidden) + mat(hidden, ffn)
    return layers * per_layer + mat(vocab, hidden)


def round_config(args, world, weight_bytes, nodes, graph_nodes):
    """The bench line's config: the same dict for both arms."""
    w = round_workload()
    return {"workload": "round_64layers_head_m1to8", "width_M": args.width, "layers": args.layers,
            "hidden": w["hidden"], "ffn": w["ffn"], "vocab": w["vocab"],
            "weight_bytes_per_round": weight_bytes, "gemm_nodes": nodes,
            "graph_nodes": graph_nodes, "round_mode": args.round_mode,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (13.8 GB of weights per round)"}


def round_workload():
    """Dimensions of the 64-layer round (hidden, ffn, vocab)."""
    from nvfp4_weight_streaming_decode_b200 import synth
    return synth.WORKLOADS[4]


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from nvfp4_weight_streaming_decode_b200 import synth
    w4 = synth.WORKLOADS[4]
    hidden = w4["hidden"]
    q_full, s_full = synth.matrix(4, 0, 3 * hidden, hidden)
    Xb = synth.activations(synth.rng(4, 0), args.width, hidden)
    per_step_rows = 2048
    times = []
    rows_done = 0
    for i in range(args.warmup + args.steps):
        lo = (i * per_step_rows) % (q_full.shape[0] - per_step_rows)
        q = np.ascontiguousarray(q_full[lo:lo + per_step_rows])
        s = np.ascontiguousarray(s_full[lo:lo + per_step_rows])
        t0 = time.perf_counter()
        oracle.gemm(Xb, q, s, synth.GSCALE)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            rows_done += per_step_rows
    total = sum(times)
    gbs = rows_done * hidden * (0.5 + 1 / 16) / total / 1e9
    sample = (f"float64 oracle GEMM, M={args.width}, {per_step_rows} rows of the round's layer-0 "
              f"q/k/v matrix (K={hidden}) per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / max(1, len(times)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": round_config(args, world, round_weight_bytes(args.layers, hidden, w4["ffn"], w4["vocab"]),
                               4 * args.layers + 1,
                               4 * args.layers + 1 if args.round_mode == "chain" else None),
        "cpu_baseline": {"value": gbs, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU legs

def gemm_sweep(dev, hbm_peak):
    """Single decode GEMMs per workload and width, timed on the device: each
    case is a chain of back-to-back launches captured as a C-ABI round (one
    graph, PDL between nodes), rotating through enough weight copies to
    exceed L2, and replayed under CUDA events."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, synth
    from nvfp4_weight_streaming_decode_b200.workloads import BYTES_PER_WEIGHT, make_matrix
    out = []
    stream = torch.cuda.Stream(device=dev)
    G, D = abi.NVFP4_DESC_GEMM, abi.NVFP4_DESC_GATEUP_SILU

    def time_chain(descs, reps=10):
        rnd = abi.Round(descs, abi.NVFP4_ROUND_CHAIN)
        with torch.cuda.stream(stream):
            for _ in range(3):
                rnd.replay(8, stream)
        torch.cuda.synchronize()
        res = {}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for M in range(1, 9):
            with torch.cuda.stream(stream):
                rnd.replay(M, stream)
                e0.record(stream)
                for _ in range(reps):
                    rnd.replay(M, stream)
                e1.record(stream)
            e1.synchronize()
            res[M] = e0.elapsed_time(e1) * 1e-3 / reps / len(descs)
        rnd.close()
        return res

    def add(name, t_by_m, wbytes, io):
        for M, t in t_by_m.items():
            b = wbytes + io(M)
            out.append({"workload": name, "M": M, "us": t * 1e6, "GBps": b / t / 1e9,
                        "frac": b / t / 1e9 / hbm_peak})

    X = synth.torch_activations(1, 8, 8, 17408, dev)
    # single projection N = K = 5120: 16 copies (236 MB > L2), 32 nodes
    mats = [make_matrix(1, 500 + c, 5120, 5120, dev) for c in range(16)]
    Y = torch.empty((8, 5120), dtype=torch.float32, device=dev)
    descs = [abi.desc(G, X, m.wq, m.ws, synth.GSCALE, Y, 5120, 5120) for m in mats + mats]
    add("proj_n5120_k5120", time_chain(descs), 5120 * 5120 * BYTES_PER_WEIGHT,
        lambda M: 2 * M * 5120 + 4 * M * 5120)
    del mats
    # head N = 151936, K = 5120 (438 MB > L2), 4 nodes
    head = make_matrix(3, 0, 151936, 5120, dev, synth.EXP_LOGU_M6_4)
    Yh = torch.empty((8, 151936), dtype=torch.float32, device=dev)
    descs = [abi.desc(G, X, head.wq, head.ws, synth.GSCALE, Yh, 151936, 5120)] * 4
    add("head_n151936_k5120", time_chain(descs, 5), 151936 * 5120 * BYTES_PER_WEIGHT,
        lambda M: 2 * M * 5120 + 4 * M * 151936)
    del head
    # fused MLP: gate/up 2 x 17408 x 5120 and down 5120 x 17408, 2 copies (300 MB > L2)
    sets = [(make_matrix(2, 600 + 3 * c, 17408, 5120, dev), make_matrix(2, 601 + 3 * c, 17408, 5120, dev),
             make_matrix(2, 602 + 3 * c, 5120, 17408, dev)) for c in range(2)]
    H = torch.empty((8, 17408), dtype=torch.bfloat16, device=dev)
    descs = [abi.desc(D, X, g.wq, g.ws, synth.GSCALE, H, 17408, 5120, u.wq, u.ws, synth.GSCALE)
             for (g, u, _) in sets + sets]
    add("mlp_gateup_2x17408_k5120", time_chain(descs), 2 * 17408 * 5120 * BYTES_PER_WEIGHT,
        lambda M: 2 * M * 5120 + 2 * M * 17408)
    descs = [abi.desc(G, X, d.wq, d.ws, synth.GSCALE, Y, 5120, 17408) for (_, _, d) in sets + sets]
    add("mlp_down_n5120_k17408", time_chain(descs), 5120 * 17408 * BYTES_PER_WEIGHT,
        lambda M: 2 * M * 17408 + 4 * M * 5120)
    del sets
    torch.cuda.synchronize()
    return out


def node_split(r, stream, widths, by_width):
    """Per node kind: the round's nodes of that kind alone, chained in one graph,
    device time per node at each width, and that kind's share of the round."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi
    kinds = {}
    for i, (name, _, _, _, _) in enumerate(r.nodes):
        kinds.setdefault(re.sub(r"\d+$", "", name), []).append(i)
    out = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for kind, idx in kinds.items():
        rnd = abi.Round([r.descs[i] for i in idx], abi.NVFP4_ROUND_CHAIN)
        reps = max(3, 200 // len(idx))
        res = {"nodes": len(idx)}
        for M in widths:
            with torch.cuda.stream(stream):
                for _ in range(3):
                    rnd.replay(M, stream)
                e0.record(stream)
                for _ in range(reps):
                    rnd.replay(M, stream)
                e1.record(stream)
            e1.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps / len(idx)
            res[f"us_per_node_M{M}"] = us
            if by_width.get(M):
                res[f"share_of_round_M{M}"] = us * len(idx) / (by_width[M] * 1e3)
        rnd.close()
        out[kind] = res
    for M in widths:
        if by_width.get(M):
            out[f"sum_over_kinds_ms_M{M}"] = sum(v[f"us_per_node_M{M}"] * v["nodes"] for k, v in out.items()
                                                  if isinstance(v, dict)) / 1e3
            out[f"round_ms_M{M}"] = by_width[M]
    return out


def round_io_bytes(r, M):
    """Algorithmic activation bytes of one round: X read and outputs written, per node."""
    from nvfp4_weight_streaming_decode_b200 import abi
    total = 0
    for (_, kind, _, _, mkeys) in r.nodes:
        m0 = r.mats[mkeys[0]]
        total += 2 * M * m0.K + (4 if kind == abi.NVFP4_DESC_GEMM else 2) * M * m0.N
    return total


def verify_sweep(dev, hbm_peak):
    """The decode GEMM at verify widths (M = 9..64: up to 32 on the decode
    kernel with several lane blocks, above on the tensor-memory kernel), timed
    on the device: for each workload and width, a CUDA graph of
    back-to-back nvfp4_gemm_decode calls rotating through enough weight
    copies to exceed L2, replayed under CUDA events."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, synth
    from nvfp4_weight_streaming_decode_b200.workloads import BYTES_PER_WEIGHT, make_matrix
    out = []
    s = torch.cuda.Stream(device=dev)
    X = synth.torch_activations(1, 9, 64, 17408, dev)
    cases = []
    mats = [make_matrix(1, 700 + c, 5120, 5120, dev) for c in range(16)]
    cases.append(("proj_n5120_k5120", [(m, 5120, 5120) for m in mats + mats]))
    head = make_matrix(3, 0, 151936, 5120, dev, synth.EXP_LOGU_M6_4)
    cases.append(("head_n151936_k5120", [(head, 151936, 5120)] * 4))
    downs = [make_matrix(2, 800 + c, 5120, 17408, dev) for c in range(4)]
    cases.append(("mlp_down_n5120_k17408", [(m, 5120, 17408) for m in downs + downs]))
    for name, calls in cases:
        N, K = calls[0][1], calls[0][2]
        for M in (9, 16, 24, 32, 40, 64):
            x = X[:M, :K].contiguous()
            Y = torch.empty((M, N), dtype=torch.float32, device=dev)
            with torch.cuda.stream(s):
                for (m, n_, k_) in calls:
                    abi.gemm_decode(x, m.wq, m.ws, synth.GSCALE, n_, k_, Y=Y, stream=s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for (m, n_, k_) in calls:
                    abi.gemm_decode(x, m.wq, m.ws, synth.GSCALE, n_, k_, Y=Y, stream=s)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            with torch.cuda.stream(s):
                g.replay()
                e0.record(s)
                for _ in range(reps):
                    g.replay()
                e1.record(s)
            e1.synchronize()
            t = e0.elapsed_time(e1) * 1e-3 / reps / len(calls)
            b = N * K * BYTES_PER_WEIGHT + 2 * M * K + 4 * M * N
            out.append({"workload": name, "M": M, "us": t * 1e6, "GBps": b / t / 1e9, "frac": b / t / 1e9 / hbm_peak,
                        "tflops": 2.0 * M * N * K / t / 1e12,
                        "kernel": ("decode_gemm_kernel, %d blocks of 8 lanes" % ((M + 7) // 8)) if M <= 32
                        else "verify_kernel (tcgen05.mma, accumulators in tensor memory)"})
            del g
    return {"kernel": "M = 9..32: decode_gemm_kernel (bf16 m16n8k16, 2..4 lane blocks); "
                      "M = 33..64: verify_kernel (tcgen05.mma, accumulators in tensor memory)", "cases": out}


def grouped_sweep(dev, hbm_peak):
    """Grouped expert decode (nvfp4_gemm_grouped) on 512 experts of the read
    Flash-Next shape: gate/up-like 768 x 2,048 (one input per lane) and
    down-like 2,048 x 768 (one input per route), for M = 1 and 8 lanes with 10
    picks each.  A CUDA graph of 8 calls rotating through 8 seeded route tables
    (so consecutive calls stream mostly different experts) is replayed under
    CUDA events; GB/s counts the distinct selected experts' bytes per call."""
    import numpy as np
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, synth
    from nvfp4_weight_streaming_decode_b200.workloads import BYTES_PER_WEIGHT, make_matrix
    out = []
    s = torch.cuda.Stream(device=dev)
    E, T = 512, 10
    for name, N, K, per_route in (("experts_768x2048", 768, 2048, False), ("experts_2048x768", 2048, 768, True)):
        m = make_matrix(5, 0 if N == 768 else 1, E * N, K, dev)
        kc = -(-K // 64)
        qb, sb = (N // 32) * kc * 1024, (N // 32) * kc * 128
        table = abi.expert_table([(m.wq[e * qb:(e + 1) * qb], m.ws[e * sb:(e + 1) * sb], synth.GSCALE)
                                  for e in range(E)], dev)
        for M in (1, 8):
            rng = np.random.default_rng(M * 31 + N)
            routes = [torch.from_numpy(np.stack([rng.choice(E, T, replace=False) for _ in range(M)]).astype(np.int32)).to(dev)
                      for _ in range(8)]
            uniq = np.mean([len(np.unique(r.cpu().numpy())) for r in routes])
            X = synth.torch_activations(5, 2, M * T if per_route else M, K, dev)
            Y = torch.empty((M, T, N), dtype=torch.float32, device=dev)
            with torch.cuda.stream(s):
                for r in routes:
                    abi.gemm_grouped(X, r, table, E, N, K, x_per_route=per_route, Y=Y, stream=s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for r in routes:
                    abi.gemm_grouped(X, r, table, E, N, K, x_per_route=per_route, Y=Y, stream=s)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s):
                g.replay()
                e0.record(s)
                for _ in range(10):
                    g.replay()
                e1.record(s)
            e1.synchronize()
            t = e0.elapsed_time(e1) * 1e-3 / 80
            b = uniq * N * K * BYTES_PER_WEIGHT
            out.append({"workload": name, "M": M, "T": T, "experts_per_call": float(uniq), "us": t * 1e6,
                        "GBps": b / t / 1e9, "frac": b / t / 1e9 / hbm_peak})
            del g
        del m, table
    return {"kernel": "grouped_kernel", "cases": out}


def percentile(xs, q):
    """q-th percentile of a list, linear between closest ranks (numpy's default)."""
    ys = sorted(xs)
    if not ys:
        return None
    pos = (len(ys) - 1) * q / 100.0
    lo = int(pos)
    hi = min(lo + 1, len(ys) - 1)
    return ys[lo] + (ys[hi] - ys[lo]) * (pos - lo)


def stream_read_peak(dev, stream, hbm_peak, gib=4, reps=10):
    """Read-only HBM bandwidth with the library's own probe (nvfp4_stream_read):
    one pass over a `gib` GiB buffer per launch, four CTAs per SM, best and
    median of `reps` launches under CUDA events.  A second denominator beside
    the measured copy peak; the roofline keeps the copy figure."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi
    nbytes = gib << 30
    buf = torch.zeros(nbytes // 4, dtype=torch.int32, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ctas = 4 * sms
    out = torch.empty((ctas,), dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            abi.stream_read(buf, ctas, out, stream)
    times = []
    for _ in range(reps):
        with torch.cuda.stream(stream):
            e0.record(stream)
            abi.stream_read(buf, ctas, out, stream)
            e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    del buf, out
    torch.cuda.empty_cache()
    best = nbytes / min(times) / 1e9
    return {"gbs": best, "median_gbs": nbytes / statistics.median(times) / 1e9, "bytes": nbytes, "ctas": ctas,
            "reps": reps, "of_copy_peak": best / hbm_peak,
            "kernel": "stream_read_kernel (nvfp4_stream_read: 16-byte cache-streaming loads, XOR per CTA)"}


def topk_detail(logits, dev, hbm_peak):
    """Device time of nvfp4_topk on the round's own head logits (FP32
    [8][151,936]), for rows 1 and 8 and k = 1, 8, 64: 50 calls captured in a
    CUDA graph, replayed 5 times, timed with CUDA events.  The logits were
    just written by the head, so they are L2-resident, as in a round."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi
    out = []
    V = logits.shape[1]
    s = torch.cuda.Stream(device=dev)
    for rows in (1, 8):
        for k in (1, 8, 64):
            x = logits[:rows]
            vals = torch.empty((rows, k), dtype=torch.float32, device=dev)
            idx = torch.empty((rows, k), dtype=torch.int32, device=dev)
            with torch.cuda.stream(s):
                abi.topk(x, k, values=vals, indices=idx, stream=s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(50):
                    abi.topk(x, k, values=vals, indices=idx, stream=s)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s):
                g.replay()
                e0.record(s)
                for _ in range(5):
                    g.replay()
                e1.record(s)
            e1.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / 250
            nbytes = rows * V * 4 + rows * k * 8
            st, splits, slice_ = abi.nvfp4_topk_splits(rows, V, k, torch.cuda.get_device_properties(dev).multi_processor_count)
            out.append({"rows": rows, "V": V, "k": k, "us": us, "GBps": nbytes / (us * 1e-6) / 1e9,
                        "frac": nbytes / (us * 1e-6) / 1e9 / hbm_peak, "splits": splits, "slice": slice_})
            del g
    return {"kernel": "topk_kernel", "l2": "logits L2-resident (just written by the head, as in a round)",
            "bytes": "rows*V*4 logits read + rows*k*8 written", "cases": out}


def run_gemm_case(args):
    """Three direct nvfp4_gemm_decode / nvfp4_gemm_gateup_silu calls on one workload matrix."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, build, synth
    from nvfp4_weight_streaming_decode_b200.workloads import make_matrix
    build.build()
    dev = torch.device("cuda", 0)
    M = args.width
    shapes = {"head": (151936, 5120, synth.EXP_LOGU_M6_4), "proj": (5120, 5120, synth.EXP_UNIFORM_M4_2),
              "qkv": (15360, 5120, synth.EXP_UNIFORM_M4_2),
              "gateup": (17408, 5120, synth.EXP_UNIFORM_M4_2), "down": (5120, 17408, synth.EXP_UNIFORM_M4_2)}
    N, K, exp = shapes[args.gemm_case]
    m = make_matrix(3, 0, N, K, dev, exp)
    X = synth.torch_activations(3, 1, M, K, dev)
    if args.gemm_case == "gateup":
        u = make_matrix(3, 1, N, K, dev, exp)
        for _ in range(3):
            abi.gemm_gateup_silu(X, m.wq, m.ws, synth.GSCALE, u.wq, u.ws, synth.GSCALE, N, K)
    else:
        for _ in range(3):
            abi.gemm_decode(X, m.wq, m.ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    print(json.dumps({"gemm_case": args.gemm_case, "M": M, "N": N, "K": K, "ok": True}))
    return 0


def run_grouped_case(args):
    """Three nvfp4_gemm_grouped calls: 512 seeded experts of 768 x 2,048, --width lanes with 10 picks
    each (three different seeded route tables)."""
    import numpy as np
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, build, synth
    from nvfp4_weight_streaming_decode_b200.workloads import make_matrix
    build.build()
    dev = torch.device("cuda", 0)
    E, T, N, K, M = 512, 10, 768, 2048, args.width
    m = make_matrix(5, 0, E * N, K, dev)
    qb, sb = (N // 32) * (K // 64) * 1024, (N // 32) * (K // 64) * 128
    table = abi.expert_table([(m.wq[e * qb:(e + 1) * qb], m.ws[e * sb:(e + 1) * sb], synth.GSCALE)
                              for e in range(E)], dev)
    rng = np.random.default_rng(7)
    X = synth.torch_activations(5, 2, M, K, dev)
    for _ in range(3):
        r = torch.from_numpy(np.stack([rng.choice(E, T, replace=False) for _ in range(M)]).astype(np.int32)).to(dev)
        abi.gemm_grouped(X, r, table, E, N, K)
    torch.cuda.synchronize()
    print(json.dumps({"grouped_case": True, "M": M, "T": T, "E": E, "N": N, "K": K, "ok": True}))


def run_topk_case(args):
    """Three nvfp4_topk calls over [--width][151,936] seeded N(0,1) logits."""
    import torch

    from nvfp4_weight_streaming_decode_b200 import abi, build
    build.build()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    x = torch.randn((args.width, 151936), generator=g, device=dev, dtype=torch.float32)
    for _ in range(3):
        abi.topk(x, args.topk_case)
    torch.cuda.synchronize()
    print(json.dumps({"topk_case": args.topk_case, "rows": args.width, "V": 151936, "ok": True}))
    return 0


def run_ours(args):
    import torch

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from nvfp4_weight_streaming_decode_b200 import abi, build, synth
    from nvfp4_weight_streaming_decode_b200.workloads import SyntheticRound
    build.build()
    abi.load()
    hbm_peak, peak_kind = peaks()
    M = args.width
    w = synth.WORKLOADS[4]

    r = SyntheticRound.build(dev, layers=args.layers, hidden=w["hidden"], ffn=w["ffn"], vocab=w["vocab"])
    mode = abi.NVFP4_ROUND_PERSISTENT if args.round_mode == "persistent" else abi.NVFP4_ROUND_CHAIN
    rnd = abi.Round(r.descs, mode)
    nodes = len(r.descs)          # GEMM nodes of the round (kernel launches in chain mode)
    graph_nodes = rnd.nodes
    weight_bytes = r.weight_bytes
    io_bytes = round_io_bytes(r, M)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            rnd.replay(M, stream)
    torch.cuda.synchronize()

    # per-width round times (detail): 20 warm-up replays, then 100 timed, an event
    # after every replay for the median and p90 beside the mean
    by_width, p50_by_width, p90_by_width = {}, {}, {}
    if args.profile:
        args.no_sweep = args.no_cpu_baseline = True
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_warm_detail, n_rep = 20, 100
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_rep + 1)]
    for m in (range(1, 9) if not args.profile else ()):
        with torch.cuda.stream(stream):
            for _ in range(n_warm_detail):
                rnd.replay(m, stream)
            evs[0].record(stream)
            for j in range(n_rep):
                rnd.replay(m, stream)
                evs[j + 1].record(stream)
        evs[-1].synchronize()
        per = [evs[j].elapsed_time(evs[j + 1]) for j in range(n_rep)]
        by_width[m] = evs[0].elapsed_time(evs[-1]) / n_rep
        p50_by_width[m] = statistics.median(per)
        p90_by_width[m] = percentile(per, 90)

    # host submission cost of one replay: host wall time around the C-ABI call that
    # launches the width's graph (through the Python binding), for 30 replays queued
    # back to back; its share of the round's device time (the pages' 2.2 %)
    submit = None
    if not args.profile:
        torch.cuda.synchronize()
        host_ns = []
        with torch.cuda.stream(stream):
            for _ in range(30):
                t0 = time.perf_counter_ns()
                rnd.replay(M, stream)
                host_ns.append(time.perf_counter_ns() - t0)
        torch.cuda.synchronize()
        med_us = statistics.median(host_ns) / 1e3
        submit = {"host_us_per_replay_p50": med_us, "host_us_per_replay_max": max(host_ns) / 1e3,
                  "share_of_round": med_us / (by_width.get(M, 0) * 1e3) if by_width.get(M) else None}

    # the timed region: K replays at width M
    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            rnd.replay(M, stream)
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed_s = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world)
    ms_per_step = elapsed_s * 1e3 / args.steps
    value = aggregate_gbps(weight_bytes, args.steps, elapsed_s, world)

    # end to end through the C ABI with host buffers: H2D of the layer-0 input,
    # the replay, D2H of the logits, every step
    x_host = torch.empty((M, w["hidden"]), dtype=torch.bfloat16).pin_memory()
    x_host.copy_(r.bufs["x0"][:M].cpu())
    y_host = torch.empty((M, w["vocab"]), dtype=torch.float32).pin_memory()
    e2e_steps = max(10, args.steps // 4) if not args.profile else 1
    with torch.cuda.stream(stream):
        for _ in range(3):
            rnd.replay_host(M, x_host, r.bufs["x0"], r.bufs["logits"][:M], y_host, stream)
        barrier(world)
        e0.record(stream)
        for _ in range(e2e_steps):
            rnd.replay_host(M, x_host, r.bufs["x0"], r.bufs["logits"][:M], y_host, stream)
        e1.record(stream)
    e1.synchronize()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world)
    e2e_value = aggregate_gbps(weight_bytes, e2e_steps, e2e_s, world)

    # roofline of the decode GEMM kernel over the round: every node is a launch of it
    launches = graph_nodes            # kernel launches per round: 1 (persistent) or one per GEMM node (chain)
    per_launch_bytes = (weight_bytes + io_bytes) / launches
    per_launch_s = (elapsed_s / args.steps) / launches
    achieved = per_launch_bytes / per_launch_s / 1e9
    traffic_round = profiled_traffic()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "traffic": (traffic_round / launches) if traffic_round else None,
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "kernel": ("round_kernel (persistent round, one launch per round)" if args.round_mode == "persistent"
                           else "decode_gemm_kernel (one launch per round node)")}

    read_peak = None
    if rank == 0 and not args.no_sweep:
        try:
            read_peak = stream_read_peak(dev, stream, hbm_peak)
        except (RuntimeError, MemoryError) as e:  # context only: never lose the bench line to it
            torch.cuda.synchronize()
            read_peak = {"gbs": None, "error": str(e)[:200]}

    topk = None
    if rank == 0 and not args.no_sweep:
        rnd.replay(8, stream)
        torch.cuda.synchronize()
        topk = topk_detail(r.bufs["logits"], dev, hbm_peak)

    # device-time split of the round by node kind: each kind's nodes of this round
    # alone, chained in their own graph (same matrices and buffers), timed at width M
    # and at width 1; the sum over kinds set against the live round
    split = None
    if rank == 0 and not args.no_sweep:
        split = node_split(r, stream, (1, M), by_width)

    sweep = None
    verify = None
    grouped = None
    if rank == 0 and not args.no_sweep:
        del rnd
        sweep = gemm_sweep(dev, hbm_peak)
        verify = verify_sweep(dev, hbm_peak)
        grouped = grouped_sweep(dev, hbm_peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, cores, sample = oracle_sample(dev, 12.0)
        cpu = {"value": gbs, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random NVFP4 codes/scales, N(0,1) bf16 activations)",
            "config": round_config(args, world, weight_bytes, nodes, graph_nodes),
            "round_ms": ms_per_step,
            "round_ms_by_width": by_width,
            "round_GBps_by_width": {m: weight_bytes / (t * 1e-3) / 1e9 for m, t in by_width.items()},
            "round_frac_by_width": {m: weight_bytes / (t * 1e-3) / 1e9 / hbm_peak for m, t in by_width.items()},
            "round_frac_of_nominal_by_width": {m: weight_bytes / (t * 1e-3) / 1e9 / NOMINAL_HBM_GBS
                                               for m, t in by_width.items()},
            "round_ms_p50_by_width": p50_by_width,
            "round_ms_p90_by_width": p90_by_width,
            "read_peak": read_peak,
            "round_frac_of_read_peak": (value / read_peak["gbs"]) if read_peak and read_peak["gbs"] else None,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": x_host.numel() * 2,
                    "d2h_bytes_per_step": y_host.numel() * 4, "ms_per_step": e2e_s * 1e3 / e2e_steps},
            "gpu_launches": graph_nodes * args.steps,
            "submission": submit,
            "node_split": split,
            "clocks": clk,
            "gemm_sweep": sweep,
            "topk": topk,
            "verify_widths": verify,
            "grouped_experts": grouped,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.gemm_case:
        return run_gemm_case(args)
    if args.topk_case:
        return run_topk_case(args)
    if args.grouped_case:
        return run_grouped_case(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
