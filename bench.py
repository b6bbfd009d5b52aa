"""Benchmark of the MSA training hot path (Index Branch + Main Branch forward
and backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 128k] [--impl ours|reference]

One step = msa_proxy_select + msa_fwd + msa_bwd over one synthetic batch of
the chosen workload, inputs resident in HBM.  Under torchrun every rank runs
its own batch (seed = rank): the path shards by independent problems with no
collective, so scaling is weak.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle (the plain C implementation the
tests check against) on a bounded sample of query rows of the same workload,
on the host cores, and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA fwd+bwd TFLOP/s (selected-block FLOPs) and tokens/s at T=128K; % of bf16 peak"
BLOCK = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=0, help="query rows in the CPU sample (0 = auto)")
    ap.add_argument("--decode", action="store_true",
                    help="time msa_decode (one new token per sequence against full-length caches) instead")
    ap.add_argument("--decode-batch", type=int, default=16, help="sequences per decode step")
    ap.add_argument("--cp", action="store_true",
                    help="context parallel: one sequence of the workload split by rows over the ranks "
                         "(key-side all-gather, dK/dV reduce-scatter); strong scaling")
    ap.add_argument("--window", type=int, default=1, help="forced blocks per query (own block included)")
    ap.add_argument("--dilation", type=int, default=1, help="stride between forced blocks")
    ap.add_argument("--bias", default=None, choices=["none", "group", "recency"],
                    help="override the workload's proxy-input structure (profiling variants)")
    ap.add_argument("--outliers", type=int, default=0,
                    help="large-norm (x8) key rows per (batch, group): the attention-sink-like variant")
    ap.add_argument("--proxy-grad", action="store_true",
                    help="also time the proxy-head gradient (forward keeping block masses + msa_proxy_bwd)")
    ap.add_argument("--groups", type=int, default=0,
                    help="run only this many of the workload's KV groups (same per-group shape; profiling "
                         "captures scale their counters by the group ratio)")
    return ap.parse_args()


def workload_name(cfg, window=1, dilation=1):
    bias = {"none": "", "group": ", per-group low-rank proxy bias", "recency": ", planted local-recency proxy bias"}
    pattern = f", forced window {window} blocks at dilation {dilation}" if window > 1 else ""
    outl = f", {cfg.k_outliers} large-norm (x8) keys per group" if cfg.k_outliers else ""
    return (f"MSA {cfg.name}: B={cfg.B} T={cfg.T} Hq={cfg.Hq} Hkv={cfg.Hkv} d={cfg.d} dp={cfg.dp} "
            f"topk={cfg.topk} (own block incl.), causal, fwd+bwd{bias[cfg.bias]}{pattern}{outl}")


# ---------------------------------------------------------------- FLOP model
def flops_from_nsel(cfg, nsel_counts):
    """Selected-block FLOPs of one batch.  pairs(i) = keys query i reads =
    128 (nsel_i - 1) + (i mod 128) + 1 (other selected blocks whole, own block
    up to i); forward 4 d per (query head, key) pair (QK^T and PV), backward
    2.5x forward; proxy 2 dp per (query, key) pair over the key blocks the
    selection actually scores (blocks before the query's own, for query
    tiles with more eligible blocks than topk)."""
    total_pairs = nsel_counts["pairs"]
    f_fwd = 4.0 * cfg.d * cfg.G * total_pairs
    f_bwd = 2.5 * f_fwd
    f_proxy = 0.0
    if cfg.topk > 1:
        for qb in range((cfg.T + BLOCK - 1) // BLOCK):
            if qb + 1 > cfg.topk:
                rows = min(BLOCK, cfg.T - qb * BLOCK)
                f_proxy += 2.0 * cfg.dp * rows * BLOCK * qb
        f_proxy *= cfg.B * cfg.Hp
    return f_proxy, f_fwd, f_bwd


def pair_count(cfg, nsel, r0=0):
    """Selected (query, key) pairs of the rows r0 .. r0 + nsel.shape[2] - 1
    whose selection sizes nsel [B, Hp, rows] holds."""
    import torch
    i = torch.arange(r0, r0 + nsel.shape[2], device=nsel.device, dtype=torch.int64)
    own = (i % BLOCK) + 1
    pairs = BLOCK * (nsel.to(torch.int64) - 1) + own.view(1, 1, -1)
    return {"pairs": float(pairs.sum().item())}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id):
        self.device_id = device_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.device_id)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def sources_sha256(names):
    """sha256 over the named files under the package's csrc/, in order (the
    key a committed traffic record was taken with); None if one is missing."""
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_attention_09_b200", "csrc")
    h = hashlib.sha256()
    for name in names:
        fp = os.path.join(csrc, name)
        if not os.path.exists(fp):
            return None
        with open(fp, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    record profiles/traffic.json (the capture's bytes times its stated scale
    to the full launch), or None when there is none or the kernel's sources
    have changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    for r in rec.get("records", []):
        if r.get("kernel") == kernel and r.get("workload") == workload:
            if sources_sha256(r["sources"]) != r["sources_sha256"]:
                return None
            return float(r["bytes_per_launch_captured"]) * float(r["scale_to_full"])
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------- ranks
def combine_ranks(dist, world, device, ms, units):
    """Whole-job figures of a weak-scaling run: each rank times its own batch,
    the job takes as long as the slowest rank (max of ms) and does the work of
    all ranks (sum of units).  One all-reduce each, same order on every rank."""
    if world <= 1:
        return ms, units
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ---------------------------------------------------------------- CPU oracle timing
def oracle_arrays(host):
    """float32 copies of the bf16 inputs (exact) for the oracle."""
    return {k: v.float().numpy() for k, v in host.items()}


def cpu_oracle_sample(cfg, x, rows_target, seed=0, window=1, dilation=1):
    """Time the oracle on a bounded sample of query rows (b, g, i) of the
    workload: selection (proxy scores of the row over all earlier keys, pool,
    top-k), then forward, dQ and the row's dK/dV contributions for each of
    the group's G heads.  Returns (credited FLOPs, seconds, rows, threads)."""
    import oracle as O
    from block_sparse_attention_09_b200.inputs import sample_rows
    m = O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=cfg.topk, window=window,
               dilation=dilation)
    threads = os.cpu_count() or 1
    srows = sample_rows(cfg.B * cfg.Hkv * cfg.T, rows_target, seed=seed + 11)
    t0 = time.perf_counter()
    idx, nsel, _ = O.select(m, x["qp"], x["kp"], rows=srows, nthreads=threads)
    qrows = []
    for r in srows:
        i = r % cfg.T
        bg = r // cfg.T
        b, g = divmod(bg, cfg.Hkv)
        for hh in range(cfg.G):
            qrows.append((b * cfg.Hq + g * cfg.G + hh) * cfg.T + i)
    o, lse = O.fwd(m, x["q"], x["k"], x["v"], idx, nsel, rows=qrows, nthreads=threads)
    dq, D = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o, lse, idx, nsel, rows=qrows, nthreads=threads)
    for c0 in range(0, len(qrows), 32):   # contributions are topk*128*d doubles per row: chunk them
        O.bwd_kv_rows(m, x["q"], x["k"], x["v"], x["dout"], lse, D, idx, nsel, rows=qrows[c0:c0 + 32],
                      nthreads=threads)
    secs = time.perf_counter() - t0
    flops = 0.0
    for r in srows:
        i = r % cfg.T
        bg = r // cfg.T
        b, g = divmod(bg, cfg.Hkv)
        bi = i // BLOCK
        ns = int(nsel[b, g, i])
        pairs = BLOCK * (ns - 1) + (i % BLOCK) + 1
        f_fwd = 4.0 * cfg.d * cfg.G * pairs
        f_proxy = 2.0 * cfg.dp * BLOCK * bi if (bi + 1 > cfg.topk and cfg.topk > 1) else 0.0
        flops += f_proxy + 3.5 * f_fwd
    return flops, secs, len(srows), threads


def calibrate_rows(cfg, x, seconds, cap=4096, window=1, dilation=1):
    """Rows of the CPU sample that take about `seconds` on this host."""
    fl, secs, n, _ = cpu_oracle_sample(cfg, x, 32, seed=99, window=window, dilation=dilation)
    return max(8, min(cap, int(n * seconds / max(secs, 1e-3))))


def run_reference(args, cfg, rank):
    if rank != 0:
        return
    from block_sparse_attention_09_b200.inputs import make_inputs
    x = oracle_arrays(make_inputs(cfg, seed=0))
    rows = args.cpu_rows or calibrate_rows(cfg, x, seconds=4.0, window=args.window, dilation=args.dilation)
    vals = []
    for s in range(args.warmup + args.steps):
        fl, secs, n, threads = cpu_oracle_sample(cfg, x, rows, seed=s, window=args.window, dilation=args.dilation)
        if s >= args.warmup:
            vals.append((fl, secs))
    fl = sum(v[0] for v in vals)
    secs = sum(v[1] for v in vals)
    value = fl / secs / 1e12
    sample = f"{rows} query rows (b, group, i) per step, all {cfg.G} heads each, same workload and seeds"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(vals),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_name(cfg, args.window, args.dilation)},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- decode arm
def run_decode(args, cfg, rank, local):
    """Decode step: every sequence of the batch attends with one new token to
    caches of the workload's full length T.  Caches are seeded N(0,1) bf16
    drawn on the device (the timing does not depend on their values).  Metric:
    tokens/s; roofline: the HBM bytes a step must read (the proxy-key scan and
    the selected K/V tiles) over the decode kernels' time."""
    import torch
    from block_sparse_attention_09_b200 import msa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, T, Hq, Hkv, D, dp, k = args.decode_batch, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    mk = lambda *shape: torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    kc, vc, kpc = mk(B, T, Hkv, D), mk(B, T, Hkv, D), mk(B, T, Hkv, dp)
    q, qp = mk(B, Hq, D), mk(B, Hkv, dp)
    dims = msa.make_dims(B, T, Hq, Hkv, D, dp, k, window=args.window, dilation=args.dilation)
    ws = msa.workspace(dims, msa.MSA_DECODE, dev)
    out = (torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev), torch.empty((B, Hq), dtype=torch.float32, device=dev),
           torch.empty((B, Hkv, k), dtype=torch.int32, device=dev), torch.empty((B, Hkv), dtype=torch.int32, device=dev))
    step = lambda: msa.decode(q, qp, kc, vc, kpc, k, ws=ws, out=out, window=args.window, dilation=args.dilation)
    step()
    if msa.check_status(ws) != 0:
        raise RuntimeError("device status on the decode workload")
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    steps = max(args.steps, 20)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = msa.kernel_launches()
    a.record()
    for _ in range(steps):
        step()
    b_.record()
    torch.cuda.synchronize()
    launches = msa.kernel_launches() - l0
    ms = a.elapsed_time(b_) / steps
    # bytes a step must read: the proxy keys of every position, and the selected K and V rows
    nb = (T + 127) // 128
    rows_sel = min(k, nb) * 128
    bytes_step = B * Hkv * (T * dp * 2 + 2 * rows_sel * D * 2)
    peaks, src = measured_peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    line = {"metric": "MSA decode tokens/s (one new token per sequence, full-length caches)",
            "value": B / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": max(args.warmup, 3),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) bf16 caches drawn on the device",
            "config": {"workload": (f"MSA decode: {B} sequences x 1 new token, caches T={T} Hq={Hq} Hkv={Hkv} d={D} "
                                    f"dp={dp} topk={k} (own block incl.)"
                                    + (f", forced window {args.window} at dilation {args.dilation}"
                                       if args.window > 1 else "")),
                       "batch": B, "T": T, "Hq": Hq, "Hkv": Hkv, "d": D, "dp": dp, "topk": k,
                       "l2": "caches larger than L2 (proxy keys alone %.2f GB), no flush" % (B * T * Hkv * dp * 2 / 1e9)},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": gbs / float(peaks["hbm_gbs"]), "traffic": None,
                         "algorithmic_bytes_per_step": bytes_step, "peak_source": src},
            "gpu_launches": launches}
    print(json.dumps(line), flush=True)


def run_cp(args, cfg, rank, local, world):
    """Context-parallel step: the workload's sequence split into zig-zag
    chunks of 128-row blocks over the ranks (block_sparse_attention_09_b200.cp):
    all-gather of k, v, kp, each rank's selection, forward and backward of its
    own query rows, reduce-scatter of the fp32 partial dK/dV.  The work is fixed as the
    ranks grow (strong scaling); value = FLOPs of the whole sequence's step /
    the slowest rank's time."""
    import torch
    import torch.distributed as dist
    from block_sparse_attention_09_b200 import cp, msa
    from block_sparse_attention_09_b200.inputs import make_inputs
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)
    chunks = cp.shard_chunks(cfg.T, world, rank)
    host = make_inputs(cfg, seed=0)   # the same sequence on every rank; each keeps its rows
    d = {k: cp.take_rows(v, chunks).to(dev) for k, v in host.items()}
    del host

    def step():
        return cp.step(d["q"], d["k"], d["v"], d["dout"], d["qp"], d["kp"], cfg.topk, cfg.T, return_selection=True)

    out = step()
    nsel = out[6]
    # selected-key pairs of this rank's rows (chunk by chunk), summed over the ranks
    own, at = 0.0, 0
    for c0, c1 in chunks:
        own += pair_count(cfg, nsel[:, :, at:at + c1 - c0], c0)["pairs"]
        at += c1 - c0
    pairs = torch.tensor([own], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(pairs)
    f_proxy, f_fwd, f_bwd = flops_from_nsel(cfg, {"pairs": float(pairs.item())})
    f_step = f_proxy + f_fwd + f_bwd
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0 = msa.kernel_launches()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        step()
    b_.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = a.elapsed_time(b_) / args.steps
    launches = msa.kernel_launches() - l0
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks, src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    tflops = f_step / (ms * 1e-3) / 1e12
    line = {"metric": METRIC + " (context parallel)", "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) bf16 inputs" + (", planted local-recency proxy bias" if cfg.bias == "recency" else ""),
            "config": {"workload": workload_name(cfg) + f", rows split over {world} ranks (zig-zag chunks)",
                       "B": cfg.B, "T": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d, "dp": cfg.dp,
                       "topk": cfg.topk, "parallelism": f"cp{world}",
                       "l2": "inputs larger than L2, no flush"},
            "tokens_per_s": cfg.B * cfg.T / (ms * 1e-3),
            "flops_per_step": {"proxy": f_proxy, "fwd": f_fwd, "bwd": f_bwd},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "traffic": None,
                         "peak_source": f"{src} bf16 sustained (whole step, collectives included)"},
            "cpu_baseline": None, "e2e": None,
            "gpu_launches": launches}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def main():
    args = parse()
    from block_sparse_attention_09_b200.inputs import CONFIGS, make_inputs
    cfg = CONFIGS[args.config]
    if args.bias is not None:
        cfg = cfg.with_(bias=args.bias)
    if args.outliers:
        cfg = cfg.with_(k_outliers=args.outliers)
    if args.groups:
        cfg = cfg.with_(name=f"{cfg.name}-g{args.groups}", Hkv=args.groups, Hq=args.groups * cfg.G)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return
    if args.decode:
        run_decode(args, cfg, rank, local)
        return
    if args.cp:
        run_cp(args, cfg, rank, local, world)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)
    from block_sparse_attention_09_b200 import msa

    # ---- inputs: seeded, generated on the host, one batch per rank
    host = make_inputs(cfg, seed=rank)
    host = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    torch.cuda.synchronize()
    B, T, Hq, Hkv, D = cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d
    dims = msa.make_dims(B, T, Hq, Hkv, D, cfg.dp, cfg.topk)
    ws_sel = msa.workspace(dims, msa.MSA_SELECT, dev)
    ws_fwd = msa.step_workspace(dims, dev)   # the backward reuses the forward's inverse index
    ws_bwd = ws_fwd
    o = torch.empty_like(d["q"])
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    stream = torch.cuda.current_stream()

    def step(inputs, ev=None):
        if ev is not None:
            ev[0].record(stream)
        idx, nsel = msa.proxy_select(inputs["qp"], inputs["kp"], cfg.topk, ws=ws_sel, window=args.window,
                                     dilation=args.dilation)
        if ev is not None:
            ev[1].record(stream)
        msa.fwd(inputs["q"], inputs["k"], inputs["v"], idx, nsel, ws=ws_fwd, out=(o, lse))
        if ev is not None:
            ev[2].record(stream)
        msa.bwd(inputs["q"], inputs["k"], inputs["v"], o, inputs["dout"], lse, idx, nsel, ws=ws_bwd,
                out=(dq, dk, dv), reuse_index=True)
        if ev is not None:
            ev[3].record(stream)
        return idx, nsel

    # correctness guard on the timed configuration: every call's device status
    # word clean (each call resets its status, so each is read right after it)
    idx, nsel = msa.proxy_select(d["qp"], d["kp"], cfg.topk, ws=ws_sel, window=args.window,
                                 dilation=args.dilation, check=True)
    msa.fwd(d["q"], d["k"], d["v"], idx, nsel, ws=ws_fwd, out=(o, lse), check=True)
    fallback = msa.fallback_rows(ws_fwd)   # rows the forward redid with its exact two-pass softmax
    msa.bwd(d["q"], d["k"], d["v"], o, d["dout"], lse, idx, nsel, ws=ws_bwd, out=(dq, dk, dv), reuse_index=True,
            check=True)
    f_proxy, f_fwd, f_bwd = flops_from_nsel(cfg, pair_count(cfg, nsel))
    f_step = f_proxy + f_fwd + f_bwd

    for _ in range(args.warmup):
        step(d)
    torch.cuda.synchronize()

    kernel_names = {msa.KERNEL_PROXY: "proxy_select", msa.KERNEL_FWD_MAIN: "fwd_main",
                    msa.KERNEL_BWD_MAIN: "bwd_main"}
    kev = {k: [] for k in kernel_names}
    pev = []
    try:
        gpu_id = str(torch.cuda.get_device_properties(local).uuid)
        gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    except Exception:
        gpu_id = str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = msa.kernel_launches()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        for kk in kernel_names:
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)      # torch creates the CUDA event on first record;
            b_.record(stream)     # the library records it again around the kernel
            kev[kk].append((a, b_))
            msa.set_kernel_events(kk, a, b_)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        pev.append(ev)
        step(d, ev)
    t_stop.record(stream)
    torch.cuda.synchronize()
    launches = msa.kernel_launches() - launches0
    for kk in kernel_names:
        msa.set_kernel_events(kk, None, None)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = t_start.elapsed_time(t_stop) / args.steps
    ms, f_job = combine_ranks(dist, world, dev, ms, f_step)

    phase = {"proxy_select": [], "fwd": [], "bwd": []}
    for ev in pev:
        phase["proxy_select"].append(ev[0].elapsed_time(ev[1]))
        phase["fwd"].append(ev[1].elapsed_time(ev[2]))
        phase["bwd"].append(ev[2].elapsed_time(ev[3]))
    phase_ms = {k: statistics.mean(v) for k, v in phase.items()}
    kern_ms = {kernel_names[k]: statistics.mean(a.elapsed_time(b_) for a, b_ in v) for k, v in kev.items()}

    # ---- the proxy-head gradient (reported apart from the step's metric)
    proxy_grad = None
    if args.proxy_grad:
        ws_pg = msa.proxy_workspace(dims, dev)
        pg_out = (torch.empty(d["qp"].shape, dtype=torch.float32, device=dev),
                  torch.empty(d["kp"].shape, dtype=torch.float32, device=dev),
                  torch.empty((B, cfg.Hkv, T), dtype=torch.float32, device=dev))

        def pg_step(ev=None):
            ix, ns = msa.proxy_select(d["qp"], d["kp"], cfg.topk, ws=ws_sel)
            if ev is not None:
                ev[0].record(stream)
            msa.fwd(d["q"], d["k"], d["v"], ix, ns, ws=ws_pg, out=(o, lse), block_mass=True)
            if ev is not None:
                ev[1].record(stream)
            msa.bwd(d["q"], d["k"], d["v"], o, d["dout"], lse, ix, ns, ws=ws_pg, out=(dq, dk, dv), reuse_index=True)
            if ev is not None:
                ev[2].record(stream)
            msa.proxy_bwd(d["q"], d["qp"], d["kp"], ix, ns, ws_pg, out=pg_out)
            if ev is not None:
                ev[3].record(stream)

        pg_step()
        if msa.check_status(ws_pg) != 0:
            raise RuntimeError("device status after the proxy-head gradient")
        for _ in range(args.warmup):
            pg_step()
        evs = []
        for _ in range(args.steps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            evs.append(ev)
            pg_step(ev)
        torch.cuda.synchronize()
        proxy_grad = {"fwd_with_block_mass_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
                      "proxy_bwd_ms": statistics.mean(e[2].elapsed_time(e[3]) for e in evs),
                      "loss_sum": float(pg_out[2].double().sum().item())}
        del ws_pg, pg_out

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # End to end through the public API: every step copies its inputs from
        # pinned host memory and its results (O, dQ, dK, dV) back.  Two device
        # buffer sets let the copies of one step overlap the compute of its
        # neighbours (H2D and D2H on their own streams, ordered by events).
        out_host = {"o": torch.empty_like(o, device="cpu").pin_memory(),
                    "dq": torch.empty_like(dq, device="cpu").pin_memory(),
                    "dk": torch.empty_like(dk, device="cpu").pin_memory(),
                    "dv": torch.empty_like(dv, device="cpu").pin_memory()}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(v.numel() * v.element_size() for v in out_host.values())
        e_steps = max(4, args.steps)   # the same K as the device-timed steps
        d_in = [d, {k: torch.empty_like(v) for k, v in d.items()}]
        d_out = [(o, lse, dq, dk, dv),
                 (torch.empty_like(o), torch.empty_like(lse), torch.empty_like(dq), torch.empty_like(dk),
                  torch.empty_like(dv))]
        hs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        # the inputs go over in the order the step reads them (proxy pair, then
        # q/k/v, then dout), each group with its own event, so the selection
        # starts while the rest is still on its way; O goes back after the
        # forward, the gradients after the backward
        groups = (("qp", "kp"), ("q", "k", "v"), ("dout",))
        in_ready = [[torch.cuda.Event() for _ in groups] for _ in range(2)]
        fwd_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n, t0=None, t1=None):
            if t0 is not None:
                t0.record(stream)
                hs.wait_stream(stream)
            for kk in range(n):
                sb = kk % 2
                if kk >= 2:
                    hs.wait_event(comp_done[sb])          # set sb's inputs no longer read
                with torch.cuda.stream(hs):
                    for gi, names in enumerate(groups):   # this step's inputs
                        for name in names:
                            d_in[sb][name].copy_(host[name], non_blocking=True)
                        in_ready[sb][gi].record(hs)
                if kk >= 2:
                    stream.wait_event(out_done[sb])       # set sb's outputs copied out
                oo, ll, qq, kk_, vv = d_out[sb]
                inp = d_in[sb]
                stream.wait_event(in_ready[sb][0])
                ix, ns = msa.proxy_select(inp["qp"], inp["kp"], cfg.topk, ws=ws_sel, window=args.window,
                                          dilation=args.dilation)
                stream.wait_event(in_ready[sb][1])
                msa.fwd(inp["q"], inp["k"], inp["v"], ix, ns, ws=ws_fwd, out=(oo, ll))
                fwd_done[sb].record(stream)
                stream.wait_event(in_ready[sb][2])
                msa.bwd(inp["q"], inp["k"], inp["v"], oo, inp["dout"], ll, ix, ns, ws=ws_bwd, out=(qq, kk_, vv),
                        reuse_index=True)
                comp_done[sb].record(stream)
                with torch.cuda.stream(ds):               # this step's results
                    ds.wait_event(fwd_done[sb])
                    out_host["o"].copy_(oo, non_blocking=True)
                    ds.wait_event(comp_done[sb])
                    out_host["dq"].copy_(qq, non_blocking=True)
                    out_host["dk"].copy_(kk_, non_blocking=True)
                    out_host["dv"].copy_(vv, non_blocking=True)
                    out_done[sb].record(ds)
            stream.wait_stream(ds)
            stream.wait_stream(hs)
            if t1 is not None:
                t1.record(stream)

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(e_steps, a, b_)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b_) / e_steps
        e_ms, _ = combine_ranks(dist, world, dev, e_ms, f_step)
        e2e = {"value": f_job / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelining": "two buffer sets; H2D, compute and D2H of neighbouring steps overlap; inputs copied "
                               "in the order the step reads them, O copied back after the forward"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = measured_peaks()
    tflops = f_job / (ms * 1e-3) / 1e12
    tok_s = world * B * T / (ms * 1e-3)
    # dominant kernel of the step
    kf = {"proxy_select": f_proxy, "fwd_main": f_fwd, "bwd_main": f_bwd}
    dom = max(kern_ms, key=lambda k: kern_ms[k])
    achieved = kf[dom] / (kern_ms[dom] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": recorded_traffic(dom, cfg.name),
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
            "frac_of_burst": achieved / float(peaks.get("bf16_tflops", peak))}

    phase_rates = {"proxy_select": f_proxy / (phase_ms["proxy_select"] * 1e-3) / 1e12,
                   "fwd": f_fwd / (phase_ms["fwd"] * 1e-3) / 1e12,
                   "bwd": f_bwd / (phase_ms["bwd"] * 1e-3) / 1e12,
                   "fwd+bwd": (f_fwd + f_bwd) / ((phase_ms["fwd"] + phase_ms["bwd"]) * 1e-3) / 1e12}

    cpu = None
    if not args.no_cpu and world == 1:
        x = oracle_arrays(host)
        rows = args.cpu_rows or calibrate_rows(cfg, x, seconds=15.0, window=args.window, dilation=args.dilation)
        fl, secs, n, threads = cpu_oracle_sample(cfg, x, rows, seed=0, window=args.window, dilation=args.dilation)
        cpu = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} query rows (b, group, i) of the same workload, all {cfg.G} heads each: "
                         f"selection, forward, dQ and dK/dV contributions; {secs:.1f} s"}

    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 inputs" + (", planted local-recency proxy bias" if cfg.bias == "recency" else ""),
        "config": {"workload": workload_name(cfg, args.window, args.dilation), "B": B, "T": T, "Hq": Hq, "Hkv": Hkv, "d": D,
                   "dp": cfg.dp, "topk": cfg.topk, "per_rank": "one batch per rank (seed = rank)",
                   "l2": "inputs larger than L2 (Q alone %.2f GB), no flush" % (d["q"].numel() * 2 / 1e9)},
        "tokens_per_s": tok_s,
        "frac_of_peak": tflops / float(peaks.get("bf16_tflops")),
        "flops_per_step": {"proxy": f_proxy, "fwd": f_fwd, "bwd": f_bwd},
        "phases_ms": phase_ms,
        "phase_tflops": phase_rates,
        "kernel_ms": kern_ms,
        # the same rates as fractions of the sustained bf16 peak (the proxy
        # selection and the fwd+bwd pair are the two targets named for the path)
        "phase_frac_of_peak": {k: v / peak for k, v in phase_rates.items()},
        # tokens/s of the main branch alone (forward + backward, no selection)
        "tokens_per_s_main": world * B * T / ((phase_ms["fwd"] + phase_ms["bwd"]) * 1e-3),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "fallback_rows": fallback,
        "proxy_grad": proxy_grad,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
