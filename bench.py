"""Decode-indexer benchmark: keys scored per second for one LatentIndex layer
group's decode step, hierarchical selection (HS) and the DSA-style per-layer
path, on synthetic inputs.

A step (default workload: 4 sequences at 128K context, e4m3 latent with a
per-token fp32 scale, 64 heads, d_c = 192, d_k = 128, k = 2048, B = 8192,
G = 4) is, for every sequence:
  HS path : build the anchor latent of the new token (W_down h, d_model 7168)
            and append it; absorb the 4 layers' queries; the anchor scans its
            full prefix and proposes the top-B candidates and its top-k; 3
            followers gather the candidates, rescore and select top-k.
  DSA path: per layer, build and append the new key (W_k h), convert the raw
            query, scan the layer's key cache and select top-k.
Keys scored per step = sum_b (N_b + 3 min(B, N_b)) + 4 sum_b N_b.

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Multi-GPU: one process per GPU (torchrun); every rank runs the same step on
its own sequences (weak scaling, no collective on the data path).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import construction_inputs, generate, workload  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
METRIC = "decode indexer keys scored/s and % HBM roofline at 8K-128K ctx; HS vs DSA path"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


def keys_per_step(wl, lengths):
    hs = sum(int(n) + (wl.group - 1) * min(wl.B, int(n)) for n in lengths)
    dsa = wl.group * sum(int(n) for n in lengths)
    return hs, dsa


def config_of(wl, paths="HS + DSA-style, with construction"):
    return {"workload": f"{wl.name}: batch {wl.batch}, ctx {wl.length_range[1]}, {wl.cache_dtype} cache, "
                        f"H {wl.heads}, d_k {wl.d_k}, d_c {wl.d_c}, k {wl.k}, B {wl.B}, G {wl.group}",
            "batch": wl.batch, "ctx": wl.length_range[1], "cache": wl.cache_dtype, "heads": wl.heads,
            "d_k": wl.d_k, "d_c": wl.d_c, "k": wl.k, "B": wl.B, "group": wl.group, "d_model": wl.d_model,
            "paths": paths, "l2": "flushed before every step (256 MiB write, outside the timed events)"}


# ------------------------------------------------------------------ CPU oracle leg

def oracle_sample_step(inp, b, hnew, Wd, Wk):
    """The oracle's version of one sequence's group step (HS + DSA-style, with
    construction of the new token's latent and keys)."""
    from oracle import indexer
    wl = inp.wl
    n = int(inp.lengths[b])
    c = inp.latent[b, :n].astype(np.float64)
    indexer.latent(hnew[b], Wd)                          # anchor latent of the new token
    qt0, _ = indexer.absorb(inp.q[0][b, 0], inp.W_K[0])
    s0 = indexer.score(c, qt0, inp.w[0][b, 0])
    cand, cn, _ = indexer.hs_anchor(s0, wl.B, wl.k, n)
    for l in range(1, wl.group):
        qt, _ = indexer.absorb(inp.q[l][b, 0], inp.W_K[l])
        sc = indexer.score(c[cand[:cn]], qt, inp.w[l][b, 0])
        indexer.hs_follower(sc, cand, cn, wl.k)
    for l in range(wl.group):
        indexer.latent(hnew[b], Wk[l])                   # the layer's new key
        s = indexer.dsa_score(c, inp.W_K[l], inp.q[l][b, 0], inp.w[l][b, 0])
        indexer.topk(s, wl.k, n)
    return n + (wl.group - 1) * min(wl.B, n) + wl.group * n


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(args.workload)
    inp = generate(wl)
    hnew, Wd, Wk = construction_inputs(wl)
    for _ in range(args.warmup):
        oracle_sample_step(inp, 0, hnew, Wd, Wk)
    t0 = time.perf_counter()
    keys = 0
    for _ in range(args.steps):
        keys += oracle_sample_step(inp, 0, hnew, Wd, Wk)
    dt = time.perf_counter() - t0
    v = keys / dt
    sample = f"sequence 0 of {wl.batch} per step (HS + DSA-style group step, fp64 NumPy oracle)"
    cores = cpu_cores()
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": config_of(wl),
           "cpu_baseline": {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return 0


def cpu_baseline(inp, hnew, Wd, Wk, budget_s=20.0):
    keys, t0 = 0, time.perf_counter()
    reps = 0
    while True:
        keys += oracle_sample_step(inp, reps % inp.wl.batch, hnew, Wd, Wk)
        reps += 1
        if time.perf_counter() - t0 > budget_s / 2 or reps >= inp.wl.batch:
            break
    dt = time.perf_counter() - t0
    return {"value": keys / dt, "unit": "keys/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{reps} of {inp.wl.batch} sequences of one step (HS + DSA-style), fp64 NumPy, {dt:.1f} s"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nme, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nme)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ roofline inputs

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def scan_source_hash():
    h = hashlib.sha256()
    for name in ("scan.cu", "sm100.cuh", "internal.h"):
        with open(os.path.join(ROOT, "cross_layer_latent_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kind):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source."""
    try:
        with open(os.path.join(ROOT, "profiles", "scan_traffic.json")) as f:
            t = json.load(f)
        if t.get("source_hash") != scan_source_hash():
            return None
        return t.get(kind)
    except Exception:
        return None


# ------------------------------------------------------------------ GPU leg

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import cross_layer_latent_b200 as li

    wl = workload(args.workload)
    dev = f"cuda:{local}"
    inp = generate(wl, seed=wl.seed + 1000 * rank)
    hnew, Wd, Wk = construction_inputs(wl, seed=wl.seed + 1000 * rank)
    ctx = li.Context(local)
    dt_code = {"f32": li.LI_F32, "bf16": li.LI_BF16, "e4m3": li.LI_E4M3}[wl.cache_dtype]
    g = li.GroupIndexer(ctx, batch=wl.batch, capacity=wl.capacity, d_c=wl.d_c, H=wl.heads, d_k=wl.d_k,
                        G=wl.group, dtype=dt_code, k=wl.k, B=wl.B, T=wl.queries, dsa=True, device=dev)
    g.load(inp.lengths, inp.W_K, inp.q, inp.w, latent=inp.latent, hidden=inp.hidden, W_down=inp.W_down,
           q_pos=inp.q_pos)
    lengths = torch.from_numpy(inp.lengths).to(dev)
    len_before = (lengths - 1).to(torch.int32)
    bf = torch.bfloat16
    h_anchor = torch.from_numpy(hnew).to(dev, bf)
    h_layers = [torch.from_numpy(hnew).to(dev, bf) for _ in range(wl.group)]
    W_down = torch.from_numpy(Wd).to(dev, bf)
    W_k = [torch.from_numpy(x).to(dev, bf) for x in Wk]
    W_K = [torch.from_numpy(x).to(dev, bf) for x in inp.W_K]
    q = [torch.from_numpy(x).to(dev, bf) for x in inp.q]
    w = [torch.from_numpy(x).to(dev) for x in inp.w]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    hs_keys, dsa_keys = keys_per_step(wl, inp.lengths)

    def reset():
        g.latent.lengths.copy_(len_before)
        for kc in g.keys:
            kc.lengths.copy_(len_before)

    def hs_path():
        g.append(h_anchor, W_down)
        for l in range(wl.group):
            g.w[l].copy_(w[l])
            li.li_absorb_query(ctx, q[l], W_K[l], wl.d_c, g.dtype, g.q_abs[l], g.q_abs_scale[l])
        g.hs_anchor(0)
        for l in range(1, wl.group):
            g.hs_follower(l)

    def dsa_path():
        for l in range(wl.group):
            g.append_keys(l, h_layers[l], W_k[l])
            li.li_absorb_query(ctx, q[l], None, wl.d_k, g.dtype, g.q_raw[l], g.q_raw_scale[l])
            g.dsa_score_topk(l)

    for _ in range(args.warmup):
        reset()
        hs_path()
        dsa_path()
    torch.cuda.synchronize()
    st = li.li_device_status(ctx, g.ws)
    if st != "LI_OK":
        raise RuntimeError(f"device status after warm-up: {st}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    li.li_profile_reset(ctx)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        torch.cuda.nvtx.range_push("timed")
        li.li_profile_enable(ctx, True)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            reset()
            ev[i][0].record(stream)
            hs_path()
            ev[i][1].record(stream)
            dsa_path()
            ev[i][2].record(stream)
        li.li_profile_enable(ctx, False)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    hs_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dsa_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = sum(hs_ms) + sum(dsa_ms)
    recs = li.li_profile_read(ctx)
    li.li_profile_reset(ctx)
    st = li.li_device_status(ctx, g.ws)
    if st != "LI_OK":
        raise RuntimeError(f"device status after the timed steps: {st}")

    t = torch.tensor([total_ms], device=dev, dtype=torch.float64)
    if dist:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    keys = hs_keys + dsa_keys
    value = world * keys * args.steps / (max_ms / 1e3)

    # ---- roofline of the dominant kernel (the scan), from the live launch profile
    kernels = [r for r in recs if r["kernel"] != "memset"]
    scans = [r for r in recs if r["kernel"] == "scan"]
    per_step = len(scans) // args.steps
    row_latent = wl.d_c * (1 if wl.cache_dtype == "e4m3" else 2 if wl.cache_dtype == "bf16" else 4) + \
        (4 if wl.cache_dtype == "e4m3" else 0)
    row_key = wl.d_k * (1 if wl.cache_dtype == "e4m3" else 2 if wl.cache_dtype == "bf16" else 4) + \
        (4 if wl.cache_dtype == "e4m3" else 0)
    ntok = int(inp.lengths.sum())
    scan_bytes = [ntok * row_latent] + [ntok * row_key] * wl.group      # anchor scan, then 4 DSA scans
    alg_bytes = sum(scan_bytes[j % len(scan_bytes)] for j in range(len(scans)))
    scan_ms = sum(r["ms"] for r in scans)
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (scan_ms / 1e3) / 1e9 if scan_ms > 0 else 0.0
    traffic = profiled_traffic("scan_dram_bytes_per_launch")
    by_kernel = {}
    for r in recs:
        d = by_kernel.setdefault(r["kernel"], {"launches": 0, "ms": 0.0})
        d["launches"] += 1
        d["ms"] += r["ms"]
    for d in by_kernel.values():
        d["ms_per_step"] = d["ms"] / args.steps
        d["ms"] = round(d["ms"], 4)

    out = {"metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": wl.cache_dtype, "data": "synthetic",
           "config": config_of(wl),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": traffic,
                        "kernel": "scan (tcgen05 latent / key scan, fused ReLU-weighted head reduction)",
                        "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                        "alg_bytes_per_key": {"latent": row_latent, "dsa_key": row_key},
                        "launches_per_step": per_step, "scan_ms_per_step": scan_ms / args.steps},
           "paths": {"hs_ms": statistics.mean(hs_ms), "dsa_ms": statistics.mean(dsa_ms),
                     "hs_keys_per_step": hs_keys, "dsa_keys_per_step": dsa_keys,
                     "hs_keys_per_s": hs_keys / (statistics.mean(hs_ms) / 1e3),
                     "dsa_keys_per_s": dsa_keys / (statistics.mean(dsa_ms) / 1e3),
                     "hs_speedup_over_dsa": statistics.mean(dsa_ms) / statistics.mean(hs_ms)},
           "kernels": by_kernel,
           "gpu_launches": len(kernels),
           "wall_s_timed_loop": t_wall}
    out["clocks"] = clk.summary()

    # ---- end to end through the public API with host buffers
    if not args.no_e2e:
        pin = lambda x: torch.from_numpy(np.ascontiguousarray(x)).pin_memory()  # noqa: E731
        host_in = {"h_anchor": pin(hnew.astype(np.float32)).to(bf).pin_memory(),
                   "h_layers": [pin(hnew.astype(np.float32)).to(bf).pin_memory() for _ in range(wl.group)],
                   "q": [pin(x).to(bf).pin_memory() for x in inp.q], "w": [pin(x) for x in inp.w]}
        host_out = [torch.empty(wl.batch, 1, wl.k, dtype=torch.int32).pin_memory() for _ in range(2 * wl.group)]
        h2d = host_in["h_anchor"].numel() * 2 + sum(x.numel() * 2 for x in host_in["h_layers"]) + \
            sum(x.numel() * 2 for x in host_in["q"]) + sum(x.numel() * 4 for x in host_in["w"])
        d2h = sum(x.numel() * 4 for x in host_out)

        def e2e_step():
            h_anchor.copy_(host_in["h_anchor"], non_blocking=True)
            for l in range(wl.group):
                h_layers[l].copy_(host_in["h_layers"][l], non_blocking=True)
                q[l].copy_(host_in["q"][l], non_blocking=True)
                w[l].copy_(host_in["w"][l], non_blocking=True)
            hs_path()
            hs_idx = [x.clone() for x in g.idx]
            dsa_path()
            for l in range(wl.group):
                host_out[l].copy_(hs_idx[l], non_blocking=True)
                host_out[wl.group + l].copy_(g.idx[l], non_blocking=True)

        for _ in range(2):
            reset()
            e2e_step()
        torch.cuda.synchronize()
        e2e_ms = []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            reset()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            e1.synchronize()
            e2e_ms.append(e0.elapsed_time(e1))
        te = torch.tensor([sum(e2e_ms)], device=dev, dtype=torch.float64)
        if dist:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        out["e2e"] = {"value": world * keys * args.steps / (float(te.item()) / 1e3), "unit": "keys/s",
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                      "ms_per_step": float(te.item()) / args.steps}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(inp, hnew, Wd, Wk)
    if rank == 0:
        print(json.dumps(out))
    ctx.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
