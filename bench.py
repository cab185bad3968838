"""Benchmark one PARK attention layer (retrieval + block-sparse attention) at
the HunyuanVideo layer shape on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl park|reference]

A step is one park_layer call: metric, query K-means, QRKC key K-means (10
iterations each), PAMA, top-p, kept-block CSR, gather and block-sparse
attention, on seeded synthetic Q/K/V of the layer's shape (B=1, H=24,
N=119,056, D=128, bf16; 930 query and 930 key clusters, p = 0.9).

Rank 0 prints one JSON line.  `value` is milliseconds per layer for the whole
job (max over ranks of the device time per step, divided by the number of
ranks: every rank runs its own layer, no collective on the data path).
Under torchrun each rank is one GPU; `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "layer ms (retrieval+sparse attn) at Wan/Hunyuan shape; tensor-pipe % of peak"
WORKLOAD = "hunyuan"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12  # 148 SMs x 64 FP64 FMA/clk x 2 flops x max clock


# ----------------------------------------------------------------------------- small pure helpers


def aggregate_ms(step_ms_local: float, world: int, reduce_max) -> tuple[float, float]:
    """(max over ranks of ms per step, whole-job ms per layer).  `reduce_max`
    maps a local float to the max over ranks (identity for one rank)."""
    worst = float(reduce_max(step_ms_local))
    return worst, worst / world


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(files) -> str:
    h = hashlib.sha256()
    for p in files:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str):
    """DRAM bytes per launch for `kernel` from the committed ncu summary, if the
    kernel source still has the digest recorded there; else None."""
    prof = os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    for name in sorted(os.listdir(prof)):
        if not name.startswith(kernel) or not name.endswith(".md"):
            continue
        text = open(os.path.join(prof, name)).read()
        m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        s = re.search(r"source_digest:\s*([0-9a-f]+)\s+\(([^)]*)\)", text)
        if m and s and source_digest(s.group(2).split(",")) == s.group(1):
            return float(m.group(1))
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- CPU oracle timing


def oracle_layer_estimate(cfg, seed: int = 0, rows: int = 1024, attn_rows: int = 256) -> dict:
    """Time the float64 oracle on one head of the workload and scale it to the
    whole layer.  Sample: one (batch 0, head 0) slice; the assign and PAMA
    steps on `rows` query/key rows against all centroids (scaled by N/rows,
    x iterations, x heads); the centroid updates and permutations on the full
    head (x iterations, x heads); top-p on one full NQ x NK map (x heads);
    sparse attention on the rows of about attn_rows*NQ/N whole query clusters
    with a kept fraction of 0.7 (scaled by N/rows, x heads).  Returns estimated ms per layer and the
    phase breakdown."""
    from oracle import park_oracle as po
    from synth import gen_slice
    rng = np.random.default_rng(1234)
    N, H, NQ, NK, it = cfg.N, cfg.B * cfg.H, cfg.NQ, cfg.NK, cfg.iters
    Q = gen_slice(cfg, "Q", 0, 0, seed).astype(np.float64)
    K = gen_slice(cfg, "K", 0, 0, seed).astype(np.float64)
    V = gen_slice(cfg, "V", 0, 0, seed).astype(np.float64)
    sel = np.sort(rng.choice(N, size=min(rows, N), replace=False))
    t = {}

    def timed(key, fn, scale):
        t0 = time.perf_counter()
        out = fn()
        t[key] = (time.perf_counter() - t0) * scale
        return out

    M = timed("metric", lambda: po.metric(Q), H)
    CQ, CK = po.strided_init(Q, NQ), po.strided_init(K, NK)
    f = N / sel.size
    timed("query_assign", lambda: po.assign(Q[sel], CQ), f * it * H)
    timed("key_assign", lambda: po.assign(K[sel], CK, M), f * it * H)
    lab_q = (np.arange(N) * NQ) // N
    lab_k = (np.arange(N) * NK) // N
    timed("query_update", lambda: po.update(Q, lab_q, CQ, cfg.dtype), it * H)
    timed("key_update", lambda: po.update(K, lab_k, CK, cfg.dtype), it * H)
    timed("permutation", lambda: po.stable_permutation(lab_q, NQ), 2 * H)
    k_counts = np.bincount(lab_k, minlength=NK)
    timed("pama", lambda: po.pama(Q[sel], lab_q[sel], NQ, CK, k_counts, 1 / math.sqrt(cfg.D)), f * H)
    I = rng.dirichlet(np.ones(NK), size=NQ)
    q_counts = np.bincount(lab_q, minlength=NQ)
    timed("top_p", lambda: po.top_p(I, cfg.p, q_counts, k_counts), H)
    mask = rng.random((NQ, NK)) < 0.7
    # whole query clusters (contiguous here), so each cluster's keys are gathered once, as in a full run
    picks = rng.choice(NQ, size=max(1, attn_rows * NQ // N), replace=False)
    arows = np.nonzero(np.isin(lab_q, picks))[0]
    attn_rows = arows.size
    timed("sparse_attention", lambda: po.sparse_attention(Q, K, V, lab_q, lab_k, mask, 1 / math.sqrt(cfg.D),
                                                          rows=arows), (N / attn_rows) * H)
    total_s = sum(t.values())
    return {"ms_per_layer": total_s * 1e3, "phases_s": {k: round(v, 2) for k, v in t.items()},
            "sample": (f"one head of {H}; assign/PAMA on {sel.size} of {N} rows; updates and permutations on the "
                       f"full head; top-p on one {NQ}x{NK} map; sparse attention on the {attn_rows} rows of whole query clusters at "
                       f"kept fraction 0.7; each phase scaled to {H} heads and {it} K-means iterations")}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_layer_estimate(cfg)
    vals, last = [], None
    for _ in range(args.steps):
        last = oracle_layer_estimate(cfg)
        vals.append(last["ms_per_layer"])
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v, 1), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg),
            "cpu_baseline": {"kind": "oracle", "value": round(v, 1), "unit": "ms", "cores": blas_threads(),
                             "sample": last["sample"]},
            "e2e": {"value": round(v, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg) -> dict:
    shaped = "Wan2.1-14B" if cfg.name.startswith("wan") else "HunyuanVideo"
    return {"workload": f"{shaped}-shaped PARK layer ({cfg.name})", "B": cfg.B, "H": cfg.H, "N": cfg.N,
            "grid": [cfg.T, cfg.Hg, cfg.W], "n_text": cfg.n_text, "D": cfg.D, "NQ": cfg.NQ, "NK": cfg.NK,
            "kmeans_iters": cfg.iters, "p": cfg.p, "parallelism": "replicas",
            "l2": f"inputs larger than L2 (Q, K, V {cfg.B * cfg.H * cfg.N * cfg.D * 2 / 1e6:.0f} MB each vs 126 MB L2); "
                  "no flush"}


# Retrieval variants: flag bits of park_retrieval.flags and the p passed (a ratio for top-k).
VARIANTS = {"park": (0, None), "no_qrkc": (0x4, None), "centroid_query": (0x8, None), "topk_0.3": (0x10, 0.3),
            "size_prior": (0x20, None), "sip_0.3": (0x40, 0.3), "hva_merge": (0x80, None),
            "hva_local": (0x100, None), "hva": (0x180, None)}
# HyperVAttention local windows: boxes of 3 frames x 15 rows x 20 columns (900 tokens,
# about seven clusters of the mean size 128), clipped to the grid
HVA_WINDOW = (3, 15, 20)


def hva_window(cfg):
    return tuple(min(a, b) for a, b in zip(HVA_WINDOW, (cfg.T, cfg.Hg, cfg.W)))


# ----------------------------------------------------------------------------- roofline of one kernel

KERNEL_SOURCES = {"k_sparse_attn_tc": ["block_sparse_attention_means_b200/csrc/k_attn_tc.cu"],
                  "k_assign_tc": ["block_sparse_attention_means_b200/csrc/k_assign_tc.cu"],
                  "k_pama_tc": ["block_sparse_attention_means_b200/csrc/k_pama_tc.cu"],
                  "k_pama_f64": ["block_sparse_attention_means_b200/csrc/k_pama.cu"],
                  "k_metric_partial": ["block_sparse_attention_means_b200/csrc/k_prep.cu"]}
# kernels of park_sparse_attn; the rest of a layer is the retrieval (k_merge_init / k_merge_planes set up
# the query-tile packing here, and also the cluster merging of the merge variant)
ATTENTION_KERNELS = ("k_sparse_attn_tc", "k_attn_schedule", "k_kv_pad_gather", "k_kv_pad_offsets",
                     "k_pack_cand", "k_pack_select", "k_items_emit", "k_item_gather", "k_merge_init",
                     "k_merge_planes")
ATTENTION_MAIN = ("k_sparse_attn_tc",)


def kernel_roofline(name: str, ms_per_launch: float, cfg, counters, peaks, peak_kind) -> dict:
    """Algorithmic work per launch of the named kernel and its roofline."""
    BH, N, D, NQ, NK = cfg.B * cfg.H, cfg.N, cfg.D, cfg.NQ, cfg.NK
    sustained = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    if name in ATTENTION_MAIN:
        work, bound, peak, unit = 4.0 * D * counters[5], "tensor", sustained, "TFLOP/s"
    elif name == "k_assign_tc":
        work, bound, peak, unit = 2.0 * BH * N * ((NQ + NK) / 2) * D, "tensor", sustained, "TFLOP/s"
    elif name == "k_pama_tc":  # one pass of the score GEMM (the second pass is overhead)
        work, bound, peak, unit = 2.0 * BH * N * NK * D, "tensor", sustained, "TFLOP/s"
    elif name == "k_metric_partial":
        work, bound, peak, unit = 2.0 * BH * N * D * D, "alu", FP64_PEAK_TFLOPS, "TFLOP/s"
    elif name == "k_pama_f64":
        rec = counters[3] if counters[3] else BH * NQ
        work = 2.0 * (rec / (BH * NQ)) * BH * N * NK * D
        bound, peak, unit = "alu", FP64_PEAK_TFLOPS, "TFLOP/s"
    else:
        return {"kernel": name, "bound": None}
    achieved = work / (ms_per_launch * 1e-3) / 1e12
    traffic = committed_traffic(name)
    extra = {}
    if name in ATTENTION_MAIN:
        # tensor work actually issued: every (128-row query tile, 128-row key tile) pair, padding included
        tile_tf = 4.0 * 128 * 128 * D * counters[7] / (ms_per_launch * 1e-3) / 1e12
        extra = {"tile_tflops": round(tile_tf, 2), "tensor_pipe_frac_on_tiles": round(tile_tf / peak, 4)}
    return {"kernel": name, "bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "ms_per_launch": round(ms_per_launch, 3), **extra,
            "peak_source": peak_kind + (" (fp64: 148 SMs x 64 FMA/clk x 1.965 GHz)" if bound == "alu" else
                                        " bf16_tflops_sustained")}


# ----------------------------------------------------------------------------- dense reference, recall


def dense_reference(park, torch, cfg, shape, Q, K, V, ws, stream, reps: int = 3) -> dict:
    """Dense attention on the same tensors, two ways: the library's own
    block-sparse attention with every block kept (a retrieval at p = 1; the
    attention kernel's time per launch and the whole park_sparse_attn call), and
    torch's scaled_dot_product_attention (library flash kernel) for context."""
    dev = Q.device
    r1 = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev)
    park.retrieve(Q, K, shape, cfg.NQ, cfg.NK, 1.0, cfg.iters, out=r1, ws=ws, stream=stream)
    O1 = torch.empty_like(Q)
    park.sparse_attn(Q, K, V, shape, cfg.NQ, cfg.NK, r1, O=O1, ws=ws, stream=stream)
    torch.cuda.synchronize(dev)
    park.profile_enable(True)
    park.profile_collect()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        park.sparse_attn(Q, K, V, shape, cfg.NQ, cfg.NK, r1, O=O1, ws=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    park.profile_enable(False)
    prof = park.profile_collect()
    call_ms = e0.elapsed_time(e1) / reps
    kt, kn = prof.get("k_sparse_attn_tc", (float("nan"), 1))
    counters = r1.counters.cpu().tolist()
    flops = 4.0 * cfg.D * counters[5]
    del O1
    import torch.nn.functional as F
    out = F.scaled_dot_product_attention(Q, K, V)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(reps):
        out = F.scaled_dot_product_attention(Q, K, V)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    sdpa_ms = e0.elapsed_time(e1) / reps
    del out
    torch.cuda.empty_cache()
    return {"k10_p1_attention_kernel_ms": round(kt / kn, 3), "k10_p1_sparse_attn_call_ms": round(call_ms, 3),
            "k10_p1_tflops": round(flops / (kt / kn * 1e-3) / 1e12, 1), "torch_sdpa_ms": round(sdpa_ms, 3),
            "torch_sdpa_tflops": round(4.0 * cfg.D * cfg.B * cfg.H * cfg.N ** 2 / (sdpa_ms * 1e-3) / 1e12, 1),
            "kept_pair_fraction_p1": round(counters[5] / (cfg.B * cfg.H * cfg.N ** 2), 4)}


def recall_per_head(torch, cfg, Q, K, r, rows: int = 1024, seed: int = 0) -> dict:
    """Attention recall of the kept blocks per head (PARK Table 1): for `rows`
    query rows per head drawn uniformly (seeded), the share of each row's dense
    attention mass (float64 softmax(Q K^T / sqrt(D)) over all keys) that falls
    on keys of the key clusters its query cluster kept; mean over the rows.  A
    measurement on the library's outputs, outside the timed region."""
    g = torch.Generator().manual_seed(seed)
    scale = 1.0 / math.sqrt(cfg.D)
    vals = []
    for b in range(cfg.B):
        for h in range(cfg.H):
            idx = torch.randperm(cfg.N, generator=g)[:rows].to(Q.device)
            S = (Q[b, h, idx].double() @ K[b, h].double().T) * scale
            A = torch.softmax(S, dim=1)
            ql = r.q_labels[b, h, idx].long()
            kl = r.k_labels[b, h].long()
            keep = r.mask[b, h][ql][:, kl].bool()
            vals.append(float((A * keep).sum(1).mean()))
            del S, A, keep
    v = np.array(vals)
    return {"per_head": [round(x, 5) for x in vals], "mean": round(float(v.mean()), 5),
            "p05": round(float(np.percentile(v, 5)), 5), "worst": round(float(v.min()), 5),
            "sample": f"{rows} uniformly drawn query rows per head (seed {seed}), dense float64 attention over "
                      f"all {cfg.N} keys"}


# ----------------------------------------------------------------------------- main (our arm)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="park", choices=["park", "reference"])
    ap.add_argument("--config", default=WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention reference")
    ap.add_argument("--no-quality", action="store_true", help="skip the recall measurement")
    ap.add_argument("--extra-flags", type=lambda x: int(x, 0), default=0,
                    help="park_retrieval flag bits added to the variant's (e.g. 0x200: no query-tile packing)")
    ap.add_argument("--heads", type=int, default=0, help="override H (small cases for profiler captures)")
    ap.add_argument("--variant", default="park", choices=sorted(VARIANTS),
                    help="retrieval variant (PARK Table 3 ablations, Table 10 top-k, size prior, AB-Attention "
                         "SIP, HyperVAttention cluster merging and local windows)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warmup must be >= 3", file=sys.stderr)
        args.warmup = 3

    from synth import CONFIGS
    from synth.generator import sweep_configs
    all_cfgs = {**CONFIGS, **{c.name: c for c in sweep_configs()}}
    if args.config not in all_cfgs:
        print(f"unknown config {args.config}; one of {sorted(all_cfgs)}", file=sys.stderr)
        return 2
    cfg = all_cfgs[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads, name=f"{cfg.name}_h{args.heads}")
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist
    import block_sparse_attention_means_b200 as park
    from synth import gen_tensor

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def reduce_max(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    # inputs: seeded per rank, bf16, pinned host copies for the end-to-end leg
    host = {}
    for name in ("Q", "K", "V"):
        host[name] = torch.from_numpy(gen_tensor(cfg, name, seed=rank)).to(torch.bfloat16).pin_memory()
    Q, K, V = (host[n].to(dev, non_blocking=True) for n in ("Q", "K", "V"))
    shape = park.Shape.of(cfg)
    vflags, vp = VARIANTS[args.variant]
    sip_u = None
    if vflags & 0x40:  # SIP draws against seeded uniforms, uploaded once
        from synth.generator import gen_uniform
        sip_u = torch.from_numpy(gen_uniform(cfg, seed=rank)).to(dev)
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev, sip_uniform=sip_u,
                               window=hva_window(cfg) if vflags & 0x100 else None)
    out.flags = vflags | args.extra_flags
    p_arg = cfg.p if vp is None else vp
    ws = park.alloc_workspace(shape, cfg.NQ, cfg.NK, dev)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)

    def step():
        park.layer(Q, K, V, shape, cfg.NQ, cfg.NK, p_arg, cfg.iters, O=O, out=out, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = out.status_code()

    # ---- device-resident timing (inputs already in HBM), no per-kernel events
    sampler = ClockSampler(dev.index)
    park.profile_enable(False)
    launches0 = park.launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    launches = park.launch_count() - launches0
    step_ms = e0.elapsed_time(e1) / args.steps
    worst_ms, value = aggregate_ms(step_ms, world, reduce_max)
    counters = out.counters.cpu().tolist()

    # ---- per-kernel breakdown: a separate pass of the same steps with an event pair
    # around every launch (on the launch stream); the rooflines below use it
    park.profile_enable(True)
    park.profile_collect()
    barrier()
    torch.cuda.synchronize(dev)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        step()
    p1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    park.profile_enable(False)
    prof = park.profile_collect()
    profiled_step_ms = p0.elapsed_time(p1) / args.steps

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        O_host = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        barrier()
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            Q.copy_(host["Q"], non_blocking=True)
            K.copy_(host["K"], non_blocking=True)
            V.copy_(host["V"], non_blocking=True)
            step()
            O_host.copy_(O, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_step = f0.elapsed_time(f1) / args.steps
        _, e2e_val = aggregate_ms(e2e_step, world, reduce_max)
        nbytes = sum(host[n].numel() * host[n].element_size() for n in ("Q", "K", "V"))
        e2e = {"value": round(e2e_val, 3), "unit": "ms", "h2d_bytes_per_step": int(nbytes),
               "d2h_bytes_per_step": int(O.numel() * O.element_size())}

    # ---- quality and the dense reference (outside the timed regions; every rank
    # takes the same steps, rank 0 reports)
    recall = None if args.no_quality else recall_per_head(torch, cfg, Q, K, out)
    dense = None if args.no_dense else dense_reference(park, torch, cfg, shape, Q, K, V, ws, stream)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks, peak_kind = load_peaks()
    kernels = {k: {"ms_per_step": round(v[0] / args.steps, 3), "launches_per_step": v[1] / args.steps,
                   "share": round(v[0] / max(1e-9, sum(x[0] for x in prof.values())), 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][0])}
    top = next(iter(kernels)) if kernels else None
    roof = kernel_roofline(top, prof[top][0] / prof[top][1], cfg, counters, peaks, peak_kind) if top else None
    attn_name = next((k for k in ATTENTION_MAIN if k in prof), None)
    attn = prof.get(attn_name) if attn_name else None
    attn_roof = kernel_roofline(attn_name, attn[0] / attn[1], cfg, counters, peaks, peak_kind) \
        if attn else None
    retrieval_ms = sum(v[0] for k, v in prof.items()
                       if k not in ATTENTION_KERNELS) / args.steps
    attention_ms = sum(v[0] for k, v in prof.items() if k in ATTENTION_KERNELS) / args.steps
    if dense:
        denom = min(dense["k10_p1_attention_kernel_ms"], dense["torch_sdpa_ms"])
        dense["retrieval_frac_of_dense"] = round(retrieval_ms / denom, 4)
        dense["layer_vs_dense"] = round(value / denom, 4)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        est = oracle_layer_estimate(cfg)
        cpu = {"value": round(est["ms_per_layer"], 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
               "sample": est["sample"], "phases_s": est["phases_s"]}

    line = {"metric": METRIC, "value": round(value, 3), "unit": "ms", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(worst_ms, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(cfg), **({"variant": args.variant} if args.variant != "park" else {}),
                       **({"extra_flags": hex(args.extra_flags)} if args.extra_flags else {}),
                       **({"window": list(hva_window(cfg))} if vflags & 0x100 else {})},
            "roofline": roof, "attention_roofline": attn_roof,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches), "clocks": clocks,
            "status": status,
            "retrieval_ms_per_layer": round(retrieval_ms, 3),
            "attention_ms_per_layer": round(attention_ms, 3),
            "profiled_ms_per_step": round(profiled_step_ms, 3),
            "dense": dense, "recall": recall,
            "kept_block_fraction": round(counters[4] / (cfg.B * cfg.H * cfg.NQ * cfg.NK), 4),
            "kept_pair_fraction": round(counters[5] / (cfg.B * cfg.H * cfg.N ** 2), 4),
            "rechecks": {"query_rows": counters[0], "key_rows": counters[1], "full_rescore_rows": counters[2],
                         "pama_clusters": counters[3]},
            "kernels": kernels, "peaks": peak_kind}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
