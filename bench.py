"""Benchmark: one layer of window-attention scoring, selection and compaction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is the whole path over one synthetic Llama-3-8B-shaped layer at
N = 131072 context tokens (32 query heads, 8 KV heads, head_dim 128, window
32, average pooling 7): window scores -> per-KV-head top-k (10 %, 13107 kept)
-> K/V gather -> all-head TSP top-k (20 %, 26214 kept) -> hidden-state gather
([N][4096] bf16).  Inputs are resident in HBM before the timed region; they
are larger than L2 (K 268 MB, X 1.07 GB), so no explicit flush is used.

With N > 1 (torchrun, one process per GPU) every rank compresses its own
layer (independent sequences: weak scaling, no collective on the data path);
time is the max over ranks.  `--impl reference` times the float64 CPU
oracle on the same workload (bounded sample per step) instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "context tokens scored+compressed/s at N=128K per layer; achieved HBM GB/s"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def algorithmic_bytes(cfg) -> dict:
    """Minimum HBM bytes of each call of one layer (reads + writes)."""
    N, Hkv, d, H, w = cfg.N, cfg.Hkv, cfg.d, cfg.H, cfg.w
    kk, kt, D = cfg.k_kv, cfg.k_tsp, cfg.hidden
    return {
        "score": N * Hkv * d * 2 + w * H * d * 2 + Hkv * N * 4,  # K once, Q_win, scores out
        "select_kv": Hkv * N * 4 + Hkv * kk * 4,                # scores in, indices out
        "gather_kv": 2 * 2 * Hkv * kk * d * 2 + Hkv * kk * 4,   # K,V rows in+out, indices
        "select_tsp": Hkv * N * 4 + kt * 4,                     # the score rows in (summed on the fly), indices out
        "gather_hidden": 2 * kt * D * 2 + kt * 4,
    }


def layer_bytes(cfg) -> int:
    """Algorithmic bytes of the whole step (scores written once and read once)."""
    b = algorithmic_bytes(cfg)
    return (b["score"] + b["gather_kv"] + b["gather_hidden"] + cfg.Hkv * cfg.N * 4
            + (cfg.Hkv * cfg.k_kv + cfg.k_tsp) * 4)


def workload_config(cfg) -> dict:
    return {"workload": cfg.name, "N": cfg.N, "H": cfg.H, "Hkv": cfg.Hkv, "d": cfg.d, "w": cfg.w,
            "pool": cfg.pool, "k_kv": cfg.k_kv, "k_tsp": cfg.k_tsp, "hidden": cfg.hidden,
            "l2": (f"inputs larger than L2 (K {cfg.N * cfg.Hkv * cfg.d * 2 / 1e6:.0f} MB, "
                   f"X {cfg.N * cfg.hidden * 2 / 1e9:.2f} GB); no flush"),
            "parallelism": "one independent layer per rank"}


# --------------------------------------------------------------------------- #
# clocks (read-only NVML sampling during the timed region)
# --------------------------------------------------------------------------- #
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Median SM clock and active slowdown reasons while the GPU works."""

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            pr = torch.cuda.get_device_properties(cuda_index)
            try:
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = self._reasons_fn(self.h)
                for b, name in _REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def load_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    source is unchanged since the capture; else None."""
    try:
        data = json.load(open(TRAFFIC_FILE))
        ent = data[kernel]
        src = os.path.join(ROOT, ent["source"])
        if hashlib.sha256(open(src, "rb").read()).hexdigest() != ent["source_sha256"]:
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


def tensor_peak_bf16():
    """Dense bf16 tensor peak: the measured cuBLAS bf16 GEMM burst figure."""
    try:
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return round(float(mp["bf16_tflops"]), 1), "measured"
    except Exception:
        return 1590.0, "fallback"


def tensor_peak_tf32():
    """Dense tf32 tensor peak: the measured bf16 GEMM peak times the nominal
    tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s)."""
    try:
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return round(float(mp["bf16_tflops"]) * 1.1 / 2.25, 1), "measured bf16 x nominal tf32/bf16"
    except Exception:
        return round(1590.0 * 1.1 / 2.25, 1), "fallback bf16 x nominal tf32/bf16"


def measured_peaks():
    try:
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(mp["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# --------------------------------------------------------------------------- #
# CPU oracle (baseline / reference arm)
# --------------------------------------------------------------------------- #
class OracleLayerSteps:
    """The float64 oracle over one layer, one KV head per step: that head's
    window scores over all N keys, its pooled top-k and K/V gather; the
    head's scores also go into the all-head (TSP) sum, and the step that adds
    the last head ranks that sum (pooled top-k) and gathers the hidden
    states.  Hkv consecutive steps are one whole layer of the method."""

    def __init__(self, orc, lay, cfg):
        self.orc, self.lay, self.cfg = orc, lay, cfg
        self.T = np.zeros(cfg.N)
        self.g = 0

    def step(self) -> None:
        orc, lay, cfg, g = self.orc, self.lay, self.cfg, self.g
        G = cfg.G
        A = orc.window_scores(lay.q[:, g * G:(g + 1) * G, :], lay.k[:, g:g + 1, :], G, 1, cfg.w, cfg.scale)[0]
        S = orc.rank_scores(A, cfg.N, cfg.w, cfg.pool)
        idx = orc.select_topk(S, cfg.N, cfg.w, cfg.k_kv)
        orc.gather_rows(lay.k[:, g, :], idx, nsrc=cfg.N)
        orc.gather_rows(lay.v[:, g, :], idx, nsrc=cfg.N)
        self.T += A
        if g == cfg.Hkv - 1:
            pt = orc.rank_scores(self.T, cfg.N, cfg.w, cfg.pool)
            orc.gather_rows(lay.x, orc.select_topk(pt, cfg.N, cfg.w, cfg.k_tsp))
            self.T[:] = 0.0
        self.g = (g + 1) % cfg.Hkv


def cpu_baseline(orc, lay, cfg) -> dict:
    """One whole layer on the oracle (Hkv head steps)."""
    steps = OracleLayerSteps(orc, lay, cfg)
    t0 = time.perf_counter()
    for _ in range(cfg.Hkv):
        steps.step()
    dt = time.perf_counter() - t0
    return {"value": cfg.N / dt, "unit": "tokens/s", "cores": orc.max_threads(), "kind": "oracle",
            "sample": f"one whole N={cfg.N} layer: {cfg.Hkv} KV heads (scores over all keys, pooled top-k, K/V "
                      f"gather), the all-head sum, its pooled top-k and the hidden gather; {dt:.1f} s wall"}


def run_reference(args, cfg, rank: int) -> None:
    if rank != 0:
        return
    import oracle
    import workloads

    orc = oracle.get()
    lay = workloads.make_layer(cfg)
    steps = OracleLayerSteps(orc, lay, cfg)
    for _ in range(args.warmup):
        steps.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        steps.step()
    dt = (time.perf_counter() - t0) / args.steps  # seconds per step (one KV head)
    value = cfg.N / (dt * cfg.Hkv)
    sample = (f"each step: one KV head of the N={cfg.N} layer (scores over all keys, pooled top-k, K/V gather) "
              f"added into the all-head sum; every {cfg.Hkv}th step also ranks that sum (pooled top-k) and "
              f"gathers the hidden states; a layer = {cfg.Hkv} steps")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": orc.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# the other configurations (per-layer time; the headline is the 128K layer)
# --------------------------------------------------------------------------- #
def other_bytes(cfg, total: int) -> int:
    """Algorithmic HBM bytes of one step of cfg.  A single sequence or a
    ragged batch: K once, Q_win, the scores written and read once, the K(/V)
    gather's rows in and out.  The 16-layer accumulation: per layer K once,
    Q_win, the scores written and read once (statistics), C_global read and
    written; then C_global read by the two selections and the K gather's rows
    in and out."""
    B = cfg.batch
    kv_rows = cfg.Hkv * B * min(cfg.k_kv, cfg.N)
    gather = (2 if cfg.with_v else 1) * 2 * kv_rows * cfg.d * 2
    per_layer = total * cfg.Hkv * cfg.d * 2 + B * cfg.w * cfg.H * cfg.d * 2 + 2 * cfg.Hkv * total * 4
    if cfg.layers > 1:
        return cfg.layers * (per_layer + 2 * cfg.Hkv * total * 4) + 2 * cfg.Hkv * total * 4 + gather
    return per_layer + gather


def run_other(args, cfg, torch, kvc, workloads, dev) -> None:
    """Time per layer of configuration cfg on one GPU.

    A single sequence: score -> per-KV-head top-k -> K(/V) gather; a ragged
    batch: the same through the varlen calls.  The 16-layer accumulation
    (StructKV): one step is the whole job -- per layer the scores are added
    into C_global and the layer statistics feed the pivot rule; after the
    last layer C_global is ranked twice (the propagation set over the sum of
    the KV-head rows, and the K set of every KV head) and the retained K rows
    of that layer are gathered."""
    layers = ([workloads.make_layer(cfg, layer=l) for l in range(1, cfg.layers + 1)] if cfg.layers > 1
              else [workloads.make_layer(cfg)])
    lay0 = layers[0]
    B, total = lay0.batch, lay0.total
    max_len = int(lay0.lengths().max())
    qs = [workloads.torch_bf16(l.q, dev).view(B, cfg.w, cfg.H, cfg.d) if B > 1 else workloads.torch_bf16(l.q, dev)
          for l in layers]
    ks = [workloads.torch_bf16(l.k, dev) for l in layers]
    vs = [workloads.torch_bf16(l.v, dev) if cfg.with_v else None for l in layers]
    cu = torch.from_numpy(lay0.cu_seqlens).to(dev)
    kk = min(cfg.k_kv, cfg.N)
    scores = torch.empty((cfg.Hkv, total), dtype=torch.float32, device=dev)
    multi = cfg.layers > 1
    accum = torch.zeros((cfg.Hkv, total), dtype=torch.float32, device=dev) if multi else None
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    p = kvc.score_params(cfg.H, cfg.Hkv, cfg.d, cfg.w)
    ws_s = torch.empty(kvc.score_workspace_size(p, B, total), dtype=torch.uint8, device=dev)
    ws_k = torch.empty(kvc.select_workspace_size(cfg.Hkv, B, total), dtype=torch.uint8, device=dev)
    ws_t = torch.empty(kvc.select_workspace_size(1, B, total), dtype=torch.uint8, device=dev)
    if B > 1:
        idx = torch.empty((B, cfg.Hkv, cfg.k_kv), dtype=torch.int32, device=dev)
        counts = torch.empty((B,), dtype=torch.int32, device=dev)
        k_c = torch.empty((B, cfg.Hkv, cfg.k_kv, cfg.d), dtype=torch.bfloat16, device=dev)
    else:
        idx = torch.empty((cfg.Hkv, kk), dtype=torch.int32, device=dev)
        k_c = torch.empty((cfg.Hkv, kk, cfg.d), dtype=torch.bfloat16, device=dev)
    v_c = torch.empty_like(k_c) if cfg.with_v else None
    idx_t = torch.empty((1, min(cfg.k_tsp, cfg.N)), dtype=torch.int32, device=dev) if multi else None
    stats = torch.empty((cfg.Hkv, 3), dtype=torch.float32, device=dev) if multi else None
    pivot = kvc.pivot_state(dev) if multi else None

    def step(st):
        if B > 1:
            q, k, v = qs[0], ks[0], vs[0]
            kvc.kvc_score_varlen(q, k, cu, max_len, scores=scores, ws=ws_s, dev_err=err, stream=st)
            kvc.kvc_select_topk_varlen(scores, cu, max_len, cfg.w, cfg.pool, cfg.k_kv, idx=idx, counts=counts,
                                       ws=ws_k, dev_err=err, stream=st)
            kvc.kvc_gather_kv_varlen(k, v, cu, idx, k_out=k_c, v_out=v_c, dev_err=err, stream=st)
            return
        if not multi:
            kvc.kvc_score(qs[0], ks[0], scores=scores, ws=ws_s, dev_err=err, stream=st)
            kvc.kvc_select_topk(scores, cfg.w, cfg.pool, cfg.k_kv, idx=idx, ws=ws_k, stream=st)
            kvc.kvc_gather_kv(ks[0], vs[0], idx, k_out=k_c, v_out=v_c, dev_err=err, stream=st)
            return
        with torch.cuda.stream(st):
            accum.zero_()
            pivot.zero_()
        for l in range(cfg.layers):
            kvc.kvc_score(qs[l], ks[l], scores=scores, accum=accum, ws=ws_s, dev_err=err, stream=st)
            kvc.kvc_layer_stats(scores, float(cfg.w * cfg.G), out=stats, stream=st)
            kvc.kvc_pivot_update(stats, l + 1, 0.05, 2, cfg.layers, pivot, dev_err=err, stream=st)
        kvc.kvc_select_topk(accum, cfg.w, cfg.pool, cfg.k_tsp, row_group=cfg.Hkv, idx=idx_t, ws=ws_t, stream=st)
        kvc.kvc_select_topk(accum, cfg.w, cfg.pool, cfg.k_kv, idx=idx, ws=ws_k, stream=st)
        kvc.kvc_gather_kv(ks[-1], None, idx, k_out=k_c, dev_err=err, stream=st)

    st = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        step(st)
    torch.cuda.synchronize(dev)
    if err.item() != 0:
        raise RuntimeError(f"device error word {err.item()}")
    nsteps = args.steps
    launches0 = kvc.launch_count()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = torch.cuda.current_stream(dev)
            for i in range(nsteps):
                step(cap)
        torch.cuda.synchronize(dev)
    launches = kvc.launch_count() - launches0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    with sampler:
        torch.cuda.synchronize(dev)
        t0.record(st)
        if graph is not None:
            graph.replay()
        else:
            for i in range(nsteps):
                step(st)
        t1.record(st)
        torch.cuda.synchronize(dev)
    if graph is None:
        launches = kvc.launch_count() - launches0
    if err.item() != 0:
        raise RuntimeError(f"device error word {err.item()} after the timed region")
    ms = t0.elapsed_time(t1) / nsteps
    alg = other_bytes(cfg, total)
    peak, peak_kind = measured_peaks()
    gbs = alg / (ms * 1e-3) / 1e9
    line = {"metric": "context tokens scored+compressed/s per layer", "value": cfg.layers * total / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": nsteps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_layer": ms / cfg.layers, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "tokens_per_layer": total, "batch": B, "layers_per_step": cfg.layers,
                       "N": cfg.N, "H": cfg.H, "Hkv": cfg.Hkv, "d": cfg.d, "w": cfg.w, "pool": cfg.pool,
                       "k_kv": cfg.k_kv, "k_tsp": cfg.k_tsp, "with_v": cfg.with_v,
                       "selection_source": "C_global after the last layer" if cfg.layers > 1 else "the layer's scores"},
            "hbm": {"alg_bytes_per_step": alg, "achieved_gbs": round(gbs, 1), "peak": peak,
                    "peak_kind": peak_kind, "frac": round(gbs / peak, 4)},
            "gpu_launches": launches, "graph": graph is not None, "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# one layer split by KV head over the ranks
# --------------------------------------------------------------------------- #
def run_split(args, cfg, world, rank, local, torch, dist, kvc, shard, workloads) -> None:
    """The 128K layer split by KV head over `world` ranks (strong scaling):
    every rank scores, selects and gathers the K/V of its KV heads; the
    partial all-head rows are summed with an NCCL all-reduce; every rank then
    ranks the summed row and gathers its column slice of the hidden states.
    Steps are launched one by one (no graph); the time is the max over ranks."""
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    lay = workloads.make_layer(cfg)  # the same layer on every rank; each reads its slices
    q, k, v, x = (workloads.torch_bf16(a, dev) for a in (lay.q, lay.k, lay.v, lay.x))
    part = shard.HeadSplitLayer(rank, world, cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden,
                                dev, pool_kernel=cfg.pool)
    reduce_sum = (lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM)) if world > 1 else None
    st = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        part.run(q, k, v, x, reduce_sum=reduce_sum)
    torch.cuda.synchronize(dev)
    if part.dev_err.item() != 0:
        raise RuntimeError(f"device error word {part.dev_err.item()}")
    launches0 = kvc.launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0.record(st)
        for _ in range(args.steps):
            part.run(q, k, v, x, reduce_sum=reduce_sum)
        t1.record(st)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    launches = kvc.launch_count() - launches0
    ms = shard.max_over_ranks(t0.elapsed_time(t1), dist, dev) / args.steps
    if rank == 0:
        conf = workload_config(cfg)
        conf["parallelism"] = f"one layer split by KV head over {world} rank(s), the TSP row all-reduced"
        line = {"metric": METRIC, "value": cfg.N / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": conf,
                "hbm_gbs": round(layer_bytes(cfg) / (ms * 1e-3) / 1e9, 1), "gpu_launches": launches,
                "graph": False, "clocks": sampler.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- #
# CUDA arm
# --------------------------------------------------------------------------- #
def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 24 for --impl reference, three layers of head steps)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="kvc", choices=["kvc", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying a CUDA graph")
    ap.add_argument("--workload", default="c3", choices=["c1", "c2", "c3", "c4", "c5"],
                    help="c3 (the 128K layer) is the headline; the others print their per-layer time")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: replicas (each rank its own layer, weak scaling; default) or heads (one layer "
                         "split by KV head over the ranks, the TSP row all-reduced; strong scaling)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="same layer structure at another N (small cases for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.e2e_steps = max(args.e2e_steps, 1)
    if args.steps is None:
        args.steps = 24 if args.impl == "reference" else 1000

    import workloads

    cfg = workloads.C3
    if args.tokens:
        cfg = workloads.shrink(cfg, name=f"{cfg.name}_at_n{args.tokens}", N=args.tokens,
                               k_kv=int(0.1 * args.tokens), k_tsp=int(0.2 * args.tokens),
                               n_hitters=min(cfg.n_hitters, args.tokens // 64))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return
    if args.workload != "c3":
        import torch
        import long_context_kv_window_b200 as kvc
        torch.cuda.set_device(local)
        run_other(args, getattr(workloads, args.workload.upper()), torch, kvc, workloads,
                  torch.device("cuda", local))
        return

    import torch
    import torch.distributed as dist

    import long_context_kv_window_b200 as kvc
    from long_context_kv_window_b200 import shard

    if args.split == "heads":
        run_split(args, cfg, world, rank, local, torch, dist, kvc, shard, workloads)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # ---- inputs: this rank's own layer, resident in HBM ----------------------
    lay = workloads.make_layer(cfg, seed=cfg.seed + 1000 * rank)
    q, k, v, x = (workloads.torch_bf16(a, dev) for a in (lay.q, lay.k, lay.v, lay.x))
    plan = kvc.LayerPlan(cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, True, dev,
                         pool_kernel=cfg.pool)
    st = torch.cuda.current_stream(dev)
    side = plan.side
    calls = ["score", "select_kv", "gather_kv", "select_tsp", "gather_hidden"]
    given_lse = [None]  # the window rows' log-sum-exp, for the one-read variant of the step

    def step(evs=None, main=None):
        """One layer: the K/V chain on a side stream, the TSP chain on the main
        stream (as LayerPlan.run), with optional per-call timing events
        recorded on the stream each call runs on."""
        st = main if main is not None else torch.cuda.current_stream(dev)
        call_stream = {"score": st, "select_kv": side, "gather_kv": side, "select_tsp": st, "gather_hidden": st}
        ev_scores, ev_side = torch.cuda.Event(), torch.cuda.Event()

        def timed(name, fn):
            if evs is not None:
                evs[name][0].record(call_stream[name])
            fn()
            if evs is not None:
                evs[name][1].record(call_stream[name])
        if given_lse[0] is None:
            timed("score", lambda: kvc.kvc_score(q, k, scores=plan.scores, ws=plan.ws_score, dev_err=plan.dev_err,
                                                 stream=st))
        else:
            timed("score", lambda: kvc.kvc_score_lse(q, k, given_lse[0], scores=plan.scores, ws=plan.ws_score,
                                                     dev_err=plan.dev_err, stream=st))
        ev_scores.record(st)
        timed("select_tsp", lambda: kvc.kvc_select_topk(plan.scores, cfg.w, cfg.pool, cfg.k_tsp, row_group=cfg.Hkv,
                                                        idx=plan.idx_tsp, ws=plan.ws_sel_tsp, stream=st))
        side.wait_event(ev_scores)
        timed("select_kv", lambda: kvc.kvc_select_topk(plan.scores, cfg.w, cfg.pool, cfg.k_kv, idx=plan.idx_kv,
                                                       ws=plan.ws_sel_kv, stream=side))
        timed("gather_kv", lambda: kvc.kvc_gather_kv(k, v, plan.idx_kv, k_out=plan.k_c, v_out=plan.v_c,
                                                     dev_err=plan.dev_err, stream=side))
        timed("gather_hidden", lambda: kvc.kvc_gather_hidden(x, plan.idx_tsp.view(-1), out=plan.x_c,
                                                             dev_err=plan.dev_err, stream=st))
        ev_side.record(side)
        st.wait_event(ev_side)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if plan.dev_err.item() != 0:
        raise RuntimeError(f"device error word {plan.dev_err.item()}")

    # ---- timed region ----------------------------------------------------------
    def timed_run(with_events: bool):
        """K steps, captured once as a CUDA graph (unless --no-graph) and
        replayed; device time per step, and per-call times when the steps
        carry per-call events.  The headline run carries none: an event
        recorded between two kernels of a stream also cuts the programmatic
        (early-launch) dependency between them."""
        evs = [{c: (torch.cuda.Event(enable_timing=True, external=not args.no_graph),
                    torch.cuda.Event(enable_timing=True, external=not args.no_graph)) for c in calls}
               if with_events else None for _ in range(args.steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        launches0 = kvc.launch_count()
        graph = None
        if not args.no_graph:
            # no host launch overhead between kernels
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                cap = torch.cuda.current_stream(dev)
                for s_ in range(args.steps):
                    step(evs[s_], main=cap)
            torch.cuda.synchronize(dev)
        launches = kvc.launch_count() - launches0
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_start.record(st)
        if graph is not None:
            graph.replay()
        else:
            for s_ in range(args.steps):
                step(evs[s_], main=st)
        t_end.record(st)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        if graph is None:
            launches = kvc.launch_count() - launches0
        ms = shard.max_over_ranks(t_start.elapsed_time(t_end), dist, dev) / args.steps
        per_call = None
        if with_events:
            per_call = {c: sum(evs[s_][c][0].elapsed_time(evs[s_][c][1]) for s_ in range(args.steps)) / args.steps
                        for c in calls}
        return ms, per_call, launches

    sampler = ClockSampler(local)
    with sampler:
        ms_step, _, launches = timed_run(with_events=False)
    ms_step_events, per_call, _ = timed_run(with_events=True)
    if plan.dev_err.item() != 0:
        raise RuntimeError(f"device error word {plan.dev_err.item()} after the timed region")

    # ---- the one-read variant: normalisers given (kvc_score_lse) ---------------
    # The window rows' log-sum-exp, as a causal prefill attention of the layer
    # would return it, formed here once with torch (input preparation only,
    # outside the timed region): lse[i, h] over keys <= N - w + i.
    with torch.no_grad():
        qf = q.float()
        lse = torch.empty((cfg.w, cfg.H), dtype=torch.float32, device=dev)
        for g in range(cfg.Hkv):
            kg = k[:, g, :].float()
            for hl in range(cfg.G):
                h = g * cfg.G + hl
                logit = (qf[:, h, :] @ kg.t()) * cfg.scale  # [w][N]
                pos = torch.arange(cfg.N, device=dev)
                lim = cfg.N - cfg.w + torch.arange(cfg.w, device=dev)
                logit.masked_fill_(pos[None, :] > lim[:, None], float("-inf"))
                lse[:, h] = torch.logsumexp(logit, dim=1)
        del qf, logit
    lse_scores = torch.empty_like(plan.scores)
    for _ in range(3):
        kvc.kvc_score_lse(q, k, lse, scores=lse_scores, ws=plan.ws_score, dev_err=plan.dev_err, stream=st)
    torch.cuda.synchronize(dev)
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_lse = 20
    l0.record(st)
    for _ in range(n_lse):
        kvc.kvc_score_lse(q, k, lse, scores=lse_scores, ws=plan.ws_score, dev_err=plan.dev_err, stream=st)
    l1.record(st)
    torch.cuda.synchronize(dev)
    ms_lse = l0.elapsed_time(l1) / n_lse
    rel_lse = float(((lse_scores - plan.scores).abs() / plan.scores.abs().clamp_min(1e-30)).max())
    del lse_scores
    # the whole step with those normalisers given (one read of K): what the
    # layer costs when its prefill attention supplies them (not the headline)
    given_lse[0] = lse
    for _ in range(3):
        step()
    ms_step_lse, _, _ = timed_run(with_events=False)
    given_lse[0] = None

    # ---- decode over the compacted cache (the consumer of the K/V retention) ----
    # One decode query per head over the retained entries.  The cache (K_c +
    # V_c, 53.7 MB) fits in L2, so the timed calls cycle through four copies
    # (215 MB) and read from HBM.
    gq = torch.Generator(device=dev)
    gq.manual_seed(17)
    q_dec = torch.randn(cfg.H, cfg.d, device=dev, generator=gq).to(torch.bfloat16)
    caches = [(plan.k_c, plan.v_c)] + [(plan.k_c.clone(), plan.v_c.clone()) for _ in range(3)]
    dec_out = torch.empty((cfg.H, cfg.d), dtype=torch.float32, device=dev)
    ws_dec = torch.zeros(kvc.decode_workspace_size(cfg.H, cfg.Hkv, cfg.d, cfg.k_kv), dtype=torch.uint8, device=dev)
    for i in range(4):
        kvc.kvc_decode_attention(q_dec, *caches[i], out=dec_out, ws=ws_dec, dev_err=plan.dev_err, stream=st)
    torch.cuda.synchronize(dev)
    # the calls are replayed from a CUDA graph: a decode call is ~10 us of GPU
    # work, less than issuing it from Python takes
    n_dec = 40
    g_dec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_dec):
        cap = torch.cuda.current_stream(dev)
        for i in range(n_dec):
            kvc.kvc_decode_attention(q_dec, *caches[i % 4], out=dec_out, ws=ws_dec, dev_err=plan.dev_err, stream=cap)
    torch.cuda.synchronize(dev)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(st)
    g_dec.replay()
    d1.record(st)
    torch.cuda.synchronize(dev)
    ms_dec = d0.elapsed_time(d1) / n_dec
    del g_dec
    dec_bytes = 2 * cfg.Hkv * cfg.k_kv * cfg.d * 2 + cfg.H * cfg.d * (2 + 4)
    del caches

    # ---- residual VQ encode of the compacted cache (K and V rows) ------------
    # Four stages of 256 codewords (random stand-ins for trained codebooks);
    # the scores are a tf32 tensor-core contraction: 2 * rows * M * d FLOP per
    # stage.
    rvq_S, rvq_M = 4, 256
    cbk = torch.from_numpy(workloads.make_codebooks(rvq_S, rvq_M, cfg.d, seed=9)).to(dev)
    cbv = torch.from_numpy(workloads.make_codebooks(rvq_S, rvq_M, cfg.d, seed=10)).to(dev)
    rows_k, rows_v = plan.k_c.view(-1, cfg.d), plan.v_c.view(-1, cfg.d)
    codes_k = torch.empty((rows_k.shape[0], rvq_S), dtype=torch.int32, device=dev)
    codes_v = torch.empty_like(codes_k)

    def rvq_both():
        kvc.kvc_rvq_encode(rows_k, cbk, codes=codes_k, dev_err=plan.dev_err, stream=st)
        kvc.kvc_rvq_encode(rows_v, cbv, codes=codes_v, dev_err=plan.dev_err, stream=st)
    rvq_both()
    torch.cuda.synchronize(dev)
    n_rvq = 5
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(st)
    for _ in range(n_rvq):
        rvq_both()
    r1.record(st)
    torch.cuda.synchronize(dev)
    ms_rvq = r0.elapsed_time(r1) / n_rvq
    rvq_rows = rows_k.shape[0] + rows_v.shape[0]
    rvq_flop = 2 * rvq_rows * rvq_M * cfg.d * rvq_S
    tf32_peak, tf32_kind = tensor_peak_tf32()

    # ---- causal prefill attention with the rows' log-sum-exp -----------------
    # The producer of the window rows' normalisers (the TSP layer's attention
    # over the prompt) and the later layers' attention over the propagated
    # tokens: random queries over the layer's first n_pre keys and values.
    pre = None
    if cfg.d == 128:
        n_pre = min(cfg.N, 32768)
        gp = torch.Generator(device=dev)
        gp.manual_seed(23)
        q_pre = torch.randn(n_pre, cfg.H, cfg.d, device=dev, generator=gp).to(torch.bfloat16)
        k_pre, v_pre = k[:n_pre], v[:n_pre]
        out_pre = torch.empty((n_pre, cfg.H, cfg.d), dtype=torch.bfloat16, device=dev)
        lse_pre = torch.empty((n_pre, cfg.H), dtype=torch.float32, device=dev)
        kvc.kvc_prefill_attention(q_pre, k_pre, v_pre, out=out_pre, lse=lse_pre, dev_err=plan.dev_err, stream=st)
        torch.cuda.synchronize(dev)
        n_p = 3
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(st)
        for _ in range(n_p):
            kvc.kvc_prefill_attention(q_pre, k_pre, v_pre, out=out_pre, lse=lse_pre, dev_err=plan.dev_err,
                                      stream=st)
        p1.record(st)
        torch.cuda.synchronize(dev)
        ms_pre = p0.elapsed_time(p1) / n_p
        pre_flop = 4 * cfg.d * cfg.H * n_pre * (n_pre + 1) / 2  # QK^T and PV over the causal half
        bf16_peak, bf16_kind = tensor_peak_bf16()
        pre = {"ms": round(ms_pre, 4), "n": n_pre, "tflops": round(pre_flop / (ms_pre * 1e-3) / 1e12, 1),
               "tflops_peak_bf16": bf16_peak, "peak_kind": bf16_kind,
               "frac": round(pre_flop / (ms_pre * 1e-3) / 1e12 / bf16_peak, 4),
               "note": f"kvc_prefill_attention: causal, {cfg.H}/{cfg.Hkv} heads, d {cfg.d}, over {n_pre} tokens, "
                       "with every row's log-sum-exp; not part of the headline step"}
        del q_pre, out_pre, lse_pre

    # ---- end to end through the public API with host buffers ------------------
    hq, hk, hv, hx = (workloads.torch_bf16(a).pin_memory() for a in (lay.q, lay.k, lay.v, lay.x))
    outs = [plan.idx_kv, plan.idx_tsp, plan.k_c, plan.v_c, plan.x_c]
    h_outs = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hx))
    d2h = sum(t.numel() * t.element_size() for t in h_outs)

    def e2e_step():
        """Inputs in from pinned host memory, the layer, and every result of
        the step back: both index sets, the compacted K/V and hidden states."""
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        x.copy_(hx, non_blocking=True)
        plan.run(q, k, v, x)
        for h, t in zip(h_outs, outs):
            h.copy_(t, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(st)
    torch.cuda.synchronize(dev)
    ms_e2e = shard.max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dist, dev)

    # ---- roofline of the dominant call -----------------------------------------
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(cfg)
    dom = max(per_call, key=per_call.get)
    ach = alg[dom] / (per_call[dom] * 1e-3) / 1e9
    breakdown = {c: {"ms": round(per_call[c], 5), "alg_bytes": alg[c],
                     "gbs": round(alg[c] / (per_call[c] * 1e-3) / 1e9, 1)} for c in calls}

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            cpu = cpu_baseline(oracle.get(), lay, cfg)
        line = {
            "metric": METRIC, "value": world * cfg.N / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(cfg),
            "hbm_gbs": round(layer_bytes(cfg) / (ms_step * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach / peak, 4),
                         "traffic": load_traffic(dom)},
            "calls": breakdown,
            "rvq_encode": {"ms": round(ms_rvq, 5), "rows": rvq_rows, "stages": rvq_S, "codebook": rvq_M,
                           "rows_per_s": round(rvq_rows / (ms_rvq * 1e-3), 1),
                           "tflops": round(rvq_flop / (ms_rvq * 1e-3) / 1e12, 2), "tflops_peak_tf32": tf32_peak,
                           "peak_kind": tf32_kind,
                           "frac": round(rvq_flop / (ms_rvq * 1e-3) / 1e12 / tf32_peak, 4),
                           "note": "kvc_rvq_encode of the compacted K and V rows (tf32 scores, exact fp32 "
                                   "decision); not part of the headline step"},
            "decode": {"ms": round(ms_dec, 5), "alg_bytes": dec_bytes, "graph": True,
                       "gbs": round(dec_bytes / (ms_dec * 1e-3) / 1e9, 1),
                       "frac": round(dec_bytes / (ms_dec * 1e-3) / 1e9 / peak, 4),
                       "note": "kvc_decode_attention: one decode query per head over the compacted cache "
                               f"({cfg.Hkv} x {cfg.k_kv} entries, K and V), cache copies cycled past L2; "
                               "not part of the headline step"},
            "prefill_attention": pre,
            "step_with_given_normalisers": {
                "ms_per_step": round(ms_step_lse, 5), "value": world * cfg.N / (ms_step_lse * 1e-3),
                "unit": "tokens/s", "hbm_gbs": round(layer_bytes(cfg) / (ms_step_lse * 1e-3) / 1e9, 1),
                "frac": round(layer_bytes(cfg) / (ms_step_lse * 1e-3) / 1e9 / peak, 4),
                "note": "the same layer step with the window rows' log-sum-exp supplied (as the layer's "
                        "prefill attention, kvc_prefill_attention, returns it) and kvc_score_lse in place of "
                        "kvc_score: one read of K; not the headline"},
            "score_lse": {"ms": round(ms_lse, 5), "alg_bytes": alg["score"],
                          "gbs": round(alg["score"] / (ms_lse * 1e-3) / 1e9, 1),
                          "max_rel_diff_vs_two_pass": rel_lse,
                          "note": "kvc_score_lse: the window rows' normalisers given (one read of K), "
                                  "timed alone; not part of the headline step"},
            "ms_per_step_with_call_events": ms_step_events,
            "e2e": {"value": world * cfg.N / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
            "gpu_launches": launches,
            "graph": not args.no_graph,
            "clocks": sampler.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
