"""Benchmark of the activation-sparse gated FFN forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole sparse inference path over one batch: the
gate GEMM with the TwELL epilogue (twell_gate_pack), then the up and down
projections from TwELL (twell_hybrid_up_down: tokens with at most K = F/512
stored entries (16 at the 1B shape) through a CUDA-core kernel, the heavier
ones through two tcgen05 spill GEMMs), on the 1B-shaped bf16
workload (N=8192 tokens, d=2048, F=8192, T=C=128, mean gate density 1%,
per-token scale LogNormal(0, 0.7)) unless --workload names another.  Inputs
are seeded synthetic data resident in HBM; L2 is flushed (a 256 MB write)
between timed steps and the flush is outside the per-step CUDA events.

Prints one JSON line (rank 0).  `value` is tokens/s over all ranks (weak
scaling: every rank runs its own batch, no collective on the data path).
Also reported: the same forward with every entry through the per-entry
kernel (twell_fused_up_down), the hybrid format's pack-and-forward path, the
library's dense bf16 FFN and a cuBLAS (torch.matmul) dense FFN on the same
inputs, the roofline of each kernel, an end-to-end number through host
buffers, and the fp64 CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse gated-FFN tokens/s at 1B shape bf16 (%HBM roofline; vs dense FFN)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
# fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flop x 1.965 GHz
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# ELL capacity of the hybrid format when it serves inference (tokens with more
# stored entries run on the tensor-core spill GEMMs)
HYB_INFER_K = 64
# K of the routed step: tokens with more stored entries take the spill GEMMs.
# A spill row costs the two GEMMs' work over all F hidden units, an entry of
# the light kernel one 8 KB weight-row copy, so the break-even grows with F:
# K = F / 512 (measured, routed call alone: 1B (F = 8192) flat for K = 12..20
# at 0.155-0.156 ms, 0.161-0.165 ms at K = 8 or 24..48; 2B at 1% (F = 10240)
# 0.594-0.608 ms at K = 16, 0.526-0.533 at K = 20, 0.518-0.524 at K = 48).
def routed_k(d_ff: int) -> int:
    return max(8, d_ff // 512)

# DRAM bytes (read + write) per launch from ncu captures of the kernels,
# keyed by the hash of the source they were taken on; a kernel whose source
# changed since its capture gets null.  Captured on the 1B workload with
# --profile (one launch per kernel, L2 cold): the gate GEMM, and the routed
# call as the sum of its seven launches.
TRAFFIC = {
    "e0bf0d70a6a99597": 79755264,    # twell_gate_pack
    "3f0db3f8024f022c": 227535616,   # twell_hybrid_up_down
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="ffn_1b_bf16")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's token count (e.g. 1..64 for decode-shaped batches)")
    p.add_argument("--impl", default="own", choices=["own", "reference"])
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--sweep", action="store_true",
                   help="density sweep of the workload (0.25%%..5%%): one JSON line per density")
    p.add_argument("--cap-sweep", action="store_true",
                   help="TwELL capacity C in {T/4, T/2, T}: footprint, overflow, truncation error, "
                        "and the hybrid path that recomputes overflowing rows: one JSON line per C")
    p.add_argument("--ell-cap", type=int, default=None,
                   help="K of the routed step: tokens with more stored entries run on the spill GEMMs "
                        "(default: d_ff / 512; 0 spills every non-empty token)")
    p.add_argument("--profile", action="store_true",
                   help="run only warmup + steps of one path (for ncu captures); no JSON")
    p.add_argument("--profile-path", default="routed", choices=["routed", "fused", "hybrid"],
                   help="with --profile: the routed step (default), the TwELL step (gate + "
                        "twell_fused_up_down) or the hybrid format's path (gate, hybrid_pack, "
                        "hybrid_ffn_fwd)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def src_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "activation_sparse_gated_epilogue_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"sge_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        loaded = [s for s, p in zip(sm, pw)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------- own arm

def reduce_max_over_ranks(v: float, device) -> float:
    """Max over the ranks of the default process group of a per-rank time
    (each rank's CUDA-event total); v itself with no group or one rank."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized():
        return v
    if torch.distributed.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(n_tokens: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each processed
    n_tokens per step for `steps` steps, timed as the slowest rank's max_ms."""
    return n_tokens * world * steps / (max_ms / 1e3)


def workload_config(args):
    """The workload's configuration, with --tokens applied."""
    from activation_sparse_gated_epilogue_b200 import synth
    cfg = synth.CONFIGS[args.workload]
    return cfg.with_(n_tokens=args.tokens) if args.tokens > 0 else cfg


def spill_rows_for(n: int) -> int:
    """S_max of the hybrid format's path: a quarter of the batch, rounded up
    to whole 256-row spill tiles."""
    return max(256, (n // 4 + 255) // 256 * 256)


def routed_split(count: torch.Tensor, cap: int, k: int, s_max: int):
    """(spill rows, stored entries of the light and past-S_max tokens, all
    stored entries) of a routed call on a TwELL with per-tile counts
    `count`: tokens with more than k stored entries are heavy and the first
    s_max of them (ascending token order) go to the spill."""
    stored = torch.clamp(count.to(torch.int64), max=cap).sum(1)
    heavy = torch.nonzero(stored > k).flatten()[:s_max]
    total = int(stored.sum().item())
    spilled = int(stored[heavy].sum().item())
    return int(heavy.numel()), total - spilled, total


def twell_bytes(count: torch.Tensor, cap: int, elt: int) -> dict:
    """Sizes of a TwELL with per-tile counts `count` ([N][F/T] u8), u8
    indices and `elt`-byte values: the allocated layout, the algorithmic
    bytes (one count per (row, tile), one index and one value per stored
    entry) and the bytes of the 32-byte DRAM sectors a reader of the stored
    entries touches.  Each tile's index run starts on a C-byte boundary and
    its value run on a C*elt-byte boundary, so for C a multiple of 32 a tile
    with c stored entries touches ceil(c/32) + ceil(c*elt/32) sectors."""
    n, nt = count.shape
    c = torch.clamp(count.to(torch.int64), max=cap)
    stored = int(c.sum().item())
    sectors = int(((c + 31) // 32 + (c * elt + 31) // 32).sum().item())
    return {"allocated": n * nt * (1 + (1 + elt) * cap), "algorithmic": n * nt + (1 + elt) * stored,
            "sector_granular": n * nt + 32 * sectors if cap % 32 == 0 else None,
            "unit": "bytes", "note": "counts read whole; sectors of the stored index and value runs"}


def run_own(args, rank, world, local_rank):
    import activation_sparse_gated_epilogue_b200 as sge
    from activation_sparse_gated_epilogue_b200 import synth

    cfg = workload_config(args)
    if cfg.dtype != "bf16":
        raise SystemExit(f"bench.py measures the bf16 workloads; {cfg.name} is a parity case "
                         "(tests/test_gpu_forward.py)")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(cfg)
    n, d, f, tile, cap = cfg.n_tokens, cfg.d_model, cfg.d_ff, cfg.tile, cfg.cap
    # S_max = N: every heavy token can take the spill (the workspace holds
    # the spill operands for N rows; the GEMMs run only the rows there are)
    k_route, s_max = routed_k(f) if args.ell_cap is None else args.ell_cap, n
    x, wg, wu, wd = (getattr(inp, k).to(dev) for k in ("x", "wg_t", "wu_t", "wd"))
    # weight layouts built once: W_up^T and W_down interleaved row by row (the
    # per-entry kernel's rows, the up GEMM's B operand with row stride 2d) and
    # W_down^T (the down GEMM's K-major B operand)
    wd_t = wd.t().contiguous()
    _w_ud, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    tw = sge.TwELL.empty(n, f, tile, cap, x.dtype, dev)
    y = torch.empty_like(x)
    y_fused = torch.empty_like(x)
    h = torch.empty((n, f), dtype=x.dtype, device=dev)
    y_dense = torch.empty_like(x)
    diag = sge.new_diag(dev)
    ws = sge.fused_workspace(n, d, dev)
    ws_r = sge.routed_workspace(n, d, f, s_max, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    def timed(fns, steps, warm):
        """Per-step CUDA events around each fn (same stream), L2 flush between."""
        evs = []
        for s in range(warm + steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            e[0].record(stream)
            for i, fn in enumerate(fns):
                fn()
                e[i + 1].record(stream)
            if s >= warm:
                evs.append(e)
        torch.cuda.synchronize(dev)
        return evs

    def reduce_max(v: float) -> float:
        return reduce_max_over_ranks(v, dev)

    gate = lambda: sge.twell_gate_pack(x, wg, tile, cap, out=tw, diag=diag)
    routed = lambda: sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd_t, k_route, s_max, y=y,
                                              workspace=ws_r, diag=diag)
    fused = lambda: sge.twell_fused_up_down(x, tw, wu_i, wd_i, y=y_fused, workspace=ws)
    dense = lambda: sge.dense_ffn_fwd(x, wg, wu, wd_t, h=h, y=y_dense)

    def hybrid_setup():
        hk, hs = HYB_INFER_K, spill_rows_for(n)
        hy = sge.Hybrid.empty(n, f, hk, hs, dev)
        hws = sge.hybrid_fwd_workspace(d, f, hs, dev)
        y_h = torch.empty_like(x)
        hdiag = sge.new_diag(dev)
        hpack = lambda: sge.hybrid_pack(tw, hk, hs, out=hy, diag=hdiag)
        hfwd = lambda: sge.hybrid_ffn_fwd(x, hy, wu, wd, wd_t, y=y_h, workspace=hws)
        return hk, hs, hy, y_h, hdiag, hpack, hfwd

    if args.profile:
        if args.profile_path == "hybrid":
            _, _, _, _, _, hpack, hfwd = hybrid_setup()
            timed([gate, hpack, hfwd], args.steps, args.warmup)
        elif args.profile_path == "fused":
            timed([gate, fused], args.steps, args.warmup)
        else:
            timed([gate, routed], args.steps, args.warmup)
        return None

    # ---- the sparse forward: timed region
    timed([gate, routed], 0, args.warmup)
    barrier()
    with ClockSampler(local_rank) as clk:
        barrier()
        evs = timed([gate, routed], args.steps, 0)
        barrier()
    clocks = clk.summary()
    t_gate = [e[0].elapsed_time(e[1]) for e in evs]
    t_routed = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = reduce_max(sum(a + b for a, b in zip(t_gate, t_routed)))
    ms_step = total_ms / args.steps
    value = replica_tokens_per_s(n, world, args.steps, total_ms)
    diag_host = diag.tolist()
    n_spill, nnz_light, nnz = routed_split(tw.count, cap, k_route, s_max)
    density = nnz / (n * f)

    # ---- the same forward through the per-entry kernel alone (TwELL step)
    evf = timed([gate, fused], min(args.steps, 100), 3)
    ms_fused_step = statistics.mean(e[0].elapsed_time(e[2]) for e in evf)
    ms_fused = statistics.mean(e[1].elapsed_time(e[2]) for e in evf)
    routed_vs_fused = float(((y.float() - y_fused.float()).abs().max()
                             / y_fused.float().abs().max().clamp_min(1e-30)).item())

    # ---- dense baselines on the same inputs (own tcgen05 and cuBLAS)
    evd = timed([dense], min(args.steps, 100), 3)
    ms_dense = statistics.mean(e[0].elapsed_time(e[1]) for e in evd)

    def cublas():
        hh = torch.relu(x @ wg.t()) * (x @ wu.t())
        return hh @ wd
    evc = timed([cublas], min(args.steps, 50), 3)
    ms_cublas = statistics.mean(e[0].elapsed_time(e[1]) for e in evc)

    # ---- end to end through host buffers (copies inside the timed region)
    x_host = inp.x.pin_memory()
    y_host = torch.empty(x_host.shape, dtype=x_host.dtype).pin_memory()
    x_dev2 = torch.empty_like(x)

    def e2e():
        x_dev2.copy_(x_host, non_blocking=True)
        sge.twell_gate_pack(x_dev2, wg, tile, cap, out=tw, diag=diag)
        sge.twell_hybrid_up_down(x_dev2, tw, wu_i, wd_i, wd_t, k_route, s_max, y=y, workspace=ws_r,
                                 diag=diag)
        y_host.copy_(y, non_blocking=True)
    e2e_steps = min(args.steps, 50)
    barrier()
    eve = timed([e2e], e2e_steps, 3)
    barrier()
    e2e_ms = reduce_max(sum(e[0].elapsed_time(e[1]) for e in eve))
    e2e_value = replica_tokens_per_s(n, world, e2e_steps, e2e_ms)

    # ---- the hybrid format's own path (pack into ELL + spill, then forward)
    hk, hs, hy, y_h, hdiag, hpack, hfwd = hybrid_setup()
    hsteps = min(args.steps, 100)
    timed([gate, hpack, hfwd], 0, 3)
    barrier()
    evh = timed([gate, hpack, hfwd], hsteps, 0)
    barrier()
    h_ms = reduce_max(sum(e[0].elapsed_time(e[3]) for e in evh)) / hsteps
    hyb = {"value": round(replica_tokens_per_s(n, world, 1, h_ms), 1), "unit": "tokens/s",
           "ms_per_step": round(h_ms, 4), "ell_cap_K": hk, "s_max": hs,
           "spill_rows": int(hy.n_spill.item()), "dropped_rows": int(hdiag[2].item()),
           "ms_parts": {"gate": round(statistics.mean(e[0].elapsed_time(e[1]) for e in evh), 4),
                        "hybrid_pack": round(statistics.mean(e[1].elapsed_time(e[2]) for e in evh), 4),
                        "hybrid_ffn_fwd": round(statistics.mean(e[2].elapsed_time(e[3]) for e in evh), 4)},
           "speedup_vs_own_dense": round(ms_dense / h_ms, 3),
           "note": "gate GEMM + TwELL, hybrid_pack (ELL + dense spill rows), hybrid_ffn_fwd (saves u)"}

    if rank != 0:
        return None

    pk = peaks()
    bf16_peak = pk["bf16_tflops"]
    mg = statistics.mean(t_gate)
    mr = statistics.mean(t_routed)
    flops_gate = 2.0 * n * d * f
    gate_tf = flops_gate / (mg / 1e3) / 1e12
    # the routed call's algorithmic work: the spill rows' two GEMMs over all F
    # hidden units on tensor cores, the other tokens' entries on CUDA cores
    flops_spill = 4.0 * n_spill * d * f
    flops_light = 4.0 * nnz_light * d
    routed_roof_ms = (flops_spill / (bf16_peak * 1e12) + flops_light / (FP32_SIMT_TFLOPS * 1e12)) * 1e3
    gate_roof_ms = flops_gate / (bf16_peak * 1e12) * 1e3
    # each hash covers the kernel's source and every header it includes
    gate_src = src_hash("gate_pack.cu", "tc_launch.cuh", "tc_gemm.cuh", "sge_common.cuh", "sge_host.h")
    routed_src = src_hash("routed.cu", "fused_kernels.cuh", "spill_gemm.cuh", "tc_launch.cuh",
                          "tc_gemm.cuh", "sparse_common.cuh", "debug_checks.cuh", "sge_common.cuh",
                          "sge_host.h")
    tr_gate, tr_routed = TRAFFIC.get(gate_src), TRAFFIC.get(routed_src)
    k_gate = {"kernel": "twell_gate_pack (tcgen05 GEMM + TwELL epilogue)", "bound": "tensor",
              "achieved": round(gate_tf, 1), "peak": bf16_peak, "unit": "TFLOP/s",
              "frac": round(gate_tf / bf16_peak, 4),
              "traffic": None if tr_gate is None else int(tr_gate),
              "ms": round(mg, 4), "share": round(mg / (mg + mr), 3),
              "algorithmic": f"2*N*d*F = {flops_gate:.3e} flop per launch",
              "peak_note": "bf16_tflops (burst) of measured peaks: the step keeps SM clocks at max"}
    k_routed = {"kernel": "twell_hybrid_up_down (plan 2 + spill prep + 2 tcgen05 spill GEMMs + "
                          "per-entry kernel)", "bound": "tensor",
                "achieved": round((flops_spill + flops_light) / (mr / 1e3) / 1e12, 1),
                "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(routed_roof_ms / mr, 4),
                "traffic": None if tr_routed is None else int(tr_routed),
                "ms": round(mr, 4), "share": round(mr / (mg + mr), 3),
                "algorithmic": f"4*S*d*F = {flops_spill:.3e} flop on tensor cores (S={n_spill} spill "
                               f"rows) + 4*nnz_light*d = {flops_light:.3e} flop on CUDA cores "
                               f"(nnz_light={nnz_light}): {routed_roof_ms:.4f} ms at the peaks",
                "frac_note": "algorithmic time at the peaks / measured time"}
    k_gate["traffic_unit"] = k_routed["traffic_unit"] = "bytes per launch (ncu dram read + write)"
    dominant = k_gate if mg >= mr else k_routed
    rest = k_routed if dominant is k_gate else k_gate
    step_roof_ms = gate_roof_ms + routed_roof_ms
    # the TwELL step's roofline (gate on tensor cores, 4*nnz*d on CUDA cores)
    twell_roof_ms = gate_roof_ms + 4.0 * nnz * d / (FP32_SIMT_TFLOPS * 1e12) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; tokens x d_model x d_ff shaped like a 1B FFN)",
        "config": {"workload": f"{cfg.name}: N={n} d={d} F={f} T={tile} C={cap} "
                               f"target density {cfg.rho} sigma={cfg.sigma}",
                   "step": f"twell_gate_pack + twell_hybrid_up_down (K={k_route}, S_max={s_max})",
                   "realised_density": round(density, 5), "nnz": nnz, "spill_rows": n_spill,
                   "nnz_per_entry_path": nnz_light,
                   "twell_bytes": twell_bytes(tw.count, cap, x.element_size()),
                   "l2": "flushed between steps (256 MB write outside the step events)",
                   "weights": "W_up^T and W_down interleaved row by row ([F][2d]) and W_down^T "
                              "([d][F]), both built once",
                   "parallelism": f"replicas x{world} (token batches independent)"},
        "roofline": {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")},
        "kernels": [dominant, rest],
        "step_roofline_ms": round(step_roof_ms, 4),
        "step_roofline_frac": round(step_roof_ms / ms_step, 4),
        "twell_roofline_ms": round(twell_roof_ms, 4),
        "twell_roofline_frac": round(twell_roof_ms / ms_step, 4),
        "roofline_note": "step roofline: gate flops and spill flops at the bf16 peak, the "
                         "per-entry tokens' 4*nnz*d at the fp32 FMA peak; twell roofline: gate "
                         "flops at the bf16 peak and all 4*nnz*d at the fp32 FMA peak",
        "dense": {"own_tcgen05_ms": round(ms_dense, 4), "cublas_ms": round(ms_cublas, 4),
                  "speedup_vs_own_dense": round(ms_dense / ms_step, 3),
                  "speedup_vs_cublas_dense": round(ms_cublas / ms_step, 3)},
        "twell_fused_step": {"ms_per_step": round(ms_fused_step, 4), "fused_ms": round(ms_fused, 4),
                             "value": round(n / (ms_fused_step / 1e3), 1), "unit": "tokens/s",
                             "speedup_vs_own_dense": round(ms_dense / ms_fused_step, 3),
                             "max_abs_rel_routed_vs_fused": round(routed_vs_fused, 6),
                             "note": "gate + twell_fused_up_down: every entry through the "
                                     "per-entry kernel"},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size())},
        "gpu_launches": (3 if n <= 64 else 8) * args.steps,
        "launches_note": "per step: gate GEMM + TwELL epilogue; twell_hybrid_up_down = count, jobs, "
                         "light-token kernel, spill prep, up GEMM, down GEMM, split sum (the last "
                         "exits at once when the down GEMM did not split K); for batches of at most "
                         "64 tokens: gate, plan and the small-batch kernel",
        "hybrid_inference": hyb,
        "clocks": clocks,
        "diag": diag_host,
        "gpu": torch.cuda.get_device_name(dev),
        "peaks_source": pk["source"],
    }
    return out


# ------------------------------------------------------- density sweep

SWEEP_RHO = (0.0025, 0.005, 0.01, 0.02, 0.05)


def run_sweep(args, local_rank):
    """The workload's shape at mean densities 0.25%..5%: the gate bias
    (last input row of W_gate, times the constant last feature of x) is the
    only input that changes, so W_gate's bias column is rewritten on the GPU
    for each density.  Per density: the sparse step (gate GEMM + TwELL, fused
    up/down), the hybrid inference path, and the dense FFNs."""
    import activation_sparse_gated_epilogue_b200 as sge
    from activation_sparse_gated_epilogue_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.workload]
    inp = synth.make_inputs(cfg)
    n, d, f, tile, cap = cfg.n_tokens, cfg.d_model, cfg.d_ff, cfg.tile, cfg.cap
    x, wg, wu, wd = (getattr(inp, k).to(dev) for k in ("x", "wg_t", "wu_t", "wd"))
    wd_t = wd.t().contiguous()
    # the fused kernel's weights: W_up^T and W_down interleaved row by row
    _w_ud, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    tw = sge.TwELL.empty(n, f, tile, cap, x.dtype, dev)
    y = torch.empty_like(x)
    ws = sge.fused_workspace(n, d, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = min(args.steps, 50)

    def timed(fns, steps, warm):
        evs = []
        for s_ in range(warm + steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            e[0].record(stream)
            for i, fn in enumerate(fns):
                fn()
                e[i + 1].record(stream)
            if s_ >= warm:
                evs.append(e)
        torch.cuda.synchronize(dev)
        return [[e[i].elapsed_time(e[i + 1]) for i in range(len(fns))] for e in evs]

    s_max_r = n
    ws_r = sge.routed_workspace(n, d, f, s_max_r, dev)
    k_r = routed_k(f) if args.ell_cap is None else args.ell_cap
    y_r = torch.empty_like(x)
    h = torch.empty((n, f), dtype=x.dtype, device=dev)
    y_dense = torch.empty_like(x)
    dense_ms = statistics.mean(t[0] for t in timed([lambda: sge.dense_ffn_fwd(x, wg, wu, wd_t, h=h, y=y_dense)],
                                                   steps, 3))
    pk = peaks()
    out = []
    for rho in SWEEP_RHO:
        tau = synth.solve_tau_density(rho, cfg.sigma, d)
        wg[:, d - 1] = -tau                      # rounded to the weight dtype
        gate = lambda: sge.twell_gate_pack(x, wg, tile, cap, out=tw)
        fused = lambda: sge.twell_fused_up_down(x, tw, wu_i, wd_i, y=y, workspace=ws)
        routed = lambda: sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd_t, k_r, s_max_r,
                                                  y=y_r, workspace=ws_r)
        tr = timed([gate, routed], steps, 3)
        routed_ms = statistics.mean(a + b for a, b in tr)
        n_spill_r, nnz_light_r, _ = routed_split(tw.count, cap, k_r, s_max_r)
        t = timed([gate, fused], steps, 3)
        mg = statistics.mean(a for a, _ in t)
        mf = statistics.mean(b for _, b in t)
        nnz = int(torch.minimum(tw.count.to(torch.int64), torch.tensor(cap, device=dev)).sum().item())
        per_tok = torch.minimum(tw.count.to(torch.int64), torch.tensor(cap, device=dev)).sum(1)
        hk = HYB_INFER_K
        hs = max(128, (int((per_tok > hk).sum().item()) + 127) // 128 * 128)
        hy = sge.Hybrid.empty(n, f, hk, hs, dev)
        hws = sge.hybrid_fwd_workspace(d, f, hs, dev)
        y_h = torch.empty_like(x)
        th = timed([gate, lambda: sge.hybrid_pack(tw, hk, hs, out=hy),
                    lambda: sge.hybrid_ffn_fwd(x, hy, wu, wd, wd_t=wd_t, y=y_h, workspace=hws)], steps, 3)
        hms = statistics.mean(sum(r) for r in th)
        flops_gate, flops_fused = 2.0 * n * d * f, 4.0 * nnz * d
        roof_ms = flops_gate / (pk["bf16_tflops"] * 1e12) * 1e3 + flops_fused / (FP32_SIMT_TFLOPS * 1e12) * 1e3
        step = mg + mf
        out.append({
            "sweep": f"{cfg.name} N={n} d={d} F={f} T={tile} C={cap}", "target_density": rho,
            "realised_density": round(nnz / (n * f), 5), "nnz": nnz, "tau": round(-float(wg[0, d - 1].item()), 5),
            "gate_ms": round(mg, 4), "fused_ms": round(mf, 4), "step_ms": round(step, 4),
            "tokens_per_s": round(n / (step / 1e3), 1),
            "fused_tflops": round(flops_fused / (mf / 1e3) / 1e12, 2),
            "fused_l2_row_tbs": round(4.0 * nnz * d / (mf / 1e3) / 1e12, 2),
            "step_roofline_ms": round(roof_ms, 4), "step_roofline_frac": round(roof_ms / step, 4),
            "dense_own_ms": round(dense_ms, 4), "speedup_vs_own_dense": round(dense_ms / step, 3),
            "hybrid_inference_ms": round(hms, 4), "hybrid_speedup_vs_own_dense": round(dense_ms / hms, 3),
            "hybrid_K": hk, "hybrid_spill_rows": int((per_tok > hk).sum().item()),
            "routed_ms": round(routed_ms, 4), "routed_tokens_per_s": round(n / (routed_ms / 1e3), 1),
            "routed_speedup_vs_own_dense": round(dense_ms / routed_ms, 3),
            "routed_K": k_r, "routed_S_max": s_max_r, "routed_spill_rows": n_spill_r,
            "routed_nnz_per_entry_path": nnz_light_r,
            "routed_step_roofline_frac": round((flops_gate + 4.0 * n_spill_r * d * f) / (pk["bf16_tflops"] * 1e12) * 1e3
                                               / routed_ms + 4.0 * nnz_light_r * d / (FP32_SIMT_TFLOPS * 1e12) * 1e3
                                               / routed_ms, 4),
        })
    return out


def run_cap_sweep(args, local_rank):
    """TwELL capacity C below the tile width T (C in {T/4, T/2, T}) on the
    workload: footprint of the TwELL against the tiles and rows that overflow
    C; the TwELL step at that C (overflowing tiles keep their first C
    entries, so those rows are truncated) and its error against C = T; and
    the hybrid inference path with the safety valve: rows with an
    overflowing tile go to the spill and the spill rows are recomputed from
    the gate (hybrid_ffn_fwd given W_gate), so the result is the C = T one."""
    import activation_sparse_gated_epilogue_b200 as sge
    from activation_sparse_gated_epilogue_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.workload]
    inp = synth.make_inputs(cfg)
    n, d, f, tile = cfg.n_tokens, cfg.d_model, cfg.d_ff, cfg.tile
    x, wg, wu, wd = (getattr(inp, k).to(dev) for k in ("x", "wg_t", "wu_t", "wd"))
    wd_t = wd.t().contiguous()
    # the fused kernel's weights: W_up^T and W_down interleaved row by row
    _w_ud, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    ws = sge.fused_workspace(n, d, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = min(args.steps, 50)

    def timed(fns, steps, warm):
        evs = []
        for s_ in range(warm + steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            e[0].record(stream)
            for fn in fns:
                fn()
            e[-1].record(stream)
            if s_ >= warm:
                evs.append(e)
        torch.cuda.synchronize(dev)
        return statistics.mean(e[0].elapsed_time(e[-1]) for e in evs)

    def rel(a, b):
        return float(((a.float() - b.float()).abs().max() / b.float().abs().max()).item())

    # the full-capacity result every C is compared with
    tw_full = sge.twell_gate_pack(x, wg, tile, tile)
    y_full = sge.twell_fused_up_down(x, tw_full, wu_i, wd_i, workspace=ws)
    torch.cuda.synchronize(dev)
    out = []
    for cap in (tile // 4, tile // 2, tile):
        tw = sge.TwELL.empty(n, f, tile, cap, x.dtype, dev)
        diag = sge.new_diag(dev)
        y = torch.empty_like(x)
        gate = lambda: sge.twell_gate_pack(x, wg, tile, cap, out=tw)
        fused = lambda: sge.twell_fused_up_down(x, tw, wu_i, wd_i, y=y, workspace=ws)
        sge.twell_gate_pack(x, wg, tile, cap, out=tw, diag=diag)
        torch.cuda.synchronize(dev)
        cnt = tw.count.to(torch.int64)
        over_rows = int((cnt > cap).any(1).sum().item())
        stored = torch.minimum(cnt, torch.tensor(cap, device=dev)).sum(1)
        step_ms = timed([gate, fused], steps, 3)
        err = rel(y, y_full)
        rows_differ = int(((y.float() - y_full.float()).abs().amax(1) > 0).sum().item())
        # hybrid with the safety valve
        hk = HYB_INFER_K
        n_sp = int(((stored > hk) | (cnt > cap).any(1)).sum().item())
        hs = max(128, (n_sp + 127) // 128 * 128)
        hy = sge.Hybrid.empty(n, f, hk, hs, dev)
        hws = sge.hybrid_fwd_workspace(d, f, hs, dev)
        y_h = torch.empty_like(x)
        hdiag = sge.new_diag(dev)
        hpack = lambda: sge.hybrid_pack(tw, hk, hs, out=hy, diag=hdiag)
        hfwd = lambda: sge.hybrid_ffn_fwd(x, hy, wu, wd, wd_t=wd_t, y=y_h, workspace=hws, wg_t=wg)
        h_ms = timed([gate, hpack, hfwd], steps, 3)
        out.append({
            "cap_sweep": f"{cfg.name} N={n} d={d} F={f} T={tile}", "C": cap,
            "twell_bytes": int(n * (f // tile) * (1 + 3 * cap)),
            "overflow_tiles": int(diag[0].item()), "rows_with_overflow": over_rows,
            "stored_entries": int(stored.sum().item()),
            "twell_step_ms": round(step_ms, 4), "twell_tokens_per_s": round(n / (step_ms / 1e3), 1),
            "twell_max_abs_rel_vs_full_capacity": round(err, 6), "twell_rows_differing": rows_differ,
            "hybrid_valve_ms": round(h_ms, 4), "hybrid_valve_tokens_per_s": round(n / (h_ms / 1e3), 1),
            "hybrid_K": hk, "hybrid_spill_rows": int(hy.n_spill.item()), "hybrid_s_max": hs,
            "hybrid_dropped_rows": int(hdiag[2].item()),
            "hybrid_max_abs_rel_vs_full_capacity": round(rel(y_h, y_full), 6),
        })
    return out


# ------------------------------------------------ training step (hybrid)

def run_train(args, local_rank):
    """One FFN training step from the hybrid format: gate GEMM + TwELL,
    hybrid_pack, hybrid_ffn_fwd, hybrid_ffn_bwd; against a dense bf16 step
    (cuBLAS matmuls under torch autograd) on the same inputs."""
    import activation_sparse_gated_epilogue_b200 as sge
    from activation_sparse_gated_epilogue_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.workload]
    inp = synth.make_inputs(cfg)
    n, d, f = cfg.n_tokens, cfg.d_model, cfg.d_ff
    x, wg, wu, wd, dy = (getattr(inp, k).to(dev) for k in ("x", "wg_t", "wu_t", "wd", "dy"))
    wd_t = wd.t().contiguous()
    tw = sge.TwELL.empty(n, f, cfg.tile, cfg.cap, x.dtype, dev)
    hy = sge.Hybrid.empty(n, f, cfg.ell_cap, cfg.s_max, dev)
    y = torch.empty_like(x)
    fws = sge.hybrid_fwd_workspace(d, f, cfg.s_max, dev)
    bws = sge.hybrid_bwd_workspace(n, d, f, cfg.ell_cap, cfg.s_max, dev)
    diag = sge.new_diag(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # weight layouts built once per weight update: W_down^T (the forward's
    # spill down GEMM) and [W_up | W_gate] (the backward's dX GEMM)
    w_ug = sge.transpose_up_gate(wu, wg)
    grads = (torch.empty_like(x),) + tuple(torch.empty((f, d), dtype=torch.float32, device=dev)
                                           for _ in range(3))

    def step():
        sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap, out=tw)
        sge.hybrid_pack(tw, cfg.ell_cap, cfg.s_max, out=hy, diag=diag)
        sge.hybrid_ffn_fwd(x, hy, wu, wd, wd_t=wd_t, y=y, workspace=fws)
        return sge.hybrid_ffn_bwd(x, dy, hy, wg, wu, wd, workspace=bws, w_ug=w_ug, out=grads)

    xr = x.detach().clone().requires_grad_(True)
    wgr, wur, wdr = (w.detach().clone().requires_grad_(True) for w in (wg, wu, wd))

    def dense_step():
        h = torch.relu(xr @ wgr.t()) * (xr @ wur.t())
        (h @ wdr).backward(dy)
        xr.grad = wgr.grad = wur.grad = wdr.grad = None

    def timed(fn, steps, warm):
        ts = []
        for i in range(warm + steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= warm:
                ts.append((e0, e1))
        torch.cuda.synchronize(dev)
        return [a.elapsed_time(b) for a, b in ts]

    if args.profile:
        timed(step, args.steps, args.warmup)
        return None
    with ClockSampler(local_rank) as clk:
        t_sparse = timed(step, args.steps, args.warmup)
    t_dense = timed(dense_step, min(args.steps, 50), 3)
    ms = statistics.mean(t_sparse)
    ms_dense = statistics.mean(t_dense)
    n_spill = int(hy.n_spill.item())
    nnz = int(hy.row_nnz.to(torch.int64).sum().item())

    # ---- activation memory, read from the caching allocator: what the
    # forward leaves allocated for the backward (plus y), and the peak over
    # forward + backward, both above what was allocated before the step
    # (weights, x, dy); buffers and workspaces are allocated inside.
    def measure(fwd, bwd):
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        saved = fwd()
        torch.cuda.synchronize(dev)
        held = torch.cuda.memory_allocated(dev) - base
        out = bwd(saved)
        torch.cuda.synchronize(dev)
        peak = torch.cuda.max_memory_allocated(dev) - base
        del saved, out
        return held, peak

    def hybrid_fwd():
        tw_ = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)     # transient
        hy_ = sge.hybrid_pack(tw_, cfg.ell_cap, cfg.s_max)      # saved for the backward
        ws_ = sge.hybrid_fwd_workspace(d, f, cfg.s_max, dev)
        y_ = sge.hybrid_ffn_fwd(x, hy_, wu, wd, wd_t, workspace=ws_)
        del tw_, ws_
        return hy_, y_

    def hybrid_bwd(saved):
        hy_, _ = saved
        ws_ = sge.hybrid_bwd_workspace(n, d, f, cfg.ell_cap, cfg.s_max, dev)
        return sge.hybrid_ffn_bwd(x, dy, hy_, wg, wu, wd, workspace=ws_, w_ug=w_ug)

    def dense_fwd():
        return (torch.relu(xr @ wgr.t()) * (xr @ wur.t())) @ wdr

    def dense_bwd(y_):
        y_.backward(dy)
        g = (xr.grad, wgr.grad, wur.grad, wdr.grad)
        xr.grad = wgr.grad = wur.grad = wdr.grad = None
        return g

    del tw, hy, y, fws, bws, grads
    h_held, h_peak = measure(hybrid_fwd, hybrid_bwd)
    d_held, d_peak = measure(dense_fwd, dense_bwd)
    return {
        "metric": "hybrid FFN training step tokens/s (1B shape, bf16)", "value": round(n / (ms / 1e3), 1),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: N={n} d={d} F={f} K={cfg.ell_cap} S_max={cfg.s_max} "
                               f"sigma={cfg.sigma} (tau for 2% expected spill)",
                   "nnz": nnz, "spill_rows": n_spill, "l2": "flushed between steps"},
        "dense_autograd_cublas_ms": round(ms_dense, 4),
        "speedup_vs_dense": round(ms_dense / ms, 3),
        "activation_memory_bytes": {
            "hybrid_held_after_forward": int(h_held), "dense_held_after_forward": int(d_held),
            "held_ratio": round(h_held / d_held, 4),
            "hybrid_peak_forward_backward": int(h_peak), "dense_peak_forward_backward": int(d_peak),
            "peak_ratio": round(h_peak / d_peak, 4),
            "how": "torch.cuda.memory_allocated / max_memory_allocated around one forward and one "
                   "backward, above the weights and inputs; held = activations saved for the "
                   "backward plus y (hybrid: ELL rows, routing and the S_max-row spill buffers; "
                   "dense autograd: relu(G), U and h); the peaks include workspaces, the "
                   "hybrid's transient TwELL (C = T) and its fp32 weight gradients (dense: bf16)"},
        "gpu_launches_per_step": 23,
        "launches_note": "library kernels per step: gate 1, pack 3 (counts, route, fill), forward 6 (ELL, "
                         "gather, up GEMM, its split-K sum, down GEMM, its split-K sum), backward 13 (ELL, "
                         "gather, dH GEMM, its split-K sum, 2 counts, scan, 2 scatters, sort, dW, dX GEMM, "
                         "its split-K sum); plus one cudaMemsetAsync of the bucket counts",
        "clocks": clk.summary(), "diag": diag.tolist(),
    }


# ------------------------------------------------------ CPU oracle timing

def oracle_sample(cfg, budget_s: float, max_tokens: int):
    """Time the fp64 oracle's sparse forward on the first tokens of the
    workload; the sample grows until it costs about `budget_s`."""
    import oracle
    from activation_sparse_gated_epilogue_b200 import synth
    inp = synth.make_inputs(cfg)
    xf, wgf, wuf, wdf = (inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd"))
    oracle.build()

    def run(k):
        t0 = time.perf_counter()
        oracle.sparse_ffn(xf[:k], wgf, wuf, wdf, cfg.tile, cfg.cap, oracle.VAL_BF16)
        return time.perf_counter() - t0

    k = min(8, max_tokens)
    t = run(k)
    while t < budget_s / 4 and k < max_tokens:
        k = min(max_tokens, int(k * max(2.0, min(8.0, budget_s / max(t, 1e-3) / 2))))
        t = run(k)
    return k, t


def cpu_baseline(cfg, budget_s=12.0):
    k, t = oracle_sample(cfg, budget_s, cfg.n_tokens)
    return {"value": round(k / t, 2), "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"first {k} of {cfg.n_tokens} tokens of {cfg.name}: fp64 gate GEMM, "
                      f"TwELL pack, fused up/down ({t:.1f} s, OpenMP over tokens)"}


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded token sample."""
    import oracle
    from activation_sparse_gated_epilogue_b200 import synth
    cfg = workload_config(args)
    inp = synth.make_inputs(cfg)
    xf, wgf, wuf, wdf = (inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd"))
    oracle.build()
    kind = oracle.VAL_F32 if cfg.dtype == "f32" else oracle.VAL_BF16
    t0 = time.perf_counter()
    oracle.sparse_ffn(xf[:4], wgf, wuf, wdf, cfg.tile, cfg.cap, kind)
    per_tok = (time.perf_counter() - t0) / 4
    budget = 150.0 / max(1, args.steps + args.warmup)
    k = int(max(1, min(cfg.n_tokens, budget / max(per_tok, 1e-6))))
    times = []
    for s in range(args.warmup + args.steps):
        off = (s * k) % max(1, cfg.n_tokens - k)
        t0 = time.perf_counter()
        oracle.sparse_ffn(xf[off:off + k], wgf, wuf, wdf, cfg.tile, cfg.cap, kind)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = k * args.steps / total
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{cfg.name}: N={cfg.n_tokens} d={cfg.d_model} F={cfg.d_ff} "
                                   f"T={cfg.tile} C={cfg.cap} target density {cfg.rho} sigma={cfg.sigma}",
                       "step": "fp64 oracle on the host cores: gate GEMM, TwELL pack, up/down over "
                               "the stored entries",
                       "sample_tokens_per_step": k},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": host_cores(),
                             "kind": "oracle",
                             "sample": f"{k} consecutive tokens of {cfg.name} per step"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.workload == "train_1b_hybrid":
        if rank == 0:
            out = run_train(args, local_rank)
            if out is not None:
                print(json.dumps(out), flush=True)
        return
    if args.sweep:
        if rank == 0:
            for line in run_sweep(args, local_rank):
                print(json.dumps(line), flush=True)
        return
    if args.cap_sweep:
        if rank == 0:
            for line in run_cap_sweep(args, local_rank):
                print(json.dumps(line), flush=True)
        return
    out = run_own(args, rank, world, local_rank)
    if rank == 0 and out is not None:
        out["cpu_baseline"] = None if args.no_cpu else cpu_baseline(workload_config(args))
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
