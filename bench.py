#!/usr/bin/env python
"""Benchmark of the sparse global attention path (s3r_sparse_attn_fwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload n1000] [--impl native|reference]

One step = one call of the whole path (pooling, compressed attention and scores, top-k,
selection attention with the gated combine) over one layer of synthetic inputs already resident
in HBM. Default workload: the 1000-view sequence, L = 1,374,000 tokens (N = 1000 views x P = 1374
tokens), H = 16, d = 64, b = 64, top-k = 32. Each GPU runs its own independent layer (weak
scaling, no data-path collective); the step time is the maximum over ranks.

Prints one JSON line (rank 0) with:

- tokens/s, algorithmic TFLOP/s and fraction of the measured bf16 peak;
- per-stage times from CUDA events recorded inside the fused call;
- the roofline of the dominant kernel (algorithmic bf16 FLOPs against the measured sustained
  tensor peak; for the compressed branch also its exp2 rate), both attention branches' fraction
  of that peak next to the 0.5 target, and the dominant kernel's recorded DRAM traffic;
- an end-to-end figure from pinned host memory through HostPipeline;
- dense attention (torch SDPA, flash) on the same inputs as context;
- the fp64 CPU oracle's timed sample;
- the kernel-launch count;
- the SM clocks sampled during the timed region.

Other workloads:

- n100, vggt32, tiny;
- n1000_k40, n100_k40: top-k = 40, which writes the score matrix and runs the stand-alone top-k
  kernel; n1000_k40_h1 is one head of n1000_k40;
- n1000_windows: 2-D key windows;
- vggt32_ref, vggt32_ref_windows: the reference view kept;
- pi3_sweep: 24 layers per (b, top-k) setting at 200 views.

--single-kernel runs the compressed branch, top-k and selection as one kernel.

The line also carries a "backward" object: s3r_sparse_attn_bwd (the gradients of q, k, v and the
gate logits, with the forward's selection lists held fixed) timed on the same inputs, with its
tokens/s, algorithmic TFLOP/s, per-stage times and the roofline of its dominant kernel
(--no-backward skips it).

--impl reference times the CPU oracle (the only other implementation of this method) on bounded
samples of the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS = {
    "n1000": dict(desc="1000-view sequence: N=1000 views x P=1374 tokens (37x37 patches + 5), "
                       "L=1,374,000, H=16, d=64, b=64, top-k=32, 1 layer",
                  L=1374000, H=16, block=64, topk=32, seed=3),
    # the same layer with top-k = 40: above the 32 the compressed branch selects on the fly, so
    # the [H, nqb, nb] score matrix (29.5 GB) is written and the stand-alone top-k kernel reads it
    "n1000_k40": dict(desc="1000-view sequence, top-k=40 (score matrix + stand-alone top-k): "
                           "L=1,374,000, H=16, d=64, b=64, 1 layer",
                      L=1374000, H=16, block=64, topk=40, seed=3),
    # one head of that layer: the same 21,470-block score rows, 1/16 of them (1.84 GB), a size
    # at which the stand-alone top-k can be profiled launch by launch
    "n1000_k40_h1": dict(desc="1000-view sequence, one head, top-k=40 (score matrix + "
                              "stand-alone top-k): L=1,374,000, H=1, d=64, b=64, 1 layer",
                         L=1374000, H=1, block=64, topk=40, seed=3),
    "n100": dict(desc="100-view layer: L=137,400, H=16, d=64, b=64, top-k=32",
                 L=137400, H=16, block=64, topk=32, seed=2),
    "n100_k40": dict(desc="100-view layer, top-k=40 (score matrix + stand-alone top-k): "
                          "L=137,400, H=16, d=64, b=64",
                     L=137400, H=16, block=64, topk=40, seed=2),
    "vggt32": dict(desc="VGGT-like layer: N=32 views x P=1374, L=43,968, H=16, d=64, b=64, top-k=16",
                   L=43968, H=16, block=64, topk=16, seed=1),
    # VGGT's hybrid: the reference view's blocks kept for every query (ceil(1374/64) = 22 leading
    # blocks; with windows, the view's 26 blocks), top-k = 16 more
    "vggt32_ref": dict(desc="VGGT-like layer with the reference view kept: N=32 x P=1374, "
                            "L=43,968, H=16, d=64, b=64, forced=22, top-k=16",
                       L=43968, H=16, block=64, topk=16, seed=1, forced=22),
    "vggt32_ref_windows": dict(desc="VGGT-like layer with 2-D key windows and the reference view "
                                    "kept: N=32 x (5 + 37x37), 8x8 windows, L=43,968, H=16, "
                                    "d=64, b=64, forced=26, top-k=16",
                               L=43968, H=16, block=64, topk=16, seed=1, forced=26,
                               geo=dict(grid_h=37, grid_w=37, special=5, win_h=8)),
    "tiny": dict(desc="tiny: N=4 x P=256, L=1024, H=2, d=64, b=64, top-k=4",
                 L=1024, H=2, block=64, topk=4, seed=0),
    # the same 1000 views with key blocks as 2-D windows: each view's 5 camera/register tokens,
    # then 8 x 8 windows of its 37 x 37 patch grid (26 blocks a view, 26,000 in all)
    "n1000_windows": dict(desc="1000-view sequence with 2-D key windows: N=1000 x P=1374 "
                               "(5 special tokens + 37x37 patches), 8x8-patch windows, L=1,374,000, "
                               "H=16, d=64, b=64, top-k=32, 1 layer",
                          L=1374000, H=16, block=64, topk=32, seed=3,
                          geo=dict(grid_h=37, grid_w=37, special=5, win_h=8)),
}

METRIC = "sparse global-attn tokens/s at 1000 views"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


# MUFU.EX2 rate of one SM per clock (4 sub-partitions x 4 lanes), as tests/test_gpu_exp2_rate.py
# measures it in SM clock cycles, and the SM count of a B200.
EX2_PER_CLK_SM = 16
SM_COUNT = 148

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the kernel that bounds
# the step at 1000 views: one ncu capture of that kernel on the 100-view layer (python bench.py
# --workload n100 --steps 1 --warmup 3 --no-backward --no-cpu-baseline --no-dense-context; 290.5
# MB read + 513.2 MB written), scaled by the ratio of rows (10.0: its traffic, Q read and O_cmp
# written, is proportional to L). With the SHA-256 of the sources that kernel was built from: once
# any of them changes, the figure no longer describes the kernel and the roofline reports null.
TRAFFIC = {
    "cmp": {"workload": "n1000", "bytes": (290472704 + 513215744) * 10,
             "sources": ["sparse_global_attention_s3r_b200/csrc/cmp_attn_tc.cu",
                         "sparse_global_attention_s3r_b200/csrc/common.cuh",
                         "sparse_global_attention_s3r_b200/csrc/sm100.cuh"],
             "sha256": "8828d658b7681ded38a8e6083a06784d26930157f351ac1ec61579703cd77c02"},
}


def _sources_sha(paths):
    import hashlib

    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(stage: str, workload: str):
    rec = TRAFFIC.get(stage)
    if not rec or rec["workload"] != workload:
        return None
    try:
        if _sources_sha(rec["sources"]) != rec["sha256"]:
            return None
    except OSError:
        return None
    return rec["bytes"]


def algorithmic(cfg):
    """Algorithmic work per call: FLOPs of Q.Kc^T + P.Vc (once) and of the selection's
    Q.K^T + P.V over the tokens actually selected; bytes of each stage's compulsory traffic."""
    L, H, d, b, k, nb, nqb = cfg.L, cfg.H, cfg.d, cfg.block, cfg.topk, cfg.nb, cfg.nqb
    # tokens selected per query block: forced + k blocks of b (an upper bound: the ragged last
    # 1-D block, and 2-D windows cut at a grid edge or a view's special-token block, hold fewer)
    sel_tokens = (getattr(cfg, "forced", 0) + k) * b
    cmp_flops = 4.0 * L * nb * d * H
    sel_flops = 4.0 * L * sel_tokens * d * H
    single = getattr(cfg, "single_kernel", False)  # the compressed stage also runs selection
    return {
        # one exp2 per (query, summary) pair in each of the two passes (+ one per selected token)
        "cmp_exp2": 2.0 * L * nb * H + (L * sel_tokens * H if single else 0.0),
        "cmp_flops": cmp_flops,
        "sel_flops": sel_flops,
        "flops": cmp_flops + sel_flops,
        "stage_work": {
            # K, V read; Kc, Vc and the head-major copies of K, V (nb*b rows) written
            "pool": ("hbm", 2.0 * (L + nb + nb * b) * H * d * 2),              # bytes
            "cmp": ("tensor", cmp_flops + (sel_flops if single else 0.0)),    # flops
            "topk": ("hbm", H * nqb * (nb * 4.0 + k * 4.0)),                  # bytes
            "sel_combine": ("tensor", 0.0 if single else sel_flops),          # flops
        },
    }


def algorithmic_bwd(cfg):
    """Algorithmic work of the backward: the five products of softmax attention's gradient
    (S, dP, dQ, dK, dV: 10 L n d H FLOPs over n keys) for both branches, and per stage what its
    kernel computes of them (the dq kernel forms S, dP and dQ; the key-side kernels S, dP, dK and
    dV); the recompute stage is the forward."""
    L, H, d = cfg.L, cfg.H, cfg.d
    n_cmp = cfg.nb
    n_sel = (getattr(cfg, "forced", 0) + cfg.topk) * cfg.block
    fwd = algorithmic(cfg)["flops"]
    return {
        "flops": 10.0 * L * H * d * (n_cmp + n_sel),
        "stage_work": {
            "recompute": ("tensor", fwd),
            # dout, O_cmp, O_sel read; the statistics and dgates written
            "prep": ("hbm", L * H * (64 * 2 + 2 * 64 * 4 + 6 * 4 + 2 * 4.0)),
            "dq": ("tensor", 6.0 * L * H * d * (n_cmp + n_sel)),
            "dkv_cmp": ("tensor", 8.0 * L * H * d * n_cmp),
            "dkv_sel": ("tensor", 8.0 * L * H * d * n_sel),
        },
    }


def time_backward(args, cfg, q, k, v, gates, idx, dev, barrier, peaks):
    """K timed calls of s3r_sparse_attn_bwd after W warm-up calls (a seeded bf16 dout)."""
    import torch

    from sparse_global_attention_s3r_b200 import _lib, api

    g = torch.Generator(device=dev).manual_seed(99)
    dout = torch.randn(q.shape, generator=g, device=dev).to(torch.bfloat16)
    # training use: the forward keeps what the backward needs (save_for_backward), and the
    # backward reads it from the same workspace instead of recomputing the forward
    cfg = dataclasses.replace(cfg, save_for_backward=True, single_kernel=False)
    ws = torch.empty(api.bwd_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    idx = torch.empty_like(idx)
    for _ in range(args.warmup):
        api.sparse_attn_fwd(cfg, q, k, v, gates, ws, out, idx)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        api.sparse_attn_fwd(cfg, q, k, v, gates, ws, out, idx)
    f1.record()
    torch.cuda.synchronize()
    fwd_save_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps, dev)
    grads = (*(torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3)),
             torch.empty(gates.shape, dtype=torch.float32, device=dev))
    for _ in range(args.warmup):
        api.sparse_attn_bwd(cfg, q, k, v, gates, idx, dout, ws, grads=grads)
    torch.cuda.synchronize()
    evs = [api.StageEvents(_lib.BWD_STAGES) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    n0 = _lib.kernel_launches()
    e0.record()
    for s in range(args.steps):
        api.sparse_attn_bwd(cfg, q, k, v, gates, idx, dout, ws, stage_events=evs[s], grads=grads)
    e1.record()
    torch.cuda.synchronize()
    launches = _lib.kernel_launches() - n0
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    stage_ms = {n: statistics.mean(e.stage_ms()[n] for e in evs) for n in _lib.BWD_STAGES}
    work = algorithmic_bwd(cfg)
    stages = {}
    for n, (b_, u_) in work["stage_work"].items():
        s_ = stage_ms[n] / 1e3
        if s_ < 1e-5:  # no launch in this stage (the recompute, after a saving forward)
            stages[n] = {"ms": stage_ms[n], "launched": False}
            continue
        stages[n] = {"ms": stage_ms[n],
                     ("GB/s" if b_ == "hbm" else "TFLOP/s"): u_ / s_ / (1e9 if b_ == "hbm" else 1e12)}
    dom = max(("dq", "dkv_cmp", "dkv_sel"), key=stage_ms.get)
    ach = work["stage_work"][dom][1] / (stage_ms[dom] / 1e3) / 1e12
    del ws, grads, dout, out
    return {
        "ms_per_step": ms, "tokens_per_s": cfg.L / (ms / 1e3),
        "forward_save_ms": fwd_save_ms,
        "train_step_ms": fwd_save_ms + ms,
        "tflops": work["flops"] / (ms / 1e3) / 1e12, "stage_ms": stages,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": ach,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": ach / peaks["bf16_tflops_sustained"],
                     "peak_source": peaks["source"] + " sustained bf16", "traffic": None},
        "gpu_launches": launches,
        "how": "s3r_sparse_attn_bwd on the forward's own selection lists and a seeded bf16 dout, "
               "reading what a save_for_backward forward kept in the same workspace (the "
               "recompute stage is empty); forward_save_ms times that forward, train_step_ms "
               "is forward + backward",
    }


def rank_seed(base: int, rank: int) -> int:
    """Seed of the independent layer a rank runs (weak scaling: one layer per GPU)."""
    return base + 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the job's step time); identity without a process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def physical_gpu(local: int) -> str:
    """nvidia-smi's name for CUDA device `local` of this process."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        return vis.split(",")[local].strip()
    return str(local)


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
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
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# the CPU oracle, timed on a bounded sample of the workload
# ---------------------------------------------------------------------------------------------

def sample_blocks(nqb: int, n_blocks: int, seed: int):
    """A seeded sample of whole query blocks, the ragged last one always included."""
    import numpy as np

    rng = np.random.default_rng(seed)
    return sorted(set(rng.choice(nqb - 1, size=max(0, min(n_blocks, nqb) - 1),
                                 replace=False).tolist() if nqb > 1 else []) | {nqb - 1})


def oracle_sample(cfg, host_bits, gates_np, n_blocks: int, seed: int, result=None):
    """Time the oracle: pooling of all K/V plus the whole path for n_blocks query blocks (all
    heads). Returns (tokens/s extrapolated to the full layer, seconds, description, threads);
    `result`, a dict, receives the sampled blocks and the oracle's outputs for them."""
    from oracle import oracle as O

    pb = O.Problem(cfg.L, cfg.H, cfg.d, cfg.block, cfg.topk, forced=cfg.forced, grid_h=cfg.grid_h,
                   grid_w=cfg.grid_w, special=cfg.special, win_h=cfg.win_h)
    blocks = sample_blocks(cfg.nqb, n_blocks, seed)
    q, k, v = host_bits
    t0 = time.perf_counter()
    kc = O.pool(pb, k)
    vc = O.pool(pb, v)
    t1 = time.perf_counter()
    ref = O.sparse_attn(pb, q, k, v, gates_np, qblocks=blocks, pooled=(kc, vc))
    t2 = time.perf_counter()
    rows = int(pb.rows_of(blocks).size)
    t_full = (t1 - t0) + (t2 - t1) * cfg.L / rows
    desc = (f"pooling of all {cfg.nb} K/V blocks + the whole path for {len(blocks)} seeded query "
            f"blocks ({rows} rows, all {cfg.H} heads); extrapolated to L={cfg.L}")
    if result is not None:
        result.update(blocks=blocks, rows=pb.rows_of(blocks), ref=ref)
    return cfg.L / t_full, t2 - t0, desc, O.hardware_threads()


def parity_stats(got_idx, got_out, ref, forced: int) -> dict:
    """The GPU's lists and output on the oracle's sampled query blocks, against the oracle run on
    its own lists: the fraction of query blocks with the same selected set, the fraction whose
    k-th/(k+1)-th score gap exceeds 1e-4 (where the sets must agree), and the output's max-abs
    and relative-L2 error over the query blocks whose sets agree."""
    import numpy as np

    g = np.sort(got_idx[..., forced:], -1)
    r = np.sort(ref.idx[..., forced:], -1)
    same = (g == r).all(-1)                       # [H, nq]
    out, want = np.asarray(got_out, np.float64), np.asarray(ref.out, np.float64)
    # a row of a query block, head h, counts where that block's set agrees for head h
    qb_of_row = ref.rows // 64
    pos = np.searchsorted(np.unique(qb_of_row), qb_of_row)
    mask = same[:, pos].T[..., None]              # [R, H, 1]
    diff = np.where(mask, out - want, 0.0)
    ref_m = np.where(mask, want, 0.0)
    return {"query_blocks": int(same.shape[1]), "sets_equal": float(same.mean()),
            "gap_separated": float((ref.gap > 1e-4).mean()),
            "max_abs": float(np.abs(diff).max()),
            "rel_l2": float(np.sqrt((diff ** 2).sum() / max((ref_m ** 2).sum(), 1e-300)))}


def workload_config(wl, world: int, l2_note: str) -> dict:
    """The `config` object of the JSON line: the same keys and values in both arms."""
    return {"workload": wl["desc"], "L": wl["L"], "H": wl["H"], "d": 64, "block": wl["block"],
            "topk": wl["topk"], "forced": wl.get("forced", 0), "qblock": 64, "seed": wl["seed"],
            **wl.get("geo", {}),
            "parallelism": "independent layer per GPU" if world > 1 else "single GPU",
            "l2": l2_note}


def l2_note(L: int, H: int) -> str:
    gb = L * H * 64 * 2 / 1e9
    if gb > 0.126:
        return "inputs exceed L2 (each of Q/K/V is %.2f GB > 126 MB); no flush" % gb
    return "inputs fit in L2 (each of Q/K/V is %.1f MB); no flush" % (gb * 1e3)


def run_reference(args, wl):
    """--impl reference: the CPU oracle on bounded samples; rank 0 only. Nothing of the CUDA
    library is loaded on this path: sizes come from the oracle's own Problem, inputs from the
    seeded generator (on the GPU when there is one, so that they equal the native arm's)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch

    from oracle import oracle as O
    from sparse_global_attention_s3r_b200 import synth

    pb = O.Problem(wl["L"], wl["H"], 64, wl["block"], wl["topk"], forced=wl.get("forced", 0),
                   **wl.get("geo", {}))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.make_inputs(pb.L, pb.H, pb.d, pb.block, wl["seed"], device=dev)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    gates = x.gates.cpu().numpy()
    del x
    n_blocks = max(1, min(4, pb.nqb))
    for w in range(args.warmup):
        oracle_sample(pb, bits, gates, n_blocks, seed=w)
    vals, secs = [], []
    desc = threads = None
    for s in range(args.steps):
        v, t, desc, threads = oracle_sample(pb, bits, gates, n_blocks, seed=100 + s)
        vals.append(v)
        secs.append(t)
    value = statistics.median(vals)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # the seconds one sampled step really took; the full layer is extrapolated below
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world, l2_note(pb.L, pb.H)),
        "extrapolated_full_layer_ms": 1e3 * pb.L / value,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": desc + f"; median of {args.steps} samples of "
                                          f"{statistics.median(secs):.1f} s"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------------------------

def run_native(args, wl):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_global_attention_s3r_b200 import _lib, api, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl native")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    cfg = api.Config(L=wl["L"], H=wl["H"], block=wl["block"], topk=wl["topk"],
                     forced=wl.get("forced", 0), single_kernel=args.single_kernel,
                     **wl.get("geo", {}))
    seed = rank_seed(wl["seed"], rank)  # an independent layer per GPU
    x = synth.make_inputs(cfg.L, cfg.H, cfg.d, cfg.block, seed, device=dev)
    q, k, v, gates = x.q, x.k, x.v, x.gates
    sa = api.SparseAttention(cfg, dev)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        sa(q, k, v, gates)
    torch.cuda.synchronize()

    stage_ev = [api.StageEvents() for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(local)) as clocks:
        time.sleep(0.3)
        n0 = _lib.kernel_launches()
        start.record()
        for s in range(args.steps):
            api.sparse_attn_fwd(cfg, q, k, v, gates, sa.workspace, sa.out, sa.idx,
                                stage_events=stage_ev[s])
        end.record()
        torch.cuda.synchronize()
        launches = _lib.kernel_launches() - n0
    barrier()
    ms_max = max_over_ranks(start.elapsed_time(end) / args.steps, dev)
    stage_ms = {n: statistics.mean(e.stage_ms()[n] for e in stage_ev) for n in _lib.STAGES}
    step_ms = [sum(e.stage_ms().values()) for e in stage_ev]
    # the GPU's lists and output on the query blocks the CPU-baseline leg will give the oracle
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    got = None
    if do_cpu:
        blocks = sample_blocks(cfg.nqb, args.oracle_blocks, 7)
        rows = torch.cat([torch.arange(64 * i, min(64 * i + 64, cfg.L)) for i in blocks]).to(dev)
        got = (sa.idx[:, blocks].cpu().numpy(), sa.out.index_select(0, rows).double().cpu().numpy())
    bwd = (time_backward(args, cfg, q, k, v, gates, sa.idx, dev, barrier, load_peaks())
           if not args.no_backward else None)

    # end to end through the public API from pinned host memory: every step copies all of its
    # inputs in and its output out. HostPipeline overlaps the copy-in of step i+1 and the
    # copy-out of step i-1 with the kernels of step i (two sets of device buffers, two copy
    # streams); the timed region runs from before the first copy-in to after the last copy-out.
    host = [t_.cpu().pin_memory() for t_ in (q, k, v, gates)]
    outs_h = [torch.empty(sa.out.shape, dtype=sa.out.dtype).pin_memory() for _ in range(2)]
    del sa
    pipe = api.HostPipeline(cfg, dev)
    # at least 12 steps: the first step's copy-in and the last one's copy-out overlap no kernels,
    # and over more steps their share of the time approaches what a long stream of steps sees
    e2e_steps = max(12, args.steps)
    pipe.submit(*host, outs_h[0])
    pipe.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s_ in range(e2e_steps):
        pipe.submit(*host, outs_h[s_ % 2], after=e0 if s_ == 0 else None)
    e1.record(pipe.copy_out)
    pipe.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    h2d = sum(t_.numel() * t_.element_size() for t_ in host)
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    del host, outs_h, pipe

    # context, not a target: dense attention on the same Q, K, V (torch's SDPA, the library's
    # flash kernel) for a seeded sample of query rows against all L keys, extrapolated linearly
    # in the rows (each row's attention is independent of the others)
    dense = None
    if rank == 0 and not args.no_dense_context:
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel

        rows = min(cfg.L, args.dense_rows)
        r0 = int(torch.randint(0, cfg.L - rows + 1, (1,), generator=torch.Generator().manual_seed(5)))
        qh = q[r0:r0 + rows].permute(1, 0, 2).unsqueeze(0)  # [1, H, rows, d] views
        kh_, vh_ = k.permute(1, 0, 2).unsqueeze(0), v.permute(1, 0, 2).unsqueeze(0)
        try:
            # the flash kernel only: a fallback would materialise rows x L logits
            with sdpa_kernel(SDPBackend.FLASH_ATTENTION):
                for _ in range(2):
                    F.scaled_dot_product_attention(qh, kh_, vh_)
                torch.cuda.synchronize()
                d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                d0.record()
                F.scaled_dot_product_attention(qh, kh_, vh_)
                d1.record()
                torch.cuda.synchronize()
            dense_ms = d0.elapsed_time(d1) * cfg.L / rows
            dense = {"ms_per_layer": dense_ms, "sparse_speedup": dense_ms / ms_max,
                     "tflops": 4.0 * cfg.L * cfg.L * cfg.d * cfg.H / (dense_ms / 1e3) / 1e12,
                     "how": f"torch SDPA (flash) on {rows} seeded query rows x all {cfg.L} keys, "
                            f"all {cfg.H} heads, extrapolated to {cfg.L} rows"}
        except RuntimeError as e:
            dense = {"unavailable": str(e).splitlines()[0][:200]}
        del qh, kh_, vh_

    cpu = parity = None
    if do_cpu:
        from oracle import oracle as O

        bits = [O.bf16_bits(t_) for t_ in (q, k, v)]
        res = {}
        val, secs, desc, threads = oracle_sample(cfg, bits, gates.cpu().numpy(),
                                                 args.oracle_blocks, seed=7, result=res)
        cpu = {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": desc + f"; {secs:.1f} s of CPU work"}
        parity = parity_stats(*got, res["ref"], cfg.forced)
        del bits, res

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = load_peaks()
    work = algorithmic(cfg)
    tokens_per_s = cfg.L * world / (ms_max / 1e3)
    tflops = work["flops"] * world / (ms_max / 1e3) / 1e12
    dom = max(stage_ms, key=stage_ms.get)
    bound, units = work["stage_work"][dom]
    dom_s = stage_ms[dom] / 1e3
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": units / dom_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": units / dom_s / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["source"] + (" sustained bf16" if bound == "tensor" else " copy")
    if dom == "cmp":
        # The compressed branch needs two exponentials per (query, summary) pair; their units
        # (MUFU.EX2 at 16 per clock per SM, tests/test_gpu_exp2_rate.py, plus the part evaluated
        # as a polynomial on the FMA pipe) bound it before its tensor work does. That exp2 rate
        # is reported beside the tensor roofline, not instead of it.
        ex2_peak = EX2_PER_CLK_SM * SM_COUNT * peaks.get("sm_max_mhz", 1965.0) * 1e6
        ach = work["cmp_exp2"] / dom_s
        roof["exp2_view"] = {"achieved": ach / 1e12, "unit": "Texp2/s",
                             "mufu_peak": ex2_peak / 1e12, "frac_of_mufu": ach / ex2_peak,
                             "mufu_peak_source": "16 ex2 per clock per SM (measured by "
                                                 "tests/test_gpu_exp2_rate.py) x 148 SMs x max "
                                                 "SM clock"}
    # both attention branches against the measured sustained bf16 peak (the stated target: 0.5)
    two_ms = stage_ms["cmp"] + stage_ms["sel_combine"]
    if two_ms > 0:
        two = work["flops"] / (two_ms / 1e3) / 1e12
        roof["two_branches"] = {"stages": ["cmp", "sel_combine"], "ms": two_ms,
                                "achieved": two, "unit": "TFLOP/s",
                                "frac": two / peaks["bf16_tflops_sustained"], "target_frac": 0.5}
    roof["traffic"] = measured_traffic(dom, args.workload)
    roof["kernel"] = dom
    stages = {}
    for n in _lib.STAGES:
        b_, u_ = work["stage_work"][n]
        s_ = stage_ms[n] / 1e3
        if s_ < 1e-5:  # no launch in this stage (top-k selected inside the compressed stage)
            stages[n] = {"ms": stage_ms[n], "launched": False}
            continue
        stages[n] = {"ms": stage_ms[n],
                     ("GB/s" if b_ == "hbm" else "TFLOP/s"): u_ / s_ / (1e9 if b_ == "hbm" else 1e12)}
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, world, l2_note(cfg.L, cfg.H)),
        "kernels": "pool + one fused kernel" if args.single_kernel else
                   "pool + compressed/top-k + selection/combine",
        "tflops": tflops,
        "frac_bf16_peak": tflops / world / peaks["bf16_tflops"],
        "frac_bf16_peak_sustained": tflops / world / peaks["bf16_tflops_sustained"],
        "stage_ms": stages,
        "roofline": roof,
        "e2e": {"value": cfg.L * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "how": "HostPipeline: pinned host inputs copied in and outputs copied out every "
                       "step, overlapped with the neighbouring steps' kernels; the timed region "
                       "runs from before the first copy-in to after the last copy-out"},
        "cpu_baseline": cpu,
        "gpu_launches": launches,
        "dense_context": dense,
        "clocks": clocks.summary(),
    }
    if bwd is not None:
        line["backward"] = bwd
    if parity is not None:
        line["parity"] = parity
    print(json.dumps(line), flush=True)
    if args.records:  # one record per (config, timed step), appended
        with open(args.records, "a") as f:
            for s_, ms_ in enumerate(step_ms):
                rec = {"workload": args.workload, "config": line["config"], "step": s_,
                       "ms": ms_, "tokens_per_s": cfg.L / (ms_ / 1e3),
                       "tflops": work["flops"] / (ms_ / 1e3) / 1e12,
                       "frac_bf16_sustained": work["flops"] / (ms_ / 1e3) / 1e12
                       / peaks["bf16_tflops_sustained"],
                       "stage_ms": {n: e_ for n, e_ in stage_ev[s_].stage_ms().items()},
                       "stage_rates": stages, "parity": parity,
                       "host_cores": cpu["cores"] if cpu else None, "clocks": line["clocks"]}
                f.write(json.dumps(rec) + "\n")


# the pi^3-like sweep at N = 200 views (L = 274,800, H = 16): each (b, top-k) setting is a stack of
# 24 layers with independent seeded inputs, generated before the timed region
SWEEP = dict(L=274800, H=16, layers=24, settings=((32, 32), (64, 16), (128, 8)), seed=4000)


def run_sweep(args):
    """One step = the whole path over all 24 layers of every setting; prints one JSON line with
    the summed attention time and tokens/s of each setting."""
    import torch

    from sparse_global_attention_s3r_b200 import _lib, api, synth

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", 0)
    L, H, layers = SWEEP["L"], SWEEP["H"], SWEEP["layers"]
    result, total_ms, launches = {}, 0.0, 0
    with ClockSampler(physical_gpu(0)) as clocks:
        for b, k in SWEEP["settings"]:
            cfg = api.Config(L=L, H=H, block=b, topk=k)
            xs = [synth.make_inputs(L, H, 64, b, SWEEP["seed"] + 100 * b + i, device=dev)
                  for i in range(layers)]
            sa = api.SparseAttention(cfg, dev)
            for _ in range(args.warmup):
                for x in xs:
                    sa(x.q, x.k, x.v, x.gates)
            torch.cuda.synchronize()
            n0 = _lib.kernel_launches()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                for x in xs:
                    sa(x.q, x.k, x.v, x.gates)
            e1.record()
            torch.cuda.synchronize()
            launches += _lib.kernel_launches() - n0
            ms = e0.elapsed_time(e1) / args.steps  # one pass over the 24-layer stack
            total_ms += ms
            result[f"b{b}_k{k}"] = {"ms_24_layers": ms, "ms_per_layer": ms / layers,
                                    "tokens_per_s": layers * L / (ms / 1e3), "nb": cfg.nb}
            del xs, sa
            torch.cuda.empty_cache()
    n_settings = len(SWEEP["settings"])
    line = {
        "metric": "sparse global-attn tokens/s, pi3-like sweep at 200 views (24 layers per setting)",
        "value": n_settings * layers * L / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "pi3-like sweep: N=200 views, L=274,800, H=16, d=64, "
                               "(b, top-k) in {(32,32), (64,16), (128,8)}, 24 layers each",
                   "L": L, "H": H, "layers": layers,
                   "l2": "each layer's Q/K/V (563 MB each) exceed L2; no flush"},
        "sweep": result, "gpu_launches": launches, "clocks": clocks.summary(),
    }
    print(json.dumps(line))


def run_sweep_records(args):
    """--sweep: run each named workload in its own process, appending to --records; a workload
    whose records are already in the file is skipped, so an interrupted sweep resumes."""
    if not args.records:
        raise SystemExit("--sweep needs --records")
    names = [n.strip() for n in args.sweep.split(",") if n.strip()]
    unknown = [n for n in names if n not in WORKLOADS]
    if unknown:
        raise SystemExit(f"unknown workloads: {unknown}")
    done = set()
    if os.path.exists(args.records):
        with open(args.records) as f:
            for ln in f:
                try:
                    done.add(json.loads(ln)["workload"])
                except (ValueError, KeyError):
                    continue
    passthrough = ["--steps", str(args.steps), "--warmup", str(args.warmup),
                   "--oracle-blocks", str(args.oracle_blocks)]
    for flag in ("no_cpu_baseline", "no_backward", "no_dense_context", "single_kernel"):
        if getattr(args, flag):
            passthrough.append("--" + flag.replace("_", "-"))
    for n in names:
        if n in done:
            print(f"sweep: {n} already recorded, skipped", flush=True)
            continue
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--workload", n,
                            "--records", args.records] + passthrough)
        if r.returncode != 0:
            raise SystemExit(f"sweep: {n} failed with exit code {r.returncode}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["pi3_sweep"], default="n1000")
    ap.add_argument("--oracle-blocks", type=int, default=32,
                    help="query blocks in the timed CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--single-kernel", action="store_true",
                    help="run the compressed branch, top-k and selection as one kernel (k <= 32)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the backward (s3r_sparse_attn_bwd) on the same inputs")
    ap.add_argument("--no-dense-context", action="store_true",
                    help="skip timing dense attention (torch SDPA) on a sample of query rows")
    ap.add_argument("--dense-rows", type=int, default=16384,
                    help="query rows of the dense-attention context sample")
    ap.add_argument("--records", default=None,
                    help="append one JSON record per (workload, timed step) to this file")
    ap.add_argument("--sweep", default=None,
                    help="comma-separated workloads, each run in its own process with --records; "
                         "workloads already in the records file are skipped (resume)")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep_records(args)
    if args.workload == "pi3_sweep":
        if args.impl == "reference":
            raise SystemExit("--impl reference times the oracle on the single-layer workloads")
        return run_sweep(args)
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_native(args, wl)


if __name__ == "__main__":
    main()
