"""Benchmark of the block-sparse video self-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload h3_768p_5s] [--top-k K] [--no-cpu-baseline] [--no-e2e]
                    [--precision bf16|fp8] [--reblock] [--tau T] [--extra-tokens N]
                    [--shard heads [--gather]]

One step = one whole attention call (pool -> summarize -> select -> attend,
all through the C ABI) over one batch of synthetic bf16 input of the 768p-5s
H3 shape (B=1, H=56, N=37,740, d=128, top_k=64, anchor-weighted summaries).
``--reblock`` times the adaptive-reblocking option: the reblocked layout
(bsa_reblock), the four stages on it (pool and summarize gathering the rows
through the permutation) and the scatter
of O back, every step.
``--precision fp8`` times the FP8 (e4m3) option instead: the same stages plus
the quantisation of the attention operands, then the e4m3 attention kernel;
its roofline peak is the measured bf16 peak times the nominal e4m3/bf16
tensor ratio (2).  ``--tau T`` times the threshold-selection option: the
selection keeps the key blocks at least T standard deviations above each
row's mean score (bsa_select_threshold) and the attention runs over those
variable-length lists (bsa_attend_lists, its schedule kernel included in
the stage time).  ``--extra-tokens N`` times the extra-token option: the N
top-scoring tokens of the unlisted blocks of every query block are read
exactly (bsa_select_extra), the blocks that lose tokens get summary rows of
their remaining tokens (bsa_extra_summaries) and the attention reads both
(bsa_attend_extra).  The default (bf16, top_k) line is the headline.
Prints ONE JSON line on rank 0.  Multi-GPU (torchrun): the (b, h) slices of
the job are split into contiguous per-rank ranges and every rank runs one
attention call over its own range, with no data-path collective (every stage
is per head).  By default the job grows with the ranks (weak scaling: the
batch holds one video per rank, each rank runs its video's 56 heads);
``--shard heads`` splits the heads of one video across the ranks instead
(strong scaling: 56 / N heads per rank), and ``--gather`` then adds an
all-gather of O over NCCL to the timed step.  The time is the max over ranks;
the effective FLOPs are summed over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

REF_QBLOCKS = 48
METRIC = "ms/attention call and effective TFLOP/s vs bf16 peak (56 heads, d=128, top_k=64)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="h3_768p_5s")
    ap.add_argument("--top-k", type=int, default=None)
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (small profiling captures only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp8"])
    ap.add_argument("--reblock", action="store_true")
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--extra-tokens", type=int, default=None)
    ap.add_argument("--shard", default=None, choices=["heads"],
                    help="split one call's heads across the ranks (strong scaling)")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard heads: all-gather O over NCCL inside the timed step")
    args = ap.parse_args()
    if args.gather and args.shard != "heads":
        ap.error("--gather needs --shard heads")
    if args.reblock and args.precision != "bf16":
        ap.error("--reblock runs the bf16 path")
    if args.tau is not None and (args.reblock or args.precision != "bf16"):
        ap.error("--tau runs the bf16 path without reblocking")
    if args.extra_tokens is not None and (args.reblock or args.precision != "bf16" or
                                          args.tau is not None):
        ap.error("--extra-tokens runs the bf16 top-k path without reblocking")
    if args.extra_tokens is not None and not (0 <= args.extra_tokens <= 512):
        ap.error("--extra-tokens takes 0 .. 512")
    return args


def reblock_launches(N: int, prefix: int) -> int:
    """Kernels bsa_reblock launches (its tree shape depends on N - prefix only):
    init + key moment (Gram, reduction) + factor + whiten, then per level a
    Gram and a split, plus a power-iteration pass and a projection on levels
    whose largest group spans more than one 2048-row chunk (single-chunk
    groups finish in their Gram CTA) and a partial-sum reduction where it
    spans four or more."""
    nv = N - prefix
    levels = 0
    while (128 << levels) < nv:
        levels += 1
    if levels == 0:
        return 1
    n, largest = 5, nv
    for _ in range(levels):
        chunks = (largest + 2047) // 2048
        n += 2 + (2 if chunks > 1 else 0) + (1 if chunks >= 4 else 0)
        largest -= ((largest + 127) // 128 // 2) * 128
    return n


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ accounting

def block_sizes(N):
    nb = -(-N // 128)
    sizes = np.full(nb, 128, dtype=np.int64)
    sizes[-1] = N - 128 * (nb - 1)
    return sizes


def effective_pairs(idx, cnt, N, prefix):
    """Computed (query, key or summary) pairs of all heads: exact pairs over
    the real tokens of each listed block plus one summary column per skipped
    video block for every video query row (masked columns excluded)."""
    sizes = block_sizes(N)
    nb = len(sizes)
    pb = prefix // 128
    idx = idx.reshape(-1, nb, idx.shape[-1])
    cnt = cnt.reshape(-1, nb)
    valid = np.arange(idx.shape[-1])[None, None, :] < cnt[:, :, None]
    exact = np.where(valid, sizes[np.clip(idx, 0, nb - 1)], 0).sum(-1)
    summ = np.where(np.arange(nb)[None, :] >= pb, (nb - pb) - (cnt - pb), 0)
    return int((sizes[None, :] * (exact + summ)).sum())


def effective_pairs_extra(idx, cnt, extra, ecnt, side_cnt, N, prefix):
    """Computed pairs of the extra-token path (all heads): exact pairs over the
    listed blocks' real tokens and the extra tokens, plus one summary column
    per unlisted video block that holds none of the row's extra tokens and one
    per side summary row, for every video query row."""
    sizes = block_sizes(N)
    nb = len(sizes)
    pb = prefix // 128
    idx = idx.reshape(-1, nb, idx.shape[-1])
    cnt = cnt.reshape(-1, nb)
    extra = extra.reshape(-1, nb, extra.shape[-1])
    ecnt = ecnt.reshape(-1, nb)
    side_cnt = side_cnt.reshape(-1, nb)
    valid = np.arange(idx.shape[-1])[None, None, :] < cnt[:, :, None]
    exact = np.where(valid, sizes[np.clip(idx, 0, nb - 1)], 0).sum(-1) + ecnt
    ev = np.arange(extra.shape[-1])[None, None, :] < ecnt[:, :, None]
    blk = np.where(ev, extra // 128, -1)
    starts = ev & np.concatenate([np.ones_like(blk[..., :1], dtype=bool),
                                  blk[..., 1:] != blk[..., :-1]], axis=-1)
    affected = starts.sum(-1)
    summ = np.where(np.arange(nb)[None, :] >= pb,
                    (nb - pb) - (cnt - pb) - affected + side_cnt, 0)
    return int((sizes[None, :] * (exact + summ)).sum())


def stage_bytes(B, H, N, nb, kcap):
    """Algorithmic HBM bytes of the pool + summarize passes (read Q, K, V once;
    write qpool, kpool fp32, k~, v~ bf16, bias, anchor)."""
    bh = B * H
    reads = 3 * bh * N * 128 * 2
    writes = bh * nb * 128 * (4 + 4 + 2 + 2) + bh * nb * 4 + bh * 128 * 4
    return reads + writes


# ------------------------------------------------------------------ ranks

def max_over_ranks(ms: float, device=None) -> float:
    """Elapsed device time of this rank -> the max over all ranks (identity
    without a process group).  The only collective of the benchmark: the
    ranks' attention calls are independent (no data-path exchange)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    """Sum of a per-rank quantity over all ranks (identity without a process
    group): the effective FLOPs of the ranks' head ranges."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_tflops(flops_per_call: float, calls_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank ran calls_per_rank independent calls
    of flops_per_call effective FLOPs; the job took max_ms (slowest rank)."""
    return world * flops_per_call * calls_per_rank / (max_ms / 1e3) / 1e12


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle

def oracle_pairs(N, out, pb, query_blocks=None):
    """Computed pairs of one oracle head (extra tokens included when the
    output holds them): exact pairs over the listed blocks' real tokens and
    the extra tokens, one summary column per unlisted video block that keeps
    at least one token out of the extra ones."""
    import oracle as orc
    extras = out.get("extras")
    if extras is None:
        return orc.effective_pairs(N, out["lists"], pb, query_blocks=query_blocks)
    bounds = orc.block_bounds(N)
    nb = len(bounds)
    total = 0
    for i, (a, b) in enumerate(bounds):
        if query_blocks is not None and i not in query_blocks:
            continue
        listed = set(int(j) for j in out["lists"][i])
        exact = sum(bounds[j][1] - bounds[j][0] for j in listed) + len(extras[i])
        summ = 0
        if i >= pb:
            taken = {}
            for u in extras[i]:
                taken[int(u) // 128] = taken.get(int(u) // 128, 0) + 1
            summ = sum(1 for j in range(pb, nb) if j not in listed and
                       taken.get(j, 0) < bounds[j][1] - bounds[j][0])
        total += (b - a) * (exact + summ)
    return total


def time_oracle(Qh, Kh, Vh, cfg, budget_s=20.0, max_heads=3, fp8=False, reblock=False,
                tau=None, extra_tokens=None):
    """The fp64 oracle as it stands, on whole heads, until ~budget_s of CPU work
    (the FP8 oracle for ``fp8``, the reblocking oracle for ``reblock``, the
    threshold oracle when ``tau`` is given, the extra-token oracle when
    ``extra_tokens`` is)."""
    import oracle as orc
    from oracle import bsa_oracle_extra as orcx
    from oracle import bsa_oracle_fp8 as orc8
    from oracle import bsa_oracle_reblock as orcr
    from oracle import bsa_oracle_threshold as orct
    head_fn = orc8.forward_head_fp8 if fp8 else (orcr.forward_head_reblock if reblock
                                                  else orc.forward_head)
    sel = cfg["top_k"]
    if tau is not None:
        head_fn, sel = orct.forward_head_threshold, tau
    if extra_tokens is not None:
        def head_fn(Q_, K_, V_, top_k_, prefix_, variant_):
            return orcx.forward_head_extra(Q_, K_, V_, top_k_, extra_tokens, prefix_, variant_)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    pairs = 0
    t0 = time.perf_counter()
    heads = 0
    for h in range(min(max_heads, len(Qh))):
        out = head_fn(Qh[h], Kh[h], Vh[h], sel, cfg["prefix"], cfg["variant"])
        pairs += oracle_pairs(len(Qh[h]), out, cfg["prefix"] // 128)
        heads += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    flops = 4 * 128 * pairs
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {cfg['H']} heads of the workload, whole "
                      f"{'FP8 ' if fp8 else ''}{'reblocked ' if reblock else ''}"
                      f"{'threshold ' if tau is not None else ''}"
                      f"{'extra-token ' if extra_tokens is not None else ''}path per head "
                      f"(numpy fp64, BLAS threads = {cores}); {dt:.1f} s, "
                      f"{dt / heads:.2f} s/head"}, dt / heads


def run_reference(args, cfg):
    """Reference arm: the fp64 CPU oracle timed on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from block_sparse_video_bsa_b200.inputs import make_tensor
    # one head of the workload per step (bounded sample), inputs built on the CPU
    B, H, N = cfg["B"], cfg["H"], cfg["N"]
    heads = [make_tensor(t, 1, 1, N, 128, cfg["kind"], seed=0, device="cpu")[0, 0]
             .double().numpy() for t in ("q", "k", "v")]
    import oracle as orc
    nb = -(-N // 128)
    pb = cfg["prefix"] // 128
    # bounded sample per step: the whole head's pool / summaries / selection
    # plus the attention of REF_QBLOCKS evenly spaced query blocks
    qblocks = set(np.linspace(0, nb - 1, min(REF_QBLOCKS, nb)).round().astype(int).tolist())
    times, pairs_l = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if args.extra_tokens is not None:
            from oracle import bsa_oracle_extra as orcx
            out = orcx.forward_head_extra(heads[0], heads[1], heads[2], cfg["top_k"],
                                          args.extra_tokens, cfg["prefix"], cfg["variant"],
                                          query_blocks=qblocks)
        elif args.tau is None:
            out = orc.forward_head(heads[0], heads[1], heads[2], cfg["top_k"], cfg["prefix"],
                                   cfg["variant"], query_blocks=qblocks)
        else:
            from oracle import bsa_oracle_threshold as orct
            out = orct.forward_head_threshold(heads[0], heads[1], heads[2], args.tau,
                                              cfg["prefix"], cfg["variant"],
                                              query_blocks=qblocks)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            pairs_l.append(oracle_pairs(N, out, pb, query_blocks=qblocks))
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    ms = 1e3 * sum(times) / len(times)
    value = 4 * 128 * sum(pairs_l) / sum(times) / 1e12
    sample = (f"per step: one head (of {H}) through pool, summaries and selection, and the "
              f"attention of {len(qblocks)} of its {nb} query blocks (evenly spaced); "
              "FLOPs counted for those rows only")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_block(cfg, sample=sample,
                               **({"selection": f"threshold tau={args.tau}"}
                                  if args.tau is not None else {}),
                               **({"extra_tokens": args.extra_tokens}
                                  if args.extra_tokens is not None else {})),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parallelism_label(args, world, total_bh, nbh, gather):
    """How the job's (b, h) slices are split over the ranks."""
    if args.shard == "heads":
        return (f"heads of one call split over {world} GPU(s): {total_bh} heads, {nbh} on rank 0, "
                f"no collective in the forward" + ("; O all-gathered over NCCL" if gather else ""))
    return (f"one video per GPU: B={world} x {total_bh // max(world, 1)} heads, each rank runs "
            f"its own video's heads, no data-path collective")


def data_label(cfg):
    """What the timed inputs are: the seeded generator kind and the workload shape."""
    kind = {"block_offset": "per-block-offset", "iid": "iid N(0,1)"}.get(cfg["kind"], cfg["kind"])
    return (f"synthetic (seeded {kind} bf16 Q/K/V, workload {cfg['name']}: B={cfg['B']}, "
            f"H={cfg['H']}, N={cfg['N']})")


def config_block(cfg, local_bh=None, **extra):
    """The workload's sizes; ``local_bh`` = (b, h) slices one rank runs."""
    bh = cfg["B"] * cfg["H"] if local_bh is None else local_bh
    d = {"workload": cfg["name"], "B": cfg["B"], "H": cfg["H"], "N": cfg["N"], "d": 128,
         "top_k": cfg["top_k"], "prefix": cfg["prefix"], "summary": cfg["variant"],
         "inputs": cfg["kind"], "l2": "inputs larger than L2 (Q+K+V = "
         f"{3 * bh * cfg['N'] * 256 / 1e9:.2f} GB per step and GPU)"}
    d.update(extra)
    return d


# ------------------------------------------------------------------ our arm

def main():
    args = parse_args()
    from block_sparse_video_bsa_b200.inputs import CONFIGS
    cfg = dict(CONFIGS[args.workload])
    cfg["name"] = args.workload
    if args.top_k is not None:
        cfg["top_k"] = args.top_k
    if args.heads is not None:
        cfg["H"] = args.heads
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist
    from block_sparse_video_bsa_b200 import bsa
    from block_sparse_video_bsa_b200.inputs import make_qkv_slices
    from block_sparse_video_bsa_b200.shard import gather_heads, head_range

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    # This rank's contiguous range of the job's (b, h) slices, run as one
    # sub-call with B = 1 and H = the range's length.
    N = cfg["N"]
    top_k, prefix, variant = cfg["top_k"], cfg["prefix"], cfg["variant"]
    B_job = cfg["B"] * (1 if args.shard == "heads" else world)
    total_bh = B_job * cfg["H"]
    bh0, nbh = head_range(total_bh, world, rank)
    if nbh == 0:
        raise SystemExit(f"rank {rank}: no heads to run ({total_bh} slices over {world} ranks)")
    Q, K, V = make_qkv_slices(B_job, cfg["H"], N, bh0, nbh, 128, cfg["kind"], seed=0, device=dev)
    B, H = 1, nbh
    gather = args.gather and world > 1
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    p = bsa.params(B, H, N, top_k, prefix, variant, dev_status=status)
    buf = bsa.stage_buffers(B, H, N, top_k, prefix, variant, device=dev)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)
    fp8 = args.precision == "fp8"
    rbl = args.reblock
    thr = args.tau is not None
    xtr = args.extra_tokens is not None
    if xtr:
        n_extra = args.extra_tokens
        buf.update(bsa.extra_buffers(B, H, N, top_k, n_extra, prefix, variant, device=dev))
    if thr:
        nb0 = bsa.bsa_num_blocks(p)
        buf["idx"] = torch.empty(B, H, nb0, bsa.bsa_threshold_capacity(p), dtype=torch.int32,
                                 device=dev)
        lists_ws = torch.empty(bsa.bsa_attend_lists_workspace_bytes(p), dtype=torch.uint8,
                               device=dev)
    if fp8:
        ops_buf, ops, _ = bsa.fp8_operands(p, dev)
    if rbl:
        perm = torch.empty(B, H, N, dtype=torch.int32, device=dev)
        rb_ws = torch.empty(max(256, bsa.bsa_reblock_workspace_bytes(p)), dtype=torch.uint8,
                            device=dev)
        Qa, Ka, Va, Oa = (torch.empty_like(Q) for _ in range(4))
    else:
        Qa, Ka, Va, Oa = Q, K, V, O
    names = (["reblock"] if rbl else []) + ["pool", "summarize", "select"] + \
        (["quantize"] if fp8 else []) + (["select_extra", "extra_summaries"] if xtr else []) + \
        ["attend"] + (["unpermute"] if rbl else []) + (["gather"] if gather else [])
    nev = len(names) + 1

    def step(ev=None):
        marks = iter(ev or [])

        def mark():
            if ev:
                next(marks).record(stream)
        mark()
        if rbl:   # the reblocked layout: pool and summarize gather Q, K, V through perm
            bsa.bsa_reblock(p, Q, K, perm, rb_ws, stream)
            mark()
            bsa.bsa_pool_permuted(p, Q, perm, Qa, buf["qpool"], buf["anchor"], stream)
        else:
            bsa.bsa_pool(p, Qa, buf["qpool"], buf["anchor"], stream)
        mark()
        if rbl:
            bsa.bsa_summarize_permuted(p, K, V, perm, Ka, Va, buf["anchor"], buf["kpool"],
                                       buf["ksum"], buf["vsum"], buf["bias"], stream)
        elif xtr:
            bsa.bsa_summarize_stats(p, K, V, buf["anchor"], buf["kpool"], buf["ksum"],
                                    buf["vsum"], buf["bias"], buf["kstat"], buf["vstat"],
                                    buf["lse_blk"], stream)
        else:
            bsa.bsa_summarize(p, Ka, Va, buf["anchor"], buf["kpool"], buf["ksum"], buf["vsum"],
                              buf["bias"], stream)
        mark()
        if thr:
            bsa.bsa_select_threshold(p, args.tau, buf["qpool"], buf["kpool"], buf["idx"],
                                     buf["cnt"], stream)
        else:
            bsa.bsa_select(p, buf["qpool"], buf["kpool"], buf["idx"], buf["cnt"], stream)
        mark()
        if xtr:
            bsa.bsa_select_extra(p, n_extra, buf["qpool"], K, buf["idx"], buf["cnt"],
                                 buf["extra"], buf["ecnt"], buf["cand"], stream)
            mark()
            bsa.bsa_extra_summaries(p, n_extra, K, V, buf["anchor"], buf["kpool"], buf["kstat"],
                                    buf["vstat"], buf["lse_blk"], buf["extra"], buf["ecnt"],
                                    buf["side_k"], buf["side_v"], buf["side_bias"],
                                    buf["side_blk"], buf["side_cnt"], stream)
            mark()
            bsa.bsa_attend_extra(p, n_extra, Q, K, V, buf["idx"], buf["cnt"], buf["extra"],
                                 buf["ecnt"], buf["ksum"], buf["vsum"], buf["bias"],
                                 buf["side_k"], buf["side_v"], buf["side_bias"],
                                 buf["side_cnt"], O, None, stream)
        elif fp8:
            bsa.bsa_quantize_fp8(p, Q, K, V, buf["ksum"], buf["vsum"], ops, stream)
            mark()
            bsa.bsa_attend_fp8(p, ops, buf["idx"], buf["cnt"], buf["bias"], O, None, stream)
        elif thr:
            bsa.bsa_attend_lists(p, Q, K, V, buf["idx"], buf["cnt"], buf["ksum"], buf["vsum"],
                                 buf["bias"], O, None, lists_ws, stream)
        else:
            bsa.bsa_attend(p, Qa, Ka, Va, buf["idx"], buf["cnt"], buf["ksum"], buf["vsum"],
                           buf["bias"], Oa, None, stream)
        mark()
        if rbl:
            bsa.bsa_unpermute(p, Oa, None, perm, O, None, stream)
            mark()
        if gather:   # every rank ends the step holding the whole O
            gather_heads(O, total_bh)
            mark()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {bsa.status_string(int(status.item()))}")
    if xtr:
        pairs = effective_pairs_extra(buf["idx"].cpu().numpy(), buf["cnt"].cpu().numpy(),
                                      buf["extra"].cpu().numpy(), buf["ecnt"].cpu().numpy(),
                                      buf["side_cnt"].cpu().numpy(), N, prefix)
    else:
        pairs = effective_pairs(buf["idx"].cpu().numpy(), buf["cnt"].cpu().numpy(), N, prefix)
    flops_step = 4 * 128 * pairs               # this rank's heads
    flops_job = sum_over_ranks(flops_step, dev)  # every rank's heads
    nb = bsa.bsa_num_blocks(p)
    mean_kept = None
    if thr:   # video blocks kept per video query block, over all heads
        c = buf["cnt"][:, :, prefix // 128:].double()
        mean_kept = float((c - prefix // 128).mean())

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)]
              for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)   # let the sampler start before the timed region
    for s in range(args.steps):
        step(events[s])
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    if world > 1:
        dist.barrier()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {bsa.status_string(int(status.item()))}")

    total_ms = sum(e[0].elapsed_time(e[-1]) for e in events)
    stage_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in events)
                for i in range(nev - 1)]
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = job_tflops(flops_job, args.steps, 1, total_ms)

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e and (fp8 or rbl or thr or xtr):
        # the option's public host-buffer call: copies in, its forward, O copied
        # back, pipelined over chunks of heads, all inside the timed region
        hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
        hO = torch.empty_like(hQ).pin_memory()
        if fp8:
            ws8 = torch.empty(bsa.bsa_forward_fp8_workspace_bytes(p), dtype=torch.uint8,
                              device=dev)
            fwd, fwd_name = bsa.bsa_forward_fp8_host, "bsa_forward_fp8_host"
        elif xtr:
            for k_ in ("kstat", "vstat", "extra", "side_k", "side_v", "side_bias", "side_blk",
                       "cand"):
                del buf[k_]
            torch.cuda.empty_cache()
            ws8 = torch.empty(bsa.bsa_forward_extra_workspace_bytes(p, n_extra),
                              dtype=torch.uint8, device=dev)

            def fwd(p_, *rest):
                bsa.bsa_forward_extra_host(p_, n_extra, *rest)
            fwd_name = "bsa_forward_extra_host"
        elif thr:
            ws8 = torch.empty(bsa.bsa_forward_threshold_workspace_bytes(p), dtype=torch.uint8,
                              device=dev)

            def fwd(p_, *rest):
                bsa.bsa_forward_threshold_host(p_, args.tau, *rest)
            fwd_name = "bsa_forward_threshold_host"
        else:
            del Qa, Ka, Va, Oa, rb_ws
            ws8 = torch.empty(bsa.bsa_forward_reblock_workspace_bytes(p), dtype=torch.uint8,
                              device=dev)
            fwd, fwd_name = bsa.bsa_forward_reblock_host, "bsa_forward_reblock_host"

        def e2e_call():
            fwd(p, hQ, hK, hV, hO, None, Q, K, V, O, None, ws8, stream)
        for _ in range(2):
            e2e_call()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_call()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": job_tflops(flops_job, args.e2e_steps, 1, e_ms),
               "unit": "TFLOP/s", "ms_per_call": e_ms / args.e2e_steps,
               "h2d_bytes_per_step": 3 * Q.numel() * Q.element_size(),
               "d2h_bytes_per_step": O.numel() * O.element_size(),
               "path": f"{fwd_name} (pinned host Q/K/V -> device -> host O, pipelined over "
                       "chunks of heads)"}
        del hQ, hK, hV, hO, ws8
    elif not args.no_e2e:
        hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
        hO = torch.empty_like(hQ).pin_memory()
        ws = bsa.workspace(p, dev)
        for _ in range(2):
            bsa.bsa_forward_host(p, hQ, hK, hV, hO, None, Q, K, V, O, None, ws, stream)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            bsa.bsa_forward_host(p, hQ, hK, hV, hO, None, Q, K, V, O, None, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": job_tflops(flops_job, args.e2e_steps, 1, e_ms),
               "unit": "TFLOP/s", "ms_per_call": e_ms / args.e2e_steps,
               "h2d_bytes_per_step": 3 * Q.numel() * Q.element_size(),
               "d2h_bytes_per_step": O.numel() * O.element_size(),
               "path": "bsa_forward_host (pinned host Q/K/V -> device -> host O)"}
        del hQ, hK, hV, hO

    peaks, peak_src = load_peaks()
    attend_ms = stage_ms[names.index("attend")]
    attend_tflops = flops_step / (attend_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"]) * (2.0 if fp8 else 1.0)
    pool_bytes = stage_bytes(B, H, N, nb, bsa.bsa_select_capacity(p))
    if xtr:   # summarize also writes the fp32 statistics of the side summaries
        pool_bytes += B * H * nb * (512 + 512 + 4)
    if rbl:   # pool and summarize also write the permuted Q, K, V
        pool_bytes += 3 * B * H * N * 256
    pool_gbs = pool_bytes / ((stage_ms[names.index("pool")] + stage_ms[names.index("summarize")])
                             / 1e3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        hh = list(range(min(3, H)))
        Qh = [Q[0, h].double().cpu().numpy() for h in hh]
        Kh = [K[0, h].double().cpu().numpy() for h in hh]
        Vh = [V[0, h].double().cpu().numpy() for h in hh]
        cpu, _ = time_oracle(Qh, Kh, Vh, cfg, fp8=fp8, reblock=rbl, tau=args.tau,
                             extra_tokens=args.extra_tokens)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None,
            "dtype": "e4m3" if fp8 else "bf16",
            "data": data_label(cfg),
            "config": config_block(cfg, local_bh=nbh,
                                   parallelism=parallelism_label(args, world, total_bh, nbh,
                                                                 gather),
                                   global_batch=B_job, heads_per_rank=nbh,
                                   **({"layout": "adaptive reblocking (q_reuse_k)"} if rbl
                                      else {}),
                                   **({"selection": f"threshold tau={args.tau}",
                                       "mean_kept_blocks": mean_kept} if thr else {}),
                                   **({"extra_tokens": args.extra_tokens} if xtr else {})),
            "ms_per_call": ms_per_step,
            "effective_tflop_per_call": flops_job / 1e12,
            "stages_ms": dict(zip(names, stage_ms)),
            "roofline": {"kernel": "attend_fp8_kernel" if fp8 else
                         ("attend_kernel (extra tokens)" if xtr else "attend_kernel"),
                         "bound": "tensor", "achieved": attend_tflops,
                         "peak": peak, "unit": "TFLOP/s", "frac": attend_tflops / peak,
                         "peak_source": f"{peak_src} bf16 burst"
                                        + (" x 2 (nominal e4m3/bf16 ratio)" if fp8 else ""),
                         "traffic": None if (xtr or thr or rbl) else
                         read_traffic(cfg, "attend_fp8" if fp8 else "attend"),
                         # the same kernel against the power-capped seconds-long
                         # cuBLAS figure (the timed region is ~0.5 s of back-to-back calls)
                         "frac_sustained": attend_tflops / (float(peaks.get(
                             "bf16_tflops_sustained", peaks["bf16_tflops"]))
                             * (2.0 if fp8 else 1.0))},
            "pool_summary": {"bound": "hbm", "achieved": pool_gbs,
                             "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                             "frac": pool_gbs / float(peaks["hbm_gbs"]),
                             "bytes_per_call": pool_bytes},
            "cpu_baseline": cpu,
            "e2e": e2e,
            # per step: pool_q, anchor, summarize, select, attend; fp8 adds five
            # quantisations and the value-scale reduction, the threshold path
            # the schedule, the extra-token path the token selection, its
            # finishing pass and the side summaries
            "gpu_launches": ((11 if fp8 else (6 if thr else
                                              (5 + (3 if args.extra_tokens else 0) if xtr else 5)))
                             + (reblock_launches(N, prefix) + 1 if rbl else 0)) * args.steps,
            "clocks": clock_info,
            "context": {"pages_rtx_pro_6000_sparse_ms": 30.7 if cfg["N"] == 37_740 else None},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def read_traffic(cfg, kernel="attend"):
    """DRAM bytes per launch of the attention kernel (source csrc/<kernel>.cu)
    from the committed ncu summary profiles/<kernel>_traffic.txt, if it was
    taken on the current kernel source and this workload; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for ln in open(path):
        if "=" in ln and not ln.startswith("#"):
            k, v = ln.split("=", 1)
            kv[k.strip()] = v.strip()
    src = os.path.join(ROOT, "block_sparse_video_bsa_b200", "csrc", f"{kernel}.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if kv.get(f"{kernel}_cu_sha256_16") != h or kv.get("workload") != cfg["name"]:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


if __name__ == "__main__":
    main()
