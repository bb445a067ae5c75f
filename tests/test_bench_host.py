"""Host-side logic of bench.py without a GPU: the effective-FLOP accounting,
the cross-rank timing reduction over two gloo ranks (the N > 1 path), and the
reference (oracle) arm's JSON line."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle as orc  # noqa: E402


def test_effective_pairs_match_the_oracle_count():
    r = np.random.default_rng(0)
    N, d, P = 1500, 16, 256
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = orc.forward_head(Q, K, V, top_k=3, prefix=P)
    nb = len(out["lists"])
    kcap = nb
    idx = np.full((1, nb, kcap), -1, dtype=np.int64)
    cnt = np.zeros((1, nb), dtype=np.int64)
    for i, L in enumerate(out["lists"]):
        idx[0, i, :len(L)] = L
        cnt[0, i] = len(L)
    assert bench.effective_pairs(idx, cnt, N, P) == orc.effective_pairs(N, out["lists"], P // 128)


def test_job_tflops_is_whole_job_throughput():
    assert bench.job_tflops(9.11e12, 50, 1, 500.0) == pytest.approx(9.11 * 50 / 0.5)
    assert bench.job_tflops(9.11e12, 50, 4, 500.0) == pytest.approx(4 * 9.11 * 50 / 0.5)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [120.0, 250.0][rank]             # rank 1 is the slow one
    m = bench.max_over_ranks(local_ms)
    # the ranks' head ranges carry different effective FLOPs; the job's is the sum
    f = bench.sum_over_ranks([4.0e12, 3.0e12][rank])
    out_q.put((rank, m, bench.job_tflops(9.11e12, 10, world, m), f))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v, f in res:
        assert m == 250.0
        assert v == pytest.approx(2 * 9.11 * 10 / 0.25)
        assert f == 7.0e12


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_prints_its_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_iid", "--steps", "1", "--warmup", "0"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["metric"] == bench.METRIC


def test_threshold_options():
    # --tau runs the bf16 path without reblocking; the reference arm times the
    # threshold oracle on the same workload and names the selection.
    for bad in (["--tau", "1.0", "--reblock"], ["--tau", "1.0", "--precision", "fp8"]):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *bad],
                             capture_output=True, text=True, timeout=120, cwd=ROOT)
        assert out.returncode != 0 and "--tau" in out.stderr
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_iid", "--tau", "1.0", "--steps", "1", "--warmup", "0"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["config"]["selection"] == "threshold tau=1.0" and line["value"] > 0


def test_shard_options():
    # --gather only makes sense when one call's heads are split over the ranks
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gather"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "--gather" in out.stderr


def test_parallelism_labels_name_the_split():
    class A:
        shard = "heads"
    assert "7 on rank 0" in bench.parallelism_label(A, 8, 56, 7, False)
    assert "all-gathered" in bench.parallelism_label(A, 8, 56, 7, True)
    A.shard = None
    assert "B=8 x 56 heads" in bench.parallelism_label(A, 8, 448, 56, False)


def test_effective_pairs_with_extra_tokens_match_the_oracle_count():
    # the device arrays (lists, extra tokens, side-row counts) give the same
    # computed-pair count as the oracle's head with its extra tokens
    from oracle import bsa_oracle_extra as ox
    r = np.random.default_rng(1)
    N, d, P, n_extra = 1500, 16, 256, 100
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = ox.forward_head_extra(Q, K, V, 3, n_extra, P, query_blocks=set())
    nb = len(out["lists"])
    idx = np.full((1, nb, nb), -1, dtype=np.int64)
    cnt = np.zeros((1, nb), dtype=np.int64)
    extra = np.full((1, nb, n_extra), -1, dtype=np.int64)
    ecnt = np.zeros((1, nb), dtype=np.int64)
    side = np.zeros((1, nb), dtype=np.int64)
    bounds = orc.block_bounds(N)
    for i, L in enumerate(out["lists"]):
        idx[0, i, :len(L)] = L
        cnt[0, i] = len(L)
        e = out["extras"][i]
        extra[0, i, :len(e)] = e
        ecnt[0, i] = len(e)
        blocks = set(int(u) // 128 for u in e)
        side[0, i] = sum(1 for j in blocks
                         if sum(1 for u in e if int(u) // 128 == j) < bounds[j][1] - bounds[j][0])
    assert ecnt[0, P // 128:].min() == n_extra
    assert bench.effective_pairs_extra(idx, cnt, extra, ecnt, side, N, P) == \
        bench.oracle_pairs(N, out, P // 128)
    # no extra tokens: the top-k count
    assert bench.effective_pairs_extra(idx, cnt, extra, ecnt * 0, side * 0, N, P) == \
        bench.effective_pairs(idx, cnt, N, P)


def test_extra_token_options():
    for bad in (["--extra-tokens", "256", "--tau", "1.0"], ["--extra-tokens", "600"],
                ["--extra-tokens", "256", "--precision", "fp8"]):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *bad],
                             capture_output=True, text=True, timeout=120, cwd=ROOT)
        assert out.returncode != 0 and "--extra-tokens" in out.stderr
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_iid", "--extra-tokens", "128", "--steps", "1", "--warmup", "0"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["config"]["extra_tokens"] == 128 and line["value"] > 0
