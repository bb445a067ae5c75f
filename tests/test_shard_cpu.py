"""The multi-GPU partition of one call without a GPU: the (b, h) slices are
split into contiguous per-rank ranges, every rank regenerates and runs only
its own slices, and the all-gather puts them back in order.  Ranks run as
gloo processes on the CPU with the oracle standing in for the device call, so
what is pinned is the partition and the reassembly: the gathered result must
equal the one-rank result bit for bit."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as orc
from block_sparse_video_bsa_b200.inputs import make_qkv, make_qkv_slices
from block_sparse_video_bsa_b200.shard import gather_heads, head_range, local_slices


@pytest.mark.parametrize("total", [0, 1, 5, 7, 56, 112, 57])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_covers_every_slice_once_and_balances(total, world):
    seen = []
    counts = []
    for r in range(world):
        s, c = head_range(total, world, r)
        assert c >= 0
        seen.extend(range(s, s + c))
        counts.append(c)
    assert seen == list(range(total))                 # in order, disjoint, complete
    assert max(counts) - min(counts) <= 1
    with pytest.raises(ValueError):
        head_range(total, world, world)


def test_slices_equal_the_whole_tensors():
    B, H, N = 2, 3, 300
    whole = make_qkv(B, H, N, 128, "block_offset", seed=4)
    for world in (2, 4):
        for r in range(world):
            s, c = head_range(B * H, world, r)
            part = make_qkv_slices(B, H, N, s, c, 128, "block_offset", seed=4)
            for w, p in zip(whole, part):
                assert torch.equal(local_slices(w, world, r), p)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASE = dict(B=1, H=5, N=300, top_k=1, prefix=128, variant="anchor", kind="block_offset", seed=2)


def _rank_main(rank, world, port, case, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    B, H, N = case["B"], case["H"], case["N"]
    start, count = head_range(B * H, world, rank)
    Q, K, V = make_qkv_slices(B, H, N, start, count, 128, case["kind"], case["seed"])
    O = torch.zeros(1, count, N, 128, dtype=torch.float64)
    for i in range(count):
        # the oracle stands in for bsa_forward on this rank's sub-call
        O[0, i] = torch.from_numpy(orc.forward_head(
            Q[0, i].double().numpy(), K[0, i].double().numpy(), V[0, i].double().numpy(),
            case["top_k"], case["prefix"], case["variant"])["O"])
    full = gather_heads(O, B * H)
    if rank == 0:
        out_q.put(full.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,B,H", [(2, 1, 5), (3, 2, 3)])
def test_sharded_call_reassembles_the_one_rank_result(world, B, H):
    case = dict(CASE, B=B, H=H)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    Q, K, V = make_qkv(B, H, case["N"], 128, case["kind"], case["seed"])
    want = np.stack([orc.forward_head(Q[b, h].double().numpy(), K[b, h].double().numpy(),
                                      V[b, h].double().numpy(), case["top_k"], case["prefix"],
                                      case["variant"])["O"]
                     for b in range(B) for h in range(H)])
    assert got.shape == want.shape
    assert np.array_equal(got, want)
