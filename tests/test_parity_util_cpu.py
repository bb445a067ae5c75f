"""The parity comparison itself, without a GPU: a query block whose list
differs from the oracle's by a permitted near-tie swap is still compared on
every row, against the oracle's attention over that list.

The "device" buffers here are built from the oracle on the CPU: pooled
blocks are arranged so that two key blocks tie exactly at the k-th place, the
fabricated lists take the other block of the pair on some rows, and the
fabricated output is either the oracle's attention over those lists (a
consistent result, which must pass) or over the oracle's own lists (an output
that does not belong to the lists it claims, which must fail)."""

import numpy as np
import pytest
import torch

import oracle as orc

from parity_util import check_head

N, D, TOP_K = 1024, 128, 3
# block means c_j * e: the top three are blocks 0, 1 and then 3 or 5 (tied)
C = [5.0, 4.0, 1.0, 3.0, 0.0, 3.0, 2.0, -1.0]
SWAP_ROWS = {2, 6}


def _inputs():
    rng = np.random.default_rng(7)
    e = np.zeros(D)
    e[0] = 1.0
    Q = rng.normal(size=(N, D))
    K = rng.normal(size=(N, D))
    V = rng.normal(size=(N, D))
    for j in range(N // 128):
        s = slice(128 * j, 128 * j + 128)
        Q[s] += -Q[s].mean(axis=0) + 2.0 * e            # every query block points along e
        K[s] += -K[s].mean(axis=0) + C[j] * e
    # block 5 reflects block 3's tokens about their common mean: same pooled
    # key (an exact score tie), different tokens, and values far apart
    m3 = K[384:512].mean(axis=0)
    K[640:768] = 2.0 * m3 - K[384:512]
    V[640:768] = V[384:512] + 5.0
    return Q, K, V


def _device_buffers(Q, K, V, consistent):
    ref = orc.forward_head(Q, K, V, TOP_K, 0, "anchor")
    lists = [np.array(l) for l in ref["lists"]]
    assert [list(lists[i]) for i in SWAP_ROWS] == [[0, 1, 3]] * 2
    S = ref["scores"]
    assert all(abs(S[i, 3] - S[i, 5]) < 1e-12 for i in range(len(lists)))
    for i in SWAP_ROWS:
        lists[i] = np.array([0, 1, 5])
    O, lse = orc.attend(Q, K, V, lists if consistent else ref["lists"], ref["ksum"],
                        ref["vsum"], ref["bias"], 0)
    idx = np.stack(lists).astype(np.int32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    buf = {k: t(ref[k]) for k in ("qpool", "kpool", "ksum", "vsum", "bias")}
    buf["anchor"] = torch.from_numpy(ref["anchor"])[None, None]
    buf["idx"] = t(idx)
    buf["cnt"] = t(np.full(len(lists), TOP_K, dtype=np.int32))
    buf["O"], buf["lse"] = t(O), t(lse)
    return buf


def test_swapped_rows_are_checked_against_the_oracle_on_the_device_lists():
    Q, K, V = _inputs()
    buf = _device_buffers(Q, K, V, consistent=True)
    tq = lambda a: torch.from_numpy(a)[None, None]
    _, _, swaps = check_head(buf, tq(Q), tq(K), tq(V), 0, 0, TOP_K, 0, "anchor")
    assert swaps == SWAP_ROWS


def test_an_output_that_does_not_follow_the_swapped_list_fails():
    Q, K, V = _inputs()
    buf = _device_buffers(Q, K, V, consistent=False)
    tq = lambda a: torch.from_numpy(a)[None, None]
    with pytest.raises(AssertionError):
        check_head(buf, tq(Q), tq(K), tq(V), 0, 0, TOP_K, 0, "anchor")
