"""The extra-token parity comparison itself, without a GPU: device buffers
fabricated from the oracle (in the layouts the C ABI writes) pass every check,
and planted faults in them (a token from a listed block, a dropped side row, a
wrong side bias, an output that ignores an extra token) are caught."""

import numpy as np
import pytest
import torch

import oracle as orc
from oracle import bsa_oracle_extra as ox

from parity_util import check_head_extra

N, TOP_K, N_EXTRA, PREFIX = 1500, 2, 100, 256


def _inputs(seed=4):
    g = torch.Generator().manual_seed(seed)
    mk = lambda: (torch.randn(N // 128 + 1, 128, generator=g).repeat_interleave(128, 0)[:N] +
                  0.5 * torch.randn(N, 128, generator=g)).to(torch.bfloat16).double().numpy()
    return mk(), mk(), mk()


def _buffers(Q, K, V, variant="anchor"):
    """What the C ABI writes for one head, computed by the oracle."""
    out = ox.forward_head_extra(Q, K, V, TOP_K, N_EXTRA, PREFIX, variant)
    nb = len(out["lists"])
    pb = PREFIX // 128
    bounds = orc.block_bounds(N)
    kcap = nb
    idx = np.full((nb, kcap), -1, np.int32)
    cnt = np.zeros(nb, np.int32)
    extra = np.full((nb, N_EXTRA), -1, np.int32)
    ecnt = np.zeros(nb, np.int32)
    scap = 128
    sk = np.zeros((nb, scap, 128))
    sv = np.zeros((nb, scap, 128))
    sb = np.full((nb, scap), -np.inf)
    sj = np.full((nb, scap), -1, np.int32)
    sc = np.zeros(nb, np.int32)
    for i, L in enumerate(out["lists"]):
        idx[i, :len(L)] = L
        cnt[i] = len(L)
        e = out["extras"][i]
        extra[i, :len(e)] = e
        ecnt[i] = len(e)
        if i < pb:
            continue
        ex = set(int(u) for u in e)
        a = 0
        for j in range(pb, nb):
            if j in set(int(x) for x in L):
                continue
            toks = np.arange(*bounds[j])
            rest = np.array([t for t in toks if t not in ex], dtype=np.int64)
            if 0 < len(rest) < len(toks):
                sk[i, a], sv[i, a], sb[i, a] = ox.summary_of_tokens(K, V, rest, out["anchor"],
                                                                    variant)
                sj[i, a] = j
                a += 1
        sc[i] = a
    if variant == "anchor":
        lse_blk = out["bias"] + out["ksum"] @ out["anchor"] / np.sqrt(128)
    else:
        lse_blk = np.log([b - a for a, b in bounds])
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    buf = dict(qpool=t(out["qpool"]), kpool=t(out["kpool"]), ksum=t(out["ksum"]),
               vsum=t(out["vsum"]), bias=t(out["bias"]), idx=t(idx), cnt=t(cnt),
               kstat=t(out["ksum"]), vstat=t(out["vsum"]), lse_blk=t(lse_blk), extra=t(extra),
               ecnt=t(ecnt), side_k=t(sk), side_v=t(sv), side_bias=t(sb), side_blk=t(sj),
               side_cnt=t(sc), O=t(out["O"]), lse=t(out["lse"]))
    buf["anchor"] = torch.from_numpy(out["anchor"])[None, None]
    return buf, out


def _check(buf, Q, K, V, variant="anchor"):
    tq = lambda a: torch.from_numpy(a)[None, None]
    return check_head_extra(buf, tq(Q), tq(K), tq(V), 0, 0, TOP_K, N_EXTRA, PREFIX, variant)


@pytest.mark.parametrize("variant", ["anchor", "mean"])
def test_oracle_buffers_pass(variant):
    Q, K, V = _inputs()
    buf, out = _buffers(Q, K, V, variant)
    assert int(buf["side_cnt"].sum()) > 0
    _check(buf, Q, K, V, variant)


def test_a_token_of_a_listed_block_is_caught():
    Q, K, V = _inputs()
    buf, out = _buffers(Q, K, V)
    i = 5
    j = int(buf["idx"][0, 0, i, 2])                   # a listed video block
    buf["extra"][0, 0, i, 0] = j * 128
    buf["extra"][0, 0, i] = torch.sort(buf["extra"][0, 0, i]).values
    with pytest.raises(AssertionError):
        _check(buf, Q, K, V)


def test_a_dropped_side_row_is_caught():
    Q, K, V = _inputs()
    buf, out = _buffers(Q, K, V)
    i = int(np.argmax(buf["side_cnt"][0, 0].numpy()))
    buf["side_cnt"][0, 0, i] -= 1
    with pytest.raises(AssertionError):
        _check(buf, Q, K, V)


def test_a_wrong_side_bias_is_caught():
    Q, K, V = _inputs()
    buf, out = _buffers(Q, K, V)
    i = int(np.argmax(buf["side_cnt"][0, 0].numpy()))
    buf["side_bias"][0, 0, i, 0] += 0.01
    with pytest.raises(AssertionError):
        _check(buf, Q, K, V)


def test_an_output_without_the_extra_tokens_is_caught():
    Q, K, V = _inputs()
    buf, out = _buffers(Q, K, V)
    plain = orc.forward_head(Q, K, V, TOP_K, PREFIX)
    buf["O"] = torch.from_numpy(plain["O"])[None, None]
    with pytest.raises(AssertionError):
        _check(buf, Q, K, V)
