"""Pins of the threshold-selection oracle against facts fixed outside it.

The pages give one set of numbers for a threshold rule: the share of key
blocks kept at three settings of tau (tests/golden/threshold_kept_fractions.txt,
with its citation).  The reading that the threshold is a z-score is checked
against those shares on score rows of arbitrary offset and spread (so a
dropped mean, a variance in place of the deviation or a divided tau fails).
The decision itself is checked against exact rational arithmetic on every
small integer row (so a sample deviation in place of the population one, a
strict comparison or a wrong floor fails), the lists against the fixed-count
oracle at the same count, and the whole path against textbook dense
attention and the anchor closed form.
"""

import math
import statistics
from fractions import Fraction
from itertools import product
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle as orc
from oracle import bsa_oracle_threshold as th

from test_oracle_pins import _closed_form_row, _dense

GOLDEN = Path(__file__).parent / "golden" / "threshold_kept_fractions.txt"


def _page_shares():
    rows = [l.split() for l in GOLDEN.read_text().splitlines() if l and not l.startswith("#")]
    return [(float(t), float(p) / 100.0) for t, p in rows]


def _normal_tail(z):
    return 0.5 * math.erfc(z / math.sqrt(2.0))


def _kept_fraction(S, tau, pb=0):
    lists = th.select_blocks_threshold(S, tau, pb)
    nb = S.shape[0]
    return sum(len(l) - pb for l in lists[pb:]) / ((nb - pb) * (nb - pb))


# ------------------------------------------------------------ the pages' shares

def test_golden_file_holds_three_settings():
    assert [t for t, _ in _page_shares()] == [1.0, 1.5, 2.0]


def test_kept_shares_match_the_pages_on_gaussian_rows():
    # Rows of normal scores, each with its own offset and spread: the share
    # kept is the normal tail at tau whatever the offset and spread, and lies
    # within the page's rounding of its printed share.
    r = np.random.default_rng(0)
    nb = 1500
    S = r.standard_normal((nb, nb)) * r.uniform(0.05, 4.0, (nb, 1)) + r.uniform(-5, 5, (nb, 1))
    for tau, page in _page_shares():
        frac = _kept_fraction(S, tau)
        assert abs(frac - _normal_tail(tau)) < 2.5e-3, (tau, frac)
        assert abs(frac - page) <= 0.01, (tau, frac, page)


def test_synthetic_workload_sits_in_the_pages_regime():
    # The block-offset inputs at the 768p-5s length (one head): pooled scores
    # over the key blocks are close to normal, so the shares come out near
    # the page's.
    from block_sparse_video_bsa_b200.inputs import make_qkv
    Q, K, _ = make_qkv(1, 1, 37_740, 128, "block_offset", seed=0)
    qp = orc.pooled_means(Q[0, 0].double().numpy())
    kp = orc.pooled_means(K[0, 0].double().numpy())
    S = orc.block_scores(qp, kp)
    for tau, page in _page_shares():
        assert abs(_kept_fraction(S, tau) - page) <= 0.015, tau


# --------------------------------------------- exact arithmetic on small rows

def _exact_keep(row, tau):
    """Kept positions from rational arithmetic: x - mu >= tau * sigma decided
    by signs and squares, sigma the population deviation; the floor keeps the
    first maximum.  Also reports whether some position sits exactly on the
    threshold with x != mu."""
    n = len(row)
    mu = Fraction(sum(row), n)
    var = sum((Fraction(x) - mu) ** 2 for x in row) / n
    keep, on_edge = [], False
    for x in row:
        dx = x - mu
        if tau >= 0:
            ok = dx >= 0 and dx * dx >= tau * tau * var
        else:
            ok = dx >= 0 or dx * dx <= tau * tau * var
        on_edge |= dx != 0 and dx * dx == tau * tau * var
        keep.append(ok)
    if not any(keep):
        keep[row.index(max(row))] = True
    return [j for j, k in enumerate(keep) if k], on_edge


@pytest.mark.parametrize("n,values", [(4, range(5)), (3, range(6)), (5, range(4)), (2, range(3))])
def test_selection_matches_exact_rational_arithmetic(n, values):
    # n = 4 (and 2): mu, sigma and tau * sigma are exact in binary whenever a
    # score sits exactly on the threshold, so every row is compared.  n = 3, 5:
    # rows with a score exactly on the threshold are left out (fp64 may round
    # either way there); the rest are compared.
    taus = [Fraction(-1), Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2)]
    rows = [list(r) for r in product(values, repeat=n)]
    compared = 0
    for tau in taus:
        for start in range(0, len(rows), n):
            batch = rows[start:start + n]
            batch += [batch[-1]] * (n - len(batch))
            lists = th.select_blocks_threshold(np.array(batch, dtype=np.float64), float(tau), 0)
            for i, row in enumerate(batch):
                want, on_edge = _exact_keep(row, tau)
                if on_edge and n not in (2, 4):
                    continue
                assert list(lists[i]) == want, (row, tau)
                compared += 1
    assert compared > 0.9 * len(taus) * len(rows)


def test_floor_and_no_contrast():
    # [0, 1]: the top block has z = 1 exactly (kept at tau = 1 by ">="); at
    # tau = 2 nothing qualifies and the floor keeps it.  [2, 2]: no contrast,
    # every block is kept even at tau = 2.
    S = np.array([[0.0, 1.0], [2.0, 2.0]])
    for tau in (0.5, 1.0, 2.0):
        lists = th.select_blocks_threshold(S, tau, 0)
        assert [list(l) for l in lists] == [[1], [0, 1]], tau
    # Equal top scores below the threshold: the floor keeps the lower index.
    S = np.array([[1.0, 3.0, 3.0], [0.0, 5.0, 5.0], [7.0, 2.0, 2.0]])
    assert [list(l) for l in th.select_blocks_threshold(S, 2.0, 0)] == [[1], [1], [0]]
    assert [list(l) for l in th.select_blocks_threshold(S, 0.5, 0)] == [[1, 2], [1, 2], [0]]
    # Equal scores whose rounded mean is off by one ulp still keep every block.
    for x, n in ((0.1, 3), (0.7, 3), (0.2, 6), (1.0, 4)):
        row = np.full(n, x)
        assert (row.mean() != x) == (x != 1.0)
        lists = th.select_blocks_threshold(np.tile(row, (n, 1)), 1.5, 0)
        assert all(list(l) == list(range(n)) for l in lists), (x, n)


def test_invariants_on_random_rows():
    r = np.random.default_rng(1)
    nb = 200
    S = r.standard_normal((nb, nb)) * r.uniform(0.1, 3.0, (nb, 1))
    base = {tau: th.select_blocks_threshold(S, tau, 0) for tau in (-0.5, 0.0, 1.0, 1.5, 2.5)}
    moved = th.select_blocks_threshold(4.0 * S + 8.0, 1.0, 0)
    for i in range(nb):
        # a positive scale and a shift of the row leave the kept set unchanged
        assert list(moved[i]) == list(base[1.0][i])
        # a larger tau keeps a subset
        for lo, hi in ((-0.5, 0.0), (0.0, 1.0), (1.0, 1.5), (1.5, 2.5)):
            assert set(base[hi][i]) <= set(base[lo][i])
        # the kept blocks are the highest-scoring ones
        kept = np.zeros(nb, bool)
        kept[base[1.0][i]] = True
        if not kept.all():
            assert S[i, kept].min() >= S[i, ~kept].max()
    # tau = 0 keeps what lies at or above the row mean
    for i in range(nb):
        assert list(base[0.0][i]) == list(np.flatnonzero(S[i] >= S[i].mean()))


def test_prefix_blocks_are_listed_and_left_out_of_the_statistic():
    # Huge prefix columns change nothing among the video blocks: the statistic
    # runs over j >= pb only; prefix blocks are listed in front; prefix query
    # rows are dense.
    r = np.random.default_rng(2)
    nb, pb = 40, 3
    S = r.standard_normal((nb, nb))
    S[:, :pb] = 1e6
    lists = th.select_blocks_threshold(S, 1.0, pb)
    video_only = th.select_blocks_threshold(S[pb:, pb:], 1.0, 0)
    for i in range(nb):
        if i < pb:
            assert list(lists[i]) == list(range(nb))
        else:
            assert list(lists[i][:pb]) == list(range(pb))
            assert list(lists[i][pb:]) == list(video_only[i - pb] + pb)


@pytest.mark.parametrize("tau", [0.3, 1.0, 2.0])
def test_lists_equal_fixed_count_lists_at_the_same_count(tau):
    r = np.random.default_rng(3)
    nb, pb = 60, 2
    S = r.standard_normal((nb, nb))
    lists = th.select_blocks_threshold(S, tau, pb)
    for i in range(pb, nb):
        count = len(lists[i]) - pb
        assert list(lists[i]) == list(orc.select_blocks(S, count, pb)[i])


@pytest.mark.parametrize("N,prefix,variant", [(700, 0, "anchor"), (900, 256, "mean"),
                                              (515, 128, "anchor")])
def test_very_low_tau_is_dense_attention(N, prefix, variant):
    r = np.random.default_rng(N)
    Q, K, V = (r.standard_normal((N, 128)) for _ in range(3))
    out = th.forward_head_threshold(Q, K, V, -1e30, prefix, variant)
    nb = -(-N // 128)
    assert all(list(l) == list(range(nb)) for l in out["lists"])
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)


@pytest.mark.parametrize("tau", [0.5, 1.0, 2.0])
def test_anchor_variant_exact_when_queries_equal_anchor(tau):
    # Every query equals q-bar, so each summary row carries its block's exact
    # mass and value: the output is dense attention whatever the lists hold.
    r = np.random.default_rng(9)
    N, d = 1100, 128
    q = r.standard_normal(d)
    Q = np.tile(q, (N, 1))
    K = r.standard_normal((N, d)) + r.standard_normal((N // 128 + 1, d)).repeat(128, 0)[:N]
    V = r.standard_normal((N, d))
    out = th.forward_head_threshold(Q, K, V, tau, 0, "anchor")
    assert any(len(l) < len(out["lists"]) for l in out["lists"])
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)


@pytest.mark.parametrize("N,prefix,tau", [(17, 0, 1.0), (21, 4, 0.5), (24, 0, 2.0)])
def test_whole_path_matches_brute_force_with_stdlib_statistics(N, prefix, tau):
    # Block size 4, d = 3; the threshold from Python's statistics module
    # (exact rational mean and population variance), the lists by plain
    # comparison, the output by the scalar closed form.
    blk, d = 4, 3
    r = np.random.default_rng(200 + N)
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = th.forward_head_threshold(Q, K, V, tau, prefix, "anchor", block=blk)
    bounds = orc.block_bounds(N, blk)
    nb, pb = len(bounds), prefix // blk
    qbar = Q[prefix:].sum(0) / (N - prefix)
    qhat = [Q[a:b].sum(0) / (b - a) for a, b in bounds]
    khat = [K[a:b].sum(0) / (b - a) for a, b in bounds]
    for i, (a, b) in enumerate(bounds):
        if i < pb:
            E = list(range(nb))
        else:
            sc = [float(qhat[i] @ khat[j]) / math.sqrt(d) for j in range(pb, nb)]
            mu, sd = statistics.fmean(sc), statistics.pstdev(sc)
            chosen = [pb + j for j, x in enumerate(sc) if x - mu >= tau * sd]
            if not chosen:
                chosen = [pb + sc.index(max(sc))]
            E = list(range(pb)) + chosen
        assert list(out["lists"][i]) == E
        skipped = [] if i < pb else [j for j in range(pb, nb) if j not in E]
        toks = [t for j in E for t in range(*bounds[j])]
        for t in range(a, b):
            want = _closed_form_row(Q[t], toks, skipped, K, V, qbar, bounds, d)
            np.testing.assert_allclose(out["O"][t], want, rtol=0, atol=1e-12)


def test_argument_checks():
    Q = np.zeros((256, 8))
    for bad in (float("nan"), float("inf")):
        with pytest.raises(ValueError):
            th.forward_head_threshold(Q, Q, Q, bad)
    with pytest.raises(ValueError):
        th.forward_head_threshold(Q, Q, Q, 1.0, prefix=100)
