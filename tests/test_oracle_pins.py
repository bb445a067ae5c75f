"""Pins of the fp64 oracle against facts fixed outside it.

Nothing here re-types the oracle's formulas: each test checks a closed form,
a textbook special case (dense softmax attention, through torch's SDPA), an
inequality the pages state (Jensen: exp(E[x]) <= E[exp(x)], Spark-H3 page,
compressed-branch figure caption) or a brute-force enumeration.  A plausible
slip anywhere in the oracle (a dropped ln n_j, a wrong sign on the anchor
term, 128 instead of the ragged block's count, a transposed score, ties to
the wrong index, prefix rows counted in the anchor) fails at least one test.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle as orc


def _rng(seed):
    return np.random.default_rng(seed)


def _dense(Q, K, V):
    """Textbook softmax attention via torch's own SDPA on CPU in fp64."""
    q = torch.from_numpy(np.asarray(Q, np.float64))[None, None]
    k = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    v = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()


def _dense_lse(Q, K):
    d = Q.shape[1]
    logits = torch.from_numpy(Q @ K.T / math.sqrt(d))
    return torch.logsumexp(logits, dim=1).numpy()


# ---------------------------------------------------------------- partition

def test_block_bounds_ragged_tail():
    assert orc.block_bounds(300) == [(0, 128), (128, 256), (256, 300)]
    assert orc.block_bounds(128) == [(0, 128)]
    assert orc.block_bounds(1) == [(0, 1)]
    assert orc.block_bounds(37_740)[-1] == (294 * 128, 37_740)
    assert len(orc.block_bounds(133_644)) == 1045


def test_pooled_means_closed_form_and_ragged_count():
    # block j: rows j + c*(+1,-1,+1,-1,...) -> mean exactly j; ragged block of 3
    # rows with values 1, 2, 6 -> mean 3 (dividing by 128 would give 9/128).
    d = 4
    rows = []
    for j in range(2):
        for t in range(128):
            rows.append(np.full(d, j + (1.0 if t % 2 == 0 else -1.0) * 0.75))
    for v in (1.0, 2.0, 6.0):
        rows.append(np.full(d, v))
    X = np.array(rows)
    m = orc.pooled_means(X)
    np.testing.assert_allclose(m, [[0.0] * d, [1.0] * d, [3.0] * d], atol=1e-15)


def test_anchor_is_mean_of_video_rows_only():
    d = 3
    Q = np.zeros((384, d))
    Q[:128] = 100.0                       # text-like prefix rows
    Q[128:256] = [1.0, 2.0, 3.0]
    Q[256:] = [3.0, 2.0, 1.0]
    np.testing.assert_allclose(orc.video_query_anchor(Q, 128), [2.0, 2.0, 2.0])
    np.testing.assert_allclose(orc.video_query_anchor(Q, 0), [(100 + 4) / 3] * 3)


def test_block_scores_orientation_and_scale():
    # qhat_i = e_i, khat_j = (j+1) e_j  ->  S[i, j] = (j+1)/sqrt(d) if i == j else 0,
    # and a transposed score S[j, i] would put the factor on the wrong axis.
    d = 16
    qpool = np.eye(3, d)
    kpool = np.eye(3, d) * np.array([[1.0], [2.0], [3.0]])
    kpool[0, 1] = 5.0                     # khat_0 . qhat_1 = 5
    S = orc.block_scores(qpool, kpool)
    assert S[1, 0] == pytest.approx(5 / 4)
    assert S[0, 1] == 0.0
    np.testing.assert_allclose(np.diag(S), [0.25, 0.5, 0.75])


# ---------------------------------------------------------------- selection

def _brute_select(S_row, k, pb, nb):
    """Max-sum k-subset of the video blocks; ties -> lexicographically smallest."""
    cand = range(pb, nb)
    best, best_t = None, None
    for sub in itertools.combinations(cand, min(k, nb - pb)):
        tot = sum(S_row[j] for j in sub)
        if best is None or tot > best + 1e-12 or (abs(tot - best) <= 1e-12 and sub < best_t):
            best, best_t = tot, sub
    return list(range(pb)) + list(best_t)


@pytest.mark.parametrize("seed", range(6))
def test_selection_matches_subset_enumeration_with_ties(seed):
    r = _rng(seed)
    nb = 7
    S = r.integers(-2, 3, size=(nb, nb)).astype(np.float64)  # many exact ties
    for pb in (0, 2):
        for k in (1, 2, 3, 5, 9):
            lists = orc.select_blocks(S, k, pb)
            for i in range(nb):
                if i < pb:
                    assert list(lists[i]) == list(range(nb))
                else:
                    assert list(lists[i]) == _brute_select(S[i], k, pb, nb)


def test_all_equal_scores_pick_lowest_indices():
    nb, pb = 9, 2
    S = np.full((nb, nb), 0.125)
    lists = orc.select_blocks(S, 3, pb)
    for i in range(pb, nb):
        assert list(lists[i]) == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------- summaries

@pytest.mark.parametrize("N", [1, 127, 128, 300, 515])
@pytest.mark.parametrize("variant", ["anchor", "mean"])
def test_topk_all_blocks_is_dense_attention(N, variant):
    r = _rng(N)
    d = 128
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    nb = -(-N // 128)
    out = orc.forward_head(Q, K, V, top_k=nb + 3, variant=variant)
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], _dense_lse(Q, K), rtol=0, atol=1e-11)


def _constant_key_blocks(N, d, r):
    K = np.zeros((N, d))
    for a, b in orc.block_bounds(N):
        K[a:b] = r.standard_normal(d)
    return K


@pytest.mark.parametrize("variant", ["anchor", "mean"])
@pytest.mark.parametrize("N,prefix,top_k", [(515, 0, 1), (515, 128, 2), (1000, 0, 3),
                                            (640, 256, 1)])
def test_identical_keys_make_summary_rows_exact(variant, N, prefix, top_k):
    # Equal keys in a block: weights are uniform, k~ = k, bias = ln n_j, so
    # exp(z) v~ = n_j exp(q.k/sqrt d) mean(v) = sum_t exp(q.k_t/sqrt d) v_t.
    # The output must then equal dense attention for every top_k, including
    # the ragged last block (ln of its real count, not ln 128).
    r = _rng(N + prefix + top_k)
    d = 128
    Q = r.standard_normal((N, d))
    K = _constant_key_blocks(N, d, r)
    V = r.standard_normal((N, d))
    out = orc.forward_head(Q, K, V, top_k=top_k, prefix=prefix, variant=variant)
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)


@pytest.mark.parametrize("N,prefix", [(515, 0), (700, 128)])
def test_anchor_variant_exact_when_queries_equal_anchor(N, prefix):
    # All queries equal q-bar: the biased summary logit at the anchor is the
    # block's exact log-mass and v~ its exact softmax-weighted value, so the
    # output equals dense attention for every top_k (the figure caption's
    # "exponential matches the expected exponential").
    r = _rng(N)
    d = 128
    q = r.standard_normal(d)
    Q = np.tile(q, (N, 1))
    K = r.standard_normal((N, d))
    V = r.standard_normal((N, d))
    dense = _dense(Q, K, V)
    for top_k in (1, 2):
        a = orc.forward_head(Q, K, V, top_k=top_k, prefix=prefix, variant="anchor")["O"]
        np.testing.assert_allclose(a, dense, rtol=0, atol=1e-11)
        # The mean-pooled variant is strictly off here (Jensen), which shows
        # the test can tell the two variants apart.
        m = orc.forward_head(Q, K, V, top_k=top_k, prefix=prefix, variant="mean")["O"]
        assert np.abs(m - dense).max() > 1e-3


def test_mean_variant_underestimates_mass_jensen():
    # Spark-H3 page: mean pooling substitutes exp(E[x]) for E[exp(x)].
    r = _rng(7)
    d, N = 128, 512
    K = r.standard_normal((N, d))
    V = r.standard_normal((N, d))
    ksum, _, bias = orc.block_summaries(K, V, np.zeros(d), "mean")
    for _ in range(20):
        q = r.standard_normal(d)
        for j, (a, b) in enumerate(orc.block_bounds(N)):
            z = q @ ksum[j] / math.sqrt(d) + bias[j]
            exact = math.log(np.exp(K[a:b] @ q / math.sqrt(d)).sum())
            assert z < exact


def test_anchor_summary_logit_equals_block_lse_at_anchor():
    r = _rng(11)
    d, N = 128, 300
    K = r.standard_normal((N, d))
    V = r.standard_normal((N, d))
    qbar = 0.3 * r.standard_normal(d)
    ksum, vsum, bias = orc.block_summaries(K, V, qbar, "anchor")
    for j, (a, b) in enumerate(orc.block_bounds(N)):
        x = K[a:b] @ qbar / math.sqrt(d)
        z = qbar @ ksum[j] / math.sqrt(d) + bias[j]
        assert z == pytest.approx(math.log(np.exp(x).sum()), abs=1e-12)
        w = np.exp(x) / np.exp(x).sum()
        np.testing.assert_allclose(vsum[j], (w[:, None] * V[a:b]).sum(0), atol=1e-13)


# ---------------------------------------------------------------- whole path

def _closed_form_row(q, E_tokens, skipped, K, V, qbar, bounds, d):
    """Anchor-variant output of one query, written from the rearranged closed
    form  exp(z_j(q)) = exp((q - qbar).k~_j/sqrt d) * sum_t exp(qbar.k_t/sqrt d),
    v~_j = sum_t exp(qbar.k_t/sqrt d) v_t / sum_t exp(qbar.k_t/sqrt d),
    with plain Python scalar loops."""
    s = 1.0 / math.sqrt(d)
    num = np.zeros(V.shape[1])
    den = 0.0
    for u in E_tokens:
        e = math.exp(float(q @ K[u]) * s)
        num += e * V[u]
        den += e
    for j in skipped:
        a, b = bounds[j]
        ws = [math.exp(float(qbar @ K[t]) * s) for t in range(a, b)]
        mass = sum(ws)
        ktil = sum(w * K[t] for w, t in zip(ws, range(a, b))) / mass
        vtil = sum(w * V[t] for w, t in zip(ws, range(a, b))) / mass
        e = math.exp(float((q - qbar) @ ktil) * s) * mass
        num += e * vtil
        den += e
    return num / den


@pytest.mark.parametrize("N,prefix,top_k", [(9, 0, 1), (11, 4, 1), (16, 0, 2)])
def test_whole_path_matches_closed_form_brute_force(N, prefix, top_k):
    # Block size 4 and d = 3 make every step small enough for scalar loops.
    blk, d = 4, 3
    r = _rng(100 + N)
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = orc.forward_head(Q, K, V, top_k=top_k, prefix=prefix, variant="anchor", block=blk)
    bounds = orc.block_bounds(N, blk)
    nb, pb = len(bounds), prefix // blk
    qbar = Q[prefix:].sum(0) / (N - prefix)
    qhat = [Q[a:b].sum(0) / (b - a) for a, b in bounds]
    khat = [K[a:b].sum(0) / (b - a) for a, b in bounds]
    for i, (a, b) in enumerate(bounds):
        if i < pb:
            E = list(range(nb))
        else:
            sc = {j: float(qhat[i] @ khat[j]) / math.sqrt(d) for j in range(pb, nb)}
            ranked = sorted(sc, key=lambda j: (-sc[j], j))[:top_k]
            E = list(range(pb)) + sorted(ranked)
        assert list(out["lists"][i]) == E
        skipped = [] if i < pb else [j for j in range(pb, nb) if j not in E]
        toks = [t for j in E for t in range(*bounds[j])]
        for t in range(a, b):
            want = _closed_form_row(Q[t], toks, skipped, K, V, qbar, bounds, d)
            np.testing.assert_allclose(out["O"][t], want, rtol=0, atol=1e-12)


def test_dense_prefix_rows_are_dense():
    r = _rng(5)
    N, d, P = 640, 128, 256
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = orc.forward_head(Q, K, V, top_k=1, prefix=P)
    np.testing.assert_allclose(out["O"][:P], _dense(Q[:P], K, V), atol=1e-12)
    for i in range(2, 5):
        assert list(out["lists"][i][:2]) == [0, 1]
        assert len(out["lists"][i]) == 3


def test_effective_pairs_counts_real_tokens_and_summaries():
    # N = 300 (blocks of 128, 128, 44), prefix 0, top_k 1:
    # each row sees one exact block plus 2 summary columns.
    r = _rng(3)
    N, d = 300, 8
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = orc.forward_head(Q, K, V, top_k=1)
    lists = out["lists"]
    sizes = [128, 128, 44]
    want = sum((b - a) * (sizes[lists[i][0]] + 2) for i, (a, b) in enumerate(orc.block_bounds(N)))
    assert orc.effective_pairs(N, lists, 0) == want


def test_argument_checks():
    Q = np.zeros((256, 8))
    with pytest.raises(ValueError):
        orc.forward_head(Q, Q, Q, top_k=0)
    with pytest.raises(ValueError):
        orc.forward_head(Q, Q, Q, top_k=1, prefix=100)
    with pytest.raises(ValueError):
        orc.forward_head(Q, Q, Q, top_k=1, prefix=256)
    with pytest.raises(ValueError):
        orc.block_summaries(Q, Q, np.zeros(8), "median")
