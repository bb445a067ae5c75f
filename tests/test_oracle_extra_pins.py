"""Pins of the extra-token oracle against facts fixed outside it.

* No extra tokens: the path is the base path, bit for bit.
* Enough extra tokens to cover every unlisted video token: every token is
  read exactly, so the output is textbook dense attention (torch SDPA) --
  which fails if an extra token were also left inside its block's summary.
* Every query at the anchor: each summary row, also one over a block's
  remaining tokens, carries those tokens' exact mass and value, so the output
  is dense attention for ANY number of extra tokens (every token once).
* The token choice against brute-force ranking at a tiny size, and the whole
  path against a scalar-loop closed form there.
"""

import math

import numpy as np
import pytest

import oracle as orc
from oracle import bsa_oracle_extra as ex

from test_oracle_pins import _dense, _dense_lse


def _qkv(N, seed, d=128):
    r = np.random.default_rng(seed)
    offs = lambda: np.repeat(r.standard_normal((-(-N // 128), d)), 128, axis=0)[:N]
    return tuple(offs() + 0.5 * r.standard_normal((N, d)) for _ in range(3))


@pytest.mark.parametrize("N,prefix,top_k,variant", [(700, 0, 2, "anchor"), (900, 256, 1, "mean")])
def test_no_extra_tokens_is_the_base_path(N, prefix, top_k, variant):
    Q, K, V = _qkv(N, N)
    base = orc.forward_head(Q, K, V, top_k, prefix, variant)
    out = ex.forward_head_extra(Q, K, V, top_k, 0, prefix, variant)
    assert all(len(e) == 0 for e in out["extras"])
    np.testing.assert_array_equal(out["O"], base["O"])
    np.testing.assert_array_equal(out["lse"], base["lse"])


@pytest.mark.parametrize("N,prefix,variant", [(700, 0, "anchor"), (900, 256, "anchor"),
                                              (515, 128, "mean")])
def test_extra_tokens_covering_everything_is_dense_attention(N, prefix, variant):
    Q, K, V = _qkv(N, N + 1)
    out = ex.forward_head_extra(Q, K, V, 1, N, prefix, variant)
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)
    np.testing.assert_allclose(out["lse"], _dense_lse(Q, K), rtol=0, atol=1e-11)


@pytest.mark.parametrize("n_extra", [1, 37, 256, 600])
def test_queries_at_the_anchor_give_dense_attention(n_extra):
    # Summary rows over a block's remaining tokens are exact at q = qbar, so
    # every token is counted exactly once whatever the extra tokens are.
    r = np.random.default_rng(9)
    N, d = 1100, 128
    q = r.standard_normal(d)
    Q = np.tile(q, (N, 1))
    K = r.standard_normal((N, d)) + np.repeat(r.standard_normal((N // 128 + 1, d)), 128, 0)[:N]
    V = r.standard_normal((N, d))
    out = ex.forward_head_extra(Q, K, V, 2, n_extra, 0, "anchor")
    partial = sum(0 < len(set(e.tolist()) & set(range(a, b))) < b - a
                  for e in out["extras"] for a, b in orc.block_bounds(N))
    assert partial > 0                       # some summaries really are over remaining tokens
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)
    np.testing.assert_allclose(out["lse"], _dense_lse(Q, K), rtol=0, atol=1e-11)


@pytest.mark.parametrize("variant", ["anchor", "mean"])
@pytest.mark.parametrize("n_extra", [5, 200])
def test_identical_keys_per_block_give_dense_attention(variant, n_extra):
    # Inside each block all keys are equal, so the summary of any subset of a
    # block (n' tokens) is k~ = k, bias = ln n', v~ = their mean: exactly the
    # subset's mass and value for every query.  Both variants must then give
    # dense attention whatever the extra tokens take out of a block.
    r = np.random.default_rng(12)
    N, d, prefix = 1000, 128, 128
    Q = r.standard_normal((N, d))
    K = np.repeat(r.standard_normal((-(-N // 128), d)), 128, axis=0)[:N]
    V = r.standard_normal((N, d))
    out = ex.forward_head_extra(Q, K, V, 2, n_extra, prefix, variant)
    np.testing.assert_allclose(out["O"], _dense(Q, K, V), rtol=0, atol=1e-11)
    np.testing.assert_allclose(out["lse"], _dense_lse(Q, K), rtol=0, atol=1e-11)


@pytest.mark.parametrize("N,prefix,top_k,n_extra", [(17, 0, 1, 3), (21, 4, 1, 5), (24, 0, 2, 4)])
def test_whole_path_matches_scalar_brute_force(N, prefix, top_k, n_extra):
    # Block size 4, d = 3: the extra tokens by ranking every candidate with a
    # plain sort, the output by summing exp-weights token by token, where a
    # block with extra tokens contributes its remaining tokens through the
    # anchor closed form exp((q - qbar).k~'/sqrt d) * sum exp(qbar.k_t/sqrt d).
    blk, d = 4, 3
    r = np.random.default_rng(300 + N)
    Q, K, V = (r.standard_normal((N, d)) for _ in range(3))
    out = ex.forward_head_extra(Q, K, V, top_k, n_extra, prefix, "anchor", block=blk)
    bounds = orc.block_bounds(N, blk)
    nb, pb = len(bounds), prefix // blk
    s = 1.0 / math.sqrt(d)
    qbar = Q[prefix:].sum(0) / (N - prefix)
    qhat = [Q[a:b].sum(0) / (b - a) for a, b in bounds]
    for i, (a, b) in enumerate(bounds):
        E = [int(j) for j in out["lists"][i]]
        if i < pb:
            assert len(out["extras"][i]) == 0
            continue
        cand = [t for j in range(pb, nb) if j not in E for t in range(*bounds[j])]
        ranked = sorted(cand, key=lambda t: (-float(qhat[i] @ K[t]) * s, t))[:n_extra]
        assert list(out["extras"][i]) == sorted(ranked)
        X = set(ranked)
        for t in range(a, b):
            num, den = np.zeros(d), 0.0
            for u in [u for j in E for u in range(*bounds[j])] + sorted(X):
                e = math.exp(float(Q[t] @ K[u]) * s)
                num += e * V[u]
                den += e
            for j in range(pb, nb):
                if j in E:
                    continue
                rest = [u for u in range(*bounds[j]) if u not in X]
                if not rest:
                    continue
                ws = [math.exp(float(qbar @ K[u]) * s) for u in rest]
                mass = sum(ws)
                kt = sum(w * K[u] for w, u in zip(ws, rest)) / mass
                vt = sum(w * V[u] for w, u in zip(ws, rest)) / mass
                e = math.exp(float((Q[t] - qbar) @ kt) * s) * mass
                num += e * vt
                den += e
            np.testing.assert_allclose(out["O"][t], num / den, rtol=0, atol=1e-12)


def test_argument_checks():
    Q = np.zeros((256, 8))
    with pytest.raises(ValueError):
        ex.forward_head_extra(Q, Q, Q, 1, -1)
    with pytest.raises(ValueError):
        ex.forward_head_extra(Q, Q, Q, 0, 4)
    with pytest.raises(ValueError):
        ex.forward_head_extra(Q, Q, Q, 1, 4, prefix=100)
