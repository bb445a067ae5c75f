"""Invariances of the method, checked on the fp64 oracles at sizes that span
several blocks, a ragged tail and a dense prefix.

Each follows from the definitions alone, not from the oracle's code:
* the attention weights of a row (exact and summary columns together) sum to
  one, and so do the anchor weights inside a summary, so adding a vector c to
  every value row adds c to every output row, and scaling V scales O;
* adding a vector c to every key moves every logit of query q, exact or
  summary, by the same q.c/sqrt(d): the block scores of a row move by a
  constant (same selection, same z-scores), the anchor weights do not move,
  k~ moves by c and the bias does not; so O is unchanged and lse moves by
  q.c/sqrt(d);
* permuting the tokens inside each block (keys with their values) changes no
  pooled mean, summary or block sum, and permuting the queries inside a block
  permutes the output rows the same way; the same holds for the FP8 path,
  whose quantisation groups are whole blocks;
* the reblocked layout is built from order-free statistics of the content,
  so the reblocked attention is equivariant to ANY order of the video tokens
  (the fixed layout is not).
A slip that breaks one of these (a bias computed from the wrong k~, a summary
value not normalised, a pooled mean over the wrong rows, a scale missing from
the bias) fails here even where the closed-form pins happen not to reach.
"""

import math

import numpy as np
import pytest

import oracle as orc
from oracle import bsa_oracle_threshold as th

CASES = [(700, 0, 2, "anchor"), (900, 256, 1, "anchor"), (1000, 128, 3, "mean")]


def _qkv(N, seed):
    r = np.random.default_rng(seed)
    offs = lambda: np.repeat(r.standard_normal((-(-N // 128), 128)), 128, axis=0)[:N]
    return tuple(offs() + 0.5 * r.standard_normal((N, 128)) for _ in range(3))


def _run(kind, Q, K, V, top_k, prefix, variant):
    if kind == "topk":
        return orc.forward_head(Q, K, V, top_k, prefix, variant)
    return th.forward_head_threshold(Q, K, V, 0.8, prefix, variant)


@pytest.mark.parametrize("kind", ["topk", "threshold"])
@pytest.mark.parametrize("N,prefix,top_k,variant", CASES)
def test_value_shift_and_scale(kind, N, prefix, top_k, variant):
    Q, K, V = _qkv(N, N)
    base = _run(kind, Q, K, V, top_k, prefix, variant)
    c = np.random.default_rng(1).standard_normal(128)
    shifted = _run(kind, Q, K, V + c, top_k, prefix, variant)
    np.testing.assert_allclose(shifted["O"], base["O"] + c, rtol=0, atol=1e-11)
    np.testing.assert_allclose(shifted["lse"], base["lse"], rtol=0, atol=1e-12)
    scaled = _run(kind, Q, K, V * 2.5, top_k, prefix, variant)
    np.testing.assert_allclose(scaled["O"], base["O"] * 2.5, rtol=0, atol=1e-11)


@pytest.mark.parametrize("kind", ["topk", "threshold"])
@pytest.mark.parametrize("N,prefix,top_k,variant", CASES)
def test_key_shift_moves_logits_by_a_row_constant(kind, N, prefix, top_k, variant):
    Q, K, V = _qkv(N, N + 1)
    base = _run(kind, Q, K, V, top_k, prefix, variant)
    c = 0.7 * np.random.default_rng(2).standard_normal(128)
    moved = _run(kind, Q, K + c, V, top_k, prefix, variant)
    assert all(list(a) == list(b) for a, b in zip(moved["lists"], base["lists"]))
    np.testing.assert_allclose(moved["O"], base["O"], rtol=0, atol=1e-10)
    np.testing.assert_allclose(moved["lse"], base["lse"] + Q @ c / math.sqrt(128),
                               rtol=0, atol=1e-10)
    np.testing.assert_allclose(moved["bias"], base["bias"], rtol=0, atol=1e-10)


@pytest.mark.parametrize("kind", ["topk", "threshold"])
@pytest.mark.parametrize("N,prefix,top_k,variant", CASES)
def test_permutation_inside_blocks(kind, N, prefix, top_k, variant):
    Q, K, V = _qkv(N, N + 2)
    base = _run(kind, Q, K, V, top_k, prefix, variant)
    r = np.random.default_rng(3)
    perm_k = np.concatenate([a + r.permutation(b - a) for a, b in orc.block_bounds(N)])
    perm_q = np.concatenate([a + r.permutation(b - a) for a, b in orc.block_bounds(N)])
    out = _run(kind, Q[perm_q], K[perm_k], V[perm_k], top_k, prefix, variant)
    assert all(list(a) == list(b) for a, b in zip(out["lists"], base["lists"]))
    np.testing.assert_allclose(out["O"], base["O"][perm_q], rtol=0, atol=1e-11)
    np.testing.assert_allclose(out["lse"], base["lse"][perm_q], rtol=0, atol=1e-11)
    for key in ("ksum", "vsum", "bias", "kpool", "qpool"):
        np.testing.assert_allclose(out[key], base[key], rtol=0, atol=1e-11)


@pytest.mark.parametrize("N,prefix,top_k", [(700, 0, 2), (900, 256, 1)])
def test_reblocked_attention_is_equivariant_to_any_token_order(N, prefix, top_k):
    # The reblocked layout is built from order-free statistics of the whitened
    # queries (sums, projections, a sort whose ties need exactly equal
    # projections), so shuffling the video tokens (queries with their keys and
    # values) shuffles O and lse the same way: the layout follows the content,
    # not the positions.  The dense prefix stays in place.
    from oracle import bsa_oracle_reblock as rb
    Q, K, V = _qkv(N, N + 3)
    base = rb.forward_head_reblock(Q, K, V, top_k, prefix, "anchor")
    r = np.random.default_rng(4)
    pi = np.concatenate([np.arange(prefix), prefix + r.permutation(N - prefix)])
    out = rb.forward_head_reblock(Q[pi], K[pi], V[pi], top_k, prefix, "anchor")
    np.testing.assert_allclose(out["O"], base["O"][pi], rtol=0, atol=1e-10)
    np.testing.assert_allclose(out["lse"], base["lse"][pi], rtol=0, atol=1e-10)
    # the fixed layout is not equivariant: the same shuffle changes its output
    fixed = orc.forward_head(Q, K, V, top_k, prefix, "anchor")["O"]
    fixed_pi = orc.forward_head(Q[pi], K[pi], V[pi], top_k, prefix, "anchor")["O"]
    assert np.abs(fixed_pi - fixed[pi]).max() > 1e-3


@pytest.mark.parametrize("N,prefix,top_k", [(700, 0, 2), (1000, 128, 3)])
def test_fp8_path_permutation_inside_blocks(N, prefix, top_k):
    # e4m3 groups are whole blocks (one amax and scale each), so permuting the
    # tokens inside blocks changes no code and no scale: the FP8 output is
    # permuted exactly like the bf16 one.
    from oracle import bsa_oracle_fp8 as o8
    Q, K, V = _qkv(N, N + 4)
    base = o8.forward_head_fp8(Q, K, V, top_k, prefix, "anchor")
    r = np.random.default_rng(5)
    perm_k = np.concatenate([a + r.permutation(b - a) for a, b in orc.block_bounds(N)])
    perm_q = np.concatenate([a + r.permutation(b - a) for a, b in orc.block_bounds(N)])
    out = o8.forward_head_fp8(Q[perm_q], K[perm_k], V[perm_k], top_k, prefix, "anchor")
    np.testing.assert_allclose(out["O"], base["O"][perm_q], rtol=0, atol=1e-11)
    np.testing.assert_allclose(out["lse"], base["lse"][perm_q], rtol=0, atol=1e-11)
