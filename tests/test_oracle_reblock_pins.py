"""Pins of the reblocking oracle against things other than itself: brute-force
cosines of score vectors, closed-form principal axes, hand-built clusters,
and dense attention (which any token permutation must leave unchanged)."""

import numpy as np
import pytest
import torch

from oracle import bsa_oracle_reblock as rb


def test_whitened_dot_is_the_cosine_of_score_vectors(monkeypatch):
    # R-a: u_s . u_t = cos(K q_s, K q_t), K the video keys (brute force).
    # Exact without the ridge; the ridge (1e-6 of the mean eigenvalue of M)
    # moves it by a few 1e-6 for these anisotropic keys.
    rng = np.random.default_rng(0)
    d, n_k, n_q = 8, 300, 40
    K = rng.standard_normal((n_k, d)) @ rng.standard_normal((d, d))   # anisotropic keys
    Q = rng.standard_normal((n_q, d))
    S = Q @ K.T                                                        # score patterns
    cos = (S @ S.T) / np.outer(np.linalg.norm(S, axis=1), np.linalg.norm(S, axis=1))
    U = rb.whiten(Q, rb.key_second_moment(K))
    np.testing.assert_allclose(U @ U.T, cos, atol=2e-5)
    monkeypatch.setattr(rb, "RIDGE", 0.0)
    U0 = rb.whiten(Q, rb.key_second_moment(K))
    np.testing.assert_allclose(U0 @ U0.T, cos, atol=1e-12)


def test_prefix_keys_and_queries_are_left_out():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((300, 6))
    np.testing.assert_allclose(rb.key_second_moment(K, 128), K[128:].T @ K[128:])
    U = rb.whiten(rng.standard_normal((300, 6)), rb.key_second_moment(K, 128), 128)
    assert U.shape == (172, 6)


def test_split_direction_closed_form():
    # Points +-a e1 +- b e2 (centre 0, scatter diag(n a^2, n b^2, 0, ...)):
    # 8 power iterations from the all-ones vector give a vector proportional
    # to ((n a^2)^8, (n b^2)^8, 0, ...).
    a, b, d = 2.0, 1.5, 5
    pts = [(sa * a, sb * b) for sa in (1, -1) for sb in (1, -1)]
    U = np.zeros((4, d))
    U[:, :2] = pts
    v = rb.split_direction(U)
    n = 4
    ref = np.zeros(d)
    ref[0], ref[1] = (n * a * a) ** 8, (n * b * b) ** 8
    np.testing.assert_allclose(v, ref / np.linalg.norm(ref), rtol=1e-12, atol=1e-15)


def test_split_sizes_ties_and_order():
    rng = np.random.default_rng(2)
    for n in (129, 256, 300, 640, 1000):
        idx = np.arange(n) * 3 + 7
        left, right = rb.split_node(rng.standard_normal((n, 4)), idx)
        b = -(-n // 128)
        assert len(left) == (b // 2) * 128 and len(right) == n - len(left)
        assert np.all(np.diff(left) > 0) and np.all(np.diff(right) > 0)
        assert set(left) | set(right) == set(idx)
    # identical rows: every projection ties -> the lowest indices go left
    left, right = rb.split_node(np.ones((300, 4)), np.arange(300))
    np.testing.assert_array_equal(left, np.arange(128))


def test_split_follows_the_principal_axis():
    # Two clusters of 128 along e1 (+ small noise): the left child is the one
    # with the smaller coordinate (the start vector makes v . e1 > 0).
    rng = np.random.default_rng(3)
    U = 0.01 * rng.standard_normal((256, 6))
    U[:128, 0] += 1.0
    U[128:, 0] -= 1.0
    order = rng.permutation(256)
    left, right = rb.split_node(U[order], np.arange(256))
    np.testing.assert_array_equal(np.sort(order[left]), np.arange(128, 256))


@pytest.mark.parametrize("n", [1, 127, 128, 129, 300, 1000, 4100])
def test_partition_leaves(n):
    rng = np.random.default_rng(n)
    leaves = rb.partition(rng.standard_normal((n, 5)))
    sizes = [len(x) for x in leaves]
    assert all(s == 128 for s in sizes[:-1]) and 1 <= sizes[-1] <= 128
    assert len(leaves) == -(-n // 128)
    allidx = np.concatenate(leaves)
    np.testing.assert_array_equal(np.sort(allidx), np.arange(n))
    assert all(np.all(np.diff(x) > 0) for x in leaves)


def test_scrambled_clusters_are_recovered():
    # Four clusters of 128 queries on an arc (angles 0, 0.3, 0.6, 0.9 rad in
    # the e1-e2 plane), scrambled over the sequence; keys with K^T K = c I so
    # the metric is the plain cosine.  Every leaf must be one whole cluster.
    rng = np.random.default_rng(4)
    d = 8
    K = np.tile(np.eye(d), (64, 1)) * 3.0                  # 512 keys, K^T K = 576 I
    labels = np.repeat(np.arange(4), 128)
    ang = labels * 0.3
    Q = np.zeros((512, d))
    Q[:, 0], Q[:, 1] = np.cos(ang), np.sin(ang)
    Q += 0.01 * rng.standard_normal(Q.shape)
    shuffle = rng.permutation(512)
    Q, labels = Q[shuffle], labels[shuffle]
    perm = rb.reblock_permutation(Q, K)
    for leaf in perm.reshape(4, 128):
        assert len(set(labels[leaf])) == 1
    assert sorted(labels[perm.reshape(4, 128)[:, 0]]) == [0, 1, 2, 3]


def test_prefix_rows_keep_their_places():
    rng = np.random.default_rng(5)
    Q, K = rng.standard_normal((700, 6)), rng.standard_normal((700, 6))
    perm = rb.reblock_permutation(Q, K, prefix=256)
    np.testing.assert_array_equal(perm[:256], np.arange(256))
    np.testing.assert_array_equal(np.sort(perm), np.arange(700))


def test_reblocked_dense_attention_is_unchanged():
    # With every block listed the method is dense attention, which no token
    # permutation changes: O and lse come back in the original order.
    rng = np.random.default_rng(6)
    N, d = 500, 16
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    out = rb.forward_head_reblock(Q, K, V, top_k=10)
    assert not np.array_equal(out["perm"], np.arange(N))
    t = lambda x: torch.from_numpy(x)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V))[0, 0].numpy()
    np.testing.assert_allclose(out["O"], ref, atol=1e-12)
    lse = torch.logsumexp(t(Q @ K.T / np.sqrt(d))[0, 0], dim=1).numpy()
    np.testing.assert_allclose(out["lse"], lse, atol=1e-12)
