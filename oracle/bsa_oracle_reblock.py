"""Adaptive reblocking of the query/key layout (Spark-Reblock): the oracle.

TEST INFRASTRUCTURE ONLY, under the same rules as ``bsa_oracle.py``: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import it.  It shares no code with the CUDA path.

Where it comes from: "Spark-H3: Block Sparse Attention Speeds Up MiniMax-H3 in
ComfyUI", section "What Spark-Attn changes", the Spark-Reblock bullet: the
fixed spatio-temporal tiles are replaced by an adaptive partition; two queries
are similar when their attention-score patterns over the keys are similar,
measured by a Mahalanobis cosine distance induced by the opposite side's
second moment; a hierarchical partitioner splits groups until every leaf holds
the target block size, in O(N log N) time.  Section "Workflows": the shipped
workflows fix ``reblock_layout=q_reuse_k``.

The pages give no formulas.  READINGS of this project:

* R-a (metric).  The score pattern of query q over the video keys is K q, so
  the cosine of two patterns is q^T M q' / sqrt(q^T M q * q'^T M q') with
  M = sum_{t >= P} k_t k_t^T, the keys' second moment.  With L L^T = M + dI
  (Cholesky; d = 1e-6 * trace(M) / 128, a ridge that keeps the factor defined
  when the keys span fewer than 128 directions) the whitened, normalised
  coordinates u = L^T q / |L^T q| turn that cosine into u . u'.
* R-b (hierarchical partitioner).  A group of n tokens holding b = ceil(n/128)
  blocks with b >= 2 is bisected along its principal axis: centre c = mean of
  u, direction v = POWER_ITERS power iterations of the centred scatter matrix
  C = sum (u - c)(u - c)^T from (1, ..., 1) / sqrt(128), projections p = u . v;
  the left child takes the floor(b/2) * 128 tokens of smallest p (ties to the
  lower original index), the right child the rest.  A group with b = 1 is a
  leaf.  Each level is linear in N and there are ceil(log2(N/128)) levels.
* R-c (layout).  Leaves in left-to-right order; inside a leaf, ascending
  original index.  Only the last leaf can be ragged.
* R-d (q_reuse_k).  Keys and values take the queries' permutation (one layout
  per head); the dense prefix rows [0, P) keep their places.
* R-e.  The attention (pool, summaries, selection, exact and compressed
  branch) runs on the permuted sequence; O and lse are put back in the
  original token order.

Pinned by tests/test_oracle_reblock_pins.py.
"""

from __future__ import annotations

import numpy as np

from .bsa_oracle import BLOCK, forward_head

POWER_ITERS = 8
RIDGE = 1e-6


def key_second_moment(K, prefix: int = 0) -> np.ndarray:
    """M = sum over the video keys (rows >= prefix) of k k^T (R-a)."""
    Kv = np.asarray(K, dtype=np.float64)[prefix:]
    return Kv.T @ Kv


def whiten(Q, M, prefix: int = 0) -> np.ndarray:
    """u_t = L^T q_t / |L^T q_t| for the video queries, L L^T = M + ridge (R-a).

    A query with L^T q = 0 gets u = 0.
    """
    d = M.shape[0]
    L = np.linalg.cholesky(M + RIDGE * np.trace(M) / d * np.eye(d))
    Y = np.asarray(Q, dtype=np.float64)[prefix:] @ L          # rows are (L^T q_t)^T
    norm = np.linalg.norm(Y, axis=1, keepdims=True)
    return np.where(norm > 0, Y / np.where(norm > 0, norm, 1.0), 0.0)


def split_direction(U) -> np.ndarray:
    """POWER_ITERS power iterations of the centred scatter matrix (R-b)."""
    U = np.asarray(U, dtype=np.float64)
    c = U.mean(axis=0)
    C = (U - c).T @ (U - c)
    v = np.full(U.shape[1], 1.0 / np.sqrt(U.shape[1]))
    for _ in range(POWER_ITERS):
        w = C @ v
        nrm = np.linalg.norm(w)
        if nrm == 0:
            break
        v = w / nrm
    return v


def split_node(U, idx, block: int = BLOCK):
    """(left, right) original indices of one bisection (R-b).

    ``idx`` lists the group's original token indices in ascending order and
    ``U`` their rows of u in the same order.
    """
    n = len(idx)
    b = -(-n // block)
    m = (b // 2) * block
    p = np.asarray(U, dtype=np.float64) @ split_direction(U)
    order = np.lexsort((np.asarray(idx), p))          # p ascending, then index
    left = np.sort(np.asarray(idx)[order[:m]])
    right = np.sort(np.asarray(idx)[order[m:]])
    return left, right


def partition(U, block: int = BLOCK):
    """Leaves (arrays of row indices of U, ascending) in left-to-right order."""
    leaves = []

    def rec(idx):
        if len(idx) <= block:
            leaves.append(idx)
            return
        pos = idx                          # rows of U are indexed by token
        left, right = split_node(U[pos], idx, block)
        rec(left)
        rec(right)

    rec(np.arange(U.shape[0]))
    return leaves


def reblock_permutation(Q, K, prefix: int = 0, block: int = BLOCK) -> np.ndarray:
    """perm[new position] = original token index (R-c, R-d)."""
    N = np.asarray(Q).shape[0]
    U = whiten(Q, key_second_moment(K, prefix), prefix)
    leaves = partition(U, block)
    video = np.concatenate(leaves) + prefix if leaves else np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(prefix), video]).astype(np.int64)


def forward_head_reblock(Q, K, V, top_k: int, prefix: int = 0, variant: str = "anchor",
                         block: int = BLOCK, perm=None, query_blocks=None):
    """The whole path on the reblocked layout; O and lse in the original order (R-e).

    ``perm`` overrides the permutation (tests pass a partition they have
    checked for validity); ``query_blocks`` restricts the attention step to
    those blocks of the permuted sequence.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if perm is None:
        perm = reblock_permutation(Q, K, prefix, block)
    out = forward_head(Q[perm], K[perm], V[perm], top_k, prefix, variant, block,
                       query_blocks=query_blocks)
    O = np.zeros_like(out["O"])
    lse = np.zeros_like(out["lse"])
    O[perm] = out["O"]
    lse[perm] = out["lse"]
    out.update(perm=perm, O=O, lse=lse)
    return out
