"""Content-adaptive block selection by a score threshold: the oracle.

TEST INFRASTRUCTURE ONLY, under the same rules as ``bsa_oracle.py``: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import it.  It shares no code with the CUDA path.

Where it comes from: "H3 Sparse Attention" (comfy.icu, WAS node page),
section "The inputs that matter", the ``method`` input: the content-adaptive
method there takes a threshold ``tau`` instead of a fixed block count, and the
page gives the share of key blocks each setting keeps exact: about 16 % at
tau = 1.0, 7 % at 1.5 and 3 % at 2.0.  "Spark-H3: Block Sparse Attention
Speeds Up MiniMax-H3 in ComfyUI", section "Availability", calls that method's
threshold content-adaptive.  The pages give no formula.

READINGS of this project:

* T-a (statistic).  Those shares are the upper tail of the standard normal,
  1 - Phi(tau) = 15.9 %, 6.7 %, 2.3 %: the threshold is a z-score.  For a
  video query block i the scores S[i, j] over the video key blocks
  j in [pb, nb) have mean mu_i and population standard deviation sigma_i
  (divided by nbv); block j is kept when S[i, j] - mu_i >= tau * sigma_i.
* T-b (no contrast).  A row whose scores are all equal (sigma_i = 0, where
  ">=" keeps everything) keeps every video block: with nothing to rank, the
  row is read exactly.  It is decided by comparing the row's largest and
  smallest score, which rounding cannot disturb (a rounded mean of equal
  values can be off by one ulp, and then so is every deviation).
* T-c (floor).  A row keeps at least one block: when no block reaches the
  threshold (possible only for tau > 0 and few blocks, since the largest
  z-score of n values is at most sqrt(n - 1)), it keeps its top-scoring block,
  ties to the lower index.
* T-d.  Everything else is unchanged from the fixed-count path: the dense
  prefix key blocks are listed in front of every video row and do not enter
  mu or sigma, prefix query rows are dense, and every video key block that is
  not listed enters through its summary row.

Pinned by tests/test_oracle_threshold_pins.py.
"""

from __future__ import annotations

import numpy as np

from .bsa_oracle import (BLOCK, attend, block_scores, block_summaries, pooled_means,
                         video_query_anchor)


def row_threshold(row, tau: float):
    """(mu, tau * sigma) of one row of video-block scores (T-a)."""
    row = np.asarray(row, dtype=np.float64)
    mu = row.mean()
    sigma = np.sqrt(np.mean((row - mu) ** 2))
    return mu, tau * sigma


def select_blocks_threshold(S: np.ndarray, tau: float, prefix_blocks: int):
    """Exact-branch block list E_i for every query block i (ascending).

    Video query block i >= pb: the video key blocks whose score is at least
    tau standard deviations above the row's mean (T-a), all of them when the
    row's scores are all equal (T-b), or else the single
    top-scoring block if none is (T-c); the pb prefix blocks in front (T-d).
    Dense-prefix query block i < pb: all nb blocks.
    """
    nb = S.shape[0]
    pb = prefix_blocks
    cand = np.arange(pb, nb)
    lists = []
    for i in range(nb):
        if i < pb:
            lists.append(np.arange(nb))
            continue
        row = S[i, cand]
        mu, margin = row_threshold(row, tau)
        if row.max() == row.min():
            chosen = cand
        else:
            chosen = cand[(row - mu) >= margin]
        if chosen.size == 0:
            chosen = cand[np.lexsort((cand, -row))[:1]]
        lists.append(np.concatenate([np.arange(pb), np.sort(chosen)]).astype(np.int64))
    return lists


def forward_head_threshold(Q, K, V, tau: float, prefix: int = 0, variant: str = "anchor",
                           block: int = BLOCK, query_blocks=None):
    """The whole path for one (batch, head) slice with threshold selection.

    Same stages and outputs as ``bsa_oracle.forward_head``; only the
    selection differs.  ``query_blocks`` restricts the attention step.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N = Q.shape[0]
    if prefix % block or not (0 <= prefix < N):
        raise ValueError("prefix must be a multiple of the block size in [0, N)")
    if not np.isfinite(tau):
        raise ValueError("tau must be finite")
    pb = prefix // block
    qpool = pooled_means(Q, block)
    kpool = pooled_means(K, block)
    qbar = video_query_anchor(Q, prefix)
    ksum, vsum, bias = block_summaries(K, V, qbar, variant, block)
    S = block_scores(qpool, kpool)
    lists = select_blocks_threshold(S, tau, pb)
    O, lse = attend(Q, K, V, lists, ksum, vsum, bias, pb, block, query_blocks)
    return dict(qpool=qpool, kpool=kpool, anchor=qbar, ksum=ksum, vsum=vsum,
                bias=bias, scores=S, lists=lists, O=O, lse=lse)
