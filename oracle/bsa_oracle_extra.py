"""Extra top-scoring tokens per query block (``extra_tokens``): the oracle.

TEST INFRASTRUCTURE ONLY, under the same rules as ``bsa_oracle.py``: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import it.  It shares no code with the CUDA path.

Where it comes from: "H3 Sparse Attention" (comfy.icu, WAS node page),
section "The inputs that matter": besides its chosen blocks, each query block
also reads a number of individually chosen top-scoring tokens (the
``extra_tokens`` input, 256 by default; 0 is the fastest setting).  The pages
describe it for a method without summary rows and give no formula.

READINGS of this project:

* X-a (score).  The score of key token u for query block i is
  s_iu = qhat_i . k_u / sqrt(d): the pooled query against the single key, the
  token analogue of the pooled block score.
* X-b (candidates).  The video tokens of the blocks NOT in E_i; the listed
  blocks' tokens are read exactly already, and dense-prefix blocks are always
  listed.  Dense-prefix query blocks read everything and take none.
* X-c (choice).  The min(n_extra, #candidates) candidates of highest score,
  ties to the lower token index.
* X-d (every token once).  In this method every key token enters the softmax
  exactly once: exactly when its block is listed, otherwise through its
  block's summary row.  An extra token is read exactly, so its block's
  summary row stands for the block's REMAINING tokens: the same summary
  definition (anchor-weighted or mean, with its bias) over those tokens only.
  A block whose tokens are all extra has no summary row.

Pinned by tests/test_oracle_extra_pins.py.
"""

from __future__ import annotations

import math

import numpy as np

from .bsa_oracle import (BLOCK, block_bounds, block_scores, block_summaries,
                         pooled_means, select_blocks, video_query_anchor)


def token_scores(qpool, K) -> np.ndarray:
    """s[i, u] = qhat_i . k_u / sqrt(d) for every query block i and token u (X-a)."""
    qpool = np.asarray(qpool, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    return (qpool @ K.T) / math.sqrt(K.shape[1])


def select_extra_tokens(s, lists, prefix_blocks: int, n_extra: int, N: int,
                        block: int = BLOCK):
    """Extra tokens of every query block, ascending (X-b, X-c)."""
    bounds = block_bounds(N, block)
    pb = prefix_blocks
    out = []
    for i in range(len(bounds)):
        if i < pb or n_extra <= 0:
            out.append(np.zeros(0, dtype=np.int64))
            continue
        listed = set(int(j) for j in lists[i])
        cand = np.concatenate([np.arange(*bounds[j]) for j in range(pb, len(bounds))
                               if j not in listed] or [np.zeros(0, dtype=np.int64)])
        order = np.lexsort((cand, -s[i, cand]))          # score descending, then index
        out.append(np.sort(cand[order[:n_extra]]).astype(np.int64))
    return out


def summary_of_tokens(K, V, tokens, anchor, variant: str):
    """(k~, v~, bias) of one set of tokens by the block-summary definition (X-d)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    ks, vs, b = block_summaries(np.asarray(K)[tokens], np.asarray(V)[tokens], anchor, variant,
                                block=len(tokens))
    return ks[0], vs[0], b[0]


def attend_extra(Q, K, V, lists, extras, ksum, vsum, bias, anchor, variant: str,
                 prefix_blocks: int, block: int = BLOCK, query_blocks=None):
    """Exact branch (listed blocks + extra tokens) and summary rows of the
    remaining tokens, one softmax per query row; returns O and lse."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    bounds = block_bounds(N, block)
    nb, pb = len(bounds), prefix_blocks
    O = np.zeros((N, V.shape[1]))
    lse = np.zeros(N)
    for i, (a, b) in enumerate(bounds):
        if query_blocks is not None and i not in query_blocks:
            continue
        listed = set(int(j) for j in lists[i])
        extra = set(int(u) for u in extras[i])
        exact = np.concatenate([np.arange(*bounds[j]) for j in lists[i]] +
                               [np.asarray(sorted(extra), dtype=np.int64)])
        rows_k, rows_v, rows_b = [], [], []
        if i >= pb:
            for j in range(pb, nb):
                if j in listed:
                    continue
                toks = np.arange(*bounds[j])
                rest = np.array([t for t in toks if t not in extra], dtype=np.int64)
                if len(rest) == len(toks):
                    rows_k.append(ksum[j]); rows_v.append(vsum[j]); rows_b.append(bias[j])
                elif len(rest):
                    k_, v_, b_ = summary_of_tokens(K, V, rest, anchor, variant)
                    rows_k.append(k_); rows_v.append(v_); rows_b.append(b_)
        logits = (Q[a:b] @ K[exact].T) * scale
        vals = V[exact]
        if rows_k:
            zl = (Q[a:b] @ np.array(rows_k).T) * scale + np.array(rows_b)[None, :]
            logits = np.concatenate([logits, zl], axis=1)
            vals = np.concatenate([vals, np.array(rows_v)], axis=0)
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        l = p.sum(axis=1)
        O[a:b] = (p @ vals) / l[:, None]
        lse[a:b] = m[:, 0] + np.log(l)
    return O, lse


def forward_head_extra(Q, K, V, top_k: int, n_extra: int, prefix: int = 0,
                       variant: str = "anchor", block: int = BLOCK, query_blocks=None):
    """The whole path for one (batch, head) slice with n_extra extra tokens per
    query block; same stages as ``bsa_oracle.forward_head`` plus the token
    choice."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N = Q.shape[0]
    if prefix % block or not (0 <= prefix < N):
        raise ValueError("prefix must be a multiple of the block size in [0, N)")
    if top_k < 1 or n_extra < 0:
        raise ValueError("top_k must be >= 1 and n_extra >= 0")
    pb = prefix // block
    qpool = pooled_means(Q, block)
    kpool = pooled_means(K, block)
    qbar = video_query_anchor(Q, prefix)
    ksum, vsum, bias = block_summaries(K, V, qbar, variant, block)
    lists = select_blocks(block_scores(qpool, kpool), top_k, pb)
    s = token_scores(qpool, K)
    extras = select_extra_tokens(s, lists, pb, n_extra, N, block)
    O, lse = attend_extra(Q, K, V, lists, extras, ksum, vsum, bias, qbar, variant, pb, block,
                          query_blocks)
    return dict(qpool=qpool, kpool=kpool, anchor=qbar, ksum=ksum, vsum=vsum, bias=bias,
                lists=lists, token_scores=s, extras=extras, O=O, lse=lse)
