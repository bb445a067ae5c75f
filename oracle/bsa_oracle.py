"""Plain fp64 CPU oracle for the block-sparse video self-attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The CUDA
library never imports, links or calls it, and the two share no code: the only
thing both sides use is the seeded input generator, which holds none of the
method's arithmetic.

Everything here is written for a reader checking it by eye against the pages:
one (batch, head) slice at a time, numpy float64, one Python loop per block,
library primitives (matmul, exp, lexsort) as single steps, no blocking, fusion
or reordering beyond what the definitions state.

Where the method comes from (web pages; cited by title and section):

* "h3-sparse-attn 0.1.0" (PyPI project page), opening description: each query
  block attends to its top-k key blocks of 128 tokens; the skipped blocks are
  folded back in as one summary row each.  Section "Use": ``top_k`` counts
  128-token key blocks.
* "Spark-H3: Block Sparse Attention Speeds Up MiniMax-H3 in ComfyUI", section
  "What Spark-Attn changes": an exact branch over the top-ranked key/value
  blocks and a compressed branch for everything else; the Spark-Reweight
  bullet replaces mean-pooled summaries with weighted summaries plus a
  log-mass bias, scored against the mean of the video queries as one anchor
  per head; the compressed-branch figure caption says the biased pooled
  logit's exponential matches the expected exponential E[exp(x)].
* "H3 Sparse Attention" (comfy.icu, WAS node), "The inputs that matter"
  (prompt rows read exactly) and "H3 Sparse Attention" (comfy.icu,
  video_budget node) (text rows stay fully dense): the dense prefix.

The pages print no formulas.  The summary formula used here (softmax-at-the-
anchor weighted means, bias = ln n_j + (logsumexp_t x_t - ln n_j - qbar.k~/sqrt d))
and the pooled block score (dot product of mean-pooled Q and K blocks) are the
fixed readings of the Spark-Reweight bullet this project builds to; every
other reading of a silent point is marked ``READING`` where it is used.

Every function below is pinned by ``tests/test_oracle_pins.py`` against
something other than itself (closed forms, textbook dense attention, torch's
SDPA, brute-force enumeration); none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 128
VARIANTS = ("anchor", "mean")


def block_bounds(N: int, block: int = BLOCK):
    """Token ranges [start, end) of the blocks of a length-N sequence.

    h3-sparse-attn 0.1.0, description: the sequence is cut into 128-token
    blocks.  READING (silent on the pages): when N is not a multiple of the
    block size the last block is ragged and holds the N - block*(nb-1)
    remaining tokens.
    """
    nb = -(-N // block)
    return [(j * block, min((j + 1) * block, N)) for j in range(nb)]


def pooled_means(X: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of the rows of each block of X ([N, d] -> [nb, d]).

    Used for both Q and K (the pooled block representatives that the block
    score compares).  READING: a ragged block is averaged over its real
    tokens, not over 128.
    """
    X = np.asarray(X, dtype=np.float64)
    return np.stack([X[a:b].mean(axis=0) for a, b in block_bounds(len(X), block)])


def video_query_anchor(Q: np.ndarray, prefix: int) -> np.ndarray:
    """Per-head anchor q-bar: the mean of the video queries (rows >= prefix).

    Spark-H3 page, Spark-Reweight bullet: scoring uses the mean of the video
    queries as one anchor per head.  The dense prefix rows are text-like
    rows, not video, so they are left out.
    """
    Q = np.asarray(Q, dtype=np.float64)
    return Q[prefix:].mean(axis=0)


def block_summaries(K: np.ndarray, V: np.ndarray, anchor: np.ndarray,
                    variant: str, block: int = BLOCK):
    """One summary row (k~_j, v~_j, bias_j) per key block j.

    ``variant == "anchor"`` (Spark-Reweight bullet, Spark-H3 page): with
    x_t = q-bar . k_t / sqrt(d) over the tokens t of block j,
        LSE_j = logsumexp_t x_t,   w_t = exp(x_t - LSE_j)   (softmax over the block)
        k~_j  = sum_t w_t k_t,     v~_j = sum_t w_t v_t
        bias_j = ln n_j + (LSE_j - ln n_j - q-bar . k~_j / sqrt(d)).
    The ln n_j terms cancel; the printed form is kept on purpose.  At the
    anchor the summary logit q-bar.k~/sqrt(d) + bias equals LSE_j, so its
    exponential is the block's exact exp-mass (the figure caption's "green
    point").

    ``variant == "mean"`` (the mean-pooled baseline the bullet replaces):
    k~_j = mean K, v~_j = mean V, bias_j = ln n_j (n_j copies of the mean key).

    Summaries are produced for every block; a dense-prefix block's summary
    is never used by ``attend``.
    """
    if variant not in VARIANTS:
        raise ValueError(f"unknown summary variant {variant!r}")
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d = K.shape[1]
    scale = 1.0 / math.sqrt(d)
    bounds = block_bounds(len(K), block)
    ksum = np.zeros((len(bounds), d))
    vsum = np.zeros((len(bounds), V.shape[1]))
    bias = np.zeros(len(bounds))
    for j, (a, b) in enumerate(bounds):
        Kj, Vj, n = K[a:b], V[a:b], b - a
        if variant == "mean":
            ksum[j] = Kj.mean(axis=0)
            vsum[j] = Vj.mean(axis=0)
            bias[j] = math.log(n)
            continue
        x = (Kj @ anchor) * scale
        xmax = x.max()
        lse = xmax + math.log(np.exp(x - xmax).sum())
        w = np.exp(x - lse)
        ksum[j] = w @ Kj
        vsum[j] = w @ Vj
        bias[j] = math.log(n) + (lse - math.log(n) - float(anchor @ ksum[j]) * scale)
    return ksum, vsum, bias


def block_scores(qpool: np.ndarray, kpool: np.ndarray) -> np.ndarray:
    """Pooled block score S[i, j] = qhat_i . khat_j / sqrt(d), all pairs.

    h3-sparse-attn 0.1.0, description: each query block picks its top-k key
    blocks.  READING: the score is the scaled dot product of the two
    mean-pooled blocks (the attention logit of the pooled pair), so a 1e-5
    gap is measured on the logit scale.
    """
    d = qpool.shape[1]
    return (qpool @ kpool.T) / math.sqrt(d)


def select_blocks(S: np.ndarray, top_k: int, prefix_blocks: int):
    """Exact-branch block list E_i for every query block i (ascending).

    Video query block i >= pb: the k_eff = min(top_k, nbv) video key blocks
    j in [pb, nb) with the largest S[i, j]; ties go to the lower index
    (order by score descending, then index ascending).  The pb dense-prefix
    key blocks are always added in front (prompt rows read exactly, WAS node
    "sink_conditioning"; text rows stay dense, video_budget node).
    Dense-prefix query block i < pb: all nb blocks (the row is dense).

    READINGS: prefix blocks do not count against top_k; top_k above the
    number of video blocks is clamped; a query block's own block is not
    forced in.
    """
    nb = S.shape[0]
    pb = prefix_blocks
    k_eff = min(top_k, nb - pb)
    cand = np.arange(pb, nb)
    lists = []
    for i in range(nb):
        if i < pb:
            lists.append(np.arange(nb))
            continue
        order = np.lexsort((cand, -S[i, cand]))      # primary: -S, secondary: j
        chosen = np.sort(cand[order[:k_eff]])
        lists.append(np.concatenate([np.arange(pb), chosen]).astype(np.int64))
    return lists


def attend(Q: np.ndarray, K: np.ndarray, V: np.ndarray, lists, ksum, vsum, bias,
           prefix_blocks: int, block: int = BLOCK, query_blocks=None):
    """Exact branch + compressed branch, one softmax per query row.

    For query row t in block i the logits are
      { q_t . k_u / sqrt(d) : u a token of a block in E_i }          (exact)
      { q_t . k~_j / sqrt(d) + bias_j : j >= pb, j not in E_i }      (summaries)
    and O_t = softmax(logits) @ [V rows ; v~ rows].  Dense-prefix query rows
    have every block in E_i and therefore no summary rows.  Also returns
    lse_t = log sum exp(logits) (natural log).  ``query_blocks`` optionally
    restricts the work to those query blocks (other rows are left at 0).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    bounds = block_bounds(N, block)
    nb = len(bounds)
    pb = prefix_blocks
    O = np.zeros((N, V.shape[1]))
    lse = np.zeros(N)
    for i, (a, b) in enumerate(bounds):
        if query_blocks is not None and i not in query_blocks:
            continue
        E = list(lists[i])
        tok = np.concatenate([np.arange(*bounds[j]) for j in E])
        logits = (Q[a:b] @ K[tok].T) * scale
        vals = V[tok]
        if i >= pb:
            inE = set(int(j) for j in E)
            skipped = [j for j in range(pb, nb) if j not in inE]
            if skipped:
                zl = (Q[a:b] @ ksum[skipped].T) * scale + bias[skipped][None, :]
                logits = np.concatenate([logits, zl], axis=1)
                vals = np.concatenate([vals, vsum[skipped]], axis=0)
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        l = p.sum(axis=1)
        O[a:b] = (p @ vals) / l[:, None]
        lse[a:b] = m[:, 0] + np.log(l)
    return O, lse


def forward_head(Q, K, V, top_k: int, prefix: int = 0, variant: str = "anchor",
                 block: int = BLOCK, query_blocks=None):
    """The whole path for one (batch, head) slice: pool, summarize, select, attend.

    Q, K, V are [N, d] arrays (any float type; widened to float64).  Returns a
    dict with every intermediate so tests can compare stage by stage.
    ``query_blocks`` restricts only the attention step (see ``attend``).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N = Q.shape[0]
    if prefix % block or not (0 <= prefix < N):
        raise ValueError("prefix must be a multiple of the block size in [0, N)")
    if top_k < 1:
        raise ValueError("top_k must be >= 1")
    pb = prefix // block
    qpool = pooled_means(Q, block)
    kpool = pooled_means(K, block)
    qbar = video_query_anchor(Q, prefix)
    ksum, vsum, bias = block_summaries(K, V, qbar, variant, block)
    S = block_scores(qpool, kpool)
    lists = select_blocks(S, top_k, pb)
    O, lse = attend(Q, K, V, lists, ksum, vsum, bias, pb, block, query_blocks)
    return dict(qpool=qpool, kpool=kpool, anchor=qbar, ksum=ksum, vsum=vsum,
                bias=bias, scores=S, lists=lists, O=O, lse=lse)


def forward(Q, K, V, top_k: int, prefix: int = 0, variant: str = "anchor",
            block: int = BLOCK):
    """[B, H, N, d] inputs: ``forward_head`` on every (b, h); returns O [B,H,N,d]."""
    Q = np.asarray(Q)
    B, H = Q.shape[:2]
    O = np.zeros(Q.shape[:3] + (np.asarray(V).shape[3],))
    for b in range(B):
        for h in range(H):
            O[b, h] = forward_head(Q[b, h], K[b, h], V[b, h], top_k, prefix,
                                   variant, block)["O"]
    return O


def effective_pairs(N: int, lists, prefix_blocks: int, block: int = BLOCK,
                    query_blocks=None) -> int:
    """Computed (query, key-or-summary) pairs of one head, masked columns excluded.

    Exact pairs count the real tokens of each listed block; summary pairs
    count one column per skipped video block for every video query row.
    Multiplied by 4*d this is the method's effective FLOP count.
    """
    bounds = block_bounds(N, block)
    nb = len(bounds)
    total = 0
    for i, (a, b) in enumerate(bounds):
        if query_blocks is not None and i not in query_blocks:
            continue
        rows = b - a
        exact = sum(bounds[j][1] - bounds[j][0] for j in lists[i])
        summ = 0 if i < prefix_blocks else (nb - prefix_blocks) - (len(lists[i]) - prefix_blocks)
        total += rows * (exact + summ)
    return total
