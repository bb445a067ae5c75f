"""GPU parity of the selection stage alone (bsa_select / bsa_select_threshold
on pooled inputs given directly), at row lengths that take every kernel
configuration:
  * tensor-core scores, two CTAs per SM (up to 512 video blocks) or one,
    32 query blocks per CTA (up to 1984 blocks), keys in registers (up to
    1504 blocks) or in shared memory beyond;
  * tensor-core scores, 16 query blocks per CTA (1985 to 3072 blocks);
  * the SIMT kernel (more than 3072 blocks).
Selection is "each query block attends to its top-k key blocks"
(h3-sparse-attn 0.1.0, opening description), or the threshold tau ("H3
Sparse Attention", WAS node page, "The inputs that matter").  Pooled vectors
of half-integers give scores that are exact on both sides, so rows with many
equal scores must match the oracle's lowest-index tie-break exactly."""

import numpy as np
import pytest
import torch

import oracle as orc
from block_sparse_video_bsa_b200 import bsa

from parity_util import check_selection, check_threshold_selection

pytestmark = pytest.mark.gpu


def _pooled(nb, kind, seed):
    g = torch.Generator().manual_seed(seed)
    if kind == "ties":   # entries in {-1, -0.5, 0, 0.5, 1}: exact products and sums
        q = torch.randint(-2, 3, (nb, 128), generator=g).float() * 0.5
        k = torch.randint(-2, 3, (nb, 128), generator=g).float() * 0.5
    else:                # a shared direction plus noise, like pooled video blocks
        base = torch.randn(1, 128, generator=g)
        q = base + 0.5 * torch.randn(nb, 128, generator=g)
        k = base + 0.5 * torch.randn(nb, 128, generator=g)
    return q, k


def _run(nbv, pb, kind, seed, top_k=None, tau=None):
    nb = nbv + pb
    N = nb * 128 - 37                      # ragged tail (pooled inputs are given)
    p = bsa.params(1, 1, N, 1 if top_k is None else top_k, pb * 128, "anchor")
    q, k = _pooled(nb, kind, seed)
    qd = q.view(1, 1, nb, 128).cuda().contiguous()
    kd = k.view(1, 1, nb, 128).cuda().contiguous()
    cnt = torch.empty(1, 1, nb, dtype=torch.int32, device="cuda")
    if tau is None:
        idx = torch.empty(1, 1, nb, bsa.bsa_select_capacity(p), dtype=torch.int32, device="cuda")
        bsa.bsa_select(p, qd, kd, idx, cnt)
    else:
        idx = torch.empty(1, 1, nb, bsa.bsa_threshold_capacity(p), dtype=torch.int32,
                          device="cuda")
        bsa.bsa_select_threshold(p, tau, qd, kd, idx, cnt)
    torch.cuda.synchronize()
    S = orc.block_scores(q.double().numpy(), k.double().numpy())
    return idx[0, 0].cpu().numpy(), cnt[0, 0].cpu().numpy(), S


@pytest.mark.parametrize("nbv,top_k,pb,kind", [
    (295, 64, 0, "gauss"),      # 32 query blocks per CTA, 13 keys per lane
    (295, 64, 0, "ties"),
    (1045, 64, 2, "gauss"),     # 2K-5s rows: 35 keys per lane, one CTA per SM
    (1400, 700, 0, "ties"),     # 47 keys per lane, half the row kept
    (1400, 1, 1, "gauss"),
    (1800, 64, 0, "gauss"),     # keys in shared memory
    (3000, 64, 0, "gauss"),     # 16 query blocks per CTA, all 512 TMEM columns
    (3000, 5, 3, "ties"),
    (5000, 64, 0, "gauss"),     # SIMT scores
])
def test_topk_row_lengths(nbv, top_k, pb, kind):
    idx, cnt, S = _run(nbv, pb, kind, seed=nbv + top_k, top_k=top_k)
    lists = orc.select_blocks(S, top_k, pb)
    if kind == "ties":
        # scores exact on both sides: the lists are the oracle's, ties included
        for i in range(nbv + pb):
            c = int(cnt[i])
            assert [int(v) for v in idx[i, :c]] == [int(v) for v in lists[i]], i
            assert (idx[i, c:] == -1).all()
    else:
        check_selection(idx, cnt, {"scores": S, "lists": lists}, pb, top_k)


def test_ties_exceed_the_threshold_count():
    # every score of a row takes one of a few values, so the k-th score is
    # shared by many more blocks than are needed: the lowest indices win
    nbv, top_k = 1045, 100
    idx, cnt, S = _run(nbv, 0, "ties", seed=3, top_k=top_k)
    lists = orc.select_blocks(S, top_k, 0)
    shared = 0
    for i in range(nbv):
        row = S[i]
        kth = np.sort(row)[::-1][top_k - 1]
        shared += int((row == kth).sum() > 1)
        assert [int(v) for v in idx[i, :top_k]] == [int(v) for v in lists[i]], i
    assert shared > nbv // 2     # the case is really exercised


@pytest.mark.parametrize("nbv,pb,tau", [(1045, 0, 1.0), (3000, 2, 0.5), (5000, 0, 1.5)])
def test_threshold_row_lengths(nbv, pb, tau):
    idx, cnt, S = _run(nbv, pb, "gauss", seed=nbv, tau=tau)
    check_threshold_selection(idx, cnt, S, tau, pb)
