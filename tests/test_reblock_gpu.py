"""GPU parity of the adaptive reblocking (Spark-Reblock) against its oracle.

The layout is a tree of floating-point split decisions, so several layouts are
correct to within rounding: the GPU stores the whitened queries u in bf16
(relative 2^-9), so a token whose projection lies within ~2^-9 of a split's
threshold may land on either side.  The tests therefore check the GPU's layout
for validity, group by group: for every group of the GPU's tree (a contiguous
range of its layout), the oracle recomputes the split of that very group in
fp64; the GPU's left part must equal the oracle's except for tokens whose
oracle projection lies within EPS of the oracle's threshold.  Everything
unique is compared exactly: the prefix stays put, the layout is a
permutation, leaves are 128 tokens (the last one ragged) in ascending order.
The attention on the GPU's layout is then checked stage by stage against the
bf16 oracle on the same permuted inputs, and bsa_forward_reblock against the
stage path put back in the original order.
"""

import numpy as np
import pytest
import torch

from oracle import bsa_oracle_reblock as rb
from block_sparse_video_bsa_b200 import bsa
from block_sparse_video_bsa_b200.inputs import CONFIGS, make_qkv

from parity_util import check_head, host, run_stages

pytestmark = pytest.mark.gpu

EPS = 4e-3          # 2 * 2^-9 (bf16 u) plus an allowance for the direction
MAX_SWAP_FRAC = 5e-3


def check_layout(perm_h, Qh, Kh, prefix):
    """Validity of one head's GPU layout; returns (groups, swapped tokens)."""
    N = len(perm_h)
    nv = N - prefix
    np.testing.assert_array_equal(perm_h[:prefix], np.arange(prefix))
    np.testing.assert_array_equal(np.sort(perm_h), np.arange(N))
    video = perm_h[prefix:] - prefix
    U = rb.whiten(Qh, rb.key_second_moment(Kh, prefix), prefix)
    stack, groups, swapped = [(0, nv)], 0, 0
    while stack:
        s, c = stack.pop()
        if c <= 128:
            assert np.all(np.diff(video[s:s + c]) > 0), "leaf not ascending"
            continue
        members = np.sort(video[s:s + c])
        m = (-(-c // 128) // 2) * 128
        p = U[members] @ rb.split_direction(U[members])
        order = np.lexsort((members, p))
        mis = set(members[order[:m]].tolist()) ^ set(video[s:s + m].tolist())
        if mis:
            lo, hi = p[order[m - 1]], p[order[m]]
            pm = dict(zip(members.tolist(), p.tolist()))
            bad = [t for t in mis if not (lo - EPS <= pm[t] <= hi + EPS)]
            assert not bad, (s, c, len(bad), lo, hi)
        groups += 1
        swapped += len(mis)
        stack += [(s, m), (s + m, c - m)]
    assert swapped <= MAX_SWAP_FRAC * max(nv, 1) + 2, (swapped, nv)
    return groups, swapped


@pytest.mark.parametrize("B,H,N,prefix,kind", [
    (1, 2, 1000, 0, "block_offset"),
    (1, 2, 1500, 256, "block_offset"),     # dense prefix + ragged
    (2, 1, 4100, 0, "block_offset"),       # ragged tail of 4 rows
    (1, 1, 300, 0, "iid"),
    (1, 1, 17_000, 0, "block_offset"),     # groups larger than one 2048-row chunk
    (1, 1, 129, 0, "iid"),                 # one split
    (1, 1, 128, 0, "iid"),                 # one block: identity
    (1, 1, 1, 0, "iid"),
])
def test_reblock_layout_is_valid(B, H, N, prefix, kind):
    Q, K, V = make_qkv(B, H, N, 128, kind, seed=N, device="cuda")
    perm = bsa.reblock(Q, K, prefix)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            check_layout(perm[b, h].cpu().numpy().astype(np.int64), host(Q[b, h]), host(K[b, h]),
                         prefix)


@pytest.mark.parametrize("B,H,N,top_k,prefix,variant", [
    (1, 2, 1000, 3, 0, "anchor"),
    (1, 2, 1500, 2, 256, "anchor"),
    (1, 1, 4100, 5, 0, "mean"),
])
def test_forward_reblock_matches_oracle_on_its_layout(B, H, N, top_k, prefix, variant):
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", seed=3, device="cuda")
    perm = bsa.reblock(Q, K, prefix)
    p = bsa.params(B, H, N, top_k, prefix, variant)
    Qp, Kp, Vp = (torch.empty_like(Q) for _ in range(3))
    bsa.bsa_permute(p, Q, K, V, perm, Qp, Kp, Vp)
    buf = run_stages(Qp, Kp, Vp, top_k, prefix, variant)
    for b in range(B):
        for h in range(H):
            check_head(buf, Qp, Kp, Vp, b, h, top_k, prefix, variant)
    O, lse = bsa.forward_reblock(Q, K, V, top_k, prefix, variant, return_lse=True)
    O2, lse2 = bsa.forward_reblock(Q, K, V, top_k, prefix, variant, return_lse=True)
    Ob, lseb = torch.empty_like(Q), torch.empty_like(lse)
    bsa.bsa_unpermute(p, buf["O"], buf["lse"], perm, Ob, lseb)
    torch.cuda.synchronize()
    assert torch.equal(O, Ob) and torch.equal(lse, lseb)
    assert torch.equal(O, O2) and torch.equal(lse, lse2)        # deterministic
    # the permuted inputs really are Q[perm]
    idx = perm.long()[..., None].expand(-1, -1, -1, 128)
    assert torch.equal(Qp, torch.gather(Q, 2, idx))


def test_scrambled_clusters_form_their_own_blocks():
    # Four clusters of 128 queries on an arc, scrambled over the sequence; keys
    # with K^T K proportional to I (the metric is the plain cosine).  Every
    # block of the GPU's layout must hold one whole cluster.
    N, d = 512, 128
    g = torch.Generator().manual_seed(0)
    labels = torch.arange(N) // 128
    ang = labels.double() * 0.3
    Q = torch.zeros(N, d, dtype=torch.float64)
    Q[:, 0], Q[:, 1] = torch.cos(ang), torch.sin(ang)
    Q += 0.01 * torch.randn(N, d, generator=g, dtype=torch.float64)
    shuffle = torch.randperm(N, generator=g)
    Q, labels = Q[shuffle], labels[shuffle]
    K = torch.eye(d, dtype=torch.float64).repeat(N // d, 1)
    Qd = Q.to(torch.bfloat16)[None, None].cuda().contiguous()
    Kd = K.to(torch.bfloat16)[None, None].cuda().contiguous()
    perm = bsa.reblock(Qd, Kd)[0, 0].cpu()
    for blk in perm.view(4, 128):
        assert len(set(labels[blk.long()].tolist())) == 1


def test_reblock_full_size_sampled_head():
    cfg = CONFIGS["h3_768p_5s"]
    B, H, N = cfg["B"], cfg["H"], cfg["N"]
    Q, K, V = make_qkv(B, H, N, 128, cfg["kind"], 0, device="cuda")
    perm = bsa.reblock(Q, K, cfg["prefix"])
    O = bsa.forward_reblock(Q, K, V, cfg["top_k"], cfg["prefix"], cfg["variant"])
    torch.cuda.synchronize()
    h = 13
    groups, swapped = check_layout(perm[0, h].cpu().numpy().astype(np.int64), host(Q[0, h]),
                                   host(K[0, h]), cfg["prefix"])
    assert groups == -(-N // 128) - 1
    # attention on the GPU's layout for that head: the stage path on the
    # permuted head, against the oracle on the same permuted inputs
    p1 = bsa.params(1, 1, N, cfg["top_k"], cfg["prefix"], cfg["variant"])
    Qh, Kh, Vh = (x[:, h:h + 1].contiguous() for x in (Q, K, V))
    Qp, Kp, Vp = (torch.empty_like(Qh) for _ in range(3))
    bsa.bsa_permute(p1, Qh, Kh, Vh, perm[:, h:h + 1].contiguous(), Qp, Kp, Vp)
    buf = run_stages(Qp, Kp, Vp, cfg["top_k"], cfg["prefix"], cfg["variant"], with_lse=True)
    check_head(buf, Qp, Kp, Vp, 0, 0, cfg["top_k"], cfg["prefix"], cfg["variant"],
               check_lse=True)
    Ob = torch.empty_like(Qh)
    bsa.bsa_unpermute(p1, buf["O"], None, perm[:, h:h + 1].contiguous(), Ob)
    torch.cuda.synchronize()
    assert torch.equal(O[:, h:h + 1], Ob)
    del Q, K, V, O
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N,prefix,variant", [(1500, 256, "anchor"), (4100, 0, "mean"),
                                              (17_000, 0, "anchor")])
def test_permuted_stages_equal_permute_then_stages(N, prefix, variant):
    # bsa_pool_permuted / bsa_summarize_permuted read through perm and write
    # the permuted rows themselves: the same bits as bsa_permute followed by
    # bsa_pool / bsa_summarize on the permuted copies
    B, H = 1, 2
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", 4, device="cuda")
    p = bsa.params(B, H, N, 8, prefix, variant)
    perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(256, bsa.bsa_reblock_workspace_bytes(p)), dtype=torch.uint8,
                     device="cuda")
    bsa.bsa_reblock(p, Q, K, perm, ws)
    Qp, Kp, Vp = (torch.empty_like(X) for X in (Q, K, V))
    bsa.bsa_permute(p, Q, K, V, perm, Qp, Kp, Vp)
    a = bsa.stage_buffers(B, H, N, 8, prefix, variant)
    bsa.bsa_pool(p, Qp, a["qpool"], a["anchor"])
    bsa.bsa_summarize(p, Kp, Vp, a["anchor"], a["kpool"], a["ksum"], a["vsum"], a["bias"])
    b = bsa.stage_buffers(B, H, N, 8, prefix, variant)
    Qq, Kq, Vq = (torch.full_like(X, float("nan")) for X in (Q, K, V))
    bsa.bsa_pool_permuted(p, Q, perm, Qq, b["qpool"], b["anchor"])
    bsa.bsa_summarize_permuted(p, K, V, perm, Kq, Vq, b["anchor"], b["kpool"], b["ksum"],
                               b["vsum"], b["bias"])
    torch.cuda.synchronize()
    assert torch.equal(Qq, Qp) and torch.equal(Kq, Kp) and torch.equal(Vq, Vp)
    for k in ("qpool", "anchor", "kpool", "ksum", "vsum", "bias"):
        assert torch.equal(a[k], b[k]), k
