"""Comparison helpers for the GPU-vs-oracle parity tests (acceptance rules of
the spec: indices exact except at score gaps under 1e-5; O max-abs <= 2e-2 and
rel-L2 <= 1e-2 against the fp64 oracle)."""

import numpy as np
import torch

import oracle as orc
from block_sparse_video_bsa_b200 import bsa

TIE_GAP = 1e-5
O_MAX_ABS = 2e-2
O_REL_L2 = 1e-2
POOL_RTOL, POOL_ATOL = 1e-5, 1e-6
SUM_RTOL, SUM_ATOL = 2.0 ** -7, 1e-3
# bf16 unit roundoff.  The GPU feeds bf16(k~) to the MMA and computes its
# bias from the same bf16(k~), so (exactly, up to fp32 slack)
#   z_gpu(q) - z_ref(q) = (q - qbar) . (bf16(k~) - k~) / sqrt(d),
# bounded by 2^-8 * sum_d |q_d - qbar_d| |k~_d| / sqrt(d); the bias alone moves
# by the same expression at q = 0.  (Mean variant: bias = ln n has no k~
# term and the logit shift is q . (bf16(k~) - k~) / sqrt(d).)  lse moves by at
# most the largest shift of any summary logit.  These bounds use oracle values
# only.
BF16_U = 2.0 ** -8
FP32_SLACK = 2e-4


def run_stages(Q, K, V, top_k, prefix, variant, with_lse=True):
    """Every stage through its own C entry point; returns all device outputs."""
    B, H, N, _ = Q.shape
    p = bsa.params(B, H, N, top_k, prefix, variant)
    buf = bsa.stage_buffers(B, H, N, top_k, prefix, variant, device=Q.device)
    bsa.bsa_pool(p, Q, buf["qpool"], buf["anchor"])
    bsa.bsa_summarize(p, K, V, buf["anchor"], buf["kpool"], buf["ksum"], buf["vsum"], buf["bias"])
    bsa.bsa_select(p, buf["qpool"], buf["kpool"], buf["idx"], buf["cnt"])
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if with_lse else None
    bsa.bsa_attend(p, Q, K, V, buf["idx"], buf["cnt"], buf["ksum"], buf["vsum"], buf["bias"],
                   O, lse)
    torch.cuda.synchronize()
    buf["O"] = O
    buf["lse"] = lse
    return buf


def host(t):
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 \
        else t.detach().cpu().numpy()


def check_selection(idx_row_block, cnt_row, ref, prefix_blocks, top_k):
    """idx/cnt of one head vs the oracle's lists; returns query blocks with a
    near-tie swap (allowed only where the oracle's scores are within 1e-5 of
    the k-th score)."""
    S, lists = ref["scores"], ref["lists"]
    nb = S.shape[0]
    pb = prefix_blocks
    k_eff = min(top_k, nb - pb)
    swapped = set()
    for i in range(nb):
        want = list(lists[i])
        c = int(cnt_row[i])
        assert c == len(want), (i, c, len(want))
        got = [int(v) for v in idx_row_block[i, :c]]
        assert all(int(v) == -1 for v in idx_row_block[i, c:]), f"padding of row {i}"
        if got == want:
            continue
        assert i >= pb, f"prefix row {i} differs"
        assert got[:pb] == list(range(pb))
        assert got == sorted(set(got)) and all(pb <= j < nb for j in got[pb:])
        cand = np.arange(pb, nb)
        kth = np.sort(S[i, cand])[::-1][k_eff - 1]
        for j in set(got) ^ set(want):
            assert abs(S[i, j] - kth) < TIE_GAP, (i, j, S[i, j], kth)
        swapped.add(i)
    return swapped


def rows_of_blocks(N, blocks):
    rows = []
    for i in sorted(blocks):
        a, b = orc.block_bounds(N)[i]
        rows.extend(range(a, b))
    return np.array(rows, dtype=np.int64)


def check_output(O_gpu, O_ref, N):
    """O of one head against the oracle on every row: max-abs and rel-L2."""
    g, r = O_gpu, O_ref
    err = np.abs(g - r)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    assert max_abs <= O_MAX_ABS, f"max-abs {max_abs}"
    assert rel_l2 <= O_REL_L2, f"rel-L2 {rel_l2}"
    return max_abs, rel_l2


def check_stages(buf, ref, b, h, pb):
    """Pools, anchor, summaries and bias of one (b, h) slice vs the oracle."""
    np.testing.assert_allclose(host(buf["qpool"][b, h]), ref["qpool"], rtol=POOL_RTOL, atol=POOL_ATOL)
    np.testing.assert_allclose(host(buf["kpool"][b, h]), ref["kpool"], rtol=POOL_RTOL, atol=POOL_ATOL)
    np.testing.assert_allclose(host(buf["anchor"][b, h]), ref["anchor"], rtol=POOL_RTOL,
                               atol=POOL_ATOL)
    v = slice(pb, None)  # summaries of prefix blocks are never used
    np.testing.assert_allclose(host(buf["ksum"][b, h])[v], ref["ksum"][v], rtol=SUM_RTOL, atol=SUM_ATOL)
    np.testing.assert_allclose(host(buf["vsum"][b, h])[v], ref["vsum"][v], rtol=SUM_RTOL, atol=SUM_ATOL)
    d = ref["ksum"].shape[1]
    kabs = np.abs(ref["ksum"][v])
    bias_tol = BF16_U * (kabs @ np.abs(ref["anchor"])) / np.sqrt(d) + FP32_SLACK
    bias_err = np.abs(host(buf["bias"][b, h])[v] - ref["bias"][v])
    assert (bias_err <= bias_tol).all(), f"bias err {bias_err.max()} > {bias_tol.min()}"


def check_lse_bound(lse_gpu, Qh, ref, lse_ref, pb, variant, N):
    """lse within the bound the bf16 summary keys allow (oracle values only),
    on every row."""
    d = ref["ksum"].shape[1]
    kabs = np.abs(ref["ksum"][pb:])
    # anchor variant: the shift is (q - qbar) . delta; mean variant: q . delta
    centre = ref["anchor"][None, :] if variant == "anchor" else 0.0
    qd = np.abs(Qh - centre)
    lse_tol = BF16_U * (qd @ kabs.T).max(axis=1) / np.sqrt(d) + FP32_SLACK \
        if kabs.size else np.full(N, FP32_SLACK)
    lse_err = np.abs(lse_gpu - lse_ref)
    assert lse_err.shape == (N,)
    assert (lse_err <= lse_tol).all(), f"lse err {lse_err.max()} (bound {lse_tol.min()})"


def gpu_lists(idx_rows, cnt_row):
    """The GPU's block lists of one head (rows already validated)."""
    return [np.array([int(v) for v in idx_rows[i, :int(cnt_row[i])]], dtype=np.int64)
            for i in range(len(cnt_row))]


def check_head(buf, Q, K, V, b, h, top_k, prefix, variant, check_lse=True):
    """Full per-stage parity of one (b, h) slice; returns (max_abs, rel_l2, swaps).

    A query block whose GPU list differs from the oracle's by a permitted
    near-tie swap is not left out: the oracle recomputes its attention over
    the GPU's list (same summaries and biases), and O and lse are then
    compared on every row."""
    N = Q.shape[2]
    Qh, Kh, Vh = host(Q[b, h]), host(K[b, h]), host(V[b, h])
    ref = orc.forward_head(Qh, Kh, Vh, top_k, prefix, variant)
    pb = prefix // 128
    check_stages(buf, ref, b, h, pb)
    idx_rows, cnt_row = host(buf["idx"][b, h]), host(buf["cnt"][b, h])
    swaps = check_selection(idx_rows, cnt_row, ref, pb, top_k)
    O_ref, lse_ref = ref["O"], ref["lse"]
    if swaps:
        O_sw, lse_sw = orc.attend(Qh, Kh, Vh, gpu_lists(idx_rows, cnt_row), ref["ksum"],
                                  ref["vsum"], ref["bias"], pb, query_blocks=swaps)
        rows = rows_of_blocks(N, swaps)
        O_ref, lse_ref = O_ref.copy(), lse_ref.copy()
        O_ref[rows], lse_ref[rows] = O_sw[rows], lse_sw[rows]
    m, r = check_output(host(buf["O"][b, h]), O_ref, N)
    if check_lse and buf.get("lse") is not None:
        check_lse_bound(host(buf["lse"][b, h]), Qh, ref, lse_ref, pb, variant, N)
    return m, r, swaps


# ------------------------------------------------------------ threshold lists

# Band around a row's threshold (logit scale) inside which the GPU's fp32
# statistic may decide a block either way: the fp32 scores are within ~1e-5 of
# the fp64 ones (the top-k tie gap), and the mean and deviation add errors of
# the same order times tau.
THRESH_BAND = 1e-4


def check_threshold_selection(idx_rows, cnt_row, S, tau, pb):
    """GPU lists of one head vs the threshold oracle.  Returns the GPU's lists
    (each checked for validity) and the rows where they differ from the
    oracle's, which is allowed only for blocks within THRESH_BAND of the row's
    threshold, or, where the oracle fell back to the top block, for a GPU top
    block within the top-k tie gap of the row maximum."""
    from oracle import bsa_oracle_threshold as th
    nb = S.shape[0]
    want_lists = th.select_blocks_threshold(S, tau, pb)
    cand = np.arange(pb, nb)
    got_lists, differ = [], set()
    for i in range(nb):
        c = int(cnt_row[i])
        assert 1 <= c <= nb, (i, c)
        got = [int(v) for v in idx_rows[i, :c]]
        assert all(int(v) == -1 for v in idx_rows[i, c:]), f"padding of row {i}"
        got_lists.append(np.array(got, dtype=np.int64))
        want = [int(v) for v in want_lists[i]]
        if got == want:
            continue
        assert i >= pb, f"prefix row {i} differs"
        assert got[:pb] == list(range(pb))
        assert got == sorted(set(got)) and all(pb <= j < nb for j in got[pb:]), i
        row = S[i, cand]
        mu, margin = th.row_threshold(row, tau)
        floor = not np.any(row - mu >= margin) and row.max() != row.min()
        if floor and len(got) == pb + 1 and S[i, got[-1]] >= row.max() - TIE_GAP:
            differ.add(i)
            continue
        for j in set(got) ^ set(want):
            assert abs(S[i, j] - mu - margin) <= THRESH_BAND, (i, j, S[i, j] - mu - margin)
        differ.add(i)
    return got_lists, differ


def run_stages_threshold(Q, K, V, tau, prefix, variant, with_lse=True):
    """The threshold path stage by stage through its C entry points."""
    B, H, N, _ = Q.shape
    p = bsa.params(B, H, N, 1, prefix, variant)
    buf = bsa.stage_buffers(B, H, N, 1, prefix, variant, device=Q.device)
    nb = bsa.bsa_num_blocks(p)
    buf["idx"] = torch.empty(B, H, nb, bsa.bsa_threshold_capacity(p), dtype=torch.int32,
                             device=Q.device)
    bsa.bsa_pool(p, Q, buf["qpool"], buf["anchor"])
    bsa.bsa_summarize(p, K, V, buf["anchor"], buf["kpool"], buf["ksum"], buf["vsum"], buf["bias"])
    bsa.bsa_select_threshold(p, tau, buf["qpool"], buf["kpool"], buf["idx"], buf["cnt"])
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if with_lse else None
    ws = torch.empty(bsa.bsa_attend_lists_workspace_bytes(p), dtype=torch.uint8, device=Q.device)
    bsa.bsa_attend_lists(p, Q, K, V, buf["idx"], buf["cnt"], buf["ksum"], buf["vsum"],
                         buf["bias"], O, lse, ws)
    torch.cuda.synchronize()
    buf["O"] = O
    buf["lse"] = lse
    return buf


def check_head_threshold(buf, Q, K, V, b, h, tau, prefix, variant, check_lse=True):
    """Per-stage parity of one (b, h) slice of the threshold path: stages and
    lists against the oracle, then O and lse against the oracle's attention
    over the GPU's (validated) lists.  Returns (max_abs, rel_l2, rows that
    differ, kept video blocks per row)."""
    from oracle import bsa_oracle_threshold as th
    N = Q.shape[2]
    Qh, Kh, Vh = host(Q[b, h]), host(K[b, h]), host(V[b, h])
    ref = th.forward_head_threshold(Qh, Kh, Vh, tau, prefix, variant, query_blocks=set())
    pb = prefix // 128
    check_stages(buf, ref, b, h, pb)
    lists, differ = check_threshold_selection(host(buf["idx"][b, h]), host(buf["cnt"][b, h]),
                                              ref["scores"], tau, pb)
    O_ref, lse_ref = orc.attend(Qh, Kh, Vh, lists, ref["ksum"], ref["vsum"], ref["bias"], pb)
    m, r = check_output(host(buf["O"][b, h]), O_ref, N)
    if check_lse and buf.get("lse") is not None:
        check_lse_bound(host(buf["lse"][b, h]), Qh, ref, lse_ref, pb, variant, N)
    kept = np.array([len(l) - pb for l in lists[pb:]])
    return m, r, differ, kept


# ------------------------------------------------------------ extra tokens

# Ordering slack of the token scores the GPU ranks: qhat enters the tensor
# cores as bf16 hi + lo (each component within 2^-18 of qhat) and the 256
# products of a score accumulate in fp32, so a GPU score is within
# (2^-18 + 2^-16) * sum_d |qhat_d k_ud| of the exact dot product; divided by
# sqrt(d) on the oracle's scale.  2^-15 covers both terms.
EXTRA_GAP_REL = 2.0 ** -15


def run_stages_extra(Q, K, V, top_k, n_extra, prefix, variant, with_lse=True):
    """The extra-token path stage by stage through its C entry points."""
    B, H, N, _ = Q.shape
    p = bsa.params(B, H, N, top_k, prefix, variant)
    buf = bsa.stage_buffers(B, H, N, top_k, prefix, variant, device=Q.device)
    buf.update(bsa.extra_buffers(B, H, N, top_k, n_extra, prefix, variant, device=Q.device))
    bsa.bsa_pool(p, Q, buf["qpool"], buf["anchor"])
    bsa.bsa_summarize_stats(p, K, V, buf["anchor"], buf["kpool"], buf["ksum"], buf["vsum"],
                            buf["bias"], buf["kstat"], buf["vstat"], buf["lse_blk"])
    bsa.bsa_select(p, buf["qpool"], buf["kpool"], buf["idx"], buf["cnt"])
    bsa.bsa_select_extra(p, n_extra, buf["qpool"], K, buf["idx"], buf["cnt"], buf["extra"],
                         buf["ecnt"], buf["cand"])
    bsa.bsa_extra_summaries(p, n_extra, K, V, buf["anchor"], buf["kpool"], buf["kstat"],
                            buf["vstat"], buf["lse_blk"], buf["extra"], buf["ecnt"], buf["side_k"],
                            buf["side_v"], buf["side_bias"], buf["side_blk"], buf["side_cnt"])
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if with_lse else None
    bsa.bsa_attend_extra(p, n_extra, Q, K, V, buf["idx"], buf["cnt"], buf["extra"], buf["ecnt"],
                         buf["ksum"], buf["vsum"], buf["bias"], buf["side_k"], buf["side_v"],
                         buf["side_bias"], buf["side_cnt"], O, lse)
    torch.cuda.synchronize()
    buf["O"] = O
    buf["lse"] = lse
    return buf


def check_extra_selection(extra_rows, ecnt_row, s, lists, Kh, qpool, n_extra, pb, N):
    """GPU extra tokens of one head vs the oracle's choice over the same block
    lists: valid candidates, the right count, and the same set except tokens
    whose oracle scores lie within the derived ordering slack of the row's
    n-th score.  Returns the GPU's extra lists."""
    from oracle import bsa_oracle_extra as ox
    want = ox.select_extra_tokens(s, lists, pb, n_extra, N)
    bounds = orc.block_bounds(N)
    nb = len(bounds)
    absk = np.abs(Kh)
    got_all = []
    for i in range(nb):
        c = int(ecnt_row[i])
        got = [int(u) for u in extra_rows[i, :c]] if n_extra > 0 else []
        if n_extra > 0:
            assert all(int(u) == -1 for u in extra_rows[i, c:]), f"padding of row {i}"
        got_all.append(np.array(got, dtype=np.int64))
        w = [int(u) for u in want[i]]
        assert c == len(w), (i, c, len(w))
        if got == w:
            continue
        assert i >= pb, f"prefix row {i}"
        listed = set(int(j) for j in lists[i])
        assert got == sorted(set(got)), f"row {i} not ascending / unique"
        assert all(u >= pb * 128 and (u // 128) not in listed and u < N for u in got), i
        cand = np.concatenate([np.arange(*bounds[j]) for j in range(pb, nb) if j not in listed])
        nth = np.sort(s[i, cand])[::-1][len(w) - 1]
        for u in set(got) ^ set(w):
            gap = EXTRA_GAP_REL * float(np.abs(qpool[i]) @ absk[u]) / np.sqrt(Kh.shape[1]) + 1e-7
            assert abs(s[i, u] - nth) <= gap, (i, u, s[i, u], nth, gap)
    return got_all


def check_side_rows(buf, b, h, Kh, Vh, anchor, lists, extras, variant, pb, N):
    """The GPU's summary rows of partly extra blocks against the summary
    definition over the remaining tokens (the oracle's summary_of_tokens)."""
    from oracle import bsa_oracle_extra as ox
    bounds = orc.block_bounds(N)
    nb = len(bounds)
    sk, sv = host(buf["side_k"][b, h]), host(buf["side_v"][b, h])
    sb, sj, sc = host(buf["side_bias"][b, h]), host(buf["side_blk"][b, h]), host(buf["side_cnt"][b, h])
    d = Kh.shape[1]
    for i in range(nb):
        if i < pb:
            assert int(sc[i]) == 0
            continue
        ex = set(int(u) for u in extras[i])
        listed = set(int(j) for j in lists[i])
        rows = []
        for j in range(pb, nb):
            if j in listed:
                continue
            toks = np.arange(*bounds[j])
            rest = np.array([t for t in toks if t not in ex], dtype=np.int64)
            if 0 < len(rest) < len(toks):
                rows.append((j, ox.summary_of_tokens(Kh, Vh, rest, anchor, variant)))
        assert int(sc[i]) == len(rows), (i, int(sc[i]), len(rows))
        for a_, (j, (k_, v_, b_)) in enumerate(rows):
            assert int(sj[i, a_]) == j, (i, a_, int(sj[i, a_]), j)
            np.testing.assert_allclose(sk[i, a_], k_, rtol=SUM_RTOL, atol=SUM_ATOL)
            np.testing.assert_allclose(sv[i, a_], v_, rtol=SUM_RTOL, atol=SUM_ATOL)
            tol = (BF16_U * float(np.abs(k_) @ np.abs(anchor)) / np.sqrt(d) if variant == "anchor"
                   else 0.0) + FP32_SLACK
            assert abs(float(sb[i, a_]) - b_) <= tol, (i, j, float(sb[i, a_]), b_, tol)
        pad = -(-len(rows) // 128) * 128
        if pad > len(rows):
            assert np.all(sk[i, len(rows):pad] == 0) and np.all(np.isneginf(sb[i, len(rows):pad]))


def check_head_extra(buf, Q, K, V, b, h, top_k, n_extra, prefix, variant, check_lse=True,
                     query_blocks=None):
    """Per-stage parity of one (b, h) slice of the extra-token path: stages,
    lists, fp32 block statistics, the extra tokens, the side summary rows, then
    O and lse against the oracle's attention over the GPU's (validated) lists
    and extra tokens on every row (or on ``query_blocks``)."""
    from oracle import bsa_oracle_extra as ox
    N = Q.shape[2]
    Qh, Kh, Vh = host(Q[b, h]), host(K[b, h]), host(V[b, h])
    ref = ox.forward_head_extra(Qh, Kh, Vh, top_k, 0, prefix, variant, query_blocks=set())
    ref["scores"] = orc.block_scores(ref["qpool"], ref["kpool"])
    pb = prefix // 128
    check_stages(buf, ref, b, h, pb)
    idx_rows, cnt_row = host(buf["idx"][b, h]), host(buf["cnt"][b, h])
    check_selection(idx_rows, cnt_row, ref, pb, top_k)
    lists = gpu_lists(idx_rows, cnt_row)
    # fp32 block statistics (the GPU's own fp32 sums; oracle fp64)
    d = Kh.shape[1]
    v = slice(pb, None)
    np.testing.assert_allclose(host(buf["kstat"][b, h])[v], ref["ksum"][v], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(host(buf["vstat"][b, h])[v], ref["vsum"][v], rtol=1e-5, atol=1e-5)
    if variant == "anchor":
        lse_ref = ref["bias"] + ref["ksum"] @ ref["anchor"] / np.sqrt(d)
    else:
        lse_ref = np.log([hi - lo for lo, hi in orc.block_bounds(N)])
    np.testing.assert_allclose(host(buf["lse_blk"][b, h])[v], lse_ref[v], rtol=1e-5, atol=1e-5)
    s = ox.token_scores(ref["qpool"], Kh)
    extras = check_extra_selection(host(buf["extra"][b, h]), host(buf["ecnt"][b, h]), s, lists,
                                   Kh, ref["qpool"], n_extra, pb, N)
    check_side_rows(buf, b, h, Kh, Vh, ref["anchor"], lists, extras, variant, pb, N)
    O_ref, lse_r = ox.attend_extra(Qh, Kh, Vh, lists, extras, ref["ksum"], ref["vsum"],
                                   ref["bias"], ref["anchor"], variant, pb,
                                   query_blocks=query_blocks)
    O_gpu = host(buf["O"][b, h])
    rows = np.arange(N) if query_blocks is None else rows_of_blocks(N, query_blocks)
    m, r = check_output(O_gpu[rows], O_ref[rows], len(rows))
    if check_lse and buf.get("lse") is not None:
        # every summary logit (global or side row) moves by at most
        # 2^-8 * sum_d |q_d - c_d| |k~_d| / sqrt(d) through the bf16 rounding
        # of the summary key the MMA reads
        centre = ref["anchor"][None, :] if variant == "anchor" else 0.0
        sk_all, scnt = host(buf["side_k"][b, h]), host(buf["side_cnt"][b, h])
        side_rows = [sk_all[i, :int(scnt[i])] for i in range(len(scnt)) if int(scnt[i]) > 0]
        kall = np.abs(np.concatenate([ref["ksum"][pb:]] + side_rows, axis=0))
        qd = np.abs(Qh[rows] - centre)
        tol = BF16_U * (qd @ kall.T).max(axis=1) / np.sqrt(d) + FP32_SLACK
        err = np.abs(host(buf["lse"][b, h])[rows] - lse_r[rows])
        assert (err <= tol).all(), f"lse err {err.max()} (bound {tol.min()})"
    return m, r, extras
