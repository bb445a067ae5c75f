"""The C ABI without a GPU: libbsa.so loads, exports every function that
include/bsa.h declares, and the host-side checks (sizes, bad arguments) that
run before any CUDA call behave as documented.  No compute call here touches
the device: every call below returns from argument validation."""

import ctypes

import pytest

from block_sparse_video_bsa_b200 import bsa


@pytest.fixture(scope="module")
def L():
    return bsa.lib()


def test_exports_every_declared_symbol(L):
    names = bsa.header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(bsa._SIGS), "binding and header disagree"


def _p(**kw):
    base = dict(B=1, H=56, N=37_740, top_k=64, prefix=0, variant="anchor")
    base.update(kw)
    return bsa.params(**base)


def test_sizes_match_the_block_arithmetic():
    p = _p()
    assert bsa.bsa_num_blocks(p) == 295
    assert bsa.bsa_select_capacity(p) == 64
    assert bsa.bsa_select_capacity(_p(N=103_996, prefix=512)) == 813
    assert bsa.bsa_select_capacity(_p(top_k=1000)) == 295       # clamped to nbv
    assert bsa.bsa_num_blocks(_p(N=1)) == 1
    ws = bsa.bsa_workspace_bytes(p)
    blocks = 56 * 295
    want = blocks * 128 * 4 * 2 + 56 * 128 * 4 + blocks * 128 * 2 * 2 + blocks * 4 \
        + blocks * 64 * 4 + blocks * 4
    assert want <= ws <= want + 8 * 256


@pytest.mark.parametrize("kw", [dict(D=64), dict(top_k=0), dict(prefix=100), dict(prefix=37_760),
                                dict(N=0), dict(B=0), dict(variant=7), dict(N=(1 << 21) + 1),
                                dict(H=70_000)])
def test_invalid_parameters_rejected_before_launch(kw):
    p = _p(**kw)
    assert bsa.bsa_num_blocks(p) == -1
    assert bsa.bsa_workspace_bytes(p) == 0
    rc = bsa.lib().bsa_pool(ctypes.byref(p), ctypes.c_void_p(4096), ctypes.c_void_p(4096),
                            ctypes.c_void_p(4096), None)
    assert rc == bsa.BSA_ERR_INVALID


def test_null_and_misaligned_pointers_rejected_before_launch():
    L = bsa.lib()
    p = _p()
    P = ctypes.byref(p)
    a = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.bsa_pool(P, None, a, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_pool(P, odd, a, a, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_summarize(P, a, a, None, a, a, a, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_select(P, a, a, None, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_attend(P, a, a, a, a, a, a, a, a, None, None, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_attend(P, a, a, a, a, a, a, a, a, odd, None, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_forward(P, a, a, a, a, None, a, 16, None) == bsa.BSA_ERR_INVALID  # too small
    assert L.bsa_forward(P, a, a, a, a, None, odd, 1 << 40, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_forward_host(P, a, a, a, a, None, a, a, a, None, None, a, 1 << 40,
                              None) == bsa.BSA_ERR_INVALID
    assert L.bsa_debug_expired_wait(None, 1000, None) == bsa.BSA_ERR_INVALID
    # The mean variant does not need an anchor, the anchor variant does.  The
    # mean-variant call passes the null-anchor check and is then stopped by a
    # misaligned bias, so it never reaches the device even on a GPU machine.
    pm = _p(variant="mean")
    bias_odd = ctypes.c_void_p((1 << 20) + 2)
    assert L.bsa_summarize(ctypes.byref(pm), a, a, None, a, a, a, bias_odd, None) == \
        bsa.BSA_ERR_ALIGN
    assert L.bsa_summarize(P, a, a, None, a, a, a, bias_odd, None) == bsa.BSA_ERR_INVALID


def test_status_strings():
    assert bsa.status_string(bsa.BSA_OK) == "ok"
    assert "aligned" in bsa.status_string(bsa.BSA_ERR_ALIGN)
    assert bsa.status_string(99) == "unknown status"


def test_density_to_topk_rounds_up():
    assert [bsa.topk_from_density(r, 133_644) for r in (0.1, 0.2, 0.3)] == [105, 209, 314]
    assert bsa.topk_from_density(0.3, 128_000) == 300
    assert bsa.topk_from_density(0.001, 2048) == 1


def test_option_sizes():
    # reblocking scratch and the FP8 operand set follow the documented layouts
    p = _p()
    bh, N, nb = 56, 37_740, 295
    ops = bsa.bsa_fp8_operands_bytes(p)
    codes = bh * N * 128 * 2 + bh * nb * 128 * 128 + bh * nb * 128 + bh * 3 * 128 * 128
    scales = (3 * bh * nb + 2 * bh * 3 + bh) * 4
    assert codes + scales <= ops <= codes + scales + 11 * 256
    assert bsa.bsa_forward_fp8_workspace_bytes(p) == bsa.bsa_workspace_bytes(p) + ops
    rb = bsa.bsa_reblock_workspace_bytes(p)
    assert rb >= bh * (N - 0) * 128 * 2 + bh * N * 4      # bf16 whitened queries + a permutation
    frb = bsa.bsa_forward_reblock_workspace_bytes(p)
    assert frb >= rb + bsa.bsa_workspace_bytes(p) + 4 * bh * N * 256
    for f in (bsa.bsa_fp8_operands_bytes, bsa.bsa_reblock_workspace_bytes,
              bsa.bsa_forward_reblock_workspace_bytes, bsa.bsa_forward_fp8_workspace_bytes):
        assert f(_p(top_k=0)) == 0


def test_option_arguments_rejected_before_launch():
    L = bsa.lib()
    p = _p()
    P = ctypes.byref(p)
    a = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    # reblocking
    assert L.bsa_reblock(P, a, a, None, a, 1 << 40, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_reblock(P, a, a, a, a, 16, None) == bsa.BSA_ERR_INVALID      # scratch too small
    assert L.bsa_reblock(P, odd, a, a, a, 1 << 40, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_permute(P, a, a, a, None, a, a, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_pool_permuted(P, a, None, a, a, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_pool_permuted(P, a, a, odd, a, a, None) == bsa.BSA_ERR_ALIGN       # Qp
    assert L.bsa_summarize_permuted(P, a, a, None, a, a, a, a, a, a, a, None) == \
        bsa.BSA_ERR_INVALID
    assert L.bsa_summarize_permuted(P, a, a, a, a, odd, a, a, a, a, a, None) == \
        bsa.BSA_ERR_ALIGN                                                             # Vp
    assert L.bsa_unpermute(P, a, None, a, a, a, None) == bsa.BSA_ERR_INVALID   # lse without lsep
    assert L.bsa_forward_reblock(P, a, a, a, a, None, a, 16, None) == bsa.BSA_ERR_INVALID
    # FP8
    ops = bsa.bsa_fp8_operands()
    assert L.bsa_quantize_fp8(P, a, a, a, a, a, ctypes.byref(ops), None) == bsa.BSA_ERR_INVALID
    assert L.bsa_attend_fp8(P, ctypes.byref(ops), a, a, a, a, None, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_fp8_operands_carve(P, a, 16, ctypes.byref(ops)) == bsa.BSA_ERR_INVALID
    assert L.bsa_fp8_operands_carve(P, odd, 1 << 40, ctypes.byref(ops)) == bsa.BSA_ERR_ALIGN
    assert L.bsa_forward_fp8(P, a, a, a, a, None, a, 16, None) == bsa.BSA_ERR_INVALID


def test_fp8_operands_carve_follows_the_field_order():
    # carving needs no device: it only computes pointers into the caller's buffer
    L = bsa.lib()
    p = _p(N=1000, H=2)
    n = bsa.bsa_fp8_operands_bytes(p)
    base = 1 << 32
    ops = bsa.bsa_fp8_operands()
    assert L.bsa_fp8_operands_carve(ctypes.byref(p), ctypes.c_void_p(base), n,
                                    ctypes.byref(ops)) == bsa.BSA_OK
    ptrs = [getattr(ops, f) for f, _ in bsa.bsa_fp8_operands._fields_]
    assert ptrs[0] == base and all(b > a for a, b in zip(ptrs, ptrs[1:]))
    assert all(x % 256 == 0 for x in ptrs) and ptrs[-1] < base + n


def _reblock_scratch(B, H, N, prefix):
    """Bytes of the reblocking scratch from the tree's shape (independent
    replica of the plan: levels, chunk counts of the largest group, partial
    slots), each piece rounded to 256 bytes."""
    r256 = lambda x: (x + 255) // 256 * 256
    nv, bh = N - prefix, B * H
    levels = 0
    while (128 << levels) < nv:
        levels += 1
    moment_chunks = -(-nv // 2048)
    maxp, largest = 1, nv
    for l in range(levels):
        chunks = -(-largest // 2048)
        if chunks > 1:
            maxp = max(maxp, (1 << l) * chunks)
        largest -= (-(-largest // 128) // 2) * 128
    maxp = max(maxp, moment_chunks)
    return sum(r256(x) for x in (bh * N * 4, bh * maxp * 128 * 128 * 4, bh * maxp * 128 * 4,
                                 bh * (1 << levels) * 128 * 4, bh * 128 * 128 * 4,
                                 bh * 128 * 128 * 2, bh * 128 * 128 * 2, bh * nv * 128 * 2,
                                 bh * nv * 4))


@pytest.mark.parametrize("B,H,N,prefix", [(1, 56, 37_740, 0), (1, 56, 133_644, 0),
                                          (1, 56, 103_996, 512), (2, 3, 4100, 0), (1, 1, 129, 0),
                                          (1, 1, 128, 0), (1, 2, 2049, 0), (1, 1, 1, 0)])
def test_reblock_scratch_follows_the_tree_shape(B, H, N, prefix):
    p = bsa.params(B, H, N, 1, prefix)
    assert bsa.bsa_reblock_workspace_bytes(p) == _reblock_scratch(B, H, N, prefix)


def test_threshold_sizes():
    # lists of up to nb blocks; the schedule holds one int per video query
    # block
    p = _p()
    bh, nb = 56, 295
    assert bsa.bsa_threshold_capacity(p) == nb
    assert bsa.bsa_threshold_capacity(_p(top_k=0)) == -1
    r256 = lambda x: (x + 255) // 256 * 256
    assert bsa.bsa_attend_lists_workspace_bytes(p) == bh * nb * 4
    pp = _p(N=103_996, prefix=512)
    assert bsa.bsa_attend_lists_workspace_bytes(pp) == bh * 809 * 4
    fw = bsa.bsa_forward_threshold_workspace_bytes(p)
    fixed = bsa.bsa_workspace_bytes(p)             # idx rows of 64 there, of 295 here
    assert fw - bsa.bsa_attend_lists_workspace_bytes(p) - fixed == \
        r256(bh * nb * nb * 4) - r256(bh * nb * 64 * 4)


def test_threshold_arguments_rejected_before_launch():
    L = bsa.lib()
    p = _p()
    P = ctypes.byref(p)
    a = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 40
    for tau in (float("nan"), float("inf"), float("-inf")):
        assert L.bsa_select_threshold(P, tau, a, a, a, a, None) == bsa.BSA_ERR_INVALID
        assert L.bsa_forward_threshold(P, tau, a, a, a, a, None, a, big, None) == \
            bsa.BSA_ERR_INVALID
    assert L.bsa_select_threshold(P, 1.0, a, a, None, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_select_threshold(P, 1.0, odd, a, a, a, None) == bsa.BSA_ERR_ALIGN
    args = lambda kcap, ws=big, o=a, w=a: (P, a, a, a, a, kcap, a, a, a, a, o, None, w, ws, None)
    assert L.bsa_attend_lists(*args(0)) == bsa.BSA_ERR_INVALID          # empty rows
    assert L.bsa_attend_lists(*args(296)) == bsa.BSA_ERR_INVALID        # wider than nb
    assert L.bsa_attend_lists(*args(295, ws=16)) == bsa.BSA_ERR_INVALID  # schedule too small
    assert L.bsa_attend_lists(*args(295, o=odd)) == bsa.BSA_ERR_ALIGN
    assert L.bsa_attend_lists(*args(295, w=odd)) == bsa.BSA_ERR_ALIGN
    # with a dense prefix the rows must hold all nb blocks
    pp = _p(N=103_996, prefix=512)
    assert L.bsa_attend_lists(ctypes.byref(pp), a, a, a, a, 812, a, a, a, a, a, None, a, big,
                              None) == bsa.BSA_ERR_INVALID
    assert L.bsa_forward_threshold(P, 1.0, a, a, a, a, None, a, 16, None) == bsa.BSA_ERR_INVALID


def test_extra_token_sizes():
    # side rows: min(n_extra, nbv) rounded up to 128; two candidate buffers
    # (token halves) of 768 keys per video query block up to 256 extra
    # tokens, 2048 above
    p = _p()
    bh, nb = 56, 295
    assert bsa.bsa_extra_side_capacity(p, 256) == 256
    assert bsa.bsa_extra_side_capacity(p, 100) == 128
    assert bsa.bsa_extra_side_capacity(p, 0) == 0
    assert bsa.bsa_extra_side_capacity(bsa.params(1, 1, 1000, 3), 300) == 128   # nbv = 8
    assert bsa.bsa_extra_side_capacity(p, 513) == -1 and bsa.bsa_extra_side_capacity(p, -1) == -1
    assert bsa.bsa_select_extra_workspace_bytes(p, 256) == 2 * bh * nb * (768 * 8 + 4)
    assert bsa.bsa_select_extra_workspace_bytes(p, 257) == 2 * bh * nb * (2048 * 8 + 4)
    assert bsa.bsa_select_extra_workspace_bytes(p, 0) == 0
    r256 = lambda x: (x + 255) // 256 * 256
    blocks = bh * nb
    want = sum(r256(x) for x in (blocks * 512, blocks * 512, blocks * 4, blocks * 256 * 4,
                                 blocks * 4, blocks * 256 * 256, blocks * 256 * 256,
                                 blocks * 256 * 4, blocks * 256 * 4, blocks * 4,
                                 2 * blocks * (768 * 8 + 4)))
    assert bsa.bsa_forward_extra_workspace_bytes(p, 256) == bsa.bsa_workspace_bytes(p) + want
    # the row gathers use 32-bit row coordinates
    assert bsa.bsa_forward_extra_workspace_bytes(bsa.params(64, 16, 1 << 21, 64), 256) == 0


def test_extra_token_arguments_rejected_before_launch():
    L = bsa.lib()
    p = _p()
    P = ctypes.byref(p)
    a = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 40
    for n in (-1, 513):
        assert L.bsa_select_extra(P, n, a, a, a, a, a, a, a, big, None) == bsa.BSA_ERR_INVALID
        assert L.bsa_forward_extra(P, n, a, a, a, a, None, a, big, None) == bsa.BSA_ERR_INVALID
        assert L.bsa_attend_extra(P, n, *([a] * 14), a, None, None) == bsa.BSA_ERR_INVALID
        assert L.bsa_extra_summaries(P, n, *([a] * 14), None) == bsa.BSA_ERR_INVALID
    assert L.bsa_select_extra(P, 256, a, a, a, a, a, a, a, 16, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_select_extra(P, 256, a, a, a, a, None, a, a, big, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_select_extra(P, 256, odd, a, a, a, a, a, a, big, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_select_extra(P, 256, a, a, a, a, a, a, odd, big, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_forward_extra(P, 256, a, a, a, a, None, a, 16, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_forward_extra(P, 256, a, a, a, odd, None, a, big, None) == bsa.BSA_ERR_ALIGN
    # the anchor variant needs the anchor; the side table needs 16-byte rows
    args = [a] * 14
    args[2] = None
    assert L.bsa_extra_summaries(P, 256, *args, None) == bsa.BSA_ERR_INVALID
    args = [a] * 14
    args[9] = odd
    assert L.bsa_extra_summaries(P, 256, *args, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_attend_extra(P, 256, *([a] * 14), odd, None, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_summarize_stats(P, a, a, a, a, a, a, a, None, a, a, None) == bsa.BSA_ERR_INVALID
    assert L.bsa_summarize_stats(P, a, a, a, a, a, a, a, odd, a, a, None) == bsa.BSA_ERR_ALIGN
