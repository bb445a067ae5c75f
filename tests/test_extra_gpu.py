"""GPU parity of the extra-token path (the `extra_tokens` input of the WAS
node page, "H3 Sparse Attention", section "The inputs that matter"), through
the C ABI, against the extra-token oracle.

The GPU ranks token scores computed on the tensor cores (qhat as bf16 hi + lo,
fp32 accumulation), so a token whose oracle score lies within the derived
ordering slack of its row's n-th score may be chosen either way; everything
else is compared exactly, every list is checked for validity, the summary rows
of partly extra blocks are compared with the summary definition over the
remaining tokens, and O and lse are compared with the oracle's attention over
the GPU's (validated) lists and extra tokens on every row."""

import random

import numpy as np
import pytest
import torch

from block_sparse_video_bsa_b200 import bsa
from block_sparse_video_bsa_b200.inputs import CONFIGS, make_qkv

from parity_util import check_head_extra, check_output, host, run_stages, run_stages_extra

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,top_k,n_extra,prefix,variant,kind", [
    (1, 2, 1000, 3, 100, 0, "anchor", "block_offset"),      # ragged tail, one partial extra tile
    (1, 2, 2048, 4, 256, 0, "mean", "iid"),                 # the small iid shape, mean variant
    (2, 1, 1500, 2, 300, 256, "anchor", "block_offset"),    # dense prefix, three extra tiles
    (1, 2, 4100, 5, 512, 0, "anchor", "block_offset"),      # the largest count, ragged tail of 4
    (1, 1, 17_000, 7, 256, 0, "anchor", "block_offset"),    # 133 blocks: two summary tiles
    (1, 2, 1500, 2, 128, 256, "mean", "block_offset"),
    (1, 1, 300, 1, 1, 0, "anchor", "iid"),                  # a single extra token
])
def test_small_cases_all_stages(B, H, N, top_k, n_extra, prefix, variant, kind):
    Q, K, V = make_qkv(B, H, N, 128, kind, seed=3, device="cuda")
    buf = run_stages_extra(Q, K, V, top_k, n_extra, prefix, variant)
    for b in range(B):
        for h in range(H):
            check_head_extra(buf, Q, K, V, b, h, top_k, n_extra, prefix, variant)


@pytest.mark.parametrize("N,prefix,variant", [(1000, 0, "anchor"), (1500, 256, "mean"),
                                              (129, 0, "anchor"), (1, 0, "anchor")])
def test_no_extra_tokens_is_the_top_k_path_bit_for_bit(N, prefix, variant):
    Q, K, V = make_qkv(1, 3, N, 128, "block_offset", seed=5, device="cuda")
    O0, l0 = bsa.forward(Q, K, V, 2, prefix, variant, return_lse=True)
    O1, l1 = bsa.forward_extra(Q, K, V, 2, 0, prefix, variant, return_lse=True)
    buf = run_stages_extra(Q, K, V, 2, 0, prefix, variant)
    torch.cuda.synchronize()
    assert torch.equal(O0, O1) and torch.equal(l0, l1)
    assert torch.equal(O0, buf["O"]) and torch.equal(l0, buf["lse"])
    assert int(buf["ecnt"].abs().sum()) == 0 and int(buf["side_cnt"].abs().sum()) == 0


@pytest.mark.parametrize("N,top_k,prefix", [(700, 2, 0), (800, 1, 256)])
def test_extra_tokens_covering_every_candidate_give_dense_attention(N, top_k, prefix):
    # every unlisted token becomes extra: no summary row is left, the row is dense
    Q, K, V = make_qkv(1, 2, N, 128, "block_offset", seed=7, device="cuda")
    O = bsa.forward_extra(Q, K, V, top_k, 512, prefix)
    buf = run_stages_extra(Q, K, V, top_k, 512, prefix, "anchor")
    torch.cuda.synchronize()
    assert torch.equal(O, buf["O"])
    assert int(buf["side_cnt"].abs().sum()) == 0
    dense = torch.nn.functional.scaled_dot_product_attention(Q.float(), K.float(), V.float())
    assert (O.float() - dense).abs().max().item() <= 2e-2
    for h in range(2):
        check_head_extra(buf, Q, K, V, 0, h, top_k, 512, prefix, "anchor")


def test_forward_extra_matches_stages_and_is_deterministic():
    N, top_k, n_extra = 3000, 4, 256
    Q, K, V = make_qkv(1, 4, N, 128, "block_offset", seed=9, device="cuda")
    buf = run_stages_extra(Q, K, V, top_k, n_extra, 0, "anchor")
    O1, l1 = bsa.forward_extra(Q, K, V, top_k, n_extra, return_lse=True)
    O2, l2 = bsa.forward_extra(Q, K, V, top_k, n_extra, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(O1, buf["O"]) and torch.equal(O1, O2)
    assert torch.equal(l1, buf["lse"]) and torch.equal(l1, l2)


def test_extra_tokens_change_the_output_where_they_should():
    # the rows read their extra tokens exactly: the output moves away from the
    # top-k path's
    N = 2048
    Q, K, V = make_qkv(1, 1, N, 128, "block_offset", seed=11, device="cuda")
    O0 = bsa.forward(Q, K, V, 3)
    O1 = bsa.forward_extra(Q, K, V, 3, 256)
    torch.cuda.synchronize()
    assert (O0.float() - O1.float()).abs().max().item() > 1e-3


def test_full_size_768p_sampled_head_and_query_blocks():
    # The 768p-5s workload with the page's default of 256 extra tokens, in the
    # launch configuration of the whole call; one seeded head checked stage by
    # stage, its attention on 24 seeded query blocks.
    cfg = CONFIGS["h3_768p_5s"]
    B, H, N = cfg["B"], cfg["H"], cfg["N"]
    Q, K, V = make_qkv(B, H, N, 128, cfg["kind"], 0, device="cuda")
    n_extra = 256
    O = bsa.forward_extra(Q, K, V, cfg["top_k"], n_extra, cfg["prefix"], cfg["variant"])
    buf = run_stages_extra(Q, K, V, cfg["top_k"], n_extra, cfg["prefix"], cfg["variant"])
    torch.cuda.synchronize()
    assert torch.equal(O, buf["O"])
    h = random.Random(2).randrange(H)
    nb = -(-N // 128)
    qb = set(random.Random(3).sample(range(nb), 24)) | {nb - 1}
    _, _, extras = check_head_extra(buf, Q, K, V, 0, h, cfg["top_k"], n_extra, cfg["prefix"],
                                    cfg["variant"], query_blocks=qb)
    assert all(len(e) == n_extra for e in extras)
    del Q, K, V, O, buf
    torch.cuda.empty_cache()
