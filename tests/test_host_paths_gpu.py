"""The host-buffer forwards of the options (FP8, threshold selection, extra
tokens, adaptive reblocking): pipelined over chunks of (b, h) slices, they must give the same O
and lse, bit for bit, as the device-buffer forward of the same option."""

import pytest
import torch

from block_sparse_video_bsa_b200 import bsa
from block_sparse_video_bsa_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

B, H, N, TOP_K, PREFIX = 1, 10, 2500, 3, 256     # 8 chunks, the last ones of one slice


def _host_run(fn, ws_bytes, Q, K, V, *lead):
    p = bsa.params(B, H, N, TOP_K, PREFIX)
    ws = torch.empty(ws_bytes(p), dtype=torch.uint8, device="cuda")
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    hO = torch.empty_like(hQ).pin_memory()
    hl = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
    dQ, dK, dV, dO = (torch.empty_like(Q) for _ in range(4))
    dl = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    fn(p, *lead, hQ, hK, hV, hO, hl, dQ, dK, dV, dO, dl, ws)
    torch.cuda.synchronize()
    return hO, hl


def test_fp8_host_forward_matches_device_forward():
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", seed=21, device="cuda")
    hO, hl = _host_run(bsa.bsa_forward_fp8_host, bsa.bsa_forward_fp8_workspace_bytes, Q, K, V)
    O, lse = bsa.forward_fp8(Q, K, V, TOP_K, PREFIX, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(hO, O.cpu()) and torch.equal(hl, lse.cpu())


def test_threshold_host_forward_matches_device_forward():
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", seed=22, device="cuda")
    hO, hl = _host_run(bsa.bsa_forward_threshold_host, bsa.bsa_forward_threshold_workspace_bytes,
                       Q, K, V, 1.0)
    O, lse = bsa.forward_threshold(Q, K, V, 1.0, PREFIX, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(hO, O.cpu()) and torch.equal(hl, lse.cpu())


def test_extra_host_forward_matches_device_forward():
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", seed=23, device="cuda")
    hO, hl = _host_run(bsa.bsa_forward_extra_host,
                       lambda p: bsa.bsa_forward_extra_workspace_bytes(p, 200), Q, K, V, 200)
    O, lse = bsa.forward_extra(Q, K, V, TOP_K, 200, PREFIX, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(hO, O.cpu()) and torch.equal(hl, lse.cpu())


def test_reblock_host_forward_matches_device_forward():
    Q, K, V = make_qkv(B, H, N, 128, "block_offset", seed=24, device="cuda")
    hO, hl = _host_run(bsa.bsa_forward_reblock_host, bsa.bsa_forward_reblock_workspace_bytes,
                       Q, K, V)
    O, lse = bsa.forward_reblock(Q, K, V, TOP_K, PREFIX, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(hO, O.cpu()) and torch.equal(hl, lse.cpu())
