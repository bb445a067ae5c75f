"""Seeded synthetic Q/K/V generators (the only module both the oracle tests
and the CUDA path use; it holds none of the method's arithmetic).

The pages' workload is MiniMax H3 video-DiT self-attention: 56 heads,
head_dim 128, bf16, sequence lengths H3 packs at 24 fps ("h3-sparse-attn
0.1.0", section "Measured").  No latents or weights exist here, so inputs are
synthetic with that shape and two value distributions:

* ``"iid"``: every element ~ N(0, 1).
* ``"block_offset"``: for each tensor X in {Q, K, V}, each (b, h) and each
  128-token block j an offset mu_{X,b,h,j} ~ N(0, I_d) is drawn; token t of
  block j is mu_{X,b,h,j} + 0.5 * eps_t with eps_t ~ N(0, I_d).  Neighbouring
  tokens share a block mean, as video tokens of one spatio-temporal tile do,
  so pooled block scores are structured and far apart (gaps >> 1e-5).

Each (tensor, b, h) slice has its own torch.Generator seeded with
``seed * 1_000_003 + tensor_id * 1009 + (b * H + h)`` so any head can be
regenerated alone.  The CPU and CUDA generators produce different streams;
a comparison always copies the exact bf16 tensor one side used to the other.
"""

from __future__ import annotations

import torch

BLOCK = 128
KINDS = ("iid", "block_offset")
_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


def slice_seed(seed: int, tensor: str, b: int, h: int, H: int) -> int:
    return seed * 1_000_003 + _TENSOR_ID[tensor] * 1009 + (b * H + h)


def _one_slice(N: int, d: int, kind: str, gen: torch.Generator, device) -> torch.Tensor:
    if kind == "iid":
        x = torch.randn(N, d, generator=gen, device=device, dtype=torch.float32)
    elif kind == "block_offset":
        nb = -(-N // BLOCK)
        mu = torch.randn(nb, d, generator=gen, device=device, dtype=torch.float32)
        eps = torch.randn(N, d, generator=gen, device=device, dtype=torch.float32)
        x = mu.repeat_interleave(BLOCK, dim=0)[:N] + 0.5 * eps
    else:
        raise ValueError(f"unknown input kind {kind!r}")
    return x.to(torch.bfloat16)


def make_tensor(tensor: str, B: int, H: int, N: int, d: int = 128, kind: str = "iid",
                seed: int = 0, device="cpu") -> torch.Tensor:
    """One of Q/K/V as a contiguous bf16 [B, H, N, d] tensor on ``device``."""
    out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=device)
    gen = torch.Generator(device=device)
    for b in range(B):
        for h in range(H):
            gen.manual_seed(slice_seed(seed, tensor, b, h, H))
            out[b, h] = _one_slice(N, d, kind, gen, device)
    return out


def make_qkv(B: int, H: int, N: int, d: int = 128, kind: str = "iid", seed: int = 0,
             device="cpu"):
    """(Q, K, V), each contiguous bf16 [B, H, N, d]."""
    return tuple(make_tensor(t, B, H, N, d, kind, seed, device) for t in ("q", "k", "v"))


def make_qkv_slices(B: int, H: int, N: int, start: int, count: int, d: int = 128,
                    kind: str = "iid", seed: int = 0, device="cpu"):
    """(Q, K, V) slices start .. start+count-1 (in (b, h) order) of the tensors
    ``make_qkv(B, H, N, ...)`` builds, each as a contiguous bf16
    [1, count, N, d] tensor: a rank regenerates only the heads it owns, bit
    for bit equal to the same slices of the whole tensors."""
    out = []
    for t in ("q", "k", "v"):
        x = torch.empty(1, count, N, d, dtype=torch.bfloat16, device=device)
        gen = torch.Generator(device=device)
        for i in range(count):
            b, h = divmod(start + i, H)
            gen.manual_seed(slice_seed(seed, t, b, h, H))
            x[0, i] = _one_slice(N, d, kind, gen, device)
        out.append(x)
    return tuple(out)


# The five workloads: shapes of the pages' "Measured" table (56 heads,
# head_dim 128, H3's 24 fps sequence lengths) plus a small iid case.
CONFIGS = {
    "tiny_iid": dict(B=1, H=2, N=2048, top_k=4, prefix=0, variant="mean", kind="iid"),
    "h3_768p_5s": dict(B=1, H=56, N=37_740, top_k=64, prefix=0, variant="anchor",
                       kind="block_offset"),
    "h3_768p_10s": dict(B=1, H=56, N=73_416, top_k=64, prefix=0, variant="anchor",
                        kind="block_offset"),
    "h3_768p_15s_prefix512": dict(B=1, H=56, N=103_996, top_k=64, prefix=512,
                                  variant="anchor", kind="block_offset"),
    "h3_2k_5s": dict(B=1, H=56, N=133_644, top_k=64, prefix=0, variant="anchor",
                     kind="block_offset"),
}
