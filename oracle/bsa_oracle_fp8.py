"""FP8 (e4m3) operands for the exact and compressed branch: the oracle.

TEST INFRASTRUCTURE ONLY, under the same rules as ``bsa_oracle.py``: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import it.  It shares no code with the CUDA path.

Where it comes from.  The pages speak of a quantised sparse kernel: "H3 Sparse
Attention" (comfy.icu, WAS node), section "What it actually does": inside the
kernel the sparse layers compute in INT8, and that quantisation is where the
softness comes from.  They give no format, granularity or rounding.  Every
choice below is a READING of this project (the FP8 row of its scope table):

* Format: OCP FP8 e4m3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
  bits; largest finite value 448; subnormal spacing 2^-9), round to nearest
  with ties to the even mantissa, saturating at +-448.
* Granularity: one scale per 128-token block of Q, K and V (real rows of a
  ragged block only) and one per 128-row tile of the summary tables.
* Codes of a group with largest magnitude amax: round_e4m3(x * r) with
  r = fp32(448 / amax), x and the product in fp32 (one rounding each); the
  dequantisation scale is fp32(amax / 448).  An all-zero group has r = 1 and
  scale 1.
* The summary tables quantised are the bf16-rounded k~ and v~ rows the bf16
  path feeds its tensor cores.  Pooling, the summaries' bias and the block
  selection are the bf16 path's, unchanged.
* The output is the bf16 path's attention (``bsa_oracle.attend``) on the
  dequantised operands.  The kernel additionally rounds its softmax
  numerators to e4m3; that is an approximation which the parity tests bound
  (it is not part of the definition).

Pinned by tests/test_oracle_fp8_pins.py (hand-computed e4m3 values, a
brute-force search over all e4m3 codes built from the bit layout, torch's own
float8_e4m3fn cast, exact round trips of representable inputs).
"""

from __future__ import annotations

import numpy as np

from .bsa_oracle import (BLOCK, attend, block_bounds, block_scores, block_summaries,
                         pooled_means, select_blocks, video_query_anchor)

E4M3_MAX = 448.0


def round_e4m3(x) -> np.ndarray:
    """Nearest e4m3 value (ties to the even mantissa), saturating at +-448.

    A normal e4m3 number with binade exponent e (-6 <= e <= 8) has spacing
    2^(e-3); below 2^-6 the subnormals have spacing 2^-9.  ``np.round`` rounds
    halves to even, and every quotient a / spacing below is exact in fp64.
    """
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.minimum(a, E4M3_MAX)
    _, ex = np.frexp(a)                     # a = m * 2^ex, m in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)              # binade exponent (subnormals use -6)
    step = np.ldexp(1.0, e - 3)
    q = np.round(a / step) * step
    return np.copysign(q, np.asarray(x, dtype=np.float64))


def quantize_group(X):
    """Codes (as values) and scale of one quantisation group (READING above)."""
    x = np.asarray(X, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    if amax == 0:
        ratio, scale = np.float32(1), np.float32(1)
    else:
        ratio = np.float32(E4M3_MAX) / amax
        scale = amax / np.float32(E4M3_MAX)
    y = (x * ratio).astype(np.float32)
    return round_e4m3(y), float(scale)


def quantize_blocks(X, block: int = BLOCK):
    """Per 128-row group of an [n, d] array: codes [n, d] (values), scales [groups]."""
    X = np.asarray(X, dtype=np.float32)
    n = X.shape[0]
    codes = np.zeros(X.shape)
    scales = []
    for a, b in block_bounds(n, block):
        c, s = quantize_group(X[a:b])
        codes[a:b] = c
        scales.append(s)
    return codes, np.array(scales)


def dequantize(codes, scales, block: int = BLOCK):
    """codes * the scale of each row's group."""
    codes = np.asarray(codes, dtype=np.float64)
    rows = np.repeat(np.asarray(scales, dtype=np.float64), block)[: codes.shape[0]]
    return codes * rows[:, None]


def bf16_round(x) -> np.ndarray:
    """Nearest bfloat16 value (ties to even) of fp64 values, as fp64.

    bfloat16 keeps 8 significant bits; numbers are finite and far from the
    bf16 range limits here.
    """
    a = np.asarray(x, dtype=np.float64)
    m, ex = np.frexp(a)                     # |m| in [0.5, 1)
    return np.ldexp(np.round(np.ldexp(m, 8)), ex - 8)


def forward_head_fp8(Q, K, V, top_k: int, prefix: int = 0, variant: str = "anchor",
                     block: int = BLOCK, query_blocks=None):
    """The FP8 path for one (batch, head) slice.

    Stages a1-a4 as in the bf16 path; then every attention operand is
    quantised per group and the attention runs on the dequantised values.
    Returns the codes and scales too, so tests can compare them bit for bit.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N = Q.shape[0]
    pb = prefix // block
    qbar = video_query_anchor(Q, prefix)
    ksum, vsum, bias = block_summaries(K, V, qbar, variant, block)
    lists = select_blocks(block_scores(pooled_means(Q, block), pooled_means(K, block)), top_k, pb)
    ksum_b, vsum_b = bf16_round(ksum), bf16_round(vsum)
    qc, sq = quantize_blocks(Q, block)
    kc, sk = quantize_blocks(K, block)
    vc, sv = quantize_blocks(V, block)
    ksc, sks = quantize_blocks(ksum_b, block)
    vsc, svs = quantize_blocks(vsum_b, block)
    Qd, Kd, Vd = dequantize(qc, sq, block), dequantize(kc, sk, block), dequantize(vc, sv, block)
    KSd, VSd = dequantize(ksc, sks, block), dequantize(vsc, svs, block)
    O, lse = attend(Qd, Kd, Vd, lists, KSd, VSd, bias, pb, block, query_blocks)
    assert N == O.shape[0]
    return dict(lists=lists, bias=bias, q_codes=qc, q_scale=sq, k_codes=kc, k_scale=sk,
                v_codes=vc, v_scale=sv, ks_codes=ksc, ks_scale=sks, vs_codes=vsc,
                vs_scale=svs, Qd=Qd, Kd=Kd, Vd=Vd, KSd=KSd, VSd=VSd, O=O, lse=lse)


def weight_moves(p, r, exp_rel_err: float = 0.0):
    """Largest move of each softmax weight w = p / sum(p) (last axis) when the
    kernel rounds p * r to e4m3 (r = s_v / s_ref <= 1) after computing p with
    relative error at most ``exp_rel_err`` = e, and divides by the sum of its
    own numerators: max(rho w, 2^-10 / (r l (1 - e)) + w 2e / (1 - e)) with
    rho = (1 + e)(1 + 2^-4) / (1 - e) - 1 and l = sum(p) (see
    fp8_output_bound for the derivation)."""
    p = np.asarray(p, dtype=np.float64)
    l = p.sum(axis=-1, keepdims=True)
    e = float(exp_rel_err)
    rho = (1 + e) * (1 + 2.0 ** -4) / (1 - e) - 1
    return np.maximum(rho * p / l, 2.0 ** -10 / (r * l * (1 - e)) + (2 * e / (1 - e)) * p / l)


def fp8_output_bound(Qd, Kd, Vd, lists, KSd, VSd, bias, v_scale, vs_scale, prefix_blocks: int,
                     block: int = BLOCK, query_blocks=None, with_variance: bool = False,
                     exp_rel_err: float = 0.0):
    """Per-element bound on |O_kernel - O| from the kernel's e4m3 numerators.

    The kernel writes each softmax numerator p (relative to a running max at
    most 2^8 below the row max, so p >= the exact numerator) times
    r = s_v / s_ref (<= 1, s_ref the largest V scale of the head) as e4m3:
    the error is at most 2^-4 relative for normal codes and 2^-10 absolute
    below 2^-6.  Dividing by the kernel's row sum (>= the exact one), a
    column's weight moves by at most max(2^-4 w, 2^-10 / (r * l)), with w the
    exact weight and l = sum_t exp(x_t - max) the exact row sum.  The bound is
    the sum of those moves times |v|, column by column.

    ``exp_rel_err`` = e: the kernel's numerators before rounding are
    p (1 + e_t) with |e_t| <= e (an approximate exponential), and its row sum
    is the sum of those, l (1 + e_l) with |e_l| <= e.  Then a normal code's
    weight is w (1 + e_t)(1 + d_t) / (1 + e_l) with |d_t| <= 2^-4, which moves
    by at most rho w, rho = (1 + e)(1 + 2^-4) / (1 - e) - 1; a subnormal
    code's by at most 2^-10 / (r l (1 - e)) + w (2 e / (1 - e)).  With e = 0
    both reduce to the moves above.

    With ``with_variance`` it also returns an upper model of each element's
    error variance: rounding to nearest leaves an error spread over at most
    half a step, so a move of at most m has variance at most m^2 / 3 (the
    uniform case); the moves of different columns are independent roundings,
    so the variances add: sum_t max-move_t^2 / 3 * v_t^2.
    """
    Qd = np.asarray(Qd, dtype=np.float64)
    N, d = Qd.shape
    scale = 1.0 / np.sqrt(d)
    bounds = block_bounds(N, block)
    nb = len(bounds)
    pb = prefix_blocks
    s_ref = max(np.max(v_scale), np.max(vs_scale))
    out = np.zeros((N, d))
    var = np.zeros((N, d))
    for i, (a, b) in enumerate(bounds):
        if query_blocks is not None and i not in query_blocks:
            continue
        E = [int(j) for j in lists[i]]
        tok = np.concatenate([np.arange(*bounds[j]) for j in E])
        logits = (Qd[a:b] @ Kd[tok].T) * scale
        vals = np.abs(Vd[tok])
        r = np.concatenate([np.full(bounds[j][1] - bounds[j][0], v_scale[j] / s_ref) for j in E])
        if i >= pb:
            skipped = [j for j in range(pb, nb) if j not in set(E)]
            if skipped:
                zl = (Qd[a:b] @ KSd[skipped].T) * scale + bias[skipped][None, :]
                logits = np.concatenate([logits, zl], axis=1)
                vals = np.concatenate([vals, np.abs(VSd[skipped])], axis=0)
                r = np.concatenate([r, np.array([vs_scale[j // block] for j in skipped]) / s_ref])
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        move = weight_moves(p, r[None, :], exp_rel_err)
        out[a:b] = move @ vals
        var[a:b] = (move ** 2 / 3) @ (vals ** 2)
    return (out, var) if with_variance else out
