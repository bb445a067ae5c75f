"""Pins of the FP8 oracle against things other than itself: hand-computed
e4m3 values, a brute-force nearest-code search over the whole e4m3 code table
built from its bit layout, torch's own float8_e4m3fn and bfloat16 casts, and
exact round trips of representable inputs."""

import numpy as np
import pytest
import torch

import oracle as orc
from oracle import bsa_oracle_fp8 as f8


def _e4m3_table():
    """Every finite e4m3 value from its bits: (value, mantissa bits), both signs."""
    out = []
    for sign in (1.0, -1.0):
        for e in range(16):
            for m in range(8):
                if e == 15 and m == 7:
                    continue                      # the NaN code
                v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
                out.append((sign * v, m))
    return out


def test_round_e4m3_hand_values():
    cases = {
        448.0: 448.0, 460.0: 448.0, 1e6: 448.0,     # largest finite; saturation
        1.0: 1.0, 1.0625: 1.0, 1.1875: 1.25,        # step 1/8 near 1; ties to even
        17.0: 16.0, 19.0: 20.0, 15.5: 16.0,         # step 2 in [16, 32)
        2.0 ** -6: 2.0 ** -6,                       # smallest normal
        2.0 ** -9: 2.0 ** -9,                       # smallest subnormal
        2.0 ** -10: 0.0,                            # tie between 0 and 2^-9 -> 0
        3 * 2.0 ** -10: 2.0 ** -8,                  # tie between 1 and 2 units -> 2
        0.75 * 2.0 ** -9: 2.0 ** -9,
        -1.0625: -1.0, 0.0: 0.0,
    }
    got = f8.round_e4m3(np.array(list(cases)))
    np.testing.assert_array_equal(got, np.array(list(cases.values())))


def test_round_e4m3_is_the_nearest_code_ties_to_even():
    table = _e4m3_table()
    vals = np.array([v for v, _ in table])
    mant = np.array([m for _, m in table])
    rng = np.random.default_rng(0)
    pos = np.unique(np.abs(vals))
    mids = (pos[1:] + pos[:-1]) / 2
    xs = np.concatenate([rng.uniform(-448, 448, 4000), rng.uniform(-1, 1, 4000) * 2.0 ** -5,
                         mids, -mids, vals])
    got = f8.round_e4m3(xs)
    for x, g in zip(xs, got):
        dist = np.abs(vals - x)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:                                  # a tie: the even mantissa
            best = [b for b in best if mant[b] % 2 == 0]
        assert g == vals[best[0]], (x, g, vals[best])


def test_round_e4m3_matches_torch_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 40, rng.standard_normal(20000) * 2.0 ** -7])
    x = np.clip(x.astype(np.float32), -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(f8.round_e4m3(x), ref)


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * 3).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(f8.bf16_round(x.astype(np.float64)), ref)


def test_quantize_group_closed_forms():
    c, s = f8.quantize_group(np.full((3, 4), -2.5, np.float32))       # constant block
    assert np.all(c == -448.0) and s == np.float32(2.5) / np.float32(448)
    c, s = f8.quantize_group(np.zeros((5, 4), np.float32))             # zero block
    assert np.all(c == 0) and s == 1.0
    x = np.array([[0.5, -3.0, 1.25, 0.0]], np.float32)
    c, s = f8.quantize_group(x)
    assert c[0, 1] == -448.0                                            # amax -> 448
    r = np.float32(448) / np.float32(3.0)
    np.testing.assert_array_equal(c, f8.round_e4m3((x * r).astype(np.float32)))


def test_quantize_relative_error_and_ragged_groups():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((300, 16)).astype(np.float32)              # groups 128, 128, 44
    codes, scales = f8.quantize_blocks(X)
    assert len(scales) == 3
    assert scales[2] == np.float32(np.abs(X[256:]).max()) / np.float32(448)
    D = f8.dequantize(codes, scales)
    big = np.abs(X) >= 2.0 ** -6 * np.repeat(scales, 128)[:300, None]
    rel = np.abs(D - X) / np.abs(X)
    assert rel[big].max() <= 2.0 ** -4 * (1 + 1e-6)


def _representable(rng, n, d, k):
    """Rows whose groups are e4m3 values times 2^k with |max| = 448 * 2^k."""
    table = np.array([v for v, _ in _e4m3_table()])
    X = rng.choice(table, size=(n, d)) * 2.0 ** k
    for a in range(0, n, 128):
        X[a, 0] = 448.0 * 2.0 ** k
    return X


def test_fp8_path_is_exact_on_representable_inputs():
    # Quantisation is lossless when every group is e4m3 values times a power of
    # two with amax = 448 * 2^k, so with every block listed (no summaries) the
    # FP8 path equals the bf16 path's definition (and dense attention).
    rng = np.random.default_rng(4)
    N, d = 300, 16
    Q, K, V = (_representable(rng, N, d, k) for k in (-9, -8, -7))
    r8 = f8.forward_head_fp8(Q, K, V, top_k=10, prefix=0)
    ref = orc.forward_head(Q, K, V, top_k=10, prefix=0)
    np.testing.assert_array_equal(r8["Qd"], Q)
    np.testing.assert_allclose(r8["O"], ref["O"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r8["lse"], ref["lse"], rtol=0, atol=1e-12)


def test_output_bound_covers_simulated_e4m3_numerators():
    # Simulate the kernel's rounding of p * r to e4m3 (running max = the row
    # max) by brute force and check the bound holds element by element.
    rng = np.random.default_rng(5)
    N, d, top_k = 700, 8, 2
    Q = rng.standard_normal((N, d)) * 1.5
    K = rng.standard_normal((N, d)) * 1.5
    V = rng.standard_normal((N, d))
    r8 = f8.forward_head_fp8(Q, K, V, top_k, 0)
    bound, var = f8.fp8_output_bound(r8["Qd"], r8["Kd"], r8["Vd"], r8["lists"], r8["KSd"],
                                     r8["VSd"], r8["bias"], r8["v_scale"], r8["vs_scale"], 0,
                                     with_variance=True)
    sq_err = 0.0
    s_ref = max(r8["v_scale"].max(), r8["vs_scale"].max())
    bounds = orc.block_bounds(N)
    nb = len(bounds)
    for i, (a, b) in enumerate(bounds):
        E = [int(j) for j in r8["lists"][i]]
        tok = np.concatenate([np.arange(*bounds[j]) for j in E])
        sk = [j for j in range(nb) if j not in E]
        logits = np.concatenate([r8["Qd"][a:b] @ r8["Kd"][tok].T / np.sqrt(d),
                                 r8["Qd"][a:b] @ r8["KSd"][sk].T / np.sqrt(d) + r8["bias"][sk]],
                                axis=1)
        vcodes = np.concatenate([r8["v_codes"][tok], r8["vs_codes"][sk]])
        r = np.concatenate([r8["v_scale"][tok // 128], r8["vs_scale"][np.array(sk) // 128]]) / s_ref
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        pq = f8.round_e4m3(p * r[None, :])
        O_sim = s_ref * (pq @ vcodes) / p.sum(axis=1, keepdims=True)
        err = np.abs(O_sim - r8["O"][a:b])
        assert (err <= bound[a:b] + 1e-12).all()
        assert err.max() > 0
        sq_err += float((err ** 2).sum())
    # the squared error over all elements stays within the variance model
    assert sq_err <= var.sum(), (sq_err, var.sum())


def test_output_bound_needs_its_subnormal_term():
    # Peaked logits: most numerators p * r fall below 2^-6, where e4m3 is
    # subnormal and its error is absolute (2^-10), not relative.  The full
    # bound must hold on the brute-force simulation; its relative part alone
    # must not (so the absolute term is load-bearing).
    rng = np.random.default_rng(6)
    N, d, top_k = 512, 8, 4
    Q = rng.standard_normal((N, d)) * 4.0
    K = rng.standard_normal((N, d)) * 4.0
    V = rng.standard_normal((N, d))
    r8 = f8.forward_head_fp8(Q, K, V, top_k, 0)
    bound = f8.fp8_output_bound(r8["Qd"], r8["Kd"], r8["Vd"], r8["lists"], r8["KSd"], r8["VSd"],
                                r8["bias"], r8["v_scale"], r8["vs_scale"], 0)
    s_ref = max(r8["v_scale"].max(), r8["vs_scale"].max())
    rel_only_violated = False
    for i, (a, b) in enumerate(orc.block_bounds(N)):
        E = [int(j) for j in r8["lists"][i]]
        tok = np.concatenate([np.arange(*orc.block_bounds(N)[j]) for j in E])
        logits = r8["Qd"][a:b] @ r8["Kd"][tok].T / np.sqrt(d)           # every block listed
        r = r8["v_scale"][tok // 128] / s_ref
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        l = p.sum(axis=1, keepdims=True)
        O_sim = s_ref * (f8.round_e4m3(p * r[None, :]) @ r8["v_codes"][tok]) / l
        err = np.abs(O_sim - r8["O"][a:b])
        assert (err <= bound[a:b] + 1e-12).all()
        rel_only = (2.0 ** -4 * p / l) @ np.abs(r8["Vd"][tok])
        rel_only_violated |= bool((err > rel_only + 1e-12).any())
    assert rel_only_violated


def test_output_bound_covers_approximate_exponentials():
    # The kernel may compute some softmax numerators with an approximate
    # exponential: p (1 + e_t), |e_t| <= e, and sums those into its row sum.
    # Simulated with the worst signs (alternating +e and -e per column, and
    # all +e or all -e), the bound with exp_rel_err = e holds element by
    # element.
    rng = np.random.default_rng(7)
    N, d, top_k = 600, 8, 2
    Q = rng.standard_normal((N, d)) * 1.5
    K = rng.standard_normal((N, d)) * 1.5
    V = rng.standard_normal((N, d))
    r8 = f8.forward_head_fp8(Q, K, V, top_k, 0)
    eps = 2.0 ** -6
    args = (r8["Qd"], r8["Kd"], r8["Vd"], r8["lists"], r8["KSd"], r8["VSd"], r8["bias"],
            r8["v_scale"], r8["vs_scale"], 0)
    bound_e = f8.fp8_output_bound(*args, exp_rel_err=eps)
    bound_0 = f8.fp8_output_bound(*args)
    s_ref = max(r8["v_scale"].max(), r8["vs_scale"].max())
    bounds = orc.block_bounds(N)
    nb = len(bounds)
    for pattern in ("alternate", "plus", "minus"):
        for i, (a, b) in enumerate(bounds):
            E = [int(j) for j in r8["lists"][i]]
            tok = np.concatenate([np.arange(*bounds[j]) for j in E])
            sk = [j for j in range(nb) if j not in E]
            logits = np.concatenate([r8["Qd"][a:b] @ r8["Kd"][tok].T / np.sqrt(d),
                                     r8["Qd"][a:b] @ r8["KSd"][sk].T / np.sqrt(d)
                                     + r8["bias"][sk]], axis=1)
            vcodes = np.concatenate([r8["v_codes"][tok], r8["vs_codes"][sk]])
            r = np.concatenate([r8["v_scale"][tok // 128],
                                r8["vs_scale"][np.array(sk) // 128]]) / s_ref
            p = np.exp(logits - logits.max(axis=1, keepdims=True))
            sign = {"alternate": np.where(np.arange(p.shape[1]) % 2 == 0, 1.0, -1.0),
                    "plus": np.ones(p.shape[1]), "minus": -np.ones(p.shape[1])}[pattern]
            pt = p * (1 + eps * sign[None, :])
            O_sim = s_ref * (f8.round_e4m3(pt * r[None, :]) @ vcodes) / pt.sum(axis=1,
                                                                           keepdims=True)
            err = np.abs(O_sim - r8["O"][a:b])
            assert (err <= bound_e[a:b] + 1e-12).all(), (pattern, i)
    assert (bound_e >= bound_0).all() and (bound_e > bound_0).any()


def test_weight_moves_need_the_approximate_exponential_term():
    # Brute force over rows of numerators, e4m3 rounding and the kernel's own
    # row sum: every weight stays within weight_moves(e).  A constructed row
    # where one numerator sits just below a rounding midpoint (so e4m3 rounds
    # it down by almost 2^-4) and is pushed down by -e while the others are
    # pushed up (so the row sum grows) moves further than the bound without
    # the term allows.
    rng = np.random.default_rng(8)
    eps = 2.0 ** -5
    for _ in range(200):
        n = 64
        p = np.exp(-rng.exponential(3.0, n))
        p[rng.integers(n)] = 1.0
        r = rng.uniform(0.2, 1.0, n)
        et = rng.choice([-eps, eps], n)
        pt = p * (1 + et)
        w_hat = f8.round_e4m3(pt * r) / (r * pt.sum())
        w = p / p.sum()
        assert (np.abs(w_hat - w) <= f8.weight_moves(p, r, eps) + 1e-15).all()
    # the constructed row
    k = 1.0 + 2.0 ** -4 - 2.0 ** -11          # rounds down to 1.0 in e4m3
    p = np.array([k / (1 - eps), 1.0, 1.0, 1.0])
    r = np.ones(4)
    pt = p * np.array([1 - eps, 1 + eps, 1 + eps, 1 + eps])
    assert f8.round_e4m3(np.array([pt[0]]))[0] == 1.0
    w_hat = f8.round_e4m3(pt * r) / (r * pt.sum())
    w = p / p.sum()
    assert abs(w_hat[0] - w[0]) <= f8.weight_moves(p, r, eps)[0]
    assert abs(w_hat[0] - w[0]) > f8.weight_moves(p, r, 0.0)[0]
