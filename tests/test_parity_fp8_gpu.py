"""GPU parity of the FP8 (e4m3) path against the FP8 oracle, through the C ABI.

* Codes and scales of Q, K, V: bit-exact (both sides take every rounding
  decision on the same fp32 values: fp32(448 / amax), one fp32 multiply,
  round to nearest even).
* Summary codes: the kernel quantises its own bf16 k~ / v~, which can differ
  from the oracle's bf16 rounding of its fp64 summaries in the last bit, so
  dequantised values agree to one e4m3 step.
* O: within the oracle's bound for the kernel's e4m3 softmax numerators
  (``fp8_output_bound``) plus bf16 output rounding, element by element; and
  the summed squared error within the summed variance model of those
  roundings (plus bf16 rounding of O).  A fixed rel-L2 such as the bf16
  path's 1e-2 does not apply: with zero-mean values O is itself an average
  of size ~ sqrt(sum w^2), so each weight's ~2^-4 rounding moves O by a
  comparable fraction of itself.
* lse: within the bias's bf16 bound (the kernel's bias is computed from
  bf16 k~, the oracle's from fp64 k~): 2^-9 * sum_d |qbar_d| |k~_jd| / sqrt(d).
"""

import numpy as np
import pytest
import torch

import oracle as orc
from oracle import bsa_oracle_fp8 as f8
from block_sparse_video_bsa_b200 import bsa
from block_sparse_video_bsa_b200.inputs import CONFIGS, make_qkv

pytestmark = pytest.mark.gpu


def _host(t):
    return t.double().cpu().numpy()


def _decode(codes_u8):
    return codes_u8.cpu().view(torch.float8_e4m3fn).double().numpy()


def run_fp8_stages(Q, K, V, top_k, prefix, variant, with_lse=True):
    B, H, N, _ = Q.shape
    p = bsa.params(B, H, N, top_k, prefix, variant)
    buf = bsa.stage_buffers(B, H, N, top_k, prefix, variant)
    bsa.bsa_pool(p, Q, buf["qpool"], buf["anchor"])
    bsa.bsa_summarize(p, K, V, buf["anchor"], buf["kpool"], buf["ksum"], buf["vsum"], buf["bias"])
    bsa.bsa_select(p, buf["qpool"], buf["kpool"], buf["idx"], buf["cnt"])
    opbuf, ops, views = bsa.fp8_operands(p)
    bsa.bsa_quantize_fp8(p, Q, K, V, buf["ksum"], buf["vsum"], ops)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda") if with_lse else None
    bsa.bsa_attend_fp8(p, ops, buf["idx"], buf["cnt"], buf["bias"], O, lse)
    torch.cuda.synchronize()
    buf.update(O=O, lse=lse, ops_buf=opbuf, ops=ops, views=views)
    return buf


def check_head_fp8(buf, Q, K, V, b, h, top_k, prefix, variant, check_lse=True, query_blocks=None):
    N = Q.shape[2]
    nb = -(-N // 128)
    vw = buf["views"]
    r8 = f8.forward_head_fp8(_host(Q[b, h]), _host(K[b, h]), _host(V[b, h]), top_k, prefix,
                             variant, query_blocks=query_blocks)
    # codes and scales of Q, K, V: bit-exact
    np.testing.assert_array_equal(_decode(vw["q8"][b, h]), r8["q_codes"])
    np.testing.assert_array_equal(_decode(vw["k8"][b, h]), r8["k_codes"])
    vt = _decode(vw["vt8"][b, h]).transpose(0, 2, 1).reshape(nb * 128, 128)
    np.testing.assert_array_equal(vt[:N], r8["v_codes"])
    assert not vt[N:].any()
    for name, key in (("q_scale", "q_scale"), ("k_scale", "k_scale"), ("v_scale", "v_scale")):
        np.testing.assert_array_equal(vw[name][b, h].cpu().numpy(), r8[key].astype(np.float32))
    # summary codes: one e4m3 step
    ksd = _decode(vw["ks8"][b, h]) * np.repeat(vw["ks_scale"][b, h].cpu().numpy(), 128)[:nb, None]
    nt = -(-nb // 128)
    vst = _decode(vw["vst8"][b, h]).transpose(0, 2, 1).reshape(nt * 128, 128)[:nb]
    vsd = vst * np.repeat(vw["vs_scale"][b, h].cpu().numpy(), 128)[:nb, None]
    for got, ref, sc in ((ksd, r8["KSd"], r8["ks_scale"]), (vsd, r8["VSd"], r8["vs_scale"])):
        floor = np.repeat(sc, 128)[:nb, None] * 2.0 ** -6
        assert (np.abs(got - ref) <= 2.0 ** -3 * np.maximum(np.abs(ref), floor) + 1e-12).all()
    assert vw["v_ref"][b, h].item() == np.float32(max(r8["v_scale"].max(), r8["vs_scale"].max()))
    # O within the e4m3-numerator bound (+ bf16 output rounding), element by
    # element, and the summed squared error within the variance model
    bound, var = f8.fp8_output_bound(r8["Qd"], r8["Kd"], r8["Vd"], r8["lists"], r8["KSd"],
                                     r8["VSd"], r8["bias"], r8["v_scale"], r8["vs_scale"],
                                     prefix // 128, query_blocks=query_blocks, with_variance=True)
    got = _host(buf["O"][b, h])
    rows = np.arange(N) if query_blocks is None else np.concatenate(
        [np.arange(i * 128, min(N, i * 128 + 128)) for i in query_blocks])
    err = np.abs(got[rows] - r8["O"][rows])
    tol = bound[rows] + 2.0 ** -8 * np.abs(r8["O"][rows]) + 1e-3
    assert (err <= tol).all(), (err.max(), (err - tol).max())
    sq_model = var[rows].sum() + ((2.0 ** -9 * r8["O"][rows]) ** 2 / 3).sum() + 1e-10 * err.size
    assert (err ** 2).sum() <= sq_model, ((err ** 2).sum(), sq_model)
    rel = np.linalg.norm(got[rows] - r8["O"][rows]) / np.linalg.norm(r8["O"][rows])
    if check_lse:
        qbar = orc.video_query_anchor(_host(Q[b, h]), prefix)
        ks_full = orc.block_summaries(_host(K[b, h]), _host(V[b, h]), qbar, variant)[0]
        lb = 2.0 ** -9 * (np.abs(qbar) @ np.abs(ks_full).T).max() / np.sqrt(128) + 2e-4
        lerr = np.abs(buf["lse"][b, h].cpu().numpy()[rows] - r8["lse"][rows])
        assert lerr.max() <= lb, (lerr.max(), lb)
    return err.max(), rel


@pytest.mark.parametrize("B,H,N,top_k,prefix,variant,kind", [
    (1, 2, 2048, 4, 0, "anchor", "iid"),
    (1, 2, 2048, 4, 0, "mean", "iid"),
    (2, 2, 1000, 3, 0, "anchor", "block_offset"),      # ragged tail (104 rows)
    (1, 3, 1500, 2, 256, "anchor", "block_offset"),    # dense prefix + ragged
    (1, 2, 4100, 5, 0, "anchor", "block_offset"),      # ragged tail of 4 rows
    (1, 1, 300, 1, 0, "anchor", "iid"),                # 3 blocks, k=1
    (1, 1, 17_000, 7, 0, "anchor", "block_offset"),    # 133 blocks: 2 summary tiles
])
def test_fp8_small_cases(B, H, N, top_k, prefix, variant, kind):
    Q, K, V = make_qkv(B, H, N, 128, kind, 0, device="cuda")
    buf = run_fp8_stages(Q, K, V, top_k, prefix, variant)
    for b in range(B):
        for h in range(H):
            check_head_fp8(buf, Q, K, V, b, h, top_k, prefix, variant)


@pytest.mark.parametrize("N", [1, 127, 129])
def test_fp8_edge_lengths(N):
    Q, K, V = make_qkv(1, 1, N, 128, "iid", N, device="cuda")
    buf = run_fp8_stages(Q, K, V, 1, 0, "anchor")
    check_head_fp8(buf, Q, K, V, 0, 0, 1, 0, "anchor")


def test_fp8_forward_matches_stages_and_is_deterministic():
    Q, K, V = make_qkv(1, 3, 3000, 128, "block_offset", 9, device="cuda")
    buf = run_fp8_stages(Q, K, V, 4, 0, "anchor")
    O1, l1 = bsa.forward_fp8(Q, K, V, 4, return_lse=True)
    O2, l2 = bsa.forward_fp8(Q, K, V, 4, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(O1, buf["O"]) and torch.equal(O1, O2)
    assert torch.equal(l1, buf["lse"]) and torch.equal(l1, l2)


@pytest.mark.parametrize("name,head,n_qb", [("h3_768p_5s", 31, 24),
                                            ("h3_768p_15s_prefix512", 5, 12),
                                            ("h3_2k_5s", 17, 8)])
def test_fp8_full_size_sampled_head(name, head, n_qb):
    # the workload through bsa_forward_fp8 (the call bench.py times with
    # --precision fp8); one head against the oracle on sampled query blocks
    # (the prefix workload's sample includes two dense-prefix query blocks)
    cfg = CONFIGS[name]
    B, H, N = cfg["B"], cfg["H"], cfg["N"]
    Q, K, V = make_qkv(B, H, N, 128, cfg["kind"], 0, device="cuda")
    O = bsa.forward_fp8(Q, K, V, cfg["top_k"], cfg["prefix"], cfg["variant"])
    buf = run_fp8_stages(Q, K, V, cfg["top_k"], cfg["prefix"], cfg["variant"], with_lse=False)
    assert torch.equal(O, buf["O"])
    qb = set(np.random.default_rng(7).choice(-(-N // 128), n_qb, replace=False).tolist())
    if cfg["prefix"]:
        qb |= {0, cfg["prefix"] // 128 - 1}
    check_head_fp8(buf, Q, K, V, 0, head, cfg["top_k"], cfg["prefix"], cfg["variant"],
                   check_lse=False, query_blocks=sorted(qb))
    del Q, K, V, O, buf
    torch.cuda.empty_cache()
