"""Thin ctypes binding over libbsa.so (include/bsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch tensors (device memory + streams); the functions
keep the C names.  There is no fallback: if libbsa.so is missing or the
device is not sm_100 the call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "bsa.h")

(BSA_OK, BSA_ERR_INVALID, BSA_ERR_ALIGN, BSA_ERR_CUDA, BSA_ERR_TIMEOUT, BSA_ERR_UNSUPPORTED,
 BSA_ERR_SCRATCH) = range(7)
BSA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024
VARIANTS = {"anchor": 0, "mean": 1}


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class bsa_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
        ("D", ctypes.c_int32), ("top_k", ctypes.c_int32), ("prefix", ctypes.c_int32),
        ("variant", ctypes.c_int32), ("dev_status", ctypes.c_void_p),
    ]


class bsa_fp8_operands(ctypes.Structure):
    """Mirror of bsa_fp8_operands (include/bsa.h): e4m3 codes and fp32 scales."""
    _fields_ = [("q8", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k8", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("vt8", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("ks8", ctypes.c_void_p), ("ks_scale", ctypes.c_void_p),
                ("vst8", ctypes.c_void_p), ("vs_scale", ctypes.c_void_p),
                ("v_ref", ctypes.c_void_p)]


_lib = None
_P = ctypes.POINTER(bsa_params)
_F8 = ctypes.POINTER(bsa_fp8_operands)
_vp = ctypes.c_void_p
_SIGS = {
    "bsa_num_blocks": (ctypes.c_int32, [_P]),
    "bsa_select_capacity": (ctypes.c_int32, [_P]),
    "bsa_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_pool": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp]),
    "bsa_summarize": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_select": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp]),
    "bsa_attend": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_forward": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "bsa_forward_host": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp, ctypes.c_size_t, _vp]),
    "bsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bsa_debug_expired_wait": (ctypes.c_int, [_vp, ctypes.c_uint64, _vp]),
    "bsa_forward_noalloc": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_reblock_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_reblock": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "bsa_permute": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_pool_permuted": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_summarize_permuted": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                              _vp, _vp]),
    "bsa_unpermute": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_forward_reblock_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_forward_reblock": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                           _vp]),
    "bsa_fp8_operands_bytes": (ctypes.c_size_t, [_P]),
    "bsa_fp8_operands_carve": (ctypes.c_int, [_P, _vp, ctypes.c_size_t, _F8]),
    "bsa_quantize_fp8": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _F8, _vp]),
    "bsa_attend_fp8": (ctypes.c_int, [_P, _F8, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsa_forward_fp8_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_forward_fp8": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "bsa_threshold_capacity": (ctypes.c_int32, [_P]),
    "bsa_select_threshold": (ctypes.c_int, [_P, ctypes.c_float, _vp, _vp, _vp, _vp, _vp]),
    "bsa_attend_lists_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_attend_lists": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, ctypes.c_int32, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "bsa_forward_threshold_workspace_bytes": (ctypes.c_size_t, [_P]),
    "bsa_forward_threshold": (ctypes.c_int, [_P, ctypes.c_float, _vp, _vp, _vp, _vp, _vp, _vp,
                                             ctypes.c_size_t, _vp]),
    "bsa_extra_side_capacity": (ctypes.c_int32, [_P, ctypes.c_int32]),
    "bsa_summarize_stats": (ctypes.c_int, [_P] + [_vp] * 11),
    "bsa_select_extra_workspace_bytes": (ctypes.c_size_t, [_P, ctypes.c_int32]),
    "bsa_select_extra": (ctypes.c_int, [_P, ctypes.c_int32] + [_vp] * 7 + [ctypes.c_size_t, _vp]),
    "bsa_extra_summaries": (ctypes.c_int, [_P, ctypes.c_int32] + [_vp] * 15),
    "bsa_attend_extra": (ctypes.c_int, [_P, ctypes.c_int32] + [_vp] * 17),
    "bsa_forward_extra_workspace_bytes": (ctypes.c_size_t, [_P, ctypes.c_int32]),
    "bsa_forward_extra": (ctypes.c_int, [_P, ctypes.c_int32] + [_vp] * 6 + [ctypes.c_size_t, _vp]),
}
_HOST12 = [_vp] * 11 + [ctypes.c_size_t, _vp]
_SIGS["bsa_forward_fp8_host"] = (ctypes.c_int, [_P] + _HOST12)
_SIGS["bsa_forward_threshold_host"] = (ctypes.c_int, [_P, ctypes.c_float] + _HOST12)
_SIGS["bsa_forward_extra_host"] = (ctypes.c_int, [_P, ctypes.c_int32] + _HOST12)
_SIGS["bsa_forward_reblock_host"] = (ctypes.c_int, [_P] + _HOST12)
BSA_MAX_EXTRA_TOKENS = 512


def lib() -> ctypes.CDLL:
    """Load libbsa.so once (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m "
                               "block_sparse_video_bsa_b200.build` first")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of the functions include/bsa.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().bsa_status_string(int(status)).decode()


def params(B, H, N, top_k, prefix=0, variant="anchor", D=128, dev_status=None) -> bsa_params:
    v = VARIANTS[variant] if isinstance(variant, str) else int(variant)
    ds = None if dev_status is None else dev_status.data_ptr()
    return bsa_params(B, H, N, D, top_k, prefix, v, ds)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc, where):
    if rc != BSA_OK:
        raise BsaError(rc, where)


# --------------------------------------------------------------- sizes

def bsa_num_blocks(p: bsa_params) -> int:
    return lib().bsa_num_blocks(ctypes.byref(p))


def bsa_select_capacity(p: bsa_params) -> int:
    return lib().bsa_select_capacity(ctypes.byref(p))


def bsa_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_workspace_bytes(ctypes.byref(p))


# --------------------------------------------------------------- stages

def bsa_pool(p, Q, qpool, anchor, stream=None):
    _check(lib().bsa_pool(ctypes.byref(p), _ptr(Q), _ptr(qpool), _ptr(anchor), _stream(stream)),
           "bsa_pool")


def bsa_summarize(p, K, V, anchor, kpool, ksum, vsum, bias, stream=None):
    _check(lib().bsa_summarize(ctypes.byref(p), _ptr(K), _ptr(V), _ptr(anchor), _ptr(kpool),
                               _ptr(ksum), _ptr(vsum), _ptr(bias), _stream(stream)),
           "bsa_summarize")


def bsa_select(p, qpool, kpool, idx, cnt, stream=None):
    _check(lib().bsa_select(ctypes.byref(p), _ptr(qpool), _ptr(kpool), _ptr(idx), _ptr(cnt),
                            _stream(stream)), "bsa_select")


def bsa_attend(p, Q, K, V, idx, cnt, ksum, vsum, bias, O, lse=None, stream=None):
    _check(lib().bsa_attend(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cnt),
                            _ptr(ksum), _ptr(vsum), _ptr(bias), _ptr(O), _ptr(lse),
                            _stream(stream)), "bsa_attend")


def bsa_forward(p, Q, K, V, O, lse, workspace, stream=None):
    _check(lib().bsa_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream)), "bsa_forward")


def bsa_forward_host(p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream=None):
    _check(lib().bsa_forward_host(ctypes.byref(p), _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO),
                                  _ptr(hlse), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dO), _ptr(dlse),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "bsa_forward_host")


def _host_args(hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream):
    return (_ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO), _ptr(hlse), _ptr(dQ), _ptr(dK), _ptr(dV),
            _ptr(dO), _ptr(dlse), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream))


def bsa_forward_fp8_host(p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream=None):
    _check(lib().bsa_forward_fp8_host(ctypes.byref(p), *_host_args(
        hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream)), "bsa_forward_fp8_host")


def bsa_forward_threshold_host(p, tau, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace,
                               stream=None):
    _check(lib().bsa_forward_threshold_host(ctypes.byref(p), float(tau), *_host_args(
        hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream)),
        "bsa_forward_threshold_host")


def bsa_forward_extra_host(p, n_extra, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace,
                           stream=None):
    _check(lib().bsa_forward_extra_host(ctypes.byref(p), int(n_extra), *_host_args(
        hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream)), "bsa_forward_extra_host")


def bsa_forward_reblock_host(p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace,
                             stream=None):
    _check(lib().bsa_forward_reblock_host(ctypes.byref(p), *_host_args(
        hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, stream)),
        "bsa_forward_reblock_host")


def bsa_forward_noalloc(p, Q, K, V, O, lse=None, stream=None):
    """bsa_forward with its workspace in the library's static device scratch,
    for callers that cannot allocate device memory (see include/bsa.h)."""
    _check(lib().bsa_forward_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                     _ptr(lse), _stream(stream)), "bsa_forward_noalloc")


def bsa_reblock_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_reblock_workspace_bytes(ctypes.byref(p))


def bsa_reblock(p, Q, K, perm, workspace, stream=None):
    _check(lib().bsa_reblock(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(perm), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "bsa_reblock")


def bsa_pool_permuted(p, Q, perm, Qp, qpool, anchor, stream=None):
    _check(lib().bsa_pool_permuted(ctypes.byref(p), _ptr(Q), _ptr(perm), _ptr(Qp), _ptr(qpool),
                                   _ptr(anchor), _stream(stream)), "bsa_pool_permuted")


def bsa_summarize_permuted(p, K, V, perm, Kp, Vp, anchor, kpool, ksum, vsum, bias, stream=None):
    _check(lib().bsa_summarize_permuted(ctypes.byref(p), _ptr(K), _ptr(V), _ptr(perm), _ptr(Kp),
                                        _ptr(Vp), _ptr(anchor), _ptr(kpool), _ptr(ksum),
                                        _ptr(vsum), _ptr(bias), _stream(stream)),
           "bsa_summarize_permuted")


def bsa_permute(p, Q, K, V, perm, Qp, Kp, Vp, stream=None):
    _check(lib().bsa_permute(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(Qp),
                             _ptr(Kp), _ptr(Vp), _stream(stream)), "bsa_permute")


def bsa_unpermute(p, Op, lsep, perm, O, lse=None, stream=None):
    _check(lib().bsa_unpermute(ctypes.byref(p), _ptr(Op), _ptr(lsep), _ptr(perm), _ptr(O),
                               _ptr(lse), _stream(stream)), "bsa_unpermute")


def bsa_forward_reblock_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_forward_reblock_workspace_bytes(ctypes.byref(p))


def bsa_forward_reblock(p, Q, K, V, O, lse, workspace, stream=None):
    _check(lib().bsa_forward_reblock(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                     _ptr(lse), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "bsa_forward_reblock")


def reblock(Q, K, prefix=0, stream=None):
    """perm [B, H, N] int32 of the reblocked layout (see bsa_reblock)."""
    B, H, N, D = Q.shape
    p = params(B, H, N, 1, prefix, D=D)
    perm = torch.empty(B, H, N, dtype=torch.int32, device=Q.device)
    ws = torch.empty(max(256, bsa_reblock_workspace_bytes(p)), dtype=torch.uint8, device=Q.device)
    bsa_reblock(p, Q, K, perm, ws, stream)
    return perm


def forward_reblock(Q, K, V, top_k, prefix=0, variant="anchor", return_lse=False, ws=None,
                    stream=None):
    """bsa_forward_reblock: block-sparse attention on the reblocked layout,
    O (and lse) returned in the original token order."""
    B, H, N, D = Q.shape
    p = params(B, H, N, top_k, prefix, variant, D=D)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if return_lse else None
    if ws is None:
        ws = torch.empty(bsa_forward_reblock_workspace_bytes(p), dtype=torch.uint8,
                         device=Q.device)
    bsa_forward_reblock(p, Q, K, V, O, lse, ws, stream)
    return (O, lse) if return_lse else O


def bsa_fp8_operands_bytes(p: bsa_params) -> int:
    return lib().bsa_fp8_operands_bytes(ctypes.byref(p))


def bsa_fp8_operands_carve(p, buf) -> bsa_fp8_operands:
    ops = bsa_fp8_operands()
    _check(lib().bsa_fp8_operands_carve(ctypes.byref(p), _ptr(buf), buf.numel() * buf.element_size(),
                                        ctypes.byref(ops)), "bsa_fp8_operands_carve")
    return ops


def bsa_quantize_fp8(p, Q, K, V, ksum, vsum, ops, stream=None):
    _check(lib().bsa_quantize_fp8(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(ksum),
                                  _ptr(vsum), ctypes.byref(ops), _stream(stream)),
           "bsa_quantize_fp8")


def bsa_attend_fp8(p, ops, idx, cnt, bias, O, lse=None, stream=None):
    _check(lib().bsa_attend_fp8(ctypes.byref(p), ctypes.byref(ops), _ptr(idx), _ptr(cnt),
                                _ptr(bias), _ptr(O), _ptr(lse), _stream(stream)), "bsa_attend_fp8")


def bsa_forward_fp8_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_forward_fp8_workspace_bytes(ctypes.byref(p))


def bsa_forward_fp8(p, Q, K, V, O, lse, workspace, stream=None):
    _check(lib().bsa_forward_fp8(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream)), "bsa_forward_fp8")


def bsa_threshold_capacity(p: bsa_params) -> int:
    return lib().bsa_threshold_capacity(ctypes.byref(p))


def bsa_select_threshold(p, tau, qpool, kpool, idx, cnt, stream=None):
    _check(lib().bsa_select_threshold(ctypes.byref(p), float(tau), _ptr(qpool), _ptr(kpool),
                                      _ptr(idx), _ptr(cnt), _stream(stream)),
           "bsa_select_threshold")


def bsa_attend_lists_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_attend_lists_workspace_bytes(ctypes.byref(p))


def bsa_attend_lists(p, Q, K, V, idx, cnt, ksum, vsum, bias, O, lse, workspace, stream=None):
    """bsa_attend over variable-length lists; the row stride is idx's last dimension."""
    _check(lib().bsa_attend_lists(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                  int(idx.shape[-1]), _ptr(cnt), _ptr(ksum), _ptr(vsum),
                                  _ptr(bias), _ptr(O), _ptr(lse), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "bsa_attend_lists")


def bsa_forward_threshold_workspace_bytes(p: bsa_params) -> int:
    return lib().bsa_forward_threshold_workspace_bytes(ctypes.byref(p))


def bsa_forward_threshold(p, tau, Q, K, V, O, lse, workspace, stream=None):
    _check(lib().bsa_forward_threshold(ctypes.byref(p), float(tau), _ptr(Q), _ptr(K), _ptr(V),
                                       _ptr(O), _ptr(lse), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "bsa_forward_threshold")


def bsa_extra_side_capacity(p: bsa_params, n_extra: int) -> int:
    return lib().bsa_extra_side_capacity(ctypes.byref(p), int(n_extra))


def bsa_summarize_stats(p, K, V, anchor, kpool, ksum, vsum, bias, kstat, vstat, lse_blk,
                        stream=None):
    _check(lib().bsa_summarize_stats(ctypes.byref(p), _ptr(K), _ptr(V), _ptr(anchor), _ptr(kpool),
                                     _ptr(ksum), _ptr(vsum), _ptr(bias), _ptr(kstat), _ptr(vstat),
                                     _ptr(lse_blk), _stream(stream)), "bsa_summarize_stats")


def bsa_select_extra_workspace_bytes(p: bsa_params, n_extra: int) -> int:
    return lib().bsa_select_extra_workspace_bytes(ctypes.byref(p), int(n_extra))


def bsa_select_extra(p, n_extra, qpool, K, idx, cnt, extra, ecnt, workspace, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bsa_select_extra(ctypes.byref(p), int(n_extra), _ptr(qpool), _ptr(K), _ptr(idx),
                                  _ptr(cnt), _ptr(extra), _ptr(ecnt), _ptr(workspace), nbytes,
                                  _stream(stream)), "bsa_select_extra")


def bsa_extra_summaries(p, n_extra, K, V, anchor, kpool, kstat, vstat, lse_blk, extra, ecnt,
                        side_k, side_v, side_bias, side_blk, side_cnt, stream=None):
    _check(lib().bsa_extra_summaries(ctypes.byref(p), int(n_extra), _ptr(K), _ptr(V), _ptr(anchor),
                                     _ptr(kpool), _ptr(kstat), _ptr(vstat), _ptr(lse_blk),
                                     _ptr(extra), _ptr(ecnt), _ptr(side_k), _ptr(side_v),
                                     _ptr(side_bias), _ptr(side_blk), _ptr(side_cnt),
                                     _stream(stream)), "bsa_extra_summaries")


def bsa_attend_extra(p, n_extra, Q, K, V, idx, cnt, extra, ecnt, ksum, vsum, bias, side_k, side_v,
                     side_bias, side_cnt, O, lse=None, stream=None):
    _check(lib().bsa_attend_extra(ctypes.byref(p), int(n_extra), _ptr(Q), _ptr(K), _ptr(V),
                                  _ptr(idx), _ptr(cnt), _ptr(extra), _ptr(ecnt), _ptr(ksum),
                                  _ptr(vsum), _ptr(bias), _ptr(side_k), _ptr(side_v),
                                  _ptr(side_bias), _ptr(side_cnt), _ptr(O), _ptr(lse),
                                  _stream(stream)), "bsa_attend_extra")


def bsa_forward_extra_workspace_bytes(p: bsa_params, n_extra: int) -> int:
    return lib().bsa_forward_extra_workspace_bytes(ctypes.byref(p), int(n_extra))


def bsa_forward_extra(p, n_extra, Q, K, V, O, lse, workspace, stream=None):
    _check(lib().bsa_forward_extra(ctypes.byref(p), int(n_extra), _ptr(Q), _ptr(K), _ptr(V),
                                   _ptr(O), _ptr(lse), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "bsa_forward_extra")


def extra_buffers(B, H, N, top_k, n_extra, prefix=0, variant="anchor", device="cuda"):
    """Device tensors for the extra-token stages (statistics, lists, side
    table, candidate scratch)."""
    p = params(B, H, N, top_k, prefix, variant)
    nb = bsa_num_blocks(p)
    scap = bsa_extra_side_capacity(p, n_extra)
    if nb < 0 or scap < 0:
        raise BsaError(BSA_ERR_INVALID, "extra_buffers")
    f32, bf16, i32 = torch.float32, torch.bfloat16, torch.int32
    return dict(
        kstat=torch.empty(B, H, nb, 128, dtype=f32, device=device),
        vstat=torch.empty(B, H, nb, 128, dtype=f32, device=device),
        lse_blk=torch.empty(B, H, nb, dtype=f32, device=device),
        extra=torch.empty(B, H, nb, max(n_extra, 1), dtype=i32, device=device),
        ecnt=torch.empty(B, H, nb, dtype=i32, device=device),
        side_k=torch.empty(B, H, nb, max(scap, 1), 128, dtype=bf16, device=device),
        side_v=torch.empty(B, H, nb, max(scap, 1), 128, dtype=bf16, device=device),
        side_bias=torch.empty(B, H, nb, max(scap, 1), dtype=f32, device=device),
        side_blk=torch.empty(B, H, nb, max(scap, 1), dtype=i32, device=device),
        side_cnt=torch.empty(B, H, nb, dtype=i32, device=device),
        cand=torch.empty(max(256, bsa_select_extra_workspace_bytes(p, n_extra)), dtype=torch.uint8,
                         device=device),
    )


def forward_extra(Q, K, V, top_k, n_extra, prefix=0, variant="anchor", return_lse=False, ws=None,
                  stream=None):
    """bsa_forward_extra: block-sparse attention plus n_extra top-scoring
    tokens per query block."""
    B, H, N, D = Q.shape
    p = params(B, H, N, top_k, prefix, variant, D=D)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if return_lse else None
    if ws is None:
        ws = torch.empty(bsa_forward_extra_workspace_bytes(p, n_extra), dtype=torch.uint8,
                         device=Q.device)
    bsa_forward_extra(p, n_extra, Q, K, V, O, lse, ws, stream)
    return (O, lse) if return_lse else O


def bsa_debug_expired_wait(dev_status, timeout_ns: int, stream=None):
    _check(lib().bsa_debug_expired_wait(_ptr(dev_status), int(timeout_ns), _stream(stream)),
           "bsa_debug_expired_wait")


# --------------------------------------------------------------- allocation helpers

def stage_buffers(B, H, N, top_k, prefix=0, variant="anchor", device="cuda"):
    """Device tensors for the intermediates of the four stages."""
    p = params(B, H, N, top_k, prefix, variant)
    nb = bsa_num_blocks(p)
    kcap = bsa_select_capacity(p)
    if nb < 0:
        raise BsaError(BSA_ERR_INVALID, "stage_buffers")
    f32, bf16, i32 = torch.float32, torch.bfloat16, torch.int32
    return dict(
        qpool=torch.empty(B, H, nb, 128, dtype=f32, device=device),
        anchor=torch.empty(B, H, 128, dtype=f32, device=device),
        kpool=torch.empty(B, H, nb, 128, dtype=f32, device=device),
        ksum=torch.empty(B, H, nb, 128, dtype=bf16, device=device),
        vsum=torch.empty(B, H, nb, 128, dtype=bf16, device=device),
        bias=torch.empty(B, H, nb, dtype=f32, device=device),
        idx=torch.empty(B, H, nb, kcap, dtype=i32, device=device),
        cnt=torch.empty(B, H, nb, dtype=i32, device=device),
    )


def workspace(p: bsa_params, device="cuda") -> torch.Tensor:
    n = bsa_workspace_bytes(p)
    if n == 0:
        raise BsaError(BSA_ERR_INVALID, "bsa_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward(Q, K, V, top_k, prefix=0, variant="anchor", return_lse=False, ws=None, stream=None):
    """O = block-sparse attention(Q, K, V), bf16 [B, H, N, 128] in and out."""
    B, H, N, D = Q.shape
    p = params(B, H, N, top_k, prefix, variant, D=D)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if return_lse else None
    if ws is None:
        ws = workspace(p, Q.device)
    bsa_forward(p, Q, K, V, O, lse, ws, stream)
    return (O, lse) if return_lse else O


def fp8_operands(p: bsa_params, device="cuda"):
    """One FP8 operand set in a fresh device buffer: (buffer, struct, views).

    ``views`` maps each field of bsa_fp8_operands to a torch view of the
    buffer with the documented shape (codes as uint8)."""
    n = bsa_fp8_operands_bytes(p)
    if n == 0:
        raise BsaError(BSA_ERR_INVALID, "bsa_fp8_operands_bytes")
    buf = torch.empty(n, dtype=torch.uint8, device=device)
    ops = bsa_fp8_operands_carve(p, buf)
    B, H, N = p.B, p.H, p.N
    nb = bsa_num_blocks(p)
    nt = -(-nb // 128)
    shapes = dict(q8=(B, H, N, 128), q_scale=(B, H, nb), k8=(B, H, N, 128), k_scale=(B, H, nb),
                  vt8=(B, H, nb, 128, 128), v_scale=(B, H, nb), ks8=(B, H, nb, 128),
                  ks_scale=(B, H, nt), vst8=(B, H, nt, 128, 128), vs_scale=(B, H, nt),
                  v_ref=(B, H))
    base = buf.data_ptr()
    views = {}
    for name, shape in shapes.items():
        off = getattr(ops, name) - base
        count = math.prod(shape)
        if name.endswith("8"):
            views[name] = buf[off:off + count].view(shape)
        else:
            views[name] = buf[off:off + 4 * count].view(torch.float32).view(shape)
    return buf, ops, views


def forward_fp8(Q, K, V, top_k, prefix=0, variant="anchor", return_lse=False, ws=None,
                stream=None):
    """bsa_forward_fp8: the same call as ``forward`` with e4m3 attention operands."""
    B, H, N, D = Q.shape
    p = params(B, H, N, top_k, prefix, variant, D=D)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if return_lse else None
    if ws is None:
        ws = torch.empty(bsa_forward_fp8_workspace_bytes(p), dtype=torch.uint8, device=Q.device)
    bsa_forward_fp8(p, Q, K, V, O, lse, ws, stream)
    return (O, lse) if return_lse else O


def forward_threshold(Q, K, V, tau, prefix=0, variant="anchor", return_lse=False, ws=None,
                      stream=None):
    """bsa_forward_threshold: block-sparse attention whose lists keep the key
    blocks at least tau standard deviations above each row's mean score."""
    B, H, N, D = Q.shape
    p = params(B, H, N, 1, prefix, variant, D=D)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=Q.device) if return_lse else None
    if ws is None:
        ws = torch.empty(bsa_forward_threshold_workspace_bytes(p), dtype=torch.uint8,
                         device=Q.device)
    bsa_forward_threshold(p, tau, Q, K, V, O, lse, ws, stream)
    return (O, lse) if return_lse else O


def topk_from_density(rho: float, N: int, prefix: int = 0) -> int:
    """Key-block ratio -> integer top_k = ceil(rho * nbv) (the caller's conversion)."""
    nbv = -(-N // 128) - prefix // 128
    return max(1, math.ceil(rho * nbv - 1e-9))
