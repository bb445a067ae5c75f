"""bsa_forward_noalloc: the forward path for callers that cannot allocate
device memory (framework plugins whose memory pool owns the device, servers
that reserve everything at start-up, code that cannot take cudaMalloc's
device-wide synchronisation).  Its intermediates live in the library's static
64 MiB device scratch instead of a caller workspace.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it passes on its own in a fresh
process and after the rest of the suite.
"""

import ctypes

import pytest
import torch

from block_sparse_video_bsa_b200 import bsa
from block_sparse_video_bsa_b200.inputs import make_qkv

from parity_util import check_output, host


def test_rejects_problems_larger_than_the_scratch():
    # The check runs before anything is enqueued, so no device is needed.
    p = bsa.params(1, 56, 133_644, 64)                 # ~105 MB of intermediates
    assert bsa.bsa_workspace_bytes(p) > bsa.BSA_NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(1 << 20)
    rc = bsa.lib().bsa_forward_noalloc(ctypes.byref(p), a, a, a, a, None, None)
    assert rc == bsa.BSA_ERR_SCRATCH
    assert "static scratch" in bsa.status_string(rc)
    p_ok = bsa.params(1, 56, 73_416, 64)
    assert bsa.bsa_workspace_bytes(p_ok) <= bsa.BSA_NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_dev):
    # Two different problems back to back: the second call runs over the
    # first call's leftovers in the shared scratch and must not be affected.
    cases = [
        dict(B=1, H=8, N=37_740, top_k=64, prefix=0, variant="anchor", kind="block_offset"),
        dict(B=2, H=2, N=1_500, top_k=2, prefix=256, variant="mean", kind="block_offset"),
    ]
    for i, c in enumerate(cases):
        Q, K, V = make_qkv(c["B"], c["H"], c["N"], 128, c["kind"], seed=40 + i, device=cuda_dev)
        O_ref, lse_ref = bsa.forward(Q, K, V, c["top_k"], c["prefix"], c["variant"],
                                     return_lse=True)
        p = bsa.params(c["B"], c["H"], c["N"], c["top_k"], c["prefix"], c["variant"])
        O = torch.empty_like(Q)
        lse = torch.empty_like(lse_ref)
        bsa.bsa_forward_noalloc(p, Q, K, V, O, lse)
        torch.cuda.synchronize()
        # The same deterministic kernels on the same inputs: the results must be
        # bitwise equal.  Anything read from the previous call's leftovers in the
        # shared scratch (a stale bias, an old list row) would break equality.
        assert torch.equal(O, O_ref), f"case {i}: O differs from bsa_forward"
        assert torch.equal(lse, lse_ref), f"case {i}: lse differs from bsa_forward"
        for b in range(c["B"]):
            for h in range(c["H"]):
                check_output(host(O[b, h]), host(O_ref[b, h]), c["N"])
