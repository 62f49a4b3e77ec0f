"""bsa_forward_noalloc: the whole call for callers that cannot allocate device
memory (a plugin handed only its tensors, a runtime with a fixed memory pool,
a loop that must not call cudaMalloc).  Its intermediates live in the
library's static scratch array instead of caller buffers.

The GPU test calls it through the C ABI twice in a row, on two different
problems, so the second call runs on scratch the first one left behind, and
compares each output with the output of the ordinary entry points (which
take caller buffers) on the same inputs, within the tolerance of the other
parity tests.  The file name sorts last so that, in a run that stops at the
first failure, every other test has already run."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_47_b200 as bsa
from gen import config
from parity_helpers import assert_close, problem, seeded_inputs, to_np64

CASES = {
    "tiny": config("tiny"),
    "ragged": dict(config("tiny"), B=2, heads=3, head_dim=128, T=8, H=12, W=20, T_valid=7,
                   H_valid=10, W_valid=17, prefix=(40, 64, 1), keep_ratio=0.3, name="ragged"),
}


def test_oversized_problem_is_refused_before_any_launch():
    """A problem whose intermediates do not fit the static scratch is refused
    on the host with the byte counts; no CUDA call is made."""
    p = problem(config("lowres"))
    rc = bsa.lib().bsa_forward_noalloc(ctypes.byref(p), 16, 16, 16, 8, 8, 8, 16, 8, 8, 8, None,
                                       None)
    assert rc == 4, bsa.lib().bsa_last_error()          # BSA_ERR_WORKSPACE
    msg = bsa.lib().bsa_last_error().decode()
    assert "scratch" in msg and str(bsa.NOALLOC_SCRATCH_BYTES) in msg


@pytest.mark.gpu
def test_noalloc_matches_the_buffered_entry_points_on_two_calls_in_a_row(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()
    for name in ("tiny", "ragged"):
        cfg = CASES[name]
        (q, k, v), _ = seeded_inputs(cfg, seed=9100 + len(name))
        prob = problem(cfg)
        # the ordinary path, with caller-owned buffers
        attn = bsa.BlockSparseAttention(prob)
        want = attn(q, k, v)
        # the path without caller buffers, through the C ABI
        got = torch.full_like(q, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        bsa.forward_noalloc(prob, q, k, v, got, status)
        torch.cuda.synchronize()
        attn.check_status()
        assert int(status.item()) == 0, name
        g, w = to_np64(got), to_np64(want)
        assert np.isfinite(g).all(), name
        assert_close(g, w, "noalloc " + name)
