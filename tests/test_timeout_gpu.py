"""The attention kernel's timeout path on the GPU, triggered on purpose.

With the bsa_debug_stall_pv test hook no PV product is issued, so the
softmax's bounded wait on the first PV runs out (2 s).  The kernel must then
report BSA_ERR_TIMEOUT through the status word and return without a fault,
and a normal call on the same context afterwards must be correct."""
import numpy as np
import pytest
import torch

import block_sparse_attention_47_b200 as bsa
from gen import config
from parity_helpers import GpuRun, seeded_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()
    bsa.lib()


def test_stalled_wait_reports_timeout_and_context_survives():
    cfg = config("tiny")
    (q, k, v), _ = seeded_inputs(cfg, seed=777)
    run = GpuRun(cfg, q, k, v)          # a normal call first
    good = run.out.clone()
    attn = run.attn
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.empty_like(attn.op)
    bsa.debug_stall_pv(True)
    try:
        bsa.sparse_attn_fwd(run.prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, attn.idx,
                            attn.cnt, o, status)
        torch.cuda.synchronize()        # returns: the kernel gave up, it did not hang
    finally:
        bsa.debug_stall_pv(False)
    assert int(status.item()) == 6, "expected BSA_ERR_TIMEOUT"
    # the context is still usable and a normal call is unaffected
    again = attn(q, k, v)
    torch.cuda.synchronize()
    attn.check_status()
    assert torch.equal(again, good)
    assert np.isfinite(again.float().cpu().numpy()).all()
