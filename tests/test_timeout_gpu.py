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
from parity_helpers import DeviceRun, seeded_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()
    bsa.lib()


def test_stalled_wait_reports_timeout_and_context_survives():
    cfg = config("tiny")
    (q, k, v), _ = seeded_inputs(cfg, seed=777)
    run = DeviceRun(cfg, q, k, v)          # a normal call first
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


def test_timeout_without_status_word_is_readable_from_the_default_word():
    """dev_status = NULL: the timeout lands in the library's own word, which
    bsa_take_default_status reports once and clears."""
    cfg = config("tiny")
    (q, k, v), _ = seeded_inputs(cfg, seed=778)
    run = DeviceRun(cfg, q, k, v)
    attn = run.attn
    assert bsa.take_default_status() == 0
    o = torch.empty_like(attn.op)
    bsa.debug_stall_pv(True)
    try:
        bsa.sparse_attn_fwd(run.prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, attn.idx,
                            attn.cnt, o, None)
    finally:
        bsa.debug_stall_pv(False)
    assert bsa.take_default_status() == 6
    assert bsa.take_default_status() == 0          # cleared by the read
    bsa.sparse_attn_fwd(run.prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, attn.idx,
                        attn.cnt, o, None)
    assert bsa.take_default_status() == 0
    assert torch.equal(o, attn.op)


def test_stall_hook_affects_only_the_calling_thread():
    """A thread that turned the test hook on does not stall launches queued
    by another thread."""
    import threading
    cfg = config("tiny")
    (q, k, v), _ = seeded_inputs(cfg, seed=779)
    run = DeviceRun(cfg, q, k, v)
    attn = run.attn
    on = threading.Event()
    done = threading.Event()

    def holder():
        bsa.debug_stall_pv(True)
        on.set()
        done.wait(60)
        bsa.debug_stall_pv(False)

    t = threading.Thread(target=holder)
    t.start()
    try:
        assert on.wait(60)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        o = torch.empty_like(attn.op)
        bsa.sparse_attn_fwd(run.prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, attn.idx,
                            attn.cnt, o, status)
        torch.cuda.synchronize()
    finally:
        done.set()
        t.join()
    assert int(status.item()) == 0
    assert torch.equal(o, attn.op)
