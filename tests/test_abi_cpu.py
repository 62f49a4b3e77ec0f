"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every symbol include/bsa.h declares, sizes match the workload
arithmetic, the keep-count closed form agrees with the oracle's exact
rational version, and invalid arguments are rejected before any launch."""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_attention_47_b200 as bsa
from gen import CONFIGS, SWEEP_KEEP_RATIOS, config, derived_sizes
from oracle import bsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from block_sparse_attention_47_b200 import build
    build.build()
    return bsa.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) == 24, names
    for n in names:
        assert hasattr(bsa.lib(), n), n
    assert set(names) == set(bsa._SIGS), "binding and header disagree"


def test_struct_layout_matches_header():
    # 10 int32 + 8 int32 prefix + keep + mode + 2 floats
    assert ctypes.sizeof(bsa.Problem) == 4 * (10 + 8 + 2 + 2)
    assert ctypes.sizeof(bsa.Sizes) == 8 * 13


def test_keep_count_matches_oracle():
    for n in (1, 2, 3, 7, 32, 504, 1440, 1920, 2016, 5000):
        for r in (0.0, 0.001, 0.01, 0.03, 0.05, 0.0625, 0.0664, 0.0793, 0.1, 0.25, 0.5, 0.75, 1.0):
            assert bsa.keep_count(n, r) == O.keep_count(n, r), (n, r)
    assert bsa.keep_count(0, 0.5) == -1
    assert bsa.keep_count(10, 1.5) == -1
    assert bsa.keep_count(10, float("nan")) == -1


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_query_sizes_match_workload(name):
    cfg = config(name)
    p = bsa.Problem.make(**cfg)
    s = bsa.query_sizes(p)
    d = derived_sizes(cfg)
    assert (s.n_tokens, s.n_prefix_tokens, s.n_blocks, s.n_prefix_blocks, s.n_video_blocks) == \
        (d["N"], d["P"], d["nb"], d["nbp"], d["nbv"])
    assert s.list_capacity == d["nbp"] + O.keep_count(d["nbv"], cfg["keep_ratio"])
    assert s.perm_tensor_bytes == cfg["B"] * cfg["heads"] * d["N"] * cfg["head_dim"] * 2
    assert s.idx_bytes == cfg["B"] * cfg["heads"] * d["nb"] * s.list_capacity * 4
    if cfg["block_mode"] == 1:
        assert s.n_regions == (cfg["T"] // 8) * (cfg["H"] // 8) * (cfg["W"] // 8)


def test_sweep_keep_counts():
    nbv = derived_sizes(config("sweep"))["nbv"]
    assert [bsa.keep_count(nbv, r) for r in SWEEP_KEEP_RATIOS] == [360, 144, 115, 96, 72, 44, 15]


def base(**kw):
    d = dict(B=1, heads=2, head_dim=64, T=8, H=16, W=16, keep_blocks=8)
    d.update(kw)
    return bsa.Problem.make(**d)


BAD_PROBLEMS = [
    (dict(head_dim=96), 3), (dict(head_dim=0), 3), (dict(B=0), 2), (dict(heads=0), 2),
    (dict(T=6), 2), (dict(W=0), 2), (dict(H_valid=12), 2), (dict(T_valid=0), 2),
    (dict(T_valid=9), 2), (dict(keep_blocks=0), 2), (dict(keep_blocks=33), 2),
    (dict(block_mode=2), 1), (dict(block_mode=1, W=12), 2), (dict(block_mode=1, H_valid=14), 2),
    (dict(block_mode=1, dyn_tau=float("nan")), 1), (dict(block_mode=1, dyn_tau=0.5), 1),
    (dict(softmax_scale=0.0), 1), (dict(softmax_scale=float("inf")), 1),
    (dict(prefix=(8192 * 64,)), 3),  # 8,224 blocks: more than the attention kernel walks
    (dict(prefix=(0,)), 2),
]


@pytest.mark.parametrize("kw,status", BAD_PROBLEMS, ids=[str(k) for k, _ in BAD_PROBLEMS])
def test_invalid_problems_rejected(kw, status):
    p = base(**kw)
    s = bsa.Sizes()
    rc = bsa.lib().bsa_query_sizes(ctypes.byref(p), ctypes.byref(s))
    assert rc == status, (rc, bsa.lib().bsa_last_error())
    assert bsa.lib().bsa_last_error().decode()
    # every entry point rejects it the same way, before touching CUDA
    rc2 = bsa.lib().bsa_permute(ctypes.byref(p), 16, 16, 8, 8, 8, 16, None)
    assert rc2 == status


def test_too_many_prefix_segments():
    p = base()
    p.n_prefix_segments = 9
    assert bsa.lib().bsa_query_sizes(ctypes.byref(p), ctypes.byref(bsa.Sizes())) == 2


def test_null_and_misaligned_pointers_rejected():
    p = base()
    L = bsa.lib()
    assert L.bsa_permute(ctypes.byref(p), None, 16, 8, 8, 8, 16, None) == 1
    assert b"layout_buf" in L.bsa_last_error()
    assert L.bsa_permute(ctypes.byref(p), 16, 24, 8, 8, 8, 16, None) == 1
    assert b"aligned" in L.bsa_last_error()
    assert L.bsa_permute(ctypes.byref(p), 16, 16, 8, 12, 8, 16, None) == 1  # stride not %8
    assert L.bsa_sparse_attn_fwd(ctypes.byref(p), 16, 16, 16, 16, None, 16, 16, None, None) == 1
    assert L.bsa_sparse_attn_fwd(ctypes.byref(p), 16, 16, 16, 16, 16, 16, 16, 2, None) == 1
    assert L.bsa_select_topk(ctypes.byref(p), 16, 16, 16, None, None) == 1
    assert L.bsa_pool(ctypes.byref(p), 16, 16, 16, 16, 8, None) == 1
    assert L.bsa_unpermute(ctypes.byref(p), 16, 16, None, 8, 8, 8, None) == 1
    assert L.bsa_layout(None, None, 0, 0, 0, 16, None) == 1
    hist = (ctypes.c_int64 * 7)()
    assert L.bsa_layout_stats(ctypes.byref(p), 16, None, None) == 1
    # fixed-mode stats need no device
    assert L.bsa_layout_stats(ctypes.byref(p), 16, hist, None) == 0
    assert list(hist) == [32, 0, 0, 0, 0, 0, 0]


def test_status_strings():
    for code, name in bsa.STATUS.items():
        assert bsa.lib().bsa_status_string(code).decode() == name
    assert bsa.lib().bsa_status_string(99).decode() == "BSA_ERR_UNKNOWN"


def test_take_default_status_validation():
    L = bsa.lib()
    assert L.bsa_take_default_status(None, None) == 1
    assert b"out" in L.bsa_last_error()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_reports_cuda_error():
    p = base()
    rc = bsa.lib().bsa_permute(ctypes.byref(p), 16, 16, 8, 8, 8, 16, None)
    assert rc == 5
    with pytest.raises(bsa.BSAError):
        bsa._check(rc)


def host_buffers(**bad):
    b = bsa.DeviceBuffers()
    for name, _ in bsa.DeviceBuffers._fields_:
        setattr(b, name, 16)
    for name, v in bad.items():
        setattr(b, name, v)
    return b


def test_forward_host_validation():
    """bsa_forward_host rejects bad arguments before touching the device."""
    p = base()
    L = bsa.lib()
    P = ctypes.byref(p)
    ok = host_buffers()
    assert L.bsa_forward_host(P, None, 16, 16, 16, ctypes.byref(ok), 1, None, None) == 1
    assert b"host" in L.bsa_last_error()
    assert L.bsa_forward_host(P, 16, 16, 16, 16, None, 1, None, None) == 1
    assert L.bsa_forward_host(P, 16, 16, 16, 16, ctypes.byref(host_buffers(v_perm=24)), 1,
                              None, None) == 1
    assert b"v_perm" in L.bsa_last_error()
    assert L.bsa_forward_host(P, 16, 16, 16, 16, ctypes.byref(host_buffers(idx=18)), 1,
                              None, None) == 1
    assert b"idx" in L.bsa_last_error()
    for hg in (0, -1, p.heads + 1):
        assert L.bsa_forward_host(P, 16, 16, 16, 16, ctypes.byref(ok), hg, None, None) == 1
    if p.heads > 1:
        assert L.bsa_forward_host(P, 16, 16, 16, 16, ctypes.byref(ok), p.heads + 1, None,
                                  None) == 1


def test_forward_host_int32_lists_need_4_byte_alignment_only():
    # idx/cnt at 4-byte (not 16-byte) boundaries pass validation; without a
    # GPU the call then stops at the device check
    p = base()
    L = bsa.lib()
    b = host_buffers(idx=20, cnt=36)
    st = L.bsa_forward_host(ctypes.byref(p), 16, 16, 16, 16, ctypes.byref(b), 1, None, None)
    assert st == 5, L.bsa_last_error()


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without libbsa.so every call that needs it raises."""
    monkeypatch.setattr(bsa, "_LIB", None)
    monkeypatch.setattr(bsa, "LIB_PATH", str(tmp_path / "libbsa.so"))
    with pytest.raises(ImportError):
        bsa.lib()
    with pytest.raises(ImportError):
        bsa.keep_count(1920, 0.25)
    p = base()
    with pytest.raises(ImportError):
        bsa.BlockSparseAttention(p, device="cpu")


def test_last_error_is_per_thread():
    """bsa_last_error() reports the calling thread's own failure."""
    import threading
    L = bsa.lib()
    barrier = threading.Barrier(2)
    seen = {}

    def fail_with(key, **bad):
        p = base(**bad)
        for _ in range(200):
            barrier.wait()
            st = L.bsa_query_sizes(ctypes.byref(p), ctypes.byref(bsa.Sizes()))
            barrier.wait()  # the other thread has made its own failing call too
            seen.setdefault(key, set()).add((st, L.bsa_last_error()))

    threads = [threading.Thread(target=fail_with, args=("dim",), kwargs=dict(head_dim=96)),
               threading.Thread(target=fail_with, args=("batch",), kwargs=dict(B=0))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert len(seen["dim"]) == 1 and len(seen["batch"]) == 1
    (st_d, msg_d), = seen["dim"]
    (st_b, msg_b), = seen["batch"]
    assert st_d == 3 and b"head_dim" in msg_d
    assert st_b == 2 and b"B and heads" in msg_b


def test_raster_attention_validation():
    """The raster attention call needs heads contiguous in a token row
    (stride_h == head_dim) and is refused before any launch otherwise."""
    p = base()              # head_dim 64
    L = bsa.lib()
    P = ctypes.byref(p)
    args = lambda sh, osh=64: (P, 16, 16, 16, 16, 4096, 128, sh, 16, 16, 16, 4096, 128, osh,
                               None, None)
    assert L.bsa_sparse_attn_fwd_raster(*args(128)) == 3
    assert b"stride_h" in L.bsa_last_error()
    assert L.bsa_sparse_attn_fwd_raster(*args(60)) == 1        # not a multiple of 8
    assert L.bsa_sparse_attn_fwd_raster(P, 16, 16, 16, 16, 4096, 128, 64, None, 16, 16, 4096,
                                        128, 64, None, None) == 1
    assert b"idx" in L.bsa_last_error()
    assert L.bsa_pool_raster(P, 16, 16, 24, 4096, 128, 64, 16, 16, None) == 1
    if not torch.cuda.is_available():
        assert L.bsa_sparse_attn_fwd_raster(*args(64)) == 5    # valid: stops at the device check
