"""GPU parity of window heads (spatial and temporal attention patterns with
full / boundary / empty tiles) against the fp64 oracle's explicit
token x token window mask.

Small cases compare every output token; the full-size 720p case (24 heads
alternating spatial, temporal and unbounded windows, B=2) compares sampled
query blocks of sampled (batch, head) pairs.  Bars as for the other outputs:
max-abs 2e-2 and relative L2 5e-3 against fp64; pad tokens exactly 0."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_47_b200 as bsa
from gen import config, make_qkv
from oracle import bsa_oracle as O
from parity_helpers import assert_close, problem, sample_blocks, to_np64

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": config("tiny"),
    "ragged": dict(config("tiny"), B=2, heads=3, head_dim=128, T=8, H=12, W=20, T_valid=7,
                   H_valid=10, W_valid=17, prefix=(40, 64, 1), keep_ratio=0.3, name="ragged"),
    "dyn": dict(config("tiny"), B=2, heads=3, head_dim=128, T=8, H=16, W=24, T_valid=8,
                H_valid=16, W_valid=24, block_mode=1, blobs=2, keep_ratio=0.25, name="dyn"),
}

# spatial (nearby frames), temporal (same place across frames), both, unbounded
WINDOWS = [(1, -1, -1), (-1, 2, 2), (2, 3, 1), (0, -1, -1), (-1, 0, 0), (-1, -1, -1)]


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()


def run_windows(cfg, q, k, v, wins):
    prob = problem(cfg)
    attn = bsa.BlockSparseAttention(prob)
    bsa.layout(prob, k, attn.layout_buf)
    windows = torch.tensor(wins, dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    bsa.window_attn_fwd_raster(prob, attn.layout_buf, q, k, v, windows, out, attn.status)
    torch.cuda.synchronize()
    attn.check_status()
    return out


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("shift", [0, 3])
def test_window_heads_small(name, shift):
    cfg = SMALL[name]
    q, k, v = make_qkv(cfg, 4300 + len(name), pad_fill=1e4, device="cuda")
    wins = [WINDOWS[(h + shift) % len(WINDOWS)] for h in range(cfg["heads"])]
    out = to_np64(run_windows(cfg, q, k, v, wins))
    geo = O.Geometry(cfg)
    host = [to_np64(t) for t in (q, k, v)]
    scale = 1 / math.sqrt(cfg["head_dim"])
    valid = geo.token_valid()
    for b in range(geo.B):
        for hh in range(geo.h):
            want = O.window_attention(geo, host[0][b, :, hh], host[1][b, :, hh],
                                      host[2][b, :, hh], wins[hh], scale)
            assert_close(out[b, :, hh], want, "%s b%d h%d window %s" % (name, b, hh, wins[hh]))
            assert not out[b, ~valid, hh].any(), "pad tokens must come out as 0"


def test_window_heads_full_size_720p():
    cfg = config("720p")
    q, k, v = make_qkv(cfg, 4400, pad_fill=1e4, device="cuda")
    wins = [WINDOWS[h % len(WINDOWS)] for h in range(cfg["heads"])]
    out = run_windows(cfg, q, k, v, wins)
    geo = O.Geometry(cfg)
    perm = O.fixed_perm(geo)
    rng = np.random.default_rng(7)
    scale = 1 / math.sqrt(cfg["head_dim"])
    for b, hh in [(0, 0), (1, 1), (0, 3), (1, 4), (0, 5), (1, 2)]:
        blocks = sample_blocks(geo, 4, rng)
        rows = np.concatenate([perm[i * 64:(i + 1) * 64] for i in blocks])
        qb, kb, vb = (to_np64(t[b, :, hh]) for t in (q, k, v))
        want = O.window_attention(geo, qb, kb, vb, wins[hh], scale, rows=rows)
        got = to_np64(out[b, :, hh])[rows]
        assert_close(got, want, "720p b%d h%d window %s" % (b, hh, wins[hh]))
    assert not torch.isnan(out).any()
