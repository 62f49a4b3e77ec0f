"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (the whole six-call sequence through BlockSparseAttention
on seeded device inputs).  The fp64 oracle checks what it can compute in
seconds: the full layout maps (bit-exact), and for a seeded sample of
(batch, head) pairs the permuted rows (bit-exact), block means, every index
list (valid against the oracle's fp32 scores, equal outside the near-tie
band), and the attention output of sampled query blocks (first, last,
prefix and padded blocks included) against fp64."""
import math

import numpy as np
import pytest
import torch

from gen import config, make_qkv
from oracle import bsa_oracle as O
from parity_helpers import (DeviceRun, assert_close, decode_map, matched_lists, sample_blocks,
                            scale_of, to_np64)

pytestmark = pytest.mark.gpu

FULL = [
    ("720p", {}),
    ("720p", {"keep_ratio": 0.0625}),
    ("720p_dyn", {}),
    ("ref_prefix", {}),
    ("lowres", {}),
    ("lowres", {"keep_ratio": 1.0}),
    ("sweep", {"keep_ratio": 0.10}),
    ("sweep", {"keep_ratio": 0.03}),
    ("sweep", {"keep_ratio": 0.01}),
    # 2,560 blocks: the selection's 8-query-block form (16 do not fit next to
    # the scores in shared memory)
    ("720p", {"B": 1, "heads": 2, "H": 64, "H_valid": 64}),
]


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()


def bh_sample(cfg, rng, count=3):
    count = min(count, cfg["B"] * cfg["heads"])
    pairs = {(0, 0), (cfg["B"] - 1, cfg["heads"] - 1)}
    while len(pairs) < count:
        pairs.add((int(rng.integers(0, cfg["B"])), int(rng.integers(0, cfg["heads"]))))
    return sorted(pairs)


# the permute-free path (raster tensors read through tensor-map boxes)
FULL_RASTER = [
    ("720p", {}),
    ("720p_dyn", {}),
    ("ref_prefix", {}),
    ("lowres", {}),
]


def _ids(cases):
    return ["%s%s" % (n, "-" + "-".join("%s=%s" % kv for kv in o.items()) if o else "")
            for n, o in cases]


@pytest.mark.parametrize("name,over", FULL, ids=_ids(FULL))
def test_full_size_parity(name, over):
    check_full_size(name, over)


@pytest.mark.parametrize("name,over", FULL_RASTER, ids=_ids(FULL_RASTER))
def test_full_size_parity_raster(name, over):
    check_full_size(name, over, raster=True)


def check_full_size(name, over, raster=False):
    """The checks of one full-size workload (also used by the maximum-size
    test, which runs last).  raster=True runs the permute-free path, which
    has no permuted tensors to compare."""
    cfg = config(name, **over)
    rng = np.random.default_rng(1234)
    q, k, v = make_qkv(cfg, 42000 + len(name), pad_fill=1e4, device="cuda")
    run = DeviceRun(cfg, q, k, v, raster=raster)
    geo = O.Geometry(cfg)
    keep = run.prob.keep_blocks
    assert keep == O.keep_count(geo.nbv, cfg["keep_ratio"])
    valid = geo.token_valid()

    # layout: full maps, bit-exact (dynamic codes up to the near-tie band)
    perms = []
    for b in range(geo.B):
        if cfg["block_mode"] == 1:
            kb = to_np64(k[b])
            vr = O.region_variation(geo, kb)
            want = np.array([O.shape_code(vr[r], cfg["dyn_tau"]) for r in range(len(vr))])
            got = run.codes[b].astype(np.int64)
            for r in np.nonzero(got != want)[0]:
                top = vr[r].max()
                near = (abs(top - cfg["dyn_tau"] * vr[r].min()) < 1e-4 * top or
                        np.sort(np.abs(vr[r][:, None] - vr[r][None, :]).ravel())[3] < 1e-4 * top)
                assert near, "region %d code %d vs oracle %d" % (r, got[r], want[r])
            nondefault = float((got != 0).mean())
            assert 0.2 <= nondefault <= 0.8, nondefault
            perm = O.dynamic_perm(geo, got)  # same codes -> the map must be identical
        else:
            perm = O.fixed_perm(geo)
        gperm, gpad = decode_map(run.perm[b])
        assert np.array_equal(gperm, perm)
        assert np.array_equal(gpad, ~valid[perm])
        perms.append(perm)

    idx, cnt = run.attn.idx.cpu().numpy(), run.attn.cnt.cpu().numpy()
    gq_pool, gk_pool = run.attn.q_pool.cpu().numpy(), run.attn.k_pool.cpu().numpy()
    out = run.out
    for b, hh in bh_sample(cfg, rng):
        perm = perms[b]
        host = [to_np64(t[b, :, hh]) for t in (q, k, v)]
        op = [O.permute(geo, perm, x) for x in host]
        # permuted rows, bit-exact
        for t_dev, ref in zip((run.attn.qp, run.attn.kp, run.attn.vp), op):
            if not raster:
                assert np.array_equal(to_np64(t_dev[b, hh]), ref)
        qpool, kpool = O.pool(geo, perm, op[0]), O.pool(geo, perm, op[1])
        np.testing.assert_allclose(gq_pool[b, hh], qpool, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(gk_pool[b, hh], kpool, rtol=1e-5, atol=1e-5)
        # every index list of this (b, h)
        S = O.block_scores_f32(geo, qpool, kpool)
        assert np.all(cnt[b, hh, :geo.nbp] == -1)
        assert np.all(cnt[b, hh, geo.nbp:] == geo.nbp + keep)
        gl = idx[b, hh, geo.nbp:, :geo.nbp + keep]
        assert np.all(gl[:, :geo.nbp] == np.arange(geo.nbp))
        vid = gl[:, geo.nbp:] - geo.nbp
        assert np.all(np.diff(vid, axis=1) > 0) if keep > 1 else True
        kth = -np.partition(-S, keep - 1, axis=1)[:, keep - 1]
        band = 1e-4 * np.abs(S).max(axis=1)
        chosen = np.zeros_like(S, dtype=bool)
        np.put_along_axis(chosen, vid, True, axis=1)
        assert not np.any(~chosen & (S > (kth + band)[:, None])), "a clearly better block was dropped"
        assert not np.any(chosen & (S < (kth - band)[:, None])), "a clearly worse block was kept"
        # attention on sampled query blocks, every one compared: the oracle's
        # list for a block is its own valid selection equal to the GPU's
        extra = []
        if cfg["H_valid"] < cfg["H"]:
            extra.append(geo.nbp + (geo.nbv - 1))
        blocks = sample_blocks(geo, 8, rng, extra)
        lists = matched_lists(geo, S, idx[b, hh], keep, rows=blocks)
        want = O.block_sparse_attention(geo, perm, *op, lists, scale_of(cfg), blocks)
        got_raster = to_np64(out[b, :, hh])
        for i in blocks:
            slots = perm[i * 64:(i + 1) * 64]
            assert_close(got_raster[slots], want[i], "%s b%d h%d block %d" % (name, b, hh, i))
    pad = torch.from_numpy(~valid).to(out.device)
    assert not bool(out[:, pad].any()), "pad tokens must come out as 0"
    assert int(run.attn.status.item()) == 0
