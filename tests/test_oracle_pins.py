"""Pins of the fp64 oracle to facts outside itself.

Each check below ties one oracle function to something the pages print, a
closed form, an invariant, a textbook/library routine or a brute-force
enumeration.  The mutation tests at the end plant plausible mistakes in the
oracle (on the CPU only) and confirm that some pin catches each of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from gen import config, derived_sizes, make_qkv
from oracle import bsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_worked_numbers.txt")


def golden_rows():
    rows = []
    for line in open(GOLDEN, encoding="utf-8"):
        if line.startswith("#") or not line.strip():
            continue
        body = line.split("|")[0].split()
        rows.append(body)
    return rows


def small_prob(**kw):
    p = dict(B=1, heads=2, head_dim=16, T=8, H=8, W=8, T_valid=8, H_valid=8,
             W_valid=8, prefix=(), keep_ratio=0.25, block_mode=0, dyn_tau=1.25, blobs=0)
    p.update(kw)
    return p


def bf16_inputs(prob, seed=7, pad_fill=1e4):
    q, k, v = make_qkv(prob, seed, pad_fill=pad_fill)
    return [t.float().numpy().astype(np.float64) for t in (q, k, v)]


# --------------------------------------------------------------------------
# the pages' worked numbers
# --------------------------------------------------------------------------
def check_pages_numbers():
    for row in golden_rows():
        kind = row[0]
        if kind == "grid":
            T, H, W, approx = int(row[1]), int(row[2]), int(row[3]), int(row[5])
            geo = O.Geometry(small_prob(T=T, H=H, W=W, T_valid=T, H_valid=H, W_valid=W))
            assert geo.N == T * H * W
            assert round(geo.N, -3) == approx
            assert geo.nbv == 1920
        elif kind == "keep":
            n, r, k = int(row[1]), float(row[2]), int(row[3])
            assert O.keep_count(n, r) == k
        elif kind == "block":
            assert math.prod(map(int, row[1:4])) == int(row[4]) == O.BLOCK
            assert O.SHAPES[0] == tuple(map(int, row[1:4]))
        elif kind == "region":
            for s in O.SHAPES:
                assert math.prod(s) == int(row[4])
                assert all(int(row[1]) % a == 0 for a in s)
        elif kind == "calls":
            assert int(row[1]) * int(row[2]) * int(row[3]) == int(row[4])


def test_pages_worked_numbers():
    check_pages_numbers()


KEEP_TABLE = [  # closed form max(1, ceil(r*n)) worked by hand
    (1920, 0.25, 480), (1920, 0.0625, 120), (504, 0.25, 126), (32, 0.25, 8),
    (2016, 0.25, 504), (1440, 0.25, 360), (1440, 0.10, 144), (1440, 0.0793, 115),
    (1440, 0.0664, 96), (1440, 0.05, 72), (1440, 0.03, 44), (1440, 0.01, 15),
    (10, 0.0, 1), (10, 1.0, 10), (7, 0.5, 4), (3, 0.001, 1)]


def check_keep_count():
    for n, r, k in KEEP_TABLE:
        assert O.keep_count(n, r) == k, (n, r)


def test_keep_count_closed_form():
    check_keep_count()


# --------------------------------------------------------------------------
# layout
# --------------------------------------------------------------------------
def coords(geo, raster):
    r = raster - geo.P
    t, rem = divmod(r, geo.H * geo.W)
    y, x = divmod(rem, geo.W)
    return t, y, x


def check_fixed_layout(prob):
    geo = O.Geometry(prob)
    perm = O.fixed_perm(geo)
    assert sorted(perm.tolist()) == list(range(geo.N))  # bijection
    assert perm[:geo.P].tolist() == list(range(geo.P))   # prefix untouched
    nbw, nbh = geo.W // 4, geo.H // 4
    for j in range(geo.nbv):
        slots = perm[geo.P + 64 * j: geo.P + 64 * (j + 1)]
        bt, rem = divmod(j, nbh * nbw)
        bh, bw = divmod(rem, nbw)
        cs = [coords(geo, int(s)) for s in slots]
        # the block is exactly the 4x4x4 cube at (bt, bh, bw)
        want = {(4 * bt + a, 4 * bh + b, 4 * bw + c)
                for a in range(4) for b in range(4) for c in range(4)}
        assert set(cs) == want
        # tokens inside the block in raster order
        assert list(slots) == sorted(slots)


def test_fixed_layout_cubes_and_bijection():
    check_fixed_layout(small_prob())
    check_fixed_layout(small_prob(T=4, H=12, W=8, T_valid=3, H_valid=11, W_valid=8,
                                  prefix=(5, 64, 70)))


def check_dynamic_tiling(prob, codes):
    geo = O.Geometry(prob)
    perm = O.dynamic_perm(geo, codes)
    assert sorted(perm.tolist()) == list(range(geo.N))
    nr_h, nr_w = geo.H // 8, geo.W // 8
    for r, code in enumerate(codes):
        rt, rem = divmod(r, nr_h * nr_w)
        rh, rw = divmod(rem, nr_w)
        region = perm[geo.P + 512 * r: geo.P + 512 * (r + 1)]
        cs = [coords(geo, int(s)) for s in region]
        # the region's 8 blocks tile exactly its 512 tokens
        assert set(cs) == {(8 * rt + a, 8 * rh + b, 8 * rw + c)
                           for a in range(8) for b in range(8) for c in range(8)}
        st, sh, sw = O.SHAPES[code]
        for blk in range(8):
            bc = cs[64 * blk: 64 * (blk + 1)]
            ts, ys, xs = zip(*bc)
            # each block is a box of the coded shape, holding 64 tokens
            assert (max(ts) - min(ts) + 1, max(ys) - min(ys) + 1, max(xs) - min(xs) + 1) == (st, sh, sw)
            assert len(set(bc)) == 64
            assert min(ts) % st == 0 and min(ys) % sh == 0 and min(xs) % sw == 0
            raster = region[64 * blk: 64 * (blk + 1)]
            assert list(raster) == sorted(raster)


def test_dynamic_layout_tiles_regions():
    prob = small_prob(T=8, H=16, W=16, T_valid=8, H_valid=16, W_valid=16, prefix=(64,),
                      block_mode=1)
    check_dynamic_tiling(prob, [0, 1, 2, 3])
    check_dynamic_tiling(prob, [4, 5, 6, 0])


def ramp_k(prob, a, b, c):
    """K(t, y, x) = a*t + b*y + c*x on every channel: |delta| along each axis
    is exactly (a, b, c)."""
    geo = O.Geometry(prob)
    k = np.zeros((1, geo.N, geo.h, geo.d))
    t, y, x = np.meshgrid(np.arange(geo.T), np.arange(geo.H), np.arange(geo.W), indexing="ij")
    k[0, geo.P:] = (a * t + b * y + c * x).reshape(-1)[:, None, None]
    return k


RULE_CASES = [  # (a, b, c) -> expected shape (t, h, w)
    ((3.0, 2.0, 1.0), (2, 4, 8)), ((3.0, 1.0, 2.0), (2, 8, 4)),
    ((2.0, 3.0, 1.0), (4, 2, 8)), ((1.0, 3.0, 2.0), (8, 2, 4)),
    ((2.0, 1.0, 3.0), (4, 8, 2)), ((1.0, 2.0, 3.0), (8, 4, 2)),
    ((1.0, 1.0, 1.0), (4, 4, 4)), ((1.2, 1.0, 1.0), (4, 4, 4)),
    ((1.3, 1.0, 1.0), (2, 4, 8)),  # ties broken by axis order t < h < w
    ((1.0, 1.0, 1.3), (4, 8, 2)), ((1.0, 1.3, 1.3), (8, 2, 4)),
    ((0.0, 0.0, 0.0), (4, 4, 4)),
]


def check_dynamic_rule():
    prob = small_prob(block_mode=1)
    for (a, b, c), want in RULE_CASES:
        k = ramp_k(prob, a, b, c)
        geo = O.Geometry(prob)
        v = O.region_variation(geo, k[0])
        assert np.allclose(v[0], [a, b, c], rtol=0, atol=1e-12)
        assert O.SHAPES[O.shape_code(v[0], 1.25)] == want, ((a, b, c), want)


def test_dynamic_rule_short_side_on_most_changing_axis():
    check_dynamic_rule()


def test_dynamic_variation_bruteforce():
    """region_variation against a plain loop over every adjacent pair."""
    prob = small_prob(T=8, H=8, W=16, T_valid=7, H_valid=8, W_valid=15, heads=2, head_dim=3,
                      block_mode=1)
    geo = O.Geometry(prob)
    rng = np.random.default_rng(3)
    kb = rng.normal(size=(geo.N, 2, 3))
    v = O.region_variation(geo, kb)
    valid = geo.token_valid()
    for r in range(2):
        sums, cnts = [0.0] * 3, [0] * 3
        for t in range(8):
            for y in range(8):
                for x in range(8 * r, 8 * r + 8):
                    p = geo.raster_index(t, y, x)
                    for axis, (dt, dy, dx) in enumerate(((1, 0, 0), (0, 1, 0), (0, 0, 1))):
                        t2, y2, x2 = t + dt, y + dy, x + dx
                        if t2 >= 8 or y2 >= 8 or x2 >= 8 * r + 8:
                            continue
                        q = geo.raster_index(t2, y2, x2)
                        if not (valid[p] and valid[q]):
                            continue
                        sums[axis] += np.abs(kb[q] - kb[p]).sum()
                        cnts[axis] += kb[p].size
        assert np.allclose(v[r], [s / c for s, c in zip(sums, cnts)], rtol=1e-12)


# --------------------------------------------------------------------------
# pooling
# --------------------------------------------------------------------------
def check_pool():
    prob = small_prob(T=4, H=8, W=8, T_valid=3, H_valid=8, W_valid=7, prefix=(70,), head_dim=4)
    geo = O.Geometry(prob)
    perm = O.fixed_perm(geo)
    rng = np.random.default_rng(0)
    # a field constant on every block pools to that constant
    const = np.zeros((geo.N, 4))
    blk_of_slot = np.repeat(np.arange(geo.nb), 64)
    vals = rng.normal(size=(geo.nb, 4))
    const[perm] = vals[blk_of_slot]
    xp = O.permute(geo, perm, const)
    assert np.allclose(O.pool(geo, perm, xp), vals, atol=1e-14)
    # against a plain loop over valid tokens
    x = rng.normal(size=(geo.N, 4))
    valid = geo.token_valid()
    xp = O.permute(geo, perm, x)
    got = O.pool(geo, perm, xp)
    for j in range(geo.nb):
        toks = [int(perm[s]) for s in range(64 * j, 64 * j + 64) if valid[perm[s]]]
        want = sum(x[t] for t in toks) / len(toks)
        assert np.allclose(got[j], want, atol=1e-13)
    # linearity
    y = rng.normal(size=(geo.N, 4))
    a = O.pool(geo, perm, O.permute(geo, perm, 2 * x - 3 * y))
    b = 2 * O.pool(geo, perm, O.permute(geo, perm, x)) - 3 * O.pool(geo, perm, O.permute(geo, perm, y))
    assert np.allclose(a, b, atol=1e-12)


def test_pool_constant_loop_linear():
    check_pool()


def test_permute_unpermute_identity():
    prob = small_prob(T=4, H=8, W=8, T_valid=3, H_valid=7, W_valid=8, prefix=(70, 3))
    geo = O.Geometry(prob)
    perm = O.fixed_perm(geo)
    x = np.random.default_rng(1).normal(size=(geo.N, 5))
    back = O.unpermute(geo, perm, O.permute(geo, perm, x))
    valid = geo.token_valid()
    assert np.array_equal(back[valid], x[valid])
    assert not back[~valid].any()


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------
def check_topk():
    rng = np.random.default_rng(5)
    for trial in range(60):
        n = int(rng.integers(2, 11))
        k = int(rng.integers(1, n + 1))
        s = rng.integers(-3, 4, size=n).astype(np.float32)  # many exact ties
        got = O.topk_row(s, k)
        assert got == O.topk_bruteforce(s, k)
        assert got == sorted(got) and len(got) == k
        # the kept set has the largest possible score sum
        best = max(sum(s[list(c)]) for c in __import__("itertools").combinations(range(n), k))
        assert sum(s[got]) == best


def test_topk_bruteforce_and_max_sum():
    check_topk()


def check_select_structure():
    prob = small_prob(T=4, H=8, W=8, prefix=(64, 100), keep_ratio=0.5)
    geo = O.Geometry(prob)
    perm = O.fixed_perm(geo)
    rng = np.random.default_rng(2)
    qp, kp = rng.normal(size=(geo.nb, 8)), rng.normal(size=(geo.nb, 8))
    keep = O.keep_count(geo.nbv, 0.5)
    lists = O.select(geo, qp, kp, keep)
    S = (qp[geo.nbp:].astype(np.float32).astype(np.float64)
         @ kp[geo.nbp:].astype(np.float32).astype(np.float64).T)
    for i, lst in enumerate(lists):
        assert list(lst) == sorted(set(lst.tolist()))
        if i < geo.nbp:  # prefix query blocks attend densely
            assert list(lst) == list(range(geo.nb))
            continue
        assert list(lst[:geo.nbp]) == list(range(geo.nbp))  # prefix keys always kept
        vid = lst[geo.nbp:] - geo.nbp
        assert len(vid) == keep
        row = S[i - geo.nbp]
        worst_kept = row[vid].min()
        others = np.delete(row, vid)
        assert worst_kept >= others.max() - 1e-6


def test_select_structure_prefix_dense():
    check_select_structure()


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def sdpa_dense_raster(q, k, v, valid, scale):
    """torch fp64 scaled_dot_product_attention with a key-padding mask."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    mask = torch.from_numpy(valid)[None, None, None, :].expand(qt.shape[0], qt.shape[1], qt.shape[2], -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def check_sparsity0_is_dense(prob):
    geo = O.Geometry(prob)
    q, k, v = bf16_inputs(prob)
    prob = dict(prob, keep_ratio=1.0)
    out, _, _, lists = O.forward(prob, q, k, v)
    assert all(len(l) == geo.nb for lb in lists for lh in lb for l in lh)
    valid = geo.token_valid()
    ref = sdpa_dense_raster(q, k, v, valid, 1 / math.sqrt(geo.d))
    assert np.abs(out[:, valid] - ref[:, valid]).max() < 1e-12
    assert not out[:, ~valid].any()


def test_sparsity0_equals_sdpa():
    check_sparsity0_is_dense(small_prob(T=4, H=8, W=12, T_valid=4, H_valid=7, W_valid=12,
                                        heads=2, head_dim=16))
    check_sparsity0_is_dense(small_prob(T=4, H=8, W=8, prefix=(30, 64), heads=1, head_dim=8))


def test_single_video_block_with_prefix_is_dense():
    """Degenerate grid: one video block (4x4x4) behind a prefix.  Top-k has a
    single candidate, so even the lowest keep ratio keeps every block, and
    the call must equal dense attention (torch fp64 SDPA with a key mask)."""
    prob = small_prob(T=4, H=4, W=4, T_valid=4, H_valid=4, W_valid=4, prefix=(20, 64),
                      heads=2, head_dim=8, keep_ratio=0.01)
    geo = O.Geometry(prob)
    assert geo.nbv == 1 and geo.nbp == 2
    assert O.keep_count(geo.nbv, prob["keep_ratio"]) == 1
    q, k, v = bf16_inputs(prob)
    out, _, _, lists = O.forward(prob, q, k, v)
    assert all(list(l) == [0, 1, 2] for lb in lists for lh in lb for l in lh)
    valid = geo.token_valid()
    ref = sdpa_dense_raster(q, k, v, valid, 1 / math.sqrt(geo.d))
    assert np.abs(out[:, valid] - ref[:, valid]).max() < 1e-12
    assert not out[:, ~valid].any()


def masked_attention_bruteforce(prob, q, k, v, perm, lists):
    """Raster-order attention under an explicit token x token mask built from
    the kept block pairs; one pass over each row with -inf outside the mask."""
    geo = O.Geometry(prob)
    valid = geo.token_valid()
    block_of = np.empty(geo.N, dtype=np.int64)
    block_of[perm] = np.arange(geo.N) // 64
    scale = 1 / math.sqrt(geo.d)
    out = np.zeros_like(q)
    for b in range(geo.B):
        for hh in range(geo.h):
            kept = np.zeros((geo.nb, geo.nb), dtype=bool)
            for i, lst in enumerate(lists[b][hh]):
                kept[i, lst] = True
            mask = kept[block_of[:, None], block_of[None, :]] & valid[None, :]
            logits = np.where(mask, q[b, :, hh] @ k[b, :, hh].T * scale, -np.inf)
            w = np.exp(logits - logits.max(axis=1, keepdims=True))
            out[b, :, hh] = (w / w.sum(axis=1, keepdims=True)) @ v[b, :, hh]
            out[b, ~valid, hh] = 0
    return out


def check_bruteforce_mask(prob):
    q, k, v = bf16_inputs(prob)
    out, perms, _, lists = O.forward(prob, q, k, v)
    ref = masked_attention_bruteforce(prob, q, k, v, perms[0], lists)
    assert np.abs(out - ref).max() < 1e-12


def test_block_sparse_equals_bruteforce_mask_tiny():
    tiny = config("tiny")
    check_bruteforce_mask(tiny)


def test_block_sparse_bruteforce_prefix_and_pads():
    check_bruteforce_mask(small_prob(T=4, H=8, W=12, T_valid=3, H_valid=7, W_valid=11,
                                     prefix=(40, 64), keep_ratio=0.34, heads=2, head_dim=16))


def test_block_sparse_bruteforce_dynamic_layout():
    """The same brute-force pin under a dynamic layout that mixes block shapes
    (regions coded 2, 1, 2, 0), with a padded row and a prefix segment: the
    mask is built from the dynamic permutation, so a block that gathers the
    wrong tokens, or a shape applied to the wrong region, fails it."""
    prob = small_prob(T=8, H=16, W=16, T_valid=8, H_valid=15, W_valid=16, prefix=(40,),
                      block_mode=1, blobs=6, keep_ratio=0.3, heads=2, head_dim=16)
    q, k, v = bf16_inputs(prob, seed=5)
    out, perms, codes, lists = O.forward(prob, q, k, v)
    assert len(set(codes[0].tolist())) >= 3  # several shapes, not only the default
    ref = masked_attention_bruteforce(prob, q, k, v, perms[0], lists)
    assert np.abs(out - ref).max() < 1e-12


def test_dynamic_vs_fixed_same_kept_tile_count():
    """The block shape changes where attention looks, not how much ([PRISM]
    section on the dynamic-block speed)."""
    prob = small_prob(T=8, H=16, W=16, T_valid=8, H_valid=16, W_valid=16, blobs=2,
                      heads=2, head_dim=8)
    q, k, v = bf16_inputs(prob, pad_fill=0)
    counts = []
    for mode in (0, 1):
        p = dict(prob, block_mode=mode)
        _, _, codes, lists = O.forward(p, q, k, v)
        counts.append(sum(len(l) for lb in lists for lh in lb for l in lh))
    assert counts[0] == counts[1] == 2 * 32 * O.keep_count(32, 0.25)


def test_generator_pads_and_shapes():
    cfg = config("lowres", heads=2, T=4)
    q, k, v = make_qkv(cfg, 1)
    sz = derived_sizes(cfg)
    assert q.shape == (1, sz["N"], 2, 128) and q.dtype == torch.bfloat16
    geo = O.Geometry(cfg)
    valid = torch.from_numpy(geo.token_valid())
    assert (q[0, ~valid] == 1e4).all() and (q[0, valid].abs() < 100).all()


# --------------------------------------------------------------------------
# planted mistakes: each must trip at least one pin
# --------------------------------------------------------------------------
def _floor_keep(n, r):
    return int(min(n, max(1, math.floor(float(r) * n))))


def _reversed_rank(v, tau):
    v32 = np.asarray(v, dtype=np.float32)
    if v32.max() == 0 or v32.max() < np.float32(tau) * v32.min():
        return 0
    order = sorted(range(3), key=lambda a: (float(v32[a]), a))  # wrong direction
    size = [0, 0, 0]
    for rank, axis in enumerate(order):
        size[axis] = (2, 4, 8)[rank]
    return O.SHAPES.index(tuple(size))


def _pool_over_64(geo, perm, x_perm_bh):
    return x_perm_bh.reshape(geo.nb, 64, -1).sum(axis=1) / 64.0


def _topk_smallest(row, k):
    return sorted(sorted(range(len(row)), key=lambda j: (float(row[j]), j))[:k])


def _attn_keeps_pads(geo, perm, q, k, v, lists, scale, query_blocks=None):
    out = {}
    for i in (query_blocks or range(geo.nb)):
        keys = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in lists[i]])
        lg = q[i * 64:(i + 1) * 64] @ k[keys].T * scale
        e = np.exp(lg - lg.max(axis=1, keepdims=True))
        out[i] = e @ v[keys] / e.sum(axis=1, keepdims=True)
        out[i][~O.slot_valid(geo, perm)[i * 64:(i + 1) * 64]] = 0
    return out


def _fixed_perm_swapped_xy(geo):
    perm = list(range(geo.P))
    for bt in range(geo.T // 4):
        for bh in range(geo.H // 4):
            for bw in range(geo.W // 4):
                for dt in range(4):
                    for dx in range(4):
                        for dy in range(4):
                            perm.append(geo.raster_index(4 * bt + dt, 4 * bh + dy, 4 * bw + dx))
    return np.asarray(perm)


def _select_prefix_rows_sparse(geo, qp, kp, keep):
    lists = O.__dict__["_orig_select"](geo, qp, kp, keep)
    return [l if i >= geo.nbp else l[-keep:] for i, l in enumerate(lists)]


MUTATIONS = [
    ("keep_count", _floor_keep, check_keep_count),
    ("shape_code", _reversed_rank, check_dynamic_rule),
    ("pool", _pool_over_64, check_pool),
    ("topk_row", _topk_smallest, check_topk),
    ("block_sparse_attention", _attn_keeps_pads,
     lambda: check_sparsity0_is_dense(small_prob(T=4, H=8, W=12, T_valid=4, H_valid=7, W_valid=12,
                                                 heads=1, head_dim=8))),
    ("fixed_perm", _fixed_perm_swapped_xy, lambda: check_fixed_layout(small_prob())),
    ("select", _select_prefix_rows_sparse, check_select_structure),
]


@pytest.mark.parametrize("name,bad,check", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, bad, check):
    check()  # passes on the real oracle
    monkeypatch.setitem(O.__dict__, "_orig_" + name, getattr(O, name))
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        check()
