"""Pins of the oracle's window heads (spatial / temporal attention patterns)
and of its full / boundary / empty tile classes, to facts outside the
window code itself:

* an unbounded window is dense attention: torch fp64 SDPA with a key mask;
* a spatial head with w_t = 0 is dense attention inside each frame (plus the
  prefix): one SDPA call per frame on that frame's tokens;
* a temporal head with w_y = w_x = 0 is dense attention along each pixel's
  time line (plus the prefix): one SDPA call per (y, x);
* a brute-force loop over query tokens with explicit comparisons;
* tile-class counts worked by hand for 4x4x4 blocks.
Planted mistakes at the end confirm that the pins catch an off-by-one
window, a prefix that is not kept dense, and a tile class judged on the
wrong pairs."""
import math

import numpy as np
import pytest
import torch

from gen import config, make_qkv
from oracle import bsa_oracle as O

U = O.UNBOUNDED


def prob(**kw):
    p = dict(B=1, heads=1, head_dim=16, T=8, H=8, W=8, T_valid=8, H_valid=8, W_valid=8,
             prefix=(), keep_ratio=0.25, block_mode=0, dyn_tau=1.25, blobs=0)
    p.update(kw)
    return p


def inputs(p, seed=11):
    q, k, v = make_qkv(p, seed, pad_fill=1e4)
    return [t[0, :, 0].float().numpy().astype(np.float64) for t in (q, k, v)]


def sdpa(q, k, v, key_ok, scale):
    """torch fp64 scaled_dot_product_attention with a key mask (library)."""
    qt, kt, vt = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    m = torch.from_numpy(key_ok)[None, None, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m,
                                                            scale=scale)[0, 0].numpy()


def check_unbounded_is_dense(p):
    geo = O.Geometry(p)
    q, k, v = inputs(p)
    scale = 1 / math.sqrt(geo.d)
    out = O.window_attention(geo, q, k, v, (U, U, U), scale)
    valid = geo.token_valid()
    ref = sdpa(q, k, v, valid, scale)
    assert np.abs(out[valid] - ref[valid]).max() < 1e-12
    assert not out[~valid].any()


def test_unbounded_window_is_dense_attention():
    check_unbounded_is_dense(prob())
    check_unbounded_is_dense(prob(T=4, H=8, W=12, T_valid=3, H_valid=7, W_valid=12,
                                  prefix=(30, 64)))


def check_spatial_head_is_per_frame(p):
    """w_t = 0: each frame's queries see their own frame and the prefix."""
    geo = O.Geometry(p)
    q, k, v = inputs(p)
    scale = 1 / math.sqrt(geo.d)
    out = O.window_attention(geo, q, k, v, (0, U, U), scale)
    valid = geo.token_valid()
    hw = geo.H * geo.W
    for t in range(geo.T):
        keys = np.concatenate([np.arange(geo.P), geo.P + t * hw + np.arange(hw)])
        rows = geo.P + t * hw + np.arange(hw)
        ref = sdpa(q[rows], k[keys], v[keys], valid[keys], scale)
        ok = valid[rows]
        if ok.any():
            assert np.abs(out[rows][ok] - ref[ok]).max() < 1e-12
    # prefix queries stay dense
    if geo.P:
        pre = np.arange(geo.P)
        ref = sdpa(q[pre], k, v, valid, scale)
        ok = valid[pre]
        assert np.abs(out[pre][ok] - ref[ok]).max() < 1e-12


def test_spatial_head_is_dense_within_each_frame():
    check_spatial_head_is_per_frame(prob())
    check_spatial_head_is_per_frame(prob(T=4, H=8, W=12, T_valid=3, H_valid=7, W_valid=11,
                                         prefix=(40,)))


def check_temporal_head_is_per_pixel(p):
    """w_y = w_x = 0: each pixel's queries see its own time line and the prefix."""
    geo = O.Geometry(p)
    q, k, v = inputs(p)
    scale = 1 / math.sqrt(geo.d)
    out = O.window_attention(geo, q, k, v, (U, 0, 0), scale)
    valid = geo.token_valid()
    for y in range(geo.H):
        for x in range(geo.W):
            line = geo.P + (np.arange(geo.T) * geo.H + y) * geo.W + x
            keys = np.concatenate([np.arange(geo.P), line])
            ref = sdpa(q[line], k[keys], v[keys], valid[keys], scale)
            ok = valid[line]
            if ok.any():
                assert np.abs(out[line][ok] - ref[ok]).max() < 1e-12


def test_temporal_head_is_dense_along_each_time_line():
    check_temporal_head_is_per_pixel(prob())
    check_temporal_head_is_per_pixel(prob(T=8, H=4, W=8, T_valid=7, H_valid=4, W_valid=7,
                                          prefix=(10,)))


def test_window_mask_bruteforce():
    """Token by token with plain comparisons, mixed windows, pads, prefix."""
    p = prob(T=4, H=4, W=8, T_valid=3, H_valid=4, W_valid=7, prefix=(5,))
    geo = O.Geometry(p)
    valid = geo.token_valid()
    for win in [(1, U, U), (U, 1, 2), (2, 0, 3), (0, 0, 0)]:
        m = O.window_mask(geo, win)
        for n in range(geo.N):
            for j in range(geo.N):
                if not valid[j]:
                    want = False
                elif n < geo.P or j < geo.P:
                    want = True
                else:
                    a = geo.P
                    tq, rq = divmod(n - a, geo.H * geo.W)
                    yq, xq = divmod(rq, geo.W)
                    tk, rk = divmod(j - a, geo.H * geo.W)
                    yk, xk = divmod(rk, geo.W)
                    want = all(w == U or abs(d) <= w
                               for w, d in zip(win, (tk - tq, yk - yq, xk - xq)))
                assert m[n, j] == want, (win, n, j)


def check_tile_class_counts():
    """4x4x4 blocks on an 8x16x16 grid (2 time slabs of 16 blocks, 32
    blocks): worked by hand.
      w_t = 0: same slab -> boundary (a block spans 4 frames), other slab
               -> empty: 2 * 16 * 16 = 512 boundary, 512 empty;
      w_t = 3: same slab -> full, other slab -> boundary (512 / 512);
      w_t = 7: every pair within 7 frames -> full (1,024);
      w_y = w_x = 0 (temporal): same (bh, bw) column, any slab -> boundary
               (16 columns * 2 * 2 = 64), the rest empty (960)."""
    geo = O.Geometry(config("tiny"))
    perm = O.fixed_perm(geo)
    for win, want in [((0, U, U), [512, 512, 0]), ((3, U, U), [0, 512, 512]),
                      ((7, U, U), [0, 0, 1024]), ((U, 0, 0), [960, 64, 0]),
                      ((U, U, U), [0, 0, 1024])]:
        got = np.bincount(O.tile_classes(geo, perm, win).ravel(), minlength=3).tolist()
        assert got == want, (win, got)


def test_tile_class_counts_worked_by_hand():
    check_tile_class_counts()


def check_tile_classes_with_prefix_and_pads():
    """Prefix rows and columns are full; a pad-only difference never makes a
    tile boundary (classes are judged on real tokens only)."""
    p = prob(T=4, H=8, W=8, T_valid=3, H_valid=8, W_valid=8, prefix=(70,))
    geo = O.Geometry(p)
    perm = O.fixed_perm(geo)
    c = O.tile_classes(geo, perm, (0, U, U))
    assert (c[:geo.nbp, :] == 2).all() and (c[:, :geo.nbp] == 2).all()
    # T_valid = 3 < 4: each video block spans frames 0..2 only; with w_t = 2
    # every same-slab pair of real tokens is within the window -> full
    c2 = O.tile_classes(geo, perm, (2, U, U))
    assert (c2[geo.nbp:, geo.nbp:] == 2).all()


def test_tile_classes_with_prefix_and_pads():
    check_tile_classes_with_prefix_and_pads()


# ---- planted mistakes --------------------------------------------------------
def _mask_strict(geo, window, rows=None):
    c = O.token_coords(geo)
    cq = c if rows is None else c[np.asarray(rows)]
    vid = c[:, 0] >= 0
    ok = np.ones((len(cq), geo.N), dtype=bool)
    for a in range(3):
        w = int(window[a])
        if w >= 0:
            ok &= np.abs(cq[:, None, a] - c[None, :, a]) < w
    ok |= ~vid[None, :]
    ok |= (cq[:, 0] < 0)[:, None]
    return ok & geo.token_valid()[None, :]


def _mask_sparse_prefix_queries(geo, window, rows=None):
    m = O.__dict__["_orig_window_mask"](geo, window, rows)
    c = O.token_coords(geo)
    cq = c if rows is None else c[np.asarray(rows)]
    vid = c[:, 0] >= 0
    m[cq[:, 0] < 0] &= ~vid[None, :]      # prefix queries lose the video keys
    return m


def _classes_with_pads(geo, perm, window):
    mask = O.window_mask(geo, window)[perm][:, perm] | ~O.slot_valid(geo, perm)[None, :]
    out = np.zeros((geo.nb, geo.nb), dtype=np.int64)
    for i in range(geo.nb):
        for j in range(geo.nb):
            sub = mask[i * 64:(i + 1) * 64, j * 64:(j + 1) * 64]
            out[i, j] = 2 if sub.all() else (1 if sub.any() else 0)
    return out


WINDOW_MUTATIONS = [
    ("window_mask", _mask_strict, lambda: check_spatial_head_is_per_frame(prob())),
    ("window_mask", _mask_sparse_prefix_queries,
     lambda: check_spatial_head_is_per_frame(prob(T=4, H=8, W=8, prefix=(40,)))),
    ("tile_classes", _classes_with_pads, check_tile_classes_with_prefix_and_pads),
]


@pytest.mark.parametrize("name,bad,check", WINDOW_MUTATIONS,
                         ids=["strict-window", "sparse-prefix-queries", "classes-on-pads"])
def test_planted_window_mistake_is_caught(monkeypatch, name, bad, check):
    check()
    monkeypatch.setitem(O.__dict__, "_orig_" + name, getattr(O, name))
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        check()
