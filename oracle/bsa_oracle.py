"""fp64 CPU oracle for block-sparse video self-attention.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow definition that the
CUDA path is checked against.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it; the product package never does,
and this module imports nothing from the product package.

Every floating-point step runs in numpy float64 on exact fp64 copies of the
bf16 inputs, with no tiling, no online softmax and no fusion.  Where a float
decides an integer (a block shape code, a top-k membership) the decision is
taken on the value rounded to float32, the precision the GPU kernels decide
in; the tests accept the documented near-tie band around each decision.

Sources (the pages; section names given in the original language with a
gloss):
  [PRISM]  oh-my-gpu.com, "Prism / Kandinsky 6 speed ablation":
           "토큰 수의 제곱으로 느는 어텐션 비용" (quadratic cost: the 32x48x80
           grid, 122,880 tokens with padding);
           "같은 계산량 안에서 볼 곳을 고르는 Prism" (Prism: 64-token blocks
           judged by the mean of their tokens, top fraction of key blocks
           kept, 480 of 1,920 at sparsity 0.75; default 4x4x4 blocks;
           8x8x8 regions whose most-changing axis gets the short side);
           "동적 블록을 켜도 그대로였던 속도" (the block shape changes where
           attention looks, not how much).
  [SVG]    aibase.it, "Sparse VideoGen TPU 최적화": "이론적 sparsity와 물리적
           sparsity의 차이" (full / boundary / empty tiles; skipping empty
           tiles is the speed-up) and "실무에서 배울 최적화 기준" (token
           permutation so masks become contiguous tiles).
  [REF2VA] pulmap.app, "Ref2VA VSA": "토큰 75%를 건너뛰는 VSA" (4x4x4 tiles,
           top-k over tiles) and "조건 토큰은 왜 다르게 다루나" (text /
           reference-image / reference-audio tokens in segment-pure tiles,
           attended 100 % densely; top-k applied only to video key tiles).

Readings taken where the pages are silent (each listed in the design notes):
  * block score = dot product of the pooled query and pooled key block
    means; the softmax scale is left out as it does not change the order;
  * selection is per (batch, head); the dynamic shape is per (batch,
    region), measured on K and shared by all heads;
  * ties are broken by the lower key-block index;
  * keep = max(1, ceil(keep_ratio * n_video_blocks)) in exact arithmetic on
    the decimal keep ratio;
  * dynamic rule: v_a = mean |K(p + e_a) - K(p)| over heads, channels and
    the adjacent valid in-region pairs along axis a; if max(v) < tau*min(v)
    or max(v) == 0 the region keeps 4x4x4, else the axes ranked by (v descending, axis
    t<h<w) get sizes 2, 4, 8;
  * prefix query blocks attend to every block; video query blocks attend to
    every prefix block plus their top-k video blocks; no forced diagonal.

parity pins: see tests/test_oracle_pins.py (every function below is pinned).
"""
from fractions import Fraction
import itertools
import math

import numpy as np

# the seven 64-token block shapes (t, h, w); index = shape code
SHAPES = ((4, 4, 4), (2, 4, 8), (2, 8, 4), (4, 2, 8), (4, 8, 2), (8, 2, 4),
          (8, 4, 2))
BLOCK = 64


# --------------------------------------------------------------------------
# geometry
# --------------------------------------------------------------------------
class Geometry:
    """Token / block bookkeeping of one problem (plain integer arithmetic).

    Raster order: prefix segments first, each padded at its end to a multiple
    of 64 tokens, then video token (t, y, x) at P + (t*H + y)*W + x.
    """

    def __init__(self, prob):
        self.prob = prob
        self.B, self.h, self.d = prob["B"], prob["heads"], prob["head_dim"]
        self.T, self.H, self.W = prob["T"], prob["H"], prob["W"]
        self.Tv, self.Hv, self.Wv = prob["T_valid"], prob["H_valid"], prob["W_valid"]
        self.seg_len = list(prob["prefix"])
        self.seg_pad = [((n + BLOCK - 1) // BLOCK) * BLOCK for n in self.seg_len]
        self.seg_off = [sum(self.seg_pad[:i]) for i in range(len(self.seg_pad))]
        self.P = sum(self.seg_pad)
        self.Nv = self.T * self.H * self.W
        self.N = self.P + self.Nv
        self.nbp = self.P // BLOCK
        self.nbv = self.Nv // BLOCK
        self.nb = self.nbp + self.nbv

    def raster_index(self, t, y, x):
        return self.P + (t * self.H + y) * self.W + x

    def token_valid(self):
        """bool [N]: is the raster token a real (non-pad) token."""
        v = np.zeros(self.N, dtype=bool)
        for off, n in zip(self.seg_off, self.seg_len):
            v[off:off + n] = True
        t, y, x = np.meshgrid(np.arange(self.T), np.arange(self.H),
                              np.arange(self.W), indexing="ij")
        vid = (t < self.Tv) & (y < self.Hv) & (x < self.Wv)
        v[self.P:] = vid.reshape(-1)
        return v


def keep_count(n_blocks, keep_ratio):
    """Kept video key blocks per query block: max(1, ceil(r * n)), at most n.

    Exact rational arithmetic on the decimal the ratio was written as, so
    0.05 * 1440 is exactly 72.  [PRISM] Prism section: sparsity 0.75 keeps
    25 % of key blocks, 480 of 1,920.
    """
    r = Fraction(repr(float(keep_ratio)))
    k = math.ceil(r * n_blocks)
    return int(min(n_blocks, max(1, k)))


# --------------------------------------------------------------------------
# layout: slot -> raster token permutation
# --------------------------------------------------------------------------
def _prefix_perm(geo):
    return list(range(geo.P))


def fixed_perm(geo):
    """int64 [N]: slot s of the block-ordered sequence -> raster token.

    Fixed 4x4x4 blocks ([PRISM] Prism section, [REF2VA] VSA section):
    blocks in raster order over (bt, bh, bw), the block's 64 tokens in
    (t, y, x) raster order.  Prefix tokens keep their place.
    """
    perm = _prefix_perm(geo)
    for bt in range(geo.T // 4):
        for bh in range(geo.H // 4):
            for bw in range(geo.W // 4):
                for dt in range(4):
                    for dy in range(4):
                        for dx in range(4):
                            perm.append(geo.raster_index(4 * bt + dt, 4 * bh + dy,
                                                         4 * bw + dx))
    return np.asarray(perm, dtype=np.int64)


def dynamic_perm(geo, codes):
    """int64 [N] for one batch element given a shape code per 8x8x8 region.

    Regions in raster order over (rt, rh, rw); each region's 8 blocks are
    contiguous; inside the region, sub-blocks of shape (st, sh, sw) in raster
    order and tokens in raster order inside each sub-block ([PRISM] Prism
    section: 8x8x8 regions, blocks stay 64 tokens).
    """
    perm = _prefix_perm(geo)
    nr_h, nr_w = geo.H // 8, geo.W // 8
    for r, code in enumerate(codes):
        rt, rem = divmod(r, nr_h * nr_w)
        rh, rw = divmod(rem, nr_w)
        st, sh, sw = SHAPES[int(code)]
        for bt in range(8 // st):
            for bh in range(8 // sh):
                for bw in range(8 // sw):
                    for dt in range(st):
                        for dy in range(sh):
                            for dx in range(sw):
                                perm.append(geo.raster_index(
                                    8 * rt + st * bt + dt, 8 * rh + sh * bh + dy,
                                    8 * rw + sw * bw + dx))
    return np.asarray(perm, dtype=np.int64)


def region_variation(geo, k_raster_b, regions=None):
    """float64 [n_regions, 3]: per-axis mean |delta K| of each 8x8x8 region.

    k_raster_b: one batch element of K, [N, heads, d] (any float dtype).
    v_a averages |K(p + e_a) - K(p)| over heads, channels and every pair of
    adjacent in-region tokens along axis a that are both valid ([PRISM]
    Prism section: the change along t, h, w is measured per region).
    A region with no valid pair along some axis reports NaN for that axis.
    With `regions` given, only those rows are evaluated (the others are 0).
    """
    T, H, W = geo.T, geo.H, geo.W
    valid = geo.token_valid()[geo.P:].reshape(T, H, W)
    vid = k_raster_b[geo.P:]
    nr_t, nr_h, nr_w = T // 8, H // 8, W // 8
    out = np.zeros((nr_t * nr_h * nr_w, 3))
    wanted = None if regions is None else set(int(r) for r in regions)
    r = -1
    for rt in range(nr_t):
        for rh in range(nr_h):
            for rw in range(nr_w):
                r += 1
                if wanted is not None and r not in wanted:
                    continue
                idx = np.array([[[(8 * rt + a) * H * W + (8 * rh + b) * W + 8 * rw + c
                                  for c in range(8)] for b in range(8)] for a in range(8)])
                x = np.asarray(vid[idx.reshape(-1)], dtype=np.float64)
                x = x.reshape(8, 8, 8, -1)
                ok = valid[8 * rt:8 * rt + 8, 8 * rh:8 * rh + 8, 8 * rw:8 * rw + 8]
                for axis in range(3):
                    diff = np.abs(np.diff(x, axis=axis))
                    pair_ok = np.logical_and(
                        np.take(ok, range(7), axis=axis),
                        np.take(ok, range(1, 8), axis=axis))
                    n = pair_ok.sum()
                    if n == 0:
                        out[r, axis] = np.nan
                    else:
                        out[r, axis] = diff[pair_ok].mean()
    return out


def shape_code(v, tau):
    """Shape code from the three per-axis variations (decided in float32).

    4x4x4 (code 0) when max(v) < tau*min(v), when nothing changes at all
    (max(v) == 0), or when some axis has no valid pair; otherwise the axes ranked by (v descending, axis index ascending) get
    sizes 2, 4, 8: the most-changing axis is cut shortest ([PRISM] Prism
    section).
    """
    if np.any(np.isnan(v)):
        return 0
    v32 = np.asarray(v, dtype=np.float32)
    tau32 = np.float32(tau)
    if v32.max() == 0 or v32.max() < tau32 * v32.min():
        return 0
    order = sorted(range(3), key=lambda a: (-float(v32[a]), a))
    size = [0, 0, 0]
    for rank, axis in enumerate(order):
        size[axis] = (2, 4, 8)[rank]
    return SHAPES.index(tuple(size))


def layout(prob, k_raster=None):
    """Per batch element: (perm [N], codes or None).

    Fixed mode ignores K.  Dynamic mode measures K per region.
    """
    geo = Geometry(prob)
    out = []
    for b in range(geo.B):
        if prob["block_mode"] == 0:
            out.append((fixed_perm(geo), None))
        else:
            v = region_variation(geo, np.asarray(k_raster[b], dtype=np.float64))
            codes = np.array([shape_code(v[r], prob["dyn_tau"]) for r in range(len(v))],
                             dtype=np.int64)
            out.append((dynamic_perm(geo, codes), codes))
    return out


def slot_valid(geo, perm):
    """bool [N]: validity of each block-ordered slot."""
    return geo.token_valid()[perm]


# --------------------------------------------------------------------------
# permute / pool / select
# --------------------------------------------------------------------------
def permute(geo, perm, x_raster_bh):
    """[N, d] raster rows -> [N, d] float64 block-ordered rows, pad slots 0
    ([SVG] practical criteria: token permutation)."""
    x = np.asarray(x_raster_bh, dtype=np.float64)[perm].copy()
    x[~slot_valid(geo, perm)] = 0.0
    return x


def unpermute(geo, perm, o_perm_bh):
    """[N, d] block-ordered -> [N, d] raster, pad tokens 0."""
    o = np.zeros_like(o_perm_bh)
    ok = slot_valid(geo, perm)
    o[perm[ok]] = o_perm_bh[ok]
    return o


def pool(geo, perm, x_perm_bh):
    """float64 [nb, d]: mean of each block's valid tokens ([PRISM] Prism
    section: a block is judged by the mean of its 64 tokens)."""
    ok = slot_valid(geo, perm).reshape(geo.nb, BLOCK)
    x = x_perm_bh.reshape(geo.nb, BLOCK, -1)
    out = np.zeros((geo.nb, x.shape[-1]))
    for j in range(geo.nb):
        n = ok[j].sum()
        if n == 0:
            raise ValueError("block %d holds no valid token" % j)
        out[j] = x[j][ok[j]].sum(axis=0) / n
    return out


def block_scores_f32(geo, q_pool, k_pool):
    """float32 [nbv, nbv] scores of video query blocks against video key
    blocks: the dot product of the pooled means (pooled values first rounded
    to float32, the dot product taken in float64 and rounded to float32)."""
    qp = np.asarray(q_pool, dtype=np.float32).astype(np.float64)[geo.nbp:]
    kp = np.asarray(k_pool, dtype=np.float32).astype(np.float64)[geo.nbp:]
    return (qp @ kp.T).astype(np.float32)


def topk_row(scores_row, k):
    """Indices of the k best entries by (score descending, index ascending),
    returned in ascending index order."""
    order = sorted(range(len(scores_row)), key=lambda j: (-float(scores_row[j]), j))
    return sorted(order[:k])


def select(geo, q_pool, k_pool, keep, rows=None):
    """Kept key-block lists for every query block of one (batch, head).

    Returns a list of length nb; entry i is a sorted int64 array of kept key
    blocks.  Prefix query blocks keep every block; video query blocks keep
    every prefix block plus their top-`keep` video blocks ([PRISM] Prism
    section; [REF2VA] condition-token section).  With `rows` given, only
    those query blocks are evaluated (the others are None).
    """
    S = block_scores_f32(geo, q_pool, k_pool)
    lists = []
    every = np.arange(geo.nb, dtype=np.int64)
    wanted = None if rows is None else set(int(r) for r in rows)
    for i in range(geo.nb):
        if wanted is not None and i not in wanted:
            lists.append(None)
        elif i < geo.nbp:
            lists.append(every)
        else:
            vid = np.asarray(topk_row(S[i - geo.nbp], keep), dtype=np.int64) + geo.nbp
            lists.append(np.concatenate([np.arange(geo.nbp, dtype=np.int64), vid]))
    return lists


def block_scores_gated_f32(geo, q_pool, k_pool, gate):
    """float32 [nbv, nbv] learned-gate scores ([REF2VA] "토큰 75%를 건너뛰는
    VSA": a trained predictor, to_gate_compress, picks the tiles that matter).
    Reading: the head's gate matrix G maps each pooled query row,
    q~_c = sum_e G[c][e] q_e, and q~ is scored against the pooled key means.
    Pooled values and G are rounded to float32 first, the products are taken
    in float64 and the scores rounded to float32."""
    qp = np.asarray(q_pool, dtype=np.float32).astype(np.float64)[geo.nbp:]
    kp = np.asarray(k_pool, dtype=np.float32).astype(np.float64)[geo.nbp:]
    G = np.asarray(gate, dtype=np.float32).astype(np.float64)
    return ((qp @ G.T) @ kp.T).astype(np.float32)


def select_gated(geo, q_pool, k_pool, keep, gate, rows=None):
    """select() with the learned-gate scores of one head's gate matrix."""
    S = block_scores_gated_f32(geo, q_pool, k_pool, gate)
    lists = []
    every = np.arange(geo.nb, dtype=np.int64)
    wanted = None if rows is None else set(int(r) for r in rows)
    for i in range(geo.nb):
        if wanted is not None and i not in wanted:
            lists.append(None)
        elif i < geo.nbp:
            lists.append(every)
        else:
            vid = np.asarray(topk_row(S[i - geo.nbp], keep), dtype=np.int64) + geo.nbp
            lists.append(np.concatenate([np.arange(geo.nbp, dtype=np.int64), vid]))
    return lists


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def block_sparse_attention(geo, perm, q_perm, k_perm, v_perm, lists, scale,
                           query_blocks=None):
    """Block-ordered output rows for the requested query blocks of one
    (batch, head).

    For each valid query token of block i: logits over every valid key token
    of the kept blocks of i, two-pass softmax (max, then normalised
    exponentials), weighted sum of values.  Pad query rows are 0.  Only kept
    tiles are touched ([SVG] logical vs physical sparsity: empty tiles are
    skipped).  Returns {i: float64 [64, d]}.
    """
    ok = slot_valid(geo, perm)
    if query_blocks is None:
        query_blocks = range(geo.nb)
    out = {}
    for i in query_blocks:
        rows = slice(i * BLOCK, (i + 1) * BLOCK)
        keys = np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in lists[i]])
        keys = keys[ok[keys]]
        logits = (q_perm[rows] @ k_perm[keys].T) * scale
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        o = (e @ v_perm[keys]) / e.sum(axis=1, keepdims=True)
        o[~ok[rows]] = 0.0
        out[i] = o
    return out


def forward(prob, q, k, v, lists_override=None):
    """The whole call on small problems: raster fp64 output [B, N, h, d].

    lists_override[b][h] replaces the oracle's own selection (the
    "conditioned" mode used to compare outputs on the GPU's selection).
    Returns (out, perms, codes, lists).
    """
    geo = Geometry(prob)
    keep = prob.get("keep_blocks") or keep_count(geo.nbv, prob["keep_ratio"])
    scale = prob.get("softmax_scale") or 1.0 / math.sqrt(geo.d)
    lay = layout(prob, k)
    out = np.zeros((geo.B, geo.N, geo.h, geo.d))
    all_lists = []
    for b in range(geo.B):
        perm = lay[b][0]
        per_b = []
        for hh in range(geo.h):
            qp = permute(geo, perm, q[b, :, hh])
            kp = permute(geo, perm, k[b, :, hh])
            vp = permute(geo, perm, v[b, :, hh])
            if lists_override is not None:
                lists = lists_override[b][hh]
            else:
                lists = select(geo, pool(geo, perm, qp), pool(geo, perm, kp), keep)
            per_b.append(lists)
            blocks = block_sparse_attention(geo, perm, qp, kp, vp, lists, scale)
            op = np.concatenate([blocks[i] for i in range(geo.nb)])
            out[b, :, hh] = unpermute(geo, perm, op)
        all_lists.append(per_b)
    return out, [p for p, _ in lay], [c for _, c in lay], all_lists


# --------------------------------------------------------------------------
# backward: gradients through the block-sparse attention
# --------------------------------------------------------------------------
# [PRISM] "같은 계산량 안에서 볼 곳을 고르는 Prism": the sparse attention is
# also used in training (a 2K training step from 26.5 to 10.6 minutes), so
# the same kept tiles carry the gradients.  With P the row-softmax of the
# masked logits and O = P V, for a loss whose gradient at O is dO:
#   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
#   dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
# Pad query rows have O = 0 by definition, so nothing flows through them.
def kept_mask(geo, perm, lists):
    """bool [N, N] in block order: query slot -> key slot is attended (its
    key block is in the query block's list and the key is a real token)."""
    kept = np.zeros((geo.nb, geo.nb), dtype=bool)
    for i, lst in enumerate(lists):
        kept[i, np.asarray(lst, dtype=np.int64)] = True
    blk = np.arange(geo.N) // BLOCK
    return kept[blk[:, None], blk[None, :]] & slot_valid(geo, perm)[None, :]


def block_sparse_attention_grad(geo, perm, q_perm, k_perm, v_perm, do_perm, lists, scale):
    """(dq, dk, dv), float64 [N, d] in block order, of one (batch, head)."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q_perm, k_perm, v_perm, do_perm))
    mask = kept_mask(geo, perm, lists)
    logits = np.where(mask, (q @ k.T) * scale, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    p = e / e.sum(axis=1, keepdims=True)
    p[~slot_valid(geo, perm)] = 0.0
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    return scale * (ds @ k), scale * (ds.T @ q), dv


# --------------------------------------------------------------------------
# helpers used by the pins (brute force on tiny inputs)
# --------------------------------------------------------------------------
def topk_bruteforce(scores_row, k):
    """The unique k-subset that dominates its complement under the order
    (score descending, index ascending), found by enumerating subsets."""
    n = len(scores_row)
    key = [(float(scores_row[j]), -j) for j in range(n)]
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        if all(key[a] > key[b] for a in inside for b in range(n) if b not in inside):
            found.append(sorted(sub))
    assert len(found) == 1
    return found[0]


# --------------------------------------------------------------------------
# window heads: spatial and temporal attention patterns, tile classes
# --------------------------------------------------------------------------
# [SVG] "Sparse VideoGen의 핵심 아이디어": a spatial head attends within the
# same or nearby frames, a temporal head to the same spatial neighbourhood
# across frames.  Both are written here as one window per head, (w_t, w_y,
# w_x): query token (t, y, x) attends to video key (t', y', x') when
# |t' - t| <= w_t, |y' - y| <= w_y and |x' - x| <= w_x, an axis with
# UNBOUNDED (-1) being free.  The conditioning prefix stays dense as in
# [REF2VA] "조건 토큰은 왜 다르게 다루나": every query attends to every prefix
# key and prefix queries attend to every key.  Pad keys are excluded and pad
# query rows are 0, as everywhere else.
# [SVG] "이론적 sparsity와 물리적 sparsity의 차이": a 64 x 64 tile of block
# pairs is full (every pair of real tokens attended), boundary (some) or
# empty (none, skipped).
UNBOUNDED = -1


def token_coords(geo):
    """int64 [N, 3]: (t, y, x) of every raster token; -1 for prefix tokens."""
    c = np.full((geo.N, 3), -1, dtype=np.int64)
    t, y, x = np.meshgrid(np.arange(geo.T), np.arange(geo.H), np.arange(geo.W), indexing="ij")
    c[geo.P:, 0] = t.reshape(-1)
    c[geo.P:, 1] = y.reshape(-1)
    c[geo.P:, 2] = x.reshape(-1)
    return c


def window_mask(geo, window, rows=None):
    """bool [N, N] in raster order: may query token n attend to key token m.
    A negative window entry leaves its axis free.  With `rows` (raster query
    indices) only those query rows are built: [len(rows), N]."""
    c = token_coords(geo)
    cq = c if rows is None else c[np.asarray(rows)]
    vid = c[:, 0] >= 0
    ok = np.ones((len(cq), geo.N), dtype=bool)
    for a in range(3):
        w = int(window[a])
        if w >= 0:
            ok &= np.abs(cq[:, None, a] - c[None, :, a]) <= w
    ok |= ~vid[None, :]                  # prefix keys: every query
    ok |= (cq[:, 0] < 0)[:, None]        # prefix queries: every key
    return ok & geo.token_valid()[None, :]


def window_attention(geo, q_bh, k_bh, v_bh, window, scale, rows=None):
    """[N, d] raster-order output of one (batch, head) under its window:
    logits over the allowed valid keys of each query, two-pass softmax,
    pad query rows 0.  With `rows` only those raster query rows are
    computed ([len(rows), d])."""
    q = np.asarray(q_bh, dtype=np.float64)
    k = np.asarray(k_bh, dtype=np.float64)
    v = np.asarray(v_bh, dtype=np.float64)
    idx = np.arange(geo.N) if rows is None else np.asarray(rows)
    mask = window_mask(geo, window, idx)
    logits = np.where(mask, (q[idx] @ k.T) * scale, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    out = (e @ v) / e.sum(axis=1, keepdims=True)
    out[~geo.token_valid()[idx]] = 0.0
    return out


def tile_classes(geo, perm, window):
    """int64 [nb, nb] over block pairs in block order: 0 empty, 1 boundary,
    2 full, judged on the pairs of real tokens (query block i, key block j)."""
    mask = window_mask(geo, window)[perm][:, perm]            # block order
    ok = slot_valid(geo, perm)
    out = np.zeros((geo.nb, geo.nb), dtype=np.int64)
    for i in range(geo.nb):
        qi = np.arange(i * BLOCK, (i + 1) * BLOCK)
        qi = qi[ok[qi]]
        for j in range(geo.nb):
            kj = np.arange(j * BLOCK, (j + 1) * BLOCK)
            kj = kj[ok[kj]]
            sub = mask[np.ix_(qi, kj)]
            out[i, j] = 2 if sub.all() else (1 if sub.any() else 0)
    return out
