"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI, compute the oracle's view of the same seeded inputs, and compare.

The oracle never receives a value computed by the CUDA path.  Where a stage
is tested on its own (attention, unpermute), its inputs are built from the
oracle's permutation and selection and uploaded."""
import math

import numpy as np
import torch

import block_sparse_attention_47_b200 as bsa
from gen import derived_sizes, make_qkv
from oracle import bsa_oracle as O

# bf16-in / fp32-accumulate vs fp64 tolerance (stated for the outputs)
MAX_ABS = 2e-2
REL_L2 = 5e-3
# near-tie band of a block-selection decision, relative to max |score| of the row
TIE_REL = 1e-4
PAD = 0x80000000


def problem(cfg, keep=None):
    keep = keep if keep is not None else O.keep_count(derived_sizes(cfg)["nbv"], cfg["keep_ratio"])
    return bsa.Problem.make(**dict(cfg, keep_blocks=keep))


def to_np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want).max() if got.size else 0.0
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, "%s max-abs %.3g rel-L2 %.3g" % (what, err, rel)
    return err, rel


class DeviceRun:
    """The whole six-call sequence on device buffers, kept for inspection."""

    def __init__(self, cfg, q, k, v, keep=None, dense=False, raster=False):
        self.cfg = cfg
        self.raster = raster
        self.prob = problem(cfg, keep)
        self.attn = bsa.BlockSparseAttention(self.prob)
        if raster:
            self.out = self.attn.raster_call(q, k, v)
        else:
            self.out = self.attn(q, k, v, dense=dense)
        torch.cuda.synchronize()
        self.attn.check_status()
        s = self.attn.sizes
        lb = self.attn.layout_buf
        B, N, nb = self.prob.B, s.n_tokens, s.n_blocks
        raw = lb.view(torch.uint8)

        def section(offset, count, dtype):
            nbytes = count * torch.tensor([], dtype=dtype).element_size()
            return raw[offset:offset + nbytes].view(dtype)

        def align(x):
            return (x + 255) // 256 * 256
        off = 0
        self.perm = section(off, B * N, torch.int32).view(B, N).cpu().numpy().astype(np.int64)
        off = align(off + 4 * B * N)
        self.iperm = section(off, B * N, torch.int32).view(B, N).cpu().numpy().astype(np.int64)
        off = align(off + 4 * B * N)
        self.bmask = section(off, B * nb, torch.int64).view(B, nb).cpu().numpy()
        off = align(off + 8 * B * nb)
        self.bcount = section(off, B * nb, torch.int32).view(B, nb).cpu().numpy()
        off = align(off + 4 * B * nb)
        nreg = max(int(s.n_regions), 1)
        self.codes = section(off, B * nreg, torch.uint8).view(B, nreg).cpu().numpy()


def decode_map(m):
    """(index, pad flag) from a GPU map entry with bit 31 marking pad."""
    m = m & 0xFFFFFFFF
    return (m & 0x7FFFFFFF).astype(np.int64), (m & PAD) != 0


def lists_to_device(geo, lists_bh, kcap, device="cuda"):
    """Oracle lists [B][h][nb] -> (idx, cnt) in the C ABI's format."""
    B, h = len(lists_bh), len(lists_bh[0])
    idx = np.zeros((B, h, geo.nb, kcap), dtype=np.int32)
    cnt = np.zeros((B, h, geo.nb), dtype=np.int32)
    for b in range(B):
        for hh in range(h):
            for i, lst in enumerate(lists_bh[b][hh]):
                if i < geo.nbp:
                    cnt[b, hh, i] = -1
                else:
                    cnt[b, hh, i] = len(lst)
                    idx[b, hh, i, :len(lst)] = lst
    return torch.from_numpy(idx).to(device), torch.from_numpy(cnt).to(device)


def check_list_row(gpu_row, scores_row, keep, nbp):
    """Validity of one GPU list against the oracle's fp32 scores: prefix
    first, ascending, `keep` video blocks, and the kept set equals the
    oracle's top-k except for entries inside the near-tie band."""
    gpu_row = np.asarray(gpu_row)
    assert list(gpu_row[:nbp]) == list(range(nbp))
    vid = gpu_row[nbp:] - nbp
    assert len(vid) == keep and np.all(np.diff(vid) > 0)
    s = np.asarray(scores_row, dtype=np.float64)
    kth = np.sort(s)[::-1][keep - 1]
    band = TIE_REL * max(np.abs(s).max(), 1e-30)
    chosen = np.zeros(len(s), dtype=bool)
    chosen[vid] = True
    assert np.all(chosen[s > kth + band]), "a clearly better block was dropped"
    assert np.all(s[chosen] >= kth - band), "a clearly worse block was kept"
    return list(vid) == O.topk_row(scores_row, keep)


def topk_alternatives(scores_row, keep, limit=256):
    """Every list the oracle accepts for one query block: the `keep`-subsets
    (ascending) that hold every block scoring above kth + band and no block
    scoring below kth - band, where kth is the keep-th largest fp32 score
    and band = TIE_REL * max |score| (the near-tie band).  Without a near tie
    this is the single list O.topk_row gives."""
    s = np.asarray(scores_row, dtype=np.float64)
    kth = np.sort(s)[::-1][keep - 1]
    band = TIE_REL * max(np.abs(s).max(), 1e-30)
    sure = np.nonzero(s > kth + band)[0]
    maybe = np.nonzero(np.abs(s - kth) <= band)[0]
    need = keep - len(sure)
    assert 0 < need <= len(maybe)
    if need == len(maybe):
        return [sorted(int(x) for x in np.concatenate([sure, maybe]))]
    if math.comb(len(maybe), need) > limit:
        raise AssertionError("near-tie band too wide to enumerate (%d of %d)" % (need, len(maybe)))
    import itertools
    return [sorted(int(x) for x in np.concatenate([sure, np.asarray(c, dtype=np.int64)]))
            for c in itertools.combinations(maybe, need)]


def matched_lists(geo, S, gpu_idx_bh, keep, rows=None):
    """The oracle's list of every query block (or of `rows`) of one
    (batch, head), chosen among its own valid alternatives
    (topk_alternatives) as the one the GPU took.  Fails unless the GPU's
    list is one of them.  Prefix query blocks keep every block."""
    lists = [None] * geo.nb
    every = np.arange(geo.nb, dtype=np.int64)
    pre = np.arange(geo.nbp, dtype=np.int64)
    for i in (range(geo.nb) if rows is None else rows):
        if i < geo.nbp:
            lists[i] = every
            continue
        gpu = [int(x) - geo.nbp for x in gpu_idx_bh[i, geo.nbp:geo.nbp + keep]]
        alts = topk_alternatives(S[i - geo.nbp], keep)
        assert gpu in alts, "query block %d: the GPU list is not a valid top-%d" % (i, keep)
        lists[i] = np.concatenate([pre, np.asarray(alts[alts.index(gpu)], dtype=np.int64)
                                   + geo.nbp])
    return lists


def oracle_forward_matched(cfg, host, gpu_idx, keep):
    """O.forward on the host inputs with, for every (batch, head) and query
    block, the oracle's valid selection that equals the GPU's (so every row
    is compared, near ties included).  gpu_idx is [B, heads, nb, kcap]."""
    geo = O.Geometry(cfg)
    qn, kn, vn = host
    lay = O.layout(cfg, kn)
    all_lists = []
    for b in range(geo.B):
        perm = lay[b][0]
        per = []
        for hh in range(geo.h):
            qp, kp, _ = oracle_bh(geo, perm, qn, kn, vn, b, hh)
            S = O.block_scores_f32(geo, O.pool(geo, perm, qp), O.pool(geo, perm, kp))
            per.append(matched_lists(geo, S, gpu_idx[b, hh], keep))
        all_lists.append(per)
    out, _, _, _ = O.forward(dict(cfg, keep_blocks=keep), qn, kn, vn, lists_override=all_lists)
    return out


def oracle_bh(geo, perm, q, k, v, b, hh):
    """Oracle permuted fp64 rows of one (batch, head)."""
    return (O.permute(geo, perm, q[b, :, hh]), O.permute(geo, perm, k[b, :, hh]),
            O.permute(geo, perm, v[b, :, hh]))


def seeded_inputs(cfg, seed, pad_fill=1e4, device="cuda"):
    """Generator tensors on the device plus fp64 host copies."""
    q, k, v = make_qkv(cfg, seed, pad_fill=pad_fill, device=device)
    return (q, k, v), [to_np64(t) for t in (q, k, v)]


def sample_blocks(geo, n, rng, extra=()):
    picks = {0, geo.nb - 1, *extra}
    if geo.nbp:
        picks |= {geo.nbp - 1, geo.nbp}
    while len(picks) < min(n, geo.nb):
        picks.add(int(rng.integers(0, geo.nb)))
    return sorted(picks)


def scale_of(cfg):
    return 1.0 / math.sqrt(cfg["head_dim"])
