"""GPU parity of the learned-gate selection (bsa_select_topk_gated) against
the oracle's gated block scores, with synthetic gate matrices standing in
for trained to_gate_compress weights.

* an identity gate gives exactly the ungated lists;
* every gated list is a valid top-k of the oracle's gated fp32 scores (near
  ties accepted), and the attention output over the gated lists matches the
  oracle on its own valid selection equal to the GPU's;
* the same at full 720p size for sampled (batch, head) pairs."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_47_b200 as bsa
from gen import config, make_gate, make_qkv
from oracle import bsa_oracle as O
from parity_helpers import (assert_close, matched_lists, problem, sample_blocks, to_np64,
                            topk_alternatives)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": config("tiny"),
    "ragged": dict(config("tiny"), B=2, heads=3, head_dim=128, T=8, H=12, W=20, T_valid=7,
                   H_valid=10, W_valid=17, prefix=(40, 64, 1), keep_ratio=0.3, name="ragged"),
}


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()


def gated_call(cfg, q, k, v, gate):
    """layout -> pool_raster -> gated select -> raster attention."""
    prob = problem(cfg)
    attn = bsa.BlockSparseAttention(prob)
    bsa.layout(prob, k, attn.layout_buf)
    bsa.pool_raster(prob, attn.layout_buf, q, k, attn.q_pool, attn.k_pool)
    bsa.select_topk_gated(prob, attn.q_pool, attn.k_pool, gate, attn.idx, attn.cnt)
    out = torch.empty_like(q)
    bsa.sparse_attn_fwd_raster(prob, attn.layout_buf, q, k, v, attn.idx, attn.cnt, out,
                               attn.status)
    torch.cuda.synchronize()
    attn.check_status()
    return attn, out


@pytest.mark.parametrize("name", sorted(SMALL))
def test_identity_gate_gives_the_plain_lists(name):
    cfg = SMALL[name]
    q, k, v = make_qkv(cfg, 4500, pad_fill=1e4, device="cuda")
    eye = torch.eye(cfg["head_dim"], device="cuda").expand(cfg["heads"], -1, -1).contiguous()
    attn, out = gated_call(cfg, q, k, v, eye)
    plain = bsa.BlockSparseAttention(attn.prob)
    want = plain.raster_call(q, k, v)
    torch.cuda.synchronize()
    nbp = attn.sizes.n_prefix_blocks
    assert torch.equal(attn.idx[:, :, nbp:], plain.idx[:, :, nbp:])
    assert torch.equal(out, want)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_gated_lists_and_output_match_oracle(name):
    cfg = SMALL[name]
    q, k, v = make_qkv(cfg, 4600, pad_fill=1e4, device="cuda")
    gate = make_gate(cfg["heads"], cfg["head_dim"], 4601, device="cuda")
    attn, out = gated_call(cfg, q, k, v, gate)
    geo = O.Geometry(cfg)
    keep = attn.prob.keep_blocks
    perm = O.fixed_perm(geo)
    host = [to_np64(t) for t in (q, k, v)]
    gate_h = gate.cpu().numpy()
    idx = attn.idx.cpu().numpy()
    all_lists, changed = [], 0
    for b in range(geo.B):
        per = []
        for hh in range(geo.h):
            qp, kp = (O.permute(geo, perm, host[i][b, :, hh]) for i in (0, 1))
            qpool, kpool = O.pool(geo, perm, qp), O.pool(geo, perm, kp)
            S = O.block_scores_gated_f32(geo, qpool, kpool, gate_h[hh])
            per.append(matched_lists(geo, S, idx[b, hh], keep))
            plain = O.select(geo, qpool, kpool, keep)
            changed += sum(not np.array_equal(a, c) for a, c in zip(per[-1], plain))
        all_lists.append(per)
    assert changed > 0, "the synthetic gate should change some lists"
    want, _, _, _ = O.forward(dict(cfg, keep_blocks=keep), *host, lists_override=all_lists)
    assert_close(to_np64(out), want, name + " gated")


def test_gated_full_size_720p():
    cfg = config("720p")
    q, k, v = make_qkv(cfg, 4700, pad_fill=1e4, device="cuda")
    gate = make_gate(cfg["heads"], cfg["head_dim"], 4701, device="cuda")
    attn, out = gated_call(cfg, q, k, v, gate)
    geo = O.Geometry(cfg)
    keep = attn.prob.keep_blocks
    perm = O.fixed_perm(geo)
    rng = np.random.default_rng(3)
    idx = attn.idx.cpu().numpy()
    gate_h = gate.cpu().numpy()
    for b, hh in [(0, 0), (1, 23), (1, 7)]:
        op = [O.permute(geo, perm, to_np64(t[b, :, hh])) for t in (q, k, v)]
        S = O.block_scores_gated_f32(geo, O.pool(geo, perm, op[0]), O.pool(geo, perm, op[1]),
                                     gate_h[hh])
        lists = matched_lists(geo, S, idx[b, hh], keep)    # every list of this (b, h)
        blocks = sample_blocks(geo, 6, rng)
        want = O.block_sparse_attention(geo, perm, *op, lists, 1 / math.sqrt(geo.d), blocks)
        got = to_np64(out[b, :, hh])
        for i in blocks:
            assert_close(got[perm[i * 64:(i + 1) * 64]], want[i], "720p gated b%d h%d" % (b, hh))
