"""Pins of the oracle's backward (gradients of the block-sparse attention)
to facts outside its own formulas:

* central finite differences of the oracle's forward (a different code path:
  two-pass softmax over kept tiles, per query block) along random directions
  of Q, K and V, on problems with a prefix, pads and a sparse selection;
* torch fp64 autograd through an explicitly masked softmax attention (a
  library routine) gives the same dQ, dK and dV;
* every block kept: torch autograd through scaled_dot_product_attention
  with a key-padding mask.
Planted mistakes (no D term, an unscaled dK, P in place of dS for dQ) must
be caught."""
import math

import numpy as np
import pytest
import torch

from gen import make_qkv
from oracle import bsa_oracle as O


def prob(**kw):
    p = dict(B=1, heads=1, head_dim=8, T=4, H=8, W=8, T_valid=3, H_valid=7, W_valid=8,
             prefix=(20,), keep_ratio=0.4, block_mode=0, dyn_tau=1.25, blobs=0)
    p.update(kw)
    return p


def case(p, seed=21):
    geo = O.Geometry(p)
    q, k, v = (t[0, :, 0].float().numpy().astype(np.float64) for t in make_qkv(p, seed, pad_fill=1e4))
    perm = O.fixed_perm(geo)
    qp, kp, vp = (O.permute(geo, perm, x) for x in (q, k, v))
    keep = O.keep_count(geo.nbv, p["keep_ratio"])
    lists = O.select(geo, O.pool(geo, perm, qp), O.pool(geo, perm, kp), keep)
    rng = np.random.default_rng(seed)
    do = rng.normal(size=qp.shape)
    return geo, perm, qp, kp, vp, do, lists


def forward_rows(geo, perm, qp, kp, vp, lists, scale):
    blocks = O.block_sparse_attention(geo, perm, qp, kp, vp, lists, scale)
    return np.concatenate([blocks[i] for i in range(geo.nb)])


def check_finite_differences(p):
    geo, perm, qp, kp, vp, do, lists = case(p)
    scale = 1 / math.sqrt(geo.d)
    grads = O.block_sparse_attention_grad(geo, perm, qp, kp, vp, do, lists, scale)
    rng = np.random.default_rng(5)
    ok = O.slot_valid(geo, perm)
    for which in range(3):
        direction = rng.normal(size=qp.shape)
        direction[~ok] = 0.0          # pad slots are not inputs of the method
        eps = 1e-5

        def loss(sign):
            xs = [qp, kp, vp]
            xs = [x + sign * eps * direction if i == which else x for i, x in enumerate(xs)]
            return float((forward_rows(geo, perm, *xs, lists, scale) * do).sum())
        numeric = (loss(1) - loss(-1)) / (2 * eps)
        analytic = float((grads[which] * direction).sum())
        assert abs(numeric - analytic) <= 1e-6 * max(1.0, abs(analytic)), (which, numeric,
                                                                          analytic)


def test_gradients_match_finite_differences():
    check_finite_differences(prob())
    check_finite_differences(prob(keep_ratio=0.01, prefix=(64, 5)))


def check_autograd(p):
    geo, perm, qp, kp, vp, do, lists = case(p, seed=8)
    scale = 1 / math.sqrt(geo.d)
    dq, dk, dv = O.block_sparse_attention_grad(geo, perm, qp, kp, vp, do, lists, scale)
    mask = torch.from_numpy(O.kept_mask(geo, perm, lists))
    valid_q = torch.from_numpy(O.slot_valid(geo, perm))
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (qp, kp, vp))
    logits = (tq @ tk.T * scale).masked_fill(~mask, float("-inf"))
    o = torch.softmax(logits, dim=-1) @ tv
    o = torch.where(valid_q[:, None], o, torch.zeros_like(o))
    (o * torch.from_numpy(do)).sum().backward()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(mine - ref.numpy()).max() < 1e-12


def test_gradients_match_torch_autograd():
    check_autograd(prob())
    check_autograd(prob(T=8, H=8, W=12, T_valid=8, H_valid=6, W_valid=11, prefix=(3, 64),
                        keep_ratio=0.3, head_dim=16))


def test_keep_everything_matches_sdpa_autograd():
    p = prob(keep_ratio=1.0, prefix=(30,))
    geo, perm, qp, kp, vp, do, lists = case(p, seed=9)
    assert all(len(l) == geo.nb for l in lists)
    scale = 1 / math.sqrt(geo.d)
    dq, dk, dv = O.block_sparse_attention_grad(geo, perm, qp, kp, vp, do, lists, scale)
    valid = torch.from_numpy(O.slot_valid(geo, perm))
    tq, tk, tv = (torch.from_numpy(x)[None, None].requires_grad_() for x in (qp, kp, vp))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=valid[None, None, None, :], scale=scale)[0, 0]
    o = torch.where(valid[:, None], o, torch.zeros_like(o))
    (o * torch.from_numpy(do)).sum().backward()
    for mine, ref in ((dq, tq.grad[0, 0]), (dk, tk.grad[0, 0]), (dv, tv.grad[0, 0])):
        assert np.abs(mine - ref.numpy()).max() < 1e-12


# ---- planted mistakes --------------------------------------------------------
def _grad_variant(kind):
    def grad(geo, perm, q_perm, k_perm, v_perm, do_perm, lists, scale):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q_perm, k_perm, v_perm, do_perm))
        mask = O.kept_mask(geo, perm, lists)
        logits = np.where(mask, (q @ k.T) * scale, -np.inf)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        p[~O.slot_valid(geo, perm)] = 0.0
        o = p @ v
        dv = p.T @ do
        dp = do @ v.T
        delta = 0.0 if kind == "no-delta" else (do * o).sum(axis=1, keepdims=True)
        ds = p * (dp - delta)
        dq = scale * ((p if kind == "p-for-ds" else ds) @ k)
        dk = (1.0 if kind == "unscaled-dk" else scale) * (ds.T @ q)
        return dq, dk, dv
    return grad


@pytest.mark.parametrize("kind", ["no-delta", "unscaled-dk", "p-for-ds"])
def test_planted_gradient_mistake_is_caught(monkeypatch, kind):
    check_finite_differences(prob())
    monkeypatch.setattr(O, "block_sparse_attention_grad", _grad_variant(kind))
    with pytest.raises(AssertionError):
        check_finite_differences(prob())
