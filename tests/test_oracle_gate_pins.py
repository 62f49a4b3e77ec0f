"""Pins of the oracle's learned-gate block scores (the VSA-style predictor
that picks the tiles) to facts outside that code:

* an identity gate gives the plain pooled scores and lists exactly;
* a positive multiple of the identity keeps every list (the order of a row
  is unchanged by a positive scale);
* a brute-force double sum over channels for a non-symmetric gate;
* the bilinear form's transpose rule: scoring K against Q with G^T gives the
  transposed score matrix.
A planted mistake (the gate applied transposed) must be caught."""
import numpy as np
import pytest

from gen import make_gate, make_qkv
from oracle import bsa_oracle as O


def prob(**kw):
    p = dict(B=1, heads=1, head_dim=16, T=8, H=8, W=8, T_valid=8, H_valid=8, W_valid=8,
             prefix=(20,), keep_ratio=0.25, block_mode=0, dyn_tau=1.25, blobs=0)
    p.update(kw)
    return p


def pooled(p, seed=3):
    geo = O.Geometry(p)
    q, k, _ = make_qkv(p, seed, pad_fill=1e4)
    perm = O.fixed_perm(geo)
    qp = O.pool(geo, perm, O.permute(geo, perm, q[0, :, 0].float().numpy()))
    kp = O.pool(geo, perm, O.permute(geo, perm, k[0, :, 0].float().numpy()))
    return geo, qp, kp


def test_identity_gate_is_the_plain_score():
    geo, qp, kp = pooled(prob())
    eye = np.eye(geo.d, dtype=np.float32)
    assert np.array_equal(O.block_scores_gated_f32(geo, qp, kp, eye),
                          O.block_scores_f32(geo, qp, kp))
    keep = O.keep_count(geo.nbv, 0.25)
    got = O.select_gated(geo, qp, kp, keep, eye)
    want = O.select(geo, qp, kp, keep)
    assert all(np.array_equal(a, b) for a, b in zip(got, want))


def test_scaled_identity_keeps_the_lists():
    geo, qp, kp = pooled(prob())
    keep = O.keep_count(geo.nbv, 0.25)
    want = O.select(geo, qp, kp, keep)
    got = O.select_gated(geo, qp, kp, keep, 4.0 * np.eye(geo.d, dtype=np.float32))
    assert all(np.array_equal(a, b) for a, b in zip(got, want))


def check_bruteforce():
    geo, qp, kp = pooled(prob(head_dim=8))
    G = make_gate(1, geo.d, 77)[0].numpy()
    assert not np.allclose(G, G.T)
    S = O.block_scores_gated_f32(geo, qp, kp, G)
    q32 = qp.astype(np.float32).astype(np.float64)
    k32 = kp.astype(np.float32).astype(np.float64)
    G64 = G.astype(np.float64)
    for i in range(geo.nbv):
        for j in range(geo.nbv):
            s = 0.0
            for c in range(geo.d):
                for e in range(geo.d):
                    s += G64[c, e] * q32[geo.nbp + i, e] * k32[geo.nbp + j, c]
            assert abs(float(S[i, j]) - s) <= 1e-6 * max(1.0, abs(s)), (i, j)


def test_gated_score_bruteforce():
    check_bruteforce()


def test_transpose_rule():
    geo, qp, kp = pooled(prob())
    G = make_gate(1, geo.d, 5)[0].numpy()
    a = O.block_scores_gated_f32(geo, qp, kp, G).astype(np.float64)
    b = O.block_scores_gated_f32(geo, kp, qp, G.T.copy()).astype(np.float64)
    np.testing.assert_allclose(a, b.T, rtol=1e-5, atol=1e-5)


def _gate_transposed(geo, q_pool, k_pool, gate):
    return O.__dict__["_orig_block_scores_gated_f32"](geo, q_pool, k_pool,
                                                       np.asarray(gate).T.copy())


def test_planted_transposed_gate_is_caught(monkeypatch):
    check_bruteforce()
    monkeypatch.setitem(O.__dict__, "_orig_block_scores_gated_f32", O.block_scores_gated_f32)
    monkeypatch.setattr(O, "block_scores_gated_f32", _gate_transposed)
    with pytest.raises(AssertionError):
        check_bruteforce()
