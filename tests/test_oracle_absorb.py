"""Pins for the absorbed-projection oracle (oracle/absorb.py), on the CPU.

* brute force with Python floats on tiny shapes, both projections;
* the absorption identity of the GQLA summary ("Caminho MQA-Absorvido"): with
  the latent query q_lat = q_nope . W_UK, the score against a latent row c
  equals q_nope . (W_UK c), the score against the decompressed key;
* linearity in the input, and the RoPE part passing through unchanged.
"""
import numpy as np

from oracle import absorb


def test_brute_force_both_projections():
    rng = np.random.default_rng(201)
    T, h, dn, dl, dr, dout = 3, 2, 4, 5, 2, 3
    q = rng.standard_normal((T, h, dn + dr))
    w_uk = rng.standard_normal((h, dn, dl))
    got = absorb.absorb_q(q, w_uk, d_nope=dn)
    for t in range(T):
        for hh in range(h):
            for n in range(dl):
                ref = sum(float(q[t, hh, k]) * float(w_uk[hh, k, n]) for k in range(dn))
                assert abs(got[t, hh, n] - ref) <= 1e-12
            for c in range(dr):
                assert got[t, hh, dl + c] == q[t, hh, dn + c]
    o = rng.standard_normal((T, h, dl))
    w_uv = rng.standard_normal((h, dl, dout))
    got = absorb.absorb_o(o, w_uv)
    for t in range(T):
        for hh in range(h):
            for n in range(dout):
                ref = sum(float(o[t, hh, k]) * float(w_uv[hh, k, n]) for k in range(dl))
                assert abs(got[t, hh, n] - ref) <= 1e-12


def test_absorbed_query_scores_equal_decompressed_key_scores():
    rng = np.random.default_rng(202)
    T, h, dn, dl = 4, 3, 16, 24
    q = rng.standard_normal((T, h, dn))
    w_uk = rng.standard_normal((h, dn, dl))
    c = rng.standard_normal((7, dl))                      # latent rows
    q_lat = absorb.absorb_q(q, w_uk, d_nope=dn)           # no RoPE part here
    for hh in range(h):
        k_full = c @ w_uk[hh].T                           # decompressed keys [7, dn]
        np.testing.assert_allclose(q_lat[:, hh] @ c.T, q[:, hh] @ k_full.T, rtol=1e-12, atol=1e-12)


def test_linearity():
    rng = np.random.default_rng(203)
    o1, o2 = rng.standard_normal((2, 5, 2, 8))
    w = rng.standard_normal((2, 8, 3))
    np.testing.assert_allclose(absorb.absorb_o(2.0 * o1 - o2, w),
                               2.0 * absorb.absorb_o(o1, w) - absorb.absorb_o(o2, w), rtol=1e-12, atol=1e-12)
