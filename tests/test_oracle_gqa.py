"""Pins for the GQA-path oracle (GQLA summary, "Arquitetura", item 2: a
group-expanded cache of per-group keys and values plus a shared RoPE key,
decoded with grouped-query attention).  All on the CPU.

* reduction: when every group's values equal its keys, each group's heads see
  exactly the MQA cache [K_k | RoPE] with value = K_k, which the already
  pinned MLA oracle computes (its d_v = the first d_head columns);
* brute force with Python floats on tiny inputs;
* group independence: a group's heads read only that group's K and V;
* the value is V_k, not K_k: O is a convex combination of V_k rows;
* the block table's page order does not matter (bitwise).
"""
import math

import numpy as np
import pytest


def _case(rng, B, s_q, hq, g, d_head, d_rope, page, lens, perm=True):
    pages = [(L + page - 1) // page for L in lens]
    nb = sum(pages) + 2
    q = rng.standard_normal((B, s_q, hq, d_head + d_rope))
    kv = rng.standard_normal((nb, page, 2 * g * d_head + d_rope))
    ids = rng.permutation(nb) if perm else np.arange(nb)
    bt = np.full((B, max(max(pages), 1)), -1, dtype=np.int32)
    k = 0
    for b, P in enumerate(pages):
        bt[b, :P] = ids[k:k + P]
        k += P
    return q, kv, bt, np.asarray(lens, dtype=np.int32)


def test_equal_keys_and_values_reduce_to_the_mla_oracle(oracle_mod):
    rng = np.random.default_rng(101)
    B, s_q, hq, g, dh, dr, page = 2, 2, 6, 3, 8, 4, 4
    q, kv, bt, sl = _case(rng, B, s_q, hq, g, dh, dr, page, [9, 14])
    kv[..., g * dh:2 * g * dh] = kv[..., 0:g * dh]          # V_k := K_k
    out, lse = oracle_mod.gqa_oracle_fwd(q, kv, bt, sl, 0.3, g, d_head=dh, causal=True)
    hpg = hq // g
    for k in range(g):
        mla_kv = np.concatenate([kv[..., k * dh:(k + 1) * dh], kv[..., 2 * g * dh:]], axis=-1)
        qk = q[:, :, k * hpg:(k + 1) * hpg, :]
        o_ref, l_ref = oracle_mod.mla_oracle_fwd(qk, mla_kv, bt, sl, 0.3, causal=True, d_v=dh)
        for b in range(B):
            for s in range(s_q):
                for i in range(hpg):
                    r = (b * s_q + s) * hq + k * hpg + i
                    rr = (b * s_q + s) * hpg + i
                    np.testing.assert_allclose(out[r], o_ref[rr], rtol=0, atol=1e-12)
                    assert abs(lse[r] - l_ref[rr]) <= 1e-12


def test_brute_force_python_floats(oracle_mod):
    rng = np.random.default_rng(102)
    for trial in range(4):
        B, s_q, hq, g, dh, dr, page = 1 + trial % 2, 1 + trial // 2, 4, 2, 3, 2, 2
        lens = [int(rng.integers(1, 8)) for _ in range(B)]
        causal = trial % 2 == 1
        q, kv, bt, sl = _case(rng, B, s_q, hq, g, dh, dr, page, lens)
        scale = float(rng.uniform(0.3, 1.2))
        out, lse = oracle_mod.gqa_oracle_fwd(q, kv, bt, sl, scale, g, d_head=dh, causal=causal)
        hpg = hq // g
        for b in range(B):
            for s in range(s_q):
                for h in range(hq):
                    r = (b * s_q + s) * hq + h
                    k = h // hpg
                    n = lens[b] - s_q + 1 + s if (causal and s_q > 1) else lens[b]
                    if n <= 0:
                        assert lse[r] == -math.inf and not out[r].any()
                        continue
                    z = []
                    for t in range(n):
                        row = kv[bt[b, t // page], t % page]
                        acc = sum(float(q[b, s, h, c]) * float(row[k * dh + c]) for c in range(dh))
                        acc += sum(float(q[b, s, h, dh + c]) * float(row[2 * g * dh + c]) for c in range(dr))
                        z.append(scale * acc)
                    m = max(z)
                    w = [math.exp(x - m) for x in z]
                    tot = sum(w)
                    for c in range(dh):
                        o = sum(w[t] * float(kv[bt[b, t // page], t % page][g * dh + k * dh + c])
                                for t in range(n)) / tot
                        assert abs(o - out[r, c]) <= 1e-12
                    assert abs(m + math.log(tot) - lse[r]) <= 1e-12


def test_groups_are_independent_and_values_are_v(oracle_mod):
    rng = np.random.default_rng(103)
    B, s_q, hq, g, dh, dr, page = 1, 1, 4, 2, 5, 3, 4
    q, kv, bt, sl = _case(rng, B, s_q, hq, g, dh, dr, page, [11])
    out, lse = oracle_mod.gqa_oracle_fwd(q, kv, bt, sl, 0.5, g, d_head=dh)
    kv2 = kv.copy()
    kv2[..., 1 * dh:2 * dh] += 7.0                    # K_1
    kv2[..., g * dh + dh:g * dh + 2 * dh] *= -3.0     # V_1
    out2, lse2 = oracle_mod.gqa_oracle_fwd(q, kv2, bt, sl, 0.5, g, d_head=dh)
    np.testing.assert_array_equal(out[:2], out2[:2])   # group 0's heads untouched
    np.testing.assert_array_equal(lse[:2], lse2[:2])
    assert np.abs(out[2:] - out2[2:]).max() > 1e-3
    # O of group 0's heads lies in the box spanned by V_0 rows (not K_0 rows)
    rows = np.stack([kv[bt[0, t // page], t % page] for t in range(11)])
    v0 = rows[:, g * dh:g * dh + dh]
    assert (out[:2] <= v0.max(axis=0) + 1e-12).all() and (out[:2] >= v0.min(axis=0) - 1e-12).all()


def test_block_table_permutation_is_bitwise_invariant(oracle_mod):
    rng = np.random.default_rng(104)
    q, kv, bt, sl = _case(rng, 2, 2, 4, 2, 6, 2, 4, [13, 7], perm=False)
    out, lse = oracle_mod.gqa_oracle_fwd(q, kv, bt, sl, 0.4, 2, d_head=6, causal=True)
    perm = rng.permutation(kv.shape[0])
    inv = np.argsort(perm)
    kv_p = kv[perm]
    bt_p = bt.copy()
    bt_p[bt_p >= 0] = inv[bt_p[bt_p >= 0]]
    out_p, lse_p = oracle_mod.gqa_oracle_fwd(q, kv_p, bt_p, sl, 0.4, 2, d_head=6, causal=True)
    np.testing.assert_array_equal(out, out_p)
    np.testing.assert_array_equal(lse, lse_p)


def test_rejects_heads_not_divisible_by_groups(oracle_mod):
    rng = np.random.default_rng(105)
    q, kv, bt, sl = _case(rng, 1, 1, 4, 2, 4, 2, 4, [5])
    with pytest.raises(RuntimeError):
        oracle_mod.gqa_oracle_fwd(q[:, :, :3], kv, bt, sl, 0.4, 2, d_head=4)
