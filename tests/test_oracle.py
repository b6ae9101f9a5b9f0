"""Pins for the fp64 oracle, checked against things other than itself.

Every test here runs on the CPU.  Each one is chosen so that a plausible slip
in the oracle (a dropped scale, a wrong sign, a transposed operand, the wrong
value columns, an off-by-one in the causal rule, a missing max-shift) fails at
least one of them:

* a case worked by hand from the definition of softmax attention
  (tests/golden/hand_worked.json);
* closed forms: one visible token gives its own value row; a zero query
  gives the mean of the values and LSE = ln L;
* invariants: rows of P sum to 1, the block table's page order does not
  matter, rows past L do not matter, a constant added to every score shifts
  LSE by that constant and leaves O alone, the 64 RoPE columns are key-only;
* the transposed evaluation S^T = K Q^T, softmax over the KV axis,
  O = (V^T P^T)^T of the FlashMLA-ETAP summary ("Mecanismo Central"),
  written here with numpy on dense gathered tensors;
* brute force with Python floats on tiny inputs;
* split associativity: two disjoint halves merged by LSE weight equal the
  whole, which also pins the merge the combine kernel performs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from mla_decode_attention_15_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _num(x):
    if isinstance(x, str):
        return {"ln3": math.log(3.0), "ln4": math.log(4.0)}[x]
    return float(x)


def _dense_case(rng, B, s_q, h, d_qk, page, lens, num_blocks=None, perm=True):
    """Random fp64 inputs with a random page placement."""
    lens = list(lens)
    pages = [(L + page - 1) // page for L in lens]
    total = sum(pages)
    nb = total + 3 if num_blocks is None else num_blocks
    q = rng.standard_normal((B, s_q, h, d_qk))
    kv = rng.standard_normal((nb, page, d_qk))
    ids = rng.permutation(nb) if perm else np.arange(nb)
    bt = np.full((B, max(max(pages), 1)), -1, dtype=np.int32)
    k = 0
    for b, P in enumerate(pages):
        bt[b, :P] = ids[k:k + P]
        k += P
    return q, kv, bt, np.asarray(lens, dtype=np.int32)


def _gather(kv, bt, b, L):
    page = kv.shape[1]
    return np.stack([kv[bt[b, t // page], t % page] for t in range(L)]) if L else np.zeros((0, kv.shape[-1]))


def test_hand_worked_golden(oracle_mod):
    spec = json.load(open(GOLDEN))
    for case in spec["cases"]:
        q = np.array(case["q"], dtype=np.float64).reshape(1, 1, 1, 2)
        rows = np.array([[_num(v) for v in r] for r in case["rows"]], dtype=np.float64)
        kv = rows.reshape(1, 2, 2)  # one page of two tokens
        bt = np.zeros((1, 1), dtype=np.int32)
        sl = np.array([2], dtype=np.int32)
        out, lse, probs = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, case["scale"], d_v=case["d_v"],
                                                    want_probs=True)
        assert abs(out[0, 0] - case["O"][0]) <= 1e-12
        assert abs(lse[0] - _num(case["LSE"])) <= 1e-12
        np.testing.assert_allclose(probs[0, :2], case["P"], atol=1e-12, rtol=0)


def test_probs_sum_to_one(oracle_mod):
    rng = np.random.default_rng(1)
    q, kv, bt, sl = _dense_case(rng, 3, 2, 3, 24, 8, [1, 17, 40])
    _, _, probs = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.3, d_v=16, want_probs=True)
    for r in range(probs.shape[0]):
        b = r // (2 * 3)
        assert abs(probs[r, :sl[b]].sum() - 1.0) <= 1e-12
        assert (probs[r, :sl[b]] > 0).all()


def test_single_token_gives_its_value_row(oracle_mod):
    rng = np.random.default_rng(2)
    q, kv, bt, sl = _dense_case(rng, 2, 1, 4, 32, 8, [1, 1])
    scale = 0.7
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, scale, d_v=20)
    for b in range(2):
        row = kv[bt[b, 0], 0]
        for h in range(4):
            r = b * 4 + h
            np.testing.assert_array_equal(out[r], row[:20])
            assert abs(lse[r] - scale * float(np.dot(q[b, 0, h], row))) <= 1e-12


def test_zero_query_gives_mean_value(oracle_mod):
    rng = np.random.default_rng(3)
    L = 77
    q, kv, bt, sl = _dense_case(rng, 1, 1, 2, 40, 16, [L])
    q[:] = 0.0
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 1.3, d_v=32)
    rows = _gather(kv, bt, 0, L)
    for r in range(2):
        np.testing.assert_allclose(out[r], rows[:, :32].mean(axis=0), atol=1e-12, rtol=0)
        assert abs(lse[r] - math.log(L)) <= 1e-12


def test_equal_scores_from_shared_key_columns(oracle_mod):
    """q nonzero only in columns where every row agrees: all scores are equal,
    so O is the plain mean of the differing value columns."""
    rng = np.random.default_rng(4)
    L, d_qk, d_v = 50, 48, 32
    q, kv, bt, sl = _dense_case(rng, 1, 1, 1, d_qk, 8, [L])
    q[:] = 0.0
    q[0, 0, 0, d_v:] = rng.standard_normal(d_qk - d_v)
    shared = rng.standard_normal(d_qk - d_v)
    kv[:, :, d_v:] = shared
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.5, d_v=d_v)
    rows = _gather(kv, bt, 0, L)
    np.testing.assert_allclose(out[0], rows[:, :d_v].mean(axis=0), atol=1e-12, rtol=0)
    z = 0.5 * float(np.dot(q[0, 0, 0, d_v:], shared))
    assert abs(lse[0] - (z + math.log(L))) <= 1e-12


def test_transposed_evaluation_agrees(oracle_mod):
    """S^T = K Q^T, column softmax over the KV axis, O = (V^T P^T)^T."""
    rng = np.random.default_rng(5)
    B, s_q, h, d_qk, d_v, page = 2, 1, 5, 64, 48, 16
    lens = [70, 128]
    q, kv, bt, sl = _dense_case(rng, B, s_q, h, d_qk, page, lens)
    scale = 0.125
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, scale, d_v=d_v)
    for b in range(B):
        K = _gather(kv, bt, b, lens[b])            # [L, d_qk]
        Qt = q[b].reshape(s_q * h, d_qk).T          # [d_qk, N]
        St = scale * (K @ Qt)                        # [L, N]
        m = St.max(axis=0, keepdims=True)
        E = np.exp(St - m)
        Pt = E / E.sum(axis=0, keepdims=True)        # softmax over the KV axis
        Ot = K[:, :d_v].T @ Pt                       # [d_v, N]
        ref_lse = (m + np.log(E.sum(axis=0, keepdims=True)))[0]
        for n in range(s_q * h):
            r = b * s_q * h + n
            np.testing.assert_allclose(out[r], Ot[:, n], atol=1e-12, rtol=0)
            assert abs(lse[r] - ref_lse[n]) <= 1e-12


def test_block_table_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(6)
    B, s_q, h, d_qk, page = 2, 2, 3, 32, 8
    lens = [37, 64]
    q, kv, bt, sl = _dense_case(rng, B, s_q, h, d_qk, page, lens, perm=False)
    nb = kv.shape[0]
    perm = rng.permutation(nb)
    inv = np.argsort(perm)
    kv2 = kv[perm]                       # physical page p of kv2 holds old page perm[p]
    bt2 = np.where(bt >= 0, inv[np.maximum(bt, 0)], -1).astype(np.int32)
    o1, l1 = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.2, causal=True, d_v=24)
    o2, l2 = oracle_mod.mla_oracle_fwd(q, kv2, bt2, sl, 0.2, causal=True, d_v=24)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_causal_consistency(oracle_mod):
    """Token s of an s_q=2 causal query sees the first L - 2 + 1 + s rows."""
    rng = np.random.default_rng(7)
    h, d_qk, page = 3, 32, 8
    L = 45
    q, kv, bt, sl = _dense_case(rng, 1, 2, h, d_qk, page, [L])
    o2, l2 = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.3, causal=True, d_v=16)
    for s, Lvis in ((0, L - 1), (1, L)):
        o1, l1 = oracle_mod.mla_oracle_fwd(q[:, s:s + 1], kv, bt, np.array([Lvis], np.int32), 0.3,
                                           d_v=16)
        np.testing.assert_array_equal(o2[s * h:(s + 1) * h], o1)
        np.testing.assert_array_equal(l2[s * h:(s + 1) * h], l1)
    # without the causal flag both tokens see all L rows
    o3, _ = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.3, causal=False, d_v=16)
    o4, _ = oracle_mod.mla_oracle_fwd(q[:, 0:1], kv, bt, sl, 0.3, d_v=16)
    np.testing.assert_array_equal(o3[:h], o4)


def test_split_associativity(oracle_mod):
    """Whole = LSE-weighted merge of two disjoint KV halves."""
    rng = np.random.default_rng(8)
    h, d_qk, d_v, page = 4, 40, 32, 8
    L1, L2 = 48, 29
    q, kv, bt, sl = _dense_case(rng, 1, 1, h, d_qk, page, [L1 + L2])
    ow, lw = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.4, d_v=d_v)
    bt_a = bt[:, :L1 // page]
    bt_b = bt[:, L1 // page:]
    oa, la = oracle_mod.mla_oracle_fwd(q, kv, bt_a, np.array([L1], np.int32), 0.4, d_v=d_v)
    ob, lb = oracle_mod.mla_oracle_fwd(q, kv, bt_b, np.array([L2], np.int32), 0.4, d_v=d_v)
    lstar = np.logaddexp(la, lb)
    merged = np.exp(la - lstar)[:, None] * oa + np.exp(lb - lstar)[:, None] * ob
    np.testing.assert_allclose(merged, ow, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lstar, lw, atol=1e-12, rtol=0)


def test_brute_force_python_floats(oracle_mod):
    rng = np.random.default_rng(9)
    for trial in range(6):
        B, s_q, h = 1 + trial % 2, 1 + (trial // 2) % 2, 1 + trial % 2
        d_qk, d_v, page = 6, 4, 2
        lens = [int(rng.integers(1, 9)) for _ in range(B)]
        causal = bool(trial % 3 == 0)
        q, kv, bt, sl = _dense_case(rng, B, s_q, h, d_qk, page, lens)
        scale = float(rng.uniform(0.2, 1.5))
        out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, scale, causal=causal, d_v=d_v)
        for b in range(B):
            for s in range(s_q):
                for hh in range(h):
                    r = (b * s_q + s) * h + hh
                    n = lens[b] - s_q + 1 + s if (causal and s_q > 1) else lens[b]
                    if n <= 0:
                        assert lse[r] == -math.inf and not out[r].any()
                        continue
                    rows = [[float(kv[bt[b, t // page], t % page, c]) for c in range(d_qk)]
                            for t in range(n)]
                    qv = [float(q[b, s, hh, c]) for c in range(d_qk)]
                    z = [scale * sum(qv[c] * rows[t][c] for c in range(d_qk)) for t in range(n)]
                    m = max(z)
                    w = [math.exp(x - m) for x in z]
                    tot = sum(w)
                    o = [sum(w[t] * rows[t][c] for t in range(n)) / tot for c in range(d_v)]
                    assert max(abs(o[c] - out[r, c]) for c in range(d_v)) <= 1e-12
                    assert abs(m + math.log(tot) - lse[r]) <= 1e-12


def test_rope_columns_are_key_only(oracle_mod):
    """For 576-wide rows the value is the first 512 columns: the 64 RoPE
    columns enter the scores only."""
    rng = np.random.default_rng(10)
    d = workloads.build(1, 1, 2, ("fixed", 70), seed=11)
    q = d["q"].double().numpy()
    kv = d["kv_cache"].double().numpy()[:, :, 0, :]
    bt, sl = d["block_table"].numpy(), d["cache_seqlens"].numpy()
    o1, l1 = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, workloads.SOFTMAX_SCALE)
    assert o1.shape == (2, 512)
    # (a) with q's RoPE part zeroed, changing the RoPE columns of the cache changes nothing
    q0 = q.copy()
    q0[..., 512:] = 0
    kv_b = kv.copy()
    kv_b[..., 512:] = rng.standard_normal(kv_b[..., 512:].shape) * 100
    oa, la = oracle_mod.mla_oracle_fwd(q0, kv, bt, sl, workloads.SOFTMAX_SCALE)
    ob, lb = oracle_mod.mla_oracle_fwd(q0, kv_b, bt, sl, workloads.SOFTMAX_SCALE)
    np.testing.assert_array_equal(oa, ob)
    np.testing.assert_array_equal(la, lb)
    # (b) with the full query, the RoPE columns do move the scores
    oc, lc = oracle_mod.mla_oracle_fwd(q, kv_b, bt, sl, workloads.SOFTMAX_SCALE)
    assert np.abs(lc - l1).max() > 1e-3
    # (c) O is a convex combination of the first 512 columns
    rows = _gather(kv, bt, 0, 70)
    assert (o1 <= rows[:, :512].max(axis=0) + 1e-12).all()
    assert (o1 >= rows[:, :512].min(axis=0) - 1e-12).all()


def test_rows_past_length_are_ignored(oracle_mod):
    d1 = workloads.build(2, 2, 2, ("list", [70, 129]), seed=12, causal=True)
    d2 = workloads.build(2, 2, 2, ("list", [70, 129]), seed=12, causal=True, tail_fill=1e4)
    assert not torch.equal(d1["kv_cache"], d2["kv_cache"])
    r1 = oracle_mod.mla_oracle_fwd(d1["q"], d1["kv_cache"], d1["block_table"], d1["cache_seqlens"],
                                   d1["softmax_scale"], causal=True)
    r2 = oracle_mod.mla_oracle_fwd(d2["q"], d2["kv_cache"], d2["block_table"], d2["cache_seqlens"],
                                   d2["softmax_scale"], causal=True)
    np.testing.assert_array_equal(r1[0], r2[0])
    np.testing.assert_array_equal(r1[1], r2[1])


def test_constant_score_shift(oracle_mod):
    """A key column shared by all rows adds scale*q_c*k_c to every score: LSE
    moves by exactly that and O does not move."""
    rng = np.random.default_rng(13)
    d_qk, d_v = 20, 12
    q, kv, bt, sl = _dense_case(rng, 1, 1, 2, d_qk, 4, [23])
    c = d_qk - 1
    kv[:, :, c] = 1.0
    q[..., c] = 0.0
    o1, l1 = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 0.6, d_v=d_v)
    q2 = q.copy()
    q2[..., c] = 2.5
    o2, l2 = oracle_mod.mla_oracle_fwd(q2, kv, bt, sl, 0.6, d_v=d_v)
    np.testing.assert_allclose(o2, o1, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l2 - l1, 0.6 * 2.5, atol=1e-12, rtol=0)


def test_empty_visible_range(oracle_mod):
    rng = np.random.default_rng(14)
    q, kv, bt, sl = _dense_case(rng, 2, 2, 2, 16, 4, [0, 1])
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 1.0, causal=True, d_v=8)
    # request 0 is empty; request 1 (L = 1) has token s=0 seeing L - 1 = 0 rows
    assert np.all(lse[:4] == -np.inf) and not out[:4].any()
    assert np.all(lse[4:6] == -np.inf) and not out[4:6].any()
    assert np.all(np.isfinite(lse[6:8]))
    np.testing.assert_array_equal(out[6], kv[bt[1, 0], 0, :8])


def test_selected_rows_match_full(oracle_mod):
    d = workloads.build(3, 2, 4, ("list", [65, 1, 200]), seed=15, causal=True)
    args = (d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"], d["softmax_scale"])
    of, lf = oracle_mod.mla_oracle_fwd(*args, causal=True)
    rows = [0, 5, 9, 17, 23]
    os_, ls = oracle_mod.mla_oracle_fwd(*args, causal=True, rows=rows)
    np.testing.assert_array_equal(os_, of[rows])
    np.testing.assert_array_equal(ls, lf[rows])


def test_bf16_bits_equal_fp64_of_same_values(oracle_mod):
    d = workloads.build(2, 1, 3, ("list", [100, 64]), seed=16)
    args_b = (d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"], d["softmax_scale"])
    ob, lb = oracle_mod.mla_oracle_fwd(*args_b)
    od, ld = oracle_mod.mla_oracle_fwd(d["q"].double().numpy(), d["kv_cache"].double().numpy(),
                                       d["block_table"], d["cache_seqlens"], d["softmax_scale"])
    np.testing.assert_array_equal(ob, od)
    np.testing.assert_array_equal(lb, ld)


def test_bad_block_table_rejected(oracle_mod):
    rng = np.random.default_rng(17)
    q, kv, bt, sl = _dense_case(rng, 1, 1, 1, 8, 4, [9])
    bt[0, 1] = kv.shape[0]
    with pytest.raises(RuntimeError, match="block table"):
        oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 1.0, d_v=4)
    bt[0, 1] = -1
    with pytest.raises(RuntimeError, match="block table"):
        oracle_mod.mla_oracle_fwd(q, kv, bt, sl, 1.0, d_v=4)
    with pytest.raises(RuntimeError, match="block table"):
        oracle_mod.mla_oracle_fwd(q, kv, bt[:, :2], np.array([13], np.int32), 1.0, d_v=4)


def test_generator_is_seeded_and_tables_are_permutations():
    a = workloads.make_inputs("b16_l4096_h16")
    b = workloads.make_inputs("b16_l4096_h16")
    c = workloads.make_inputs("b16_l4096_h16", seed=5)
    for k in ("q", "kv_cache", "block_table", "cache_seqlens"):
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["q"], c["q"])
    bt = a["block_table"]
    used = bt[bt >= 0]
    assert used.numel() == 16 * 64 and used.unique().numel() == used.numel()
    ident = workloads.make_inputs("b1_l1024_h16")["block_table"]
    assert torch.equal(ident[0], torch.arange(16, dtype=torch.int32))
    assert workloads.SOFTMAX_SCALE == pytest.approx(0.0721687836, abs=1e-10)


def test_large_scores_stay_finite_and_exact(oracle_mod):
    """Scores near 1e3 overflow exp() unless the running max is subtracted
    first; the result must still equal the two-token closed form."""
    q = np.array([0.0, 1.0]).reshape(1, 1, 1, 2)
    kv = np.array([[1.0, 1000.0], [3.0, 1000.0 + math.log(3.0)]]).reshape(1, 2, 2)
    out, lse = oracle_mod.mla_oracle_fwd(q, kv, np.zeros((1, 1), np.int32),
                                         np.array([2], np.int32), 1.0, d_v=1)
    assert abs(out[0, 0] - 2.5) <= 1e-12
    assert abs(lse[0] - (1000.0 + math.log(4.0))) <= 1e-9
