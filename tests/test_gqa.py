"""GQA path over a group-expanded cache (GQLA summary, "Arquitetura", item 2):
C-ABI checks on the CPU and parity of the sm_100a path against the fp64 GQA
oracle on the GPU (tolerances of helpers.py)."""
import ctypes

import numpy as np
import pytest
import torch

import helpers
import oracle
from mla_decode_attention_15_b200 import _build, binding as bd, workloads


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return bd.lib()


def test_gqa_sizes_and_rejections(lib):
    # 8 KV groups share each work range (one CTA per group): 148 // 8 = 18 ranges,
    # one plan row per request, 2 partial slots per range and group
    d = bd.make_gqa_dims(16, 2, 8, 1000, 64, True, 148)
    G, BG = 148 // 8, 16
    assert bd.mla_gqa_decode_schedule_bytes(d) == 4 * (16 + 8 * G + 3 * BG + 1)
    assert bd.mla_gqa_decode_workspace_bytes(d) == 2 * G * 8 * 32 * (128 + 1) * 4
    # one KV group, or too few SMs for one range per group: one plan row per request-group
    d1 = bd.make_gqa_dims(16, 2, 1, 1000, 64, True, 148)
    assert bd.mla_gqa_decode_schedule_bytes(d1) == 4 * (16 + 8 * 148 + 3 * 16 + 1)
    d7 = bd.make_gqa_dims(16, 2, 8, 1000, 64, True, 7)
    assert bd.mla_gqa_decode_schedule_bytes(d7) == 4 * (16 + 8 * 7 + 3 * 128 + 1)
    for change, code in [(dict(num_q_heads=24), bd.MLA_ERR_UNSUPPORTED), (dict(s_q=3), bd.MLA_ERR_UNSUPPORTED),
                         (dict(d_head=64), bd.MLA_ERR_UNSUPPORTED), (dict(page_size=32), bd.MLA_ERR_UNSUPPORTED),
                         (dict(batch=0), bd.MLA_ERR_INVALID_ARG), (dict(flags=0x100), bd.MLA_ERR_INVALID_ARG),
                         (dict(num_kv_groups=0), bd.MLA_ERR_INVALID_ARG)]:
        bad = bd.make_gqa_dims(2, 1, 2, 100, 10, False, 148)
        for k, v in change.items():
            setattr(bad, k, v)
        assert bd.mla_gqa_decode_schedule_bytes(bad) == 0, change
        rc = lib.mla_gqa_decode_fwd(ctypes.byref(bad), 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000,
                                    ctypes.c_float(0.07), 0x70000, 0x80000, None)
        assert rc == code, (change, rc)


# ------------------------------------------------------------------ GPU parity
@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    oracle.build()
    return torch.device("cuda:0")


def run_gqa(d, dev, num_sms=0, flags=0):
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    B, s_q = g["q"].shape[0], g["q"].shape[1]
    dec = bd.GqaDecoder(B, s_q, d["groups"], g["kv_cache"].shape[0], g["block_table"].shape[1], g["causal"],
                        num_sms, dev)
    dec.dims.flags = flags
    dec.plan(g["cache_seqlens"])
    out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    if flags & bd.MLA_FLAG_NO_COMBINE:
        bd.mla_gqa_decode_combine(dec.dims, dec.schedule, dec.workspace, dec.out, dec.lse)
    torch.cuda.synchronize()
    assert dec.status() == 0
    return out.clone(), lse.clone()


def ref(d, rows=None):
    kv = d["kv_cache"].cpu() if d["kv_cache"].is_cuda else d["kv_cache"]
    return oracle.gqa_oracle_fwd(d["q"], kv, d["block_table"], d["cache_seqlens"], d["softmax_scale"],
                                 d["groups"], causal=d["causal"], rows=rows)


@pytest.mark.gpu
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True)])
@pytest.mark.parametrize("groups", [1, 2, 8])
@pytest.mark.parametrize("num_sms", [148, 7, 1])
def test_gqa_ragged_tails(dev, s_q, causal, groups, num_sms):
    lens = [1, 63, 64, 65, 1000, 300]
    d = workloads.build_gqa(len(lens), s_q, groups, ("list", lens), seed=500 + groups * 10 + s_q, causal=causal)
    out, lse = run_gqa(d, dev, num_sms=num_sms)
    ro, rl = ref(d)
    helpers.compare(out, lse, ro, rl)


@pytest.mark.gpu
def test_gqa_explicit_combine_matches_fused(dev):
    d = workloads.build_gqa(3, 2, 2, ("list", [5000, 64, 2222]), seed=520, causal=True)
    o1, l1 = run_gqa(d, dev, num_sms=16)
    o2, l2 = run_gqa(d, dev, num_sms=16, flags=bd.MLA_FLAG_NO_COMBINE)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_gqa_bench_shape_sampled_rows(dev):
    """bs16, s_q 2 causal, 8 KV groups (128 query heads), 16K context: the
    shape bench.py times for this path."""
    d = workloads.build_gqa(16, 2, 8, ("fixed", 16384), seed=1005, causal=True, pool_device="cuda")
    out, lse = run_gqa(d, dev)
    rng = np.random.default_rng(5)
    rows = sorted(set(int(x) for x in rng.integers(0, 16 * 2 * 128, 24)))
    ro, rl = ref(d, rows)
    m = helpers.compare(out, lse, ro, rl, rows=rows)
    print(m)
