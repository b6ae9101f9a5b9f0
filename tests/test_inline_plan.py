"""MLA_FLAG_INLINE_PLAN: the decode kernel builds its split-KV plan from the
lengths in its own prologue, instead of reading the plan the schedule kernel
wrote.  GPU checks: the plan it leaves in the schedule buffer equals the host
plan word for word; its outputs are bitwise those of the two-launch path (the
same kernels on the same plan); it follows lengths that change between calls
with no new mla_decode_get_schedule; and the status word keeps the documented
rule (cleared only by mla_decode_get_schedule)."""
import numpy as np
import pytest
import torch

import helpers
import oracle
from mla_decode_attention_15_b200 import _build, binding as bd, workloads

pytestmark = pytest.mark.gpu

HDR_STATUS = 7


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    oracle.build()
    return torch.device("cuda:0")


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def decoder(g, inline, num_sms=0, fp32_out=False, dev=None):
    B, s_q, h, _ = g["q"].shape
    return bd.MlaDecoder(B, s_q, h, g["kv_cache"].shape[0], g["block_table"].shape[1], g["causal"], num_sms,
                         dev, fp32_out=fp32_out, inline_plan=inline)


def run(g, dev, inline, num_sms=0, fp32_out=False, no_combine=False):
    dec = decoder(g, inline, num_sms, fp32_out, dev)
    if no_combine:
        dec.dims.flags |= bd.MLA_FLAG_NO_COMBINE
    dec.plan(g["cache_seqlens"])
    out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    if no_combine:
        bd.mla_decode_combine(dec.dims, dec.schedule, dec.workspace, dec.out, dec.lse)
    torch.cuda.synchronize()
    return out.clone(), lse.clone(), dec


def same_as_two_launch_path(d, dev, num_sms=0, fp32_out=False):
    g = to_dev(d, dev)
    o1, l1, d1 = run(g, dev, False, num_sms, fp32_out)
    o2, l2, d2 = run(g, dev, True, num_sms, fp32_out)
    assert d1.status() == 0 and d2.status() == 0
    assert torch.equal(o1, o2), (o1 - o2).abs().max()
    assert torch.equal(torch.nan_to_num(l1, neginf=-1e30), torch.nan_to_num(l2, neginf=-1e30))
    return o2, l2


@pytest.mark.parametrize("name", ["b1_l1024_h16", "b16_l4096_h16", "b16_sq2_ragged1k16k_h16_peaked"])
def test_workloads_match_two_launch_path_and_oracle(dev, name):
    d = workloads.make_inputs(name)
    out, lse = same_as_two_launch_path(d, dev)
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], causal=d["causal"])
    helpers.compare(out, lse, ro, rl)


@pytest.mark.parametrize("num_sms", [1, 3, 148])
@pytest.mark.parametrize("heads,s_q", [(16, 1), (16, 2), (1, 1), (3, 2), (24, 2), (40, 1), (64, 1), (128, 2)])
def test_ragged_heads_and_grids_match_two_launch_path(dev, heads, s_q, num_sms):
    lens = [1, 2, 0, 63, 64, 65, 127, 128, 130, 1000, 4099]
    d = workloads.build(len(lens), s_q, heads, ("list", lens), seed=5 + heads + num_sms, causal=s_q > 1)
    same_as_two_launch_path(d, dev, num_sms)


@pytest.mark.parametrize("lens,s_q", [([66000], 1), ([9000, 3000], 2)])
def test_many_splits_match_two_launch_path_and_oracle(dev, lens, s_q):
    """Short batches over long contexts: 148, 71 and 24 splits per column,
    merged in d_v slices by the small combine grid."""
    d = workloads.build(len(lens), s_q, 16, ("list", lens), seed=9 + s_q, causal=s_q > 1)
    out, lse = same_as_two_launch_path(d, dev, 148)
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], causal=d["causal"])
    helpers.compare(out, lse, ro, rl)


def test_fp32_output_matches_two_launch_path(dev):
    lens = [5000, 64, 2222, 1]
    d = workloads.build(len(lens), 2, 16, ("list", lens), seed=17, causal=True)
    same_as_two_launch_path(d, dev, 148, fp32_out=True)


@pytest.mark.parametrize("lens,heads,s_q,G", [
    ([1024], 16, 1, 148), ([4096] * 16, 16, 1, 148), ([0, 5, 64, 65, 9000, 1, 130], 16, 2, 148),
    ([0, 5, 64, 65, 9000, 1, 130], 16, 2, 3), ([300, 77, 1025], 24, 2, 148), ([65536] * 2, 16, 1, 148),
    ([0, 0, 0], 16, 1, 148)])
def test_written_plan_equals_host_plan(dev, lens, heads, s_q, G):
    """Every word of the schedule buffer but the status word is rewritten by
    the decode kernel and equals the host plan; the status word is kept."""
    d = workloads.build(len(lens), s_q, heads, ("list", lens), seed=29, causal=s_q > 1)
    g = to_dev(d, dev)
    dec = decoder(g, True, G, dev=dev)
    dec.plan(g["cache_seqlens"])
    words = dec.schedule.view(torch.int32)
    words[:HDR_STATUS] = 0x7FAB7FAB
    words[HDR_STATUS + 1:] = 0x7FAB7FAB
    dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() == 0
    host = torch.zeros(dec.schedule.numel(), dtype=torch.uint8)
    bd.mla_decode_get_schedule_host(dec.dims, d["cache_seqlens"], host)
    got = dec.schedule.cpu().view(torch.int32).numpy()
    want = host.view(torch.int32).numpy()
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, (diff[:10], got[diff[:10]], want[diff[:10]])


def test_plan_at_the_shared_memory_limit(dev):
    """18,384 one-page requests: the largest plan the kernel builds in one page
    stage; one more request and the call runs the schedule kernel first."""
    for B in (18384, 18385):
        lens = [1 + (i * 37) % 64 for i in range(B)]
        d = workloads.build(B, 1, 16, ("list", lens), seed=B, spare_pages=1, pool_device="cuda")
        g = to_dev(d, dev)
        o1, l1, d1 = run(g, dev, False)
        o2, l2, d2 = run(g, dev, True)
        assert d1.status() == 0 and d2.status() == 0
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        assert torch.equal(d1.schedule[:4 * HDR_STATUS], d2.schedule[:4 * HDR_STATUS])
    rows = list(range(0, 18384, 997))
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"].cpu(), d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], causal=False, rows=rows)
    helpers.compare(o2, l2, ro, rl, rows=rows)


def test_gqa_matches_two_launch_path(dev):
    """8 KV groups walk shared ranges (one plan row per request: 6 and 1,300
    rows); one KV group with 10,200 requests has more plan rows than the
    kernel builds in one 40 KB page stage, so the call runs the schedule
    kernel first."""
    for B, groups, lens in ((6, 8, [1, 64, 65, 1000, 0, 3000]), (1300, 8, None), (10200, 1, None)):
        if lens is None:
            lens = [1 + (i * 53) % 130 for i in range(B)]
        d = workloads.build_gqa(B, 2, groups, ("list", lens), seed=B, causal=True, pool_device="cuda")
        g = to_dev(d, dev)
        res = []
        for inline in (False, True):
            dec = bd.GqaDecoder(B, 2, groups, g["kv_cache"].shape[0], g["block_table"].shape[1], True, 0, dev,
                                inline_plan=inline)
            dec.plan(g["cache_seqlens"])
            out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
            torch.cuda.synchronize()
            assert dec.status() == 0
            res.append((out.clone(), lse.clone()))
        assert torch.equal(res[0][0], res[1][0])
        assert torch.equal(torch.nan_to_num(res[0][1], neginf=-1e30), torch.nan_to_num(res[1][1], neginf=-1e30))


def test_explicit_combine_matches_fused_launch(dev):
    d = workloads.build(3, 1, 16, ("list", [5000, 64, 2222]), seed=71)
    g = to_dev(d, dev)
    o1, l1, _ = run(g, dev, True, 16)
    o2, l2, _ = run(g, dev, True, 16, no_combine=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lengths_that_change_need_no_new_plan(dev):
    """The plan follows cache_seqlens at every call: the lengths change on the
    device between calls, with no mla_decode_get_schedule in between."""
    lens_a = [9000, 70, 0, 2049]
    lens_b = [130, 70, 0, 1]  # within each request's block-table row
    d = workloads.build(4, 2, 16, ("list", lens_a), seed=73, causal=True)
    g = to_dev(d, dev)
    dec = decoder(g, True, 0, dev=dev)
    dec.plan(g["cache_seqlens"])
    dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    g["cache_seqlens"].copy_(torch.tensor(lens_b, dtype=torch.int32))
    out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() == 0
    db = dict(d)
    db["cache_seqlens"] = torch.tensor(lens_b, dtype=torch.int32)
    ro, rl = oracle.mla_oracle_fwd(db["q"], db["kv_cache"], db["block_table"], db["cache_seqlens"],
                                   db["softmax_scale"], causal=True)
    helpers.compare(out, lse, ro, rl)


def test_status_word_is_sticky_until_get_schedule(dev):
    lens = [300, 200]
    d = workloads.build(2, 1, 16, ("list", lens), seed=91)
    g = to_dev(d, dev)
    dec = decoder(g, True, 0, dev=dev)
    dec.plan(g["cache_seqlens"])
    assert dec.status() == 0
    bad = g["cache_seqlens"].clone()
    bad[1] = 64 * g["block_table"].shape[1] + 1  # beyond the table: clamped and reported
    dec(g["q"], g["kv_cache"], g["block_table"], bad, g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() & bd.MLA_STATUS_BAD_SEQLEN
    dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() & bd.MLA_STATUS_BAD_SEQLEN  # kept: only get_schedule clears it
    dec.plan(g["cache_seqlens"])
    torch.cuda.synchronize()
    assert dec.status() == 0


def test_poisoned_workspace_and_outputs(dev):
    lens = [1, 64, 1000, 5000, 130, 0, 4099, 3000]
    d = workloads.build(len(lens), 2, 16, ("list", lens), seed=777, causal=True)
    g = to_dev(d, dev)
    dec = decoder(g, True, 148, dev=dev)
    dec.workspace.view(torch.float32).fill_(float("nan"))
    dec.out.fill_(float("nan"))
    dec.lse.fill_(float("nan"))
    dec.plan(g["cache_seqlens"])
    dec.schedule.view(torch.int32)[HDR_STATUS + 1:] = -1
    out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() == 0
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], causal=True)
    helpers.compare(out, lse, ro, rl)


@pytest.mark.parametrize("groups,G", [(8, 148), (2, 148), (8, 7), (1, 148)])
def test_gqa_written_plan_equals_host_plan(dev, groups, G):
    """The GQA plan built in the decode kernel (shared ranges for 2 and 8 KV
    groups on 148 SMs; one row per request-group for 8 groups on 7 SMs and
    for one group) equals the host plan word for word."""
    lens = [0, 5, 64, 65, 9000, 1, 130, 2500]
    d = workloads.build_gqa(len(lens), 2, groups, ("list", lens), seed=31 + groups, causal=True)
    g = to_dev(d, dev)
    dec = bd.GqaDecoder(len(lens), 2, groups, g["kv_cache"].shape[0], g["block_table"].shape[1], True, G, dev,
                        inline_plan=True)
    dec.plan(g["cache_seqlens"])
    words = dec.schedule.view(torch.int32)
    words[:HDR_STATUS] = 0x7FAB7FAB
    words[HDR_STATUS + 1:] = 0x7FAB7FAB
    dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    assert dec.status() == 0
    host = torch.zeros(dec.schedule.numel(), dtype=torch.uint8)
    bd.mla_gqa_decode_get_schedule_host(dec.dims, d["cache_seqlens"], host)
    got = dec.schedule.cpu().view(torch.int32).numpy()
    want = host.view(torch.int32).numpy()
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, (diff[:10], got[diff[:10]], want[diff[:10]])
