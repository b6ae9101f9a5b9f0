"""Integer invariants of the split-KV plan, computed on the host by
mla_decode_get_schedule_host (the same plan the device kernel builds; a GPU
test checks the two are bit-identical)."""
import numpy as np
import pytest
import torch

import helpers
from mla_decode_attention_15_b200 import _build, binding as bd, workloads


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bd.lib()


def host_plan(seqlens, s_q, heads, G, max_blocks=None):
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).contiguous()
    B = seqlens.numel()
    if max_blocks is None:
        max_blocks = max(1, (int(seqlens.clamp(min=0).max()) + 63) // 64)
    d = bd.make_dims(B, s_q, heads, 10 ** 6, max_blocks, False, G)
    n = bd.mla_decode_schedule_bytes(d)
    buf = torch.zeros(n, dtype=torch.uint8)
    bd.mla_decode_get_schedule_host(d, seqlens, buf)
    N = heads * s_q
    words = buf.numpy().view(np.int32)
    if N <= 64:  # one-CTA kernels: one plan row per request-group, 64-token pages
        Hg, BG, Gp, shift, share = 1, B, G, 6, 1
    else:        # CTA pairs: one row per request, 128-token steps, ranges shared by the groups
        share = (N + 127) // 128
        Hg, BG, Gp, shift = 1, B, max(1, max(1, G // 2) // share), 7
    assert (int(words[1]), int(words[2]), int(words[3]), int(words[11]), int(words[12])) == (Gp, BG, Hg, shift, share)
    hdr, meta, bginfo, prefix = helpers.read_plan(buf.numpy(), Gp, BG)
    return dict(hdr=hdr, meta=meta, bginfo=bginfo, prefix=prefix, Hg=Hg, BG=BG, G=Gp, shift=shift, share=share,
                seqlens=seqlens.numpy(), max_blocks=max_blocks)


def check_invariants(pl):
    seq, Hg, BG, G, mb = pl["seqlens"], pl["Hg"], pl["BG"], pl["G"], pl["max_blocks"]
    hdr, meta, bginfo = pl["hdr"], pl["meta"], pl["bginfo"]
    assert hdr[0] == 0x4D4C4144 and hdr[1] == G and hdr[2] == BG and hdr[3] == Hg
    T = int(hdr[6])
    unit = 1 << pl["shift"]
    items = helpers.walk_plan(meta, bginfo, seq, Hg, mb, pl["shift"])
    pages = [(min(max(int(seq[bg // Hg]), 0), mb * 64) + unit - 1) // unit for bg in range(BG)]
    covered = [np.zeros(P, dtype=np.int64) for P in pages]
    pieces = [[] for _ in range(BG)]
    for k, its in enumerate(items):
        load = 0
        for (bg, p0, p1, unsplit, slot) in its:
            covered[bg][p0:p1] += 1
            pieces[bg].append((k, p0, p1, unsplit, slot))
            load += (p1 - p0)
        # a CTA never carries more than its share of units (pages + 1 per item)
        assert load + len(its) * helpers.OVERHEAD <= T + helpers.OVERHEAD, (k, its, T)
        # only the first and the last item of a CTA can be partial
        for (bg, p0, p1, unsplit, slot) in its[1:-1]:
            assert unsplit
    for bg in range(BG):
        assert (covered[bg] == 1).all(), bg  # every page exactly once
        ns = int(bginfo[bg, 1])
        assert ns == len(pieces[bg]), (bg, ns, pieces[bg])
        if ns == 1:
            assert pieces[bg][0][3]  # unsplit, written directly
        if ns > 1:
            slots = [pc[4] for pc in pieces[bg]]  # in split order (ascending range)
            base = int(bginfo[bg, 0])
            if pl["shift"] == 6:
                # the slots the combine reads (split_slot) are the ones the pieces were written to
                expect = [base if i == 0 else 2 * ((base >> 1) + i) for i in range(ns)]
                assert slots == expect, (bg, slots, expect)
                assert pieces[bg][0][0] == base >> 1  # split 0 sits on the group's first range
            else:
                assert sorted(slots) == list(range(base, base + ns))
            assert not any(pc[3] for pc in pieces[bg])
    used = [pc[4] for bg in range(BG) for pc in pieces[bg] if not pc[3]]
    assert len(used) == len(set(used)), "two partials share a slot"
    if pl["shift"] == 6:
        assert all(0 <= x < 2 * G for x in used)
    total_slots = sum(int(bginfo[bg, 1]) for bg in range(BG) if bginfo[bg, 1] > 1)
    assert total_slots == int(hdr[5]) <= 2 * G
    return items


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_plan_of_each_workload(name):
    w = workloads.WORKLOADS[name]
    g = torch.Generator().manual_seed(w.seed)
    if w.lens[0] == "fixed":
        lens = [w.lens[1]] * w.batch
    else:
        lens = torch.randint(w.lens[1], w.lens[2] + 1, (w.batch,), generator=g).tolist()
    pl = host_plan(lens, w.s_q, w.heads, 148)
    items = check_invariants(pl)
    busy = sum(1 for its in items if its)
    W = int(pl["hdr"][8])
    assert busy == min(pl["G"], -(-W // int(pl["hdr"][6])))


@pytest.mark.parametrize("G", [1, 2, 7, 148, 300])
@pytest.mark.parametrize("heads,s_q", [(16, 1), (16, 2), (1, 1), (3, 2), (24, 2), (40, 2), (128, 1), (128, 2)])
def test_plan_random_ragged(G, heads, s_q):
    rng = np.random.default_rng(G * 1000 + heads * 10 + s_q)
    lens = rng.integers(0, 3000, size=int(rng.integers(1, 40))).tolist()
    lens[0] = 0
    check_invariants(host_plan(lens, s_q, heads, G))


def test_plan_long_single_request_spreads_over_all_ctas():
    pl = host_plan([65536], 1, 16, 148)
    items = check_invariants(pl)
    busy = [its for its in items if its]
    assert all(len(its) == 1 for its in busy)
    T = int(pl["hdr"][6])
    assert T == -(-(1024 + 1) // 148)
    assert len(busy) == -(-(1024 + 1) // T) >= 140
    assert int(pl["bginfo"][0, 1]) == len(busy)


def test_plan_short_batch_uses_few_ctas():
    pl = host_plan([1024], 1, 16, 148)  # 16 pages: 17 units, at least 2 per range (1 page + the item's unit)
    items = check_invariants(pl)
    busy = [its for its in items if its]
    assert int(pl["hdr"][6]) == 2
    assert len(busy) == 9
    assert all(p1 - p0 >= 1 for its in busy for (_, p0, p1, _, _) in its)


def test_plan_clamps_and_flags_bad_lengths():
    pl = host_plan([100, -5, 10 ** 6], 1, 16, 8, max_blocks=4)
    assert pl["hdr"][7] & bd.MLA_STATUS_BAD_SEQLEN
    items = check_invariants(pl)
    assert int(pl["bginfo"][1, 1]) == 0          # negative length: empty request
    total = sum(p1 - p0 for its in items for (bg, p0, p1, _, _) in its if bg == 2)
    assert total == 4                            # clamped to the table's 4 pages
    ok = host_plan([100, 5], 1, 16, 8, max_blocks=4)
    assert ok["hdr"][7] == 0


def gqa_host_plan(seqlens, s_q, groups, G, max_blocks=None):
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).contiguous()
    B = seqlens.numel()
    if max_blocks is None:
        max_blocks = max(1, (int(seqlens.clamp(min=0).max()) + 63) // 64)
    d = bd.make_gqa_dims(B, s_q, groups, 10 ** 6, max_blocks, s_q > 1, G)
    buf = torch.zeros(bd.mla_gqa_decode_schedule_bytes(d), dtype=torch.uint8)
    bd.mla_gqa_decode_get_schedule_host(d, seqlens, buf)
    if groups > 1 and G // groups >= 1:   # shared ranges: one plan row per request
        Gp, BG, Hg, share = G // groups, B, 1, groups
    else:                                 # one plan row per request-group
        Gp, BG, Hg, share = G, B * groups, groups, 1
    words = buf.numpy().view(np.int32)
    assert (int(words[1]), int(words[2]), int(words[3]), int(words[4]), int(words[11]), int(words[12])) == \
        (Gp, BG, Hg, 16 * s_q, 6, share)
    hdr, meta, bginfo, prefix = helpers.read_plan(buf.numpy(), Gp, BG)
    return dict(hdr=hdr, meta=meta, bginfo=bginfo, prefix=prefix, Hg=Hg, BG=BG, G=Gp, shift=6, share=share,
                seqlens=seqlens.numpy(), max_blocks=max_blocks)


@pytest.mark.parametrize("G", [1, 7, 16, 148])
@pytest.mark.parametrize("groups", [1, 2, 8])
@pytest.mark.parametrize("s_q", [1, 2])
def test_gqa_plan_random_ragged(G, groups, s_q):
    """The GQA plan: with several KV groups (and at least one range per group)
    one row per request, each range walked by all groups; every page of every
    request once, partial slots unique and split counts consistent."""
    rng = np.random.default_rng(G * 100 + groups * 10 + s_q)
    lens = rng.integers(0, 5000, size=int(rng.integers(1, 30))).tolist()
    lens[0] = 0
    pl = gqa_host_plan(lens, s_q, groups, G)
    check_invariants(pl)
    # the slots a shared range's CTAs write (fixed slot x groups + group) fit the workspace
    d = bd.make_gqa_dims(len(lens), s_q, groups, 10 ** 6, pl["max_blocks"], s_q > 1, G)
    slot_bytes = 16 * s_q * (128 + 1) * 4
    assert bd.mla_gqa_decode_workspace_bytes(d) == 2 * pl["G"] * pl["share"] * slot_bytes
