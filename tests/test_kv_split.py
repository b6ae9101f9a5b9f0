"""Split-KV across ranks: the page split and causal assignment (host logic of
mla_decode_attention_15_b200.kv_split), the merge oracle, a world-size-2 gloo
run of the exchange on the CPU, and on one GPU the CUDA merge
(mla_decode_combine_ranks) of R shard decodes run one after another.

The merge oracle (oracle/merge.py) is pinned here against the whole-context
decode oracle: merging the shards' exact results must reproduce it to fp64
rounding, with causal s_q = 2 and with ranks that hold no page of a request."""
import datetime
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import helpers
import oracle
from oracle import merge
from mla_decode_attention_15_b200 import _build, binding as bd, kv_split, workloads


def test_page_ranges_tile_each_request():
    for P in range(0, 41):
        for R in range(1, 9):
            ranges = [kv_split.page_range(P, R, r) for r in range(R)]
            assert ranges[0][0] == 0 and ranges[-1][1] == P
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0 and a0 <= a1
            if P >= 1:
                assert ranges[-1][1] - ranges[-1][0] >= 1  # the last rank holds the tail
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        kv_split.page_range(4, 2, 2)


def test_shard_reassembles_the_batch():
    d = workloads.build(5, 1, 2, ("list", [1, 63, 64, 65, 700]), seed=61)
    sl, bt = d["cache_seqlens"], d["block_table"]
    for R in (1, 2, 3, 5):
        parts = [kv_split.shard(sl, bt, R, r) for r in range(R)]
        for b in range(5):
            L = int(sl[b])
            lens = [int(p[0][b]) for p in parts]
            assert sum(lens) == L
            assert all(x % 64 == 0 for x in lens[:-1])  # only the last rank has a partial page
            pages = [int(x) for p in parts for x in p[1][b] if x >= 0]
            assert pages == [int(x) for x in bt[b, :(L + 63) // 64]]
    assert [kv_split.rank_causal(True, 3, r) for r in range(3)] == [False, False, True]
    assert not kv_split.rank_causal(False, 3, 2)


def test_split_takes_one_or_two_new_tokens():
    """With s_q = 3 the two hidden positions of query token 0 can straddle a
    rank boundary (L = 65 over 2 ranks: rank 0 holds position 63), so the split
    refuses it, as the decode library does."""
    kv_split.check_s_q(1)
    kv_split.check_s_q(2)
    for bad in (0, 3, 4):
        with pytest.raises(ValueError):
            kv_split.check_s_q(bad)
        with pytest.raises(ValueError):
            kv_split.KvSplitDecoder(1, bad, 16, 10, 10, causal=True)
        with pytest.raises(ValueError):
            kv_split.KvSplitGqaDecoder(1, bad, 1, 10, 10, causal=True)


def _shard_oracle(d, R, causal):
    outs, lses = [], []
    for r in range(R):
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], R, r)
        o, l = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], bt, sl, d["softmax_scale"],
                                     causal=kv_split.rank_causal(causal, R, r))
        outs.append(o)
        lses.append(l)
    return outs, lses


@pytest.mark.parametrize("R,s_q,causal", [(2, 1, False), (3, 2, True), (4, 2, True)])
def test_merge_oracle_reproduces_the_whole(oracle_mod, R, s_q, causal):
    lens = [1, 2, 64, 65, 130, 257]  # requests shorter than R pages leave ranks empty
    d = workloads.build(len(lens), s_q, 2, ("list", lens), seed=62 + R)
    ow, lw = oracle_mod.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                       d["softmax_scale"], causal=causal)
    outs, lses = _shard_oracle(d, R, causal)
    assert any(np.isneginf(l).any() for l in lses)  # an empty shard took part
    om, lm = merge.merge_partials(np.stack(outs), np.stack(lses))
    np.testing.assert_allclose(om, ow, rtol=0, atol=1e-12)
    fin = np.isfinite(lw)
    assert np.array_equal(np.isneginf(lm), np.isneginf(lw))
    np.testing.assert_allclose(lm[fin], lw[fin], rtol=0, atol=1e-12)


def test_merge_oracle_special_cases():
    o = np.arange(12, dtype=np.float64).reshape(1, 3, 4)
    l = np.array([[0.5, -1.0, 2.0]])
    om, lm = merge.merge_partials(o, l)  # one part: identity
    np.testing.assert_array_equal(om, o[0])
    np.testing.assert_array_equal(lm, l[0])
    o2 = np.stack([o[0], 100 + o[0]])
    l2 = np.stack([l[0], np.full(3, -np.inf)])  # an empty part weighs nothing
    om, lm = merge.merge_partials(o2, l2)
    np.testing.assert_array_equal(om, o[0])
    np.testing.assert_array_equal(lm, l[0])
    om, lm = merge.merge_partials(o2, np.full((2, 3), -np.inf))  # nothing visible anywhere
    assert not om.any() and np.isneginf(lm).all()
    l3 = np.stack([np.zeros(3), np.zeros(3)])  # equal shares: the mean, LSE + ln 2
    om, lm = merge.merge_partials(o2, l3)
    np.testing.assert_allclose(om, (o2[0] + o2[1]) / 2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, np.log(2.0), rtol=0, atol=1e-15)


def _gloo_rank(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = workloads.build(4, 2, 2, ("list", [3, 64, 200, 129]), seed=71)
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], world, rank)
        o, l = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], bt, sl, d["softmax_scale"],
                                     causal=kv_split.rank_causal(True, world, rank))
        o_all = kv_split.gather(torch.from_numpy(o), None)
        l_all = kv_split.gather(torch.from_numpy(l), None)
        om, lm = merge.merge_partials(o_all.numpy(), l_all.numpy())
        ow, lw = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                       d["softmax_scale"], causal=True)
        ok = np.allclose(om, ow, rtol=0, atol=1e-12) and np.allclose(lm, lw, rtol=0, atol=1e-12)
        with open("%s.%d" % (result_path, rank), "w") as f:
            f.write("ok" if ok else "mismatch %g" % np.abs(om - ow).max())
    finally:
        dist.destroy_process_group()


def test_gloo_world2_exchange_and_merge(oracle_mod, tmp_path):
    """Two CPU ranks: shard, decode with the oracle, all-gather over gloo
    with kv_split.gather, merge; both ranks reproduce the whole decode."""
    port = 29000 + os.getpid() % 1000
    path = str(tmp_path / "res")
    mp.start_processes(_gloo_rank, args=(2, port, path), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        assert open("%s.%d" % (path, r)).read() == "ok"


def _gloo_rank_gqa(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = workloads.build_gqa(3, 2, 2, ("list", [2, 129, 300]), seed=72, causal=True)
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], world, rank)
        o, l = oracle.gqa_oracle_fwd(d["q"], d["kv_cache"], bt, sl, d["softmax_scale"], d["groups"],
                                     causal=kv_split.rank_causal(True, world, rank))
        om, lm = merge.merge_partials(kv_split.gather(torch.from_numpy(o), None).numpy(),
                                      kv_split.gather(torch.from_numpy(l), None).numpy())
        ow, lw = oracle.gqa_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                       d["softmax_scale"], d["groups"], causal=True)
        fin = np.isfinite(lw)
        ok = (np.allclose(om, ow, rtol=0, atol=1e-12) and np.array_equal(np.isneginf(lm), np.isneginf(lw))
              and np.allclose(lm[fin], lw[fin], rtol=0, atol=1e-12))
        with open("%s.%d" % (result_path, rank), "w") as f:
            f.write("ok" if ok else "mismatch %g" % np.abs(om - ow).max())
    finally:
        dist.destroy_process_group()


def test_gloo_world2_gqa_path(oracle_mod, tmp_path):
    """The same exchange for the GQA path: two CPU ranks, GQA oracle on each
    shard (causal s_q 2, 2 KV groups), gather over gloo, merge = whole."""
    port = 29000 + (os.getpid() + 500) % 1000
    path = str(tmp_path / "res_gqa")
    mp.start_processes(_gloo_rank_gqa, args=(2, port, path), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        assert open("%s.%d" % (path, r)).read() == "ok"


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return bd.lib()


def test_combine_ranks_rejections(lib):
    f = lib.mla_decode_combine_ranks
    good = (2, 4, 1, 16, 512, 0x1000, 0x2000, 0x3000, 0x4000, None)
    for i, v in [(0, 0), (0, 65), (1, 0), (2, 0), (3, 0), (5, None), (6, 0x2004), (7, None), (8, 0x4008)]:
        args = list(good)
        args[i] = v
        assert f(*args) == bd.MLA_ERR_INVALID_ARG, (i, v)
    args = list(good)
    args[4] = 576
    assert f(*args) == bd.MLA_ERR_UNSUPPORTED


# ------------------------------------------------------------------ GPU
@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    oracle.build()
    return torch.device("cuda:0")


@pytest.mark.gpu
@pytest.mark.parametrize("parts", ["fp32", "bf16"])
@pytest.mark.parametrize("R,s_q,causal,heads", [(2, 1, False, 16), (3, 2, True, 16), (4, 2, True, 128),
                                                (8, 1, False, 16)])
def test_split_decode_then_merge_matches_whole_oracle(dev, R, s_q, causal, heads, parts):
    """R ranks emulated on one GPU, one after another (no kernel waits on
    another): each decodes its shard with the C-ABI path, the stacked
    results are merged by mla_decode_combine_ranks(_f32), and the merge is
    compared with the whole-context oracle.  With fp32 parts (what
    KvSplitDecoder exchanges) the merged row is rounded once, so its RMSE
    stays within 1.1x of the unsplit single-GPU decode's on the same inputs."""
    lens = [1, 65, 640, 1000, 4096, 3000]
    d = workloads.build(len(lens), s_q, heads, ("list", lens), seed=90 + R, sigma=0.5 if heads == 128 else 1.0)
    B = len(lens)
    f32 = parts == "fp32"
    q, kv = d["q"].to(dev), d["kv_cache"].to(dev)
    o_parts = torch.empty(R, B, s_q, heads, 512, dtype=torch.float32 if f32 else torch.bfloat16, device=dev)
    l_parts = torch.empty(R, B, heads, s_q, dtype=torch.float32, device=dev)
    for r in range(R):
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], R, r)
        dec = bd.MlaDecoder(B, s_q, heads, kv.shape[0], bt.shape[1], kv_split.rank_causal(causal, R, r), 0, dev,
                            fp32_out=f32)
        sl_d, bt_d = sl.to(dev), bt.to(dev)
        dec.plan(sl_d)
        o, l = dec(q, kv, bt_d, sl_d, d["softmax_scale"])
        o_parts[r].copy_(o)
        l_parts[r].copy_(l)
        torch.cuda.synchronize()
        assert dec.status() == 0
    out = torch.empty(B, s_q, heads, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, heads, s_q, dtype=torch.float32, device=dev)
    bd.mla_decode_combine_ranks(o_parts, l_parts, out, lse)
    torch.cuda.synchronize()
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], causal=causal)
    m = helpers.compare(out, lse, ro, rl)
    if f32:
        whole = bd.MlaDecoder(B, s_q, heads, kv.shape[0], d["block_table"].shape[1], causal, 0, dev)
        sl_d, bt_d = d["cache_seqlens"].to(dev), d["block_table"].to(dev)
        whole.plan(sl_d)
        ow, lw = whole(q, kv, bt_d, sl_d, d["softmax_scale"])
        torch.cuda.synchronize()
        mw = helpers.compare(ow, lw, ro, rl)
        assert m["rmse"] <= 1.1 * mw["rmse"], (m, mw)


@pytest.mark.gpu
@pytest.mark.parametrize("R,groups", [(2, 2), (3, 8)])
def test_gqa_split_decode_then_merge_matches_whole_oracle(dev, R, groups):
    """The GQA path split over R emulated ranks (causal s_q 2): shard decodes
    through the C ABI one after another, merged by mla_decode_combine_ranks
    (d_v 128), against the whole-context GQA oracle."""
    lens = [1, 65, 640, 3000]
    d = workloads.build_gqa(len(lens), 2, groups, ("list", lens), seed=96 + R, causal=True)
    B, h = len(lens), 16 * groups
    q, kv = d["q"].to(dev), d["kv_cache"].to(dev)
    o_parts = torch.empty(R, B, 2, h, 128, dtype=torch.bfloat16, device=dev)
    l_parts = torch.empty(R, B, h, 2, dtype=torch.float32, device=dev)
    for r in range(R):
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], R, r)
        dec = bd.GqaDecoder(B, 2, groups, kv.shape[0], bt.shape[1], kv_split.rank_causal(True, R, r), 0, dev)
        sl_d, bt_d = sl.to(dev), bt.to(dev)
        dec.plan(sl_d)
        o, l = dec(q, kv, bt_d, sl_d, d["softmax_scale"])
        o_parts[r].copy_(o)
        l_parts[r].copy_(l)
        torch.cuda.synchronize()
        assert dec.status() == 0
    out = torch.empty(B, 2, h, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, h, 2, dtype=torch.float32, device=dev)
    bd.mla_decode_combine_ranks(o_parts, l_parts, out, lse)
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                   d["softmax_scale"], groups, causal=True)
    helpers.compare(out, lse, ro, rl)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_combine_ranks_kernel_against_merge_oracle(dev, dtype):
    """The merge kernel alone on random partials (d_v 512 and 128; bf16 or
    fp32 parts), with empty ranks and an all-empty row, against the fp64
    merge oracle: one bf16 rounding of an fp32 sum of R terms."""
    g = torch.Generator().manual_seed(93)
    for d_v in (512, 128):
        R, B, s_q, h = 5, 3, 2, 16
        o = (torch.randn(R, B, s_q, h, d_v, generator=g)).to(dtype)
        l = torch.randn(R, B, h, s_q, generator=g) * 4
        l[1] = -float("inf")
        l[:, 0, 3, 1] = -float("inf")
        out = torch.empty(B, s_q, h, d_v, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
        bd.mla_decode_combine_ranks(o.to(dev), l.to(dev), out, lse)
        torch.cuda.synchronize()
        rows = B * s_q * h
        # merge oracle over flattened rows (b*s_q+s)*h+head; LSE rows in the same order
        lo = l.permute(0, 1, 3, 2).reshape(R, rows).double().numpy()
        om, lm = merge.merge_partials(o.reshape(R, rows, d_v).double().numpy(), lo)
        got = out.reshape(rows, d_v).double().cpu().numpy()
        mag = merge.merge_partials(np.abs(o.reshape(R, rows, d_v).double().numpy()), lo)[0]
        tol = 2.0 ** -8 * np.abs(om) + 1e-5 * mag + 1e-30
        assert (np.abs(got - om) <= tol).all()
        gl = lse.permute(0, 2, 1).reshape(rows).double().cpu().numpy()
        assert np.array_equal(np.isneginf(gl), np.isneginf(lm))
        fin = np.isfinite(lm)
        assert np.abs(gl[fin] - lm[fin]).max() <= 1e-5 * max(1.0, np.abs(lm[fin]).max())
        assert not got[~fin].any()


def _nccl_one_rank(rank, port, result_path):
    """KvSplitDecoder end to end in a one-rank NCCL group: local decode,
    NCCL all-gather, CUDA merge (a single rank waits on no other)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    msg = "not run"
    try:
        dev = torch.device("cuda:0")
        d = workloads.build(3, 2, 16, ("list", [1, 65, 3000]), seed=95)
        sl, bt = kv_split.shard(d["cache_seqlens"], d["block_table"], 1, 0)
        dec = kv_split.KvSplitDecoder(3, 2, 16, d["kv_cache"].shape[0], bt.shape[1], causal=True, device=dev)
        sl_d, bt_d = sl.to(dev), bt.to(dev)
        dec.plan(sl_d)
        out, lse = dec(d["q"].to(dev), d["kv_cache"].to(dev), bt_d, sl_d, d["softmax_scale"])
        torch.cuda.synchronize()
        assert dec.dec.status() == 0
        ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                       d["softmax_scale"], causal=True)
        helpers.compare(out, lse, ro, rl)
        msg = "ok"
    except Exception as e:  # reported to the parent through the result file
        msg = "error: %r" % (e,)
    finally:
        dist.destroy_process_group()
        with open(result_path, "w") as f:
            f.write(msg)


@pytest.mark.gpu
def test_kv_split_decoder_one_rank_nccl(dev, tmp_path):
    port = 30000 + os.getpid() % 1000
    path = str(tmp_path / "nccl_res")
    mp.start_processes(_nccl_one_rank, args=(port, path), nprocs=1, start_method="spawn", join=True)
    assert open(path).read() == "ok"
