"""The allocation-free entry point, mla_decode_fwd_noalloc.

Some callers cannot allocate device memory: a runtime or plugin host that
plans every device buffer in advance and hands a kernel library no allocator,
or a decode loop that cannot pay cudaMalloc's implicit device
synchronisation.  For them the library offers one call that takes only the
inputs and outputs and keeps its schedule and split partials in a fixed
device array of its own.

These tests call it through the C ABI, twice in a row on the same inputs
(the second call finds the first call's leftovers in that array), and check
both results against the allocating path (mla_decode_get_schedule +
mla_decode_fwd with caller buffers), within the same tolerances as the
parity tests.  This file is collected last so that a run that stops at the
first failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import helpers
from mla_decode_attention_15_b200 import _build, binding as bd, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    return torch.device("cuda:0")


def _allocating(d, dims, dev):
    sched = torch.empty(bd.mla_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
    ws = torch.empty(bd.mla_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    B, s_q, h, _ = d["q"].shape
    out = torch.empty(B, s_q, h, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
    bd.mla_decode_get_schedule(dims, d["cache_seqlens"], sched)
    bd.mla_decode_fwd(dims, sched, ws, d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                      d["softmax_scale"], out, lse)
    torch.cuda.synchronize()
    assert bd.mla_decode_get_status(sched) == 0
    return out, lse


def _noalloc(d, dims, dev):
    B, s_q, h, _ = d["q"].shape
    out = torch.full((B, s_q, h, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, h, s_q), float("nan"), dtype=torch.float32, device=dev)
    L = bd.lib()
    rc = L.mla_decode_fwd_noalloc(ctypes.byref(dims), d["q"].data_ptr(), d["kv_cache"].data_ptr(),
                                  d["block_table"].data_ptr(), d["cache_seqlens"].data_ptr(),
                                  ctypes.c_float(d["softmax_scale"]), out.data_ptr(), lse.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == bd.MLA_OK, bd.mla_decode_strerror(rc)
    torch.cuda.synchronize()
    return out, lse


def _close(out, lse, ref_out, ref_lse):
    """The parity tolerances, with the allocating path as the reference."""
    o = out.double().cpu().numpy()
    r = ref_out.double().cpu().numpy()
    err = np.abs(o - r)
    assert np.isfinite(o).all()
    assert err.max() <= helpers.MAX_REL * max(np.abs(r).max(), 1e-30)
    assert np.sqrt(np.mean(err ** 2)) <= helpers.RMSE_BAR
    l, rl = lse.double().cpu().numpy(), ref_lse.double().cpu().numpy()
    assert np.array_equal(np.isneginf(l), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert (np.abs(l[fin] - rl[fin]) <= helpers.LSE_REL * np.maximum(1.0, np.abs(rl[fin]))).all()


@pytest.mark.parametrize("name,seed", [("b16_l4096_h16", None), ("b16_sq2_ragged1k16k_h16_peaked", None)])
def test_noalloc_matches_allocating_path_on_two_calls_in_a_row(dev, name, seed):
    w = workloads.WORKLOADS[name]
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
         for k, v in workloads.make_inputs(w, seed=seed).items()}
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    dims = bd.make_dims(w.batch, w.s_q, w.heads, d["kv_cache"].shape[0], d["block_table"].shape[1],
                        w.causal, sms)
    ref_out, ref_lse = _allocating(d, dims, dev)
    for _ in range(2):
        out, lse = _noalloc(d, dims, dev)
        _close(out, lse, ref_out, ref_lse)


def test_noalloc_after_a_different_shape_still_matches(dev):
    """A call with other lengths first leaves a different plan in the shared
    scratch; the next call must not depend on it."""
    a = workloads.build(3, 1, 16, ("list", [5000, 64, 2222]), seed=7)
    b = workloads.build(2, 2, 16, ("list", [130, 9000]), seed=8, causal=True)
    for d in (a, b, a):
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        B, s_q, h, _ = d["q"].shape
        dims = bd.make_dims(B, s_q, h, d["kv_cache"].shape[0], d["block_table"].shape[1], d["causal"], 148)
        ref_out, ref_lse = _allocating(d, dims, dev)
        out, lse = _noalloc(d, dims, dev)
        _close(out, lse, ref_out, ref_lse)


def test_noalloc_rejects_requests_beyond_its_scratch(dev):
    # 10000 persistent CTAs would need ~650 MB of split partials: refused
    # before anything is enqueued.
    dims = bd.make_dims(16, 1, 16, 100, 10, False, 10000)
    L = bd.lib()
    rc = L.mla_decode_fwd_noalloc(ctypes.byref(dims), 0x1000, 0x2000, 0x3000, 0x4000, ctypes.c_float(0.07),
                                  0x5000, 0x6000, None)
    assert rc == bd.MLA_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in bd.mla_decode_strerror(rc)
    flags = bd.make_dims(16, 1, 16, 100, 10, False, 148, bd.MLA_FLAG_NO_COMBINE)
    assert L.mla_decode_fwd_noalloc(ctypes.byref(flags), 0x1000, 0x2000, 0x3000, 0x4000, ctypes.c_float(0.07),
                                    0x5000, 0x6000, None) == bd.MLA_ERR_INVALID_ARG
