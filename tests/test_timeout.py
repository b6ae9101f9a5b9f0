"""The decode kernel's bounded waits, exercised on the GPU without a fault.

MLA_FLAG_TEST_STALL makes every CTA's producer leave one page unloaded, so a
wait in the kernel runs out after its 1 s limit.  The call must report
MLA_STATUS_TIMEOUT through the status word, and the same CUDA context must
decode correctly afterwards."""
import pytest
import torch

import helpers
import oracle
from mla_decode_attention_15_b200 import _build, binding as bd, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    oracle.build()
    return torch.device("cuda:0")


def _decode(d, dev, flags=0, num_sms=4):
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    B, s_q, h, _ = g["q"].shape
    dec = bd.MlaDecoder(B, s_q, h, g["kv_cache"].shape[0], g["block_table"].shape[1], g["causal"], num_sms, dev)
    dec.dims.flags = flags
    dec.plan(g["cache_seqlens"])
    out, lse = dec(g["q"], g["kv_cache"], g["block_table"], g["cache_seqlens"], g["softmax_scale"])
    torch.cuda.synchronize()
    return out, lse, dec.status()


@pytest.mark.parametrize("heads", [16, 128])
def test_wait_timeout_is_reported_and_the_device_stays_usable(dev, heads):
    d = workloads.build(2, 2, heads, ("list", [700, 300]), seed=95, causal=True)
    _, _, status = _decode(d, dev, flags=bd.MLA_FLAG_TEST_STALL)
    assert status & bd.MLA_STATUS_TIMEOUT, hex(status)
    good = workloads.build(2, 2, heads, ("list", [700, 300]), seed=96, causal=True)
    out, lse, status = _decode(good, dev)
    assert status == 0
    ro, rl = oracle.mla_oracle_fwd(good["q"], good["kv_cache"], good["block_table"], good["cache_seqlens"],
                                   good["softmax_scale"], causal=True)
    helpers.compare(out, lse, ro, rl)
