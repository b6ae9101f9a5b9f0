"""Absorbed projections (GQLA summary, "Caminho MQA-Absorvido"): the latent
query q_nope . W_UK and the output projection O . W_UV, as tcgen05 kernels
behind mla_absorb_q / mla_absorb_o.  C-ABI checks on the CPU; parity with the
fp64 oracle (oracle/absorb.py) on the GPU.

Tolerance, from the arithmetic: the kernel accumulates K = 128 (query side) or
512 (output side) bf16 products exactly in fp32 and rounds once to bf16, so
per element |gpu - exact| <= 2^-8 |exact| (bf16 rounding, half an ulp of an
8-bit significand) + K 2^-24 sum_k |a_k b_k| (fp32 summation), with a factor
1 + 2^-8 on the second term for the final rounding.  sum_k |a_k b_k| is the
oracle applied to |a| and |b|.  The RoPE part passes through bit for bit."""
import ctypes

import numpy as np
import pytest
import torch

import helpers
from mla_decode_attention_15_b200 import _build, binding as bd, workloads


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return bd.lib()


def test_absorb_rejections(lib):
    ok = bd.make_absorb_dims(16, 16)
    for fn in (lib.mla_absorb_q, lib.mla_absorb_o):
        assert fn(None, 0x1000, 0x2000, 0x3000, None, None) == bd.MLA_ERR_INVALID_ARG
        for i in range(3):
            ptrs = [0x1000, 0x2000, 0x3000]
            ptrs[i] = None
            assert fn(ctypes.byref(ok), *ptrs, None, None) == bd.MLA_ERR_INVALID_ARG, i
            ptrs[i] = 0x4008
            assert fn(ctypes.byref(ok), *ptrs, None, None) == bd.MLA_ERR_INVALID_ARG, i
        assert fn(ctypes.byref(ok), 0x1000, 0x2000, 0x3000, 0x5002, None) == bd.MLA_ERR_INVALID_ARG
        for change, code in [(dict(tokens=0), bd.MLA_ERR_INVALID_ARG),
                             (dict(tokens=65535 * 64 + 1), bd.MLA_ERR_INVALID_ARG),
                             (dict(num_heads=0), bd.MLA_ERR_INVALID_ARG),
                             (dict(d_nope=64), bd.MLA_ERR_UNSUPPORTED), (dict(d_rope=0), bd.MLA_ERR_UNSUPPORTED),
                             (dict(d_latent=576), bd.MLA_ERR_UNSUPPORTED),
                             (dict(d_v_head=64), bd.MLA_ERR_UNSUPPORTED)]:
            d = bd.make_absorb_dims(16, 16)
            for k, v in change.items():
                setattr(d, k, v)
            assert fn(ctypes.byref(d), 0x1000, 0x2000, 0x3000, None, None) == code, change


def test_absorb_python_wrappers_check_shapes():
    q = torch.zeros(4, 2, 192, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bd.absorb_q(q, torch.zeros(2, 128, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        bd.absorb_o(torch.zeros(4, 2, 512, dtype=torch.float32), torch.zeros(2, 512, 128, dtype=torch.bfloat16))


# ------------------------------------------------------------------ GPU parity
@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _build.build()
    bd.lib()
    return torch.device("cuda:0")


def _f64(t):
    return t.double().numpy()


def _check_product(got, a, b, exact_fn, K):
    """got: bf16 tensor; exact_fn(a, b) the fp64 oracle product."""
    exact = exact_fn(a, b)
    mag = exact_fn(a.abs(), b.abs())
    tol = 2.0 ** -8 * np.abs(exact) + K * 2.0 ** -24 * mag * (1 + 2.0 ** -8)
    err = np.abs(_f64(got.cpu()) - exact)
    bad = err > tol
    assert not bad.any(), "max err %g at %s (tol %g)" % (err.max(), np.argwhere(bad)[0], tol.flat[err.argmax()])


def _run(dev, T, h, seed):
    from oracle import absorb
    x = workloads.build_absorb(T, h, seed)
    g = {k: v.to(dev) for k, v in x.items()}
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    # Outputs get a guard row past the end: nothing may be written there.
    q_buf = torch.full((T + 1, h, 576), 7.0, dtype=torch.bfloat16, device=dev)
    o_buf = torch.full((T + 1, h, 128), 7.0, dtype=torch.bfloat16, device=dev)
    d = bd.make_absorb_dims(T, h)
    bd.mla_absorb_q(d, g["q_in"], g["w_uk"], q_buf[:T], status)
    bd.mla_absorb_o(d, g["o"], g["w_uv"], o_buf[:T], status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    assert bool((q_buf[T] == 7.0).all()) and bool((o_buf[T] == 7.0).all())
    q_out, out = q_buf[:T].cpu(), o_buf[:T].cpu()
    _check_product(q_out[..., :512], x["q_in"], x["w_uk"], lambda a, b: absorb.absorb_q(a, b)[..., :512], 128)
    assert torch.equal(q_out[..., 512:], x["q_in"][..., 128:])
    _check_product(out, x["o"], x["w_uv"], absorb.absorb_o, 512)
    return q_out, out


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1, 16, 63, 64, 65, 130])
@pytest.mark.parametrize("h", [1, 3, 16])
def test_absorb_parity_ragged_tokens(dev, T, h):
    _run(dev, T, h, seed=700 + 7 * T + h)


@pytest.mark.gpu
@pytest.mark.parametrize("T,h", [(16, 128), (64, 128), (32, 16)])
def test_absorb_parity_decode_sizes(dev, T, h):
    """Decode batches of the measured configurations: bs16 / bs32 x s_q 1-2
    tokens with 16 or 128 heads."""
    _run(dev, T, h, seed=800 + T + h)


@pytest.mark.gpu
def test_absorb_wrappers_and_streams(dev):
    """The tensor-level wrappers give the same bits as the C-ABI calls, on a
    side stream too, for a [B, s_q, h, .] layout."""
    x = workloads.build_absorb(2 * 8, 16, seed=901)
    q = x["q_in"].view(8, 2, 16, 192).to(dev)
    o = x["o"].view(8, 2, 16, 512).to(dev)
    w_uk, w_uv = x["w_uk"].to(dev), x["w_uv"].to(dev)
    ref_q, ref_o = bd.absorb_q(q, w_uk), bd.absorb_o(o, w_uv)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got_q, got_o = bd.absorb_q(q, w_uk, stream=s), bd.absorb_o(o, w_uv, stream=s)
    s.synchronize()
    assert got_q.shape == (8, 2, 16, 576) and got_o.shape == (8, 2, 16, 128)
    assert torch.equal(got_q, ref_q) and torch.equal(got_o, ref_o)


@pytest.mark.gpu
@pytest.mark.parametrize("inline", [False, True])
@pytest.mark.parametrize("heads,s_q,causal", [(16, 1, False), (128, 2, True)])
def test_absorbed_decode_step_matches_oracle_chain(dev, heads, s_q, causal, inline):
    """absorb_q -> decode over the latent cache -> absorb_o through the C
    ABI, step by step, against the oracle chain started from the GPU's own
    latent query (whose projection is checked element by element in the
    tests above):
      - the decode's output and LSE meet the decode tolerances against the
        fp64 decode oracle of that query;
      - each element of the projected output is within the error the decode
        carried into it, pushed through W_UV exactly (|e| . |W_UV|), plus one
        bf16 rounding of the result and the fp32 summation of 512 products;
      - the one-call chain ``absorbed_mla_decode`` gives the same bits.
    With ``inline`` the decode builds its plan and loads its first pages
    while the query projection before it (which lets its dependents start
    early) is still running: it must still read the projected query."""
    import oracle
    from oracle import absorb
    lens = [1, 70, 1000, 2500]
    B = len(lens)
    d = workloads.build(B, s_q, heads, ("list", lens), seed=950 + heads, causal=causal,
                        sigma=0.5 if heads == 128 else 1.0)
    x = workloads.build_absorb(B * s_q, heads, seed=960 + heads)
    q_in = x["q_in"].view(B, s_q, heads, 192)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    w_uk, w_uv = x["w_uk"].to(dev), x["w_uv"].to(dev)
    dec = bd.MlaDecoder(B, s_q, heads, g["kv_cache"].shape[0], g["block_table"].shape[1], causal, 0, dev,
                        inline_plan=inline)
    dec.plan(g["cache_seqlens"])
    q_lat = bd.absorb_q(q_in.to(dev), w_uk)
    o_lat, lse = dec(q_lat, g["kv_cache"], g["block_table"], g["cache_seqlens"], d["softmax_scale"])
    o_lat, lse = o_lat.clone(), lse.clone()
    out = bd.absorb_o(o_lat, w_uv)
    out_chain, lse_chain = bd.absorbed_mla_decode(q_in.to(dev), w_uk, w_uv, g["kv_cache"], g["block_table"],
                                                  g["cache_seqlens"], d["softmax_scale"], dec)
    torch.cuda.synchronize()
    assert dec.status() == 0 and out.shape == (B, s_q, heads, 128)
    assert torch.equal(out_chain, out) and torch.equal(lse_chain, lse)
    o_ref, l_ref = oracle.mla_oracle_fwd(q_lat.cpu(), d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                         d["softmax_scale"], causal=causal)
    helpers.compare(o_lat, lse, o_ref, l_ref)
    T = B * s_q
    ref = absorb.absorb_o(o_ref.reshape(T, heads, 512), x["w_uv"])          # [T, h, 128]
    o_got = o_lat.double().cpu().numpy().reshape(T, heads, 512)
    w_abs = np.abs(x["w_uv"].double().numpy())
    e = np.abs(o_got - o_ref.reshape(T, heads, 512))
    bound = (np.einsum("thk,hkn->thn", e, w_abs) + 2.0 ** -8 * np.abs(ref)
             + 512 * 2.0 ** -24 * np.einsum("thk,hkn->thn", np.abs(o_got), w_abs) + 1e-30)
    got = out.double().cpu().numpy().reshape(T, heads, 128)
    assert (np.abs(got - ref) <= bound).all()
