"""fp64 CPU oracle for absorbed-MQA MLA decode (and for the GQLA GQA path over
a group-expanded cache, ``gqa_oracle_fwd``): TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports, links or calls it, and it
shares no code with them.

The arithmetic lives in ``mla_oracle.c`` (plain C99 + OpenMP, fp64); this file
only compiles that source with gcc and marshals arguments through ctypes.  See
the header of ``mla_oracle.c`` for the definition computed and the passages of
the FlashMLA-ETAP and GQLA pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

ERRORS = {0: "ok", -1: "bad argument", -2: "bad block table", -3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.mla_oracle_fwd.restype = ctypes.c_int
        lib.mla_oracle_fwd.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_longlong,
            ctypes.c_int,
        ]
        lib.gqa_oracle_fwd.restype = ctypes.c_int
        lib.gqa_oracle_fwd.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ]
        lib.mla_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().mla_oracle_max_threads())


def _as_np(x, dtype):
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu()
        if x.dtype == torch.bfloat16:
            return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16))
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def mla_oracle_fwd(q, kv, block_table, cache_seqlens, softmax_scale, causal=False,
                   d_v=None, rows=None, want_probs=False, num_threads=0):
    """Run the oracle.

    q: [B, s_q, h, d_qk]; kv: [num_blocks, page, (1,) d_qk] -- both bf16 torch
    tensors (their bits are passed through exactly) or float64 arrays.
    block_table [B, max_blocks] int32, cache_seqlens [B] int32.  d_v defaults
    to 512 for 576-wide rows (the latent part of the row), else to d_qk.

    Returns (out [R, d_v] float64, lse [R] float64[, probs [R, max_L]]) for
    the flattened query rows r = (b*s_q + s)*h + head: all of them in that
    order, or those listed in ``rows``.
    """
    lib = _load()
    is_bf16 = isinstance(q, torch.Tensor) and q.dtype == torch.bfloat16
    if isinstance(kv, torch.Tensor) and (kv.dtype == torch.bfloat16) != is_bf16:
        raise TypeError("q and kv must both be bf16 or both be float64")
    qn = _as_np(q, np.float64)
    kvn = _as_np(kv, np.float64)
    B, s_q, h, d_qk = qn.shape
    num_blocks, page = kvn.shape[0], kvn.shape[1]
    if kvn.shape[-1] != d_qk:
        raise ValueError("kv row width must equal q width")
    if d_v is None:
        d_v = 512 if d_qk == 576 else d_qk
    bt = _as_np(block_table, np.int32).astype(np.int32)
    sl = _as_np(cache_seqlens, np.int32).astype(np.int32)
    if bt.ndim != 2 or bt.shape[0] != B or sl.shape != (B,):
        raise ValueError("block_table must be [B, max_blocks] and cache_seqlens [B]")
    if rows is None:
        nrows = B * s_q * h
        rows_np = None
    else:
        rows_np = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nrows = rows_np.shape[0]
    out = np.zeros((nrows, d_v), dtype=np.float64)
    lse = np.zeros((nrows,), dtype=np.float64)
    probs = None
    stride = 0
    if want_probs:
        stride = max(int(sl.max()) if B else 1, 1)
        probs = np.zeros((nrows, stride), dtype=np.float64)
    rc = lib.mla_oracle_fwd(
        B, s_q, h, d_qk, d_v, page, int(bool(causal)), bt.shape[1], num_blocks,
        qn.ctypes.data, kvn.ctypes.data, int(is_bf16),
        bt.ctypes.data, sl.ctypes.data,
        float(softmax_scale),
        rows_np.ctypes.data if rows_np is not None else None, int(nrows),
        out.ctypes.data, lse.ctypes.data,
        probs.ctypes.data if probs is not None else None, stride,
        int(num_threads))
    if rc != 0:
        raise RuntimeError("mla_oracle_fwd failed: %s (%d)" % (ERRORS.get(rc, "?"), rc))
    if want_probs:
        return out, lse, probs
    return out, lse


def gqa_oracle_fwd(q, kv, block_table, cache_seqlens, softmax_scale, groups, d_head=128, causal=False,
                   rows=None, num_threads=0):
    """Run the GQA-path oracle (see ``gqa_oracle_fwd`` in mla_oracle.c).

    q: [B, s_q, h_q, d_head + d_rope]; kv: [num_blocks, page, (1,)
    2*groups*d_head + d_rope]; both bf16 torch tensors or float64 arrays.
    Returns (out [R, d_head] float64, lse [R] float64) for the flattened
    query rows r = (b*s_q + s)*h_q + head, all of them or those in ``rows``.
    """
    lib = _load()
    is_bf16 = isinstance(q, torch.Tensor) and q.dtype == torch.bfloat16
    if isinstance(kv, torch.Tensor) and (kv.dtype == torch.bfloat16) != is_bf16:
        raise TypeError("q and kv must both be bf16 or both be float64")
    qn = _as_np(q, np.float64)
    kvn = _as_np(kv, np.float64)
    B, s_q, h, d_q = qn.shape
    d_rope = d_q - d_head
    num_blocks, page = kvn.shape[0], kvn.shape[1]
    if d_rope < 0 or kvn.shape[-1] != 2 * groups * d_head + d_rope:
        raise ValueError("kv row width must be 2*groups*d_head + d_rope")
    bt = _as_np(block_table, np.int32).astype(np.int32)
    sl = _as_np(cache_seqlens, np.int32).astype(np.int32)
    if rows is None:
        nrows, rows_np = B * s_q * h, None
    else:
        rows_np = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nrows = rows_np.shape[0]
    out = np.zeros((nrows, d_head), dtype=np.float64)
    lse = np.zeros((nrows,), dtype=np.float64)
    rc = lib.gqa_oracle_fwd(
        B, s_q, h, int(groups), int(d_head), int(d_rope), page, int(bool(causal)), bt.shape[1], num_blocks,
        qn.ctypes.data, kvn.ctypes.data, int(is_bf16), bt.ctypes.data, sl.ctypes.data,
        float(softmax_scale), rows_np.ctypes.data if rows_np is not None else None, int(nrows),
        out.ctypes.data, lse.ctypes.data, int(num_threads))
    if rc != 0:
        raise RuntimeError("gqa_oracle_fwd failed: %s (%d)" % (ERRORS.get(rc, "?"), rc))
    return out, lse
