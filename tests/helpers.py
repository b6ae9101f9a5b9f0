"""Shared test helpers: comparison against the oracle and a reader of the
split-KV plan.  Test infrastructure only."""
from __future__ import annotations

import re
import os

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")

# Tolerances (bf16 inputs and outputs, fp32 accumulation):
#   max|O - O_ref| <= 1e-2 * max|O_ref|
#   RMSE(O - O_ref) <= 5e-4, or 5e-4 + q where q = RMSE(bf16(O_ref) - O_ref) > 2.5e-4
#     (rounding the exact result to bf16 alone already costs q; peaked rows)
#   |LSE - LSE_ref| <= 1e-5 * max(1, |LSE_ref|), and -inf exactly where the oracle has -inf
MAX_REL = 1e-2
RMSE_BAR = 5e-4
LSE_REL = 1e-5


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(mla_(?:(?:gqa_)?decode|absorb)_\w+)\s*\(", text, re.M)))


def bf16_floor(ref: np.ndarray) -> float:
    r = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    return float(np.sqrt(np.mean((r - ref) ** 2))) if ref.size else 0.0


def compare(out_gpu: torch.Tensor, lse_gpu: torch.Tensor, ref_out: np.ndarray, ref_lse: np.ndarray,
            rows=None, heads=None, s_q=None):
    """out_gpu [B,s_q,h,512] bf16 (or fp32), lse_gpu [B,h,s_q] fp32 (device or host);
    ref_* from the oracle over flattened rows r = (b*s_q+s)*h+head (all, or ``rows``).
    Returns a dict of metrics and asserts the tolerances.  An fp32 output (the
    result before any bf16 rounding) is held to the literal RMSE bar, with no
    allowance for the bf16 rounding floor."""
    B, sq, h, dv = out_gpu.shape
    o = out_gpu.detach().double().cpu().numpy().reshape(B * sq * h, dv)
    l = lse_gpu.detach().double().cpu().numpy()  # [B, h, s_q]
    l = np.transpose(l, (0, 2, 1)).reshape(B * sq * h)
    if rows is not None:
        o = o[np.asarray(rows)]
        l = l[np.asarray(rows)]
    err = o - ref_out
    finite = np.isfinite(ref_lse)
    m = dict(
        max_abs_err=float(np.abs(err).max()) if err.size else 0.0,
        max_ref=float(np.abs(ref_out).max()) if ref_out.size else 0.0,
        rmse=float(np.sqrt(np.mean(err ** 2))) if err.size else 0.0,
        q_floor=bf16_floor(ref_out),
    )
    lse_err = np.abs(l[finite] - ref_lse[finite]) / np.maximum(1.0, np.abs(ref_lse[finite]))
    m["lse_rel_err"] = float(lse_err.max()) if lse_err.size else 0.0
    literal = out_gpu.dtype == torch.float32 or m["q_floor"] <= 2.5e-4
    m["rmse_bar"] = RMSE_BAR if literal else RMSE_BAR + m["q_floor"]
    assert np.isfinite(o).all(), "non-finite output"
    assert np.array_equal(np.isneginf(l), np.isneginf(ref_lse)), "LSE -inf pattern differs"
    assert not np.isnan(l).any()
    assert m["max_abs_err"] <= MAX_REL * max(m["max_ref"], 1e-30) or m["max_abs_err"] == 0.0, m
    assert m["rmse"] <= m["rmse_bar"], m
    assert m["lse_rel_err"] <= LSE_REL, m
    return m


# ---------------------------------------------------------------- plan reader
HDR_WORDS, META_WORDS, BG_WORDS = 16, 8, 2
OVERHEAD = 1


def read_plan(buf: np.ndarray, G: int, BG: int):
    w = buf.view(np.int32)
    hdr = w[:HDR_WORDS]
    meta = w[HDR_WORDS:HDR_WORDS + META_WORDS * G].reshape(G, META_WORDS)
    off = HDR_WORDS + META_WORDS * G
    bginfo = w[off:off + BG_WORDS * BG].reshape(BG, BG_WORDS)
    prefix = w[off + BG_WORDS * BG: off + BG_WORDS * BG + BG + 1]
    return hdr, meta, bginfo, prefix


def walk_plan(meta, bginfo, seqlens, Hg, max_blocks, shift=6):
    """Items each work range holds, exactly as the decode kernels walk it:
    list per range of (bg, p0, p1, unsplit, slot), in units of 2^shift tokens
    (64-token pages, or the CTA-pair kernel's 128-token steps).  The one-CTA
    kernels (64-token units) put the partial of range k's first item in slot
    2k and that of its last in 2k + 1; the CTA-pair plans count slots per
    request (slot base of the request + split index; the head group offset is
    left out here)."""
    BG = bginfo.shape[0]
    unit = 1 << shift
    out = []
    for k in range(meta.shape[0]):
        bb, bp, eb, ep, fs = (int(x) for x in meta[k, :5])
        items = []
        bg = bb
        while bg <= eb and bg < BG:
            cur = bg
            bg += 1
            L = min(max(int(seqlens[cur // Hg]), 0), max_blocks * 64)
            P = (L + unit - 1) // unit
            p0 = bp if cur == bb else 0
            p1 = ep if cur == eb else P
            p1 = min(p1, P)
            if p0 >= p1:
                continue
            unsplit = p0 == 0 and p1 == P
            if unsplit:
                slot = -1
            elif shift == 6:
                slot = 2 * k + (0 if cur == bb else 1)
            else:
                slot = int(bginfo[cur, 0]) + (fs if cur == bb else 0)
            items.append((cur, p0, p1, unsplit, slot))
        out.append(items)
    return out
