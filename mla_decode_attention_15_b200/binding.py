"""Python binding of the C ABI in include/mla_decode.h (ctypes).

Argument marshalling only: every step of the decode runs in the CUDA kernels
of libmla_decode.so.  PyTorch supplies device memory and the stream.  There is
no fallback: if the library is missing or the device is not an sm_100 part,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import _build

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_BAD_SCHEDULE = -4
MLA_ERR_SCRATCH_TOO_SMALL = -5
MLA_NOALLOC_SCRATCH_BYTES = 24 << 20

MLA_STATUS_BAD_BLOCK_TABLE = 0x1
MLA_STATUS_TIMEOUT = 0x2
MLA_STATUS_BAD_SEQLEN = 0x4
MLA_STATUS_BAD_SCHEDULE = 0x8
MLA_STATUS_SMEM_ALIGN = 0x10

MLA_FLAG_NO_COMBINE = 0x1
MLA_FLAG_TEST_STALL = 0x2
MLA_FLAG_FP32_OUT = 0x4
MLA_FLAG_INLINE_PLAN = 0x8

PAGE_SIZE = 64
D_QK = 576
D_V = 512

EXPORTED = (
    "mla_decode_schedule_bytes",
    "mla_decode_workspace_bytes",
    "mla_decode_get_schedule",
    "mla_decode_get_schedule_host",
    "mla_decode_fwd",
    "mla_decode_fwd_noalloc",
    "mla_decode_combine",
    "mla_decode_get_status",
    "mla_decode_strerror",
    "mla_decode_version",
    "mla_gqa_decode_schedule_bytes",
    "mla_gqa_decode_workspace_bytes",
    "mla_gqa_decode_get_schedule",
    "mla_gqa_decode_get_schedule_host",
    "mla_gqa_decode_fwd",
    "mla_gqa_decode_combine",
    "mla_absorb_q",
    "mla_absorb_o",
    "mla_decode_combine_ranks",
    "mla_decode_combine_ranks_f32",
)

GQA_D_HEAD = 128
GQA_D_ROPE = 64
GQA_HEADS_PER_GROUP = 16

ABSORB_D_NOPE = 128
ABSORB_D_ROPE = 64
ABSORB_D_LATENT = 512
ABSORB_D_V_HEAD = 128


class MlaDecodeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, mla_decode_strerror(code), code))


class mla_decode_dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "batch", "s_q", "num_heads", "num_blocks", "max_blocks_per_seq", "page_size",
        "d_qk", "d_v", "causal", "num_sms", "flags", "reserved")]


class mla_gqa_dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "batch", "s_q", "num_q_heads", "num_kv_groups", "num_blocks", "max_blocks_per_seq", "page_size",
        "d_head", "d_rope", "causal", "num_sms", "flags")]


class mla_absorb_dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "tokens", "num_heads", "d_nope", "d_rope", "d_latent", "d_v_head")]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load libmla_decode.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_build.LIB):
            raise RuntimeError("CUDA library %s is not built; run __graft_entry__.build() "
                               "(nvcc, sm_100a)" % _build.LIB)
        L = ctypes.CDLL(_build.LIB)
        P = ctypes.POINTER(mla_decode_dims)
        vp = ctypes.c_void_p
        L.mla_decode_schedule_bytes.restype = ctypes.c_size_t
        L.mla_decode_schedule_bytes.argtypes = [P]
        L.mla_decode_workspace_bytes.restype = ctypes.c_size_t
        L.mla_decode_workspace_bytes.argtypes = [P]
        L.mla_decode_get_schedule.restype = ctypes.c_int
        L.mla_decode_get_schedule.argtypes = [P, vp, vp, vp]
        L.mla_decode_get_schedule_host.restype = ctypes.c_int
        L.mla_decode_get_schedule_host.argtypes = [P, vp, vp]
        L.mla_decode_fwd.restype = ctypes.c_int
        L.mla_decode_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp]
        L.mla_decode_fwd_noalloc.restype = ctypes.c_int
        L.mla_decode_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp]
        L.mla_decode_combine.restype = ctypes.c_int
        L.mla_decode_combine.argtypes = [P, vp, vp, vp, vp, vp]
        L.mla_decode_get_status.restype = ctypes.c_int
        L.mla_decode_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.mla_decode_strerror.restype = ctypes.c_char_p
        L.mla_decode_strerror.argtypes = [ctypes.c_int]
        L.mla_decode_version.restype = ctypes.c_int
        L.mla_decode_version.argtypes = []
        Q = ctypes.POINTER(mla_gqa_dims)
        L.mla_gqa_decode_schedule_bytes.restype = ctypes.c_size_t
        L.mla_gqa_decode_schedule_bytes.argtypes = [Q]
        L.mla_gqa_decode_workspace_bytes.restype = ctypes.c_size_t
        L.mla_gqa_decode_workspace_bytes.argtypes = [Q]
        L.mla_gqa_decode_get_schedule.restype = ctypes.c_int
        L.mla_gqa_decode_get_schedule.argtypes = [Q, vp, vp, vp]
        L.mla_gqa_decode_get_schedule_host.restype = ctypes.c_int
        L.mla_gqa_decode_get_schedule_host.argtypes = [Q, vp, vp]
        L.mla_gqa_decode_fwd.restype = ctypes.c_int
        L.mla_gqa_decode_fwd.argtypes = [Q, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp]
        L.mla_gqa_decode_combine.restype = ctypes.c_int
        L.mla_gqa_decode_combine.argtypes = [Q, vp, vp, vp, vp, vp]
        i32 = ctypes.c_int32
        for name in ("mla_decode_combine_ranks", "mla_decode_combine_ranks_f32"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        A = ctypes.POINTER(mla_absorb_dims)
        for name in ("mla_absorb_q", "mla_absorb_o"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = [A, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def make_dims(batch: int, s_q: int, num_heads: int, num_blocks: int, max_blocks_per_seq: int,
              causal: bool = False, num_sms: int = 0, flags: int = 0) -> mla_decode_dims:
    return mla_decode_dims(int(batch), int(s_q), int(num_heads), int(num_blocks),
                           int(max_blocks_per_seq), PAGE_SIZE, D_QK, D_V, int(bool(causal)),
                           int(num_sms), int(flags), 0)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, where: str) -> None:
    if rc != MLA_OK:
        raise MlaDecodeError(rc, where)


def mla_decode_strerror(code: int) -> str:
    return lib().mla_decode_strerror(int(code)).decode()


def mla_decode_version() -> int:
    return int(lib().mla_decode_version())


def mla_decode_schedule_bytes(dims: mla_decode_dims) -> int:
    return int(lib().mla_decode_schedule_bytes(ctypes.byref(dims)))


def mla_decode_workspace_bytes(dims: mla_decode_dims) -> int:
    return int(lib().mla_decode_workspace_bytes(ctypes.byref(dims)))


def mla_decode_get_schedule(dims, cache_seqlens: torch.Tensor, schedule: torch.Tensor, stream=None) -> None:
    _check(lib().mla_decode_get_schedule(ctypes.byref(dims), _ptr(cache_seqlens), _ptr(schedule),
                                         _stream(stream)), "mla_decode_get_schedule")


def mla_decode_get_schedule_host(dims, cache_seqlens, schedule) -> None:
    """Host version; ``cache_seqlens`` (int32) and ``schedule`` are CPU tensors."""
    _check(lib().mla_decode_get_schedule_host(ctypes.byref(dims), _ptr(cache_seqlens), _ptr(schedule)),
           "mla_decode_get_schedule_host")


def mla_decode_fwd(dims, schedule, workspace, q, kv_cache, block_table, cache_seqlens,
                   softmax_scale: float, out, lse, stream=None) -> None:
    _check(lib().mla_decode_fwd(ctypes.byref(dims), _ptr(schedule), _ptr(workspace), _ptr(q),
                                _ptr(kv_cache), _ptr(block_table), _ptr(cache_seqlens),
                                float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream)),
           "mla_decode_fwd")


def mla_decode_fwd_noalloc(dims, q, kv_cache, block_table, cache_seqlens, softmax_scale: float,
                           out, lse, stream=None) -> None:
    """Schedule + decode + combine without caller-provided schedule or
    workspace: the library uses its own fixed device scratch (see the header).
    For callers that cannot allocate device memory.  Calls that overlap on the
    GPU share that scratch and race; serialise them."""
    _check(lib().mla_decode_fwd_noalloc(ctypes.byref(dims), _ptr(q), _ptr(kv_cache), _ptr(block_table),
                                        _ptr(cache_seqlens), float(softmax_scale), _ptr(out), _ptr(lse),
                                        _stream(stream)), "mla_decode_fwd_noalloc")


def mla_decode_combine(dims, schedule, workspace, out, lse, stream=None) -> None:
    _check(lib().mla_decode_combine(ctypes.byref(dims), _ptr(schedule), _ptr(workspace), _ptr(out),
                                    _ptr(lse), _stream(stream)), "mla_decode_combine")


def mla_decode_get_status(schedule: torch.Tensor) -> int:
    v = ctypes.c_int32(0)
    _check(lib().mla_decode_get_status(_ptr(schedule), ctypes.byref(v)), "mla_decode_get_status")
    return int(v.value)


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


class MlaDecoder:
    """Owns the schedule and workspace buffers for one shape of decode batch.

    ``plan(cache_seqlens)`` builds the split-KV schedule (once per decode step);
    ``__call__`` runs the decode kernel + combine and returns (out, lse).
    With ``fp32_out`` the output is fp32 (MLA_FLAG_FP32_OUT): the result before
    any rounding to bf16.  With ``inline_plan`` (MLA_FLAG_INLINE_PLAN) every
    call builds the plan itself; ``plan()`` is then needed once, to clear the
    status word of the new buffer.
    """

    def __init__(self, batch: int, s_q: int, num_heads: int, num_blocks: int,
                 max_blocks_per_seq: int, causal: bool = False, num_sms: int = 0,
                 device: Optional[torch.device] = None, fp32_out: bool = False, inline_plan: bool = False):
        self.device = torch.device(device or "cuda")
        if num_sms == 0:
            num_sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.dims = make_dims(batch, s_q, num_heads, num_blocks, max_blocks_per_seq, causal, num_sms,
                              (MLA_FLAG_FP32_OUT if fp32_out else 0) | (MLA_FLAG_INLINE_PLAN if inline_plan else 0))
        sb = mla_decode_schedule_bytes(self.dims)
        wb = mla_decode_workspace_bytes(self.dims)
        if sb == 0 or wb == 0:
            raise MlaDecodeError(MLA_ERR_INVALID_ARG, "MlaDecoder dims")
        self.schedule = torch.empty(sb, dtype=torch.uint8, device=self.device)
        self.workspace = torch.empty(wb, dtype=torch.uint8, device=self.device)
        self.out = torch.empty(batch, s_q, num_heads, D_V, dtype=torch.float32 if fp32_out else torch.bfloat16,
                               device=self.device)
        self.lse = torch.empty(batch, num_heads, s_q, dtype=torch.float32, device=self.device)

    def check_inputs(self, q, kv_cache, block_table, cache_seqlens) -> None:
        d = self.dims
        _require(q.dtype == torch.bfloat16 and q.is_contiguous() and
                 tuple(q.shape) == (d.batch, d.s_q, d.num_heads, D_QK), "q must be bf16 [B, s_q, h, 576]")
        _require(kv_cache.dtype == torch.bfloat16 and kv_cache.is_contiguous() and
                 kv_cache.shape[0] == d.num_blocks and kv_cache.shape[1] == PAGE_SIZE and
                 kv_cache.shape[-1] == D_QK and kv_cache.numel() == d.num_blocks * PAGE_SIZE * D_QK,
                 "kv_cache must be bf16 [num_blocks, 64, 1, 576]")
        _require(block_table.dtype == torch.int32 and block_table.is_contiguous() and
                 tuple(block_table.shape) == (d.batch, d.max_blocks_per_seq),
                 "block_table must be int32 [B, max_blocks_per_seq]")
        _require(cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous() and
                 tuple(cache_seqlens.shape) == (d.batch,), "cache_seqlens must be int32 [B]")
        for t in (q, kv_cache, block_table, cache_seqlens):
            _require(t.device == self.out.device, "all tensors must be on %s" % self.out.device)

    def plan(self, cache_seqlens: torch.Tensor, stream=None) -> None:
        mla_decode_get_schedule(self.dims, cache_seqlens, self.schedule, stream)

    def __call__(self, q, kv_cache, block_table, cache_seqlens, softmax_scale: float,
                 stream=None, check: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
        if check:
            self.check_inputs(q, kv_cache, block_table, cache_seqlens)
        mla_decode_fwd(self.dims, self.schedule, self.workspace, q, kv_cache, block_table,
                       cache_seqlens, softmax_scale, self.out, self.lse, stream)
        return self.out, self.lse

    def status(self) -> int:
        return mla_decode_get_status(self.schedule)


def mla_decode(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
               cache_seqlens: torch.Tensor, softmax_scale: float, causal: bool = False,
               num_sms: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """One-shot convenience: plan + decode on the current stream; returns (out, lse)."""
    B, s_q, h, _ = q.shape
    dec = MlaDecoder(B, s_q, h, kv_cache.shape[0], block_table.shape[1], causal, num_sms, q.device)
    dec.plan(cache_seqlens)
    out, lse = dec(q, kv_cache, block_table, cache_seqlens, softmax_scale)
    return out.clone(), lse.clone()


# ---------------------------------------------------------------- GQA path
def make_gqa_dims(batch: int, s_q: int, num_kv_groups: int, num_blocks: int, max_blocks_per_seq: int,
                  causal: bool = False, num_sms: int = 0, flags: int = 0,
                  num_q_heads: Optional[int] = None) -> mla_gqa_dims:
    h = GQA_HEADS_PER_GROUP * num_kv_groups if num_q_heads is None else num_q_heads
    return mla_gqa_dims(int(batch), int(s_q), int(h), int(num_kv_groups), int(num_blocks),
                        int(max_blocks_per_seq), PAGE_SIZE, GQA_D_HEAD, GQA_D_ROPE, int(bool(causal)),
                        int(num_sms), int(flags))


def mla_gqa_decode_schedule_bytes(dims: mla_gqa_dims) -> int:
    return int(lib().mla_gqa_decode_schedule_bytes(ctypes.byref(dims)))


def mla_gqa_decode_workspace_bytes(dims: mla_gqa_dims) -> int:
    return int(lib().mla_gqa_decode_workspace_bytes(ctypes.byref(dims)))


def mla_gqa_decode_get_schedule(dims, cache_seqlens, schedule, stream=None) -> None:
    _check(lib().mla_gqa_decode_get_schedule(ctypes.byref(dims), _ptr(cache_seqlens), _ptr(schedule),
                                             _stream(stream)), "mla_gqa_decode_get_schedule")


def mla_gqa_decode_get_schedule_host(dims, cache_seqlens, schedule) -> None:
    """Host version; ``cache_seqlens`` (int32) and ``schedule`` are CPU tensors."""
    _check(lib().mla_gqa_decode_get_schedule_host(ctypes.byref(dims), _ptr(cache_seqlens), _ptr(schedule)),
           "mla_gqa_decode_get_schedule_host")


def mla_gqa_decode_fwd(dims, schedule, workspace, q, kv_cache, block_table, cache_seqlens,
                       softmax_scale: float, out, lse, stream=None) -> None:
    _check(lib().mla_gqa_decode_fwd(ctypes.byref(dims), _ptr(schedule), _ptr(workspace), _ptr(q),
                                    _ptr(kv_cache), _ptr(block_table), _ptr(cache_seqlens),
                                    float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream)),
           "mla_gqa_decode_fwd")


def mla_gqa_decode_combine(dims, schedule, workspace, out, lse, stream=None) -> None:
    _check(lib().mla_gqa_decode_combine(ctypes.byref(dims), _ptr(schedule), _ptr(workspace), _ptr(out),
                                        _ptr(lse), _stream(stream)), "mla_gqa_decode_combine")


class GqaDecoder:
    """Schedule and workspace buffers for one shape of GQA-path decode batch
    (group-expanded cache, 16 query heads per KV group); same use as
    MlaDecoder."""

    def __init__(self, batch: int, s_q: int, num_kv_groups: int, num_blocks: int, max_blocks_per_seq: int,
                 causal: bool = False, num_sms: int = 0, device: Optional[torch.device] = None,
                 fp32_out: bool = False, inline_plan: bool = False):
        self.device = torch.device(device or "cuda")
        if num_sms == 0:
            num_sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.dims = make_gqa_dims(batch, s_q, num_kv_groups, num_blocks, max_blocks_per_seq, causal, num_sms,
                                  (MLA_FLAG_FP32_OUT if fp32_out else 0) | (MLA_FLAG_INLINE_PLAN if inline_plan else 0))
        sb = mla_gqa_decode_schedule_bytes(self.dims)
        wb = mla_gqa_decode_workspace_bytes(self.dims)
        if sb == 0 or wb == 0:
            raise MlaDecodeError(MLA_ERR_INVALID_ARG, "GqaDecoder dims")
        h = self.dims.num_q_heads
        self.row_width = 2 * num_kv_groups * GQA_D_HEAD + GQA_D_ROPE
        self.schedule = torch.empty(sb, dtype=torch.uint8, device=self.device)
        self.workspace = torch.empty(wb, dtype=torch.uint8, device=self.device)
        self.out = torch.empty(batch, s_q, h, GQA_D_HEAD, dtype=torch.float32 if fp32_out else torch.bfloat16,
                               device=self.device)
        self.lse = torch.empty(batch, h, s_q, dtype=torch.float32, device=self.device)

    def check_inputs(self, q, kv_cache, block_table, cache_seqlens) -> None:
        d = self.dims
        _require(q.dtype == torch.bfloat16 and q.is_contiguous() and
                 tuple(q.shape) == (d.batch, d.s_q, d.num_q_heads, GQA_D_HEAD + GQA_D_ROPE),
                 "q must be bf16 [B, s_q, 16*g, 192]")
        _require(kv_cache.dtype == torch.bfloat16 and kv_cache.is_contiguous() and
                 kv_cache.shape[0] == d.num_blocks and kv_cache.shape[1] == PAGE_SIZE and
                 kv_cache.shape[-1] == self.row_width and
                 kv_cache.numel() == d.num_blocks * PAGE_SIZE * self.row_width,
                 "kv_cache must be bf16 [num_blocks, 64, 1, 2*g*128 + 64]")
        _require(block_table.dtype == torch.int32 and block_table.is_contiguous() and
                 tuple(block_table.shape) == (d.batch, d.max_blocks_per_seq),
                 "block_table must be int32 [B, max_blocks_per_seq]")
        _require(cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous() and
                 tuple(cache_seqlens.shape) == (d.batch,), "cache_seqlens must be int32 [B]")
        for t in (q, kv_cache, block_table, cache_seqlens):
            _require(t.device == self.out.device, "all tensors must be on %s" % self.out.device)

    def plan(self, cache_seqlens: torch.Tensor, stream=None) -> None:
        mla_gqa_decode_get_schedule(self.dims, cache_seqlens, self.schedule, stream)

    def __call__(self, q, kv_cache, block_table, cache_seqlens, softmax_scale: float,
                 stream=None, check: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
        if check:
            self.check_inputs(q, kv_cache, block_table, cache_seqlens)
        mla_gqa_decode_fwd(self.dims, self.schedule, self.workspace, q, kv_cache, block_table,
                           cache_seqlens, softmax_scale, self.out, self.lse, stream)
        return self.out, self.lse

    def status(self) -> int:
        return mla_decode_get_status(self.schedule)


# ---------------------------------------------------------------- absorbed projections
def make_absorb_dims(tokens: int, num_heads: int) -> mla_absorb_dims:
    return mla_absorb_dims(int(tokens), int(num_heads), ABSORB_D_NOPE, ABSORB_D_ROPE, ABSORB_D_LATENT,
                           ABSORB_D_V_HEAD)


def mla_absorb_q(dims: mla_absorb_dims, q_in, w_uk, q_out, status=None, stream=None) -> None:
    _check(lib().mla_absorb_q(ctypes.byref(dims), _ptr(q_in), _ptr(w_uk), _ptr(q_out), _ptr(status),
                              _stream(stream)), "mla_absorb_q")


def mla_absorb_o(dims: mla_absorb_dims, o, w_uv, out, status=None, stream=None) -> None:
    _check(lib().mla_absorb_o(ctypes.byref(dims), _ptr(o), _ptr(w_uv), _ptr(out), _ptr(status),
                              _stream(stream)), "mla_absorb_o")


def _bf16_on(t, shape, what, device):
    _require(t.dtype == torch.bfloat16 and t.is_contiguous() and tuple(t.shape) == tuple(shape),
             "%s must be contiguous bf16 %s" % (what, list(shape)))
    _require(t.device == device, "%s must be on %s" % (what, device))


def absorb_q(q_in: torch.Tensor, w_uk: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """q_in [..., h, 192] (each head's 128-wide part, then its RoPE part) and
    w_uk [h, 128, 512] -> [..., h, 576]: the latent query q_nope . W_UK with the
    RoPE part after it, the layout mla_decode takes as q."""
    h = q_in.shape[-2]
    T = q_in.numel() // (h * (ABSORB_D_NOPE + ABSORB_D_ROPE)) if q_in.numel() else 0
    _require(T >= 1 and q_in.shape[-1] == ABSORB_D_NOPE + ABSORB_D_ROPE, "q_in must be [..., h, 192]")
    _bf16_on(q_in, q_in.shape, "q_in", q_in.device)
    _bf16_on(w_uk, (h, ABSORB_D_NOPE, ABSORB_D_LATENT), "w_uk", q_in.device)
    shape = tuple(q_in.shape[:-1]) + (ABSORB_D_LATENT + ABSORB_D_ROPE,)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=q_in.device)
    _bf16_on(out, shape, "out", q_in.device)
    mla_absorb_q(make_absorb_dims(T, h), q_in, w_uk, out, None, stream)
    return out


def absorb_o(o: torch.Tensor, w_uv: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """o [..., h, 512] (the decode's output over latent rows) and w_uv
    [h, 512, 128] -> [..., h, 128] = O . W_UV per head."""
    h = o.shape[-2]
    T = o.numel() // (h * ABSORB_D_LATENT) if o.numel() else 0
    _require(T >= 1 and o.shape[-1] == ABSORB_D_LATENT, "o must be [..., h, 512]")
    _bf16_on(o, o.shape, "o", o.device)
    _bf16_on(w_uv, (h, ABSORB_D_LATENT, ABSORB_D_V_HEAD), "w_uv", o.device)
    shape = tuple(o.shape[:-1]) + (ABSORB_D_V_HEAD,)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=o.device)
    _bf16_on(out, shape, "out", o.device)
    mla_absorb_o(make_absorb_dims(T, h), o, w_uv, out, None, stream)
    return out


# ---------------------------------------------------------------- split-KV across ranks
def mla_decode_combine_ranks(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: torch.Tensor,
                             lse: torch.Tensor, stream=None) -> None:
    """o_parts bf16 or fp32 [R, B, s_q, h, d_v], lse_parts fp32 [R, B, h, s_q]
    -> out bf16 [B, s_q, h, d_v], lse fp32 [B, h, s_q]: the LSE-weighted merge
    of the ranks' results (d_v 512 or 128); fp32 parts are rounded once, after
    the merge."""
    _require(o_parts.dim() == 5 and o_parts.dtype in (torch.bfloat16, torch.float32) and o_parts.is_contiguous(),
             "o_parts must be contiguous bf16 or fp32 [R, B, s_q, h, d_v]")
    R, B, s_q, h, d_v = o_parts.shape
    _require(lse_parts.dtype == torch.float32 and lse_parts.is_contiguous() and
             tuple(lse_parts.shape) == (R, B, h, s_q), "lse_parts must be contiguous fp32 [R, B, h, s_q]")
    _require(out.dtype == torch.bfloat16 and out.is_contiguous() and tuple(out.shape) == (B, s_q, h, d_v),
             "out must be contiguous bf16 [B, s_q, h, d_v]")
    _require(lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, h, s_q),
             "lse must be contiguous fp32 [B, h, s_q]")
    for t in (lse_parts, out, lse):
        _require(t.device == o_parts.device, "all tensors must be on %s" % o_parts.device)
    fn = lib().mla_decode_combine_ranks_f32 if o_parts.dtype == torch.float32 else lib().mla_decode_combine_ranks
    _check(fn(int(R), int(B), int(s_q), int(h), int(d_v), _ptr(o_parts), _ptr(lse_parts), _ptr(out), _ptr(lse),
              _stream(stream)), "mla_decode_combine_ranks")


def absorbed_mla_decode(q_in: torch.Tensor, w_uk: torch.Tensor, w_uv: torch.Tensor, kv_cache: torch.Tensor,
                        block_table: torch.Tensor, cache_seqlens: torch.Tensor, softmax_scale: float,
                        decoder: "MlaDecoder", stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One absorbed-MLA decode step for one layer: q_in [B, s_q, h, 192]
    (each head's 128-wide part, then its RoPE part) -> the latent query
    (mla_absorb_q), attention over the latent cache (mla_decode_fwd with
    ``decoder``'s plan, already built by ``decoder.plan``), then the output
    projection (mla_absorb_o).  Returns (out [B, s_q, h, 128] bf16, lse
    [B, h, s_q] fp32: the attention's log-sum-exp)."""
    q_lat = absorb_q(q_in, w_uk, stream=stream)
    o_lat, lse = decoder(q_lat, kv_cache, block_table, cache_seqlens, softmax_scale, stream)
    return absorb_o(o_lat, w_uv, stream=stream), lse
