"""C-ABI surface checks that need no GPU: the library loads, exports every
function the header declares, and rejects bad arguments before it touches
the device."""
import ctypes
import math
import subprocess

import pytest

import helpers
from mla_decode_attention_15_b200 import _build, binding as bd


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return bd.lib()


def test_header_declares_the_boundary():
    names = helpers.header_functions()
    for required in ("mla_decode_get_schedule", "mla_decode_fwd", "mla_decode_combine",
                     "mla_decode_schedule_bytes", "mla_decode_workspace_bytes",
                     "mla_decode_get_status", "mla_decode_strerror"):
        assert required in names, names


def test_library_exports_every_header_symbol(lib):
    names = helpers.header_functions()
    dyn = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], capture_output=True, text=True).stdout
    for n in names:
        assert hasattr(lib, n), n
        assert (" T " + n) in dyn, n
    assert set(bd.EXPORTED) == set(names)


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", _build.LIB], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout
    assert "sm_90" not in out.stdout and "sm_80" not in out.stdout


def test_version_and_strerror(lib):
    assert bd.mla_decode_version() == 6
    for code in (0, -1, -2, -3, -4):
        assert bd.mla_decode_strerror(code)
    assert "unknown" in bd.mla_decode_strerror(-99)


def _dims(**kw):
    base = dict(batch=16, s_q=1, num_heads=16, num_blocks=100, max_blocks_per_seq=10,
                causal=False, num_sms=148)
    base.update(kw)
    return bd.make_dims(**base)


def test_sizes_need_valid_dims(lib):
    d = _dims()
    assert bd.mla_decode_schedule_bytes(d) == 4 * (16 + 8 * 148 + 3 * 16 + 1)
    assert bd.mla_decode_workspace_bytes(d) == 2 * 148 * 16 * (512 + 1) * 4
    d32 = _dims(s_q=2)
    assert bd.mla_decode_workspace_bytes(d32) == 2 * 148 * 32 * 513 * 4
    # 256 columns -> 2 groups of 128 on CTA pairs: 74 clusters, 37 ranges each
    # walked by both groups; the plan has one row per request
    wide = _dims(s_q=2, num_heads=128, batch=32)
    assert bd.mla_decode_schedule_bytes(wide) == 4 * (16 + 8 * 37 + 3 * 32 + 1)
    assert bd.mla_decode_workspace_bytes(wide) == (2 * 37 * 2) * 128 * 513 * 4
    mid = _dims(s_q=2, num_heads=24)  # 48 columns -> one group of 64, one-CTA kernel
    assert bd.mla_decode_workspace_bytes(mid) == 2 * 148 * 64 * 513 * 4
    for bad in (dict(batch=0), dict(s_q=0), dict(s_q=3), dict(num_heads=0), dict(num_blocks=0),
                dict(max_blocks_per_seq=0), dict(num_sms=-1)):
        assert bd.mla_decode_schedule_bytes(_dims(**bad)) == 0, bad
        assert bd.mla_decode_workspace_bytes(_dims(**bad)) == 0, bad


def _rc_fwd(lib, d, ptrs=None, scale=0.07):
    p = dict(sched=0x10000, ws=0x20000, q=0x30000, kv=0x40000, bt=0x50000, sl=0x60000,
             out=0x70000, lse=0x80000)
    if ptrs:
        p.update(ptrs)
    return lib.mla_decode_fwd(ctypes.byref(d), p["sched"], p["ws"], p["q"], p["kv"], p["bt"], p["sl"],
                              ctypes.c_float(scale), p["out"], p["lse"], None)


def test_fwd_rejects_bad_dims_before_any_launch(lib):
    cases = [
        (dict(page_size=32), bd.MLA_ERR_UNSUPPORTED),
        (dict(d_qk=512), bd.MLA_ERR_UNSUPPORTED),
        (dict(d_v=576), bd.MLA_ERR_UNSUPPORTED),
        (dict(num_heads=129, s_q=2), bd.MLA_ERR_UNSUPPORTED),
        (dict(s_q=3), bd.MLA_ERR_UNSUPPORTED),
        (dict(s_q=4, num_heads=2), bd.MLA_ERR_UNSUPPORTED),
        (dict(batch=0), bd.MLA_ERR_INVALID_ARG),
        (dict(causal=2), bd.MLA_ERR_INVALID_ARG),
        (dict(reserved=1), bd.MLA_ERR_INVALID_ARG),
        (dict(flags=0x100), bd.MLA_ERR_INVALID_ARG),
    ]
    for change, code in cases:
        d = _dims()
        for k, v in change.items():
            setattr(d, k, v)
        assert _rc_fwd(lib, d) == code, change
    assert lib.mla_decode_fwd(None, 0, 0, 0, 0, 0, 0, ctypes.c_float(1.0), 0, 0, None) == bd.MLA_ERR_INVALID_ARG


def test_fwd_rejects_null_or_misaligned_pointers(lib):
    d = _dims()
    for name in ("sched", "ws", "q", "kv", "bt", "sl", "out", "lse"):
        assert _rc_fwd(lib, d, {name: None}) == bd.MLA_ERR_INVALID_ARG, name
        assert _rc_fwd(lib, d, {name: 0x30008}) == bd.MLA_ERR_INVALID_ARG, name
    assert _rc_fwd(lib, d, scale=math.nan) == bd.MLA_ERR_INVALID_ARG
    assert _rc_fwd(lib, d, scale=math.inf) == bd.MLA_ERR_INVALID_ARG


def test_other_entry_points_reject_bad_arguments(lib):
    d = _dims()
    assert lib.mla_decode_get_schedule(ctypes.byref(d), None, 0x1000, None) == bd.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_get_schedule(ctypes.byref(d), 0x1004, 0x1000, None) == bd.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_combine(ctypes.byref(d), 0x1000, None, 0x2000, 0x3000, None) == bd.MLA_ERR_INVALID_ARG
    st = ctypes.c_int32(0)
    assert lib.mla_decode_get_status(None, ctypes.byref(st)) == bd.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_get_status(0x1000, None) == bd.MLA_ERR_INVALID_ARG
    bad = _dims()
    bad.page_size = 128
    assert lib.mla_decode_combine(ctypes.byref(bad), 0x1000, 0x2000, 0x3000, 0x4000, None) == bd.MLA_ERR_UNSUPPORTED
    host0 = _dims(num_sms=0)
    assert lib.mla_decode_get_schedule_host(ctypes.byref(host0), 0x1000, 0x2000) == bd.MLA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(bd, "_lib", None)
    monkeypatch.setattr(_build, "LIB", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        bd.lib()


def test_build_entry_point_compiles_and_imports():
    """The build check: __graft_entry__.build() compiles (or finds up to date)
    the library and the oracle and imports the package at the ABI version it
    expects."""
    import __graft_entry__
    __graft_entry__.build()
