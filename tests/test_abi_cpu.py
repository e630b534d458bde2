"""The C ABI library loads and exports what include/fva.h declares; host-side checks
(no device work is enqueued by any call here)."""
import ctypes
import os
import re

import pytest

from adaptive_block_sparse_hilbert_b200 import fva

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fva.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FVA_API\s+[\w\s\*]*?\b(fva_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 16
    lib = ctypes.CDLL(fva.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(fva.EXPORTED)


def test_no_internal_symbols_exported():
    out = os.popen(f"nm -D --defined-only {fva.LIB_PATH}").read()
    syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert syms, out
    assert all(s.startswith("fva_") or s.startswith("_init") or s.startswith("_fini") for s in syms), syms


def test_status_strings():
    assert fva.status_string(0) == "ok"
    assert "capacity" in fva.status_string(fva.FVA_ERR_CAPACITY)
    assert fva.status_string(-99) == "unknown status"


@pytest.mark.parametrize("wid", [0, 1, 2, 3])
def test_derived_sizes(wid):
    from adaptive_block_sparse_hilbert_b200 import synth
    wl = synth.WORKLOADS[wid]
    s = fva.make_shape(wl.B, wl.H, wl.d, wl.T, wl.Hg, wl.Wg, wl.dtype)
    N = wl.T * wl.Hg * wl.Wg
    nB = (N + 63) // 64
    assert fva.fva_num_tokens(s) == N
    assert fva.fva_num_blocks(s) == nB
    assert fva.fva_num_tiles(s) == wl.H * ((nB + 1) // 2)
    assert fva.fva_mask_capacity(s) == wl.H * nB * nB
    assert fva.fva_tile_capacity(s) == wl.H * ((nB + 1) // 2) * nB
    ws0 = fva.fva_route_workspace_bytes(s, False)
    ws1 = fva.fva_route_workspace_bytes(s, True)
    assert ws0 >= wl.H * nB * nB * 8 and ws1 >= ws0 + 2 * wl.H * nB * wl.d * 8
    assert 0 < fva.fva_tiles_workspace_bytes(s) < ws0


def test_invalid_shapes_rejected():
    bad = [
        fva.make_shape(1, 2, 64, 0, 16, 16),       # T = 0
        fva.make_shape(1, 2, 60, 4, 16, 16),       # d*2 not a multiple of 16
        fva.fva_shape(1, 2, 64, 4, 16, 16, 32, fva.FVA_BF16),  # block != 64
        fva.fva_shape(1, 2, 64, 4, 16, 16, 64, 7),  # bad dtype
    ]
    for s in bad:
        assert fva.fva_num_tokens(s) == -1
        assert fva.fva_route_workspace_bytes(s) == 0


def test_routing_limit_on_block_count():
    """Routing keeps two rows' float64 working sets in one CTA's shared memory, which
    bounds nB at 11326; one block more is rejected on the host before any launch."""
    P = ctypes.c_void_p
    one = P(16)  # non-null dummy pointer; every call below fails validation first
    ok = fva.make_shape(1, 1, 64, 1, 837, 866)        # N = 724,842: nB = 11326
    over = fva.make_shape(1, 1, 64, 1, 840, 863)      # N = 724,920: nB = 11327
    assert fva.fva_num_blocks(ok) == 11326 and fva.fva_num_blocks(over) == 11327
    assert fva.fva_route_workspace_bytes(ok, 0) > 0 and fva.fva_route_workspace_bytes(ok, 1) > 0
    assert fva.fva_sasa_workspace_bytes(ok) > 0
    assert fva.fva_route_workspace_bytes(over, 0) == 0 and fva.fva_route_workspace_bytes(over, 1) == 0
    assert fva.fva_sasa_workspace_bytes(over) == 0
    small = fva.fva_mask(16, 16, 10, 16, 16, 16, 10, 16, 16)
    args = (one, one, None, None, 0.9, 4, 2, ctypes.byref(small), one, 1 << 30, None, None)
    assert fva.call_raw("fva_route", ctypes.byref(over), *args) == fva.FVA_ERR_UNSUPPORTED_SHAPE
    # the limit shape passes the shape checks and stops at the (too small) mask capacity
    assert fva.call_raw("fva_route", ctypes.byref(ok), *args) == fva.FVA_ERR_CAPACITY
    assert fva.call_raw("fva_route_noalloc", ctypes.byref(over), one, one, None, None, 0.9, 4, 2,
                        ctypes.byref(small), None, None) == fva.FVA_ERR_UNSUPPORTED_SHAPE
    # tile building from a caller-made mask has no such limit
    assert fva.fva_tiles_workspace_bytes(over) > 0


def test_host_validation_before_any_launch():
    s = fva.make_shape(1, 2, 64, 4, 16, 16, "f32")
    P = ctypes.c_void_p
    one = P(16)  # a non-null dummy pointer; validation fails before it is ever used
    rc = fva.call_raw("fva_reorder", ctypes.byref(s), None, one, None, one, 0, None)
    assert rc == fva.FVA_ERR_INVALID_ARG
    rc = fva.call_raw("fva_reorder", ctypes.byref(s), one, one, None, one, 5, None)
    assert rc == fva.FVA_ERR_INVALID_ARG
    rc = fva.call_raw("fva_reorder", ctypes.byref(s), one, P(48), P(64), one, fva.FVA_INV, None)
    assert rc == fva.FVA_ERR_INVALID_ARG  # INV takes no pooled output
    rc = fva.call_raw("fva_reorder", ctypes.byref(s), P(17), P(48), None, one, 0, None)
    assert rc == fva.FVA_ERR_ALIGNMENT
    m = fva.fva_mask(16, 16, 10, 16, 16, 16, 10, 16, 16)
    # p out of range, negative floor, bad order, too-small capacity, too-small workspace
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 0.0, 2, 2, ctypes.byref(m), one, 1 << 30,
                        None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 1.5, 2, 2, ctypes.byref(m), one, 1 << 30,
                        None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, float("nan"), 2, 2, ctypes.byref(m), one,
                        1 << 30, None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 0.9, -1, 2, ctypes.byref(m), one, 1 << 30,
                        None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 0.9, 2, 9, ctypes.byref(m), one, 1 << 30,
                        None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 0.9, 2, 2, ctypes.byref(m), one, 1 << 30,
                        None, None) == fva.FVA_ERR_CAPACITY
    big = fva.fva_mask(16, 16, 1 << 20, 16, 16, 16, 1 << 20, 16, 16)
    assert fva.call_raw("fva_route", ctypes.byref(s), one, one, None, None, 0.9, 2, 2, ctypes.byref(big), one, 64,
                        None, None) == fva.FVA_ERR_WORKSPACE
    # bf16 attention supports d in {64, 128} only
    s96 = fva.make_shape(1, 2, 96, 4, 16, 16, "bf16")
    assert fva.call_raw("fva_dense_attn", ctypes.byref(s96), one, one, one, fva.FVA_F16, P(4096), ctypes.c_float(0.0),
                        None, None) == fva.FVA_ERR_UNSUPPORTED_SHAPE
    assert fva.call_raw("fva_sparse_attn", ctypes.byref(s), one, one, one, fva.FVA_F32, None, P(4096),
                        ctypes.c_float(0.0), None, None) == fva.FVA_ERR_INVALID_ARG
    # v_dtype must match: fp32 layers take fp32 V; bf16 layers take bf16 or fp16 V
    assert fva.call_raw("fva_dense_attn", ctypes.byref(s), one, one, one, fva.FVA_F16, P(4096), ctypes.c_float(0.0),
                        None, None) == fva.FVA_ERR_INVALID_ARG
    sb = fva.make_shape(1, 2, 64, 4, 16, 16, "bf16")
    assert fva.call_raw("fva_dense_attn", ctypes.byref(sb), one, one, one, fva.FVA_F32, P(4096), ctypes.c_float(0.0),
                        None, None) == fva.FVA_ERR_INVALID_ARG
    # fp16 conversion is a forward reorder of bf16 data only
    assert fva.call_raw("fva_reorder", ctypes.byref(s), one, P(48), None, one, fva.FVA_FWD_F16, None) == \
        fva.FVA_ERR_INVALID_ARG


def test_cta_trace_argument_checks():
    # host-side checks only; the pointers below are never dereferenced, and tracing is
    # switched off again before the test ends
    L = fva.lib()
    try:
        assert L.fva_set_cta_trace(None, 5) == fva.FVA_ERR_INVALID_ARG
        assert L.fva_set_cta_trace(1024, 0) == fva.FVA_ERR_INVALID_ARG
        assert L.fva_set_cta_trace(1024, -1) == fva.FVA_ERR_INVALID_ARG
        assert L.fva_set_cta_trace(1028, 4) == fva.FVA_ERR_ALIGNMENT
        assert L.fva_set_cta_trace(1024, 4) == fva.FVA_OK
    finally:
        assert L.fva_set_cta_trace(None, 0) == fva.FVA_OK


def test_curve_perm_rejects_unknown_curve():
    s = fva.make_shape(1, 1, 64, 2, 8, 8, "bf16")
    assert fva.lib().fva_curve_perm(ctypes.byref(s), 7, 1024, 2048, None, None) == fva.FVA_ERR_INVALID_ARG
    assert fva.lib().fva_curve_perm(ctypes.byref(s), fva.FVA_CURVE_RECT, None, 2048, None, None) == fva.FVA_ERR_INVALID_ARG


def test_copy_strided_argument_checks():
    L = fva.lib()
    assert L.fva_copy_strided(None, 16, 1024, 16, 16, 1, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_copy_strided(1024, 8, 2048, 16, 16, 1, None) == fva.FVA_ERR_INVALID_ARG   # width > dst pitch
    assert L.fva_copy_strided(1024, 16, 2048, 8, 16, 1, None) == fva.FVA_ERR_INVALID_ARG   # width > src pitch
    assert L.fva_copy_strided(1024, 16, 2048, 16, 16, -1, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_copy_strided(1024, 16, 2048, 16, 16, 0, None) == fva.FVA_OK               # nothing to move


def test_sparse_attn_range_host_checks():
    """fva_sparse_attn_range turns away slot ranges outside the work list, and fp32 inputs,
    before anything is enqueued (the pointers here are never dereferenced)."""
    s = fva.make_shape(1, 2, 128, 2, 16, 16, "bf16")    # nB = 8, 4 tiles per head, 8 tiles
    assert fva.fva_num_tiles(s) == 8
    m = fva.fva_mask(16, 16, 10, 16, 16, 16, 10, 16, 16)
    p = ctypes.c_void_p(256)
    o = ctypes.c_void_p(512)

    def rng(first, n, shape=s, vd=fva.FVA_F16):
        return fva.call_raw("fva_sparse_attn_range", ctypes.byref(shape), p, p, p, vd, ctypes.byref(m), o,
                            ctypes.c_float(0.0), first, n, None, None)
    assert rng(-1, 2) == fva.FVA_ERR_INVALID_ARG
    assert rng(0, -1) == fva.FVA_ERR_INVALID_ARG
    assert rng(5, 4) == fva.FVA_ERR_INVALID_ARG       # past the 8 tiles
    assert rng(9, 0) == fva.FVA_ERR_INVALID_ARG
    f32 = fva.make_shape(1, 2, 64, 2, 16, 16, "f32")
    assert rng(0, 2, f32, fva.FVA_F32) == fva.FVA_ERR_UNSUPPORTED_SHAPE
    assert fva.call_raw("fva_sparse_attn_range", ctypes.byref(s), p, p, p, fva.FVA_F16, ctypes.byref(m), p,
                        ctypes.c_float(0.0), 0, 1, None, None) == fva.FVA_ERR_INVALID_ARG  # o aliases q
