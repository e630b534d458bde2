"""Thin ctypes binding of libfva (argument marshalling only).

Every function here forwards to the C entry point of the same name in libfva.so; all
compute runs in the library's sm_100a kernels. Tensors are torch CUDA tensors (device
memory and streams are the only things PyTorch provides). Importing this module loads
libfva.so and raises if it is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfva.so")

FVA_OK = 0
FVA_ERR_INVALID_ARG = -1
FVA_ERR_UNSUPPORTED_SHAPE = -2
FVA_ERR_CAPACITY = -3
FVA_ERR_CUDA = -4
FVA_ERR_DEVICE_TIMEOUT = -5
FVA_ERR_WORKSPACE = -6
FVA_ERR_ALIGNMENT = -7
FVA_ERR_TOO_LARGE = -8
ROUTE_NOALLOC_SCRATCH_BYTES = 64 << 20

FVA_DEVERR_NONE = 0
FVA_DEVERR_TIMEOUT = 1
FVA_DEVERR_MASK = 2
FVA_DEVERR_BAD_LIST = 3

FVA_F32 = 0
FVA_BF16 = 1
FVA_F16 = 2
FVA_FWD = 0
FVA_INV = 1
FVA_FWD_F16 = 2
FVA_ORDER_NATURAL = 0
FVA_ORDER_LPT = 1
FVA_ORDER_HEAD_LPT = 2

BLOCK = 64


class fva_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("T", ctypes.c_int32), ("Hg", ctypes.c_int32), ("Wg", ctypes.c_int32),
                ("block", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class fva_mask(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("head_kept", ctypes.c_void_p), ("tile_ptr", ctypes.c_void_p), ("tile_col", ctypes.c_void_p),
                ("tile_capacity", ctypes.c_int64), ("tile_cost", ctypes.c_void_p), ("worklist", ctypes.c_void_p),
                ("logits", ctypes.c_void_p)]


class fva_rlb_move(ctypes.Structure):
    _fields_ = [("head", ctypes.c_int32), ("from_rank", ctypes.c_int32), ("to_rank", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("gain_ms", ctypes.c_double)]


class FvaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libfva.so not built at {LIB_PATH}; run python -m adaptive_block_sparse_hilbert_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    S = ctypes.POINTER(fva_shape)
    M = ctypes.POINTER(fva_mask)
    i32, i64, sz, dbl, flt = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_double, ctypes.c_float
    sig = {
        "fva_status_string": (ctypes.c_char_p, [i32]),
        "fva_version": (i32, []),
        "fva_set_diagnostics": (None, [ctypes.c_uint64, i32]),
        "fva_set_cta_trace": (i32, [P, i64]),
        "fva_rlb_plan": (i32, [ctypes.POINTER(ctypes.c_double), i32, i32, dbl, dbl, dbl, i32,
                               ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(fva_rlb_move), i32,
                               ctypes.POINTER(ctypes.c_int)]),
        "fva_num_tokens": (i64, [S]),
        "fva_num_blocks": (i64, [S]),
        "fva_num_tiles": (i64, [S]),
        "fva_mask_capacity": (i64, [S]),
        "fva_tile_capacity": (i64, [S]),
        "fva_route_workspace_bytes": (sz, [S, i32]),
        "fva_tiles_workspace_bytes": (sz, [S]),
        "fva_hilbert_perm": (i32, [S, P, P, P]),
        "fva_curve_perm": (i32, [S, i32, P, P, P, P]),
        "fva_copy_strided": (i32, [P, sz, P, sz, sz, i64, P]),
        "fva_sasa_budgets": (i32, [ctypes.POINTER(ctypes.c_double), i32, dbl, dbl, dbl, ctypes.POINTER(ctypes.c_int64)]),
        "fva_sasa_workspace_bytes": (sz, [S]),
        "fva_sasa_augment": (i32, [S, P, P, P, i32, P, i32, M, P, sz, P, P, P]),
        "fva_reorder": (i32, [S, P, P, P, P, i32, P]),
        "fva_pool": (i32, [S, P, P, P]),
        "fva_route": (i32, [S, P, P, P, P, dbl, i32, i32, M, P, sz, P, P]),
        "fva_build_tiles": (i32, [S, M, i32, P, sz, P, P]),
        "fva_route_noalloc": (i32, [S, P, P, P, P, dbl, i32, i32, M, P, P]),
        "fva_sparse_attn": (i32, [S, P, P, P, i32, M, P, flt, P, P]),
        "fva_sparse_attn_range": (i32, [S, P, P, P, i32, M, P, flt, i64, i64, P, P]),
        "fva_dense_attn": (i32, [S, P, P, P, i32, P, flt, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()
EXPORTED = (
    "fva_status_string", "fva_version", "fva_set_diagnostics", "fva_num_tokens", "fva_num_blocks", "fva_num_tiles", "fva_mask_capacity",
    "fva_tile_capacity", "fva_route_workspace_bytes", "fva_tiles_workspace_bytes", "fva_hilbert_perm", "fva_reorder",
    "fva_pool", "fva_route", "fva_build_tiles", "fva_sparse_attn", "fva_dense_attn", "fva_route_noalloc",
    "fva_set_cta_trace", "fva_rlb_plan", "fva_curve_perm", "fva_sasa_budgets", "fva_sasa_workspace_bytes",
    "fva_sasa_augment", "fva_copy_strided", "fva_sparse_attn_range",
)


def lib():
    return _lib


FVA_DIAG_WITHHOLD_Q = 1


def fva_set_diagnostics(wait_limit_ns: int = 0, flags: int = 0) -> None:
    """Attention-kernel diagnostics: wait time limit (0 = 2 s default) and flags
    (FVA_DIAG_WITHHOLD_Q: skip the Q load so the waits behind it run out)."""
    _lib.fva_set_diagnostics(int(wait_limit_ns), int(flags))


def fva_set_cta_trace(trace=None) -> None:
    """Per-CTA trace of the bf16 attention kernels: `trace` is an int64 device tensor of
    shape [ctas, 4] (SM id, list length, start ns, end ns per CTA), or None to stop."""
    if trace is None:
        st = _lib.fva_set_cta_trace(None, 0)
    else:
        if trace.dtype != torch.int64 or trace.dim() != 2 or trace.shape[1] != 4 or not trace.is_contiguous():
            raise ValueError("trace must be a contiguous int64 tensor of shape [ctas, 4]")
        st = _lib.fva_set_cta_trace(_ptr(trace), int(trace.shape[0]))
    if st != 0:
        raise FvaError("fva_set_cta_trace", st)


def fva_rlb_plan(head_load_ms, n_ranks: int, comm_ms: float, sched_ms: float, threshold: float = 1.10,
                 max_per_rank: int = 1):
    """Runtime Load Balancing plan (host): returns (rank_of int32[n_heads], moves) with
    moves = [(head, from_rank, to_rank, gain_ms)] in the order they are applied."""
    import numpy as np
    load = np.ascontiguousarray(head_load_ms, dtype=np.float64)
    H = int(load.shape[0])
    cap = max(1, min(H, n_ranks * max_per_rank))
    rank_of = np.zeros(H, dtype=np.int32)
    moves = (fva_rlb_move * cap)()
    n = ctypes.c_int(0)
    st = _lib.fva_rlb_plan(load.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), H, int(n_ranks), float(comm_ms),
                           float(sched_ms), float(threshold), int(max_per_rank),
                           rank_of.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), moves, cap, ctypes.byref(n))
    if st != 0:
        raise FvaError("fva_rlb_plan", st)
    return rank_of, [(m.head, m.from_rank, m.to_rank, m.gain_ms) for m in moves[:n.value]]


def fva_sasa_budgets(rank_load_ms, block_ms: float, n1: float = 0.8, n2: float = 0.07):
    """Blocks each rank may add (host): floor(n1 * slack / block_ms) where slack >= n2 * critical."""
    import numpy as np
    load = np.ascontiguousarray(rank_load_ms, dtype=np.float64)
    out = np.zeros(load.shape[0], dtype=np.int64)
    st = _lib.fva_sasa_budgets(load.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(load.shape[0]),
                               float(block_ms), float(n1), float(n2), out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    if st != 0:
        raise FvaError("fva_sasa_budgets", st)
    return out


def status_string(status: int) -> str:
    return _lib.fva_status_string(int(status)).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, rc):
    if rc != FVA_OK:
        raise FvaError(fn, rc)


# ------------------------------------------------------------------------------ shapes

def make_shape(B, H, d, T, Hg, Wg, dtype="bf16") -> fva_shape:
    dt = {"bf16": FVA_BF16, "f32": FVA_F32, FVA_BF16: FVA_BF16, FVA_F32: FVA_F32}[dtype]
    return fva_shape(B, H, d, T, Hg, Wg, BLOCK, dt)


def fva_num_tokens(s): return _lib.fva_num_tokens(ctypes.byref(s))
def fva_num_blocks(s): return _lib.fva_num_blocks(ctypes.byref(s))
def fva_num_tiles(s): return _lib.fva_num_tiles(ctypes.byref(s))
def fva_mask_capacity(s): return _lib.fva_mask_capacity(ctypes.byref(s))
def fva_tile_capacity(s): return _lib.fva_tile_capacity(ctypes.byref(s))
def fva_route_workspace_bytes(s, need_pool=False): return _lib.fva_route_workspace_bytes(ctypes.byref(s), int(need_pool))
def fva_tiles_workspace_bytes(s): return _lib.fva_tiles_workspace_bytes(ctypes.byref(s))


# ------------------------------------------------------------------------------ masks

@dataclasses.dataclass
class Mask:
    """Device buffers of one block mask (owned by torch; passed to libfva as fva_mask)."""

    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    head_kept: torch.Tensor
    tile_ptr: torch.Tensor
    tile_col: torch.Tensor
    tile_cost: torch.Tensor
    worklist: torch.Tensor
    logits: torch.Tensor | None = None  # optional float64 [B*H, nB, nB]: the exported block logits

    @staticmethod
    def allocate(s: fva_shape, device="cuda", logits: bool = False) -> "Mask":
        B, H = s.B, s.H
        nB = fva_num_blocks(s)
        tiles = fva_num_tiles(s)
        i32 = dict(dtype=torch.int32, device=device)
        return Mask(
            row_ptr=torch.empty(B * H * nB + 1, **i32),
            col_idx=torch.empty(fva_mask_capacity(s), **i32),
            head_kept=torch.empty(B * H, dtype=torch.int64, device=device),
            tile_ptr=torch.empty(tiles + 1, **i32),
            tile_col=torch.empty(fva_tile_capacity(s), **i32),
            tile_cost=torch.empty(tiles, **i32),
            worklist=torch.empty(tiles, **i32),
            logits=torch.empty((B * H, nB, nB), dtype=torch.float64, device=device) if logits else None,
        )

    def c(self) -> fva_mask:
        return fva_mask(self.row_ptr.data_ptr(), self.col_idx.data_ptr(), self.col_idx.numel(),
                        self.head_kept.data_ptr(), self.tile_ptr.data_ptr(), self.tile_col.data_ptr(),
                        self.tile_col.numel(), self.tile_cost.data_ptr(), self.worklist.data_ptr(),
                        None if self.logits is None else self.logits.data_ptr())


# ------------------------------------------------------------------------------ entry points

def fva_hilbert_perm(s, perm, inv, stream=None):
    _check("fva_hilbert_perm", _lib.fva_hilbert_perm(ctypes.byref(s), _ptr(perm), _ptr(inv), _stream(stream)))


FVA_CURVE_HILBERT = 0
FVA_CURVE_RECT = 1


def fva_curve_perm(s, curve, perm, inv, dev_status=None, stream=None):
    _check("fva_curve_perm", _lib.fva_curve_perm(ctypes.byref(s), int(curve), _ptr(perm), _ptr(inv), _ptr(dev_status),
                                                 _stream(stream)))


def fva_reorder(s, x_in, x_out, pooled, perm, direction=FVA_FWD, stream=None):
    _check("fva_reorder", _lib.fva_reorder(ctypes.byref(s), _ptr(x_in), _ptr(x_out), _ptr(pooled), _ptr(perm),
                                           int(direction), _stream(stream)))


def fva_pool(s, x_bhnd, pooled, stream=None):
    _check("fva_pool", _lib.fva_pool(ctypes.byref(s), _ptr(x_bhnd), _ptr(pooled), _stream(stream)))


def fva_route(s, q, k, pooled_q, pooled_k, p, k_floor, mask: Mask, workspace, order=FVA_ORDER_HEAD_LPT,
              dev_status=None, stream=None):
    m = mask.c() if isinstance(mask, Mask) else mask
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("fva_route", _lib.fva_route(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(pooled_q), _ptr(pooled_k), float(p),
                                       int(k_floor), int(order), ctypes.byref(m), _ptr(workspace), ws_bytes,
                                       _ptr(dev_status), _stream(stream)))


def fva_route_noalloc(s, q, k, pooled_q, pooled_k, p, k_floor, mask: Mask, order=FVA_ORDER_HEAD_LPT,
                      dev_status=None, stream=None):
    """fva_route without a workspace, for callers that cannot allocate device memory: the
    scratch is a fixed 64 MiB array inside libfva (see include/fva.h)."""
    m = mask.c() if isinstance(mask, Mask) else mask
    _check("fva_route_noalloc", _lib.fva_route_noalloc(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(pooled_q),
                                                       _ptr(pooled_k), float(p), int(k_floor), int(order),
                                                       ctypes.byref(m), _ptr(dev_status), _stream(stream)))


def fva_copy_strided(dst, dst_pitch_bytes, src, src_pitch_bytes, width_bytes, rows, stream=None):
    """Pitched async copy between device and page-locked host memory (pointers or tensors)."""
    _check("fva_copy_strided", _lib.fva_copy_strided(_ptr(dst), int(dst_pitch_bytes), _ptr(src), int(src_pitch_bytes),
                                                     int(width_bytes), int(rows), _stream(stream)))


def fva_sasa_workspace_bytes(s): return _lib.fva_sasa_workspace_bytes(ctypes.byref(s))


def fva_sasa_augment(s, pooled_q, pooled_k, rank_of_head, budget, mask: Mask, workspace, order=FVA_ORDER_HEAD_LPT,
                     added=None, dev_status=None, stream=None):
    """Slack-aware augmentation of a routed mask in place (rank_of_head int32 [B*H] and
    budget int64 [n_ranks] on the device)."""
    m = mask.c() if isinstance(mask, Mask) else mask
    _check("fva_sasa_augment", _lib.fva_sasa_augment(
        ctypes.byref(s), _ptr(pooled_q), _ptr(pooled_k), _ptr(rank_of_head), int(budget.shape[0]), _ptr(budget),
        int(order), ctypes.byref(m), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(added), _ptr(dev_status), _stream(stream)))


def fva_build_tiles(s, mask: Mask, workspace, order=FVA_ORDER_HEAD_LPT, dev_status=None, stream=None):
    m = mask.c() if isinstance(mask, Mask) else mask
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("fva_build_tiles", _lib.fva_build_tiles(ctypes.byref(s), ctypes.byref(m), int(order), _ptr(workspace),
                                                   ws_bytes, _ptr(dev_status), _stream(stream)))


def _dtype_code(t):
    return {torch.float32: FVA_F32, torch.bfloat16: FVA_BF16, torch.float16: FVA_F16}[t.dtype]


def fva_sparse_attn(s, q, k, v, mask: Mask, o, scale=0.0, dev_status=None, stream=None, v_dtype=None):
    m = mask.c() if isinstance(mask, Mask) else mask
    vd = _dtype_code(v) if v_dtype is None else int(v_dtype)
    _check("fva_sparse_attn", _lib.fva_sparse_attn(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), vd, ctypes.byref(m),
                                                   _ptr(o), float(scale), _ptr(dev_status), _stream(stream)))


def fva_sparse_attn_range(s, q, k, v, mask: Mask, o, first_slot, n_slots, scale=0.0, dev_status=None, stream=None,
                          v_dtype=None):
    """The tiles at work-list positions [first_slot, first_slot + n_slots) only."""
    m = mask.c() if isinstance(mask, Mask) else mask
    vd = _dtype_code(v) if v_dtype is None else int(v_dtype)
    _check("fva_sparse_attn_range", _lib.fva_sparse_attn_range(
        ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), vd, ctypes.byref(m), _ptr(o), float(scale), int(first_slot),
        int(n_slots), _ptr(dev_status), _stream(stream)))


def fva_dense_attn(s, q, k, v, o, scale=0.0, dev_status=None, stream=None, v_dtype=None):
    vd = _dtype_code(v) if v_dtype is None else int(v_dtype)
    _check("fva_dense_attn", _lib.fva_dense_attn(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), vd, _ptr(o),
                                                 float(scale), _ptr(dev_status), _stream(stream)))


def call_raw(name, *args):
    """Call an entry point and return its status instead of raising (for error-path tests)."""
    return getattr(_lib, name)(*args)
