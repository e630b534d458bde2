"""One attention layer through libfva: Hilbert reorder (+ pooling) -> route -> block-sparse
attention -> inverse reorder. Orchestration and buffer ownership only; every step is a
libfva entry point.

    layer = SparseAttentionLayer(shape, p=0.9, k_floor=4)
    layer.forward(q_bnhd, k_bnhd, v_bnhd, o_bnhd)   # torch CUDA tensors, raster order
"""
from __future__ import annotations

import torch

from . import fva


class SparseAttentionLayer:
    def __init__(self, shape: fva.fva_shape, p: float, k_floor: int, order: int = fva.FVA_ORDER_HEAD_LPT,
                 device: str = "cuda", v_fp16: bool = True, curve: int = fva.FVA_CURVE_HILBERT):
        self.shape = shape
        self.p = float(p)
        self.k_floor = int(k_floor)
        self.order = int(order)
        s = shape
        self.N = fva.fva_num_tokens(s)
        self.nB = fva.fva_num_blocks(s)
        dt = torch.bfloat16 if s.dtype == fva.FVA_BF16 else torch.float32
        self.dtype = dt
        bhnd = (s.B, s.H, self.N, s.d)
        self.perm = torch.empty(self.N, dtype=torch.int32, device=device)
        self.inv = torch.empty(self.N, dtype=torch.int32, device=device)
        self.qh = torch.empty(bhnd, dtype=dt, device=device)
        self.kh = torch.empty(bhnd, dtype=dt, device=device)
        # bf16 layers keep the Hilbert-ordered V in fp16 so P.V runs with fp16 P (8x finer
        # rounding of the attention weights than bf16); the conversion is fused into the reorder
        self.v_fp16 = bool(v_fp16) and s.dtype == fva.FVA_BF16
        self.vh = torch.empty(bhnd, dtype=torch.float16 if self.v_fp16 else dt, device=device)
        self.oh = torch.empty(bhnd, dtype=dt, device=device)
        self.pooled_q = torch.empty((s.B, s.H, self.nB, s.d), dtype=torch.float64, device=device)
        self.pooled_k = torch.empty_like(self.pooled_q)
        self.mask = fva.Mask.allocate(s, device)
        ws = fva.fva_route_workspace_bytes(s, False)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=device)
        self.curve = int(curve)
        fva.fva_curve_perm(s, self.curve, self.perm, self.inv, self.dev_status)

    def reorder_inputs(self, q, k, v, stream=None):
        s = self.shape
        fva.fva_reorder(s, q, self.qh, self.pooled_q, self.perm, fva.FVA_FWD, stream)
        fva.fva_reorder(s, k, self.kh, self.pooled_k, self.perm, fva.FVA_FWD, stream)
        fva.fva_reorder(s, v, self.vh, None, self.perm, fva.FVA_FWD_F16 if self.v_fp16 else fva.FVA_FWD, stream)

    def route(self, stream=None):
        fva.fva_route(self.shape, None, None, self.pooled_q, self.pooled_k, self.p, self.k_floor, self.mask,
                      self.workspace, self.order, self.dev_status, stream)

    def attend(self, stream=None, scale: float = 0.0):
        fva.fva_sparse_attn(self.shape, self.qh, self.kh, self.vh, self.mask, self.oh, scale, self.dev_status, stream)

    def restore_output(self, o_out, stream=None):
        fva.fva_reorder(self.shape, self.oh, o_out, None, self.perm, fva.FVA_INV, stream)

    def forward(self, q, k, v, o_out, stream=None):
        self.reorder_inputs(q, k, v, stream)
        self.route(stream)
        self.attend(stream)
        self.restore_output(o_out, stream)
        return o_out
