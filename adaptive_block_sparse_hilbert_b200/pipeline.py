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


def ramp_sizes(H: int, steady: int = 4):
    """Head-group sizes for the pipelined layer: groups of 1, 2, 3 heads first (the first
    group's copy-in is the only one nothing overlaps), then `steady`-head groups, and a
    half-size last group (its copy-out is the only one after the compute). Sums to H."""
    sizes, left = [], H
    for n in (1, 2, 3):
        n = min(n, steady, left)
        if n > 0:
            sizes.append(n)
            left -= n
    tail = min(max(1, steady // 2), left)
    left -= tail
    while left > 0:
        n = min(steady, left)
        sizes.append(n)
        left -= n
    if tail > 0:
        sizes.append(tail)
    return sizes


class HostPipelinedLayer:
    """One layer from page-locked host Q, K, V [B, N, H, d] to host O, pipelined over head
    groups: one stream copies group g+1's head slices in while the compute streams run
    groups' reorder -> route -> attention -> inverse reorder and another stream copies group
    g-1's output back. Groups alternate between two compute streams, so a group's launches
    can start on the SMs that the previous group's attention tail leaves idle. Heads are
    independent along the whole path, so every group is an ordinary SparseAttentionLayer on
    a shape with fewer heads, and the output equals the one-shot layer's bit for bit.

    Consecutive forward() calls overlap too: a call's copy-in of a group waits only for the
    previous call's compute of that group (the last reader of the group's input buffers),
    and its compute waits for the previous call's copy-out of that group (the last reader of
    its output buffer). So one layer's copies run during its neighbours' compute. The
    caller's stream is never made to wait: call wait() (or synchronize) before reading
    o_host, and do not overwrite a host input before the call that reads it has finished.

        layer = HostPipelinedLayer(shape, p=0.9, k_floor=4)   # ramp of head groups
        layer.forward(q_host, k_host, v_host, o_host)   # pinned CPU tensors, raster order
        layer.wait()
    """

    def __init__(self, shape: fva.fva_shape, p: float, k_floor: int, groups=None,
                 order: int = fva.FVA_ORDER_HEAD_LPT, device: str = "cuda", v_fp16: bool = True,
                 curve: int = fva.FVA_CURVE_HILBERT, sizes=None, compute_streams: int = 2):
        """groups: None for the ramp schedule (ramp_sizes), or a number of equal groups;
        sizes: explicit head counts per group (overrides groups); compute_streams: streams
        the groups' compute alternates between (1 runs the groups one after another)."""
        s = shape
        H = s.H
        if sizes is None and groups is None:
            sizes = ramp_sizes(H)
        elif sizes is None:
            groups = max(1, min(int(groups), H))
            sizes = [H // groups + (1 if g < H % groups else 0) for g in range(groups)]
        sizes = [int(n) for n in sizes if int(n) > 0]
        if sum(sizes) != H:
            raise ValueError(f"group sizes {sizes} do not add up to {H} heads")
        self.shape = s
        self.heads = []  # (first head, count) per group
        h0 = 0
        for n in sizes:
            self.heads.append((h0, n))
            h0 += n
        self.N = fva.fva_num_tokens(s)
        dt = torch.bfloat16 if s.dtype == fva.FVA_BF16 else torch.float32
        self.esize = 2 if s.dtype == fva.FVA_BF16 else 4
        self.layers, self.q_in, self.k_in, self.v_in, self.o_out = [], [], [], [], []
        for _, n in self.heads:
            gs = fva.make_shape(s.B, n, s.d, s.T, s.Hg, s.Wg, s.dtype)
            self.layers.append(SparseAttentionLayer(gs, p, k_floor, order, device, v_fp16, curve))
            for lst in (self.q_in, self.k_in, self.v_in, self.o_out):
                lst.append(torch.empty((s.B, self.N, n, s.d), dtype=dt, device=device))
        self.s_in = torch.cuda.Stream(device=device)
        self.s_comp = [torch.cuda.Stream(device=device) for _ in range(max(1, int(compute_streams)))]
        self.s_out = torch.cuda.Stream(device=device)
        G = len(self.heads)
        self.in_ready = [torch.cuda.Event() for _ in range(G)]    # group's inputs on the device
        self.comp_done = [torch.cuda.Event() for _ in range(G)]   # group's compute finished
        self.out_done = [torch.cuda.Event() for _ in range(G)]    # group's output in host memory
        self.started = False
        # the buffers (and each group's token order) were made on the current stream
        made = torch.cuda.Event()
        made.record(torch.cuda.current_stream())
        for st in self._streams():
            st.wait_event(made)

    def _streams(self):
        return [self.s_in, *self.s_comp, self.s_out]

    def forward(self, q_host, k_host, v_host, o_host):
        """Enqueue one layer and return the stream that copies its output out (see the
        class notes: nothing is made to wait on it; wait() does that)."""
        s = self.shape
        row = s.H * s.d * self.esize
        rows = s.B * self.N
        for g, ((h0, n), qd, kd, vd) in enumerate(zip(self.heads, self.q_in, self.k_in, self.v_in)):
            if self.started:
                self.s_in.wait_event(self.comp_done[g])
            width = n * s.d * self.esize
            for dst, src in ((qd, q_host), (kd, k_host), (vd, v_host)):
                fva.fva_copy_strided(dst, width, src[:, :, h0:h0 + n, :], row, width, rows, self.s_in)
            self.in_ready[g].record(self.s_in)
        for g, ((h0, n), layer) in enumerate(zip(self.heads, self.layers)):
            st = self.s_comp[g % len(self.s_comp)]
            st.wait_event(self.in_ready[g])
            if self.started:
                st.wait_event(self.out_done[g])
            layer.forward(self.q_in[g], self.k_in[g], self.v_in[g], self.o_out[g], st)
            self.comp_done[g].record(st)
            self.s_out.wait_event(self.comp_done[g])
            width = n * s.d * self.esize
            fva.fva_copy_strided(o_host[:, :, h0:h0 + n, :], row, self.o_out[g], width, width, rows, self.s_out)
            self.out_done[g].record(self.s_out)
        self.started = True
        return self.s_out

    def after(self, stream=None):
        """Make the layer's streams wait for the work already enqueued on `stream` (default:
        the current stream), e.g. a timing event or a producer of the host inputs."""
        st = torch.cuda.current_stream() if stream is None else stream
        for side in self._streams():
            side.wait_stream(st)

    def wait(self, stream=None):
        """Make `stream` (default: the current stream) wait until every enqueued forward()
        has finished, its output copied to host memory."""
        st = torch.cuda.current_stream() if stream is None else stream
        for side in self._streams():
            st.wait_stream(side)

    def dev_status(self):
        """Largest device error code any group reported (0 = none)."""
        return max(int(l.dev_status.item()) for l in self.layers)
