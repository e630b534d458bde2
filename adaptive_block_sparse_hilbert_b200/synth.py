"""Seeded synthetic video-shaped Q/K/V for the routing + block-sparse attention path.

This module only draws inputs. It holds none of the method's arithmetic (no Hilbert
order, no pooling, no routing, no attention) and imports nothing from the library or
from the oracle, so both sides can take their inputs from it.

Recipe (one layer of a video DiT, B=1, tokens in raster order n = t*Hg*Wg + y*Wg + x):

* a smooth field F[n, :] in R^d: 32 random Fourier features of u = (t/T, y/Hg, x/Wg)
  with frequencies omega_j ~ N(0, 3^2 I_3), features
  phi(u) = [cos(2 pi omega_j.u), sin(2 pi omega_j.u)]_j / sqrt(32) (64 features, unit
  norm), projected by one seeded d x 64 standard-normal matrix W: F = phi W^T;
* per-head temperature tau_h (log-uniform on [0.5, 4], or bimodal for the
  head-heterogeneity workload);
* Q = tau_h (0.5 noise_Q + 0.5 F), K = tau_h (0.5 noise_K + 0.5 F) with independent
  N(0,1) noise, the SAME field for Q and K so that q.k tracks spatial proximity;
* V ~ N(0, 1).

Values are drawn in float32 and then rounded to the workload's dtype (bf16 by
round-to-nearest-even, or kept as fp32). The rounded values are what both the CUDA
path and the oracle consume. A batch of B > 1 (test cases only) stacks B such layers,
each drawn from its own seed.

The pages describe Wan2.x video DiTs at 720p/81 frames (21 latent frames x 3600
tokens = 75,600 tokens); no trained weights are available, so these synthetic tensors
stand in for that workload with its token-grid shape.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# --------------------------------------------------------------------------------------
# Workload table (the five video-shaped configurations)
# --------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    Hg: int
    Wg: int
    H: int
    d: int
    dtype: str  # "f32" or "bf16"
    p: float
    k_floor: int
    tau: tuple  # ("logU", lo, hi) or ("bimodal", flat_frac, tau_flat, tau_conc)
    seed: int
    steps: int = 1
    alphas: tuple = (0.0,)
    B: int = 1
    block: int = 64

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def nB(self) -> int:
        return (self.N + self.block - 1) // self.block


WORKLOADS = {
    0: Workload("tiny_4x16x16_h2_d64_f32", 4, 16, 16, 2, 64, "f32", 0.9, 2, ("logU", 0.5, 4.0), 1000),
    1: Workload("480p_21x30x52_h40_d128_bf16", 21, 30, 52, 40, 128, "bf16", 0.9, 4, ("logU", 0.5, 4.0), 1001),
    2: Workload("720p_21x45x80_h40_d128_bf16", 21, 45, 80, 40, 128, "bf16", 0.9, 4, ("logU", 0.5, 4.0), 1002),
    3: Workload("hetero_13x30x45_h48_d64_bf16", 13, 30, 45, 48, 64, "bf16", 0.9, 2,
                ("bimodal", 0.2, 0.3, 4.0), 1003),
    4: Workload("drift_21x45x80_h40_d128_bf16_4step", 21, 45, 80, 40, 128, "bf16", 0.9, 4,
                ("logU", 0.5, 4.0), 1004, steps=4, alphas=(0.0, 0.3, 0.6, 0.9)),
}

P_SWEEP_720P = (0.8, 0.9, 0.95)


def custom_workload(T, Hg, Wg, H, d, dtype="bf16", p=0.9, k_floor=4, seed=7, tau=("logU", 0.5, 4.0), B=1):
    """A workload of any grid/head/batch shape with the same recipe (used for small test cases).
    With B > 1 each batch entry is drawn as a layer of its own (see make_layer)."""
    name = f"custom_{T}x{Hg}x{Wg}_h{H}_d{d}_{dtype}" + (f"_b{B}" if B > 1 else "")
    return Workload(name, T, Hg, Wg, H, d, dtype, p, k_floor, tau, seed, B=B)


# --------------------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even), numpy only
# --------------------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns (round-to-nearest-even; inputs finite).
    Works through the array in chunks that stay in cache."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.reshape(-1).view(np.uint32)
    out = np.empty(u.size, dtype=np.uint16)
    tmp = np.empty(min(chunk, max(u.size, 1)), dtype=np.uint32)
    for s in range(0, u.size, chunk):
        c = u[s:s + chunk]
        t = tmp[:c.size]
        np.right_shift(c, 16, out=t)
        np.bitwise_and(t, 1, out=t)  # lowest kept bit: ties go to even
        t += np.uint32(0x7FFF)
        t += c
        t >>= 16
        out[s:s + c.size] = t
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    flat = b.reshape(-1)
    out = np.empty(flat.size, dtype=np.uint32)
    for s in range(0, flat.size, chunk):
        o = out[s:s + chunk]
        o[:] = flat[s:s + chunk]
        o <<= 16
    return out.view(np.float32).reshape(b.shape)


# --------------------------------------------------------------------------------------
# Drawing
# --------------------------------------------------------------------------------------


@dataclasses.dataclass
class Layer:
    """One layer's inputs in raster token order, layout [B, N, H, d].

    ``q``, ``k``, ``v`` are float32 arrays holding exactly the values of the workload
    dtype (already bf16-rounded for bf16). ``q_bits`` etc. hold the raw bf16 bit
    patterns (uint16) for bf16 workloads and are None for fp32.
    """

    wl: Workload
    step: int
    tau: np.ndarray
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_bits: np.ndarray | None
    k_bits: np.ndarray | None
    v_bits: np.ndarray | None


def _streams(seed: int, step: int):
    ss = np.random.SeedSequence([seed, step])
    names = ("noise_q", "noise_k", "v", "omega", "w", "tau", "perm")
    return {n: np.random.Generator(np.random.PCG64(s)) for n, s in zip(names, ss.spawn(len(names)))}


def _fourier_field(wl: Workload, rng_omega, rng_w) -> np.ndarray:
    """Smooth field F [N, d] over the (t, y, x) latent grid (float64)."""
    omega = rng_omega.normal(0.0, 3.0, size=(32, 3))
    t = np.arange(wl.T) / wl.T
    y = np.arange(wl.Hg) / wl.Hg
    x = np.arange(wl.Wg) / wl.Wg
    tt, yy, xx = np.meshgrid(t, y, x, indexing="ij")
    u = np.stack([tt.ravel(), yy.ravel(), xx.ravel()], axis=1)  # [N, 3] raster order
    ang = 2.0 * math.pi * (u @ omega.T)  # [N, 32]
    phi = np.concatenate([np.cos(ang), np.sin(ang)], axis=1) / math.sqrt(32.0)  # [N, 64]
    w = rng_w.standard_normal(size=(wl.d, 64))
    return phi @ w.T  # [N, d]


def _tau(wl: Workload, rng) -> np.ndarray:
    kind = wl.tau[0]
    if kind == "logU":
        lo, hi = wl.tau[1], wl.tau[2]
        return np.exp(rng.uniform(math.log(lo), math.log(hi), size=wl.H))
    if kind == "bimodal":
        frac, t_flat, t_conc = wl.tau[1], wl.tau[2], wl.tau[3]
        n_flat = int(round(frac * wl.H))
        tau = np.full(wl.H, t_conc)
        flat = rng.permutation(wl.H)[:n_flat]
        tau[flat] = t_flat
        return tau
    raise ValueError(kind)


def _round(wl: Workload, x32: np.ndarray):
    if wl.dtype == "bf16":
        bits = f32_to_bf16_bits(x32)
        return bf16_bits_to_f32(bits), bits
    return x32, None


def make_layer(wl: Workload, step: int = 0) -> Layer:
    """Draw one layer (one denoising step for the multi-step drift workload). With B > 1
    every batch entry is a layer of its own (own field, tau, noise and V), drawn with the
    seed 1000 * seed + b, so that the entries route differently."""
    if wl.B > 1:
        parts = [make_layer(dataclasses.replace(wl, B=1, seed=wl.seed * 1000 + b), step) for b in range(wl.B)]
        cat = lambda xs: None if xs[0] is None else np.concatenate(xs, axis=0)  # noqa: E731
        return Layer(wl, step, np.stack([x.tau for x in parts]), cat([x.q for x in parts]),
                     cat([x.k for x in parts]), cat([x.v for x in parts]), cat([x.q_bits for x in parts]),
                     cat([x.k_bits for x in parts]), cat([x.v_bits for x in parts]))
    if wl.steps > 1:
        # field of step s = (1 - a_s) field_{s-1} + a_s fresh_s ; step 0 is a fresh field
        field = None
        for s in range(step + 1):
            st = _streams(wl.seed, s)
            fresh = _fourier_field(wl, st["omega"], st["w"])
            a = wl.alphas[s]
            field = fresh if field is None else (1.0 - a) * field + a * fresh
        rng = _streams(wl.seed, step)
    else:
        rng = _streams(wl.seed, step)
        field = _fourier_field(wl, rng["omega"], rng["w"])
    tau = _tau(wl, rng["tau"])
    shape = (wl.B, wl.N, wl.H, wl.d)
    f32 = field.astype(np.float32)[None, :, None, :]  # [1, N, 1, d]
    tau32 = tau.astype(np.float32)[None, None, :, None]
    q = rng["noise_q"].standard_normal(size=shape, dtype=np.float32)
    q *= 0.5
    q += 0.5 * f32
    q *= tau32
    k = rng["noise_k"].standard_normal(size=shape, dtype=np.float32)
    k *= 0.5
    k += 0.5 * f32
    k *= tau32
    v = rng["v"].standard_normal(size=shape, dtype=np.float32)
    q, qb = _round(wl, q)
    k, kb = _round(wl, k)
    v, vb = _round(wl, v)
    return Layer(wl, step, tau, q, k, v, qb, kb, vb)


def random_rows(n_rows: int, n_cols: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain Gaussian matrix (float64), for small synthetic test cases."""
    return np.random.Generator(np.random.PCG64(seed)).standard_normal((n_rows, n_cols)) * scale
