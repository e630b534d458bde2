// Hilbert token order, token reorder with fused float64 block mean-pooling, and its
// inverse ("video-aware block organization", aixai.ru FVAttn blog, "Sparse-routing
// frontend"; pooled Q/K, PaperDaily FVAttn article, 方法揭秘).
//
// The permute kernels are pure data movement and HBM-bound: each CTA owns one
// 64-token block of one (b, h), so every 16-byte vector is read once and written once,
// and the block's pooled row is reduced inside the CTA (no atomics).
#include "fva_internal.cuh"

namespace fva {

// ---------------------------------------------------------------------------------
// Hilbert order of one frame
// ---------------------------------------------------------------------------------

// Cell (x, y) at distance t along the Hilbert curve of side 2^m. Walks the base-4
// digits of t from the least significant: each digit picks a quadrant of the current
// sub-square, and the cells found so far are reflected into that quadrant's
// orientation (lower-left: swap axes; lower-right: reflect about the anti-diagonal).
__device__ __forceinline__ void hilbert_cell(int m, uint32_t t, int* px, int* py) {
  int x = 0, y = 0;
  for (int level = 0; level < m; ++level) {
    const int side = 1 << level;
    const int hi = (t >> 1) & 1;           // right half?
    const int up = (t ^ hi) & 1;           // upper half?
    if (!up) {
      if (hi) {
        x = side - 1 - x;
        y = side - 1 - y;
      }
      const int tmp = x;
      x = y;
      y = tmp;
    }
    x += side * hi;
    y += side * up;
    t >>= 2;
  }
  *px = x;
  *py = y;
}

constexpr int kHilbertChunk = 1024;  // indices per pass: 4^5, one aligned 32 x 32 sub-square

// Index of the first chunk (a multiple of 1024, so an aligned 32 x 32 sub-square) at or
// after b that holds an in-grid cell. The 4^k indices from an index aligned to 4^k form
// one aligned 2^k x 2^k sub-square (every level of the curve only reflects, swaps and
// translates by multiples of the side), so a sub-square whose lower corner lies at or
// beyond the frame is skipped whole, largest first. A wrong skip could only leave cells
// out (perm is written at most Hg * Wg times), never write past the frame.

__device__ uint64_t hilbert_next_chunk(uint64_t b, uint64_t total, int m, int Hg, int Wg) {
  while (b < total) {
    int k = m;
    while (k > 5 && (b & ((1ull << (2 * k)) - 1)) != 0) --k;
    int x, y;
    hilbert_cell(m, static_cast<uint32_t>(b), &x, &y);
    bool skipped = false;
    for (; k >= 5; --k) {
      const int corner = ~((1 << k) - 1);
      if ((x & corner) >= Wg || (y & corner) >= Hg) {
        b += 1ull << (2 * k);
        skipped = true;
        break;
      }
    }
    if (!skipped) return b;
  }
  return total;
}

// One CTA: walk the curve of the enclosing square in order, 1024 indices at a time,
// skipping sub-squares outside the frame, keep in-grid cells (block-wide scan for their
// output slots) and write frame 0's order to perm[0, HW). The square has up to 4^16
// cells, so indices are 64-bit; the work follows the frame's area, not the square's.
__global__ void __launch_bounds__(kHilbertChunk) hilbert_frame_kernel(int m, int Hg, int Wg, int32_t* perm) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  __shared__ uint64_t next_base;
  const uint64_t total = 1ull << (2 * m);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    next_base = hilbert_next_chunk(0, total, m, Hg, Wg);
  }
  __syncthreads();
  while (true) {
    const uint64_t base = next_base;
    if (base >= total) break;
    const uint64_t t = base + threadIdx.x;
    int x = 0, y = 0, valid = 0;
    if (t < total) {
      hilbert_cell(m, static_cast<uint32_t>(t), &x, &y);
      valid = (x < Wg && y < Hg) ? 1 : 0;
    }
    const uint32_t ballot = __ballot_sync(0xffffffffu, valid);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < kHilbertChunk / 32; ++w) {
      const int c = warp_tot[w];
      if (w < warp) before += c;
      all += c;
    }
    const int pos = carry + before + in_warp;
    if (valid) perm[pos] = y * Wg + x;
    __syncthreads();
    if (threadIdx.x == 0) {
      carry += all;
      next_base = hilbert_next_chunk(base + kHilbertChunk, total, m, Hg, Wg);
    }
    __syncthreads();
  }
}

// Replicate frame 0's order over the T frames and build the inverse.
__global__ void hilbert_frames_kernel(int64_t HW, int64_t N, int32_t* perm, int32_t* inv) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / HW;
    const int32_t cell = perm[i - t * HW];
    const int64_t src = t * HW + cell;
    if (t > 0) perm[i] = static_cast<int32_t>(src);
    inv[src] = static_cast<int32_t>(i);
  }
}

// Generalized Hilbert curve over the Hg x Wg frame itself (J. Cerveny's construction): a
// region (first cell, major vector a, minor vector b) one cell thick is walked straight;
// one at least 1.5x longer than thick is cut across a into two halves; otherwise it is cut
// into three parts (half of b first with the roles of a and b swapped, the far part of b,
// then back along -b). Halves are rounded to even lengths so the pieces join by unit
// steps. One thread walks the frame with an explicit stack of pending regions; a stack
// that would overflow, or a cell count other than Hg * Wg, is reported, never written past.
struct RectRegion {
  int x, y, ax, ay, bx, by;
};
constexpr int kRectStack = 256;

__device__ __forceinline__ int isign(int v) { return (v > 0) - (v < 0); }

__global__ void rect_curve_frame_kernel(int Hg, int Wg, int32_t* perm, int32_t* dev_status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  RectRegion stack[kRectStack];
  int top = 0;
  stack[top++] = Wg >= Hg ? RectRegion{0, 0, Wg, 0, 0, Hg} : RectRegion{0, 0, 0, Hg, Wg, 0};
  const int total = Hg * Wg;
  int n = 0;
  while (top > 0) {
    const RectRegion r = stack[--top];
    const int w = abs(r.ax + r.ay), h = abs(r.bx + r.by);
    const int ux = isign(r.ax), uy = isign(r.ay), vx = isign(r.bx), vy = isign(r.by);
    if (h == 1 || w == 1) {
      const int len = h == 1 ? w : h;
      const int sx = h == 1 ? ux : vx, sy = h == 1 ? uy : vy;
      for (int i = 0; i < len; ++i) {
        const int cx = r.x + i * sx, cy = r.y + i * sy;
        if (n >= total || cx < 0 || cx >= Wg || cy < 0 || cy >= Hg) {
          report(dev_status, FVA_DEVERR_MASK);
          return;
        }
        perm[n++] = cy * Wg + cx;
      }
      continue;
    }
    if (top + 3 > kRectStack) {
      report(dev_status, FVA_DEVERR_MASK);
      return;
    }
    int na = w / 2, nb = h / 2;
    if (2 * w > 3 * h) {
      if ((na & 1) && w > 2) ++na;
      // children pushed last-first so the first one is walked next
      stack[top++] = RectRegion{r.x + ux * na, r.y + uy * na, r.ax - ux * na, r.ay - uy * na, r.bx, r.by};
      stack[top++] = RectRegion{r.x, r.y, ux * na, uy * na, r.bx, r.by};
    } else {
      if ((nb & 1) && h > 2) ++nb;
      const int a2x = ux * na, a2y = uy * na, b2x = vx * nb, b2y = vy * nb;
      stack[top++] = RectRegion{r.x + (r.ax - ux) + (b2x - vx), r.y + (r.ay - uy) + (b2y - vy), -b2x, -b2y,
                                -(r.ax - a2x), -(r.ay - a2y)};
      stack[top++] = RectRegion{r.x + b2x, r.y + b2y, r.ax, r.ay, r.bx - b2x, r.by - b2y};
      stack[top++] = RectRegion{r.x, r.y, b2x, b2y, a2x, a2y};
    }
  }
  if (n != total) report(dev_status, FVA_DEVERR_MASK);
}

cudaError_t launch_rect_curve_perm(const Dims& D, int Hg, int Wg, int32_t* perm, int32_t* inv,
                                   int32_t* dev_status, cudaStream_t st) {
  rect_curve_frame_kernel<<<1, 32, 0, st>>>(Hg, Wg, perm, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t HW = static_cast<int64_t>(Hg) * Wg;
  int grid = static_cast<int>((D.N + 255) / 256);
  if (grid > 148 * 16) grid = 148 * 16;
  hilbert_frames_kernel<<<grid, 256, 0, st>>>(HW, D.N, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_hilbert_perm(const Dims& D, int T, int Hg, int Wg, int32_t* perm, int32_t* inv,
                                cudaStream_t st) {
  int m = 0;
  while ((1 << m) < (Hg > Wg ? Hg : Wg)) ++m;
  hilbert_frame_kernel<<<1, kHilbertChunk, 0, st>>>(m, Hg, Wg, perm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t HW = static_cast<int64_t>(Hg) * Wg;
  int grid = static_cast<int>((D.N + 255) / 256);
  if (grid > 148 * 16) grid = 148 * 16;
  // frame 0 entries are read by every frame; the kernel only rewrites frames t > 0, so
  // the reads of perm[0, HW) never race with writes.
  hilbert_frames_kernel<<<grid, 256, 0, st>>>(HW, D.N, perm, inv);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------
// Reorder / pool
// ---------------------------------------------------------------------------------

template <typename T>
__device__ __forceinline__ void add_vec(double* acc, const uint4& v);

template <>
__device__ __forceinline__ void add_vec<__nv_bfloat16>(double* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += static_cast<double>(__uint_as_float(w[i] << 16));
    acc[2 * i + 1] += static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
  }
}
template <>
__device__ __forceinline__ void add_vec<float>(double* acc, const uint4& v) {
  acc[0] += static_cast<double>(__uint_as_float(v.x));
  acc[1] += static_cast<double>(__uint_as_float(v.y));
  acc[2] += static_cast<double>(__uint_as_float(v.z));
  acc[3] += static_cast<double>(__uint_as_float(v.w));
}

constexpr int kReorderThreads = 256;

// Eight bf16 values -> eight fp16 values (exact in range, saturated to +-65504 outside).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = fminf(fmaxf(__uint_as_float(w[i] << 16), -65504.0f), 65504.0f);
    const float hi = fminf(fmaxf(__uint_as_float(w[i] & 0xFFFF0000u), -65504.0f), 65504.0f);
    o[i] = pack_f16x2(lo, hi);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// MODE 0: forward permute [B,N,H,d] -> [B,H,N,d] (+ pool)
// MODE 1: inverse permute [B,H,N,d] -> [B,N,H,d]
// MODE 2: pool only, input already [B,H,N,d]
// MODE 3: forward permute with the output converted bf16 -> fp16
// One CTA per (block a, group of G adjacent heads, batch b); VPR = 16-byte vectors per
// (token, head) row. The G heads of one token are adjacent in [B,N,H,d], so a token's
// G * VPR vectors are one contiguous run: short rows (d * sizeof(T) < 256 B) are moved
// G heads at a time and every CTA moves 64 rows of 256 B or more. Every thread keeps one
// vector column and loads all of its rows before storing any, so a CTA has its whole
// 64-row block in flight.
template <typename T, int MODE, bool POOL, int VPR, int G>
__global__ void __launch_bounds__(kReorderThreads) reorder_kernel(
    const uint8_t* __restrict__ x_in, uint8_t* __restrict__ x_out, double* __restrict__ pooled,
    const int32_t* __restrict__ perm, int N, int H) {
  constexpr int EPV = 16 / sizeof(T);          // elements per 16-byte vector
  constexpr int VPT = VPR * G;                 // vectors per token (its G heads)
  constexpr int RPP = kReorderThreads / VPT;   // rows per pass
  constexpr int NPASS = (kBlock + RPP - 1) / RPP;
  constexpr int64_t kRowBytes = VPR * 16;
  constexpr int kWidth = VPR * EPV;            // = d
  __shared__ double red[POOL ? RPP * kWidth * G : 1];
  const int a = blockIdx.x, h0 = blockIdx.y * G, b = blockIdx.z;
  const int v = threadIdx.x % VPT;             // vector within the token's G heads
  const int g = v / VPR, vc = v % VPR;         // its head within the group, its column
  const int r0 = threadIdx.x / VPT;
  const int row_lo = a * kBlock;
  const int n_valid = min(kBlock, N - row_lo);
  uint4 buf[NPASS];
#pragma unroll
  for (int ps = 0; ps < NPASS; ++ps) {
    const int r = r0 + ps * RPP;
    if (r < n_valid) {
      const int i = row_lo + r;
      const uint4* src;
      if (MODE == 0 || MODE == 3) {
        src = reinterpret_cast<const uint4*>(x_in + ((static_cast<int64_t>(b) * N + perm[i]) * H + h0) * kRowBytes) + v;
      } else {
        src = reinterpret_cast<const uint4*>(x_in + ((static_cast<int64_t>(b) * H + h0 + g) * N + i) * kRowBytes) + vc;
      }
      buf[ps] = __ldg(src);
    }
  }
  double acc[POOL ? EPV : 1];
  if (POOL) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] = 0.0;
  }
#pragma unroll
  for (int ps = 0; ps < NPASS; ++ps) {
    const int r = r0 + ps * RPP;
    if (r < n_valid) {
      const int i = row_lo + r;
      if (MODE != 2) {
        uint4* dst;
        if (MODE == 0 || MODE == 3) {
          dst = reinterpret_cast<uint4*>(x_out + ((static_cast<int64_t>(b) * H + h0 + g) * N + i) * kRowBytes) + vc;
        } else {
          dst = reinterpret_cast<uint4*>(x_out + ((static_cast<int64_t>(b) * N + perm[i]) * H + h0) * kRowBytes) + v;
        }
        *dst = (MODE == 3) ? bf16x8_to_f16x8(buf[ps]) : buf[ps];
      }
      if (POOL) add_vec<T>(acc, buf[ps]);
    }
  }
  if (POOL) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) red[r0 * (G * kWidth) + v * EPV + e] = acc[e];
    __syncthreads();
    // column sums over the RPP partial rows, fixed order; column c of the group is column
    // c % d of head h0 + c / d
    for (int c = threadIdx.x; c < G * kWidth; c += kReorderThreads) {
      double sum = 0.0;
#pragma unroll 8
      for (int r = 0; r < RPP; ++r) sum += red[r * (G * kWidth) + c];
      const int hh = h0 + c / kWidth;
      pooled[((static_cast<int64_t>(b) * H + hh) * gridDim.x + a) * kWidth + (c % kWidth)] =
          sum / static_cast<double>(n_valid);
    }
  }
}

template <typename T, int VPR, int G>
static cudaError_t launch_reorder_g(const Dims& D, const void* x_in, void* x_out, double* pooled,
                                    const int32_t* perm, int mode, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(D.nB), static_cast<unsigned>(D.H / G), static_cast<unsigned>(D.B));
  const uint8_t* in = static_cast<const uint8_t*>(x_in);
  uint8_t* out = static_cast<uint8_t*>(x_out);
  const int N = static_cast<int>(D.N), H = static_cast<int>(D.H);
  if (mode == 0 && pooled) {
    reorder_kernel<T, 0, true, VPR, G><<<grid, kReorderThreads, 0, st>>>(in, out, pooled, perm, N, H);
  } else if (mode == 0) {
    reorder_kernel<T, 0, false, VPR, G><<<grid, kReorderThreads, 0, st>>>(in, out, nullptr, perm, N, H);
  } else if (mode == 1) {
    reorder_kernel<T, 1, false, VPR, G><<<grid, kReorderThreads, 0, st>>>(in, out, nullptr, perm, N, H);
  } else if (mode == 3) {
    reorder_kernel<T, 3, false, VPR, G><<<grid, kReorderThreads, 0, st>>>(in, out, nullptr, perm, N, H);
  } else {
    reorder_kernel<T, 2, true, VPR, G><<<grid, kReorderThreads, 0, st>>>(in, nullptr, pooled, nullptr, N, H);
  }
  return cudaGetLastError();
}

// Heads moved together: enough that a token's group spans 16 vectors (256 B), and a
// divisor of H.
template <typename T, int VPR>
static cudaError_t launch_reorder_v(const Dims& D, const void* x_in, void* x_out, double* pooled,
                                    const int32_t* perm, int mode, cudaStream_t st) {
  if constexpr (VPR == 4) {
    if (D.H % 4 == 0) return launch_reorder_g<T, VPR, 4>(D, x_in, x_out, pooled, perm, mode, st);
  }
  if constexpr (VPR <= 8) {
    if (D.H % 2 == 0) return launch_reorder_g<T, VPR, 2>(D, x_in, x_out, pooled, perm, mode, st);
  }
  return launch_reorder_g<T, VPR, 1>(D, x_in, x_out, pooled, perm, mode, st);
}

template <typename T>
static cudaError_t launch_reorder_t(const Dims& D, const void* x_in, void* x_out, double* pooled,
                                    const int32_t* perm, int mode, cudaStream_t st) {
  switch (D.d * static_cast<int64_t>(sizeof(T)) / 16) {
    case 4: return launch_reorder_v<T, 4>(D, x_in, x_out, pooled, perm, mode, st);
    case 8: return launch_reorder_v<T, 8>(D, x_in, x_out, pooled, perm, mode, st);
    case 16: return launch_reorder_v<T, 16>(D, x_in, x_out, pooled, perm, mode, st);
    case 32: return launch_reorder_v<T, 32>(D, x_in, x_out, pooled, perm, mode, st);
    case 64: return launch_reorder_v<T, 64>(D, x_in, x_out, pooled, perm, mode, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_reorder(const Dims& D, const void* x_in, void* x_out, double* pooled,
                           const int32_t* perm, int direction, cudaStream_t st) {
  const int mode = direction == FVA_FWD ? 0 : (direction == FVA_INV ? 1 : 3);
  if (D.esize == 2) return launch_reorder_t<__nv_bfloat16>(D, x_in, x_out, pooled, perm, mode, st);
  return launch_reorder_t<float>(D, x_in, x_out, pooled, perm, mode, st);
}

cudaError_t launch_pool(const Dims& D, const void* x_bhnd, double* pooled, cudaStream_t st) {
  if (D.esize == 2) return launch_reorder_t<__nv_bfloat16>(D, x_bhnd, nullptr, pooled, nullptr, 2, st);
  return launch_reorder_t<float>(D, x_bhnd, nullptr, pooled, nullptr, 2, st);
}

}  // namespace fva
