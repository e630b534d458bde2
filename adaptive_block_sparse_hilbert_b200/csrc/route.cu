// Top-p block routing with a Top-k safety floor, CSR mask, per-head kept counts,
// tile lists and the longest-first work list.
//
// Method (aixai.ru FVAttn blog, "Top-p vs Top-k" and "Sparse-routing frontend";
// PaperDaily FVAttn article, 方法揭秘 and 龙迷三问): block importance from pooled Q/K,
// keep key blocks in importance order until the cumulative importance reaches p, and
// never fewer than k_floor blocks.
//
// Kernels (all float64 where a value decides the mask):
//   route_scores_kernel   S = pooled_q pooled_k^T / sqrt(d), a GEMM on the FP64 tensor-core
//                         MMA (mma.sync m8n8k4.f64)
//   route_select_kernel   one warp per row: softmax, bucket refinement to the cut,
//                         exact (logit desc, index asc) order inside the last bucket,
//                         kept bitmask, kept count, per-tile union cost
//   finish_kernel         row_ptr / tile_ptr scans, head_kept, per-head load
//   order_*_kernel        work list (natural, global LPT, head-grouped LPT)
//   emit_kernel           col_idx (ascending) and tile_col (union + membership bits)
#include <math.h>

#include "fva_internal.cuh"

namespace fva {

// ---------------------------------------------------------------------------------
// Block logits
// ---------------------------------------------------------------------------------
constexpr int kDK = 16;       // d-chunk per pipeline stage (every supported d is a multiple of 16)
constexpr int kDP = kDK + 4;  // padded row (doubles): a half-warp's fragment loads hit 32 banks
constexpr int kStages = 3;    // d-chunks in flight, so one barrier per chunk suffices

__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// 16-byte global -> shared copy; with `valid` false the destination is zero-filled and
// nothing is read
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_but_one() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// A warp computes MI x NI MMA tiles of 8 x 8 (lane (g, t) holds A[g][t], B[t][g] and
// C[g][2t], C[g][2t+1] of a tile); a CTA is WR x WC warps.
template <int MI, int NI, int WR, int WC>
struct ScoresCfg {
  static constexpr int kMI = MI, kNI = NI, kWR = WR, kWC = WC;
  static constexpr int kBM = 8 * MI * WR;            // CTA tile rows (query blocks)
  static constexpr int kBN = 8 * NI * WC;            // CTA tile columns (key blocks)
  static constexpr int kThreads = 32 * WR * WC;
  static constexpr int kStageD = (kBM + kBN) * kDP;  // doubles per stage
  static constexpr size_t kSmem = static_cast<size_t>(kStages) * kStageD * 8;
};
// 128 x 64 logits per CTA as 4 x 2 warps of 32 x 32, two CTAs per SM: sixteen warps hide
// the MMA and shared-memory latencies, and one CTA's epilogue overlaps the other's products.
using Scores = ScoresCfg<4, 4, 4, 2>;
constexpr int kScoresCtasPerSm = 2;

// grid: (ceil(nB / kBN), ceil(nB / kBM), B*H). Every logit is the sum over d in ascending
// order, four products per MMA step, divided by sqrt(d) at the end; the tiling changes no
// bit of it.
template <class C>
__global__ void __launch_bounds__(C::kThreads, kScoresCtasPerSm)
    route_scores_kernel(const double* __restrict__ pq, const double* __restrict__ pk, double* __restrict__ S,
                        int nB, int d, double sqrt_d) {
  constexpr int MI = C::kMI, NI = C::kNI, BM = C::kBM, BN = C::kBN;
  extern __shared__ __align__(16) double sm_d[];
  const int bh = blockIdx.z;
  const int a0 = blockIdx.y * BM, b0 = blockIdx.x * BN;
  const double* Q = pq + static_cast<int64_t>(bh) * nB * d;
  const double* K = pk + static_cast<int64_t>(bh) * nB * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wm = warp % C::kWR, wn = warp / C::kWR;
  const int g = lane >> 2, t = lane & 3;
  double acc[MI][NI][2];
#pragma unroll
  for (int mi = 0; mi < MI; ++mi)
#pragma unroll
    for (int ni = 0; ni < NI; ++ni) acc[mi][ni][0] = acc[mi][ni][1] = 0.0;

  // stage rows: BM rows of pooled Q, then BN rows of pooled K, 8 x 16 bytes each
  auto issue = [&](int chunk) {
    double* st = sm_d + (chunk % kStages) * C::kStageD;
    const int i0 = chunk * kDK;
    for (int c = threadIdx.x; c < (BM + BN) * 8; c += C::kThreads) {
      const int r = c >> 3, part = c & 7;
      const bool is_q = r < BM;
      const int gr = is_q ? a0 + r : b0 + (r - BM);
      const bool ok = gr < nB;
      const double* src = (is_q ? Q : K) + static_cast<int64_t>(ok ? gr : 0) * d + i0 + 2 * part;
      cp_async16(st + r * kDP + 2 * part, src, ok);
    }
  };
  const int nk = d / kDK;
  issue(0);
  cp_async_commit();
  if (nk > 1) issue(1);
  cp_async_commit();
  for (int c = 0; c < nk; ++c) {
    cp_async_wait_all_but_one();  // this thread's copies of chunk c have landed
    __syncthreads();              // everyone's have, and chunk c - 1 is no longer read
    if (c + 2 < nk) issue(c + 2);
    cp_async_commit();
    const double* As = sm_d + (c % kStages) * C::kStageD;
    const double* Bs = As + BM * kDP;
#pragma unroll
    for (int kk = 0; kk < kDK; kk += 4) {
      double af[MI], bf[NI];
#pragma unroll
      for (int mi = 0; mi < MI; ++mi) af[mi] = As[(wm * 8 * MI + mi * 8 + g) * kDP + kk + t];
#pragma unroll
      for (int ni = 0; ni < NI; ++ni) bf[ni] = Bs[(wn * 8 * NI + ni * 8 + g) * kDP + kk + t];
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni) dmma_8x8x4(acc[mi][ni][0], acc[mi][ni][1], af[mi], bf[ni]);
    }
  }
#pragma unroll
  for (int mi = 0; mi < MI; ++mi) {
    const int a = a0 + wm * 8 * MI + mi * 8 + g;
    if (a >= nB) continue;
    double* dst = S + (static_cast<int64_t>(bh) * nB + a) * nB;
#pragma unroll
    for (int ni = 0; ni < NI; ++ni) {
      const int b = b0 + wn * 8 * NI + ni * 8 + 2 * t;
      if (b < nB) dst[b] = acc[mi][ni][0] / sqrt_d;
      if (b + 1 < nB) dst[b + 1] = acc[mi][ni][1] / sqrt_d;
    }
  }
}

// ---------------------------------------------------------------------------------
// Selection
// ---------------------------------------------------------------------------------
constexpr int kNBK = 128;                       // buckets per refinement level
constexpr int kMaxLevels = 12;
constexpr double kFix = 4503599627370496.0;     // 2^52: fixed-point unit of importance

// Shared memory of one row's warp. The importances exp(s - max) are recomputed where they
// are needed rather than kept (the same operation on the same inputs, so the same bits): an
// fp64 copy of them beside the logits would nearly double the arena and cut the rows that fit
// on an SM, and kept in place of the logits (which the passes then read again from L2) they
// made the kernel slower. Candidates are 16-bit block indices for the same reason.
struct WarpArena {
  double* s;          // [nB] the row's logits
  uint64_t* hw;       // [kNBK] bucket mass (fixed point); last: masses of the final candidates
  uint16_t* list;     // [nB] candidate block indices (routable nB < 2^16)
  int32_t* hcnt;      // [kNBK] bucket counts
  uint32_t* words;    // [nWords] kept bitmask of the row
};

__host__ __device__ inline size_t warp_arena_bytes(int nB, int nWords) {
  size_t b = 0;
  b += align_up(static_cast<size_t>(nB) * 8, 16);
  b += kNBK * 8;
  b += align_up(static_cast<size_t>(nB) * 2, 16);
  b += kNBK * 4;
  b += align_up(static_cast<size_t>(nWords) * 4, 16);
  return b;
}

__device__ inline WarpArena make_arena(uint8_t* base, int nB, int nWords) {
  WarpArena A;
  size_t off = 0;
  A.s = reinterpret_cast<double*>(base + off);
  off += align_up(static_cast<size_t>(nB) * 8, 16);
  A.hw = reinterpret_cast<uint64_t*>(base + off);
  off += kNBK * 8;
  A.list = reinterpret_cast<uint16_t*>(base + off);
  off += align_up(static_cast<size_t>(nB) * 2, 16);
  A.hcnt = reinterpret_cast<int32_t*>(base + off);
  off += kNBK * 4;
  A.words = reinterpret_cast<uint32_t*>(base + off);
  return A;
}

// (s_j, j) precedes (s_i, i) in the routing order: larger logit, or equal logit and
// lower block index.
__device__ __forceinline__ bool precedes(double sj, int j, double si, int i) {
  return sj > si || (sj == si && j < i);
}

// importance e/Z in units of 2^-52 (zscale = 2^52 / Z), truncated
__device__ __forceinline__ uint64_t fixed_mass(double e, double zscale) {
  return static_cast<uint64_t>(e * zscale);
}

struct Pivot {
  int found;   // 0: the mass target is never reached (keep everything)
  int L;       // 1-based position of the pivot in the routing order
  double s;    // pivot logit
  int b;       // pivot block
};

// Find the pivot of the routing order for one row.
// by_mass: the first position whose cumulative fixed-point mass reaches `pth`
// (= p * 2^52); otherwise the position `cnt_target` (1-based) by count.
__device__ Pivot select_pivot(const WarpArena& A, int nB, double smax, double smin, double zscale, bool by_mass,
                              double pth, int cnt_target) {
  const double* srow = A.s;
  const int lane = threadIdx.x & 31;
  uint64_t above_w = 0;
  int above_c = 0;
  double lo = smin, hi = smax;
  int c = nB;            // candidates
  bool implicit = true;  // candidates are all blocks [0, nB)
  for (int level = 0; level < kMaxLevels; ++level) {
    if (c <= 32 || !(hi > lo)) break;
    const double kappa = static_cast<double>(kNBK) / (hi - lo);
    for (int i = lane; i < kNBK; i += 32) {
      A.hcnt[i] = 0;
      A.hw[i] = 0;
    }
    __syncwarp();
    for (int i = lane; i < c; i += 32) {
      const int b = implicit ? i : A.list[i];
      const double s = srow[b];
      int bk = static_cast<int>((hi - s) * kappa);
      bk = bk < 0 ? 0 : (bk >= kNBK ? kNBK - 1 : bk);
      atomicAdd(&A.hcnt[bk], 1);
      if (by_mass) atomicAdd(reinterpret_cast<unsigned long long*>(&A.hw[bk]),
                             static_cast<unsigned long long>(fixed_mass(exp(s - smax), zscale)));
    }
    __syncwarp();
    // lane owns buckets 4*lane .. 4*lane+3
    int cnt4[4];
    uint64_t w4[4];
    int csum = 0;
    uint64_t wsum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      cnt4[q] = A.hcnt[4 * lane + q];
      w4[q] = A.hw[4 * lane + q];
      csum += cnt4[q];
      wsum += w4[q];
    }
    // exclusive prefix over lanes
    int cpre = csum;
    uint64_t wpre = wsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int cn = __shfl_up_sync(0xffffffffu, cpre, o);
      const uint64_t wn = __shfl_up_sync(0xffffffffu, wpre, o);
      if (lane >= o) {
        cpre += cn;
        wpre += wn;
      }
    }
    cpre -= csum;
    wpre -= wsum;
    // first bucket (lowest index = highest logits) where the running total reaches the target
    int hit = kNBK;
    int hit_c_before = 0;
    uint64_t hit_w_before = 0;
    {
      int cc = cpre;
      uint64_t ww = wpre;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool reach = by_mass ? (static_cast<double>(above_w + ww + w4[q]) >= pth)
                                   : (above_c + cc + cnt4[q] >= cnt_target);
        if (reach && hit == kNBK) {
          hit = 4 * lane + q;
          hit_c_before = cc;
          hit_w_before = ww;
        }
        cc += cnt4[q];
        ww += w4[q];
      }
    }
    // lowest lane with a hit decides
    const unsigned hmask = __ballot_sync(0xffffffffu, hit < kNBK);
    if (hmask == 0) {
      Pivot none;
      none.found = 0;
      none.L = nB;
      none.s = smin;
      none.b = nB - 1;
      return none;  // mass target not reached by the whole row
    }
    const int src = __ffs(hmask) - 1;
    const int B = __shfl_sync(0xffffffffu, hit, src);
    above_c += __shfl_sync(0xffffffffu, hit_c_before, src);
    above_w += __shfl_sync(0xffffffffu, hit_w_before, src);
    // compact the candidates of bucket B (ascending block index is kept)
    int newc = 0;
    double nlo = INFINITY, nhi = -INFINITY;
    for (int i0 = 0; i0 < c; i0 += 32) {
      const int i = i0 + lane;
      int b = -1;
      bool in = false;
      double s = 0.0;
      if (i < c) {
        b = implicit ? i : A.list[i];
        s = srow[b];
        int bk = static_cast<int>((hi - s) * kappa);
        bk = bk < 0 ? 0 : (bk >= kNBK ? kNBK - 1 : bk);
        in = (bk == B);
      }
      const unsigned m = __ballot_sync(0xffffffffu, in);
      __syncwarp();
      if (in) {
        A.list[newc + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(b);
        nlo = fmin(nlo, s);
        nhi = fmax(nhi, s);
      }
      newc += __popc(m);
      __syncwarp();
    }
    c = newc;
    implicit = false;
    lo = warp_min_d(nlo);
    hi = warp_max_d(nhi);
  }
  if (implicit) {
    for (int i = lane; i < c; i += 32) A.list[i] = static_cast<uint16_t>(i);
    __syncwarp();
  }
  // masses of the remaining candidates, kept in the bucket array when they fit (the
  // levels normally leave <= 32; equal logits can leave more, which recompute)
  const bool cached = by_mass && c <= kNBK;
  if (cached) {
    for (int i = lane; i < c; i += 32) A.hw[i] = fixed_mass(exp(srow[A.list[i]] - smax), zscale);
    __syncwarp();
  }
  // exact order inside the remaining candidates: rank and inclusive cumulative mass
  int best_rank = 0x7fffffff;
  int best_b = -1;
  double best_s = 0.0;
  for (int i0 = 0; i0 < c; i0 += 32) {
    const int i = i0 + lane;
    if (i < c) {
      const int bi = A.list[i];
      const double si = srow[bi];
      int rank = 0;
      uint64_t cw = 0;
      for (int j = 0; j < c; ++j) {
        const int bj = A.list[j];
        const double sj = srow[bj];
        if (precedes(sj, bj, si, bi)) {
          ++rank;
          if (by_mass) cw += cached ? A.hw[j] : fixed_mass(exp(sj - smax), zscale);
        }
      }
      bool ok;
      if (by_mass) {
        cw += cached ? A.hw[i] : fixed_mass(exp(si - smax), zscale);
        ok = static_cast<double>(above_w + cw) >= pth;
      } else {
        ok = (above_c + rank + 1 == cnt_target);
      }
      if (ok && rank < best_rank) {
        best_rank = rank;
        best_b = bi;
        best_s = si;
      }
    }
  }
  // warp argmin over rank
  int r = best_rank;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r = min(r, __shfl_xor_sync(0xffffffffu, r, o));
  const unsigned who = __ballot_sync(0xffffffffu, best_rank == r && best_b >= 0);
  Pivot pv;
  if (who == 0) {
    pv.found = 0;  // mass target not reached (truncated total below p)
    pv.L = nB;
    pv.s = smin;
    pv.b = nB - 1;
    return pv;
  }
  const int src = __ffs(who) - 1;
  pv.found = 1;
  pv.L = above_c + r + 1;
  pv.b = __shfl_sync(0xffffffffu, best_b, src);
  pv.s = __shfl_sync(0xffffffffu, best_s, src);
  return pv;
}

// grid: (ceil(nB / rows_per_cta), BH); block: 32 * rows_per_cta (rows_per_cta even)
__global__ void route_select_kernel(const double* __restrict__ S, int nB, int nWords, int nPairs,
                                    double p, int k_floor, uint32_t* __restrict__ bits,
                                    int32_t* __restrict__ row_cnt, int32_t* __restrict__ tile_cost,
                                    int32_t* dev_status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_cta = blockDim.x >> 5;
  const int bh = blockIdx.y;
  const int a0 = blockIdx.x * rows_per_cta;
  const int a = a0 + warp;
  const size_t arena = warp_arena_bytes(nB, nWords);
  WarpArena A = make_arena(smem_raw + arena * warp, nB, nWords);

  if (a < nB) {
    const int64_t row = static_cast<int64_t>(bh) * nB + a;
    const double* grow = S + row * nB;
    double* srow = A.s;
    double smax = -INFINITY, smin = INFINITY;
    for (int b = lane; b < nB; b += 32) {
      const double s = grow[b];
      srow[b] = s;
      smax = fmax(smax, s);
      smin = fmin(smin, s);
    }
    smax = warp_max_d(smax);
    smin = warp_min_d(smin);
    double z = 0.0;
    for (int b = lane; b < nB; b += 32) {
      z += exp(srow[b] - smax);
    }
    const double Z = warp_sum_d(z);
    const double zscale = kFix / Z;
    __syncwarp();

    const int L_k = k_floor < nB ? k_floor : nB;
    bool all = (p >= 1.0) || (L_k >= nB);
    Pivot pv;
    pv.found = 0;
    pv.L = nB;
    pv.s = smin;
    pv.b = nB - 1;
    if (!all) {
      pv = select_pivot(A, nB, smax, smin, zscale, true, p * kFix, 0);
      if (!pv.found) {
        all = true;
      } else if (pv.L < L_k) {
        pv = select_pivot(A, nB, smax, smin, zscale, false, 0.0, L_k);
        if (!pv.found) all = true;
      }
    }
    int kept = 0;
    for (int k = 0; k < nWords; ++k) {
      const int b = 32 * k + lane;
      bool keep = false;
      if (b < nB) keep = all || precedes(srow[b], b, pv.s, pv.b) || b == pv.b;
      const unsigned w = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) A.words[k] = w;
      kept += __popc(w);
    }
    __syncwarp();
    for (int k = lane; k < nWords; k += 32) bits[row * nWords + k] = A.words[k];
    if (lane == 0) {
      row_cnt[row] = kept;
      if (kept != (all ? nB : pv.L)) report(dev_status, FVA_DEVERR_MASK);
    }
  }
  __syncthreads();
  // per-tile union cost for the pairs (2t, 2t+1) inside this CTA (a0 is even)
  if ((warp & 1) == 0 && a < nB) {
    const int t = a >> 1;
    const bool has_b = (a + 1 < nB);
    const WarpArena Bn = make_arena(smem_raw + arena * (warp + 1), nB, nWords);
    int u = 0;
    for (int k = lane; k < nWords; k += 32) u += __popc(A.words[k] | (has_b ? Bn.words[k] : 0u));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
    if (lane == 0) tile_cost[static_cast<int64_t>(bh) * nPairs + t] = u;
  }
}

// ---------------------------------------------------------------------------------
// Scans, per-head counts
// ---------------------------------------------------------------------------------
// Exclusive scan of n int32 into out[0..n] by one 1024-thread block; returns the total.
// The block walks the array in chunks of 4 x blockDim.x consecutive elements (each thread
// four neighbours, so loads and stores are coalesced), loading the next chunk before it
// combines the current one; `smem` holds 33 int64.
__device__ int64_t block_exclusive_scan(const int32_t* __restrict__ in, int32_t* __restrict__ out,
                                        int64_t n, int64_t* smem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = 4 * static_cast<int64_t>(blockDim.x);
  auto load = [&](int64_t base, int32_t* v) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t i = base + 4 * tid + q;
      v[q] = i < n ? in[i] : 0;
    }
  };
  int32_t cur[4], nxt[4];
  load(0, cur);
  int64_t run = 0;  // sum of every chunk before this one
  for (int64_t base = 0; base < n; base += chunk) {
    if (base + chunk < n) load(base + chunk, nxt);
    const int64_t local = static_cast<int64_t>(cur[0]) + cur[1] + cur[2] + cur[3];
    int64_t inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) smem[warp] = inc;
    __syncthreads();
    if (warp == 0) {  // scan of the warp totals
      const int nw = static_cast<int>(blockDim.x >> 5);
      const int64_t wv = lane < nw ? smem[lane] : 0;
      int64_t wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      if (lane < nw) smem[lane] = wi - wv;
      if (lane == 31) smem[32] = wi;
    }
    __syncthreads();
    int64_t x = run + smem[warp] + inc - local;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t i = base + 4 * tid + q;
      if (i < n) out[i] = static_cast<int32_t>(x);
      x += cur[q];
    }
    run += smem[32];
    __syncthreads();  // smem is rewritten by the next chunk
#pragma unroll
    for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
  }
  if (tid == 0) out[n] = static_cast<int32_t>(run);
  __syncthreads();
  return run;
}

__global__ void __launch_bounds__(1024) finish_kernel(const int32_t* __restrict__ row_cnt, int64_t rows,
                                                      const int32_t* __restrict__ tile_cost, int64_t tiles,
                                                      int nB, int nPairs, int BH, int32_t* row_ptr,
                                                      int32_t* tile_ptr, int64_t* head_kept, int64_t* head_load,
                                                      int64_t capacity, int64_t tile_capacity,
                                                      int32_t* dev_status) {
  __shared__ int64_t sw[33];
  int64_t total_rows = -1;
  if (row_cnt) total_rows = block_exclusive_scan(row_cnt, row_ptr, rows, sw);
  const int64_t total_tiles = block_exclusive_scan(tile_cost, tile_ptr, tiles, sw);
  __syncthreads();
  for (int bh = threadIdx.x; bh < BH; bh += blockDim.x) {
    head_kept[bh] = static_cast<int64_t>(row_ptr[static_cast<int64_t>(bh + 1) * nB]) -
                    row_ptr[static_cast<int64_t>(bh) * nB];
    head_load[bh] = static_cast<int64_t>(tile_ptr[static_cast<int64_t>(bh + 1) * nPairs]) -
                    tile_ptr[static_cast<int64_t>(bh) * nPairs];
  }
  if (threadIdx.x == 0) {
    if (total_rows > capacity || total_tiles > tile_capacity) report(dev_status, FVA_DEVERR_MASK);
  }
}

// ---------------------------------------------------------------------------------
// Work list orders
// ---------------------------------------------------------------------------------
__global__ void order_natural_kernel(int32_t* worklist, int64_t tiles) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < tiles;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    worklist[i] = static_cast<int32_t>(i);
}

// rank(t) = #{t' : cost' > cost or (cost' == cost and t' < t)}; worklist[rank] = t
__global__ void __launch_bounds__(256) order_lpt_kernel(const int32_t* __restrict__ cost, int64_t tiles,
                                                        int32_t* worklist) {
  __shared__ int32_t sc[2048];
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int32_t ct = t < tiles ? cost[t] : 0;
  int64_t rank = 0;
  for (int64_t base = 0; base < tiles; base += 2048) {
    const int64_t n = tiles - base < 2048 ? tiles - base : 2048;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) sc[i] = cost[base + i];
    __syncthreads();
    if (t < tiles) {
      for (int i = 0; i < n; ++i) {
        const int32_t c = sc[i];
        rank += (c > ct) || (c == ct && base + i < t);
      }
    }
  }
  if (t < tiles) worklist[rank] = static_cast<int32_t>(t);
}

// One CTA per (b, h): heads ordered by load desc (index asc), tiles of a head by cost desc
// (index asc).
__global__ void __launch_bounds__(256) order_head_lpt_kernel(const int32_t* __restrict__ cost,
                                                             const int64_t* __restrict__ head_load, int BH,
                                                             int nPairs, int32_t* worklist) {
  extern __shared__ int32_t sc[];  // [nPairs]
  __shared__ int64_t head_rank;
  const int bh = blockIdx.x;
  if (threadIdx.x == 0) {
    const int64_t my = head_load[bh];
    int64_t r = 0;
    for (int j = 0; j < BH; ++j) {
      const int64_t l = head_load[j];
      r += (l > my) || (l == my && j < bh);
    }
    head_rank = r;
  }
  for (int i = threadIdx.x; i < nPairs; i += blockDim.x) sc[i] = cost[static_cast<int64_t>(bh) * nPairs + i];
  __syncthreads();
  for (int t = threadIdx.x; t < nPairs; t += blockDim.x) {
    const int32_t ct = sc[t];
    int r = 0;
    for (int i = 0; i < nPairs; ++i) {
      const int32_t c = sc[i];
      r += (c > ct) || (c == ct && i < t);
    }
    worklist[head_rank * nPairs + r] = bh * nPairs + t;
  }
}

// ---------------------------------------------------------------------------------
// Emission of col_idx and tile_col from the bitmasks
// ---------------------------------------------------------------------------------
// One warp per tile (query blocks 2t and 2t+1 of one (b, h)). The warp walks the two
// rows' bitmasks one 32-block word at a time; lane i owns block 32 k + i, and its output
// slot is the number of set bits below it, so every store instruction writes one
// contiguous run of entries.
__global__ void __launch_bounds__(256) emit_kernel(const uint32_t* __restrict__ bits, int nB, int nWords,
                                                   int nPairs, int64_t tiles, const int32_t* __restrict__ row_ptr,
                                                   const int32_t* __restrict__ tile_ptr, int32_t* col_idx,
                                                   int32_t* tile_col, int write_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t tile = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (tile >= tiles) return;
  const int64_t bh = tile / nPairs;
  const int t = static_cast<int>(tile - bh * nPairs);
  const int64_t rA = bh * nB + 2 * t;
  const bool hasB = 2 * t + 1 < nB;
  const int64_t rB = rA + 1;
  int32_t* outA = col_idx + row_ptr[rA];
  int32_t* outB = hasB ? col_idx + row_ptr[rB] : nullptr;
  int32_t* outT = tile_col + tile_ptr[tile];
  const uint32_t below = (1u << lane) - 1u;
  for (int k0 = 0; k0 < nWords; k0 += 32) {
    // lane q holds word k0 + q of both rows
    const uint32_t myA = k0 + lane < nWords ? bits[rA * nWords + k0 + lane] : 0u;
    const uint32_t myB = (hasB && k0 + lane < nWords) ? bits[rB * nWords + k0 + lane] : 0u;
    const int kn = nWords - k0 < 32 ? nWords - k0 : 32;
    for (int q = 0; q < kn; ++q) {
      const uint32_t wa = __shfl_sync(0xffffffffu, myA, q);
      const uint32_t wb = __shfl_sync(0xffffffffu, myB, q);
      const uint32_t wu = wa | wb;
      const int blk = 32 * (k0 + q) + lane;
      const uint32_t inA = (wa >> lane) & 1u, inB = (wb >> lane) & 1u;
      if (write_rows) {
        if (inA) outA[__popc(wa & below)] = blk;
        if (inB) outB[__popc(wb & below)] = blk;
        outA += __popc(wa);
        if (hasB) outB += __popc(wb);
      }
      if ((wu >> lane) & 1u)
        outT[__popc(wu & below)] = (blk << 2) | static_cast<int>(inA) | (static_cast<int>(inB) << 1);
      outT += __popc(wu);
    }
  }
}

// ---------------------------------------------------------------------------------
// Tiles from a caller-made CSR
// ---------------------------------------------------------------------------------
// One warp per row: the row's bitmask is built in shared memory (nWords words per warp),
// then written out in whole words.
__global__ void __launch_bounds__(256) csr_to_bits_kernel(const int32_t* __restrict__ row_ptr,
                                                          const int32_t* __restrict__ col_idx, int64_t rows,
                                                          int nB, int nWords, uint32_t* bits, int32_t* dev_status) {
  extern __shared__ uint32_t row_words[];  // [8][nWords]
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  uint32_t* w = row_words + (threadIdx.x >> 5) * nWords;
  for (int k = lane; k < nWords; k += 32) w[k] = 0u;
  __syncwarp();
  const int32_t lo = row_ptr[r], hi = row_ptr[r + 1];
  for (int32_t i = lo + lane; i < hi; i += 32) {
    const int32_t c = col_idx[i];
    if (c < 0 || c >= nB) {
      report(dev_status, FVA_DEVERR_BAD_LIST);
      continue;
    }
    atomicOr(&w[c >> 5], 1u << (c & 31));
  }
  __syncwarp();
  for (int k = lane; k < nWords; k += 32) bits[r * nWords + k] = w[k];
}

__global__ void __launch_bounds__(256) tile_cost_kernel(const uint32_t* __restrict__ bits, int nB, int nWords,
                                                        int nPairs, int64_t tiles, int32_t* tile_cost) {
  const int lane = threadIdx.x & 31;
  const int64_t tile = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (tile >= tiles) return;
  const int64_t bh = tile / nPairs;
  const int t = static_cast<int>(tile - bh * nPairs);
  const int64_t rA = bh * nB + 2 * t;
  const bool hasB = 2 * t + 1 < nB;
  int u = 0;
  for (int k = lane; k < nWords; k += 32)
    u += __popc(bits[rA * nWords + k] | (hasB ? bits[(rA + 1) * nWords + k] : 0u));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
  if (lane == 0) tile_cost[tile] = u;
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------
// Rows (warps) per CTA: the even count that fits the most warps on an SM (228 KB of shared
// memory, 1 KB of it reserved per CTA, at most 64 warps), fewer rows per CTA on a tie; 0 if
// not even two rows fit in one CTA's 227 KB.
static int select_rows_per_cta(const Dims& D) {
  const size_t arena = warp_arena_bytes(static_cast<int>(D.nB), static_cast<int>(D.nWords));
  constexpr size_t kCta = 227 * 1024, kSm = 228 * 1024, kReserved = 1024;
  int best = 0, best_warps = 0;
  for (int r = 2; r <= 16; r += 2) {
    const size_t smem = arena * r;
    if (smem > kCta) break;
    int ctas = static_cast<int>(kSm / (smem + kReserved));
    if (ctas * r > 64) ctas = 64 / r;
    if (ctas * r > best_warps) {
      best_warps = ctas * r;
      best = r;
    }
  }
  return best;
}

static cudaError_t launch_order_and_emit(const Dims& D, const fva_mask* m, int order, const RouteScratch& ws,
                                         int write_rows, cudaStream_t st) {
  if (order == FVA_ORDER_NATURAL) {
    int grid = static_cast<int>((D.tiles + 255) / 256);
    order_natural_kernel<<<grid, 256, 0, st>>>(m->worklist, D.tiles);
  } else if (order == FVA_ORDER_LPT) {
    order_lpt_kernel<<<static_cast<int>((D.tiles + 255) / 256), 256, 0, st>>>(m->tile_cost, D.tiles, m->worklist);
  } else {
    const size_t smem = static_cast<size_t>(D.nPairs) * 4;
    const cudaError_t ea = cudaFuncSetAttribute(order_head_lpt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(smem));
    if (ea != cudaSuccess) return ea;
    order_head_lpt_kernel<<<static_cast<int>(D.BH), 256, smem, st>>>(m->tile_cost, ws.head_load,
                                                                     static_cast<int>(D.BH),
                                                                     static_cast<int>(D.nPairs), m->worklist);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  emit_kernel<<<static_cast<int>((D.tiles + 7) / 8), 256, 0, st>>>(
      ws.bits, static_cast<int>(D.nB), static_cast<int>(D.nWords), static_cast<int>(D.nPairs), D.tiles,
      m->row_ptr, m->tile_ptr, m->col_idx, m->tile_col, write_rows);
  return cudaGetLastError();
}

cudaError_t launch_route(const Dims& D, const double* pq, const double* pk, double p, int k_floor, int order,
                         const fva_mask* m, const RouteScratch& ws, int32_t* dev_status, cudaStream_t st) {
  const int nB = static_cast<int>(D.nB);
  {
    cudaError_t e = launch_route_scores(D, pq, pk, ws.scores, st);
    if (e != cudaSuccess) return e;
  }
  {
    const int rpc = select_rows_per_cta(D);
    const size_t smem = warp_arena_bytes(nB, static_cast<int>(D.nWords)) * rpc;
    const cudaError_t ea = cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(smem));
    if (ea != cudaSuccess) return ea;
    const dim3 grid((nB + rpc - 1) / rpc, static_cast<unsigned>(D.BH));
    route_select_kernel<<<grid, 32 * rpc, smem, st>>>(ws.scores, nB, static_cast<int>(D.nWords),
                                                     static_cast<int>(D.nPairs), p, k_floor, ws.bits, ws.row_cnt,
                                                     m->tile_cost, dev_status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  finish_kernel<<<1, 1024, 0, st>>>(ws.row_cnt, D.rows, m->tile_cost, D.tiles, nB, static_cast<int>(D.nPairs),
                                    static_cast<int>(D.BH), m->row_ptr, m->tile_ptr, m->head_kept, ws.head_load,
                                    m->capacity, m->tile_capacity, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_order_and_emit(D, m, order, ws, 1, st);
}

cudaError_t launch_route_scores(const Dims& D, const double* pq, const double* pk, double* scores, cudaStream_t st) {
  const int nB = static_cast<int>(D.nB);
  const dim3 grid((nB + Scores::kBN - 1) / Scores::kBN, (nB + Scores::kBM - 1) / Scores::kBM,
                  static_cast<unsigned>(D.BH));
  cudaError_t e = cudaFuncSetAttribute(route_scores_kernel<Scores>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Scores::kSmem));
  if (e != cudaSuccess) return e;
  route_scores_kernel<Scores><<<grid, Scores::kThreads, Scores::kSmem, st>>>(pq, pk, scores, nB, static_cast<int>(D.d),
                                                                             sqrt(static_cast<double>(D.d)));
  return cudaGetLastError();
}

cudaError_t launch_csr_to_bits(const Dims& D, const fva_mask* m, uint32_t* bits, int32_t* dev_status,
                               cudaStream_t st) {
  const size_t smem = static_cast<size_t>(D.nWords) * 4 * 8;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(csr_to_bits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  csr_to_bits_kernel<<<static_cast<int>((D.rows + 7) / 8), 256, smem, st>>>(
      m->row_ptr, m->col_idx, D.rows, static_cast<int>(D.nB), static_cast<int>(D.nWords), bits, dev_status);
  return cudaGetLastError();
}

// From per-row bitmasks in ws.bits: tile costs, row_ptr (from row_cnt, or kept as given
// when row_cnt is null), tile_ptr, head_kept, the work list, then the lists themselves
// (col_idx too when write_rows).
cudaError_t launch_tiles_from_bits(const Dims& D, const fva_mask* m, int order, const RouteScratch& ws,
                                   const int32_t* row_cnt, int write_rows, int32_t* dev_status, cudaStream_t st) {
  tile_cost_kernel<<<static_cast<int>((D.tiles + 7) / 8), 256, 0, st>>>(
      ws.bits, static_cast<int>(D.nB), static_cast<int>(D.nWords), static_cast<int>(D.nPairs), D.tiles, m->tile_cost);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  finish_kernel<<<1, 1024, 0, st>>>(row_cnt, D.rows, m->tile_cost, D.tiles, static_cast<int>(D.nB),
                                    static_cast<int>(D.nPairs), static_cast<int>(D.BH), m->row_ptr, m->tile_ptr,
                                    m->head_kept, ws.head_load, m->capacity, m->tile_capacity, dev_status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_order_and_emit(D, m, order, ws, write_rows, st);
}

cudaError_t launch_build_tiles(const Dims& D, const fva_mask* m, int order, const RouteScratch& ws,
                               int32_t* dev_status, cudaStream_t st) {
  cudaError_t e = launch_csr_to_bits(D, m, ws.bits, dev_status, st);
  if (e != cudaSuccess) return e;
  return launch_tiles_from_bits(D, m, order, ws, nullptr, 0, dev_status, st);
}

bool route_shape_supported(const Dims& D) { return select_rows_per_cta(D) > 0; }

}  // namespace fva
