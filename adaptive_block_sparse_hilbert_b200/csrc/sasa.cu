// Slack-Aware Sparse Augmentation (SASA) of a routed block mask, and its budget rule.
//
// Method: aixai.ru FVAttn blog, section "Slack-Aware Sparse Augmentation (SASA)" -- ranks
// that wait for the critical path spend their slack on additional high-value blocks
// (augmentation coefficient n1 = 0.8, trigger threshold n2 = 0.07); section
// "Sparse-routing frontend" -- the routing pass provides the importance order of key
// blocks. PaperDaily article, 方法揭秘 -- from the blocks the mask skipped, the most
// important ones are added within each rank's idle-time budget.
//
// A rank's budget goes to the skipped (row, block) entries of its heads with the largest
// routing importance P_ab = softmax_b(s_ab), ties to the lower head, query block and key
// block. On the device:
//   1. the block logits (exported by the routing pass, or recomputed) give, for every
//      skipped entry, a 64-bit key that orders like P (the bits of the positive double P,
//      plus one; kept entries get 0);
//   2. an exact radix select fixes, 8 bits per pass from the top, the key tau_r of each
//      rank's budget-th largest entry (per-CTA shared histograms, one picking step per pass).
//      Once two digits are fixed, the entries that still match their rank's prefix are
//      copied into a compact list (key and row), and the remaining six passes and the tie
//      count read that list instead of every entry; when the list would not fit its
//      capacity they read every entry, with the same result;
//   3. entries equal to tau_r are shared out in (head, query block) order, lower key block
//      first within a row, to fill the budget exactly;
//   4. the new kept bitmask is old | key > tau_r | the allotted ties, and the tile lists,
//      row pointers and work list are rebuilt from it.
#include <math.h>

#include "fva_internal.cuh"

namespace fva {

namespace {

constexpr int kSasaBins = 256;
constexpr int kSasaMaxRanks = FVA_SASA_MAX_RANKS;

__device__ __forceinline__ int rank_of_row(const int32_t* rank_of, int64_t row, int nB, int R) {
  const int r = rank_of[row / nB];
  return (r >= 0 && r < R) ? r : -1;
}

// per row: row maximum, Z = sum exp(s - max), then one key per entry; counts candidates.
// `logits` and `keys_out` may be the same array (the keys then replace the logits: every
// lane writes only the entries it has just read, after the row's reductions). Rows of a
// rank without a budget are left alone: no later pass reads their keys.
__global__ void __launch_bounds__(256) sasa_keys_kernel(const double* logits, uint64_t* keys_out,
                                                        const uint32_t* __restrict__ bits, int64_t rows, int nB,
                                                        int nWords, const int32_t* __restrict__ rank_of, int R,
                                                        const int64_t* __restrict__ budget,
                                                        unsigned long long* total, int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const double* s = logits + r * nB;
  const int rk = rank_of_row(rank_of, r, nB, R);
  if (rk < 0 && lane == 0 && (r % nB) == 0) report(dev_status, FVA_DEVERR_BAD_LIST);
  if (rk >= 0 && budget[rk] <= 0) return;
  double mx = -INFINITY;
  for (int b = lane; b < nB; b += 32) mx = fmax(mx, s[b]);
  mx = warp_max_d(mx);
  double z = 0.0;
  for (int b = lane; b < nB; b += 32) z += exp(s[b] - mx);
  z = warp_sum_d(z);
  uint64_t* key = keys_out + r * nB;
  unsigned cnt = 0;
  for (int b = lane; b < nB; b += 32) {
    const bool kept = (bits[r * nWords + (b >> 5)] >> (b & 31)) & 1u;
    uint64_t k = 0;
    if (!kept && rk >= 0) {
      const double p = exp(s[b] - mx) / z;
      k = static_cast<uint64_t>(__double_as_longlong(p)) + 1ull;
      ++cnt;
    }
    key[b] = k;  // the same element this lane just read
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0 && rk >= 0 && cnt) atomicAdd(&total[rk], static_cast<unsigned long long>(cnt));
}

// need[r]: -1 = take every candidate; 0 = take none; > 0 = still to place by the select
__global__ void sasa_init_kernel(const int64_t* __restrict__ budget, int R, const unsigned long long* total,
                                 unsigned long long* prefix, unsigned long long* pmask, long long* need,
                                 int64_t* added) {
  const int r = threadIdx.x;
  if (r >= R) return;
  const long long b = budget[r] > 0 ? budget[r] : 0;
  const long long t = static_cast<long long>(total[r]);
  prefix[r] = 0;
  pmask[r] = 0;
  need[r] = b == 0 ? 0 : (t <= b ? -1 : b);
  if (added) added[r] = b < t ? b : t;
}

// The entries (key, row) of selecting ranks that match their rank's prefix after two
// digits. `count` keeps counting past `capacity`, so a list that did not fit is known.
struct CompactList {
  uint64_t* keys;
  int64_t* rows;
  unsigned long long* count;
  unsigned long long capacity;
  __device__ bool holds_all() const { return count != nullptr && *count <= capacity; }
};

__global__ void __launch_bounds__(512) sasa_compact_kernel(const uint64_t* __restrict__ keys, int64_t rows, int nB,
                                                           const int32_t* __restrict__ rank_of, int R,
                                                           const unsigned long long* __restrict__ prefix,
                                                           const unsigned long long* __restrict__ pmask,
                                                           const long long* __restrict__ need, CompactList cl) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int rk = rank_of_row(rank_of, r, nB, R);
    if (rk < 0 || need[rk] <= 0) continue;
    const uint64_t pf = prefix[rk], pm = pmask[rk];
    const uint64_t* k = keys + r * nB;
    for (int b0 = 0; b0 < nB; b0 += 32) {
      const int b = b0 + lane;
      const uint64_t v = b < nB ? k[b] : 0ull;
      const bool in = v != 0 && (v & pm) == pf;
      const unsigned m = __ballot_sync(0xffffffffu, in);
      if (m == 0) continue;
      unsigned long long base = 0;
      if (lane == 0) base = atomicAdd(cl.count, static_cast<unsigned long long>(__popc(m)));
      base = __shfl_sync(0xffffffffu, base, 0);
      const unsigned long long j = base + __popc(m & ((1u << lane) - 1u));
      if (in && j < cl.capacity) {
        cl.keys[j] = v;
        cl.rows[j] = r;
      }
    }
  }
}

// histogram of the next 8-bit digit of the keys that match their rank's prefix
// (reads the compact list instead of every entry when `cl` is given and holds them all)
__global__ void __launch_bounds__(512) sasa_hist_kernel(const uint64_t* __restrict__ keys, int64_t rows, int nB,
                                                        const int32_t* __restrict__ rank_of, int R,
                                                        const unsigned long long* __restrict__ prefix,
                                                        const unsigned long long* __restrict__ pmask,
                                                        const long long* __restrict__ need, int shift,
                                                        unsigned* hist, CompactList cl) {
  extern __shared__ unsigned sh[];
  for (int i = threadIdx.x; i < R * kSasaBins; i += blockDim.x) sh[i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  if (cl.holds_all()) {
    const int64_t n = static_cast<int64_t>(*cl.count);
    for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < n;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const uint64_t v = cl.keys[j];
      const int rk = rank_of_row(rank_of, cl.rows[j], nB, R);
      if (rk >= 0 && need[rk] > 0 && (v & pmask[rk]) == prefix[rk])
        atomicAdd(&sh[rk * kSasaBins + static_cast<int>((v >> shift) & 255u)], 1u);
    }
  } else {
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
      const int rk = rank_of_row(rank_of, r, nB, R);
      if (rk < 0 || need[rk] <= 0) continue;
      const uint64_t pf = prefix[rk], pm = pmask[rk];
      const uint64_t* k = keys + r * nB;
      for (int b = lane; b < nB; b += 32) {
        const uint64_t v = k[b];
        if (v != 0 && (v & pm) == pf) atomicAdd(&sh[rk * kSasaBins + static_cast<int>((v >> shift) & 255u)], 1u);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < R * kSasaBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&hist[i], sh[i]);
}

// one warp per rank: the digit where the count from the top reaches `need`. Lane l holds
// bins 8l .. 8l+7; a suffix sum over the lanes above gives each lane the count of the
// digits above its bins, and the lane whose bins hold the crossing picks it.
__global__ void __launch_bounds__(32) sasa_pick_kernel(unsigned* hist, int R, int shift, unsigned long long* prefix,
                                                       unsigned long long* pmask, long long* need,
                                                       int32_t* dev_status) {
  const int r = blockIdx.x;
  const int lane = threadIdx.x;
  if (r >= R) return;
  unsigned* h = hist + r * kSasaBins;
  unsigned c[8];
  long long mine = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    c[q] = h[8 * lane + q];
    mine += c[q];
  }
  const long long nd = need[r];
  if (nd > 0) {
    long long above = mine;  // inclusive suffix sum: bins 8 lane .. 255
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_down_sync(0xffffffffu, above, o);
      if (lane + o < 32) above += t;
    }
    above -= mine;  // bins above this lane's eight
    int d = -1;
    long long before = 0;
    if (above < nd && above + mine >= nd) {
      long long run = above;
      for (int q = 7; q >= 0; --q) {
        if (run + c[q] >= nd) {
          d = 8 * lane + q;
          before = run;
          break;
        }
        run += c[q];
      }
    }
    const unsigned who = __ballot_sync(0xffffffffu, d >= 0);
    if (who == 0) {  // fewer matching entries than needed: cannot happen when counts are right
      if (lane == 0) {
        report(dev_status, FVA_DEVERR_MASK);
        need[r] = 0;
      }
    } else if (lane == __ffs(who) - 1) {
      prefix[r] |= static_cast<unsigned long long>(d) << shift;
      pmask[r] |= 255ull << shift;
      need[r] = nd - before;
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) h[8 * lane + q] = 0u;
}

// entries equal to tau_r per row (tie candidates)
// (every entry is read only when the compact list does not hold them all; tie_take starts
// at zero)
__global__ void __launch_bounds__(256) sasa_ties_count_kernel(const uint64_t* __restrict__ keys, int64_t rows,
                                                              int nB, const int32_t* __restrict__ rank_of, int R,
                                                              const unsigned long long* __restrict__ prefix,
                                                              const long long* __restrict__ need, int32_t* tie_take,
                                                              CompactList cl) {
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows || cl.holds_all()) return;
  const int rk = rank_of_row(rank_of, r, nB, R);
  int n = 0;
  if (rk >= 0 && need[rk] > 0) {
    const uint64_t tau = prefix[rk];
    for (int b = lane; b < nB; b += 32) n += keys[r * nB + b] == tau ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0) tie_take[r] = n;
}

// the same counts from the compact list, when it holds every candidate (ties match the
// prefix, so all of them are in it)
__global__ void __launch_bounds__(512) sasa_ties_compact_kernel(int nB, const int32_t* __restrict__ rank_of, int R,
                                                                const unsigned long long* __restrict__ prefix,
                                                                const long long* __restrict__ need, int32_t* tie_take,
                                                                CompactList cl) {
  if (!cl.holds_all()) return;
  const int64_t n = static_cast<int64_t>(*cl.count);
  for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = cl.rows[j];
    const int rk = rank_of_row(rank_of, row, nB, R);
    if (rk >= 0 && need[rk] > 0 && cl.keys[j] == prefix[rk]) atomicAdd(&tie_take[row], 1);
  }
}

// rows in (head, query block) order take the ties each rank still needs. Ties are rare:
// each thread flags whether its contiguous chunk of rows holds any, and one thread then
// walks only the flagged chunks, in row order.
__global__ void __launch_bounds__(1024) sasa_ties_alloc_kernel(int64_t rows, int nB,
                                                               const int32_t* __restrict__ rank_of, int R,
                                                               const long long* __restrict__ need, int32_t* tie_take) {
  __shared__ int has[1024];
  __shared__ long long left[kSasaMaxRanks];
  const int64_t chunk = (rows + blockDim.x - 1) / blockDim.x;
  has[threadIdx.x] = 0;
  if (threadIdx.x < R) left[threadIdx.x] = need[threadIdx.x] > 0 ? need[threadIdx.x] : 0;
  __syncthreads();
  for (int64_t row = threadIdx.x; row < rows; row += blockDim.x)  // coalesced
    if (tie_take[row] != 0) has[row / chunk] = 1;
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int c = 0; c < static_cast<int>(blockDim.x); ++c) {
    if (!has[c]) continue;
    const int64_t clo = c * chunk;
    const int64_t chi = clo + chunk < rows ? clo + chunk : rows;
    for (int64_t row = clo; row < chi; ++row) {
      const int n = tie_take[row];
      if (n == 0) continue;
      const int rk = rank_of_row(rank_of, row, nB, R);
      const long long t = rk < 0 ? 0 : (left[rk] < n ? left[rk] : n);
      if (rk >= 0) left[rk] -= t;
      tie_take[row] = static_cast<int32_t>(t);
    }
  }
}

// new kept bitmask and kept count per row
__global__ void __launch_bounds__(256) sasa_bits_kernel(const uint64_t* __restrict__ keys, int64_t rows, int nB,
                                                        int nWords, const int32_t* __restrict__ rank_of, int R,
                                                        const unsigned long long* __restrict__ prefix,
                                                        const unsigned long long* __restrict__ pmask,
                                                        const long long* __restrict__ need,
                                                        const int32_t* __restrict__ tie_take, uint32_t* bits,
                                                        int32_t* row_cnt) {
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int rk = rank_of_row(rank_of, r, nB, R);
  const bool all = rk >= 0 && need[rk] < 0;
  const bool thr = rk >= 0 && pmask[rk] != 0;
  if (!all && !thr) {  // nothing added to this row: count its kept blocks, keys unread
    int kept = 0;
    for (int k = lane; k < nWords; k += 32) kept += __popc(bits[r * nWords + k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
    if (lane == 0) row_cnt[r] = kept;
    return;
  }
  const uint64_t tau = thr ? prefix[rk] : ~0ull;
  const int ties = tie_take[r];
  int tie_seen = 0, kept = 0;
  for (int k = 0; k < nWords; ++k) {
    const int b = 32 * k + lane;
    const uint64_t v = b < nB ? keys[r * nB + b] : 0ull;
    const bool eq = thr && v != 0 && v == tau;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const int my_tie = tie_seen + __popc(eqm & ((1u << lane) - 1u));
    tie_seen += __popc(eqm);
    const bool add = v != 0 && (all || (thr && (v > tau || (eq && my_tie < ties))));
    const unsigned w = bits[r * nWords + k] | __ballot_sync(0xffffffffu, add);
    if (lane == 0) bits[r * nWords + k] = w;
    kept += __popc(w);
  }
  if (lane == 0) row_cnt[r] = kept;
}

}  // namespace

// compact list capacity: a sixteenth of all entries (at least 256)
static size_t sasa_compact_capacity(const Dims& D) {
  const size_t c = (static_cast<size_t>(D.rows) * static_cast<size_t>(D.nB) + 15) / 16;
  return c < 256 ? 256 : c;
}

size_t sasa_extra_bytes(const Dims& D) {
  return align_up(static_cast<size_t>(D.rows) * 4, 256) + align_up(kSasaMaxRanks * kSasaBins * 4, 256) +
         4 * align_up(kSasaMaxRanks * 8, 256) + align_up(8, 256) + align_up(sasa_compact_capacity(D) * 8, 256) * 2;
}

cudaError_t launch_sasa(const Dims& D, const double* pq, const double* pk, const int32_t* rank_of, int R,
                        const int64_t* budget, int order, const fva_mask* m, const RouteScratch& ws, uint8_t* extra,
                        int64_t* added, int32_t* dev_status, cudaStream_t st) {
  int32_t* tie_take = reinterpret_cast<int32_t*>(extra);
  size_t off = align_up(static_cast<size_t>(D.rows) * 4, 256);
  unsigned* hist = reinterpret_cast<unsigned*>(extra + off);
  off += align_up(kSasaMaxRanks * kSasaBins * 4, 256);
  unsigned long long* total = reinterpret_cast<unsigned long long*>(extra + off);
  off += align_up(kSasaMaxRanks * 8, 256);
  unsigned long long* prefix = reinterpret_cast<unsigned long long*>(extra + off);
  off += align_up(kSasaMaxRanks * 8, 256);
  unsigned long long* pmask = reinterpret_cast<unsigned long long*>(extra + off);
  off += align_up(kSasaMaxRanks * 8, 256);
  long long* need = reinterpret_cast<long long*>(extra + off);
  off += align_up(kSasaMaxRanks * 8, 256);
  CompactList cl;
  cl.count = reinterpret_cast<unsigned long long*>(extra + off);
  off += align_up(8, 256);
  cl.capacity = sasa_compact_capacity(D);
  cl.keys = reinterpret_cast<uint64_t*>(extra + off);
  off += align_up(cl.capacity * 8, 256);
  cl.rows = reinterpret_cast<int64_t*>(extra + off);
  CompactList full = cl;  // the same list, not used yet: passes read every entry
  full.count = nullptr;

  const int nB = static_cast<int>(D.nB), nWords = static_cast<int>(D.nWords);
  const unsigned row_grid = static_cast<unsigned>((D.rows + 7) / 8);
  cudaError_t e = cudaMemsetAsync(hist, 0, kSasaMaxRanks * kSasaBins * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(total, 0, kSasaMaxRanks * 8, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(cl.count, 0, 8, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(tie_take, 0, static_cast<size_t>(D.rows) * 4, st);
  // the block logits: exported by the routing pass (mask->logits), else recomputed
  const double* logits = m->logits;
  if (!logits && e == cudaSuccess) {
    e = launch_route_scores(D, pq, pk, ws.scores, st);
    logits = ws.scores;
  }
  if (e == cudaSuccess) e = launch_csr_to_bits(D, m, ws.bits, dev_status, st);
  if (e != cudaSuccess) return e;
  sasa_keys_kernel<<<row_grid, 256, 0, st>>>(logits, reinterpret_cast<uint64_t*>(ws.scores), ws.bits, D.rows, nB,
                                             nWords, rank_of, R, budget, total, dev_status);
  sasa_init_kernel<<<1, kSasaMaxRanks, 0, st>>>(budget, R, total, prefix, pmask, need, added);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint64_t* keys = reinterpret_cast<const uint64_t*>(ws.scores);
  const size_t hist_smem = static_cast<size_t>(R) * kSasaBins * 4;
  if (hist_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(sasa_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(hist_smem));
    if (e != cudaSuccess) return e;
  }
  for (int shift = 56; shift >= 0; shift -= 8) {
    sasa_hist_kernel<<<148 * 4, 512, hist_smem, st>>>(keys, D.rows, nB, rank_of, R, prefix, pmask, need, shift, hist,
                                                      shift < 48 ? cl : full);
    sasa_pick_kernel<<<R, 32, 0, st>>>(hist, R, shift, prefix, pmask, need, dev_status);
    if (shift == 48)
      sasa_compact_kernel<<<148 * 4, 512, 0, st>>>(keys, D.rows, nB, rank_of, R, prefix, pmask, need, cl);
  }
  sasa_ties_count_kernel<<<row_grid, 256, 0, st>>>(keys, D.rows, nB, rank_of, R, prefix, need, tie_take, cl);
  sasa_ties_compact_kernel<<<148 * 4, 512, 0, st>>>(nB, rank_of, R, prefix, need, tie_take, cl);
  sasa_ties_alloc_kernel<<<1, 1024, 0, st>>>(D.rows, nB, rank_of, R, need, tie_take);
  sasa_bits_kernel<<<row_grid, 256, 0, st>>>(keys, D.rows, nB, nWords, rank_of, R, prefix, pmask, need, tie_take,
                                              ws.bits, ws.row_cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_tiles_from_bits(D, m, order, ws, ws.row_cnt, 1, dev_status, st);
}

}  // namespace fva
