// Block-sparse (and dense) flash-style forward attention on sm_100a tensor cores.
//
// Method: aixai.ru FVAttn blog, sparse-attention section -- attention is computed only
// over the key blocks the router kept for a query block; the dense case (every block
// kept) is the FlashAttention-style baseline the pages compare against.
//
// Design (B200):
//   * One CTA per tile = two Hilbert-adjacent query blocks (128 query rows) of one
//     (b, h). It walks the union of the two rows' kept key-block lists; each list entry
//     carries which of the two query blocks keeps it, and the other half's scores are
//     masked to -inf. A 128-row tile never costs more tensor time than two 64-row
//     (M=64, half-rate) tiles, and Hilbert-adjacent blocks share most of their lists.
//   * Warp roles: warp 4 issues TMA tile loads (Q once, then K and V blocks of 64 keys
//     into a ring of stages), warp 5 issues tcgen05.mma (one thread), warps 0-3 own one
//     query row per thread (TMEM lane) for the online softmax and the epilogue.
//   * S = Q K^T (M=128, N=64, K=d, bf16 -> fp32) goes to one of two TMEM buffers (three at
//     d = 64, where the QK product runs two steps ahead of P V); the softmax warps read
//     it, write P back over it as packed fp16 (bf16 in the bf16-V variant) and the MMA
//     warp issues O += P V with P taken straight from TMEM (A operand) and V from shared
//     memory (B operand, MN-major). O stays in TMEM until the epilogue.
//   * O is rescaled only when a row maximum grows by more than 2^8 (log2 units), so
//     the exponentials stay <= 256 and the TMEM read-modify-write of O is rare.
//   * Two CTAs per SM (<= 256 TMEM columns and ~97 KB smem each): while one CTA runs
//     its softmax, the other keeps the tensor core busy.
//   * CTA i runs the tile at work-list position first_slot + i (longest first); the
//     hardware block scheduler hands each free CTA slot the next CTA, i.e. greedy list
//     scheduling, as long as it dispatches in blockIdx order (the per-CTA trace shows
//     that it does). A work-list entry that names no tile is reported, not followed.
//   * Every mbarrier wait is bounded (~2 s); on expiry the CTA reports
//     FVA_DEVERR_TIMEOUT, drains its own TMA loads and MMAs, frees TMEM and exits.
#include <math.h>

#include "fva_internal.cuh"

namespace fva {

constexpr int kAttnThreads = 192;
constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 64;   // keys per step (one key block)
constexpr uint32_t kTmemCols = 256;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

// Bounded wait taken by a whole warp: the result is the same on every lane, so the
// warp stays converged for the .sync.aligned TMEM instructions that follow.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
struct AttnCfg {
  static constexpr int kChunks = D / 64;                    // 128-byte swizzle rows per d
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kQBytes = kChunks * kBM * 128;        // 128 rows x 128 B per chunk
  static constexpr int kKVBytes = kChunks * kBN * 128;       // 64 rows x 128 B per chunk
  static constexpr int kSmemData = kQBytes + 2 * kStages * kKVBytes;
  // S buffers of 64 TMEM columns each, then O: two buffers at d = 128 (2 x 64 + 128 = 256
  // columns), three at d = 64 (3 x 64 + 64 = 256), so at d = 64 the QK product runs two
  // steps ahead of P.V and S(j + 3), not S(j + 2), is the one that waits for P(j)
  static constexpr int kSBufs = (D == 128) ? 2 : 3;
  static constexpr uint32_t kOCol = kSBufs * 64;             // O columns [kOCol, kOCol + D)
};

template <int D>
struct __align__(8) AttnBars {
  uint64_t q_full;
  uint64_t k_full[AttnCfg<D>::kStages];
  uint64_t k_empty[AttnCfg<D>::kStages];
  uint64_t v_full[AttnCfg<D>::kStages];
  uint64_t v_empty[AttnCfg<D>::kStages];
  uint64_t s_full[AttnCfg<D>::kSBufs];
  uint64_t p_full[AttnCfg<D>::kSBufs];
  // one per S buffer: P.V of step i completes pv_done[i % kSBufs], so a wait for step j - 1
  // never sees more than one phase of ambiguity (S(j) arriving implies every P.V of a step
  // <= j - kSBufs is complete)
  uint64_t pv_done[AttnCfg<D>::kSBufs];
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr size_t attn_smem_bytes() {
  return 1024 /*alignment slack*/ + AttnCfg<D>::kSmemData + sizeof(AttnBars<D>);
}

// VF16: V and P in fp16 for P.V (else both bf16); Q and K are bf16 either way.
template <int D, bool DENSE, bool VF16>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, __nv_bfloat16* __restrict__ out,
                     const int32_t* __restrict__ tile_ptr, const int32_t* __restrict__ tile_col,
                     const int32_t* __restrict__ worklist, int slot0, int ntiles, int N, int nB, int nPairs, float scale_log2,
                     uint64_t kWaitLimitNs, uint32_t diag_flags, int32_t* dev_status, int64_t* cta_trace) {
  using Cfg = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + Cfg::kQBytes;
  uint8_t* sV = sK + Cfg::kStages * Cfg::kKVBytes;
  AttnBars<D>& bar = *reinterpret_cast<AttnBars<D>*>(smem + Cfg::kSmemData);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = static_cast<int>(blockIdx.x) + slot0;  // position in the work list
  int tile = DENSE ? static_cast<int>(blockIdx.x) : worklist[slot];
  // a work-list entry that names no tile is reported; its CTA then runs an empty list on
  // tile 0 and writes nothing
  const bool tile_ok = DENSE || (tile >= 0 && tile < ntiles);
  if (!tile_ok) {
    if (threadIdx.x == 0) report(dev_status, FVA_DEVERR_BAD_LIST);
    tile = 0;
  }
  const int bh = tile / nPairs;
  const int t = tile - bh * nPairs;
  int n_iter, list_base;
  if (DENSE) {
    n_iter = nB;
    list_base = 0;
  } else if (!tile_ok) {
    n_iter = 0;
    list_base = 0;
  } else {
    list_base = tile_ptr[tile];
    n_iter = tile_ptr[tile + 1] - list_base;
  }

  const uint64_t t_start = cta_trace != nullptr && threadIdx.x == 0 ? global_timer_ns() : 0;
  if (threadIdx.x == 128) {
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int i = 0; i < Cfg::kSBufs; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_full[i], 128);
      mbar_init(&bar.pv_done[i], 1);
    }
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.drain, 1);
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  volatile int* abort_flag = &bar.abort;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_q = 0;
      int k_uses[Cfg::kStages], v_uses[Cfg::kStages];
      for (int s = 0; s < Cfg::kStages; ++s) k_uses[s] = v_uses[s] = 0;
      bool ok = true;
      // FVA_DIAG_WITHHOLD_Q: the Q tile is never requested, so every wait behind it runs out
      if (!(diag_flags & FVA_DIAG_WITHHOLD_Q)) {
        mbar_arrive_expect_tx(&bar.q_full, Cfg::kQBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sQ + c * (kBM * 128) + hf * (64 * 128), &tmq, &bar.q_full, c * 64, t * kBM + hf * 64, bh);
        last_q = 1;
      }
      // K runs kStages blocks ahead of V: the MMA warp needs K(j+1) before V(j), and a K
      // stage is free as soon as its QK product has run, long before the V stage of the
      // same step (whose PV waits for the softmax)
      auto key_block = [&](int j, int* kb) -> bool {
        *kb = DENSE ? j : (tile_col[list_base + j] >> 2);
        if (*kb < 0 || *kb >= nB) {
          report(dev_status, FVA_DEVERR_BAD_LIST);
          *abort_flag = 1;
          return false;
        }
        return true;
      };
      auto load_k = [&](int j) -> bool {
        int kb;
        if (!key_block(j, &kb)) return false;
        const int s = j % Cfg::kStages;
        const uint32_t use = static_cast<uint32_t>(j / Cfg::kStages);
        if (j >= Cfg::kStages && !mbar_wait(&bar.k_empty[s], (use - 1) & 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          return false;
        }
        mbar_arrive_expect_tx(&bar.k_full[s], Cfg::kKVBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_3d(sK + s * Cfg::kKVBytes + c * (kBN * 128), &tmk, &bar.k_full[s], c * 64, kb * kBN, bh);
        ++k_uses[s];
        return true;
      };
      auto load_v = [&](int j) -> bool {
        int kb;
        if (!key_block(j, &kb)) return false;
        const int s = j % Cfg::kStages;
        const uint32_t use = static_cast<uint32_t>(j / Cfg::kStages);
        if (j >= Cfg::kStages && !mbar_wait(&bar.v_empty[s], (use - 1) & 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          return false;
        }
        mbar_arrive_expect_tx(&bar.v_full[s], Cfg::kKVBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_3d(sV + s * Cfg::kKVBytes + c * (kBN * 128), &tmv, &bar.v_full[s], c * 64, kb * kBN, bh);
        ++v_uses[s];
        return true;
      };
      bool go = true;
      for (int j = 0; j < Cfg::kStages && j < n_iter && go; ++j) go = load_k(j);
      for (int j = 0; j < n_iter && go; ++j) {
        go = load_v(j);
        if (go && j + Cfg::kStages < n_iter) go = load_k(j + Cfg::kStages);
      }
      if (!ok) {
        report(dev_status, FVA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the last load issued into every buffer
        volatile int never = 0;
        if (last_q) mbar_wait(&bar.q_full, 0, &never, 100000000ull);
        for (int s = 0; s < Cfg::kStages; ++s) {
          if (k_uses[s] > 0) mbar_wait(&bar.k_full[s], (k_uses[s] - 1) & 1, &never, 100000000ull);
          if (v_uses[s] > 0) mbar_wait(&bar.v_full[s], (v_uses[s] - 1) & 1, &never, 100000000ull);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16kind_f32(kBM, kBN, 0, 0, kFmtBF16);
      constexpr uint32_t idesc_pv = idesc_f16kind_f32(kBM, D, 0, 1, VF16 ? kFmtF16 : kFmtBF16);
      bool ok = mbar_wait(&bar.q_full, 0, abort_flag, kWaitLimitNs);
      bool issued = false;
      constexpr int kLag = Cfg::kSBufs - 1;  // P.V of step j - kLag follows the QK of step j
      auto issue_pv = [&](int i) -> bool {
        const int sb = i % Cfg::kSBufs;
        const int s = i % Cfg::kStages;
        if (!mbar_wait(&bar.p_full[sb], (i / Cfg::kSBufs) & 1, abort_flag, kWaitLimitNs)) return false;
        if (!mbar_wait(&bar.v_full[s], (i / Cfg::kStages) & 1, abort_flag, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sV + s * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(v_base + kk * 2048, kBN * 128, 1024);
          mma_ts(tmem + Cfg::kOCol, tmem + sb * 64 + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar.v_empty[s]);
        tc_commit(&bar.pv_done[sb]);
        return true;
      };
      if (ok) tc_fence_after();
      for (int j = 0; j < n_iter && ok; ++j) {
        const int s = j % Cfg::kStages;
        const int sb = j % Cfg::kSBufs;
        if (!mbar_wait(&bar.k_full[s], (j / Cfg::kStages) & 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ);
        const uint32_t k_base = smem_u32(sK + s * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2;
          const uint32_t ko = (kk & 3) * 32;
          const uint64_t adesc = sdesc_sw128(q_base + c * (kBM * 128) + ko, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(k_base + c * (kBN * 128) + ko, 16, 1024);
          mma_ss(tmem + sb * 64, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        issued = true;
        tc_commit(&bar.k_empty[s]);
        tc_commit(&bar.s_full[sb]);
        if (j >= kLag && !issue_pv(j - kLag)) {
          ok = false;
          break;
        }
      }
      for (int i = n_iter > kLag ? n_iter - kLag : 0; i < n_iter && ok; ++i) ok = issue_pv(i);
      if (ok) {
        tc_commit(&bar.o_full);
      } else {
        report(dev_status, FVA_DEVERR_TIMEOUT);
        *abort_flag = 1;
        if (issued) {
          // drain every MMA issued so far before TMEM is freed
          volatile int never = 0;
          tc_commit(&bar.drain);
          mbar_wait(&bar.drain, 0, &never, 100000000ull);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int half = warp >> 1;
    float m_ref = -INFINITY;
    float l_sum = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_iter; ++j) {
      const int entry = DENSE ? ((j << 2) | 3) : tile_col[list_base + j];
      const int kb = entry >> 2;
      const bool keep = (entry >> half) & 1;
      const int sb = j % Cfg::kSBufs;
      if (!warp_wait(&bar.s_full[sb], (j / Cfg::kSBufs) & 1, abort_flag, kWaitLimitNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t pk[32];
      if (keep) {
        uint32_t r[64];
        tmem_ld64(lane_base + sb * 64, r);
        if (kb == nB - 1) {  // ragged last key block: keys past N score -inf
          const int nvalid = N - kb * kBN;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= nvalid) r[c] = 0xFF800000u;
        }
        // row maximum of the raw scores: four independent chains, seeded with r[0..7], then
        // three-input maxima over r[8..63]
        float mx4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mx4[q] = fmaxf(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
#pragma unroll
        for (int c = 8; c < 64; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mx4[q] = fmax3(mx4[q], __uint_as_float(r[c + 2 * q]), __uint_as_float(r[c + 2 * q + 1]));
        }
        const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * scale_log2;
        const float m_new = fmaxf(m_ref, mx);
        const bool need = m_new > m_ref + 8.0f;
        const bool need_o = need && (l_sum > 0.0f);
        if (__any_sync(0xffffffffu, need_o)) {
          // O holds rows rescaled to the old maximum: wait for the PV of step j-1, then
          // O_row *= 2^(m_ref - m_new) for the rows whose maximum moved.
          if (!warp_wait(&bar.pv_done[(j - 1) % Cfg::kSBufs], ((j - 1) / Cfg::kSBufs) & 1, abort_flag,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need_o ? ex2_approx(m_ref - m_new) : 1.0f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(lane_base + Cfg::kOCol + cc * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(lane_base + Cfg::kOCol + cc * 32, o);
          }
        }
        if (need) {
          l_sum *= ex2_approx(m_ref - m_new);
          m_ref = m_new;
        }
        // p = 2^(s * scale * log2 e - m_ref) on pairs of scores: one packed FFMA and two
        // MUFU.EX2; the row sum runs in two packed accumulators
        const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
        const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])),
                                            sc2, nm2));
          const uint64_t p2 = f2_pack(ex2_approx(x.x), ex2_approx(x.y));
          const float2 p = f2_unpack(p2);
          pk[c] = VF16 ? pack_f16x2(p.x, p.y) : pack_bf16x2(p.x, p.y);
          acc2[c & 1] = f2_add(acc2[c & 1], p2);
        }
        const float2 la = f2_unpack(f2_add(acc2[0], acc2[1]));
        l_sum += la.x + la.y;
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      tmem_st32(lane_base + sb * 64, pk);
      tc_fence_before();
      mbar_arrive(&bar.p_full[sb]);
    }
    // ------------------------------------------------------------------ epilogue
    if (ok && !warp_wait(&bar.o_full, 0, abort_flag, kWaitLimitNs)) ok = false;
    if (!ok) {
      report(dev_status, FVA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      const float inv_l = l_sum > 0.0f ? 1.0f / l_sum : 0.0f;
      const int grow = t * kBM + row;
      const bool valid = grow < N && n_iter > 0;
      uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(bh) * N + grow) * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(lane_base + Cfg::kOCol + cc * 32, o);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[cc * 4 + q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      if (n_iter == 0 && grow < N && tile_ok) {
        for (int q = 0; q < D / 8; ++q) dst[q] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (cta_trace != nullptr && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    int64_t* rec = cta_trace + 4 * static_cast<int64_t>(DENSE ? static_cast<int>(blockIdx.x) : slot);
    rec[0] = smid;
    rec[1] = n_iter;
    rec[2] = static_cast<int64_t>(t_start);
    rec[3] = static_cast<int64_t>(global_timer_ns());
  }
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------
static uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;
static uint32_t g_diag_flags = 0;
static int64_t* g_cta_trace = nullptr;
static int64_t g_cta_trace_capacity = 0;
void set_attn_cta_trace(int64_t* trace, int64_t capacity_ctas) {
  g_cta_trace = trace;
  g_cta_trace_capacity = capacity_ctas;
}
bool attn_cta_trace_fits(int64_t ctas) { return g_cta_trace == nullptr || g_cta_trace_capacity >= ctas; }
uint64_t attn_wait_limit_ns() { return g_wait_limit_ns; }
uint32_t attn_diag_flags() { return g_diag_flags; }
void set_attn_diagnostics(uint64_t ns, uint32_t flags) {
  g_wait_limit_ns = ns == 0 ? kDefaultWaitLimitNs : ns;
  g_diag_flags = flags;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over a [B*H, N, d] 16-bit tensor, box = 64 elements (128 B) x 64 rows x 1.
static bool make_map(CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t d, bool f16) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(N * d * 2)};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool DENSE, bool VF16>
static cudaError_t launch_attn_t(const Dims& Dm, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                 const fva_mask* m, void* o, float scale_log2, int first_slot, int n_slots,
                                 int32_t* dev_status, cudaStream_t st) {
  const size_t smem = attn_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<D, DENSE, VF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(DENSE ? Dm.tiles : n_slots);
  if (grid == 0) return cudaSuccess;
  attn_bf16_kernel<D, DENSE, VF16><<<grid, kAttnThreads, smem, st>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), DENSE ? nullptr : m->tile_ptr, DENSE ? nullptr : m->tile_col,
      DENSE ? nullptr : m->worklist, DENSE ? 0 : first_slot, static_cast<int>(Dm.tiles), static_cast<int>(Dm.N), static_cast<int>(Dm.nB), static_cast<int>(Dm.nPairs),
      scale_log2, attn_wait_limit_ns(), attn_diag_flags(), dev_status, g_cta_trace);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_attn_d(const Dims& Dm, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                 bool v_f16, const fva_mask* m, bool dense, void* o, float scale_log2, int first_slot,
                                 int n_slots, int32_t* dev_status, cudaStream_t st) {
  if (v_f16) {
    return dense ? launch_attn_t<D, true, true>(Dm, mq, mk, mv, m, o, scale_log2, 0, 0, dev_status, st)
                 : launch_attn_t<D, false, true>(Dm, mq, mk, mv, m, o, scale_log2, first_slot, n_slots, dev_status, st);
  }
  return dense ? launch_attn_t<D, true, false>(Dm, mq, mk, mv, m, o, scale_log2, 0, 0, dev_status, st)
               : launch_attn_t<D, false, false>(Dm, mq, mk, mv, m, o, scale_log2, first_slot, n_slots, dev_status, st);
}

cudaError_t launch_attn_bf16(const Dims& Dm, const void* q, const void* k, const void* v, bool v_f16,
                             const fva_mask* m, bool dense, void* o, float scale, int64_t first_slot, int64_t n_slots,
                             int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, Dm.BH, Dm.N, Dm.d, false) || !make_map(&mk, k, Dm.BH, Dm.N, Dm.d, false) ||
      !make_map(&mv, v, Dm.BH, Dm.N, Dm.d, v_f16))
    return cudaErrorInvalidValue;
  const float scale_log2 = scale * 1.4426950408889634f;
  const int fs = static_cast<int>(first_slot), ns = static_cast<int>(n_slots);
  if (Dm.d == 128) return launch_attn_d<128>(Dm, mq, mk, mv, v_f16, m, dense, o, scale_log2, fs, ns, dev_status, st);
  return launch_attn_d<64>(Dm, mq, mk, mv, v_f16, m, dense, o, scale_log2, fs, ns, dev_status, st);
}

}  // namespace fva
