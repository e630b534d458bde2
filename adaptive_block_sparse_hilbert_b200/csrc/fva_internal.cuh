// Internal helpers of libfva: shape arithmetic, launch checks and thin inline-PTX
// wrappers for the sm_100a features the kernels use (mbarrier, TMA tile loads,
// tcgen05 MMA / TMEM). Nothing here is exported.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fva.h"

namespace fva {

constexpr int kBlock = 64;

struct Dims {
  int64_t B, H, d, N, nB, nPairs, BH, rows, tiles, nWords;
  int esize;
};

// Returns false for shapes no entry point accepts.
bool make_dims(const fva_shape* s, Dims* out);

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------------
// kernel launchers (defined in their .cu files); each returns a cudaError_t
// ---------------------------------------------------------------------------------
cudaError_t launch_hilbert_perm(const Dims& D, int T, int Hg, int Wg, int32_t* perm, int32_t* inv,
                                cudaStream_t st);
cudaError_t launch_rect_curve_perm(const Dims& D, int Hg, int Wg, int32_t* perm, int32_t* inv,
                                   int32_t* dev_status, cudaStream_t st);
cudaError_t launch_reorder(const Dims& D, const void* x_in, void* x_out, double* pooled,
                           const int32_t* perm, int direction, cudaStream_t st);
cudaError_t launch_pool(const Dims& D, const void* x_bhnd, double* pooled, cudaStream_t st);

struct RouteScratch {
  double* scores;     // [BH, nB, nB]
  uint32_t* bits;     // [BH*nB, nWords]
  int32_t* row_cnt;   // [BH*nB]
  int64_t* head_load; // [BH] total tile cost per (b, h)
};
cudaError_t launch_route(const Dims& D, const double* pq, const double* pk, double p, int k_floor,
                         int order, const fva_mask* m, const RouteScratch& ws, int32_t* dev_status,
                         cudaStream_t st);
cudaError_t launch_build_tiles(const Dims& D, const fva_mask* m, int order, const RouteScratch& ws,
                               int32_t* dev_status, cudaStream_t st);
size_t sasa_extra_bytes(const Dims& D);
cudaError_t launch_sasa(const Dims& D, const double* pq, const double* pk, const int32_t* rank_of, int R,
                        const int64_t* budget, int order, const fva_mask* m, const RouteScratch& ws, uint8_t* extra,
                        int64_t* added, int32_t* dev_status, cudaStream_t st);
cudaError_t launch_route_scores(const Dims& D, const double* pq, const double* pk, double* scores, cudaStream_t st);
cudaError_t launch_csr_to_bits(const Dims& D, const fva_mask* m, uint32_t* bits, int32_t* dev_status,
                               cudaStream_t st);
cudaError_t launch_tiles_from_bits(const Dims& D, const fva_mask* m, int order, const RouteScratch& ws,
                                   const int32_t* row_cnt, int write_rows, int32_t* dev_status, cudaStream_t st);

// Sparse: the CTAs of work-list slots [first_slot, first_slot + n_slots); dense: every tile.
cudaError_t launch_attn_bf16(const Dims& D, const void* q, const void* k, const void* v, bool v_f16,
                             const fva_mask* m, bool dense, void* o, float scale, int64_t first_slot,
                             int64_t n_slots, int32_t* dev_status, cudaStream_t st);
uint64_t attn_wait_limit_ns();
uint32_t attn_diag_flags();
void set_attn_diagnostics(uint64_t wait_limit_ns, uint32_t flags);
void set_attn_cta_trace(int64_t* trace, int64_t capacity_ctas);
bool attn_cta_trace_fits(int64_t ctas);
cudaError_t launch_attn_f32(const Dims& D, const float* q, const float* k, const float* v,
                            const int32_t* row_ptr, const int32_t* col_idx, bool dense, float* o,
                            float scale, cudaStream_t st);

// ---------------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report(int32_t* dev_status, int code) {
  if (dev_status) atomicCAS(dev_status, 0, code);
}

// ---- mbarrier ------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true once the phase with this parity has completed; false if `abort`
// became nonzero or about `limit_ns` passed (the caller then reports and unwinds). Each
// try_wait may suspend the thread for a hardware-chosen time, so the clock is read after
// every attempt.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// ---- TMA (tile mode, no multicast) ------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ---- tcgen05 ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once all tcgen05.mma issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (sm_100 format:
// start>>4 in bits 0-13, leading byte offset>>4 in 16-29, stride byte offset>>4 in
// 32-45, descriptor version 1 in bits 46-47, base offset 0, layout type 2 =
// SWIZZLE_128B in bits 61-63). Tiles are 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  desc |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  desc |= static_cast<uint64_t>(1) << 46;
  desc |= static_cast<uint64_t>(2) << 61;
  return desc;
}

// Instruction descriptor, kind::f16 with an fp32 accumulator: c_format bits 4-5 = 1
// (F32); a_format 7-9 and b_format 10-12 = ab_format (0 = F16, 1 = BF16; A and B always
// share it); a_major bit 15, b_major bit 16 (1 = MN-major); N>>3 in bits 17-22; M>>4 in
// bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16kind_f32(int M, int N, int a_mn_major, int b_mn_major,
                                                         uint32_t ab_format) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t kFmtF16 = 0, kFmtBF16 = 1;

#define FVA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                  "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FVA_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                  "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// Load 32 consecutive 32-bit TMEM columns of this thread's lane and wait for them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FVA_R8(0), FVA_R8(8), FVA_R8(16), FVA_R8(24)
      : "r"(taddr)
      : "memory");
}
// Load 64 consecutive 32-bit TMEM columns of this thread's lane and wait for them.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FVA_R8(0), FVA_R8(8), FVA_R8(16), FVA_R8(24), FVA_R8(32), FVA_R8(40), FVA_R8(48), FVA_R8(56)
      : "r"(taddr)
      : "memory");
}
// Store 32 consecutive 32-bit TMEM columns of this thread's lane and wait for the store.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      FVA_W8(0), FVA_W8(8), FVA_W8(16), FVA_W8(24)
      : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16x2 / f16x2 packs: `lo` goes to the low 16 bits (element k), `hi` to the high
// (element k+1).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t v;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(v) : "f"(hi), "f"(lo));
  return v;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t v;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(v) : "f"(hi), "f"(lo));
  return v;
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) ------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


// Warp reductions with a fixed butterfly order (deterministic).
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_min_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace fva
