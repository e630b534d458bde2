// C ABI of libfva: argument validation, workspace carving and kernel dispatch.
// Every check that can be made on the host is made here, before anything is enqueued.
#include <math.h>
#include <string.h>

#include "fva_internal.cuh"

namespace fva {

bool route_shape_supported(const Dims& D);

bool make_dims(const fva_shape* s, Dims* out) {
  if (!s) return false;
  if (s->B < 1 || s->H < 1 || s->d < 1 || s->T < 1 || s->Hg < 1 || s->Wg < 1) return false;
  if (s->block != kBlock) return false;
  if (s->dtype != FVA_F32 && s->dtype != FVA_BF16) return false;
  Dims D;
  D.B = s->B;
  D.H = s->H;
  D.d = s->d;
  D.N = static_cast<int64_t>(s->T) * s->Hg * s->Wg;
  D.nB = (D.N + kBlock - 1) / kBlock;
  D.nPairs = (D.nB + 1) / 2;
  D.BH = D.B * D.H;
  D.rows = D.BH * D.nB;
  D.tiles = D.BH * D.nPairs;
  D.nWords = (D.nB + 31) / 32;
  D.esize = s->dtype == FVA_BF16 ? 2 : 4;
  if (D.N > 0x7fffffffLL || D.rows > 0x7fffffffLL) return false;
  const int64_t row_bytes = D.d * D.esize;
  if (row_bytes != 64 && row_bytes != 128 && row_bytes != 256 && row_bytes != 512 && row_bytes != 1024) return false;
  if (s->Hg > 65536 || s->Wg > 65536) return false;
  if (D.BH > 65535 || D.nB > 65535 * 8) return false;
  *out = D;
  return true;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? FVA_OK : FVA_ERR_CUDA; }

struct Carver {
  uint8_t* base;
  size_t off;
  template <typename T>
  T* take(size_t bytes) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = align_up(off + bytes, 256);
    return p;
  }
};

static size_t route_scratch_layout(const Dims& D, int need_pool, void* ws, RouteScratch* rs, double** pq,
                                   double** pk, bool with_scores) {
  Carver c{static_cast<uint8_t*>(ws), 0};
  RouteScratch r;
  r.scores = with_scores ? c.take<double>(static_cast<size_t>(D.BH * D.nB * D.nB) * 8) : nullptr;
  r.bits = c.take<uint32_t>(static_cast<size_t>(D.rows * D.nWords) * 4);
  r.row_cnt = c.take<int32_t>(static_cast<size_t>(D.rows) * 4);
  r.head_load = c.take<int64_t>(static_cast<size_t>(D.BH) * 8);
  double* q = nullptr;
  double* k = nullptr;
  if (need_pool) {
    q = c.take<double>(static_cast<size_t>(D.rows * D.d) * 8);
    k = c.take<double>(static_cast<size_t>(D.rows * D.d) * 8);
  }
  if (rs) *rs = r;
  if (pq) *pq = q;
  if (pk) *pk = k;
  return c.off;
}

}  // namespace fva

using namespace fva;

extern "C" {

const char* fva_status_string(int status) {
  switch (status) {
    case FVA_OK: return "ok";
    case FVA_ERR_INVALID_ARG: return "invalid argument";
    case FVA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or dtype";
    case FVA_ERR_CAPACITY: return "mask buffer capacity too small";
    case FVA_ERR_CUDA: return "CUDA error";
    case FVA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case FVA_ERR_WORKSPACE: return "workspace too small";
    case FVA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case FVA_ERR_TOO_LARGE: return "shape needs more scratch than the fixed no-alloc array holds";
    default: return "unknown status";
  }
}

int fva_version(void) { return 100; }

void fva_set_diagnostics(uint64_t wait_limit_ns, int flags) {
  set_attn_diagnostics(wait_limit_ns, static_cast<uint32_t>(flags));
}

int fva_set_cta_trace(int64_t* trace_dev, int64_t capacity_ctas) {
  if ((trace_dev == nullptr) != (capacity_ctas == 0) || capacity_ctas < 0) return FVA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(trace_dev) % 8 != 0) return FVA_ERR_ALIGNMENT;
  set_attn_cta_trace(trace_dev, capacity_ctas);
  return FVA_OK;
}

int64_t fva_num_tokens(const fva_shape* s) {
  Dims D;
  return make_dims(s, &D) ? D.N : -1;
}
int64_t fva_num_blocks(const fva_shape* s) {
  Dims D;
  return make_dims(s, &D) ? D.nB : -1;
}
int64_t fva_num_tiles(const fva_shape* s) {
  Dims D;
  return make_dims(s, &D) ? D.tiles : -1;
}
int64_t fva_mask_capacity(const fva_shape* s) {
  Dims D;
  return make_dims(s, &D) ? D.BH * D.nB * D.nB : -1;
}
int64_t fva_tile_capacity(const fva_shape* s) {
  Dims D;
  return make_dims(s, &D) ? D.BH * D.nPairs * D.nB : -1;
}

size_t fva_route_workspace_bytes(const fva_shape* s, int need_pool) {
  Dims D;
  if (!make_dims(s, &D) || !route_shape_supported(D)) return 0;
  return route_scratch_layout(D, need_pool, nullptr, nullptr, nullptr, nullptr, true);
}

size_t fva_tiles_workspace_bytes(const fva_shape* s) {
  Dims D;
  if (!make_dims(s, &D)) return 0;
  return route_scratch_layout(D, 0, nullptr, nullptr, nullptr, nullptr, false);
}

int fva_hilbert_perm(const fva_shape* s, int32_t* perm_dev, int32_t* inv_dev, fva_stream_t stream) {
  Dims D;
  if (!s || !perm_dev || !inv_dev) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  return cuda_status(launch_hilbert_perm(D, s->T, s->Hg, s->Wg, perm_dev, inv_dev, stream));
}

int fva_curve_perm(const fva_shape* s, int curve, int32_t* perm_dev, int32_t* inv_dev, int32_t* dev_status,
                   fva_stream_t stream) {
  Dims D;
  if (!s || !perm_dev || !inv_dev) return FVA_ERR_INVALID_ARG;
  if (curve != FVA_CURVE_HILBERT && curve != FVA_CURVE_RECT) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (curve == FVA_CURVE_HILBERT) return cuda_status(launch_hilbert_perm(D, s->T, s->Hg, s->Wg, perm_dev, inv_dev, stream));
  return cuda_status(launch_rect_curve_perm(D, s->Hg, s->Wg, perm_dev, inv_dev, dev_status, stream));
}

int fva_reorder(const fva_shape* s, const void* x_in_dev, void* x_out_dev, double* pooled_dev,
                const int32_t* perm_dev, int direction, fva_stream_t stream) {
  Dims D;
  if (!s || !x_in_dev || !x_out_dev || !perm_dev) return FVA_ERR_INVALID_ARG;
  if (direction != FVA_FWD && direction != FVA_INV && direction != FVA_FWD_F16) return FVA_ERR_INVALID_ARG;
  if (direction != FVA_FWD && pooled_dev) return FVA_ERR_INVALID_ARG;
  if (direction == FVA_FWD_F16 && s->dtype != FVA_BF16) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x_in_dev) || !aligned16(x_out_dev) || (pooled_dev && !aligned16(pooled_dev)))
    return FVA_ERR_ALIGNMENT;
  if (x_in_dev == x_out_dev) return FVA_ERR_INVALID_ARG;
  return cuda_status(launch_reorder(D, x_in_dev, x_out_dev, pooled_dev, perm_dev, direction, stream));
}

int fva_pool(const fva_shape* s, const void* x_bhnd_dev, double* pooled_dev, fva_stream_t stream) {
  Dims D;
  if (!s || !x_bhnd_dev || !pooled_dev) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x_bhnd_dev) || !aligned16(pooled_dev)) return FVA_ERR_ALIGNMENT;
  return cuda_status(launch_pool(D, x_bhnd_dev, pooled_dev, stream));
}

static int check_mask_outputs(const Dims& D, const fva_mask* m) {
  if (!m || !m->row_ptr || !m->col_idx || !m->head_kept || !m->tile_ptr || !m->tile_col || !m->tile_cost ||
      !m->worklist)
    return FVA_ERR_INVALID_ARG;
  if (m->capacity < D.BH * D.nB * D.nB || m->tile_capacity < D.BH * D.nPairs * D.nB) return FVA_ERR_CAPACITY;
  if (D.BH * D.nB * D.nB > 0x7fffffffLL) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (m->logits && !aligned16(m->logits)) return FVA_ERR_ALIGNMENT;
  return FVA_OK;
}

int fva_route(const fva_shape* s, const void* q_bhnd_dev, const void* k_bhnd_dev, const double* pooled_q_dev,
              const double* pooled_k_dev, double p, int k_floor, int order, const fva_mask* mask,
              void* workspace_dev, size_t workspace_bytes, int32_t* dev_status, fva_stream_t stream) {
  Dims D;
  if (!s) return FVA_ERR_INVALID_ARG;
  if (!(p > 0.0 && p <= 1.0)) return FVA_ERR_INVALID_ARG;
  if (k_floor < 0) return FVA_ERR_INVALID_ARG;
  if (order != FVA_ORDER_NATURAL && order != FVA_ORDER_LPT && order != FVA_ORDER_HEAD_LPT) return FVA_ERR_INVALID_ARG;
  const bool have_pooled = pooled_q_dev && pooled_k_dev;
  if ((pooled_q_dev == nullptr) != (pooled_k_dev == nullptr)) return FVA_ERR_INVALID_ARG;
  if (!have_pooled && (!q_bhnd_dev || !k_bhnd_dev)) return FVA_ERR_INVALID_ARG;
  if (!workspace_dev) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!route_shape_supported(D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_mask_outputs(D, mask);
  if (rc != FVA_OK) return rc;
  const int need_pool = have_pooled ? 0 : 1;
  if (workspace_bytes < route_scratch_layout(D, need_pool, nullptr, nullptr, nullptr, nullptr, true))
    return FVA_ERR_WORKSPACE;
  if (!aligned16(workspace_dev)) return FVA_ERR_ALIGNMENT;
  RouteScratch rs;
  double* pq = const_cast<double*>(pooled_q_dev);
  double* pk = const_cast<double*>(pooled_k_dev);
  double* wq = nullptr;
  double* wk = nullptr;
  route_scratch_layout(D, need_pool, workspace_dev, &rs, &wq, &wk, true);
  if (need_pool) {
    if (!aligned16(q_bhnd_dev) || !aligned16(k_bhnd_dev)) return FVA_ERR_ALIGNMENT;
    cudaError_t e = launch_pool(D, q_bhnd_dev, wq, stream);
    if (e == cudaSuccess) e = launch_pool(D, k_bhnd_dev, wk, stream);
    if (e != cudaSuccess) return FVA_ERR_CUDA;
    pq = wq;
    pk = wk;
  }
  if (mask->logits) rs.scores = mask->logits;  // the logits go to the caller's buffer
  return cuda_status(launch_route(D, pq, pk, p, k_floor, order, mask, rs, dev_status, stream));
}

int fva_copy_strided(void* dst, size_t dst_pitch_bytes, const void* src, size_t src_pitch_bytes, size_t width_bytes,
                     int64_t rows, fva_stream_t stream) {
  if (!dst || !src || rows < 0) return FVA_ERR_INVALID_ARG;
  if (width_bytes > dst_pitch_bytes || width_bytes > src_pitch_bytes) return FVA_ERR_INVALID_ARG;
  if (rows == 0 || width_bytes == 0) return FVA_OK;
  return cuda_status(cudaMemcpy2DAsync(dst, dst_pitch_bytes, src, src_pitch_bytes, width_bytes,
                                       static_cast<size_t>(rows), cudaMemcpyDefault, stream));
}

size_t fva_sasa_workspace_bytes(const fva_shape* s) {
  Dims D;
  if (!make_dims(s, &D) || !route_shape_supported(D)) return 0;
  return route_scratch_layout(D, 0, nullptr, nullptr, nullptr, nullptr, true) + sasa_extra_bytes(D);
}

int fva_sasa_augment(const fva_shape* s, const double* pooled_q_dev, const double* pooled_k_dev,
                     const int32_t* rank_of_head_dev, int n_ranks, const int64_t* budget_dev, int order,
                     const fva_mask* mask, void* workspace_dev, size_t workspace_bytes, int64_t* added_dev,
                     int32_t* dev_status, fva_stream_t stream) {
  Dims D;
  if (!s || !rank_of_head_dev || !budget_dev || !workspace_dev) return FVA_ERR_INVALID_ARG;
  if (!mask) return FVA_ERR_INVALID_ARG;
  if (!mask->logits && (!pooled_q_dev || !pooled_k_dev)) return FVA_ERR_INVALID_ARG;
  if (n_ranks < 1 || n_ranks > FVA_SASA_MAX_RANKS) return FVA_ERR_INVALID_ARG;
  if (order != FVA_ORDER_NATURAL && order != FVA_ORDER_LPT && order != FVA_ORDER_HEAD_LPT) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!route_shape_supported(D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_mask_outputs(D, mask);
  if (rc != FVA_OK) return rc;
  const size_t base = route_scratch_layout(D, 0, nullptr, nullptr, nullptr, nullptr, true);
  if (workspace_bytes < base + sasa_extra_bytes(D)) return FVA_ERR_WORKSPACE;
  if (!aligned16(workspace_dev)) return FVA_ERR_ALIGNMENT;
  if (!mask->logits && (!aligned16(pooled_q_dev) || !aligned16(pooled_k_dev))) return FVA_ERR_ALIGNMENT;
  RouteScratch rs;
  route_scratch_layout(D, 0, workspace_dev, &rs, nullptr, nullptr, true);
  return cuda_status(launch_sasa(D, pooled_q_dev, pooled_k_dev, rank_of_head_dev, n_ranks, budget_dev, order, mask,
                                 rs, static_cast<uint8_t*>(workspace_dev) + base, added_dev, dev_status, stream));
}

int fva_sasa_budgets(const double* rank_load_ms, int n_ranks, double block_ms, double n1, double n2,
                     int64_t* budget_out) {
  if (!rank_load_ms || !budget_out || n_ranks < 1) return FVA_ERR_INVALID_ARG;
  if (!(block_ms > 0.0) || !(n1 >= 0.0) || !(n2 >= 0.0)) return FVA_ERR_INVALID_ARG;
  double crit = 0.0;
  for (int r = 0; r < n_ranks; ++r) {
    if (!(rank_load_ms[r] >= 0.0) || isinf(rank_load_ms[r])) return FVA_ERR_INVALID_ARG;
    if (rank_load_ms[r] > crit) crit = rank_load_ms[r];
  }
  for (int r = 0; r < n_ranks; ++r) {
    const double slack = crit - rank_load_ms[r];
    budget_out[r] = (crit > 0.0 && slack >= n2 * crit) ? static_cast<int64_t>(floor(n1 * slack / block_ms)) : 0;
  }
  return FVA_OK;
}

int fva_build_tiles(const fva_shape* s, const fva_mask* mask, int order, void* workspace_dev, size_t workspace_bytes,
                    int32_t* dev_status, fva_stream_t stream) {
  Dims D;
  if (!s || !workspace_dev) return FVA_ERR_INVALID_ARG;
  if (order != FVA_ORDER_NATURAL && order != FVA_ORDER_LPT && order != FVA_ORDER_HEAD_LPT) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_mask_outputs(D, mask);
  if (rc != FVA_OK) return rc;
  if (workspace_bytes < route_scratch_layout(D, 0, nullptr, nullptr, nullptr, nullptr, false)) return FVA_ERR_WORKSPACE;
  if (!aligned16(workspace_dev)) return FVA_ERR_ALIGNMENT;
  if (D.nPairs * 4 > 200 * 1024) return FVA_ERR_UNSUPPORTED_SHAPE;
  RouteScratch rs;
  route_scratch_layout(D, 0, workspace_dev, &rs, nullptr, nullptr, false);
  return cuda_status(launch_build_tiles(D, mask, order, rs, dev_status, stream));
}

static int attn_common(const fva_shape* s, const void* q, const void* k, const void* v, int v_dtype,
                       const fva_mask* m, void* o, float scale, bool dense, int64_t first_slot, int64_t n_slots,
                       bool whole, int32_t* dev_status, fva_stream_t stream) {
  Dims D;
  if (!s || !q || !k || !v || !o) return FVA_ERR_INVALID_ARG;
  if (!make_dims(s, &D)) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FVA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v) return FVA_ERR_INVALID_ARG;
  if (whole) {
    first_slot = 0;
    n_slots = D.tiles;
  }
  if (first_slot < 0 || n_slots < 0 || first_slot + n_slots > D.tiles) return FVA_ERR_INVALID_ARG;
  if (!(scale > 0.0f)) scale = 1.0f / sqrtf(static_cast<float>(D.d));
  if (s->dtype == FVA_BF16) {
    if (v_dtype != FVA_BF16 && v_dtype != FVA_F16) return FVA_ERR_INVALID_ARG;
    if (D.d != 64 && D.d != 128) return FVA_ERR_UNSUPPORTED_SHAPE;
    if (!dense && (!m || !m->tile_ptr || !m->tile_col || !m->worklist)) return FVA_ERR_INVALID_ARG;
    if (!attn_cta_trace_fits(D.tiles)) return FVA_ERR_CAPACITY;
    return cuda_status(launch_attn_bf16(D, q, k, v, v_dtype == FVA_F16, m, dense, o, scale, first_slot, n_slots,
                                        dev_status, stream));
  }
  if (v_dtype != FVA_F32) return FVA_ERR_INVALID_ARG;
  if (D.d != 32 && D.d != 64 && D.d != 128) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (!whole) return FVA_ERR_UNSUPPORTED_SHAPE;  // the fp32 path reads the CSR, not the work list
  if (!dense && (!m || !m->row_ptr || !m->col_idx)) return FVA_ERR_INVALID_ARG;
  return cuda_status(launch_attn_f32(D, static_cast<const float*>(q), static_cast<const float*>(k),
                                     static_cast<const float*>(v), dense ? nullptr : m->row_ptr,
                                     dense ? nullptr : m->col_idx, dense, static_cast<float*>(o), scale, stream));
}

int fva_sparse_attn(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev, int v_dtype,
                    const fva_mask* mask, void* o_dev, float scale, int32_t* dev_status, fva_stream_t stream) {
  return attn_common(s, q_dev, k_dev, v_dev, v_dtype, mask, o_dev, scale, false, 0, 0, true, dev_status, stream);
}

int fva_sparse_attn_range(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev, int v_dtype,
                          const fva_mask* mask, void* o_dev, float scale, int64_t first_slot, int64_t n_slots,
                          int32_t* dev_status, fva_stream_t stream) {
  return attn_common(s, q_dev, k_dev, v_dev, v_dtype, mask, o_dev, scale, false, first_slot, n_slots, false,
                     dev_status, stream);
}

int fva_dense_attn(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev, int v_dtype,
                   void* o_dev, float scale, int32_t* dev_status, fva_stream_t stream) {
  return attn_common(s, q_dev, k_dev, v_dev, v_dtype, nullptr, o_dev, scale, true, 0, 0, true, dev_status, stream);
}

}  // extern "C"
