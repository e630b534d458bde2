/*
 * fva.h -- C ABI of libfva: Hilbert-ordered block routing and block-sparse attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operations follow the FVAttn pages (arXiv 2607.16190):
 *   [aixai] aixai.ru FVAttn blog -- "Sparse-routing frontend", "Top-p vs Top-k",
 *           "Runtime Load Balancing (RLB)", sparse-attention section;
 *   [PD]    longzhangge.com PaperDaily FVAttn article -- 方法揭秘 (method), 龙迷三问 (Q&A);
 *   [abs]   mlsanity.com "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing
 *           for Video Generation" -- abstract.
 *
 * Conventions (all entry points):
 *   - Every function returns an int status: FVA_OK (0) or a negative FVA_ERR_* code.
 *     fva_status_string() gives its text. No exception crosses the ABI.
 *   - The caller owns all memory. Pointers named *_dev are device pointers (cudaMalloc /
 *     torch CUDA tensors), 16-byte aligned unless stated otherwise. The library allocates
 *     no device memory; scratch space is passed in as a caller-owned workspace.
 *   - Work is enqueued asynchronously on the given stream (NULL = legacy default
 *     stream); outputs are valid after the stream is synchronised.
 *   - Host-detectable errors (null pointers, unsupported shapes, capacity or workspace
 *     too small, p outside (0, 1], negative k_floor) return before anything is
 *     enqueued. Errors found on the device (a bounded wait that ran out, an
 *     inconsistent mask) are written to the optional caller-provided int32 dev_status
 *     (device memory, expected to hold 0 on entry; set to a nonzero FVA_DEVERR_* code)
 *     and leave the device usable.
 *   - Layouts: x_bnhd = [B, N, H, d] raster token order (n = t*Hg*Wg + y*Wg + x);
 *     x_bhnd = [B, H, N, d] Hilbert order; pooled = [B, H, nB, d] float64.
 *   - Sizes: N = T*Hg*Wg, block = 64, nB = ceil(N / 64), nPairs = ceil(nB / 2);
 *     a "row" is one (b, h, query block a), r = (b*H + h)*nB + a; a "tile" is a pair
 *     of adjacent query blocks (2t, 2t+1) of one (b, h), id = (b*H + h)*nPairs + t.
 */
#ifndef FVA_H_
#define FVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FVA_API __attribute__((visibility("default")))
#else
#define FVA_API
#endif

typedef struct CUstream_st* fva_stream_t; /* identical to cudaStream_t */

enum {
  FVA_OK = 0,
  FVA_ERR_INVALID_ARG = -1,       /* null pointer, bad enum, p or k_floor out of range */
  FVA_ERR_UNSUPPORTED_SHAPE = -2, /* shape/dtype combination the library does not handle */
  FVA_ERR_CAPACITY = -3,          /* mask buffers smaller than fva_mask_capacity() etc. */
  FVA_ERR_CUDA = -4,              /* a CUDA runtime/driver call failed */
  FVA_ERR_DEVICE_TIMEOUT = -5,    /* reported through dev_status only */
  FVA_ERR_WORKSPACE = -6,         /* workspace smaller than the query function says */
  FVA_ERR_ALIGNMENT = -7,         /* a device pointer is not 16-byte aligned */
  FVA_ERR_TOO_LARGE = -8          /* the shape needs more scratch than fva_route_noalloc holds */
};

/* Codes written to dev_status by kernels. */
enum {
  FVA_DEVERR_NONE = 0,
  FVA_DEVERR_TIMEOUT = 1,   /* an mbarrier wait in the attention kernel ran out (~2 s) */
  FVA_DEVERR_MASK = 2,      /* a routed row's kept count disagreed with max(L_p, L_k) */
  FVA_DEVERR_BAD_LIST = 3   /* a tile list entry was out of range */
};

/* Element types. FVA_F16 appears only as the type of a Hilbert-ordered V (see
 * FVA_FWD_F16 and the v_dtype argument of the attention entry points). */
enum { FVA_F32 = 0, FVA_BF16 = 1, FVA_F16 = 2 };
/* Reorder directions: forward, inverse, forward with the output converted bf16 -> fp16. */
enum { FVA_FWD = 0, FVA_INV = 1, FVA_FWD_F16 = 2 };
/* Order of the attention work list (tiles are launched in this order). */
enum {
  FVA_ORDER_NATURAL = 0,    /* tile id order */
  FVA_ORDER_LPT = 1,        /* longest first over all tiles (cost desc, id asc) */
  FVA_ORDER_HEAD_LPT = 2    /* heads by total cost desc (id asc), longest first inside a head */
};

/* Problem shape. block must be 64. dtype is FVA_F32 or FVA_BF16.
 * Limits (a shape outside them gives FVA_ERR_UNSUPPORTED_SHAPE, or -1 / 0 from the size
 * queries, before anything is enqueued):
 *   B, H, d, T, Hg, Wg >= 1 (an empty layer is rejected, not treated as a no-op);
 *   Hg, Wg <= 65536; N = T*Hg*Wg <= 2^31 - 1; nB <= 524280; B*H <= 65535;
 *   B*H*nB <= 2^31 - 1;
 *   d * sizeof(dtype) in {64, 128, 256, 512, 1024} bytes;
 *   routing (fva_route, fva_route_noalloc, fva_sasa_augment): nB <= 11326, the largest
 *   count for which two rows' float64 working sets fit one CTA's 227 KB of shared
 *   memory, and B*H*nB*nB <= 2^31 - 1 (int32 CSR offsets);
 *   attention: see fva_sparse_attn. */
typedef struct fva_shape {
  int32_t B, H, d;
  int32_t T, Hg, Wg;
  int32_t block;
  int32_t dtype;
} fva_shape;

/* Block mask in CSR form plus the tile-level lists the attention kernel reads.
 * All pointers are device pointers owned by the caller.
 *   row_ptr   int32 [B*H*nB + 1]       CSR offsets over rows r
 *   col_idx   int32 [capacity]         kept key blocks of each row, ascending
 *   head_kept int64 [B*H]              kept (query block, key block) pairs per head:
 *                                      the head's load L_h ([aixai] RLB section)
 *   tile_ptr  int32 [B*H*nPairs + 1]   offsets into tile_col
 *   tile_col  int32 [tile_capacity]    union of the two rows' lists, ascending; entry =
 *                                      key_block*4 | (row 2t keeps it) | (row 2t+1 keeps it)<<1
 *   tile_cost int32 [B*H*nPairs]       number of entries of each tile (its work)
 *   worklist  int32 [B*H*nPairs]       tile ids in launch order (see FVA_ORDER_*)
 *   logits    float64 [B*H, nB, nB]    OPTIONAL (NULL: not used). When set, fva_route writes
 *                                      every row's block logits s_ab here: the importance
 *                                      order of the row's key blocks (larger logit first,
 *                                      lower block on ties) and, through the row softmax,
 *                                      their importances. fva_sasa_augment then reads them
 *                                      instead of recomputing them ([aixai] "Sparse-routing
 *                                      frontend": the one routing pass yields both the
 *                                      per-head density and the importance order that the
 *                                      augmentation uses). 16-byte aligned.
 */
typedef struct fva_mask {
  int32_t* row_ptr;
  int32_t* col_idx;
  int64_t capacity;
  int64_t* head_kept;
  int32_t* tile_ptr;
  int32_t* tile_col;
  int64_t tile_capacity;
  int32_t* tile_cost;
  int32_t* worklist;
  double* logits;
} fva_mask;

FVA_API const char* fva_status_string(int status);
FVA_API int fva_version(void);

/* Diagnostics of the attention kernels (process-wide; for failure-detection tests).
 * wait_limit_ns: time limit of every mbarrier wait (default 2 s; 0 restores it). A wait
 *   that runs out sets FVA_DEVERR_TIMEOUT in dev_status, and its CTA drains its own loads
 *   and MMAs, frees TMEM and exits; the device stays usable.
 * flags: FVA_DIAG_WITHHOLD_Q makes each CTA skip its Q tile load, so the waits behind it
 *   can never complete and run out after wait_limit_ns (a wait on a flag nothing sets).
 * fva_set_diagnostics(0, 0) restores normal operation. */
enum { FVA_DIAG_WITHHOLD_Q = 1 };
FVA_API void fva_set_diagnostics(uint64_t wait_limit_ns, int flags);

/*
 * Per-CTA trace of the attention kernels (measurement aid; the pages have no
 * counterpart). While set, every bf16 fva_sparse_attn / fva_dense_attn launch (the
 * tensor-core kernel; fp32 inputs are not traced) has each CTA write four int64 at
 * trace_dev[4 * c ..] for CTA (tile launch slot) c:
 *   [0] the SM it ran on (%smid), [1] its list length in 64-key blocks,
 *   [2] %globaltimer (ns) when it started, [3] %globaltimer when it finished.
 * trace_dev: device memory owned by the caller, capacity_ctas * 4 int64, 8-byte aligned;
 * slot c of a sparse launch is the c-th tile of the work list. A launch with more CTAs
 * than capacity_ctas fails with FVA_ERR_CAPACITY before launching.
 * fva_set_cta_trace(NULL, 0) turns tracing off (the default). Process-wide setting; not
 * thread-safe against concurrent launches. Returns FVA_OK or FVA_ERR_INVALID_ARG. */
FVA_API int fva_set_cta_trace(int64_t* trace_dev, int64_t capacity_ctas);

/* Derived sizes; -1 for an invalid shape. */
FVA_API int64_t fva_num_tokens(const fva_shape* s);
FVA_API int64_t fva_num_blocks(const fva_shape* s);
FVA_API int64_t fva_num_tiles(const fva_shape* s);
/* Entries col_idx / tile_col must hold: B*H*nB*nB and B*H*nPairs*nB. */
FVA_API int64_t fva_mask_capacity(const fva_shape* s);
FVA_API int64_t fva_tile_capacity(const fva_shape* s);
/* Bytes of workspace fva_route needs (with need_pool != 0: also room to pool Q and K);
 * 0 when the shape is outside the routing limits above. */
FVA_API size_t fva_route_workspace_bytes(const fva_shape* s, int need_pool);

/*
 * Hilbert token order ("video-aware block organization": [aixai] "Sparse-routing
 * frontend"; [PD] 方法揭秘). Per frame, the cells (y, x) are visited in the order of the
 * 2-D Hilbert curve on the enclosing 2^m x 2^m square (m = ceil(log2(max(Hg, Wg))),
 * out-of-grid cells skipped, first step (0,0) -> (x=0, y=1)); frames follow in t order.
 * perm_dev[i] = raster index of the token at Hilbert position i; inv_dev = perm^-1.
 * Both int32 [N], device memory.
 */
FVA_API int fva_hilbert_perm(const fva_shape* s, int32_t* perm_dev, int32_t* inv_dev, fva_stream_t stream);

/*
 * Token order by a chosen curve. FVA_CURVE_HILBERT is fva_hilbert_perm's order.
 * FVA_CURVE_RECT is a variant the pages leave open: a generalized Hilbert curve laid over
 * the Hg x Wg frame itself (J. Cerveny's construction: rectangles cut along the long side
 * into two halves, or across it into three parts, halves rounded to even lengths), which
 * keeps every step between grid neighbours where the plain curve on the enclosing 2^m
 * square jumps over skipped cells; on 2^m x 2^m frames the two orders are equal. The
 * curve starts at (x, y) = (0, 0) and runs first along the longer side. perm_dev / inv_dev
 * as for fva_hilbert_perm; dev_status (optional) receives FVA_DEVERR_MASK if the walk
 * fails its own consistency checks. Returns FVA_OK, FVA_ERR_INVALID_ARG (unknown curve),
 * FVA_ERR_UNSUPPORTED_SHAPE or FVA_ERR_CUDA.
 */
enum { FVA_CURVE_HILBERT = 0, FVA_CURVE_RECT = 1 };
FVA_API int fva_curve_perm(const fva_shape* s, int curve, int32_t* perm_dev, int32_t* inv_dev, int32_t* dev_status,
                           fva_stream_t stream);

/*
 * Token reorder with fused block mean-pooling ([aixai] "Sparse-routing frontend"; [PD]
 * 方法揭秘: block importance from pooled Q/K).
 *   FVA_FWD: x_out[b, h, i, :] = x_in[b, perm[i], h, :]   ([B,N,H,d] -> [B,H,N,d]);
 *            if pooled_dev != NULL also pooled[b, h, a, :] = mean of x_out rows
 *            [64a, min(64a+64, N)) in float64 (exact sum of the inputs, then / n_a).
 *   FVA_INV: x_out[b, perm[i], h, :] = x_in[b, h, i, :]   ([B,H,N,d] -> [B,N,H,d]);
 *            pooled_dev must be NULL.
 *   FVA_FWD_F16: as FVA_FWD for a bf16 input, with x_out written as float16 (exact for
 *            |x| < 65504, saturated to +-65504 beyond); pooled_dev must be NULL. This is
 *            how V is prepared for the fp16 P.V path of the attention kernel.
 * Element type from s->dtype; d * sizeof(elem) must be 64, 128, 256, 512 or 1024 bytes.
 * x_in and x_out must not overlap.
 */
FVA_API int fva_reorder(const fva_shape* s, const void* x_in_dev, void* x_out_dev, double* pooled_dev,
                const int32_t* perm_dev, int direction, fva_stream_t stream);

/* Block mean-pool of an already Hilbert-ordered [B,H,N,d] tensor into float64 [B,H,nB,d]. */
FVA_API int fva_pool(const fva_shape* s, const void* x_bhnd_dev, double* pooled_dev, fva_stream_t stream);

/*
 * Top-p routing with a Top-k safety floor ([aixai] "Top-p vs Top-k", "Sparse-routing
 * frontend"; [PD] 方法揭秘, 龙迷三问). For every row (b, h, a):
 *   s_ab = pooled_q[a] . pooled_k[b] / sqrt(d)          (float64)
 *   P_ab = softmax_b(s_ab)                              (float64)
 *   order key blocks by s descending, ties to the lower block index;
 *   L_p  = length of the shortest prefix whose cumulative P reaches p (p = 1: all);
 *   L    = max(L_p, min(k_floor, nB));  the first L blocks of the order are kept.
 * Cumulative masses are summed exactly in 2^-52 fixed point, so a row's decision can
 * differ from an exact float64 evaluation only when a cumulative mass lies within
 * ~nB*2^-52 of p.
 * Inputs: either pooled_q_dev/pooled_k_dev (float64 [B,H,nB,d], e.g. from fva_reorder)
 * or, when both are NULL, q_bhnd_dev/k_bhnd_dev (Hilbert-ordered, pooled here into the
 * workspace; needs fva_route_workspace_bytes(s, 1)).
 * Outputs: every array of *mask (row_ptr, col_idx, head_kept, tile_ptr, tile_col,
 * tile_cost, worklist), and mask->logits when it is not NULL (the block logits, which
 * otherwise stay in the workspace); mask->capacity >= fva_mask_capacity(s) and
 * mask->tile_capacity >= fva_tile_capacity(s) are required. order is a FVA_ORDER_*.
 * 0 < p <= 1, k_floor >= 0.
 */
FVA_API int fva_route(const fva_shape* s, const void* q_bhnd_dev, const void* k_bhnd_dev,
              const double* pooled_q_dev, const double* pooled_k_dev, double p, int k_floor,
              int order, const fva_mask* mask, void* workspace_dev, size_t workspace_bytes,
              int32_t* dev_status, fva_stream_t stream);

/* Bytes of workspace fva_build_tiles needs. */
FVA_API size_t fva_tiles_workspace_bytes(const fva_shape* s);

/*
 * Tile lists for a caller-made row-level CSR mask (mask->row_ptr / col_idx filled, each
 * row ascending, unique, in [0, nB)). Fills tile_ptr, tile_col, tile_cost, worklist and
 * head_kept the same way fva_route does.
 */
FVA_API int fva_build_tiles(const fva_shape* s, const fva_mask* mask, int order, void* workspace_dev,
                    size_t workspace_bytes, int32_t* dev_status, fva_stream_t stream);

/*
 * Block-sparse attention ([aixai] sparse-attention section: only the kept key blocks of
 * a query block are computed). For each query i in block a of (b, h):
 *   o_i = sum_j softmax_j(scale * q_i . k_j) v_j  over the valid keys j of the kept blocks
 * (no causal mask). q, k, o: [B,H,N,d] Hilbert order, dtype s->dtype; v: [B,H,N,d] of
 * type v_dtype.
 *   s->dtype == FVA_BF16 (tensor cores, d in {64, 128}, fp32 accumulation, bf16 output):
 *     v_dtype == FVA_F16: P is rounded to fp16 for P.V (the accurate path; prepare V
 *                         with fva_reorder(FVA_FWD_F16));
 *     v_dtype == FVA_BF16: P is rounded to bf16 for P.V.
 *   s->dtype == FVA_F32 (CUDA cores, d in {32, 64, 128}): v_dtype must be FVA_F32.
 * scale <= 0 selects 1/sqrt(d). Reads mask->tile_ptr, tile_col, worklist (bf16) or
 * mask->row_ptr, col_idx (fp32). o must not overlap q, k or v. A work-list entry that names
 * no tile, or a tile-list entry naming a key block out of range, sets FVA_DEVERR_BAD_LIST in
 * dev_status; that CTA writes no output rows (bf16 path).
 * A row that keeps no key block (possible only in a caller-made mask: fva_route keeps at
 * least one block per row) has an empty softmax; its output rows are written as zeros.
 */
FVA_API int fva_sparse_attn(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev,
                            int v_dtype, const fva_mask* mask, void* o_dev, float scale, int32_t* dev_status,
                            fva_stream_t stream);

/*
 * Part of a sparse attention launch: the tiles at work-list positions
 * [first_slot, first_slot + n_slots) of mask->worklist (bf16 inputs only; fp32 inputs give
 * FVA_ERR_UNSUPPORTED_SHAPE). Output rows of the other tiles are left untouched, so
 * consecutive ranges that together cover the list give fva_sparse_attn's result; a range
 * may also leave tiles out (with FVA_ORDER_HEAD_LPT a head's tiles are consecutive in the
 * list, so a head that another GPU computes can be skipped: [aixai] "Runtime Load
 * Balancing (RLB)", migration of a heavy head to a less loaded rank).
 * 0 <= first_slot, 0 <= n_slots, first_slot + n_slots <= fva_num_tiles(s), else
 * FVA_ERR_INVALID_ARG; n_slots == 0 enqueues nothing. Other arguments as fva_sparse_attn.
 */
FVA_API int fva_sparse_attn_range(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev,
                                  int v_dtype, const fva_mask* mask, void* o_dev, float scale, int64_t first_slot,
                                  int64_t n_slots, int32_t* dev_status, fva_stream_t stream);

/* Dense attention (every block kept): the in-house density-1 reference. Same layouts. */
FVA_API int fva_dense_attn(const fva_shape* s, const void* q_dev, const void* k_dev, const void* v_dev,
                           int v_dtype, void* o_dev, float scale, int32_t* dev_status, fva_stream_t stream);

/*
 * Routing without a caller-provided workspace. The pages have no counterpart of this
 * entry point; it exists for callers that cannot allocate device memory: a plugin inside
 * a host application whose allocator owns all device memory, a service that forbids
 * allocation after start-up to keep its footprint fixed, or any caller that holds only
 * its input and output buffers.
 * Same arguments and results as fva_route minus the workspace: the scratch lives in one
 * fixed device array inside the library, FVA_ROUTE_NOALLOC_SCRATCH_BYTES (64 MiB) on
 * every GPU that loads the library, held until the process exits. Nothing is allocated
 * (no cudaMalloc/cudaFree, no allocating library call).
 *   - Shapes whose fva_route_workspace_bytes(s, pooled == NULL) exceeds the array return
 *     FVA_ERR_TOO_LARGE before anything is enqueued (e.g. 48 heads x 275 blocks fit;
 *     40 heads x 512 blocks do not).
 *   - The first call on a device looks up the array's device address with that device
 *     current (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture.
 *   - Every call uses the same array and leaves its contents behind; every byte a call
 *     reads is written earlier in the same call. Calls whose work overlaps on the GPU
 *     (other streams, other host threads, the same device) race on the array: order them
 *     on one stream or synchronise between them.
 */
#define FVA_ROUTE_NOALLOC_SCRATCH_BYTES (64ull << 20)
FVA_API int fva_route_noalloc(const fva_shape* s, const void* q_bhnd_dev, const void* k_bhnd_dev,
                              const double* pooled_q_dev, const double* pooled_k_dev, double p, int k_floor,
                              int order, const fva_mask* mask, int32_t* dev_status, fva_stream_t stream);

/*
 * Runtime Load Balancing planner (host code; [aixai] "Runtime Load Balancing (RLB)", [PD]
 * 方法揭秘). Plans head migrations for a virtual n_ranks-way head split of the measured
 * per-head loads: heads start in the contiguous split (rank r owns heads
 * [r * n_heads / n_ranks, (r + 1) * n_heads / n_ranks)); while the slowest / fastest rank
 * load ratio is >= threshold, the heaviest own head of the most loaded rank whose move to
 * the least loaded rank has positive net gain G = K - P - C is moved there, where
 * K = (max rank load before - max after) and P = comm_ms, C = sched_ms; a rank exports at
 * most max_per_rank of its own heads, and received heads never move again. Ties go to the
 * lower rank / head index.
 *   head_load_ms: host double[n_heads], >= 0 (per-head compute time, e.g. blocks x c);
 *   rank_of_out: host int32[n_heads], the final rank of every head;
 *   moves_out: host array of moves_capacity records, filled in the order applied;
 *     moves_capacity must be >= min(n_heads, n_ranks * max_per_rank) (FVA_ERR_CAPACITY);
 *   n_moves_out: number of records written.
 * threshold >= 1 (the pages' regime boundary k2 = 1.10 is the usual value). Returns FVA_OK,
 * FVA_ERR_INVALID_ARG or FVA_ERR_CAPACITY; enqueues no device work.
 */
typedef struct {
  int32_t head;
  int32_t from_rank;
  int32_t to_rank;
  int32_t reserved;
  double gain_ms; /* net gain G of this move */
} fva_rlb_move;

FVA_API int fva_rlb_plan(const double* head_load_ms, int n_heads, int n_ranks, double comm_ms, double sched_ms,
                         double threshold, int max_per_rank, int32_t* rank_of_out, fva_rlb_move* moves_out,
                         int moves_capacity, int* n_moves_out);

/*
 * Slack-Aware Sparse Augmentation ([aixai] "Slack-Aware Sparse Augmentation (SASA)",
 * "Sparse-routing frontend"; [PD] 方法揭秘), on a head split over n_ranks ranks.
 *
 * fva_sasa_budgets (host): blocks each rank may add. With L_crit the largest of
 * rank_load_ms[0..n_ranks), a rank whose slack L_crit - L_r is >= n2 * L_crit gets
 * floor(n1 * slack / block_ms) blocks, every other rank 0 (the pages' n1 = 0.8,
 * n2 = 0.07; block_ms = compute time of one block). Returns FVA_OK or FVA_ERR_INVALID_ARG.
 *
 * fva_sasa_augment (device): adds to `mask` -- a mask fva_route produced for the same
 * pooled Q/K, whose rows keep prefixes of their routing order -- each rank's budget of
 * skipped (row, key block) entries with the largest routing importance P_ab (the row
 * softmax of the block logits; ties to the lower head, query block, key block), over the
 * rows of the heads with rank_of_head_dev[h] == r. A rank with fewer skipped entries than
 * its budget gets all of them. The mask is rewritten in place: CSR, head_kept, tile lists
 * and the work list in `order` (FVA_ORDER_*).
 *   pooled_q_dev / pooled_k_dev: float64 [B, H, nB, d] as for fva_route; both may be NULL
 *     when mask->logits is set, and are then not read;
 *   mask->logits: when not NULL, the block logits fva_route wrote there for this mask (the
 *     same pooled Q/K); the augmentation takes the importances from them instead of
 *     recomputing the logits (one float64 read of B*H*nB*nB values instead of a GEMM);
 *   rank_of_head_dev: int32 [B*H] device, values in [0, n_ranks) (others: FVA_DEVERR_BAD_LIST
 *     in dev_status, and the head is left unchanged); n_ranks in [1, FVA_SASA_MAX_RANKS];
 *   budget_dev: int64 [n_ranks] device (negative counts as 0);
 *   added_dev: optional int64 [n_ranks] device, the entries added per rank;
 *   workspace: fva_sasa_workspace_bytes(s) bytes, 16-byte aligned.
 * Returns FVA_OK, FVA_ERR_INVALID_ARG, FVA_ERR_UNSUPPORTED_SHAPE, FVA_ERR_CAPACITY,
 * FVA_ERR_WORKSPACE, FVA_ERR_ALIGNMENT or FVA_ERR_CUDA.
 */
#define FVA_SASA_MAX_RANKS 64
FVA_API int fva_sasa_budgets(const double* rank_load_ms, int n_ranks, double block_ms, double n1, double n2,
                             int64_t* budget_out);
FVA_API size_t fva_sasa_workspace_bytes(const fva_shape* s);
FVA_API int fva_sasa_augment(const fva_shape* s, const double* pooled_q_dev, const double* pooled_k_dev,
                             const int32_t* rank_of_head_dev, int n_ranks, const int64_t* budget_dev, int order,
                             const fva_mask* mask, void* workspace_dev, size_t workspace_bytes, int64_t* added_dev,
                             int32_t* dev_status, fva_stream_t stream);

/*
 * Strided asynchronous copy (data movement for the host-pipelined layer; the pages have
 * no counterpart): `rows` rows of `width_bytes` each, from src (consecutive rows
 * src_pitch_bytes apart) to dst (dst_pitch_bytes apart), enqueued on `stream`. Either
 * pointer may be device memory or page-locked host memory (the direction follows from the
 * pointers). With host rows of H * d elements and a device buffer of G * d, this moves the
 * slice of G heads of a [B, N, H, d] tensor in one call. Returns FVA_OK,
 * FVA_ERR_INVALID_ARG (null pointer, width > a pitch, negative sizes) or FVA_ERR_CUDA.
 */
FVA_API int fva_copy_strided(void* dst, size_t dst_pitch_bytes, const void* src, size_t src_pitch_bytes,
                             size_t width_bytes, int64_t rows, fva_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FVA_H_ */
