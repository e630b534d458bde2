// Float32 block-sparse / dense attention on CUDA cores: the correctness path for fp32
// inputs (the tiny 4x16x16 workload), where tolerances of 1e-4 rule out bf16/tf32
// tensor-core arithmetic. Same semantics as the tensor-core kernel (aixai.ru FVAttn
// blog, sparse-attention section): softmax over the valid keys of each query block's
// kept key blocks.
//
// One CTA per (b, h, query block); one thread per query row with its q and o rows in
// registers; each kept key block is staged once in shared memory and consumed with an
// online (running max / running sum) softmax, one score per key.
#include <math.h>

#include "fva_internal.cuh"

namespace fva {

template <int D>
__global__ void __launch_bounds__(64) attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                      const float* __restrict__ v, const int32_t* __restrict__ row_ptr,
                                                      const int32_t* __restrict__ col_idx, int dense, float* __restrict__ o,
                                                      int N, int nB, float scale) {
  extern __shared__ float smem_f32[];
  float(*sk)[D + 1] = reinterpret_cast<float(*)[D + 1]>(smem_f32);
  float(*sv)[D] = reinterpret_cast<float(*)[D]>(smem_f32 + kBlock * (D + 1));
  const int a = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int i = a * kBlock + threadIdx.x;
  const bool valid = i < N;
  const float* qb = q + bh * N * D;
  const float* kbase = k + bh * N * D;
  const float* vbase = v + bh * N * D;
  float qr[D], acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = valid ? qb[static_cast<int64_t>(i) * D + c] * scale : 0.0f;
    acc[c] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  int lo = 0, hi = nB;
  if (!dense) {
    lo = row_ptr[bh * nB + a];
    hi = row_ptr[bh * nB + a + 1];
  }
  for (int e = lo; e < hi; ++e) {
    const int kb = dense ? e : col_idx[e];
    const int n_valid = min(kBlock, N - kb * kBlock);
    __syncthreads();
    for (int idx = threadIdx.x; idx < kBlock * D; idx += blockDim.x) {
      const int r = idx / D, c = idx % D;
      const bool in = r < n_valid;
      const int64_t g = static_cast<int64_t>(kb * kBlock + r) * D + c;
      sk[r][c] = in ? kbase[g] : 0.0f;
      sv[r][c] = in ? vbase[g] : 0.0f;
    }
    __syncthreads();
    for (int r = 0; r < n_valid; ++r) {
      float s = 0.0f;
#pragma unroll
      for (int c = 0; c < D; ++c) s = fmaf(qr[c], sk[r][c], s);
      const float m_new = fmaxf(m, s);
      const float corr = expf(m - m_new);
      const float p = expf(s - m_new);
      l = l * corr + p;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(p, sv[r][c], acc[c] * corr);
      m = m_new;
    }
  }
  if (valid) {
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    float* ob = o + (bh * N + i) * D;
#pragma unroll
    for (int c = 0; c < D; ++c) ob[c] = acc[c] * inv;
  }
}

template <int D>
static cudaError_t launch_f32_t(dim3 grid, const float* q, const float* k, const float* v, const int32_t* row_ptr,
                                const int32_t* col_idx, bool dense, float* o, int N, int nB, float scale,
                                cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kBlock) * (2 * D + 1) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  attn_f32_kernel<D><<<grid, 64, smem, st>>>(q, k, v, row_ptr, col_idx, dense ? 1 : 0, o, N, nB, scale);
  return cudaGetLastError();
}

cudaError_t launch_attn_f32(const Dims& Dm, const float* q, const float* k, const float* v, const int32_t* row_ptr,
                            const int32_t* col_idx, bool dense, float* o, float scale, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(Dm.nB), static_cast<unsigned>(Dm.BH));
  const int N = static_cast<int>(Dm.N), nB = static_cast<int>(Dm.nB);
  switch (Dm.d) {
    case 32:
      return launch_f32_t<32>(grid, q, k, v, row_ptr, col_idx, dense, o, N, nB, scale, st);
    case 64:
      return launch_f32_t<64>(grid, q, k, v, row_ptr, col_idx, dense, o, N, nB, scale, st);
    case 128:
      return launch_f32_t<128>(grid, q, k, v, row_ptr, col_idx, dense, o, N, nB, scale, st);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace fva
