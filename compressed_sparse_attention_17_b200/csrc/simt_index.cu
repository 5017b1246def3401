// simt_index.cu - CUDA-core lightning-indexer scores and radix top-k.
//
// These kernels accept every dtype and shape the C ABI accepts. They are the
// FP32 path (FP32 arithmetic throughout, as the FP32 workloads require) and
// the path for shapes the tensor-core kernels do not cover.
//
// Equations: "Evidence Ledger" CSA Eqs 9-19, HCA Eqs 20-26, Shared attention
// details (Sec 2.3.3, Eq 27); "DeepSeek-V4" study 03 (pooling and index-score
// formulas).
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

// ---------------------------------------------------------------------------
// Index scores on CUDA cores: I[q,s] = sum_h w[q,h] ReLU(qI[q,h] . KI[s]).
// Block = 128 entries of one query; KI tile staged in shared memory with a
// padded row stride; each thread accumulates its entry's H_I head dots.
// ---------------------------------------------------------------------------
template <typename Tin, int HMAX>
__global__ void __launch_bounds__(128) index_scores_simt_kernel(
    csa_geom g, const Tin* __restrict__ qI, const float* __restrict__ w,
    const Tin* __restrict__ KI, int64_t ldK, int nseq, const int32_t* __restrict__ seq_of_q,
    const int64_t* __restrict__ pos, const int64_t* __restrict__ n_entries, int H_I, int c_I,
    float* __restrict__ scores, int64_t ld_scores) {
  extern __shared__ float smem[];
  const int q = blockIdx.y;
  const int b = seq_of_q[q];
  if (b < 0 || b >= nseq) return;
  const int64_t nv = n_visible(pos[q], g.m, g.vis_offset, min(n_entries[b], ldK));
  const int64_t s0 = (int64_t)blockIdx.x * 128;
  if (s0 >= nv) return;
  float* qs = smem;                   // [H_I][c_I]
  float* ws = qs + H_I * c_I;         // [H_I]
  float* ks = ws + HMAX;              // [128][c_I + 1]
  for (int e = threadIdx.x; e < H_I * c_I; e += 128) qs[e] = to_f32(qI[(int64_t)q * H_I * c_I + e]);
  for (int e = threadIdx.x; e < H_I; e += 128) ws[e] = w[(int64_t)q * H_I + e];
  const int ld = c_I + 1;
  const Tin* kb = KI + ((int64_t)b * ldK + s0) * c_I;
  for (int e = threadIdx.x; e < 128 * c_I; e += 128) {
    int rr = e / c_I, j = e % c_I;
    ks[rr * ld + j] = (s0 + rr < nv) ? to_f32(kb[(int64_t)rr * c_I + j]) : 0.f;
  }
  __syncthreads();
  const int64_t s = s0 + threadIdx.x;
  if (s >= nv) return;
  float acc[HMAX];
#pragma unroll
  for (int h = 0; h < HMAX; ++h) acc[h] = 0.f;
  const float* kr = ks + threadIdx.x * ld;
  for (int j = 0; j < c_I; ++j) {
    const float kv = kr[j];
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
      if (h < H_I) acc[h] = fmaf(qs[h * c_I + j], kv, acc[h]);
  }
  float I = 0.f;
#pragma unroll
  for (int h = 0; h < HMAX; ++h)
    if (h < H_I) I = fmaf(ws[h], fmaxf(acc[h], 0.f), I);
  scores[(int64_t)q * ld_scores + s] = I;
}

}  // namespace

template <typename Tin, int HMAX>
static cudaError_t index_simt_t(const csa_geom& g, const void* qI, const float* w, const void* KI,
                                int64_t ldK, int nseq, const int32_t* seq_of_q, const int64_t* pos,
                                const int64_t* n_entries, int Q, int H_I, int c_I, float* scores,
                                int64_t ld_scores, cudaStream_t s) {
  size_t smem = sizeof(float) * ((size_t)H_I * c_I + HMAX + 128 * (size_t)(c_I + 1));
  auto kern = index_scores_simt_kernel<Tin, HMAX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((ldK + 127) / 128), (unsigned)Q);
  count_launches();
  kern<<<grid, 128, smem, s>>>(g, reinterpret_cast<const Tin*>(qI), w,
                               reinterpret_cast<const Tin*>(KI), ldK, nseq, seq_of_q, pos, n_entries,
                               H_I, c_I, scores, ld_scores);
  return cudaGetLastError();
}

cudaError_t launch_index_scores_simt(const csa_geom& g, int dt, const void* qI, const float* w,
                                     const void* KI, int64_t ldK, int nseq,
                                     const int32_t* seq_of_q,
                                     const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                                     int c_I, float* scores, int64_t ld_scores, cudaStream_t s) {
  if (Q == 0 || ldK == 0) return cudaSuccess;
#define CSA_IDX_CASE(HM)                                                                       \
  if (H_I <= HM)                                                                               \
    return dt == CSA_F32                                                                       \
               ? index_simt_t<float, HM>(g, qI, w, KI, ldK, nseq, seq_of_q, pos, n_entries, Q, H_I,  \
                                         c_I, scores, ld_scores, s)                            \
               : index_simt_t<__nv_bfloat16, HM>(g, qI, w, KI, ldK, nseq, seq_of_q, pos, n_entries,  \
                                                 Q, H_I, c_I, scores, ld_scores, s);
  CSA_IDX_CASE(8)
  CSA_IDX_CASE(32)
  CSA_IDX_CASE(64)
  CSA_IDX_CASE(128)
#undef CSA_IDX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace csa
