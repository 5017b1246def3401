// tc_index.cu - lightning-indexer scores on the 5th-generation tensor cores.
//
// I[q, s] = sum_h w[q,h] * ReLU(qI[q,h,:] . KI[b, s, :])
// ("Evidence Ledger", CSA Eqs 13-17; "DeepSeek-V4" study 03, index-score
// formula).
//
// One CTA computes one tile of 128 compressed entries against a group of
// queries of the same sequence: the entries are the MMA's M dimension (one
// TMEM lane each), the group's (query, head) pairs its N dimension, the key
// width its K dimension. TMA brings both operands into shared memory in the
// 128-byte-swizzled K-major layout; one thread issues tcgen05.mma into a
// TMEM accumulator; four epilogue warps read their lanes back and apply the
// ReLU, the head weights and the head sum in registers, so each thread owns
// one entry and no cross-thread reduction is needed.
//
// Warp roles (192 threads): warp 0 issues the TMA loads, warp 1 owns the
// TMEM allocation and issues the MMAs, warps 2-5 run the epilogue.
#include "internal.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kThreads = 192;
constexpr int kTileM = 128;
constexpr int kChunkBytesA = kTileM * 128;  // 128 rows x 64 BF16

struct Params {
  int Q, H_I, c_I, G, nseq;
  int64_t ldK;
  int m, vis_offset;
  const int32_t* seq_of_q;
  const int64_t* pos;
  const int64_t* n_entries;
  const float* w;
  float* scores;
  int64_t ld_scores;
  int* err;
  uint32_t tmem_cols;
};

__device__ __forceinline__ int64_t query_nvis(const Params& P, int q) {
  const int b = P.seq_of_q[q];
  if (b < 0 || b >= P.nseq) return 0;
  return n_visible(P.pos[q], P.m, P.vis_offset, min(P.n_entries[b], P.ldK));
}

__global__ void __launch_bounds__(kThreads, 2)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmQ, Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int KCH = P.c_I / 64;
  const int Nmax = P.G * P.H_I;
  uint8_t* sA = smem;
  uint8_t* sB = sA + KCH * kChunkBytesA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + KCH * Nmax * 128);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  float* wsm = reinterpret_cast<float*>(tslot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * P.G;
  const int qn = min(P.G, P.Q - q0);
  const int64_t s0 = (int64_t)blockIdx.y * kTileM;

  int64_t nv_max = 0;
  for (int j = 0; j < qn; ++j) nv_max = max(nv_max, query_nvis(P, q0 + j));
  if (s0 >= nv_max) return;  // same decision in every thread of the CTA

  const uint32_t full_bar = tc::smem_u32(&bars[0]);
  const uint32_t mma_bar = tc::smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    tc::mbar_init(full_bar, 1);
    tc::mbar_init(mma_bar, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmQ);
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_u32(tslot), P.tmem_cols);
  for (int e = threadIdx.x; e < qn * P.H_I; e += kThreads) wsm[e] = P.w[(int64_t)q0 * P.H_I + e];
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tslot;

  uint32_t phase = 0;
  int j0 = 0;
  while (j0 < qn) {
    // one pass per run of consecutive queries of the same sequence
    const int b = P.seq_of_q[q0 + j0];
    int j1 = j0 + 1;
    while (j1 < qn && P.seq_of_q[q0 + j1] == b) ++j1;
    int64_t nv_run = 0;
    for (int j = j0; j < j1; ++j) nv_run = max(nv_run, query_nvis(P, q0 + j));
    if (s0 < nv_run) {
      const int nq = j1 - j0;
      const int N = nq * P.H_I;
      if (threadIdx.x == 0) {
        tc::mbar_arrive_expect_tx(full_bar, (uint32_t)(KCH * kChunkBytesA + KCH * N * 128));
        const int32_t yk = (int32_t)((int64_t)b * P.ldK + s0);
        for (int ch = 0; ch < KCH; ++ch)
          tc::tma_load_2d(tc::smem_u32(sA + ch * kChunkBytesA), &tmK, ch * 64, yk, full_bar);
        for (int j = j0; j < j1; ++j)
          for (int ch = 0; ch < KCH; ++ch)
            tc::tma_load_2d(tc::smem_u32(sB + ch * Nmax * 128 + (j - j0) * P.H_I * 128), &tmQ,
                            ch * 64, (q0 + j) * P.H_I, full_bar);
      }
      if (warp == 1) {
        if (lane == 0) {
          if (tc::mbar_wait(full_bar, phase, P.err)) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16_f32(kTileM, N);
            for (int kk = 0; kk < KCH * 4; ++kk) {
              const int ch = kk >> 2;
              const uint32_t off = (uint32_t)(kk & 3) * 32;
              const uint64_t ad = tc::sdesc_kmajor_sw128(tc::smem_u32(sA + ch * kChunkBytesA) + off);
              const uint64_t bd = tc::sdesc_kmajor_sw128(tc::smem_u32(sB + ch * Nmax * 128) + off);
              tc::mma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(mma_bar);
          } else {
            *abort_flag = 1;
          }
        }
        __syncwarp();
      } else if (warp >= 2) {
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        if (tc::mbar_wait(mma_bar, phase, P.err)) {
          tc::tc_fence_after();
          const int64_t s = s0 + row;
          for (int j = j0; j < j1; ++j) {
            float acc = 0.f;
            const float* wq = wsm + j * P.H_I;
            for (int h0 = 0; h0 < P.H_I; h0 += 16) {
              float v[16];
              tc::tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)((j - j0) * P.H_I + h0), v);
#pragma unroll
              for (int i = 0; i < 16; ++i) acc = fmaf(wq[h0 + i], fmaxf(v[i], 0.f), acc);
            }
            if (s < query_nvis(P, q0 + j)) P.scores[(int64_t)(q0 + j) * P.ld_scores + s] = acc;
          }
        } else {
          *abort_flag = 1;
        }
      }
      phase ^= 1u;
      tc::tc_fence_before();
      __syncthreads();
      tc::tc_fence_after();
      if (*abort_flag) break;
    }
    j0 = j1;
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, P.tmem_cols);
}

}  // namespace

bool index_tc_supported(int dt, int H_I, int c_I) {
  return dt == CSA_BF16 && H_I % 16 == 0 && H_I >= 16 && H_I <= 128 && c_I % 64 == 0 &&
         c_I >= 64 && c_I <= 256;
}

cudaError_t launch_index_scores_tc(const csa_geom& g, const void* qI, const float* w,
                                   const void* KI, int64_t ldK, int nseq,
                                   const int32_t* seq_of_q, const int64_t* pos,
                                   const int64_t* n_entries, int Q, int H_I, int c_I,
                                   float* scores, int64_t ld_scores, cudaStream_t s) {
  if (Q == 0 || ldK == 0 || nseq == 0) return cudaSuccess;
  // query groups share one entry tile; many queries per call means prefill
  int G = Q >= 512 ? 256 / H_I : 1;
  if (G < 1) G = 1;
  CUtensorMap tmK, tmQ;
  if (!encode_tmap_2d_bf16(&tmK, KI, (uint64_t)c_I, (uint64_t)nseq * ldK, (uint64_t)c_I * 2, 64,
                           kTileM))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d_bf16(&tmQ, qI, (uint64_t)c_I, (uint64_t)Q * H_I, (uint64_t)c_I * 2, 64,
                           (uint32_t)H_I))
    return cudaErrorInvalidValue;
  Params P;
  P.Q = Q;
  P.H_I = H_I;
  P.c_I = c_I;
  P.G = G;
  P.nseq = nseq;
  P.ldK = ldK;
  P.m = g.m;
  P.vis_offset = g.vis_offset;
  P.seq_of_q = seq_of_q;
  P.pos = pos;
  P.n_entries = n_entries;
  P.w = w;
  P.scores = scores;
  P.ld_scores = ld_scores;
  P.err = device_error_ptr();
  uint32_t cols = 32;
  while (cols < (uint32_t)(G * H_I)) cols <<= 1;
  P.tmem_cols = cols;
  const int KCH = c_I / 64;
  const size_t smem = 1024 + (size_t)KCH * kChunkBytesA + (size_t)KCH * G * H_I * 128 + 64 +
                      sizeof(float) * (size_t)G * H_I;
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (ldK + kTileM - 1) / kTileM;
  if (tiles > 65535) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((Q + G - 1) / G), (unsigned)tiles);
  count_launches();
  index_scores_tc_kernel<<<grid, kThreads, smem, s>>>(tmK, tmQ, P);
  return cudaGetLastError();
}

}  // namespace csa
