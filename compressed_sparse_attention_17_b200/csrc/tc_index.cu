// tc_index.cu - lightning-indexer scores on the 5th-generation tensor cores.
//
// I[q, s] = sum_h w[q,h] * ReLU(qI[q,h,:] . KI[b, s, :])
// ("Evidence Ledger", CSA Eqs 13-17; "DeepSeek-V4" study 03, index-score
// formula).
//
// A tile of 128 compressed entries against one query: the entries are the
// MMA's M dimension (one TMEM lane each), the query's heads its N dimension,
// the key width its K dimension. TMA brings both operands into shared memory
// in the 128-byte-swizzled K-major layout; one thread issues tcgen05.mma into
// a TMEM accumulator; four epilogue warps read their lanes back and apply the
// ReLU, the head weights and the head sum in registers, so each thread owns
// one entry and no cross-thread reduction is needed.
//
// Warp roles (192 threads): warp 0 issues the TMA loads, warp 1 owns the
// TMEM allocation and issues the MMAs, warps 2-5 run the epilogue.
#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kThreads = 192;
constexpr int kTileM = 128;
constexpr int kChunkBytesA = kTileM * 128;  // 128 rows x 64 BF16

// ---------------------------------------------------------------------------
// Persistent, pipelined kernel (one CTA per SM) over (query, 128-entry tile)
// units: with few queries (decode) every CTA takes a balanced contiguous
// range of units, which may span query boundaries; with many (prefill) CTA i
// takes every tile of queries i, i + grid, ... Warp 0 streams the key tiles
// through a ring of shared-memory stages (TMA, evict-first L2 policy) and
// loads a query's qI into one of two slots when the query changes; warp 1
// issues the MMAs into one of four TMEM accumulators; warps 2-5 reduce the
// accumulator while the next tile is multiplied and later tiles load.
// ---------------------------------------------------------------------------
constexpr int kDecAcc = 4;  // TMEM accumulators in flight between the MMA and the epilogue

struct DecParams {
  int Q, H_I, c_I, nseq, stages;
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
  int interleave;  // 1: CTA i takes queries i, i + grid, ...; 0: contiguous unit ranges
};

__device__ __forceinline__ int64_t dec_nvis(const DecParams& P, int q) {
  const int b = P.seq_of_q[q];
  if (b < 0 || b >= P.nseq) return 0;
  return n_visible(P.pos[q], P.m, P.vis_offset, min(P.n_entries[b], P.ldK));
}

__device__ __forceinline__ int dec_ntiles(const DecParams& P, int q) {
  return (int)((dec_nvis(P, q) + kTileM - 1) / kTileM);
}

// The (query, entry tile) units of one CTA, in order. Contiguous mode: units
// [u0, u1) of the query-major order, prefix[q] = first unit of query q (few
// queries: a query's tiles spread over several CTAs). Interleaved mode: every
// tile of queries blockIdx.x, blockIdx.x + gridDim.x, ... (many queries; the
// causal tile counts balance across CTAs).
struct UnitWalk {
  const int* prefix;
  const DecParams* P;
  int Q;
  int q;
  int64_t t;
  int nt;  // tiles of query q (interleaved mode)
  __device__ void start(const DecParams& prm, const int* pre, int u0) {
    P = &prm;
    prefix = pre;
    Q = prm.Q;
    if (prm.interleave) {
      q = blockIdx.x;
      t = 0;
      nt = q < Q ? dec_ntiles(prm, q) : 0;
      while (q < Q && nt == 0) {
        q += gridDim.x;
        nt = q < Q ? dec_ntiles(prm, q) : 0;
      }
      return;
    }
    int lo = 0, hi = Q - 1;  // largest q with prefix[q] <= u0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= u0) lo = mid;
      else hi = mid - 1;
    }
    q = lo;
    t = u0 - prefix[q];
    while (q < Q - 1 && t >= prefix[q + 1] - prefix[q]) {
      t -= prefix[q + 1] - prefix[q];
      ++q;
    }
  }
  __device__ void next() {
    ++t;
    if (P->interleave) {
      while (q < Q && t >= nt) {
        q += gridDim.x;
        t = 0;
        nt = q < Q ? dec_ntiles(*P, q) : 0;
      }
      return;
    }
    while (q < Q - 1 && t >= prefix[q + 1] - prefix[q]) {
      t = 0;
      ++q;
    }
  }
};

// HREG = H_I when the head weights of the current query are kept in
// registers (reloaded when the query changes), 0 for read-through loads.
template <int HREG>
__global__ void __launch_bounds__(kThreads, 1)
    index_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                        DecParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int KCH = P.c_I / 64;
  const int S = P.stages;
  const int bytesA = KCH * kChunkBytesA;
  const int bytesB = KCH * P.H_I * 128;
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * bytesA;
  float* wsm = reinterpret_cast<float*>(sB + 2 * bytesB);
  int* prefix = reinterpret_cast<int*>(wsm + 128);
  uint64_t* bars = reinterpret_cast<uint64_t*>(prefix + (P.interleave ? 2 : ((P.Q + 2 + 1) & ~1)));
  // bars: Afull[S], Aempty[S], Bfull[2], Bempty[2], accfull[kDecAcc], accempty[kDecAcc]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4 + 2 * kDecAcc);
  __shared__ int scan_tmp[kThreads / 32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int u0 = 0, u1 = 0;
  if (P.interleave) {
    // ---- this CTA's tile count over its queries ----
    int cnt = 0;
    for (int q = blockIdx.x + threadIdx.x * gridDim.x; q < P.Q; q += kThreads * gridDim.x)
      cnt += dec_ntiles(P, q);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) scan_tmp[warp] = cnt;
    __syncthreads();
    for (int i = 0; i < kThreads / 32; ++i) u1 += scan_tmp[i];
    __syncthreads();
  } else {
    // ---- units per query and their prefix (every CTA computes it) ----
    int carry = 0;
    for (int base = 0; base < P.Q; base += kThreads) {
      const int q = base + threadIdx.x;
      const int nt = q < P.Q ? dec_ntiles(P, q) : 0;
      int x = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) scan_tmp[warp] = x;
      __syncthreads();
      int wbase = 0, tot = 0;
      for (int i = 0; i < kThreads / 32; ++i) {
        wbase += i < warp ? scan_tmp[i] : 0;
        tot += scan_tmp[i];
      }
      if (q < P.Q) prefix[q] = carry + wbase + x - nt;
      carry += tot;
      __syncthreads();
    }
    if (threadIdx.x == 0) prefix[P.Q] = carry;
    __syncthreads();
    const int U = prefix[P.Q];
    u0 = (int)((int64_t)blockIdx.x * U / gridDim.x);
    u1 = (int)((int64_t)(blockIdx.x + 1) * U / gridDim.x);
  }
  if (u0 >= u1) return;  // same decision in every thread of the CTA

  auto afull = [&](int s) { return tc::smem_u32(&bars[s]); };
  auto aempty = [&](int s) { return tc::smem_u32(&bars[S + s]); };
  auto bfull = [&](int s) { return tc::smem_u32(&bars[2 * S + s]); };
  auto bempty = [&](int s) { return tc::smem_u32(&bars[2 * S + 2 + s]); };
  auto accfull = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + s]); };
  auto accempty = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + kDecAcc + s]); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(afull(s), 1);
      tc::mbar_init(aempty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bfull(s), 1);
      tc::mbar_init(bempty(s), 1);
    }
    for (int s = 0; s < kDecAcc; ++s) {
      tc::mbar_init(accfull(s), 1);
      tc::mbar_init(accempty(s), 4);
    }
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmQ);
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_u32(tslot), P.tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tslot;
  const int nunits = u1 - u0;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer ----
      const uint64_t pol = tc::l2_policy_evict_first();
      UnitWalk wk;
      wk.start(P, prefix, u0);
      int last_q = -1, gc = -1;
      for (int i = 0; i < nunits; ++i, wk.next()) {
        const int q = wk.q;
        if (q != last_q) {
          ++gc;
          const int bs = gc & 1;
          if (gc >= 2 && !tc::mbar_wait(bempty(bs), ((gc >> 1) - 1) & 1, P.err)) break;
          tc::mbar_arrive_expect_tx(bfull(bs), (uint32_t)bytesB);
          for (int ch = 0; ch < KCH; ++ch)
            tc::tma_load_2d(tc::smem_u32(sB + bs * bytesB + ch * P.H_I * 128), &tmQ, ch * 64,
                            q * P.H_I, bfull(bs));
          last_q = q;
        }
        const int s = i % S;
        if (i >= S && !tc::mbar_wait(aempty(s), ((i / S) - 1) & 1, P.err)) break;
        tc::mbar_arrive_expect_tx(afull(s), (uint32_t)bytesA);
        const int32_t y = (int32_t)((int64_t)P.seq_of_q[q] * P.ldK + wk.t * kTileM);
        for (int ch = 0; ch < KCH; ++ch)
          tc::tma_load_2d_hint(tc::smem_u32(sA + s * bytesA + ch * kChunkBytesA), &tmK, ch * 64, y,
                               afull(s), pol);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      const uint32_t idesc = tc::idesc_bf16_f32(kTileM, P.H_I);
      UnitWalk wk;
      wk.start(P, prefix, u0);
      int last_q = -1, gc = -1;
      for (int i = 0; i < nunits; ++i, wk.next()) {
        const int q = wk.q;
        if (q != last_q) {
          if (gc >= 0) tc::mma_commit(bempty(gc & 1));  // previous query's qI slot is free
          ++gc;
          if (!tc::mbar_wait(bfull(gc & 1), (gc >> 1) & 1, P.err)) break;
          last_q = q;
        }
        const int s = i % S, a = i % kDecAcc;
        if (!tc::mbar_wait(afull(s), (i / S) & 1, P.err)) break;
        if (i >= kDecAcc && !tc::mbar_wait(accempty(a), ((i / kDecAcc) - 1) & 1, P.err)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * P.H_I);
        for (int kk = 0; kk < KCH * 4; ++kk) {
          const int ch = kk >> 2;
          const uint32_t off = (uint32_t)(kk & 3) * 32;
          tc::mma_bf16(d, tc::sdesc_kmajor_sw128(tc::smem_u32(sA + s * bytesA + ch * kChunkBytesA) + off),
                       tc::sdesc_kmajor_sw128(tc::smem_u32(sB + (gc & 1) * bytesB + ch * P.H_I * 128) + off),
                       idesc, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(aempty(s));
        tc::mma_commit(accfull(a));
      }
    }
    __syncwarp();
  } else {
    // ---- epilogue: one entry per thread ----
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    UnitWalk wk;
    wk.start(P, prefix, u0);
    int last_q = -1;
    int64_t nv = 0;
    float* out = nullptr;
    const float* wq = nullptr;
    float wr[HREG > 0 ? HREG : 1];
    for (int i = 0; i < nunits; ++i, wk.next()) {
      const int q = wk.q;
      if (q != last_q) {
        nv = dec_nvis(P, q);
        out = P.scores + (int64_t)q * P.ld_scores;
        wq = P.w + (int64_t)q * P.H_I;
        if (HREG > 0) {
#pragma unroll
          for (int h = 0; h < HREG; h += 4) {
            const float4 t4 = __ldg(reinterpret_cast<const float4*>(wq + h));
            wr[h] = t4.x;
            wr[h + 1] = t4.y;
            wr[h + 2] = t4.z;
            wr[h + 3] = t4.w;
          }
        }
        last_q = q;
      }
      const int a = i % kDecAcc;
      if (!tc::mbar_wait_warp(accfull(a), (i / kDecAcc) & 1, P.err)) break;
      tc::tc_fence_after();
      float acc4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains over the heads
      if (HREG > 0) {
#pragma unroll
        for (int h0 = 0; h0 < (HREG > 0 ? HREG : 16); h0 += 32) {
          float v[32];
          tc::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * HREG + h0), v);
#pragma unroll
          for (int j = 0; j < 32; ++j) acc4[j & 3] = fmaf(wr[h0 + j], fmaxf(v[j], 0.f), acc4[j & 3]);
        }
      } else {
        for (int h0 = 0; h0 < P.H_I; h0 += 16) {
          float v[16];
          tc::tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * P.H_I + h0), v);
#pragma unroll
          for (int j = 0; j < 16; ++j) acc4[j & 3] = fmaf(__ldg(wq + h0 + j), fmaxf(v[j], 0.f), acc4[j & 3]);
        }
      }
      const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(accempty(a));
      const int64_t sidx = wk.t * kTileM + row;
      if (sidx < nv) out[sidx] = acc;
    }
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
  CUtensorMap tmK, tmQ;
  if (!encode_tmap_2d_bf16(&tmK, KI, (uint64_t)c_I, (uint64_t)nseq * ldK, (uint64_t)c_I * 2, 64,
                           kTileM) ||
      !encode_tmap_2d_bf16(&tmQ, qI, (uint64_t)c_I, (uint64_t)Q * H_I, (uint64_t)c_I * 2, 64,
                           (uint32_t)H_I))
    return cudaErrorInvalidValue;
  DecParams P{};
  P.Q = Q;
  P.H_I = H_I;
  P.c_I = c_I;
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
  int nsm = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  P.interleave = Q >= 4 * nsm ? 1 : 0;
  uint32_t cols = 32;
  while (cols < (uint32_t)(kDecAcc * H_I)) cols <<= 1;
  P.tmem_cols = cols;
  const int KCH = c_I / 64;
  const size_t prefix_ints = P.interleave ? 2 : (size_t)Q + 3;
  const size_t fixed = 1024 + 2 * (size_t)KCH * H_I * 128 + 128 * 4 + prefix_ints * 4 + 256;
  const size_t per_stage = (size_t)KCH * kChunkBytesA;
  const int stages = (int)std::min<size_t>(6, (220 * 1024 - fixed) / per_stage);
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = fixed + stages * per_stage;
  // w rows are read as float4 in the register path: 16-byte aligned rows
  const bool wreg = H_I == 64 && (reinterpret_cast<uintptr_t>(w) & 15) == 0;
  auto kern = wreg ? index_decode_kernel<64> : index_decode_kernel<0>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  count_launches();
  kern<<<nsm, kThreads, smem, s>>>(tmK, tmQ, P);
  return cudaGetLastError();
}

}  // namespace csa
