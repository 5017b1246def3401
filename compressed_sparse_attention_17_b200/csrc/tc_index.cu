// tc_index.cu - lightning-indexer scores on the 5th-generation tensor cores.
//
// I[q, s] = sum_h w[q,h] * ReLU(qI[q,h,:] . KI[b, s, :])
// ("Evidence Ledger", CSA Eqs 13-17; "DeepSeek-V4" study 03, index-score
// formula).
//
// A tile of 128 compressed entries against one query, or against a group of
// four consecutive queries of one sequence: the entries are the MMA's M
// dimension (one TMEM lane each), the (query, head) rows its N dimension, the
// key width its K dimension. TMA brings both operands into shared memory in
// the 128-byte-swizzled K-major layout; one thread issues tcgen05.mma into a
// TMEM accumulator; the epilogue warps read their lanes back and apply the
// ReLU, the head weights and the head sum in registers, so each thread owns
// one entry and no cross-thread reduction is needed.
//
// Warp roles: warp 0 issues the TMA loads, warp 1 owns the TMEM allocation
// and issues the MMAs, the remaining warps (4, or 8 for query groups) run the
// epilogue.
#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kTileM = 128;
constexpr int kChunkBytesA = kTileM * 128;  // 128 rows x 64 BF16

// ---------------------------------------------------------------------------
// Persistent, pipelined kernel (one CTA per SM) over (query group, 128-entry
// tile) units. A group is G consecutive queries of one sequence: its G x H_I
// (query, head) rows form the MMA's N dimension, so one key tile serves the
// whole group (G = 4 for long single-sequence runs such as prefill, where the
// same keys are read by every query; G = 1 otherwise). With few groups every
// CTA takes a balanced contiguous range of units, which may span group
// boundaries; with many, CTA i takes every tile of groups i, i + grid, ...
// Warp 0 streams the key tiles through a ring of shared-memory stages (TMA,
// evict-first L2 policy) and loads a group's qI into one of two slots when
// the group changes; warp 1 issues the MMAs into one of the TMEM accumulators;
// warps 2-5 reduce an accumulator while the next tile is multiplied and later
// tiles load.
// ---------------------------------------------------------------------------
constexpr int kDecAcc = 4;  // G = 1: TMEM accumulators in flight between the MMA and the epilogue
constexpr int kGrpAcc = 2;  // G > 1: two accumulators of G x H_I columns

// Warp roles: warp 0 loads, warp 1 issues the MMAs, the rest run the
// epilogue (G = 1: 4 warps, one per TMEM lane quadrant; G > 1: 8 warps, two
// per quadrant, each taking half of the group's queries).
template <int G>
struct GroupCfg {
  static constexpr int acc = G == 1 ? kDecAcc : kGrpAcc;
  static constexpr int epi_warps = G == 1 ? 4 : 8;
  // qI slots: two for single queries (the next query loads while the current
  // one is multiplied); one 64 KB slot for groups, which leaves room for a
  // fourth key stage (the next group's qI is first pulled into L2)
  static constexpr int qslots = G == 1 ? 2 : 1;
  static constexpr int threads = 64 + 32 * epi_warps;
};

struct DecParams {
  int Q, H_I, c_I, nseq, stages;
  int NG;  // query groups of G consecutive queries
  const void* qI;
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

// Entry tiles of group g: those of its member that sees the most entries.
template <int G>
__device__ __forceinline__ int grp_ntiles(const DecParams& P, int g) {
  int nt = 0;
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int q = g * G + j;
    if (q < P.Q) nt = max(nt, dec_ntiles(P, q));
  }
  return nt;
}

// The (group, entry tile) units of one CTA, in order. Contiguous mode: units
// [u0, u1) of the group-major order, prefix[g] = first unit of group g (few
// groups: a group's tiles spread over several CTAs). Interleaved mode: every
// tile of groups blockIdx.x, blockIdx.x + gridDim.x, ... (many groups; the
// causal tile counts balance across CTAs). q below is the group index.
template <int G>
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
    Q = prm.NG;
    if (prm.interleave) {
      q = blockIdx.x;
      t = 0;
      nt = q < Q ? grp_ntiles<G>(prm, q) : 0;
      while (q < Q && nt == 0) {
        q += gridDim.x;
        nt = q < Q ? grp_ntiles<G>(prm, q) : 0;
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
        nt = q < Q ? grp_ntiles<G>(*P, q) : 0;
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
// registers (reloaded when the query changes; G = 1), 0 for read-through
// loads. G = queries per group (1, or 4 with H_I = 64).
template <int HREG, int G>
__global__ void __launch_bounds__(GroupCfg<G>::threads, 1)
    index_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                        DecParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int KCH = P.c_I / 64;
  const int S = P.stages;
  constexpr int NACC = GroupCfg<G>::acc;
  const int NW = G * P.H_I;  // MMA N: the group's (query, head) rows
  const int bytesA = KCH * kChunkBytesA;
  const int bytesB = KCH * NW * 128;
  constexpr int QS = GroupCfg<G>::qslots;
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * bytesA;
  // groups: the head weights of two groups (double-buffered, bulk-copied)
  float* wsm = reinterpret_cast<float*>(sB + QS * bytesB);
  int* prefix = reinterpret_cast<int*>(wsm + (G > 1 ? 2 * NW : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(prefix + (P.interleave ? 2 : ((P.NG + 2 + 1) & ~1)));
  // bars: Afull[S], Aempty[S], Bfull[2], Bempty[2], accfull[NACC], accempty[NACC], Wfull[2], Wempty[2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4 + 2 * NACC + 4);
  constexpr int kThreads = GroupCfg<G>::threads;
  constexpr int kEpi = GroupCfg<G>::epi_warps;
  __shared__ int scan_tmp[kThreads / 32];
  pdl_wait();  // the previous kernel's writes are visible from here on

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int u0 = 0, u1 = 0;
  if (P.interleave) {
    // ---- this CTA's tile count over its groups ----
    int cnt = 0;
    for (int q = blockIdx.x + threadIdx.x * gridDim.x; q < P.NG; q += kThreads * gridDim.x)
      cnt += grp_ntiles<G>(P, q);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) scan_tmp[warp] = cnt;
    __syncthreads();
    for (int i = 0; i < kThreads / 32; ++i) u1 += scan_tmp[i];
    __syncthreads();
  } else {
    // ---- units per group and their prefix (every CTA computes it) ----
    int carry = 0;
    for (int base = 0; base < P.NG; base += kThreads) {
      const int q = base + threadIdx.x;
      const int nt = q < P.NG ? grp_ntiles<G>(P, q) : 0;
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
      if (q < P.NG) prefix[q] = carry + wbase + x - nt;
      carry += tot;
      __syncthreads();
    }
    if (threadIdx.x == 0) prefix[P.NG] = carry;
    __syncthreads();
    const int U = prefix[P.NG];
    u0 = (int)((int64_t)blockIdx.x * U / gridDim.x);
    u1 = (int)((int64_t)(blockIdx.x + 1) * U / gridDim.x);
  }
  if (u0 >= u1) return;  // same decision in every thread of the CTA

  auto afull = [&](int s) { return tc::smem_u32(&bars[s]); };
  auto aempty = [&](int s) { return tc::smem_u32(&bars[S + s]); };
  auto bfull = [&](int s) { return tc::smem_u32(&bars[2 * S + s]); };
  auto bempty = [&](int s) { return tc::smem_u32(&bars[2 * S + 2 + s]); };
  auto accfull = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + s]); };
  auto accempty = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + NACC + s]); };
  auto wfull = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + 2 * NACC + s]); };
  auto wempty = [&](int s) { return tc::smem_u32(&bars[2 * S + 4 + 2 * NACC + 2 + s]); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(afull(s), 1);
      tc::mbar_init(aempty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bfull(s), 1);
      tc::mbar_init(bempty(s), 1);
    }
    for (int s = 0; s < NACC; ++s) {
      tc::mbar_init(accfull(s), 1);
      tc::mbar_init(accempty(s), kEpi);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(wfull(s), 1);
      tc::mbar_init(wempty(s), kEpi);
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
      UnitWalk<G> wk;
      wk.start(P, prefix, u0);
      int last_q = -1, gc = -1;
      // qI of a new query (group) into its slot once the slot's previous
      // occupant has left the MMA
      auto load_q = [&](int q) {
        ++gc;
        const int bs = gc % QS;
        if (gc >= QS && !tc::mbar_wait(bempty(bs), ((gc / QS) - 1) & 1, P.err)) return false;
        tc::mbar_arrive_expect_tx(bfull(bs), (uint32_t)bytesB);
        for (int ch = 0; ch < KCH; ++ch)
          tc::tma_load_2d(tc::smem_u32(sB + bs * bytesB + ch * NW * 128), &tmQ, ch * 64, q * NW, bfull(bs));
        return true;
      };
      for (int i = 0; i < nunits; ++i, wk.next()) {
        const int q = wk.q;
        const bool newq = q != last_q;
        if (G == 1 && newq && !load_q(q)) break;
        const int s = i % S;
        if (i >= S && !tc::mbar_wait(aempty(s), ((i / S) - 1) & 1, P.err)) break;
        tc::mbar_arrive_expect_tx(afull(s), (uint32_t)bytesA);
        // groups of several queries are formed only over a single sequence
        const int64_t seq = G == 1 ? (int64_t)P.seq_of_q[q] : 0;
        const int32_t y = (int32_t)(seq * P.ldK + wk.t * kTileM);
        for (int ch = 0; ch < KCH; ++ch)
          tc::tma_load_2d_hint(tc::smem_u32(sA + s * bytesA + ch * kChunkBytesA), &tmK, ch * 64, y,
                               afull(s), pol);
        if (G > 1 && newq) {
          // the key tile goes first: it needs no qI slot and lands while the
          // previous group drains from the single slot
          if (!load_q(q)) break;
          const int ws = gc & 1;
          if (gc >= 2 && !tc::mbar_wait(wempty(ws), ((gc >> 1) - 1) & 1, P.err)) break;
          const uint32_t wbytes = (uint32_t)(min(G, P.Q - q * G) * P.H_I * 4);
          tc::mbar_arrive_expect_tx(wfull(ws), wbytes);
          tc::bulk_copy_g2s(tc::smem_u32(wsm + ws * NW), P.w + (int64_t)q * NW, wbytes, wfull(ws));
          // the next group's qI into L2, so that its load at the next change
          // is an L2 hit
          const int qn = P.interleave ? q + (int)gridDim.x : q + 1;
          if (qn < P.NG) {
            const int64_t r0 = (int64_t)qn * NW;
            const int64_t r1 = min((int64_t)(qn + 1) * NW, (int64_t)P.Q * P.H_I);
            tc::prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(P.qI) + r0 * P.c_I * 2,
                                 (uint32_t)((r1 - r0) * P.c_I * 2));
          }
        }
        last_q = q;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      const uint32_t idesc = tc::idesc_bf16_f32(kTileM, NW);
      UnitWalk<G> wk;
      wk.start(P, prefix, u0);
      int last_q = -1, gc = -1;
      for (int i = 0; i < nunits; ++i, wk.next()) {
        const int q = wk.q;
        if (q != last_q) {
          if (gc >= 0) tc::mma_commit(bempty(gc % QS));  // previous query's qI slot is free
          ++gc;
          if (!tc::mbar_wait(bfull(gc % QS), (gc / QS) & 1, P.err)) break;
          last_q = q;
        }
        const int s = i % S, a = i % NACC;
        if (!tc::mbar_wait(afull(s), (i / S) & 1, P.err)) break;
        if (i >= NACC && !tc::mbar_wait(accempty(a), ((i / NACC) - 1) & 1, P.err)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * NW);
        for (int kk = 0; kk < KCH * 4; ++kk) {
          const int ch = kk >> 2;
          const uint32_t off = (uint32_t)(kk & 3) * 32;
          tc::mma_bf16(d, tc::sdesc_kmajor_sw128(tc::smem_u32(sA + s * bytesA + ch * kChunkBytesA) + off),
                       tc::sdesc_kmajor_sw128(tc::smem_u32(sB + (gc % QS) * bytesB + ch * NW * 128) + off),
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
    UnitWalk<G> wk;
    wk.start(P, prefix, u0);
    if constexpr (G > 1) {
      constexpr int GH = G / 2;             // queries of the group this warp reduces
      const int j0 = (warp - 2) / 4 * GH;   // warps 2-5: the first half, 6-9: the second
      int last_q = -1, gce = -1;
      int64_t nv[GH];
      const float* wg = wsm;
      for (int i = 0; i < nunits; ++i, wk.next()) {
        const int g = wk.q;
        if (g != last_q) {
          // the previous group's weights are no longer read by this warp
          if (gce >= 0 && lane == 0) tc::mbar_arrive(wempty(gce & 1));
          ++gce;
          if (!tc::mbar_wait_warp(wfull(gce & 1), (gce >> 1) & 1, P.err)) break;
          wg = wsm + (gce & 1) * NW;
#pragma unroll
          for (int j = 0; j < GH; ++j) {
            const int q = g * G + j0 + j;
            nv[j] = q < P.Q ? dec_nvis(P, q) : 0;
          }
          last_q = g;
        }
        const int a = i % NACC;
        if (!tc::mbar_wait_warp(accfull(a), (i / NACC) & 1, P.err)) break;
        tc::tc_fence_after();
        float sc[GH];
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const int j = j0 + jj;
          sc[jj] = 0.f;
          const int q = g * G + j;
          if (q >= P.Q) continue;  // same for the whole warp
          // H_I = 64 here; the same four chains over the heads as for G = 1
          const float* wq = wg + j * 64;  // shared memory: one broadcast read per four heads
          float v[64];
          tc::tmem_ld64(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * NW + j * 64), v);
          float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 64; h += 4) {
            const float4 w4 = *reinterpret_cast<const float4*>(wq + h);
            acc4[0] = fmaf(w4.x, fmaxf(v[h], 0.f), acc4[0]);
            acc4[1] = fmaf(w4.y, fmaxf(v[h + 1], 0.f), acc4[1]);
            acc4[2] = fmaf(w4.z, fmaxf(v[h + 2], 0.f), acc4[2]);
            acc4[3] = fmaf(w4.w, fmaxf(v[h + 3], 0.f), acc4[3]);
          }
          sc[jj] = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(accempty(a));
        const int64_t sidx = wk.t * kTileM + row;
#pragma unroll
        for (int jj = 0; jj < GH; ++jj)
          if (sidx < nv[jj]) P.scores[(int64_t)(g * G + j0 + jj) * P.ld_scores + sidx] = sc[jj];
      }
    } else {
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
        const int a = i % NACC;
        if (!tc::mbar_wait_warp(accfull(a), (i / NACC) & 1, P.err)) break;
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
  // w rows are read as float4 by the register and grouped paths
  const bool w16 = (reinterpret_cast<uintptr_t>(w) & 15) == 0;
  // one sequence and many queries (prefill): groups of 4 queries share each key tile
  const int G = (nseq == 1 && H_I == 64 && c_I <= 128 && w16 && Q >= 64) ? 4 : 1;
  CUtensorMap tmK, tmQ;
  if (!encode_tmap_2d_bf16(&tmK, KI, (uint64_t)c_I, (uint64_t)nseq * ldK, (uint64_t)c_I * 2, 64,
                           kTileM) ||
      !encode_tmap_2d_bf16(&tmQ, qI, (uint64_t)c_I, (uint64_t)Q * H_I, (uint64_t)c_I * 2, 64,
                           (uint32_t)(G * H_I)))
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
  P.NG = (Q + G - 1) / G;
  P.qI = qI;
  P.interleave = P.NG >= 4 * nsm ? 1 : 0;
  const int nacc = G == 1 ? kDecAcc : kGrpAcc;
  uint32_t cols = 32;
  while (cols < (uint32_t)(nacc * G * H_I)) cols <<= 1;
  if (cols > 512) return cudaErrorInvalidValue;
  P.tmem_cols = cols;
  const int KCH = c_I / 64;
  const size_t prefix_ints = P.interleave ? 2 : (size_t)P.NG + 3;
  const int qslots = G > 1 ? GroupCfg<4>::qslots : GroupCfg<1>::qslots;
  const size_t fixed = 1024 + (size_t)qslots * KCH * G * H_I * 128 +
                       (G > 1 ? 2 * (size_t)G * H_I * 4 : 0) + prefix_ints * 4 + 256;
  const size_t per_stage = (size_t)KCH * kChunkBytesA;
  // the grouped kernel takes all of shared memory (one 64 KB query group + 4 stages)
  const size_t cap = G > 1 ? 227 * 1024 : 220 * 1024;
  if (fixed + 2 * per_stage > cap) return cudaErrorInvalidValue;
  const int stages = (int)std::min<size_t>(6, (cap - fixed) / per_stage);
  P.stages = stages;
  const size_t smem = fixed + stages * per_stage;
  auto kern = G > 1 ? index_decode_kernel<0, 4>
                    : (H_I == 64 && w16 ? index_decode_kernel<64, 1> : index_decode_kernel<0, 1>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  count_launches();
  return launch_pdl(kern, dim3(nsm), dim3(G > 1 ? GroupCfg<4>::threads : GroupCfg<1>::threads),
                    smem, s, tmK, tmQ, P);
}

}  // namespace csa
