// tc_attend_cluster.cu - shared-KV multi-query core attention on the
// 5th-generation tensor cores, one thread-block cluster per query token:
// compressed entries (selected by the indexer, or every visible one for HCA)
// plus the sliding window, one softmax whose denominator carries the sink,
// RMSNorm + RoPE on the queries and inverse RoPE on the outputs ("Evidence
// Ledger", CSA Eqs 18-19, Shared attention details Sec 2.3.3 and Eq 27;
// "DeepSeek-V4" study 03).
//
// Split. A query's key slots (selected entries, then the window) are cut into
// 64-key tiles; the C CTAs of its cluster take contiguous tile ranges. C
// depends only on the call's slot capacity (k or the cache length, plus the
// window), never on the batch, and the partial results are combined in rank
// order, so a query's output does not depend on the batch it is in.
//
// Per CTA, per tile (all 64 heads at once; the one shared-memory tile is both
// K and V, as the shared-KV MQA prescribes):
//   S  [head, key]   = Qhat (K-major A, K = 512 dims) x K_tile^T      M = 64
//   O^T[dim, head]  += K_tile^T (MN-major A, K = keys) x P^T (K-major B)
//                                                                   M = 128
// With M = 64, S occupies lanes 0-15 of each 32-lane TMEM quadrant: softmax
// thread (warp w, lane l < 16) owns head 16 w + l and its 64 keys, so a
// head's row max and sum stay in one thread. Key tiles, S and P are
// double-buffered; the MMA warp issues S(t+1) and PV(t) in whichever order
// their inputs become ready, so the gather of tile t+1 and the S MMA of tile
// t+1 overlap the softmax of tile t.
//
// Softmax. The per-head reference value m_h (log2 units) starts at the sink
// logit and is raised only when a tile's maximum exceeds it by more than
// 2^8 (then O^T and the running sums are rescaled): every weight exp(l -
// m_h) stays below 2^8, so the FP32 sums and the BF16 weights neither
// overflow nor lose range, and the result is the exact softmax up to
// rounding.
//
// Combine. Each CTA publishes (m_h, l_h) in shared memory; every CTA derives
// its weight 2^(m_h - M_h) / (2^(z'_h - M_h) + sum_r l_r,h 2^(m_r,h - M_h))
// and stores its scaled O^T slice for dims [r' 512/C, (r'+1) 512/C) into CTA
// r''s shared memory (distributed shared memory); CTA r' then sums the C
// slices in rank order, applies inverse RoPE and stores BF16. Every remote
// store lands before the second cluster barrier, and no CTA reads another's
// memory after it.
//
// Loads. The raw queries arrive by eight TMA tile loads (64 dims x 64 heads,
// 128-byte swizzle) straight into the Qhat layout and are normalised in
// place. Key rows are gathered 16 bytes a lane with cp.async (BF16) or
// dequantised through registers (FP8-mixed rows).
//
// Warps (288 threads): 0-3 prepare Qhat, then run the softmax; 4-7 gather key
// rows; 8 owns TMEM and issues the MMAs. All eight data warps share the
// combine.
#include <cooperative_groups.h>

#include "internal.h"
#include "tc_common.cuh"

namespace cg = cooperative_groups;

namespace csa {

namespace {

constexpr int kThreads = 288;
constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kTile = 64;           // keys per tile
constexpr int kChunks = kDim / 64;  // 64-dim chunks of a key row
constexpr int kMaxCluster = 8;
constexpr int kTilesPerCta = 5;     // target tiles per CTA when choosing the cluster size
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // O^T: 4 blocks (128 dims each) x 64 head columns
constexpr uint32_t kColS = 256;  // S: 2 buffers x 64 columns (lanes 0-15 of each quadrant)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

// shared memory map (offsets from the 1024-aligned base)
constexpr int kTileBytes = kChunks * kTile * 128;  // 64 KB: 8 chunks x 64 keys x 128 B
constexpr int kOffQ = 0;                           // Qhat: 8 chunks x 64 heads x 128 B
constexpr int kOffK = kOffQ + kChunks * 8192;      // 2 key tiles (reused by the combine)
constexpr int kOffP = kOffK + 2 * kTileBytes;      // 2 x 64 heads x 128 B
constexpr int kOffBar = kOffP + 2 * 8192;          // mbarriers
constexpr int kOffMisc = kOffBar + 128;            // TMEM slot, flags
constexpr int kOffAlpha = kOffMisc + 64;           // 2 x 64 floats
constexpr int kOffMl = kOffAlpha + 2 * kHeads * 4; // 64 x (m, l), read by the cluster
constexpr int kOffW = kOffMl + kHeads * 8;         // 64 floats: combine weights
constexpr int kOffRope = kOffW + kHeads * 4;       // 32 x (cos, sin) at the query position
constexpr int kOffVote = kOffRope + 32 * 8;        // 2 x 4 rescale votes
constexpr int kOffList = kOffVote + 64;            // compacted entry list (k ints)
constexpr int kStageBytes = kHeads * kDim * 4;     // combine staging, over the key tiles
static_assert(kStageBytes <= 2 * kTileBytes, "staging must fit the key tiles");
static_assert(kOffList % 16 == 0, "entry list must be 16-byte aligned");

enum Bar { kFull0 = 0, kSFull0 = 2, kPFull0 = 4, kEmpty0 = 6, kODone = 8, kQReady = 9, kQRaw = 10 };

struct Params {
  int Q, r, m, vis_offset, n_win, win_ring, kv_dt, k, dense, nseq, csize;
  double base;
  float eps;
  const __nv_bfloat16* q;
  const float* q_gain;
  const float* sink;
  const void* E;
  int64_t ldE;
  const int64_t* n_entries;
  const int32_t* idx;
  const __nv_bfloat16* win;
  int64_t ldW;
  const int32_t* seq_of_q;
  const int64_t* pos;
  __nv_bfloat16* O;
  int* err;
};

__device__ __forceinline__ void cluster_sync_all(int C) {
  if (C > 1) {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
  } else {
    __syncthreads();
  }
}

template <typename T>
__device__ __forceinline__ T* peer(T* p, int r, int C) {
  return C > 1 ? cg::this_cluster().map_shared_rank(p, r) : p;
}

__device__ __forceinline__ void st_shared_v4(uint32_t dst, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 2^x by the hardware approximation (relative error below 2^-22; the
// weights it produces are rounded to BF16 before use). 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int clamp_tile(int64_t v) {
  return (int)(v < 0 ? 0 : (v > kTile ? kTile : v));
}

__global__ void __launch_bounds__(kThreads, 1)
    attend_cluster_kernel(const __grid_constant__ CUtensorMap tq, Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = tc::smem_u32(sm + kOffQ);
  const uint32_t sK = tc::smem_u32(sm + kOffK);
  const uint32_t sP = tc::smem_u32(sm + kOffP);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  int* flags = reinterpret_cast<int*>(sm + kOffMisc + 16);  // [0] abort, [1] compacted count
  float* alpha_s = reinterpret_cast<float*>(sm + kOffAlpha);
  float* ml = reinterpret_cast<float*>(sm + kOffMl);
  float* wgt = reinterpret_cast<float*>(sm + kOffW);
  float2* rope = reinterpret_cast<float2*>(sm + kOffRope);
  int* vote = reinterpret_cast<int*>(sm + kOffVote);
  int32_t* list = reinterpret_cast<int32_t*>(sm + kOffList);
  auto bar = [&](int i) { return tc::smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();  // the previous kernel's writes (the selected entries) are visible from here on
  const int C = P.csize;
  const int rank = (int)(blockIdx.x % (unsigned)C);
  const int qi = (int)(blockIdx.x / (unsigned)C);
  const int b = P.seq_of_q[qi];
  const int64_t p = P.pos[qi];
  const bool valid_seq = b >= 0 && b < P.nseq;

  // ---- setup: barriers, TMEM, RoPE table, compacted entry list ----
  if (threadIdx.x == 0) {
    tc::mbar_init(bar(kFull0), 128);
    tc::mbar_init(bar(kFull0 + 1), 128);
    tc::mbar_init(bar(kSFull0), 1);
    tc::mbar_init(bar(kSFull0 + 1), 1);
    tc::mbar_init(bar(kPFull0), 128);
    tc::mbar_init(bar(kPFull0 + 1), 128);
    tc::mbar_init(bar(kEmpty0), 1);
    tc::mbar_init(bar(kEmpty0 + 1), 1);
    tc::mbar_init(bar(kODone), 1);
    tc::mbar_init(bar(kQReady), 128);
    tc::mbar_init(bar(kQRaw), 1);
    flags[0] = 0;
    flags[1] = 0;
    tc::fence_barrier_init();
  }
  if (warp == 8) {
    tc::tmem_alloc(tc::smem_u32(tslot), kTmemCols);
    if (lane < P.r / 2) {
      float cs, sn;
      rope_cs(p, lane, P.r, P.base, &cs, &sn);
      rope[lane] = make_float2(cs, sn);
    }
  }
  const int64_t ldE = P.ldE;
  int64_t nsel = 0;
  if (valid_seq) {
    if (P.dense) {
      nsel = n_visible(p, P.m, P.vis_offset, min(P.n_entries[b], ldE));
    } else if (warp < 8) {
      const int32_t* row = P.idx + (int64_t)qi * P.k;
      if ((P.k & 3) == 0) {
        for (int g = threadIdx.x; g < P.k / 4; g += 256)
          tc::cp_async16(tc::smem_u32(list + 4 * g), row + 4 * g);
      } else {
        for (int j = threadIdx.x; j < P.k; j += 256) list[j] = row[j];
      }
      tc::cp_async_wait_all();
      tc::named_bar(2, 256);
      // keep the slots that hold an entry inside the cache, in order, in
      // place: each 256-slot chunk is read before any of it is written, and
      // writes never pass the chunk's end
      __shared__ int wcount[8];
      int base_total = 0;
      for (int j0 = 0; j0 < P.k; j0 += 256) {
        const int j = j0 + threadIdx.x;
        const int32_t e = j < P.k ? list[j] : -1;
        const bool ok = e >= 0 && e < ldE;
        const unsigned msk = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) wcount[warp] = __popc(msk);
        tc::named_bar(2, 256);
        int before = 0, tot = 0;
        for (int w = 0; w < 8; ++w) {
          before += w < warp ? wcount[w] : 0;
          tot += wcount[w];
        }
        if (ok) list[base_total + before + __popc(msk & ((1u << lane) - 1u))] = e;
        base_total += tot;
        tc::named_bar(2, 256);
      }
      if (threadIdx.x == 0) flags[1] = base_total;
    }
  }
  tc::tc_fence_before();
  __syncthreads();  // barriers, entry list, RoPE table and TMEM address ready
  tc::tc_fence_after();
  const uint32_t tmem = *tslot;
  if (valid_seq && !P.dense) nsel = flags[1];

  // ---- this CTA's tiles ----
  const int64_t w0 = p - P.n_win + 1 > 0 ? p - P.n_win + 1 : 0;
  const int64_t nwin = (valid_seq && P.n_win > 0) ? p - w0 + 1 : 0;
  const int64_t nslots = valid_seq ? nsel + nwin : 0;
  const int64_t ntiles = (nslots + kTile - 1) / kTile;
  const int64_t t0 = ntiles * rank / C;
  const int T = (int)(ntiles * (rank + 1) / C - t0);
  const float sink2 = P.sink[threadIdx.x & (kHeads - 1)] * kLog2e;  // head = thread % 64
  if (threadIdx.x == 0 && T > 0) {
    // raw queries: 8 tiles of 64 dims x 64 heads, already in the Qhat layout
    tc::mbar_arrive_expect_tx(bar(kQRaw), 65536u);
    for (int c = 0; c < kChunks; ++c) tc::tma_load_2d(sQ + c * 8192, &tq, 64 * c, qi * kHeads, bar(kQRaw));
  }

  float ref = 0.f, lsum = 0.f;  // softmax state of warps 0-3, lanes 0-15 (head 16 w + l)
  if (warp < 4) {
    const int h = 16 * warp + (lane & 15);
    const bool owner = lane < 16;
    ref = P.sink[h] * kLog2e;
    if (T > 0) {
      // ---- Qhat = RoPE_p(RMSNorm(q_h) * gain) in BF16, in place: lane l
      //      holds dims 16 l .. 16 l + 15 of each head (granules 2 l, 2 l + 1
      //      of chunk l / 4); four heads at a time ----
      float gn[16];
      float2 rt[8];  // (cos, sin) of each pair of this lane, (1, 0) outside the rotated dims
      float qscale = 1.f;  // RMSNorm factor of head h when it is applied to the logits
#pragma unroll
      for (int i = 0; i < 16; ++i) gn[i] = P.q_gain ? P.q_gain[16 * lane + i] : 1.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int d = 16 * lane + 2 * i;
        rt[i] = d >= kDim - P.r ? rope[(d - (kDim - P.r)) >> 1] : make_float2(1.f, 0.f);
      }
      if (!tc::mbar_wait_warp(bar(kQRaw), 0, P.err)) flags[0] = 1;
      uint8_t* qch = sm + kOffQ + (lane >> 2) * 8192;
      const uint32_t g0 = (uint32_t)((2 * lane) & 7);
      if (P.q_gain == nullptr) {
        // Without a gain, RMSNorm scales each head by one factor, applied to
        // its logits instead: only the rotated dims change here, in place,
        // and the MMA starts as soon as they are written.
        if (16 * lane + 16 > kDim - P.r) {
          for (int j = 0; j < 16; ++j) {
            const uint32_t hh = (uint32_t)(16 * warp + j);
            uint4* p0 = reinterpret_cast<uint4*>(qch + tc::sw128_offset(hh, g0));
            uint4* p1 = reinterpret_cast<uint4*>(qch + tc::sw128_offset(hh, g0 + 1));
            const uint4 r0 = *p0, r1 = *p1;
            const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float a = bf16_lo(w[i]), bb = bf16_hi(w[i]);
              o[i] = pack_bf16x2(a * rt[i].x - bb * rt[i].y, a * rt[i].y + bb * rt[i].x);
            }
            *p0 = make_uint4(o[0], o[1], o[2], o[3]);
            *p1 = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
        __syncwarp();  // the rotated dims are read back below by every lane
        tc::fence_proxy_async();
        tc::mbar_arrive(bar(kQReady));
        // RMSNorm factors of this warp's heads (the rotation keeps the sum
        // of squares); lanes l and l + 16 keep head 16 w + l % 16's
        for (int j0 = 0; j0 < 16; j0 += 4) {
          float ss[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t hh = (uint32_t)(16 * warp + j0 + jj);
            const uint4 r0 = *reinterpret_cast<const uint4*>(qch + tc::sw128_offset(hh, g0));
            const uint4 r1 = *reinterpret_cast<const uint4*>(qch + tc::sw128_offset(hh, g0 + 1));
            const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            float s2 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
              s2 = fmaf(lo, lo, fmaf(hi, hi, s2));
            }
            ss[jj] = s2;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) ss[jj] += __shfl_xor_sync(0xffffffffu, ss[jj], o);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            if ((lane & 15) == j0 + jj) qscale = rsqrtf(ss[jj] * (1.f / (float)kDim) + P.eps);
        }
      } else {
        for (int j0 = 0; j0 < 16; j0 += 4) {
          uint4* ptr[4][2];
          uint4 raw[4][2];
          float ss[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t hh = (uint32_t)(16 * warp + j0 + jj);
            ptr[jj][0] = reinterpret_cast<uint4*>(qch + tc::sw128_offset(hh, g0));
            ptr[jj][1] = reinterpret_cast<uint4*>(qch + tc::sw128_offset(hh, g0 + 1));
            raw[jj][0] = *ptr[jj][0];
            raw[jj][1] = *ptr[jj][1];
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t w[8] = {raw[jj][0].x, raw[jj][0].y, raw[jj][0].z, raw[jj][0].w,
                                   raw[jj][1].x, raw[jj][1].y, raw[jj][1].z, raw[jj][1].w};
            float s2 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
              s2 = fmaf(lo, lo, fmaf(hi, hi, s2));
            }
            ss[jj] = s2;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) ss[jj] += __shfl_xor_sync(0xffffffffu, ss[jj], o);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const float inv = rsqrtf(ss[jj] * (1.f / (float)kDim) + P.eps);
            const uint32_t w[8] = {raw[jj][0].x, raw[jj][0].y, raw[jj][0].z, raw[jj][0].w,
                                   raw[jj][1].x, raw[jj][1].y, raw[jj][1].z, raw[jj][1].w};
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float a = bf16_lo(w[i]) * inv * gn[2 * i];
              const float bb = bf16_hi(w[i]) * inv * gn[2 * i + 1];
              o[i] = pack_bf16x2(a * rt[i].x - bb * rt[i].y, a * rt[i].y + bb * rt[i].x);
            }
            *ptr[jj][0] = make_uint4(o[0], o[1], o[2], o[3]);
            *ptr[jj][1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
        tc::fence_proxy_async();
        tc::mbar_arrive(bar(kQReady));
      }

      // ---- softmax over this CTA's tiles ----
      const float sc = kLog2e / sqrtf((float)kDim) * qscale;
      const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
      for (int t = 0; t < T; ++t) {
        const int buf = t & 1;
        const uint32_t par = (uint32_t)(t >> 1) & 1u;
        const int nvalid = clamp_tile(nslots - (t0 + t) * kTile);  // keys of the tile that exist
        if (!tc::mbar_wait_warp(bar(kSFull0 + buf), par, P.err)) flags[0] = 1;
        tc::tc_fence_after();
        float s[64];
        tc::tmem_ld32(tmem + lane_addr + kColS + buf * 64, s);
        tc::tmem_ld32(tmem + lane_addr + kColS + buf * 64 + 32, s + 32);
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          s[i] = i < nvalid ? s[i] * sc : -INFINITY;
          m8[i & 7] = fmaxf(m8[i & 7], s[i]);
        }
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        float a = 1.f;
        const bool need = owner && mx > ref + kRescaleLog2;
        if (need) {
          a = ex2(ref - mx);
          ref = mx;
        }
        if (owner) alpha_s[buf * kHeads + h] = a;
        const int anyw = __any_sync(0xffffffffu, need) ? 1 : 0;
        if (lane == 0) vote[buf * 4 + warp] = anyw;
        tc::named_bar(1, 128);
        const bool any = (vote[buf * 4] | vote[buf * 4 + 1] | vote[buf * 4 + 2] | vote[buf * 4 + 3]) != 0;
        if (any && t > 0) {
          // O^T holds tiles 0..t-1: once the last of them is in, scale head
          // column h by alpha_h (each thread: its dim of every block)
          if (!tc::mbar_wait_warp(bar(kODone), (uint32_t)(t - 1) & 1u, P.err)) flags[0] = 1;
          tc::tc_fence_after();
          const float* al = alpha_s + buf * kHeads;
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
              float o[32];
              const uint32_t ta = tmem + lane_addr + kColO + blk * kHeads + hf * 32;
              tc::tmem_ld32(ta, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= al[hf * 32 + i];
              tc::tmem_st32(ta, o);
            }
          }
        }
        if (owner) {
          // weights in BF16: row h of P, keys 0..63 = granules 0..7
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int gi = 0; gi < 8; ++gi) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float p0 = ex2(s[8 * gi + 2 * i] - ref), p1 = ex2(s[8 * gi + 2 * i + 1] - ref);
              l4[i] += p0 + p1;
              pk[i] = pack_bf16x2(p0, p1);
            }
            st_shared_v4(sP + buf * 8192 + tc::sw128_offset((uint32_t)h, (uint32_t)gi), pk[0], pk[1],
                         pk[2], pk[3]);
          }
          lsum = lsum * a + ((l4[0] + l4[1]) + (l4[2] + l4[3]));
        }
        tc::fence_proxy_async();
        tc::tc_fence_before();
        tc::mbar_arrive(bar(kPFull0 + buf));
      }
      if (!tc::mbar_wait_warp(bar(kODone), (uint32_t)(T - 1) & 1u, P.err)) flags[0] = 1;
      tc::tc_fence_after();
    }
    if (owner) {
      ml[2 * h] = ref;
      ml[2 * h + 1] = T > 0 ? lsum : 0.f;
    }
  } else if (warp < 8) {
    // ---- gather of key rows: warp 4 + i takes rows i, i + 4, ..., 16 B a lane ----
    const int pw = warp - 4;
    const int row_bytes_e = (int)row_bytes(P.kv_dt, kDim);
    const bool mixed_kv = P.kv_dt == CSA_FP8_MIXED;
    for (int t = 0; t < T; ++t) {
      const int buf = t & 1;
      if (t >= 2 && !tc::mbar_wait_warp(bar(kEmpty0 + buf), (uint32_t)((t >> 1) - 1) & 1u, P.err))
        flags[0] = 1;
      const uint32_t base = sK + buf * kTileBytes;
      for (int rr = pw; rr < kTile; rr += 4) {
        const int64_t slot = (t0 + t) * kTile + rr;
        const uint8_t* row = nullptr;
        bool mixed = false;
        if (slot < nslots) {
          if (slot < nsel) {
            const int64_t e = P.dense ? slot : (int64_t)list[slot];
            row = reinterpret_cast<const uint8_t*>(P.E) + ((int64_t)b * ldE + e) * row_bytes_e;
            mixed = mixed_kv;
          } else {
            const int64_t j = w0 + (slot - nsel);
            const int64_t wr = P.win_ring ? (j % P.n_win) : j;
            if (wr < P.ldW)
              row = reinterpret_cast<const uint8_t*>(P.win + ((int64_t)b * P.ldW + wr) * kDim);
          }
        }
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int g = lane + 32 * gg;  // 16-byte granule of the row: dims 8 g .. 8 g + 7
          const uint32_t dst = base + (g >> 3) * 8192 + tc::sw128_offset((uint32_t)rr, (uint32_t)(g & 7));
          if (row == nullptr) {
            st_shared_v4(dst, 0u, 0u, 0u, 0u);
          } else if (!mixed) {
            tc::cp_async16(dst, row + 16 * g);
          } else if (8 * g < kMixedFp8Dims) {
            const float sc = *reinterpret_cast<const float*>(row + kMixedScaleOffset);
            const uint2 codes = *reinterpret_cast<const uint2*>(row + 8 * g);
            auto dq = [&](uint32_t w, int i) { return e4m3_to_f32(byte_of(w, i)) * sc; };
            st_shared_v4(dst, pack_bf16x2(dq(codes.x, 0), dq(codes.x, 1)),
                         pack_bf16x2(dq(codes.x, 2), dq(codes.x, 3)),
                         pack_bf16x2(dq(codes.y, 0), dq(codes.y, 1)),
                         pack_bf16x2(dq(codes.y, 2), dq(codes.y, 3)));
          } else {
            const uint4 v = *reinterpret_cast<const uint4*>(row + kMixedFp8Dims +
                                                            2 * (8 * g - kMixedFp8Dims));
            st_shared_v4(dst, v.x, v.y, v.z, v.w);
          }
        }
      }
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::mbar_arrive(bar(kFull0 + buf));
    }
  } else if (lane == 0 && T > 0) {
    // ---- MMA issue: S(t) once tile t is in and PV(t-2) issued, PV(t) once
    //      its weights are written; whichever is ready first ----
    if (!tc::mbar_wait(bar(kQReady), 0, P.err)) flags[0] = 1;
    const uint32_t id_s = tc::idesc_bf16_f32(64, kTile);
    const uint32_t id_pv = tc::idesc_bf16_f32_major(128, kHeads, 1, 0);
    int ns = 0, npv = 0;
    uint64_t t_idle = 0;
    while (npv < T) {
      bool did = false;
      if (ns < T && ns <= npv + 1 && tc::mbar_test(bar(kFull0 + (ns & 1)), (uint32_t)(ns >> 1) & 1u)) {
        const int buf = ns & 1;
        tc::tc_fence_after();
        const uint32_t kb = sK + buf * kTileBytes;
        const uint64_t dq = tc::sdesc_kmajor_sw128(sQ), dk = tc::sdesc_kmajor_sw128(kb);
        const uint32_t ds = tmem + kColS + buf * 64;
#pragma unroll 4
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint32_t o = (uint32_t)((kk >> 2) * 8192 + (kk & 3) * 32);
          tc::mma_bf16(ds, tc::sdesc_add(dq, o), tc::sdesc_add(dk, o), id_s, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar(kSFull0 + buf));
        ++ns;
        did = true;
      }
      if (npv < ns && tc::mbar_test(bar(kPFull0 + (npv & 1)), (uint32_t)(npv >> 1) & 1u)) {
        const int buf = npv & 1;
        tc::tc_fence_after();
        const uint32_t kb = sK + buf * kTileBytes;
        const uint64_t da = tc::sdesc_mnmajor_sw128(kb, 8192, 1024);
        const uint64_t db = tc::sdesc_kmajor_sw128(sP + buf * 8192);
        const uint32_t acc0 = npv > 0 ? 1u : 0u;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            tc::mma_bf16(tmem + kColO + blk * kHeads, tc::sdesc_add(da, (2 * blk) * 8192 + kk * 2048),
                         tc::sdesc_add(db, kk * 32), id_pv, kk > 0 ? 1u : acc0);
        }
        tc::mma_commit(bar(kEmpty0 + buf));
        tc::mma_commit(bar(kODone));
        ++npv;
        did = true;
      }
      if (did) {
        t_idle = 0;
        continue;
      }
      __nanosleep(64);  // leave the issue slots to the softmax warps
      if (t_idle == 0) {
        t_idle = tc::global_timer_ns();
      } else if (tc::global_timer_ns() - t_idle > tc::kWaitLimitNs) {
        record_device_error(P.err, CSA_ERR_TIMEOUT);
        flags[0] = 1;
        break;
      }
    }
  }

  // ---- combine over the cluster ----
  __syncwarp();
  tc::tc_fence_before();
  cluster_sync_all(C);  // every CTA's (m, l) published; its MMAs are complete
  tc::tc_fence_after();
  if (threadIdx.x < kHeads) {
    const int hh = threadIdx.x;
    float M = sink2;
    for (int r = 0; r < C; ++r) M = fmaxf(M, peer(ml, r, C)[2 * hh]);
    float den = exp2f(sink2 - M);
    for (int r = 0; r < C; ++r) {
      const float* pm = peer(ml, r, C);
      den += pm[2 * hh + 1] * exp2f(pm[2 * hh] - M);
    }
    wgt[hh] = T > 0 ? exp2f(ml[2 * hh] - M) / den : 0.f;
  }
  __syncthreads();
  // staging of CTA r': [C][16 head quads][D dims][4 heads], slot r holding
  // CTA r's scaled O for the dims r' owns; every CTA stores its slices into
  // their owners, 16 bytes (4 heads of one dim) at a time
  const int D = kDim / C;
  float* stage = reinterpret_cast<float*>(sm + kOffK);
  if (warp < 8) {
    const int quad = warp & 3;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
#pragma unroll 1
    for (int bi = 0; bi < 2; ++bi) {
      const int blk = 2 * (warp >> 2) + bi;
      const int d = blk * 128 + 32 * quad + lane;
      const int own = d / D;
      float* dst = peer(stage, own, C) + ((int64_t)rank * 16 * D + (d - own * D)) * 4;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        float o[32];
        if (T > 0) {
          tc::tmem_ld32(tmem + lane_addr + kColO + blk * kHeads + hf * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4) {
          const int h0 = hf * 32 + 4 * g4;
          *reinterpret_cast<float4*>(dst + (int64_t)(h0 / 4) * D * 4) =
              make_float4(o[4 * g4] * wgt[h0], o[4 * g4 + 1] * wgt[h0 + 1],
                          o[4 * g4 + 2] * wgt[h0 + 2], o[4 * g4 + 3] * wgt[h0 + 3]);
        }
      }
    }
  }
  cluster_sync_all(C);  // every slice is in its owner's staging
  {
    // sum the C slices of this CTA's dims in rank order, inverse RoPE, BF16.
    // Item = (head quad, dim); the 32 lanes of a warp take 32 consecutive
    // dims (16 D and 288 are multiples of 32), so the partner of a rotated
    // pair (d, d ^ 1) is the neighbouring lane.
    const int items = 16 * D;
    for (int it = threadIdx.x; it < items; it += kThreads) {
      const int hq = it / D, dd = it % D;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = 0; r < C; ++r) {
        const float4 v = *reinterpret_cast<const float4*>(stage + ((int64_t)(r * 16 + hq) * D + dd) * 4);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const int d = rank * D + dd;
      float4 oth;
      oth.x = __shfl_xor_sync(0xffffffffu, acc.x, 1);
      oth.y = __shfl_xor_sync(0xffffffffu, acc.y, 1);
      oth.z = __shfl_xor_sync(0xffffffffu, acc.z, 1);
      oth.w = __shfl_xor_sync(0xffffffffu, acc.w, 1);
      if (d >= kDim - P.r) {
        // rotate the pair (d & ~1, d | 1) by -p
        const float2 tr = rope[(d - (kDim - P.r)) >> 1];
        const float cs = tr.x, sn = (d & 1) ? -tr.y : tr.y;
        acc = make_float4(acc.x * cs + oth.x * sn, acc.y * cs + oth.y * sn, acc.z * cs + oth.z * sn,
                          acc.w * cs + oth.w * sn);
      }
      __nv_bfloat16* op = P.O + ((int64_t)qi * kHeads + 4 * hq) * kDim + d;
      op[0] = __float2bfloat16_rn(acc.x);
      op[kDim] = __float2bfloat16_rn(acc.y);
      op[2 * kDim] = __float2bfloat16_rn(acc.z);
      op[3 * kDim] = __float2bfloat16_rn(acc.w);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int attend_cluster_size(int64_t max_slots) {
  const int64_t tiles = (max_slots + kTile - 1) / kTile;
  int c = 1;
  while (c < kMaxCluster && (int64_t)c * kTilesPerCta < tiles) c *= 2;
  return c;
}

bool attend_cluster_supported(int q_dt, int kv_dt, int c, int H_q, int k, int rope_dims) {
  return q_dt == CSA_BF16 && (kv_dt == CSA_BF16 || kv_dt == CSA_FP8_MIXED) && c == kDim &&
         H_q == kHeads && k <= CSA_MAX_TOPK && rope_dims % 4 == 0 && rope_dims <= 64;
}

cudaError_t launch_attend_cluster(const csa_geom& g, int kv_dt, const void* q, const float* q_gain,
                                  const float* sink, const void* E, int64_t ldE, int nseq,
                                  const int64_t* n_entries, const int32_t* idx, int k, int dense,
                                  const void* win, int64_t ldW, const int32_t* seq_of_q,
                                  const int64_t* pos, int Q, void* O, cudaStream_t s) {
  if (Q == 0) return cudaSuccess;
  const int64_t max_slots = (dense ? ldE : (int64_t)k) + g.n_win;
  Params P{};
  P.Q = Q;
  P.r = g.rope_dims;
  P.m = g.m;
  P.vis_offset = g.vis_offset;
  P.n_win = g.n_win;
  P.win_ring = g.win_ring;
  P.kv_dt = kv_dt;
  P.k = k;
  P.dense = dense;
  P.nseq = nseq;
  P.csize = attend_cluster_size(max_slots);
  P.base = g.rope_base;
  P.eps = g.eps;
  P.q = reinterpret_cast<const __nv_bfloat16*>(q);
  P.q_gain = q_gain;
  P.sink = sink;
  P.E = E;
  P.ldE = ldE;
  P.n_entries = n_entries;
  P.idx = idx;
  P.win = reinterpret_cast<const __nv_bfloat16*>(win);
  P.ldW = ldW;
  P.seq_of_q = seq_of_q;
  P.pos = pos;
  P.O = reinterpret_cast<__nv_bfloat16*>(O);
  P.err = device_error_ptr();
  // the queries [Q * 64 heads, 512] in tiles of 64 dims x 64 heads
  CUtensorMap tq{};
  if ((uint64_t)Q * kHeads >= (1ull << 31) ||
      !encode_tmap_2d_bf16(&tq, q, kDim, (uint64_t)Q * kHeads, kDim * 2, 64, 64))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)kOffList + (dense ? 0 : (size_t)k * 4) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attend_cluster_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)Q * P.csize;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launches();
  return cudaLaunchKernelEx(&cfg, attend_cluster_kernel, tq, P);
}

}  // namespace csa
