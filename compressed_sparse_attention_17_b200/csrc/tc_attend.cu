// tc_attend.cu - shared-KV multi-query core attention on the 5th-generation
// tensor cores: compressed entries (selected by the indexer, or every
// visible one for HCA) plus the sliding window, one softmax whose
// denominator carries the sink, RMSNorm + RoPE on the queries and inverse
// RoPE on the outputs ("Evidence Ledger", CSA Eqs 18-19, Shared attention
// details Sec 2.3.3 and Eq 27; "DeepSeek-V4" study 03).
//
// Orientation. One CTA serves one query token (all 64 heads). Keys are
// gathered 128 at a time into a 128-byte-swizzled K-major tile
// sK[key][dim]; the heads are the MMA's N dimension:
//   S^T[key, head]  = sK (K-major A, K = dims) x Qhat (K-major B)
//   O^T[dim, head] += sK^T (MN-major A, K = keys) x P^T (MN-major B)
// so the one shared-memory tile is both K and V, as the shared-KV MQA
// prescribes. S^T takes 64 TMEM columns, O^T 4 x 64 (512 dims).
//
// Softmax. Each epilogue thread owns one key (TMEM lane) and its 64 head
// logits. The per-head reference value m_h starts at the sink logit and is
// raised only when a tile's maximum exceeds it by more than 2^8 (then O^T
// and the running sums are rescaled): every weight exp(l - m_h) stays below
// 2^8, so the FP32 sums and the BF16 weights neither overflow nor lose
// range, and the result is the exact softmax up to rounding.
//
// This kernel serves large batches (prefill), one CTA per query; small
// batches run on the cluster kernel (tc_attend_cluster.cu), which splits a
// query's keys over several CTAs.
//
// Warps (288 threads): 0-3 gather key rows (cp.async) and prepare Qhat with
// 4-7; 4-7 run the softmax and the output epilogue (TMEM lane quadrant =
// warp % 4); 8 owns TMEM and issues the MMAs.
#include "internal.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kThreads = 288;
constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kTile = 128;          // keys per tile
constexpr int kChunks = kDim / 64;  // 64-dim chunks of a key row
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;       // S^T: 64 columns
constexpr uint32_t kColO = 256;     // O^T: 4 blocks x 64 columns
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

// shared memory map (offsets from the 1024-aligned base)
constexpr int kOffK = 0;                           // 8 x 16 KB
constexpr int kOffQ = kOffK + kChunks * 16384;     // 8 x 8 KB
constexpr int kOffP = kOffQ + kChunks * 8192;      // 16 KB
constexpr int kOffRed = kOffP + 16384;             // 4 x 64 floats
constexpr int kOffRef = kOffRed + 4 * kHeads * 4;  // 64 floats (log2 units)
constexpr int kOffAlpha = kOffRef + kHeads * 4;    // 64 floats
constexpr int kOffMisc = kOffAlpha + kHeads * 4;   // barriers, tmem slot, flags
constexpr int kOffRope = kOffMisc + 64;            // 32 x (cos, sin) at the query position
constexpr int kOffInv = kOffRope + 32 * 8;         // 64 floats: 1 / denominator per head
constexpr int kOffList = kOffInv + kHeads * 4;     // compacted entry list
constexpr int kSmemFixed = kOffList + 1024;        // + alignment slack

struct Params {
  int Q, r, m, vis_offset, n_win, win_ring, kv_dt, k, dense, nseq;
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

__device__ __forceinline__ int order_int(float f) {
  int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float from_order_int(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF);
}

__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sK = tc::smem_u32(sm + kOffK);
  const uint32_t sQ = tc::smem_u32(sm + kOffQ);
  const uint32_t sP = tc::smem_u32(sm + kOffP);
  float* red = reinterpret_cast<float*>(sm + kOffRed);
  float* ref2 = reinterpret_cast<float*>(sm + kOffRef);
  float* alpha = reinterpret_cast<float*>(sm + kOffAlpha);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffMisc + 16);
  int* flags = reinterpret_cast<int*>(sm + kOffMisc + 32);  // [0] abort, [1] rescale, [2] nvalid
  int32_t* list = reinterpret_cast<int32_t*>(sm + kOffList);
  float2* rope = reinterpret_cast<float2*>(sm + kOffRope);
  float* inv_den = reinterpret_cast<float*>(sm + kOffInv);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();  // the previous kernel's writes (the selected entries) are visible from here on
  const int qi = blockIdx.x;
  const int b = P.seq_of_q[qi];
  const int64_t p = P.pos[qi];
  const bool valid_seq = b >= 0 && b < P.nseq;
  const uint32_t s_bar = tc::smem_u32(&bars[0]);
  const uint32_t o_bar = tc::smem_u32(&bars[1]);

  // ---- setup: barriers, TMEM, compacted entry list ----
  if (threadIdx.x == 0) {
    tc::mbar_init(s_bar, 1);
    tc::mbar_init(o_bar, 1);
    flags[0] = 0;
    flags[1] = 0;
    tc::fence_barrier_init();
  }
  if (warp == 8) {
    tc::tmem_alloc(tc::smem_u32(tslot), kTmemCols);
    // cos/sin of the query position for each rotated pair (FP64 angles)
    if (lane < P.r / 2) {
      float cs, sn;
      rope_cs(p, lane, P.r, P.base, &cs, &sn);
      rope[lane] = make_float2(cs, sn);
    }
  }
  const int64_t ldE = P.ldE;
  const int row_bytes_e = (int)row_bytes(P.kv_dt, kDim);
  // ---- stage the raw queries (64 KB, linear) and the index row in shared
  //      memory with one burst of asynchronous copies ----
  if (valid_seq && warp < 8) {
    {
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(P.q + (int64_t)qi * kHeads * kDim);
      for (int g = threadIdx.x; g < kHeads * kDim * 2 / 16; g += 256) tc::cp_async16(sQ + 16 * g, qsrc + 16 * g);
    }
    if (!P.dense) {
      const int32_t* row = P.idx + (int64_t)qi * P.k;
      if ((P.k & 3) == 0) {
        for (int g = threadIdx.x; g < P.k / 4; g += 256) tc::cp_async16(tc::smem_u32(list + 4 * g), row + 4 * g);
      } else {
        for (int j = threadIdx.x; j < P.k; j += 256) list[j] = row[j];
      }
    }
    tc::cp_async_wait_all();
    tc::named_bar(2, 256);
  }
  int64_t nsel = 0;
  if (valid_seq) {
    if (P.dense) {
      nsel = n_visible(p, P.m, P.vis_offset, min(P.n_entries[b], ldE));
    } else if (warp < 8) {
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
      if (threadIdx.x == 0) flags[2] = base_total;
    }
  }
  if (threadIdx.x < kHeads) ref2[threadIdx.x] = P.sink[threadIdx.x] * kLog2e;
  tc::tc_fence_before();
  __syncthreads();  // entry list, RoPE table and TMEM address ready
  tc::tc_fence_after();
  const uint32_t tmem = *tslot;
  if (valid_seq && !P.dense) nsel = flags[2];

  // ---- key slots of this CTA ----
  const int64_t w0 = p - P.n_win + 1 > 0 ? p - P.n_win + 1 : 0;
  const int64_t nwin = (valid_seq && P.n_win > 0) ? p - w0 + 1 : 0;
  const int64_t nslots = valid_seq ? nsel + nwin : 0;
  const int64_t ntiles = (nslots + kTile - 1) / kTile;
  const int64_t t_begin = 0, t_end = ntiles;

  // gather of key tile t into sK by warps 0-7 (one 1 KB row per warp-step,
  // 16 bytes per lane and instruction; asynchronous for BF16 rows)
  auto issue_gather = [&](int64_t t) {
    for (int rr = warp; rr < kTile; rr += 8) {
      const int64_t slot = t * kTile + rr;
      const uint8_t* row = nullptr;
      bool mixed = false;
      if (slot < nslots) {
        if (slot < nsel) {
          const int64_t e = P.dense ? slot : (int64_t)list[slot];
          row = reinterpret_cast<const uint8_t*>(P.E) + ((int64_t)b * ldE + e) * row_bytes_e;
          mixed = P.kv_dt == CSA_FP8_MIXED;
        } else {
          const int64_t j = w0 + (slot - nsel);
          const int64_t wr = P.win_ring ? (j % P.n_win) : j;
          if (wr < P.ldW)
            row = reinterpret_cast<const uint8_t*>(P.win + ((int64_t)b * P.ldW + wr) * kDim);
        }
      }
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = lane + 32 * gg;  // 16-byte granule of the row: dims 8g .. 8g+7
        const uint32_t dst = sK + (g >> 3) * 16384 + tc::sw128_offset((uint32_t)rr, (uint32_t)(g & 7));
        if (row == nullptr) {
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0) : "memory");
        } else if (!mixed) {
          tc::cp_async16(dst, row + 16 * g);
        } else {
          uint32_t o[4];
          if (8 * g < kMixedFp8Dims) {
            const float sc = *reinterpret_cast<const float*>(row + kMixedScaleOffset);
            const uint2 codes = *reinterpret_cast<const uint2*>(row + 8 * g);
            const uint8_t* cb = reinterpret_cast<const uint8_t*>(&codes);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              __nv_bfloat162 pr = __floats2bfloat162_rn(e4m3_to_f32(cb[2 * i]) * sc,
                                                        e4m3_to_f32(cb[2 * i + 1]) * sc);
              o[i] = *reinterpret_cast<uint32_t*>(&pr);
            }
          } else {
            const uint4 v = *reinterpret_cast<const uint4*>(row + kMixedFp8Dims + 2 * (8 * g - kMixedFp8Dims));
            o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]),
                       "r"(o[2]), "r"(o[3])
                       : "memory");
        }
      }
    }
  };
  // the first tile's rows travel while the queries are normalised
  if (warp < 8 && t_begin < t_end) issue_gather(t_begin);

  // ---- q-hat = RoPE_p(RMSNorm(q_h) * gain) in BF16, K-major swizzled, in
  //      place: every raw value is read before any swizzled row is written ----
  if (valid_seq && warp < 8) {
    uint32_t raw[8][8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int h = warp + 8 * j;
      const uint4 a = *reinterpret_cast<const uint4*>(sm + kOffQ + h * 1024 + 32 * lane);
      const uint4 c2 = *reinterpret_cast<const uint4*>(sm + kOffQ + h * 1024 + 32 * lane + 16);
      raw[j][0] = a.x; raw[j][1] = a.y; raw[j][2] = a.z; raw[j][3] = a.w;
      raw[j][4] = c2.x; raw[j][5] = c2.y; raw[j][6] = c2.z; raw[j][7] = c2.w;
    }
    tc::named_bar(2, 256);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int h = warp + 8 * j;
      float v[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[j][i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) ss += v[i] * v[i];
      ss = warp_sum(ss);
      const float inv = 1.f / sqrtf(ss / (float)kDim + P.eps);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const int d = 16 * lane + i;
        float a = v[i] * inv * (P.q_gain ? P.q_gain[d] : 1.f);
        float bb = v[i + 1] * inv * (P.q_gain ? P.q_gain[d + 1] : 1.f);
        if (d >= kDim - P.r) {
          const float2 t = rope[(d - (kDim - P.r)) >> 1];
          const float a2 = a * t.x - bb * t.y;
          bb = a * t.y + bb * t.x;
          a = a2;
        }
        v[i] = a;
        v[i + 1] = bb;
      }
      // dims 16*lane .. +15 = granules 2*lane, 2*lane+1 of chunk lane/4
      const int chunk = lane >> 2;
#pragma unroll
      for (int gq = 0; gq < 2; ++gq) {
        const uint32_t g = (uint32_t)((2 * lane + gq) & 7);
        __nv_bfloat162 pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pk[i] = __floats2bfloat162_rn(v[8 * gq + 2 * i], v[8 * gq + 2 * i + 1]);
        const uint32_t dst = sQ + chunk * 8192 + tc::sw128_offset((uint32_t)h, g);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                     "r"(*reinterpret_cast<uint32_t*>(&pk[0])), "r"(*reinterpret_cast<uint32_t*>(&pk[1])),
                     "r"(*reinterpret_cast<uint32_t*>(&pk[2])), "r"(*reinterpret_cast<uint32_t*>(&pk[3]))
                     : "memory");
      }
    }
  }
  // the bulk copy of q-hat must have landed before any MMA and before exit
  const float scale2 = kLog2e / sqrtf((float)kDim);
  // softmax/epilogue layout: warps 0-7, TMEM lane quadrant = warp % 4 (one
  // key, or one output dim, per lane), head half = warp / 4 (32 heads)
  const int quad = warp & 3, half = (warp >> 2) & 1;
  const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
  float lsum[32];
#pragma unroll
  for (int h = 0; h < 32; ++h) lsum[h] = 0.f;

  uint32_t phase = 0;
  for (int64_t t = t_begin; t < t_end; ++t) {
    if (warp < 8) {
      if (t > t_begin) issue_gather(t);
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    // ---- S^T = K Qhat^T ----
    if (warp == 8 && lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, kHeads);
      const uint64_t dk = tc::sdesc_kmajor_sw128(sK), dq = tc::sdesc_kmajor_sw128(sQ);
#pragma unroll 4
      for (int kk = 0; kk < kDim / 16; ++kk) {
        const uint32_t ch = kk >> 2, off = (uint32_t)(kk & 3) * 32;
        tc::mma_bf16(tmem + kColS, tc::sdesc_add(dk, ch * 16384 + off), tc::sdesc_add(dq, ch * 8192 + off),
                     idesc, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(s_bar);
    }
    // ---- softmax on the key lanes: 32 heads per thread ----
    if (warp < 8) {
      const int key = quad * 32 + lane;
      const int64_t slot = t * kTile + key;
      const bool kvalid = slot < nslots;
      float s[32];
      const bool ok = tc::mbar_wait_warp(s_bar, phase, P.err);
      if (!ok) flags[0] = 1;
      tc::tc_fence_after();
      tc::tmem_ld32(tmem + lane_addr + kColS + half * 32, s);
#pragma unroll
      for (int h = 0; h < 32; ++h) s[h] = kvalid ? s[h] * scale2 : -INFINITY;
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        const int mx = __reduce_max_sync(0xffffffffu, order_int(s[h]));
        if (lane == 0) red[quad * kHeads + half * 32 + h] = from_order_int(mx);
      }
      tc::named_bar(1, 256);
      if (warp < 2) {
        const int h = threadIdx.x;  // 0..63
        const float tmax = fmaxf(fmaxf(red[h], red[kHeads + h]), fmaxf(red[2 * kHeads + h], red[3 * kHeads + h]));
        float a = 1.f;
        if (tmax > ref2[h] + kRescaleLog2) {
          a = exp2f(ref2[h] - tmax);
          ref2[h] = tmax;
          flags[1] = 1;
        }
        alpha[h] = a;
      }
      tc::named_bar(1, 256);
      // weights in BF16: key row of 128 bytes, this half's 4 granules
      const float* rf = ref2 + half * 32;
      const float* al = alpha + half * 32;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int h = 8 * g + 2 * i;
          const float p0 = exp2f(s[h] - rf[h]), p1 = exp2f(s[h + 1] - rf[h + 1]);
          lsum[h] = lsum[h] * al[h] + p0;
          lsum[h + 1] = lsum[h + 1] * al[h + 1] + p1;
          __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<uint32_t*>(&pr);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sP + tc::sw128_offset((uint32_t)key, (uint32_t)(4 * half + g))),
                     "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                     : "memory");
      }
      // rescale the accumulated O^T: this lane's dim in each block, this half's heads
      if (flags[1] && t > t_begin) {
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          float o[32];
          const uint32_t ta = tmem + lane_addr + kColO + blk * kHeads + half * 32;
          tc::tmem_ld32(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= al[i];
          tc::tmem_st32(ta, o);
        }
      }
      tc::fence_proxy_async();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (threadIdx.x == 0) flags[1] = 0;
    // ---- O^T += K^T P^T ----
    if (warp == 8 && lane == 0) {
      if (!flags[0]) {
        const uint32_t idesc = tc::idesc_bf16_f32_major(128, kHeads, 1, 1);
        const uint64_t da = tc::sdesc_mnmajor_sw128(sK, 16384, 1024);
        const uint64_t db = tc::sdesc_mnmajor_sw128(sP, 8192, 1024);
        const uint32_t acc0 = t > t_begin ? 1u : 0u;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            tc::mma_bf16(tmem + kColO + blk * kHeads, tc::sdesc_add(da, (2 * blk) * 16384 + kk * 2048),
                         tc::sdesc_add(db, kk * 2048), idesc, kk > 0 ? 1u : acc0);
        }
      }
      tc::mma_commit(o_bar);
    }
    if (!tc::mbar_wait_warp(o_bar, phase, P.err)) flags[0] = 1;
    tc::tc_fence_after();
    phase ^= 1u;
    __syncthreads();
    if (flags[0]) break;
  }

  // ---- epilogue: sums over keys, normalisation, inverse RoPE, store ----
  const bool have = t_end > t_begin && !flags[0];
  if (warp < 8) {
    // per-head sums over the 32 keys of this warp: butterfly transpose-
    // reduce, lane j ends with the sum for head half*32 + j
#pragma unroll
    for (int off = 16, n = 16; off >= 1; off >>= 1, n >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < n) {
          const float send = upper ? lsum[i] : lsum[i + n];
          const float keep = upper ? lsum[i + n] : lsum[i];
          lsum[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
    }
    red[quad * kHeads + half * 32 + lane] = lsum[0];
    tc::named_bar(1, 256);
    if (warp < 2) {
      const int h = threadIdx.x;
      const float l = red[h] + red[kHeads + h] + red[2 * kHeads + h] + red[3 * kHeads + h];
      inv_den[h] = 1.f / (l + exp2f(P.sink[h] * kLog2e - ref2[h]));
    }
    tc::named_bar(1, 256);
    const int dim_in_blk = quad * 32 + lane;
    for (int blk = 0; blk < 4; ++blk) {
      const int d = blk * 128 + dim_in_blk;
      float o[32];
      if (have) {
        tc::tmem_ld32(tmem + lane_addr + kColO + blk * kHeads + half * 32, o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      float cs = 1.f, sn = 0.f;
      const bool rot = d >= kDim - P.r;
      if (rot) {
        const float2 tt = rope[(d - (kDim - P.r)) >> 1];
        cs = tt.x;
        sn = tt.y;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int h = half * 32 + i;
        float val = valid_seq ? o[i] * inv_den[h] : 0.f;
        if (rot) {
          // pair (d, d^1) sits in the neighbouring lane; rotate by -p
          const float other = __shfl_xor_sync(0xffffffffu, val, 1);
          val = (d & 1) ? (-other * sn + val * cs) : (val * cs + other * sn);
        }
        P.O[((int64_t)qi * kHeads + h) * kDim + d] = __float2bfloat16_rn(val);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool attend_tc_supported(int q_dt, int kv_dt, int c, int H_q, int k, int rope_dims) {
  return q_dt == CSA_BF16 && (kv_dt == CSA_BF16 || kv_dt == CSA_FP8_MIXED) && c == kDim &&
         H_q == kHeads && k <= CSA_MAX_TOPK && rope_dims % 32 == 0 && rope_dims <= 64;
}

cudaError_t launch_attend_tc(const csa_geom& g, int kv_dt, const void* q, const float* q_gain,
                             const float* sink, const void* E, int64_t ldE, int nseq,
                             const int64_t* n_entries, const int32_t* idx, int k, int dense,
                             const void* win, int64_t ldW, const int32_t* seq_of_q,
                             const int64_t* pos, int Q, void* O, cudaStream_t s) {
  if (Q == 0) return cudaSuccess;
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
  const size_t smem = (size_t)kSmemFixed + (dense ? 0 : (size_t)k * 4) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  count_launches();
  return launch_pdl(attend_tc_kernel, dim3((unsigned)Q), dim3(kThreads), smem, s, P);
}

}  // namespace csa
