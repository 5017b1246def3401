// simt_rows.cu - CUDA-core kernels: row preparation, FP8 packing, projection GEMM, compressor pooling (prefill and decode).
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

constexpr int kMaxPairsPerLane = 16;  // c <= 1024 for the row kernels

// ---------------------------------------------------------------------------
// Row preparation: y = RoPE_pos(RMSNorm(x) * gain), one warp per row.
// Lane l owns element pairs (2(l+32j), 2(l+32j)+1), so each RoPE pair is
// thread-local.
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void rmsnorm_rope_kernel(const Tin* __restrict__ x, int64_t rows, int c, int r,
                                    double base, float eps, const int64_t* __restrict__ pos,
                                    int64_t pos0, int64_t pos_step, const float* __restrict__ gain,
                                    void* __restrict__ out, const int64_t* __restrict__ out_row,
                                    int out_dt, int do_norm, int do_rope) {
  pdl_wait();
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int npairs = (c / 2 + 31) / 32;  // pair slots per lane
  const Tin* xr = x + row * c;
  float v[2 * kMaxPairsPerLane];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxPairsPerLane; ++j) {
    v[2 * j] = v[2 * j + 1] = 0.f;
    if (lane + 32 * j < c / 2) {
      int e = 2 * (lane + 32 * j);
      v[2 * j] = to_f32(xr[e]);
      v[2 * j + 1] = to_f32(xr[e + 1]);
      ss += v[2 * j] * v[2 * j] + v[2 * j + 1] * v[2 * j + 1];
    }
  }
  float inv = 1.f;
  if (do_norm) {
    ss = warp_sum(ss);
    inv = 1.f / sqrtf(ss / (float)c + eps);
  }
  const int64_t p = pos ? pos[row] : pos0 + row * pos_step;
  const int npair_rot = do_rope ? r / 2 : 0;
#pragma unroll
  for (int j = 0; j < kMaxPairsPerLane; ++j) {
    if (lane + 32 * j < c / 2) {
      int e = 2 * (lane + 32 * j);
      v[2 * j] *= inv * (gain ? gain[e] : 1.f);
      v[2 * j + 1] *= inv * (gain ? gain[e + 1] : 1.f);
    }
  }
  // RoPE: lane i computes the angle of pairs i, i+32, ... once (FP64), and
  // the owners of the rotated pairs fetch it with a shuffle
  for (int k0 = 0; k0 < npair_rot; k0 += 32) {
    float cs = 1.f, sn = 0.f;
    if (k0 + lane < npair_rot) rope_cs(p, k0 + lane, r, base, &cs, &sn);
#pragma unroll
    for (int j = 0; j < kMaxPairsPerLane; ++j) {
      const int e = 2 * (lane + 32 * j);
      const int i = (e - (c - r)) >> 1;  // rotated-pair index of this lane's pair j
      const bool mine = lane + 32 * j < c / 2 && e >= c - r && i >= k0 && i < k0 + 32;
      const float tc_ = __shfl_sync(0xffffffffu, cs, mine ? (i - k0) : 0);
      const float ts_ = __shfl_sync(0xffffffffu, sn, mine ? (i - k0) : 0);
      if (mine) {
        const float a = v[2 * j], b = v[2 * j + 1];
        v[2 * j] = a * tc_ - b * ts_;
        v[2 * j + 1] = a * ts_ + b * tc_;
      }
    }
  }
  const int64_t orow = out_row ? out_row[row] : row;
  if (out_dt == CSA_F32) {
    float* o = reinterpret_cast<float*>(out) + orow * c;
#pragma unroll
    for (int j = 0; j < kMaxPairsPerLane; ++j) {
      const int e = 2 * (lane + 32 * j);
      if (j < npairs && e < c) *reinterpret_cast<float2*>(o + e) = make_float2(v[2 * j], v[2 * j + 1]);
    }
  } else if (out_dt == CSA_BF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + orow * c;
#pragma unroll
    for (int j = 0; j < kMaxPairsPerLane; ++j) {
      const int e = 2 * (lane + 32 * j);
      if (j < npairs && e < c)
        *reinterpret_cast<uint32_t*>(o + e) = pack_bf16x2(v[2 * j], v[2 * j + 1]);
    }
  } else {  // mixed row, c == 512
    uint8_t* o = reinterpret_cast<uint8_t*>(out) + orow * (int64_t)kMixedRowBytes;
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxPairsPerLane; ++j) {
      const int e = 2 * (lane + 32 * j);
      if (j < npairs && e < kMixedFp8Dims)
        amax = fmaxf(amax, fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1])));
    }
    amax = warp_max(amax);
    const float scale = amax / 448.0f;
#pragma unroll
    for (int j = 0; j < kMaxPairsPerLane; ++j) {
      const int e = 2 * (lane + 32 * j);
      if (j >= npairs) continue;
      if (e < kMixedFp8Dims) {
        uint8_t c0 = scale > 0.f ? f32_to_e4m3(v[2 * j] / scale) : 0;
        uint8_t c1 = scale > 0.f ? f32_to_e4m3(v[2 * j + 1] / scale) : 0;
        *reinterpret_cast<uint16_t*>(o + e) = (uint16_t)c0 | ((uint16_t)c1 << 8);
      } else {
        *reinterpret_cast<uint32_t*>(o + kMixedFp8Dims + 2 * (e - kMixedFp8Dims)) =
            pack_bf16x2(v[2 * j], v[2 * j + 1]);
      }
    }
    if (lane == 0) *reinterpret_cast<float*>(o + kMixedScaleOffset) = scale;
    if (lane >= 1 && lane <= 3) *reinterpret_cast<uint32_t*>(o + kMixedScaleOffset + 4 * lane) = 0u;
  }
}

// ---------------------------------------------------------------------------
// Projection GEMM P = H @ [W_0 | ... | W_{nW-1}] on CUDA cores, FP32
// accumulation. 64x64 output tile per 256-thread block, 4x4 per thread.
// ---------------------------------------------------------------------------
struct WPtrs {
  const void* w[4];
};

template <typename Tin>
__global__ void __launch_bounds__(256) proj_simt_kernel(const Tin* __restrict__ H, int64_t T,
                                                        int d, int c, int nW, WPtrs W,
                                                        float* __restrict__ P) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int ncol = nW * c;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += BK) {
    for (int e = threadIdx.x; e < BM * BK; e += 256) {
      int mm = e / BK, kk = e % BK;
      int64_t row = m0 + mm;
      int kcol = k0 + kk;
      As[kk][mm] = (row < T && kcol < d) ? to_f32(H[row * d + kcol]) : 0.f;
    }
    for (int e = threadIdx.x; e < BN * BK; e += 256) {
      int kk = e / BN, nn = e % BN;
      int col = n0 + nn, krow = k0 + kk;
      float v = 0.f;
      if (col < ncol && krow < d) {
        int wi = col / c, ch = col % c;
        v = to_f32(reinterpret_cast<const Tin*>(W.w[wi])[(int64_t)krow * c + ch]);
      }
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int64_t row = m0 + ty * 4 + i;
    if (row >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int col = n0 + tx * 4 + j;
      if (col < ncol) P[row * ncol + col] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Pooling of one entry per 128-thread block from candidate values/logits,
// then RMSNorm and RoPE at position i*m; shared by prefill and decode.
// Candidate r (r < ncand) of channel ch: value vals(r)[ch], logit
// logits(r)[ch] + bias[r][ch]; `present` masks absent candidates.
// Thread t owns channel pairs (2(t+128j), +1).
// ---------------------------------------------------------------------------
__device__ void store_entry(const csa_geom& g, float* pooled_pairs, int npairs_thread,
                            int64_t entry_pos, const float* gain, int out_dt, void* E_row,
                            float* red) {
  const int c = g.c, r = g.rope_dims;
  const int t = threadIdx.x;
  float ss = 0.f;
  for (int j = 0; j < npairs_thread; ++j) {
    ss += pooled_pairs[2 * j] * pooled_pairs[2 * j] + pooled_pairs[2 * j + 1] * pooled_pairs[2 * j + 1];
  }
  ss = warp_sum(ss);
  if ((t & 31) == 0) red[t >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
  const float inv = 1.f / sqrtf(tot / (float)c + g.eps);
  float amax = 0.f;
  for (int j = 0; j < npairs_thread; ++j) {
    int e = 2 * (t + 128 * j);
    float a = pooled_pairs[2 * j] * inv * (gain ? gain[e] : 1.f);
    float b = pooled_pairs[2 * j + 1] * inv * (gain ? gain[e + 1] : 1.f);
    if (e >= c - r) {
      float cs, sn;
      rope_cs(entry_pos, (e - (c - r)) >> 1, r, g.rope_base, &cs, &sn);
      float a2 = a * cs - b * sn;
      b = a * sn + b * cs;
      a = a2;
    }
    pooled_pairs[2 * j] = a;
    pooled_pairs[2 * j + 1] = b;
    if (e < kMixedFp8Dims) amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
  }
  if (out_dt == CSA_F32) {
    for (int j = 0; j < npairs_thread; ++j) {
      int e = 2 * (t + 128 * j);
      *reinterpret_cast<float2*>(reinterpret_cast<float*>(E_row) + e) =
          make_float2(pooled_pairs[2 * j], pooled_pairs[2 * j + 1]);
    }
  } else if (out_dt == CSA_BF16) {
    for (int j = 0; j < npairs_thread; ++j) {
      int e = 2 * (t + 128 * j);
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(E_row) + e) =
          __floats2bfloat162_rn(pooled_pairs[2 * j], pooled_pairs[2 * j + 1]);
    }
  } else {
    __syncthreads();
    amax = warp_max(amax);
    if ((t & 31) == 0) red[t >> 5] = amax;
    __syncthreads();
    float am = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) am = fmaxf(am, red[w]);
    const float scale = am / 448.0f;
    uint8_t* o = reinterpret_cast<uint8_t*>(E_row);
    for (int j = 0; j < npairs_thread; ++j) {
      int e = 2 * (t + 128 * j);
      float a = pooled_pairs[2 * j], b = pooled_pairs[2 * j + 1];
      if (e < kMixedFp8Dims) {
        uint8_t c0 = scale > 0.f ? f32_to_e4m3(a / scale) : 0;
        uint8_t c1 = scale > 0.f ? f32_to_e4m3(b / scale) : 0;
        *reinterpret_cast<uint16_t*>(o + e) = (uint16_t)c0 | ((uint16_t)c1 << 8);
      } else {
        *reinterpret_cast<__nv_bfloat162*>(o + kMixedFp8Dims + 2 * (e - kMixedFp8Dims)) =
            __floats2bfloat162_rn(a, b);
      }
    }
    if (t == 0) *reinterpret_cast<float*>(o + kMixedScaleOffset) = scale;
    if (t >= 1 && t <= 3) *reinterpret_cast<uint32_t*>(o + kMixedScaleOffset + 4 * t) = 0u;
  }
}

constexpr int kPoolThreads = 128;
constexpr int kMaxPoolPairs = 8;  // c <= 2048

// Prefill pool: block i; P rows are tokens with columns
// [C^a | Z^a | C^b | Z^b] (CSA) or [C | Z] (HCA).
__global__ void __launch_bounds__(kPoolThreads) pool_prefill_kernel(
    csa_geom g, const float* __restrict__ P, const float* __restrict__ bias,
    const float* __restrict__ gain, int out_dt, void* __restrict__ E) {
  __shared__ float red[kPoolThreads / 32];
  const int64_t i = blockIdx.x;
  const int c = g.c, m = g.m;
  const int nW = g.overlap ? 4 : 2;
  const int64_t ld = (int64_t)nW * c;
  const int npairs = (c / 2 + kPoolThreads - 1) / kPoolThreads;
  float pooled[2 * kMaxPoolPairs];
  for (int j = 0; j < npairs; ++j) {
    for (int u = 0; u < 2; ++u) {
      const int ch = 2 * (threadIdx.x + kPoolThreads * j) + u;
      float res = 0.f;
      if (ch < c) {
        float mx = -FLT_MAX;
        const int nb = (g.overlap && i >= 1) ? m : 0;
        for (int rr = 0; rr < nb; ++rr) {
          const float* row = P + ((i - 1) * m + rr) * ld;
          mx = fmaxf(mx, row[3 * c + ch] + bias[rr * c + ch]);
        }
        const int abase = g.overlap ? m : 0;
        for (int rr = 0; rr < m; ++rr) {
          const float* row = P + (i * m + rr) * ld;
          mx = fmaxf(mx, row[c + ch] + bias[(abase + rr) * c + ch]);
        }
        float den = 0.f, num = 0.f;
        for (int rr = 0; rr < nb; ++rr) {
          const float* row = P + ((i - 1) * m + rr) * ld;
          float e = __expf(row[3 * c + ch] + bias[rr * c + ch] - mx);
          den += e;
          num = fmaf(e, row[2 * c + ch], num);
        }
        for (int rr = 0; rr < m; ++rr) {
          const float* row = P + (i * m + rr) * ld;
          float e = __expf(row[c + ch] + bias[(abase + rr) * c + ch] - mx);
          den += e;
          num = fmaf(e, row[ch], num);
        }
        res = num / den;
      }
      pooled[2 * j + u] = res;
    }
  }
  // threads beyond c/2 pairs hold zeros and contribute nothing
  int my_pairs = 0;
  for (int j = 0; j < npairs; ++j)
    if (2 * (threadIdx.x + kPoolThreads * j) < c) my_pairs = j + 1;
  void* E_row = reinterpret_cast<uint8_t*>(E) + i * row_bytes(out_dt, c);
  store_entry(g, pooled, my_pairs, i * m, gain, out_dt, E_row, red);
}

// ---------------------------------------------------------------------------
// Decode compressor. State per sequence: [nslot][m][nW][c] FP32 with
// nslot = 1 + overlap; block i's tokens live in slot i % nslot, series in
// the order [C^a, Z^a, C^b, Z^b] (CSA) or [C, Z] (HCA).
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) decode_proj_kernel(
    csa_geom g, const Tin* __restrict__ h, const int64_t* __restrict__ pos, int B, int d, WPtrs W,
    int nW, float* __restrict__ state) {
  constexpr int TB = 8;  // tokens per thread
  const int c = g.c, m = g.m;
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  const int b0 = blockIdx.y * TB;
  const int ncol = nW * c;
  __shared__ float hs[TB][256];
  float acc[TB] = {};
  const int wi = col / c, ch = col % c;
  const Tin* Wp = col < ncol ? reinterpret_cast<const Tin*>(W.w[wi]) : nullptr;
  for (int k0 = 0; k0 < d; k0 += 256) {
    for (int e = threadIdx.x; e < TB * 256; e += blockDim.x) {
      int bb = e / 256, kk = e % 256;
      hs[bb][kk] = (b0 + bb < B && k0 + kk < d) ? to_f32(h[(int64_t)(b0 + bb) * d + k0 + kk]) : 0.f;
    }
    __syncthreads();
    if (Wp) {
      const int kend = min(256, d - k0);
      for (int kk = 0; kk < kend; ++kk) {
        float wv = to_f32(Wp[(int64_t)(k0 + kk) * c + ch]);
#pragma unroll
        for (int bb = 0; bb < TB; ++bb) acc[bb] = fmaf(hs[bb][kk], wv, acc[bb]);
      }
    }
    __syncthreads();
  }
  if (!Wp) return;
  const int nslot = 1 + g.overlap;
  const int64_t per_seq = (int64_t)nslot * m * nW * c;
  for (int bb = 0; bb < TB; ++bb) {
    const int b = b0 + bb;
    if (b >= B) break;
    const int64_t p = pos[b];
    const int64_t blk = p / m;
    const int rr = (int)(p % m);
    const int slot = (int)(blk % nslot);
    state[b * per_seq + (((int64_t)slot * m + rr) * nW + wi) * c + ch] = acc[bb];
  }
}

__global__ void __launch_bounds__(kPoolThreads) decode_pool_kernel(
    csa_geom g, const int64_t* __restrict__ pos, const float* __restrict__ bias,
    const float* __restrict__ gain, const float* __restrict__ state, int out_dt,
    void* __restrict__ E, int64_t ldE) {
  __shared__ float red[kPoolThreads / 32];
  pdl_wait();
  const int b = blockIdx.x;
  const int c = g.c, m = g.m;
  const int64_t p = pos[b];
  if ((p + 1) % m != 0) return;
  const int64_t i = p / m;
  if (i >= ldE) return;
  const int nslot = 1 + g.overlap;
  const int nW = g.overlap ? 4 : 2;
  const int64_t per_seq = (int64_t)nslot * m * nW * c;
  const float* st = state + b * per_seq;
  const float* own = st + (int64_t)(i % nslot) * m * nW * c;
  const float* prev = st + (int64_t)((i + nslot - 1) % nslot) * m * nW * c;
  const int npairs = (c / 2 + kPoolThreads - 1) / kPoolThreads;
  float pooled[2 * kMaxPoolPairs];
  for (int j = 0; j < npairs; ++j) {
    for (int u = 0; u < 2; ++u) {
      const int ch = 2 * (threadIdx.x + kPoolThreads * j) + u;
      float res = 0.f;
      if (ch < c) {
        float mx = -FLT_MAX;
        const int nb = (g.overlap && i >= 1) ? m : 0;
        const int abase = g.overlap ? m : 0;
        for (int rr = 0; rr < nb; ++rr)
          mx = fmaxf(mx, prev[((int64_t)rr * nW + 3) * c + ch] + bias[rr * c + ch]);
        for (int rr = 0; rr < m; ++rr)
          mx = fmaxf(mx, own[((int64_t)rr * nW + 1) * c + ch] + bias[(abase + rr) * c + ch]);
        float den = 0.f, num = 0.f;
        for (int rr = 0; rr < nb; ++rr) {
          float e = __expf(prev[((int64_t)rr * nW + 3) * c + ch] + bias[rr * c + ch] - mx);
          den += e;
          num = fmaf(e, prev[((int64_t)rr * nW + 2) * c + ch], num);
        }
        for (int rr = 0; rr < m; ++rr) {
          float e = __expf(own[((int64_t)rr * nW + 1) * c + ch] + bias[(abase + rr) * c + ch] - mx);
          den += e;
          num = fmaf(e, own[((int64_t)rr * nW + 0) * c + ch], num);
        }
        res = num / den;
      }
      pooled[2 * j + u] = res;
    }
  }
  int my_pairs = 0;
  for (int j = 0; j < npairs; ++j)
    if (2 * (threadIdx.x + kPoolThreads * j) < c) my_pairs = j + 1;
  void* E_row = reinterpret_cast<uint8_t*>(E) + ((int64_t)b * ldE + i) * row_bytes(out_dt, c);
  store_entry(g, pooled, my_pairs, i * m, gain, out_dt, E_row, red);
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_rmsnorm_rope(const csa_geom& g, int in_dt, int out_dt, const void* x,
                                int64_t rows, const int64_t* pos, int64_t pos0, int64_t pos_step,
                                const float* gain, void* out, const int64_t* out_row,
                                cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  count_launches();
  dim3 block(256), grid((unsigned)((rows + 7) / 8));
  if (in_dt == CSA_F32)
    return launch_pdl(rmsnorm_rope_kernel<float>, grid, block, 0, s,
                      reinterpret_cast<const float*>(x), rows, g.c, g.rope_dims, g.rope_base,
                      g.eps, pos, pos0, pos_step, gain, out, out_row, out_dt, 1, 1);
  return launch_pdl(rmsnorm_rope_kernel<__nv_bfloat16>, grid, block, 0, s,
                    reinterpret_cast<const __nv_bfloat16*>(x), rows, g.c, g.rope_dims,
                    g.rope_base, g.eps, pos, pos0, pos_step, gain, out, out_row, out_dt, 1, 1);
}

cudaError_t launch_quantize_mixed(int in_dt, const void* x, int64_t rows, void* out,
                                  cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  count_launches();
  dim3 block(256), grid((unsigned)((rows + 7) / 8));
  if (in_dt == CSA_F32)
    rmsnorm_rope_kernel<float><<<grid, block, 0, s>>>(reinterpret_cast<const float*>(x), rows,
                                                      512, 64, 10000.0, 0.f, nullptr, 0, 0,
                                                      nullptr, out, nullptr, CSA_FP8_MIXED, 0, 0);
  else
    rmsnorm_rope_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), rows, 512, 64, 10000.0, 0.f, nullptr, 0, 0,
        nullptr, out, nullptr, CSA_FP8_MIXED, 0, 0);
  return cudaGetLastError();
}

cudaError_t launch_proj_simt(int dt, const void* H, int64_t T, int d, int c, int nW,
                             const void* const* W, float* P, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  count_launches();
  WPtrs wp{};
  for (int i = 0; i < nW; ++i) wp.w[i] = W[i];
  dim3 grid((unsigned)((nW * c + 63) / 64), (unsigned)((T + 63) / 64));
  if (dt == CSA_F32)
    proj_simt_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(H), T, d, c, nW,
                                                 wp, P);
  else
    proj_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(H), T, d, c, nW, wp, P);
  return cudaGetLastError();
}

cudaError_t launch_pool_prefill(const csa_geom& g, const float* P, int64_t T, const float* bias,
                                const float* gain, int out_dt, void* E, cudaStream_t s) {
  const int64_t nb = T / g.m;
  if (nb == 0) return cudaSuccess;
  count_launches();
  pool_prefill_kernel<<<(unsigned)nb, kPoolThreads, 0, s>>>(g, P, bias, gain, out_dt, E);
  return cudaGetLastError();
}

cudaError_t launch_decode_proj(const csa_geom& g, int dt, const void* h, const int64_t* pos,
                               int B, int d, const void* const* W, int nW, float* state,
                               cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  count_launches();
  WPtrs wp{};
  for (int i = 0; i < nW; ++i) wp.w[i] = W[i];
  dim3 grid((unsigned)((nW * g.c + 255) / 256), (unsigned)((B + 7) / 8));
  if (dt == CSA_F32)
    decode_proj_kernel<float><<<grid, 256, 0, s>>>(g, reinterpret_cast<const float*>(h), pos, B,
                                                   d, wp, nW, state);
  else
    decode_proj_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        g, reinterpret_cast<const __nv_bfloat16*>(h), pos, B, d, wp, nW, state);
  return cudaGetLastError();
}

cudaError_t launch_decode_pool(const csa_geom& g, const int64_t* pos, int B, const float* bias,
                               const float* gain, const float* state, int out_dt, void* E,
                               int64_t ldE, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  count_launches();
  return launch_pdl(decode_pool_kernel, dim3(B), dim3(kPoolThreads), 0, s, g, pos, bias, gain,
                    state, out_dt, E, ldE);
}

}  // namespace csa
