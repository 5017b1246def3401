// tc_proj.cu - compressor projections on the 5th-generation tensor cores.
//
// The compressor's four projections C^a = H W_aKV, Z^a = H W_aZ,
// C^b = H W_bKV, Z^b = H W_bZ ("Evidence Ledger", CSA Eqs 9-10; HCA Eqs
// 20-26 with one KV and one gate projection) form one GEMM
// D[tokens, cols] = H[tokens, d] x W[d, cols]: H is the K-major A operand
// (128 tokens per tile, TMA-fed), the weights the MN-major B operand (four
// 64-column slices, TMA-fed straight from the row-major [d, c] matrices),
// FP32 accumulation in TMEM (256 columns).
//
// Epilogues:
//  kRaw     - store D as FP32 split-K partials (decode: one new token per
//             sequence, the weights are streamed once across all SMs);
//  kPoolCsa - overlapping softmax pool of each entry's 2m candidates
//             ("Evidence Ledger" CSA Eqs 11-12; "DeepSeek-V4" study 03):
//             a tile of 128 token rows starting m rows before a block
//             boundary yields (128-m)/m complete entries, so the projections
//             never leave the SM; only pooled rows [T/m, c] are written;
//  kPoolHca - non-overlapping pool of m' candidates (HCA).
// Normalisation and RoPE of the pooled rows follow in the row kernel.
//
// Warps (192 threads): 0 = TMA producer, 1 = TMEM owner + MMA issuer,
// 2-5 = epilogue (TMEM lane quadrant = warp % 4). Four pipeline stages of
// 48 KB (A 16 KB + B 32 KB per 64-deep K chunk).
#include "internal.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kBytesA = 128 * 128;        // 128 tokens x 64 BF16
constexpr int kBytesBSlice = 64 * 128;    // 64 K rows x 64 BF16
constexpr int kBytesStage = kBytesA + 4 * kBytesBSlice;
constexpr int kSmem = 1024 + kStages * kBytesStage + 256;
constexpr int kLd = 129;  // column stride of the staged accumulator (floats)

enum Mode { kRaw = 0, kPoolCsa = 1, kPoolHca = 2 };

struct Params {
  int mode;
  int64_t T;
  int d, c, m, nW;
  int chunks_per_split;  // 64-deep K chunks per CTA
  int entries_per_tile;  // pool modes
  int64_t nblocks;       // T / m
  const float* bias;
  float* out;            // kRaw: [ksplit][T][nW*c]; pool: [T/m][c]
  int* err;
};

__device__ __forceinline__ void slice_of(const Params& P, int ntile, int s, int* map, int* x) {
  if (P.mode == kRaw) {
    const int v = ntile * 256 + s * 64;
    *map = v / P.c;
    *x = v % P.c;
  } else if (P.mode == kPoolCsa) {
    *map = s;  // C^a, Z^a, C^b, Z^b
    *x = ntile * 64;
  } else {
    *map = s >> 1;  // C, C, Z, Z
    *x = ntile * 128 + 64 * (s & 1);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                   const __grid_constant__ CUtensorMap tmW3, Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kStages * kBytesStage);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = blockIdx.x, mtile = blockIdx.y, split = blockIdx.z;

  int64_t tok0;
  if (P.mode == kPoolCsa) tok0 = (int64_t)mtile * (128 - P.m) - P.m;
  else tok0 = (int64_t)mtile * 128;
  const int total_chunks = P.d / 64;
  const int kc0 = split * P.chunks_per_split;
  const int kc1 = min(total_chunks, kc0 + P.chunks_per_split);
  const int nchunks = kc1 - kc0;

  auto full_bar = [&](int s) { return tc::smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return tc::smem_u32(&bars[kStages + s]); };
  const uint32_t done_bar = tc::smem_u32(&bars[2 * kStages]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    tc::mbar_init(done_bar, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_u32(tslot), 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();               // inputs of the previous kernel visible from here on

  if (warp == 0 && lane == 0) {
    // ---- TMA producer ----
    const CUtensorMap* maps[4] = {&tmW0, &tmW1, &tmW2, &tmW3};
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % kStages;
      if (i >= kStages && !tc::mbar_wait(empty_bar(s), ((i / kStages) + 1) & 1, P.err)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = sm + s * kBytesStage;
      const int k0 = (kc0 + i) * 64;
      tc::mbar_arrive_expect_tx(full_bar(s), kBytesStage);
      tc::tma_load_2d(tc::smem_u32(st), &tmA, k0, (int32_t)tok0, full_bar(s));
      for (int sl = 0; sl < 4; ++sl) {
        int mi, x;
        slice_of(P, ntile, sl, &mi, &x);
        tc::tma_load_2d(tc::smem_u32(st + kBytesA + sl * kBytesBSlice), maps[mi], x, k0,
                        full_bar(s));
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    const uint32_t idesc = tc::idesc_bf16_f32_major(128, 256, 0, 1);
    bool ok = true;
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % kStages;
      if (!tc::mbar_wait(full_bar(s), (i / kStages) & 1, P.err)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t a0 = tc::smem_u32(sm + s * kBytesStage);
      const uint32_t b0 = a0 + kBytesA;
      for (int kk = 0; kk < 4; ++kk) {
        tc::mma_bf16(tmem, tc::sdesc_kmajor_sw128(a0 + kk * 32),
                     tc::sdesc_mnmajor_sw128(b0 + kk * 2048, kBytesBSlice, 1024), idesc,
                     (i > 0 || kk > 0) ? 1u : 0u);
      }
      tc::mma_commit(empty_bar(s));
    }
    if (!ok) *abort_flag = 1;
    tc::mma_commit(done_bar);
  } else if (warp >= 2) {
    // ---- epilogue ----
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // token row of the tile
    const bool ok = tc::mbar_wait_warp(done_bar, 0, P.err);
    tc::tc_fence_after();
    if (P.mode == kRaw) {
      const int64_t t = tok0 + row;
      const int ncols = P.nW * P.c;
      float* dst = P.out + ((int64_t)split * P.T + t) * ncols + (int64_t)ntile * 256;
      for (int c0 = 0; c0 < 256; c0 += 32) {
        float v[32];
        tc::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
        if (ok && !*abort_flag && t < P.T && nchunks > 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
    } else {
      // stage D column-major in shared memory (the pipeline buffers are idle)
      float* sD = reinterpret_cast<float*>(sm);  // [256 cols][129]: padded column stride
      for (int c0 = 0; c0 < 256; c0 += 32) {
        float v[32];
        tc::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) sD[(c0 + i) * kLd + row] = v[i];
      }
      tc::named_bar(1, 128);
      const int tid = threadIdx.x - 64;
      if (ok && !*abort_flag) {
        const int m = P.m, c = P.c;
        if (P.mode == kPoolCsa) {
          const int ch0 = ntile * 64;
          for (int it = tid; it < P.entries_per_tile * 64; it += 128) {
            const int e = it / 64, j = it % 64;
            const int64_t blk = (int64_t)mtile * P.entries_per_tile + e;
            if (blk >= P.nblocks) continue;
            const int ch = ch0 + j;
            const bool has_b = blk >= 1;
            float mx = -INFINITY;
            // rows m*e .. m*e+m-1: preceding block (b-series); +m: own block (a-series)
            if (has_b)
              for (int r = 0; r < m; ++r) mx = fmaxf(mx, sD[(192 + j) * kLd + m * e + r] + P.bias[r * c + ch]);
            for (int r = 0; r < m; ++r)
              mx = fmaxf(mx, sD[(64 + j) * kLd + m * e + m + r] + P.bias[(m + r) * c + ch]);
            float den = 0.f, num = 0.f;
            if (has_b)
              for (int r = 0; r < m; ++r) {
                const float w = __expf(sD[(192 + j) * kLd + m * e + r] + P.bias[r * c + ch] - mx);
                den += w;
                num = fmaf(w, sD[(128 + j) * kLd + m * e + r], num);
              }
            for (int r = 0; r < m; ++r) {
              const float w = __expf(sD[(64 + j) * kLd + m * e + m + r] + P.bias[(m + r) * c + ch] - mx);
              den += w;
              num = fmaf(w, sD[j * kLd + m * e + m + r], num);
            }
            P.out[blk * c + ch] = num / den;
          }
        } else {
          const int ch0 = ntile * 128;
          const int per_tile = 128 / m;
          for (int it = tid; it < per_tile * 128; it += 128) {
            const int e = it / 128, j = it % 128;
            const int64_t blk = (int64_t)mtile * per_tile + e;
            if (blk >= P.nblocks) continue;
            const int ch = ch0 + j;
            float mx = -INFINITY;
            for (int r = 0; r < m; ++r) mx = fmaxf(mx, sD[(128 + j) * kLd + m * e + r] + P.bias[r * c + ch]);
            float den = 0.f, num = 0.f;
            for (int r = 0; r < m; ++r) {
              const float w = __expf(sD[(128 + j) * kLd + m * e + r] + P.bias[r * c + ch] - mx);
              den += w;
              num = fmaf(w, sD[j * kLd + m * e + r], num);
            }
            P.out[blk * c + ch] = num / den;
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

// Sum of the split-K partials in split order, scattered into the decode
// state [B][slot][m][nW][c] at the token's position.
__global__ void __launch_bounds__(256) decode_reduce_kernel(const float* __restrict__ part,
                                                            int ksplit, int B, int nW, int c,
                                                            int m, int overlap,
                                                            const int64_t* __restrict__ pos,
                                                            float* __restrict__ state) {
  pdl_wait();
  const int ncols = nW * c;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)B * ncols) return;
  const int b = (int)(i / ncols), col = (int)(i % ncols);
  float acc = 0.f;
  for (int s = 0; s < ksplit; ++s) acc += part[((int64_t)s * B + b) * ncols + col];
  const int nslot = 1 + overlap;
  const int64_t p = pos[b];
  const int slot = (int)((p / m) % nslot), r = (int)(p % m);
  const int series = col / c, ch = col % c;
  const int64_t per_seq = (int64_t)nslot * m * nW * c;
  state[b * per_seq + (((int64_t)slot * m + r) * nW + series) * c + ch] = acc;
}

bool make_maps(const void* H, int64_t T, int d, const void* const* W, int nW, int c,
               CUtensorMap* tmA, CUtensorMap* tmW) {
  if (!encode_tmap_2d_bf16(tmA, H, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, 64, 128)) return false;
  for (int i = 0; i < 4; ++i) {
    const void* w = W[i < nW ? i : 0];
    if (!encode_tmap_2d_bf16(&tmW[i], w, (uint64_t)c, (uint64_t)d, (uint64_t)c * 2, 64, 64))
      return false;
  }
  return true;
}

cudaError_t launch(const CUtensorMap& tmA, const CUtensorMap* tmW, const Params& P, dim3 grid,
                   cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmem);
  if (e != cudaSuccess) return e;
  count_launches();
  return launch_pdl(proj_tc_kernel, grid, dim3(kThreads), kSmem, s, tmA, tmW[0], tmW[1], tmW[2],
                    tmW[3], P);
}

// Split-K factor of a decode projection: about enough splits that the N
// tiles times the splits fill the SMs once, at most 16 (the partials are
// summed by decode_reduce_kernel; 64 splits of the 512-wide index-key
// projection, which has two N tiles, made the decode step slower).
int decode_ksplit(int ntiles, int mtiles, int total_chunks, int* chunks_per_split) {
  const int target = min(16, max(1, 148 / max(1, ntiles * mtiles)));
  const int cps = max(1, (total_chunks + target - 1) / target);
  *chunks_per_split = cps;
  return (total_chunks + cps - 1) / cps;
}

}  // namespace

bool proj_tc_supported(const csa_geom& g, int dt, int d) {
  if (dt != CSA_BF16 || d % 64 != 0 || g.c % 64 != 0) return false;
  if (g.m >= 128 ? (g.m != 128) : (128 % g.m != 0)) return false;
  if (g.overlap && g.m >= 128) return false;
  if (!g.overlap && g.c % 128 != 0) return false;
  return true;
}

size_t proj_pool_workspace(const csa_geom& g, int64_t T) {
  return (size_t)(T / g.m) * g.c * sizeof(float);
}

size_t proj_decode_workspace(const csa_geom& g, int B, int d) {
  const int nW = g.overlap ? 4 : 2;
  const int ntiles = nW * g.c / 256, mtiles = (B + 127) / 128;
  int cps;
  const int ksplit = decode_ksplit(ntiles, mtiles, d / 64, &cps);
  return (size_t)ksplit * B * nW * g.c * sizeof(float);
}

bool proj_decode_supported(const csa_geom& g, int dt, int d) {
  const int nW = g.overlap ? 4 : 2;
  return dt == CSA_BF16 && d % 64 == 0 && g.c % 64 == 0 && (nW * g.c) % 256 == 0;
}

cudaError_t launch_compress_tc(const csa_geom& g, const void* H, int64_t T, int d,
                               const void* const* W, const float* bias, float* pooled,
                               cudaStream_t s) {
  const int nW = g.overlap ? 4 : 2;
  CUtensorMap tmA, tmW[4];
  if (!make_maps(H, T, d, W, nW, g.c, &tmA, tmW)) return cudaErrorInvalidValue;
  Params P{};
  P.mode = g.overlap ? kPoolCsa : kPoolHca;
  P.T = T;
  P.d = d;
  P.c = g.c;
  P.m = g.m;
  P.nW = nW;
  P.chunks_per_split = d / 64;
  P.nblocks = T / g.m;
  P.entries_per_tile = g.overlap ? (128 - g.m) / g.m : 128 / g.m;
  P.bias = bias;
  P.out = pooled;
  P.err = device_error_ptr();
  if (P.nblocks == 0) return cudaSuccess;
  const int64_t mtiles = (P.nblocks + P.entries_per_tile - 1) / P.entries_per_tile;
  const int ntiles = g.overlap ? g.c / 64 : g.c / 128;
  if (mtiles > 65535) return cudaErrorInvalidValue;
  return launch(tmA, tmW, P, dim3((unsigned)ntiles, (unsigned)mtiles, 1), s);
}

cudaError_t launch_decode_proj_tc(const csa_geom& g, const void* h, const int64_t* pos, int B,
                                  int d, const void* const* W, float* part, float* state,
                                  cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int nW = g.overlap ? 4 : 2;
  CUtensorMap tmA, tmW[4];
  if (!make_maps(h, B, d, W, nW, g.c, &tmA, tmW)) return cudaErrorInvalidValue;
  Params P{};
  P.mode = kRaw;
  P.T = B;
  P.d = d;
  P.c = g.c;
  P.m = g.m;
  P.nW = nW;
  const int ntiles = nW * g.c / 256, mtiles = (B + 127) / 128;
  int cps;
  const int ksplit = decode_ksplit(ntiles, mtiles, d / 64, &cps);
  P.chunks_per_split = cps;
  P.out = part;
  P.err = device_error_ptr();
  cudaError_t e = launch(tmA, tmW, P, dim3((unsigned)ntiles, (unsigned)mtiles, (unsigned)ksplit), s);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)B * nW * g.c;
  count_launches();
  return launch_pdl(decode_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s,
                    (const float*)part, ksplit, B, nW, g.c, g.m, g.overlap, pos, state);
}

}  // namespace csa
