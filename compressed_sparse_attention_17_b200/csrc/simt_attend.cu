// simt_attend.cu - CUDA-core shared-KV attention with window and sink.
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
// Attention on CUDA cores, one block per query, all heads. Online softmax
// seeded with the sink (running max starts at z'_h with weight 1 and no
// value), keys streamed in tiles of 32 rows through shared memory.
// ---------------------------------------------------------------------------
constexpr int kAttThreads = 256;
constexpr int kAttKT = 32;

__device__ __forceinline__ const void* key_row(const csa_geom& g, int kv_dt, const void* E,
                                               int64_t ldE, const void* win, int64_t ldW, int c,
                                               int b, int64_t slot, int64_t nsel,
                                               const int32_t* idx_row, int dense, int64_t w0) {
  if (slot < nsel) {
    int64_t s = dense ? slot : (int64_t)idx_row[slot];
    if (s < 0 || s >= ldE) return nullptr;  // absent, or outside the cache: not read
    return reinterpret_cast<const uint8_t*>(E) + ((int64_t)b * ldE + s) * row_bytes(kv_dt, c);
  }
  int64_t j = w0 + (slot - nsel);
  int64_t rowi = g.win_ring ? (j % g.n_win) : j;
  if (rowi >= ldW) return nullptr;  // outside the window buffer: not read
  const int wdt = kv_dt == CSA_FP8_MIXED ? CSA_BF16 : kv_dt;
  return reinterpret_cast<const uint8_t*>(win) + ((int64_t)b * ldW + rowi) * row_bytes(wdt, c);
}

template <typename Tq, int OPT>
__global__ void __launch_bounds__(kAttThreads) attend_simt_kernel(
    csa_geom g, int kv_dt, const Tq* __restrict__ q, const float* __restrict__ q_gain,
    const float* __restrict__ sink, const void* __restrict__ E, int64_t ldE, int nseq,
    const int64_t* __restrict__ n_entries, const int32_t* __restrict__ idx, int k, int dense,
    const void* __restrict__ win, int64_t ldW, const int32_t* __restrict__ seq_of_q,
    const int64_t* __restrict__ pos, int H_q, Tq* __restrict__ O) {
  extern __shared__ float sm[];
  const int c = g.c, r = g.rope_dims;
  const int ldk = c + 1;
  float* qh = sm;                         // [H_q][c]
  float* kt = qh + H_q * c;               // [KT][c+1]
  float* S = kt + kAttKT * ldk;           // [H_q][KT]
  float* mh = S + H_q * kAttKT;           // [H_q]
  float* lh = mh + H_q;                   // [H_q]
  float* al = lh + H_q;                   // [H_q]
  const int qi = blockIdx.x;
  const int b = seq_of_q[qi];
  const int64_t p = pos[qi];
  if (b < 0 || b >= nseq) {  // no such sequence: zero output
    for (int e = threadIdx.x; e < H_q * c; e += kAttThreads)
      O[(int64_t)qi * H_q * c + e] = from_f32<Tq>(0.f);
    return;
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nwarps = kAttThreads / 32;
  // q-hat = RoPE_p(RMSNorm(q_h) * q_gain), one warp per head
  for (int h = wid; h < H_q; h += nwarps) {
    const Tq* qr = q + ((int64_t)qi * H_q + h) * c;
    float ss = 0.f;
    for (int e = lane; e < c; e += 32) {
      float v = to_f32(qr[e]);
      ss += v * v;
    }
    ss = warp_sum(ss);
    const float inv = 1.f / sqrtf(ss / (float)c + g.eps);
    for (int pr = lane; pr < c / 2; pr += 32) {
      int e = 2 * pr;
      float a = to_f32(qr[e]) * inv * (q_gain ? q_gain[e] : 1.f);
      float bb = to_f32(qr[e + 1]) * inv * (q_gain ? q_gain[e + 1] : 1.f);
      if (e >= c - r) {
        float cs, sn;
        rope_cs(p, (e - (c - r)) >> 1, r, g.rope_base, &cs, &sn);
        float a2 = a * cs - bb * sn;
        bb = a * sn + bb * cs;
        a = a2;
      }
      qh[h * c + e] = a;
      qh[h * c + e + 1] = bb;
    }
  }
  for (int h = threadIdx.x; h < H_q; h += kAttThreads) {
    mh[h] = sink[h];
    lh[h] = 1.f;
  }
  const int64_t nv = dense ? n_visible(p, g.m, g.vis_offset, min(n_entries[b], ldE)) : 0;
  const int64_t nsel = dense ? nv : k;
  const int64_t w0 = p - g.n_win + 1 > 0 ? p - g.n_win + 1 : 0;
  const int64_t nwin = g.n_win > 0 ? p - w0 + 1 : 0;
  const int64_t nslots = nsel + nwin;
  const int32_t* idx_row = dense ? nullptr : idx + (int64_t)qi * k;
  const float scale = 1.f / sqrtf((float)c);
  float acc[OPT];
#pragma unroll
  for (int u = 0; u < OPT; ++u) acc[u] = 0.f;
  const int total_pairs = H_q * c / 2;
  __syncthreads();
  for (int64_t t0 = 0; t0 < nslots; t0 += kAttKT) {
    // load the key tile (zeros for absent slots)
    for (int e = threadIdx.x; e < kAttKT * c; e += kAttThreads) {
      const int kk = e / c, i = e % c;
      const int64_t slot = t0 + kk;
      float v = 0.f;
      if (slot < nslots) {
        const void* row = key_row(g, kv_dt, E, ldE, win, ldW, c, b, slot, nsel, idx_row, dense, w0);
        if (row) v = load_elem(row, i, slot < nsel ? kv_dt : (kv_dt == CSA_FP8_MIXED ? CSA_BF16 : kv_dt));
      }
      kt[kk * ldk + i] = v;
    }
    __syncthreads();
    // logits
    for (int pi = threadIdx.x; pi < H_q * kAttKT; pi += kAttThreads) {
      const int h = pi / kAttKT, kk = pi % kAttKT;
      const int64_t slot = t0 + kk;
      float l = -INFINITY;
      bool valid = slot < nslots &&
                   key_row(g, kv_dt, E, ldE, win, ldW, c, b, slot, nsel, idx_row, dense, w0) != nullptr;
      if (valid) {
        float d = 0.f;
        const float* qr = qh + h * c;
        const float* kr = kt + kk * ldk;
        for (int i = 0; i < c; ++i) d = fmaf(qr[i], kr[i], d);
        l = d * scale;
      }
      S[h * kAttKT + kk] = l;
    }
    __syncthreads();
    // online softmax update per head
    for (int h = threadIdx.x; h < H_q; h += kAttThreads) {
      float tmax = -INFINITY;
      for (int kk = 0; kk < kAttKT; ++kk) tmax = fmaxf(tmax, S[h * kAttKT + kk]);
      const float mnew = fmaxf(mh[h], tmax);
      const float alpha = __expf(mh[h] - mnew);
      float sum = 0.f;
      for (int kk = 0; kk < kAttKT; ++kk) {
        float pv = __expf(S[h * kAttKT + kk] - mnew);
        S[h * kAttKT + kk] = pv;
        sum += pv;
      }
      lh[h] = lh[h] * alpha + sum;
      mh[h] = mnew;
      al[h] = alpha;
    }
    __syncthreads();
    // O update
#pragma unroll
    for (int u = 0; u < OPT / 2; ++u) {
      const int pi = threadIdx.x + kAttThreads * u;
      if (pi < total_pairs) {
        const int h = (2 * pi) / c, i = (2 * pi) % c;
        const float alpha = al[h];
        float a0 = acc[2 * u] * alpha, a1 = acc[2 * u + 1] * alpha;
        const float* Sh = S + h * kAttKT;
        for (int kk = 0; kk < kAttKT; ++kk) {
          const float pv = Sh[kk];
          a0 = fmaf(pv, kt[kk * ldk + i], a0);
          a1 = fmaf(pv, kt[kk * ldk + i + 1], a1);
        }
        acc[2 * u] = a0;
        acc[2 * u + 1] = a1;
      }
    }
    __syncthreads();
  }
  // normalise, inverse RoPE, store
#pragma unroll
  for (int u = 0; u < OPT / 2; ++u) {
    const int pi = threadIdx.x + kAttThreads * u;
    if (pi < total_pairs) {
      const int h = (2 * pi) / c, i = (2 * pi) % c;
      const float inv = 1.f / lh[h];
      float a = acc[2 * u] * inv, bb = acc[2 * u + 1] * inv;
      if (i >= c - r) {
        float cs, sn;
        rope_cs(p, (i - (c - r)) >> 1, r, g.rope_base, &cs, &sn);
        float a2 = a * cs + bb * sn;  // rotation by -p
        bb = -a * sn + bb * cs;
        a = a2;
      }
      Tq* orow = O + ((int64_t)qi * H_q + h) * c;
      orow[i] = from_f32<Tq>(a);
      orow[i + 1] = from_f32<Tq>(bb);
    }
  }
}

size_t attend_smem_bytes(int c, int H_q) {
  return sizeof(float) * ((size_t)H_q * c + (size_t)kAttKT * (c + 1) + (size_t)H_q * kAttKT +
                          3 * (size_t)H_q);
}

int attend_opt(int c, int H_q) {
  int per = (H_q * c + kAttThreads - 1) / kAttThreads;
  int o = 2;
  while (o < per) o <<= 1;
  return o;
}

}  // namespace

bool attend_simt_supported(int c, int H_q) {
  return attend_smem_bytes(c, H_q) <= 227 * 1024 && attend_opt(c, H_q) <= 128;
}

template <typename Tq, int OPT>
static cudaError_t attend_t(const csa_geom& g, int kv_dt, const void* q, const float* q_gain,
                            const float* sink, const void* E, int64_t ldE, int nseq,
                            const int64_t* n_entries, const int32_t* idx, int k, int dense,
                            const void* win, int64_t ldW, const int32_t* seq_of_q,
                            const int64_t* pos, int Q, int H_q, void* O, cudaStream_t s) {
  size_t smem = attend_smem_bytes(g.c, H_q);
  auto kern = attend_simt_kernel<Tq, OPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  count_launches();
  kern<<<Q, kAttThreads, smem, s>>>(g, kv_dt, reinterpret_cast<const Tq*>(q), q_gain, sink, E,
                                    ldE, nseq, n_entries, idx, k, dense, win, ldW, seq_of_q, pos, H_q,
                                    reinterpret_cast<Tq*>(O));
  return cudaGetLastError();
}

cudaError_t launch_attend_simt(const csa_geom& g, int q_dt, int kv_dt, const void* q,
                               const float* q_gain, const float* sink, const void* E,
                               int64_t ldE, int nseq, const int64_t* n_entries,
                               const int32_t* idx, int k,
                               int dense, const void* win, int64_t ldW, const int32_t* seq_of_q,
                               const int64_t* pos, int Q, int H_q, void* O, cudaStream_t s) {
  if (Q == 0) return cudaSuccess;
  const int opt = attend_opt(g.c, H_q);
#define CSA_ATT_CASE(OP)                                                                        \
  if (opt == OP)                                                                                \
    return q_dt == CSA_F32 ? attend_t<float, OP>(g, kv_dt, q, q_gain, sink, E, ldE, nseq, n_entries,  \
                                                 idx, k, dense, win, ldW, seq_of_q, pos, Q,     \
                                                 H_q, O, s)                                     \
                           : attend_t<__nv_bfloat16, OP>(g, kv_dt, q, q_gain, sink, E, ldE,     \
                                                         nseq, n_entries, idx, k, dense, win, ldW,    \
                                                         seq_of_q, pos, Q, H_q, O, s);
  CSA_ATT_CASE(2)
  CSA_ATT_CASE(4)
  CSA_ATT_CASE(8)
  CSA_ATT_CASE(16)
  CSA_ATT_CASE(32)
  CSA_ATT_CASE(64)
  CSA_ATT_CASE(128)
#undef CSA_ATT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace csa
