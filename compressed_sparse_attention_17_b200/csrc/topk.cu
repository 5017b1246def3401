// topk.cu - exact top-k selection of lightning-indexer scores.
//
// Keeps, per query, the k_eff = min(k, n_vis) entries with the largest
// score; equal scores keep the lower entry index; the kept indices are
// written in ascending order and padded with -1 ("Evidence Ledger", CSA
// Eqs 13-17: top-k selects compressed blocks).
//
// Two levels, both exact. Stage 1: the visible range of a query is cut into
// chunks; one block per chunk caches the chunk's order-preserving keys in
// shared memory and radix-selects the chunk's own top-k (four 8-bit digit
// passes with per-warp histograms). Every member of the global top-k is in
// its chunk's top-k under the same (score, lower index) order. Stage 2 runs
// the same selection over the concatenated chunk candidates, which are
// already in index order. With a single chunk stage 1 writes the answer.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = lane < kWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) sh[lane] = s;
  }
  __syncthreads();
  const int base = wid > 0 ? sh[wid - 1] : 0;
  *total = sh[kWarps - 1];
  __syncthreads();
  return base + x - v;
}

struct SelectScratch {
  int hist[256];
  int scan[kWarps];
  uint32_t prefix;
  int remaining;
};

// Radix select over keys[0..n): returns the k-th largest key (thr) and how
// many keys equal to thr are kept (ties), for k < n.
__device__ void radix_threshold(const uint32_t* keys, int n, int k, SelectScratch& S,
                                uint32_t* thr_out, int* ties_out) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) S.hist[tid] = 0;
    __syncthreads();
    // warp-aggregated increments: lanes with the same digit add once
    for (int i0 = wid * 32; i0 < n; i0 += kThreads) {
      const int i = i0 + lane;
      const uint32_t key = i < n ? keys[i] : 0u;
      const bool act = i < n && (key & mask) == prefix;
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t dg = (key >> shift) & 255u;
        const unsigned peers = __match_any_sync(am, dg);
        if ((int)(__ffs(peers) - 1) == lane) atomicAdd(&S.hist[dg], __popc(peers));
      }
    }
    __syncthreads();
    if (wid == 0) {
      // lane L owns digits 255-8L .. 248-8L (descending)
      int cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = S.hist[255 - (8 * lane + j)];
        cnt[j] = c;
        sum += c;
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int cum = incl - sum;  // keys with a larger digit than this lane's first
      if (cum < remaining && remaining <= incl) {
        for (int j = 0; j < 8; ++j) {
          if (cum + cnt[j] >= remaining) {
            S.prefix = prefix | ((uint32_t)(255 - (8 * lane + j)) << shift);
            S.remaining = remaining - cum;
            break;
          }
          cum += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix = S.prefix;
    remaining = S.remaining;
    mask |= 255u << shift;
    __syncthreads();
  }
  *thr_out = prefix;
  *ties_out = remaining;
}

// Keeps the k largest keys (ties to lower position) and writes their ids in
// position order: out_idx[j] = ids[pos] (or base + pos when ids == nullptr),
// out_key[j] = key when out_key != nullptr. Returns the number written.
__device__ int select_and_compact(const uint32_t* keys, const int32_t* ids, int64_t base, int n,
                                  int k, SelectScratch& S, int32_t* out_idx, uint32_t* out_key) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < n; i += kThreads) {
      out_idx[i] = ids ? ids[i] : (int32_t)(base + i);
      if (out_key) out_key[i] = keys[i];
    }
    return n;
  }
  uint32_t thr;
  int take;
  radix_threshold(keys, n, k, S, &thr, &take);
  const int per = (n + kThreads - 1) / kThreads;
  const int a0 = min(n, tid * per), a1 = min(n, a0 + per);
  int nsel = 0, ntie = 0;
  for (int i = a0; i < a1; ++i) {
    nsel += keys[i] > thr;
    ntie += keys[i] == thr;
  }
  int tot;
  const int tie_base = block_exclusive_scan(ntie, S.scan, &tot);
  int mine = take - tie_base;
  mine = mine < 0 ? 0 : (mine > ntie ? ntie : mine);
  int o = block_exclusive_scan(nsel + mine, S.scan, &tot);
  int seen = 0;
  for (int i = a0; i < a1; ++i) {
    bool keep = keys[i] > thr;
    if (keys[i] == thr) keep = seen++ < mine;
    if (keep) {
      out_idx[o] = ids ? ids[i] : (int32_t)(base + i);
      if (out_key) out_key[o] = keys[i];
      ++o;
    }
  }
  return k;
}

struct Params {
  csa_geom g;
  const float* scores;
  int64_t ld_scores;
  int nseq;
  const int32_t* seq_of_q;
  const int64_t* pos;
  const int64_t* n_entries;
  int k;
  int64_t chunk;
  int nchunks;
  int32_t* idx_out;
  float* scores_dbg;
  int64_t ld_dbg;
  uint32_t* cand_key;  // [Q][nchunks][k]
  int32_t* cand_idx;   // [Q][nchunks][k]
  int32_t* cand_n;     // [Q][nchunks]
};

__device__ __forceinline__ int64_t nvis_of(const Params& P, int q) {
  const int b = P.seq_of_q[q];
  if (b < 0 || b >= P.nseq) return 0;
  return n_visible(P.pos[q], P.g.m, P.g.vis_offset, min(P.n_entries[b], P.ld_scores));
}

__global__ void __launch_bounds__(kThreads) topk_chunk_kernel(Params P) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectScratch S;
  const int q = blockIdx.y, ch = blockIdx.x;
  const int64_t nv = nvis_of(P, q);
  const int64_t c0 = (int64_t)ch * P.chunk;
  const int n = (int)max((int64_t)0, min(P.chunk, nv - c0));
  const float* sc = P.scores + (int64_t)q * P.ld_scores + c0;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const float f = sc[i];
    keys[i] = order_key(f);
    if (P.scores_dbg) P.scores_dbg[(int64_t)q * P.ld_dbg + c0 + i] = f;
  }
  __syncthreads();
  if (P.nchunks == 1) {
    int32_t* out = P.idx_out + (int64_t)q * P.k;
    const int w = select_and_compact(keys, nullptr, c0, n, P.k, S, out, nullptr);
    for (int j = w + threadIdx.x; j < P.k; j += kThreads) out[j] = -1;
  } else {
    const int64_t off = ((int64_t)q * P.nchunks + ch) * P.k;
    const int w = select_and_compact(keys, nullptr, c0, n, P.k, S, P.cand_idx + off, P.cand_key + off);
    if (threadIdx.x == 0) P.cand_n[(int64_t)q * P.nchunks + ch] = w;
  }
}

__global__ void __launch_bounds__(kThreads) topk_merge_kernel(Params P) {
  extern __shared__ uint32_t sm[];
  __shared__ SelectScratch S;
  __shared__ int offs[65];
  const int q = blockIdx.x;
  if (threadIdx.x == 0) {
    int o = 0;
    for (int c = 0; c < P.nchunks; ++c) {
      offs[c] = o;
      o += P.cand_n[(int64_t)q * P.nchunks + c];
    }
    offs[P.nchunks] = o;
  }
  __syncthreads();
  const int n = offs[P.nchunks];
  uint32_t* keys = sm;
  int32_t* ids = reinterpret_cast<int32_t*>(sm + (int64_t)P.nchunks * P.k);
  for (int c = 0; c < P.nchunks; ++c) {
    const int cnt = offs[c + 1] - offs[c];
    const int64_t off = ((int64_t)q * P.nchunks + c) * P.k;
    for (int i = threadIdx.x; i < cnt; i += kThreads) {
      keys[offs[c] + i] = P.cand_key[off + i];
      ids[offs[c] + i] = P.cand_idx[off + i];
    }
  }
  __syncthreads();
  int32_t* out = P.idx_out + (int64_t)q * P.k;
  const int w = select_and_compact(keys, ids, 0, n, P.k, S, out, nullptr);
  for (int j = w + threadIdx.x; j < P.k; j += kThreads) out[j] = -1;
}

constexpr int64_t kMaxChunk = 51200;  // keys per stage-1 block (200 KB of shared memory)

void plan(int64_t ld_scores, int k, int64_t* chunk, int* nchunks) {
  const int max_chunks = (int)max((int64_t)1, min((int64_t)16, (int64_t)24576 / k));
  int64_t c = max((int64_t)8192, (ld_scores + max_chunks - 1) / max_chunks);
  c = min(kMaxChunk, (c + 1023) / 1024 * 1024);
  *chunk = c;
  *nchunks = (int)max((int64_t)1, (ld_scores + c - 1) / c);
}

}  // namespace

bool topk_supported(int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, k, &chunk, &nchunks);
  return nchunks <= 16 && (int64_t)nchunks * k * 8 <= 200 * 1024;
}

size_t topk_workspace(int Q, int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, k, &chunk, &nchunks);
  if (nchunks == 1) return 0;
  return (size_t)Q * nchunks * ((size_t)k * 8 + 4);
}

cudaError_t launch_topk(const csa_geom& g, const float* scores, int64_t ld_scores, int nseq,
                        const int32_t* seq_of_q, const int64_t* pos, const int64_t* n_entries,
                        int Q, int k, int32_t* idx_out, float* scores_dbg, int64_t ld_dbg,
                        void* cand_ws, cudaStream_t s) {
  if (Q == 0) return cudaSuccess;
  Params P{};
  P.g = g;
  P.scores = scores;
  P.ld_scores = ld_scores;
  P.nseq = nseq;
  P.seq_of_q = seq_of_q;
  P.pos = pos;
  P.n_entries = n_entries;
  P.k = k;
  P.idx_out = idx_out;
  P.scores_dbg = scores_dbg;
  P.ld_dbg = ld_dbg;
  plan(ld_scores, k, &P.chunk, &P.nchunks);
  if (P.nchunks > 1) {
    if (!cand_ws) return cudaErrorInvalidValue;
    P.cand_key = reinterpret_cast<uint32_t*>(cand_ws);
    P.cand_idx = reinterpret_cast<int32_t*>(P.cand_key + (size_t)Q * P.nchunks * k);
    P.cand_n = P.cand_idx + (size_t)Q * P.nchunks * k;
  }
  const size_t smem1 = (size_t)P.chunk * 4;
  cudaError_t e = cudaFuncSetAttribute(topk_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem1);
  if (e != cudaSuccess) return e;
  if (Q > 65535) return cudaErrorInvalidValue;
  count_launches();
  topk_chunk_kernel<<<dim3((unsigned)P.nchunks, (unsigned)Q), kThreads, smem1, s>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess || P.nchunks == 1) return e;
  const size_t smem2 = (size_t)P.nchunks * k * 8;
  e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (e != cudaSuccess) return e;
  count_launches();
  topk_merge_kernel<<<Q, kThreads, smem2, s>>>(P);
  return cudaGetLastError();
}

}  // namespace csa
