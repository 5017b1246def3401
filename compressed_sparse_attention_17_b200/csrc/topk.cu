// topk.cu - exact top-k selection of lightning-indexer scores.
//
// Keeps, per query, the k_eff = min(k, n_vis) entries with the largest
// score; equal scores keep the lower entry index; the kept indices are
// written in ascending order and padded with -1 ("Evidence Ledger", CSA
// Eqs 13-17: top-k selects compressed blocks).
//
// The order is total on pairs (score, -index). A block finds the k-th
// largest pair of its keys and keeps every pair at or above it, in index
// order. Finding it: a value histogram between the block's minimum and
// maximum score (2048 bins; the bin is a non-decreasing function of the
// score, so every key of a higher bin has a larger score) locates the bin
// of the k-th largest key; only that bin's keys are then ranked exactly -
// by counting when they are few, else by radix select on unique 64-bit
// (order-preserving score, inverted index) keys.
//
// Long score rows are cut into chunks of up to 32,768 keys (one block
// each, keys cached in shared memory); each chunk keeps its own top k and a
// second pass selects from the concatenated chunk results, which are in
// index order. Every member of the global top k is in its chunk's top k
// under the same order.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxChunk = 32768;
constexpr int kCandCap = 4096;  // candidates of the k-th key's bin kept in shared memory
constexpr int kRankMax = 1024;  // candidates ranked by counting

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Unique key of (score, index): larger is better.
__device__ __forceinline__ uint64_t pair_key(float s, int32_t id) {
  return ((uint64_t)order_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)id);
}

struct Scratch {
  int hist[kBins];
  uint64_t cand[kCandCap];
  float red_f[2][kWarps];
  int scan[kWarps];
  int ncand;
  int bstar;
  int above;
  uint64_t kth;
  uint64_t prefix;
  int remaining;
};

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

// k-th largest (1-based k) of n unique 64-bit keys given by key_of(i),
// by radix select over 8-bit digits. Slow path: many equal scores.
template <typename KeyOf>
__device__ uint64_t radix_kth64(KeyOf key_of, int n, int k, Scratch& S) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint64_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    if (tid < 256) S.hist[tid] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint64_t key = key_of(i);
      if ((key & mask) == prefix) atomicAdd(&S.hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (wid == 0) {
      int cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = S.hist[255 - (8 * lane + j)];
        sum += cnt[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int cum = incl - sum;
      if (cum < remaining && remaining <= incl) {
        for (int j = 0; j < 8; ++j) {
          if (cum + cnt[j] >= remaining) {
            S.prefix = prefix | ((uint64_t)(255 - (8 * lane + j)) << shift);
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
    mask |= (uint64_t)255u << shift;
    __syncthreads();
  }
  return prefix;  // keys are unique: exactly one key matches
}

// k-th largest pair among n > k keys (scores sc[i], ids id_of(i)).
template <typename IdOf>
__device__ uint64_t kth_pair(const float* sc, IdOf id_of, int n, int k, Scratch& S) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // 1. score range
  float mn = INFINITY, mx = -INFINITY;
  for (int i = tid; i < n; i += kThreads) {
    mn = fminf(mn, sc[i]);
    mx = fmaxf(mx, sc[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    S.red_f[0][wid] = mn;
    S.red_f[1][wid] = mx;
  }
  for (int i = tid; i < kBins; i += kThreads) S.hist[i] = 0;
  if (tid == 0) S.ncand = 0;
  __syncthreads();
  mn = INFINITY;
  mx = -INFINITY;
  for (int w = 0; w < kWarps; ++w) {
    mn = fminf(mn, S.red_f[0][w]);
    mx = fmaxf(mx, S.red_f[1][w]);
  }
  const float span = mx - mn;
  const float scale = (span > 0.f && span < INFINITY) ? (float)kBins / span : 0.f;
  auto bin_of = [&](float s) {
    const int b = (int)((s - mn) * scale);
    return b < 0 ? 0 : (b >= kBins ? kBins - 1 : b);
  };
  // 2. value histogram
  for (int i = tid; i < n; i += kThreads) atomicAdd(&S.hist[bin_of(sc[i])], 1);
  __syncthreads();
  // 3. bin of the k-th largest: lane L owns bins 2047-64L .. 1984-64L
  if (wid == 0) {
    int sum = 0;
    for (int j = 0; j < 64; ++j) sum += S.hist[kBins - 1 - (64 * lane + j)];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int cum = incl - sum;
    if (cum < k && k <= incl) {
      for (int j = 0; j < 64; ++j) {
        const int b = kBins - 1 - (64 * lane + j);
        if (cum + S.hist[b] >= k) {
          S.bstar = b;
          S.above = cum;
          break;
        }
        cum += S.hist[b];
      }
    }
  }
  __syncthreads();
  const int bstar = S.bstar, need = k - S.above, c = S.hist[bstar];
  if (c <= kCandCap) {
    // 4. the k-th pair is the need-th largest key of bin bstar
    for (int i = tid; i < n; i += kThreads) {
      if (bin_of(sc[i]) == bstar) S.cand[atomicAdd(&S.ncand, 1)] = pair_key(sc[i], id_of(i));
    }
    __syncthreads();
    if (c <= kRankMax) {
      if (tid < c) {
        const uint64_t me = S.cand[tid];
        int rank = 0;
        for (int j = 0; j < c; ++j) rank += S.cand[j] > me;
        if (rank == need - 1) S.kth = me;
      }
      __syncthreads();
      return S.kth;
    }
    return radix_kth64([&](int i) { return S.cand[i]; }, c, need, S);
  }
  // many keys share a bin (e.g. equal scores): radix over all keys
  return radix_kth64([&](int i) { return pair_key(sc[i], id_of(i)); }, n, k, S);
}

// Keeps every key whose pair is >= the k-th largest (all keys when n <= k),
// writing ids (and scores) in position order; returns the count kept.
template <typename IdOf>
__device__ int select_block(const float* sc, IdOf id_of, int n, int k, Scratch& S, int32_t* out_idx,
                            float* out_score) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < n; i += kThreads) {
      out_idx[i] = id_of(i);
      if (out_score) out_score[i] = sc[i];
    }
    return n;
  }
  const uint64_t kth = kth_pair(sc, id_of, n, k, S);
  const int per = (n + kThreads - 1) / kThreads;
  const int a0 = min(n, tid * per), a1 = min(n, a0 + per);
  int cnt = 0;
  for (int i = a0; i < a1; ++i) cnt += pair_key(sc[i], id_of(i)) >= kth;
  int tot;
  int o = block_exclusive_scan(cnt, S.scan, &tot);
  for (int i = a0; i < a1; ++i) {
    if (pair_key(sc[i], id_of(i)) >= kth) {
      out_idx[o] = id_of(i);
      if (out_score) out_score[o] = sc[i];
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
  float* cand_score;  // [Q][nchunks][k]
  int32_t* cand_idx;  // [Q][nchunks][k]
  int32_t* cand_n;    // [Q][nchunks]
};

__device__ __forceinline__ int64_t nvis_of(const Params& P, int q) {
  const int b = P.seq_of_q[q];
  if (b < 0 || b >= P.nseq) return 0;
  return n_visible(P.pos[q], P.g.m, P.g.vis_offset, min(P.n_entries[b], P.ld_scores));
}

__global__ void __launch_bounds__(kThreads) topk_chunk_kernel(Params P) {
  extern __shared__ float sc[];
  __shared__ Scratch S;
  const int q = blockIdx.y, ch = blockIdx.x;
  const int64_t nv = nvis_of(P, q);
  const int64_t c0 = (int64_t)ch * P.chunk;
  const int n = (int)max((int64_t)0, min(P.chunk, nv - c0));
  const float* src = P.scores + (int64_t)q * P.ld_scores + c0;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const float f = src[i];
    sc[i] = f;
    if (P.scores_dbg) P.scores_dbg[(int64_t)q * P.ld_dbg + c0 + i] = f;
  }
  __syncthreads();
  auto id_of = [&](int i) { return (int32_t)(c0 + i); };
  if (P.nchunks == 1) {
    int32_t* out = P.idx_out + (int64_t)q * P.k;
    const int w = select_block(sc, id_of, n, P.k, S, out, nullptr);
    for (int j = w + threadIdx.x; j < P.k; j += kThreads) out[j] = -1;
  } else {
    const int64_t off = ((int64_t)q * P.nchunks + ch) * P.k;
    const int w = select_block(sc, id_of, n, P.k, S, P.cand_idx + off, P.cand_score + off);
    if (threadIdx.x == 0) P.cand_n[(int64_t)q * P.nchunks + ch] = w;
  }
}

__global__ void __launch_bounds__(kThreads) topk_merge_kernel(Params P) {
  extern __shared__ float sm[];
  __shared__ Scratch S;
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
  float* sc = sm;
  int32_t* ids = reinterpret_cast<int32_t*>(sm + (int64_t)P.nchunks * P.k);
  for (int c = 0; c < P.nchunks; ++c) {
    const int cnt = offs[c + 1] - offs[c];
    const int64_t off = ((int64_t)q * P.nchunks + c) * P.k;
    for (int i = threadIdx.x; i < cnt; i += kThreads) {
      sc[offs[c] + i] = P.cand_score[off + i];
      ids[offs[c] + i] = P.cand_idx[off + i];
    }
  }
  __syncthreads();
  int32_t* out = P.idx_out + (int64_t)q * P.k;
  const int w = select_block(sc, [&](int i) { return ids[i]; }, n, P.k, S, out, nullptr);
  for (int j = w + threadIdx.x; j < P.k; j += kThreads) out[j] = -1;
}

void plan(int64_t ld_scores, int64_t* chunk, int* nchunks) {
  int64_t c = ld_scores <= kMaxChunk ? ld_scores : kMaxChunk;
  if (c < 1) c = 1;
  *chunk = c;
  *nchunks = (int)max((int64_t)1, (ld_scores + c - 1) / c);
}

}  // namespace

bool topk_supported(int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, &chunk, &nchunks);
  // merge block: candidates (8 bytes each) plus the static selection scratch
  return nchunks <= 64 && (int64_t)nchunks * k * 8 <= 180 * 1024;
}

size_t topk_workspace(int Q, int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, &chunk, &nchunks);
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
  plan(ld_scores, &P.chunk, &P.nchunks);
  if (P.nchunks > 1) {
    if (!cand_ws) return cudaErrorInvalidValue;
    P.cand_score = reinterpret_cast<float*>(cand_ws);
    P.cand_idx = reinterpret_cast<int32_t*>(P.cand_score + (size_t)Q * P.nchunks * k);
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
