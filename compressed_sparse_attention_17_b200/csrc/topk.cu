// topk.cu - exact top-k selection of lightning-indexer scores.
//
// Keeps, per query, the k_eff = min(k, n_vis) entries with the largest
// score; equal scores keep the lower entry index; the kept indices are
// written in ascending order and padded with -1 ("Evidence Ledger", CSA
// Eqs 13-17: top-k selects compressed blocks).
//
// The order is total on pairs (score, -index), encoded as unique 64-bit keys
// (order-preserving score bits, inverted index). A selection finds the k-th
// largest key of a segment and keeps every key at or above it, in index
// order.
//
// One thread-block cluster (up to 8 CTAs) works on one segment; each thread
// holds its keys in registers (warp w of CTA r owns a contiguous span, lane
// l the keys span + 32 j + l, so every load is one coalesced line per warp).
// The CTAs exchange partial results through distributed shared memory:
//   1. the score range [min, max] of the segment;
//   2. a 2048-bin value histogram over that range (the bin is a
//      non-decreasing function of the score, so every key of a higher bin is
//      larger); the cluster's totals of 8 slices of 256 bins locate the slice
//      holding the k-th largest key, and that slice's bins, summed over the
//      cluster, the bin and how many keys lie above it;
//   3. that bin's keys (usually a few dozen) are gathered into every CTA and
//      ranked exactly - by counting, or by radix select when there are many;
//      when they do not fit (many equal scores), a cluster-wide radix select
//      over all keys takes over;
//   4. ordered compaction: per-warp ballots, a block scan and the cluster's
//      per-CTA counts give each kept key its output slot.
// Rows longer than one cluster's capacity (65,536 keys) are cut into chunks;
// each chunk keeps its own top k (every member of the row's top k is in its
// chunk's top k under the same order) and a second selection runs over the
// chunk results, which are dense and in index order.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace csa {

namespace {

constexpr int kBins = 2048;
constexpr int kKptMax = 16;     // keys per thread
constexpr int kMaxCluster = 8;  // portable cluster size
constexpr int kBigThreads = 512;
constexpr int kSmallThreads = 256;
constexpr int64_t kSegMax = (int64_t)kMaxCluster * kBigThreads * kKptMax;  // 65,536 keys
constexpr int kLocCap = 1024;   // a CTA's keys of the k-th key's bin
constexpr int kGathCap = 2048;  // the cluster's keys of that bin
constexpr int kRankMax = 256;   // ranked by counting up to this many

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Unique key of (score, index): larger is better.
__device__ __forceinline__ uint64_t pair_key(float s, int32_t id) {
  return ((uint64_t)order_key(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)id);
}

template <int NT>
struct Smem {
  int hist[kBins];  // this CTA's value histogram
  int stot[8];      // this CTA's counts in 8 slices of 256 bins
  uint64_t loc[kLocCap];
  uint64_t gath[kGathCap];
  int rhist[2][256];
  int scan[NT / 32];
  float red[2][NT / 32];
  int cnt[kMaxCluster], off[kMaxCluster];
  float mn, mx, gmn, gmx;
  int nloc, tot, over;
  int bstar, above, sstar, above0;
  int digit, rem;
  int kept, cbase, ctot;
  uint64_t kth;
};

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Barrier over the cluster's CTAs (a block barrier when the cluster is one CTA).
__device__ __forceinline__ void csync(int C) {
  if (C > 1) {
    cluster_arrive();
    cluster_wait();
  } else {
    __syncthreads();
  }
}
// The same shared-memory object in CTA r of the cluster.
template <typename T>
__device__ __forceinline__ T* peer(T* p, int r, int C) {
  return C > 1 ? cg::this_cluster().map_shared_rank(p, r) : p;
}

template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  constexpr int W = NT / 32;
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
    int s = lane < W ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < W) sh[lane] = s;
  }
  __syncthreads();
  const int base = wid > 0 ? sh[wid - 1] : 0;
  *total = sh[W - 1];
  __syncthreads();
  return base + x - v;
}

// need-th largest (1-based) of unique 64-bit keys, by radix select over
// 8-bit digits. Every thread hands its keys to the callback of for_each;
// with C > 1 the keys are spread over the cluster's CTAs and the digit
// histograms are summed across it (double-buffered: a CTA clears buffer
// pass & 1 only after the barrier of the previous pass, which every peer
// reaches after its last read of that buffer).
template <int NT, typename ForEach>
__device__ uint64_t radix_select(ForEach for_each, int need, Smem<NT>& S, int C) {
  const int tid = threadIdx.x;
  uint64_t prefix = 0, mask = 0;
  int rem = need;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    int* h = S.rhist[pass & 1];
    for (int i = tid; i < 256; i += NT) h[i] = 0;
    __syncthreads();
    for_each([&](uint64_t key) {
      if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1);
    });
    csync(C);
    int cnt = 0;
    if (tid < 256) {
      for (int r = 0; r < C; ++r) cnt += peer(h, r, C)[255 - tid];
    }
    int tot;
    const int ex = block_exclusive_scan<NT>(cnt, S.scan, &tot);
    if (tid < 256 && ex < rem && rem <= ex + cnt) {
      S.digit = 255 - tid;
      S.rem = rem - ex;
    }
    __syncthreads();
    prefix |= (uint64_t)S.digit << shift;
    rem = S.rem;
    mask |= (uint64_t)0xFFu << shift;
  }
  return prefix;  // the keys are unique: exactly one matches
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
  int64_t chunk;  // keys per chunk of a score row
  int nchunks;
  int csize;  // CTAs per cluster (one cluster per segment)
  int kpt;    // keys per thread
  int32_t* idx_out;
  float* scores_dbg;
  int64_t ld_dbg;
  float* cand_score;  // [Q][nchunks][k]: chunk results (when nchunks > 1)
  int32_t* cand_idx;
};

__device__ __forceinline__ int64_t nvis_of(const Params& P, int q) {
  const int b = P.seq_of_q[q];
  if (b < 0 || b >= P.nseq) return 0;
  return n_visible(P.pos[q], P.g.m, P.g.vis_offset, min(P.n_entries[b], P.ld_scores));
}

__device__ __forceinline__ int chunk_len(const Params& P, int64_t nv, int c) {
  const int64_t c0 = (int64_t)c * P.chunk;
  return (int)max((int64_t)0, min(P.chunk, nv - c0));
}

// CAND = false: segment = chunk ch of query q's score row; the result goes
// to idx_out (one chunk) or to the chunk's candidate slots.
// CAND = true: segment = query q's chunk results, concatenated (dense: every
// chunk before the last non-empty one kept exactly k); result to idx_out.
// Every branch that contains a cluster barrier depends only on values that
// all CTAs of the cluster share, so each CTA takes the same barriers.
template <int NT, int KPT, bool CAND>
__global__ void __launch_bounds__(NT, CAND ? 1 : 1024 / NT) topk_cluster_kernel(Params P) {
  __shared__ Smem<NT> S;
  pdl_wait();  // the scores of the previous kernel are visible from here on
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int C = P.csize, kpt = P.kpt, k = P.k;
  const int rank = (int)(blockIdx.x % (unsigned)C);
  const int64_t seg = blockIdx.x / (unsigned)C;
  const int nseg = CAND ? 1 : P.nchunks;
  const int q = (int)(seg / nseg), ch = (int)(seg % nseg);
  const int64_t nv = nvis_of(P, q);
  int n;
  int64_t c0 = 0;
  const float* src_s;
  const int32_t* src_i = nullptr;
  if (!CAND) {
    n = chunk_len(P, nv, ch);
    c0 = (int64_t)ch * P.chunk;
    src_s = P.scores + (int64_t)q * P.ld_scores + c0;
  } else {
    n = 0;
    for (int c = 0; c < P.nchunks; ++c) n += min(k, chunk_len(P, nv, c));
    const int64_t o = (int64_t)q * P.nchunks * k;
    src_s = P.cand_score + o;
    src_i = P.cand_idx + o;
  }

  // ---- keys of this thread (registers)
  const int base = (rank * NT + wid * 32) * kpt;  // index of this warp's first key
  float s[KPT];
  int32_t idc[CAND ? KPT : 1];  // entry indices (computed from the position otherwise)
  uint32_t vm = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    s[j] = 0.f;
    const int i = base + 32 * j + lane;
    if (j < kpt && i < n) {
      vm |= 1u << j;
      s[j] = src_s[i];
    }
    if (CAND) idc[CAND ? j : 0] = (vm >> j & 1u) ? src_i[i] : 0;
  }
  auto id_of = [&](int j) -> int32_t {
    return CAND ? idc[CAND ? j : 0] : (int32_t)(c0 + base + 32 * j + lane);
  };
  if (!CAND && P.scores_dbg) {
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (vm >> j & 1u) P.scores_dbg[(int64_t)q * P.ld_dbg + id_of(j)] = s[j];
  }

  uint64_t kth = 0;  // keep every key when n <= k
  if (n > k) {
    // 1. score range of the segment
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (vm >> j & 1u) {
        mn = fminf(mn, s[j]);
        mx = fmaxf(mx, s[j]);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
      S.red[0][wid] = mn;
      S.red[1][wid] = mx;
    }
    for (int i = tid; i < kBins; i += NT) S.hist[i] = 0;
    if (tid == 0) S.nloc = 0;
    __syncthreads();
    if (wid == 0) {
      mn = lane < NT / 32 ? S.red[0][lane] : INFINITY;
      mx = lane < NT / 32 ? S.red[1][lane] : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        S.mn = mn;
        S.mx = mx;
      }
    }
    csync(C);
    if (wid == 0) {
      mn = lane < C ? *peer(&S.mn, lane, C) : INFINITY;
      mx = lane < C ? *peer(&S.mx, lane, C) : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        S.gmn = mn;
        S.gmx = mx;
      }
    }
    __syncthreads();
    mn = S.gmn;
    mx = S.gmx;
    const float span = mx - mn;
    const float scale = (span > 0.f && span < INFINITY) ? (float)kBins / span : 0.f;
    auto bin_of = [&](float v) {
      const int b = (int)((v - mn) * scale);
      return b < 0 ? 0 : (b >= kBins ? kBins - 1 : b);
    };

    // 2. value histogram, summed over the cluster
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (vm >> j & 1u) atomicAdd(&S.hist[bin_of(s[j])], 1);
    if (C > 1) {
      // slice totals: warp s counts bins [256 s, 256 s + 256)
      __syncthreads();
      if (wid < 8) {
        int v = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) v += S.hist[256 * wid + 32 * e + lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) S.stot[wid] = v;
      }
      csync(C);
      // the slice holding the k-th largest key, from the top slice down
      if (wid == 0) {
        int tot = 0;
        if (lane < 8)
          for (int r = 0; r < C; ++r) tot += peer(S.stot, r, C)[lane];
        // suffix sums over the slices (inclusive, then exclusive)
        int suf = lane < 8 ? tot : 0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 8) suf += y;
        }
        const int ex = suf - (lane < 8 ? tot : 0);
        if (lane < 8 && ex < k && k <= suf) {
          S.sstar = lane;
          S.above0 = ex;
        }
      }
      __syncthreads();
      // its 256 bins summed over the cluster; thread t takes bin 255 - t of the slice
      const int sl = S.sstar;
      int v = 0;
      if (tid < 256) {
        const int b = 256 * sl + 255 - tid;
        for (int r = 0; r < C; ++r) v += peer(S.hist, r, C)[b];
      }
      int tot;
      const int cum = block_exclusive_scan<NT>(v, S.scan, &tot);
      const int need0 = k - S.above0;
      if (tid < 256 && cum < need0 && need0 <= cum + v) {
        S.bstar = 256 * sl + 255 - tid;
        S.above = S.above0 + cum;
      }
      __syncthreads();
    } else {
      // one CTA: bin of the k-th largest over the whole local histogram;
      // thread t owns bins 2047 - BPT t - e, e < BPT
      __syncthreads();
      constexpr int BPT = kBins / NT;
      int cnt[BPT], sum = 0;
#pragma unroll
      for (int e = 0; e < BPT; ++e) {
        cnt[e] = S.hist[kBins - 1 - (BPT * tid + e)];
        sum += cnt[e];
      }
      int tot;
      int cum = block_exclusive_scan<NT>(sum, S.scan, &tot);
      if (cum < k && k <= cum + sum) {
#pragma unroll
        for (int e = 0; e < BPT; ++e) {
          if (cum < k && k <= cum + cnt[e]) {
            S.bstar = kBins - 1 - (BPT * tid + e);
            S.above = cum;
          }
          cum += cnt[e];
        }
      }
      __syncthreads();
    }
    const int bstar = S.bstar, need = k - S.above;

    // 3. keys of that bin, gathered and ranked
    uint64_t* list = C > 1 ? S.loc : S.gath;
    const int cap = C > 1 ? kLocCap : kGathCap;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if ((vm >> j & 1u) && bin_of(s[j]) == bstar) {
        const int p = atomicAdd(&S.nloc, 1);
        if (p < cap) list[p] = pair_key(s[j], id_of(j));
      }
    csync(C);
    if (wid == 0) {
      const int c = lane < C ? *peer(&S.nloc, lane, C) : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const bool bad = __any_sync(0xffffffffu, c > cap);
      if (lane < C) {
        S.cnt[lane] = c;
        S.off[lane] = incl - c;
      }
      if (lane == 31) {
        S.tot = incl;
        S.over = bad || incl > kGathCap;
      }
    }
    __syncthreads();
    const int tot = S.tot;
    if (!S.over) {
      if (C > 1) {
        for (int r = 0; r < C; ++r) {
          const uint64_t* rl = peer(S.loc, r, C);
          const int c = S.cnt[r], o = S.off[r];
          for (int i = tid; i < c; i += NT) S.gath[o + i] = rl[i];
        }
        __syncthreads();
      }
      if (tot <= kRankMax) {
        if (tid < tot) {
          const uint64_t me = S.gath[tid];
          int r = 0;
          for (int j = 0; j < tot; ++j) r += S.gath[j] > me;
          if (r == need - 1) S.kth = me;
        }
        __syncthreads();
        kth = S.kth;
      } else {
        kth = radix_select<NT>(
            [&](auto&& f) {
              for (int i = tid; i < tot; i += NT) f(S.gath[i]);
            },
            need, S, 1);
      }
    } else {
      // many keys in one bin (equal scores): radix select over all keys
      kth = radix_select<NT>(
          [&](auto&& f) {
#pragma unroll
            for (int j = 0; j < KPT; ++j)
              if (vm >> j & 1u) f(pair_key(s[j], id_of(j)));
          },
          k, S, C);
    }
  }

  // 4. ordered compaction of the keys >= kth (ballots taken twice: to count,
  // then to place)
  auto keep_mask = [&](int j) {
    return __ballot_sync(0xffffffffu, (vm >> j & 1u) && pair_key(s[j], id_of(j)) >= kth);
  };
  int wcnt = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) wcnt += __popc(keep_mask(j));
  if (lane == 0) S.scan[wid] = wcnt;
  __syncthreads();
  int woff = 0, ckept = 0;
  for (int w = 0; w < NT / 32; ++w) {
    const int v = S.scan[w];
    woff += w < wid ? v : 0;
    ckept += v;
  }
  if (tid == 0) S.kept = ckept;
  csync(C);
  if (wid == 0) {
    const int c = lane < C ? *peer(&S.kept, lane, C) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == rank) S.cbase = incl - c;
    if (lane == 31) S.ctot = incl;
  }
  __syncthreads();
  if (C > 1) cluster_arrive();  // this CTA reads no peer memory from here on
  const int cbase = S.cbase, ctot = S.ctot;
  const bool to_cand = !CAND && P.nchunks > 1;
  int32_t* out_i = to_cand ? P.cand_idx + ((int64_t)q * P.nchunks + ch) * k
                           : P.idx_out + (int64_t)q * k;
  float* out_s = to_cand ? P.cand_score + ((int64_t)q * P.nchunks + ch) * k : nullptr;
  const uint32_t lt = (1u << lane) - 1u;
  int o = cbase + woff;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const uint32_t ball = keep_mask(j);
    if (ball >> lane & 1u) {
      const int p = o + __popc(ball & lt);
      if (p < k) {
        out_i[p] = id_of(j);
        if (to_cand) out_s[p] = s[j];
      }
    }
    o += __popc(ball);
  }
  if (!to_cand && rank == C - 1)
    for (int p = ctot + tid; p < k; p += NT) out_i[p] = -1;
  if (C > 1) cluster_wait();  // peers have finished reading this CTA's memory
}

struct Shape {
  int nt, csize, kpt;
};

// Threads per CTA, cluster size and keys per thread for segments of up to
// len keys (about 8 keys a thread, at most kKptMax).
Shape shape_for(int64_t len) {
  Shape sh;
  sh.nt = len <= (int64_t)kSmallThreads * 8 ? kSmallThreads : kBigThreads;
  const int64_t per8 = (int64_t)sh.nt * 8;
  const int64_t c = (len + per8 - 1) / per8;
  sh.csize = (int)(c < 1 ? 1 : (c > kMaxCluster ? kMaxCluster : c));
  const int64_t per_cta = (len + sh.csize - 1) / sh.csize;
  sh.kpt = (int)((per_cta + sh.nt - 1) / sh.nt);
  if (sh.kpt < 1) sh.kpt = 1;
  return sh;
}

void plan(int64_t ld_scores, int64_t* chunk, int* nchunks) {
  if (ld_scores <= kSegMax) {
    *chunk = ld_scores < 1 ? 1 : ld_scores;
    *nchunks = 1;
    return;
  }
  const int64_t nc = (ld_scores + kSegMax - 1) / kSegMax;
  *nchunks = (int)nc;
  *chunk = (ld_scores + nc - 1) / nc;
}

template <int NT, int KPT, bool CAND>
cudaError_t launch_one(const Params& P, int64_t nseg, cudaStream_t s) {
  const int64_t blocks = nseg * P.csize;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = 0;
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
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<NT, KPT, CAND>, P);
}

template <bool CAND>
cudaError_t launch_shape(Params P, const Shape& sh, int64_t nseg, cudaStream_t s) {
  P.csize = sh.csize;
  P.kpt = sh.kpt;
  if (sh.nt == kSmallThreads) return launch_one<kSmallThreads, 8, CAND>(P, nseg, s);
  if (sh.kpt <= 8) return launch_one<kBigThreads, 8, CAND>(P, nseg, s);
  if (sh.kpt <= 12) return launch_one<kBigThreads, 12, CAND>(P, nseg, s);
  return launch_one<kBigThreads, kKptMax, CAND>(P, nseg, s);
}

}  // namespace

bool topk_supported(int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, &chunk, &nchunks);
  // the chunk results of a row form one segment of the second selection
  return nchunks == 1 || ((int64_t)nchunks * k <= kSegMax && chunk >= k);
}

size_t topk_workspace(int Q, int64_t ld_scores, int k) {
  int64_t chunk;
  int nchunks;
  plan(ld_scores, &chunk, &nchunks);
  if (nchunks == 1) return 0;
  return (size_t)Q * nchunks * (size_t)k * 8;
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
  }
  cudaError_t e = launch_shape<false>(P, shape_for(P.chunk), (int64_t)Q * P.nchunks, s);
  if (e != cudaSuccess || P.nchunks == 1) return e;
  return launch_shape<true>(P, shape_for((int64_t)P.nchunks * k), Q, s);
}

}  // namespace csa
