// api.cu - the extern "C" entry points of libcsa: argument validation on
// the host, then dispatch to the kernels. See include/csa.h for the contract
// of every function.
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace csa {
__device__ int g_device_error = 0;

// Device address of the error word for the current device.
int* device_error_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return reinterpret_cast<int*>(p);
}

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace csa

namespace {

using csa::launch_attend_simt;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline csa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

bool geom_ok(const csa_geom* g) {
  if (!g) return false;
  if (g->m < 1 || (g->overlap != 0 && g->overlap != 1)) return false;
  if (g->c < 16 || g->c > 1024 || (g->c % 16) != 0) return false;
  if (g->rope_dims < 0 || (g->rope_dims & 1) || g->rope_dims > g->c) return false;
  if (!(g->rope_base > 0.0) || !(g->eps >= 0.0f)) return false;
  if (g->vis_offset != 0 && g->vis_offset != 1) return false;
  if (g->n_win < 0 || (g->win_ring != 0 && g->win_ring != 1)) return false;
  if (g->win_ring && g->n_win < 1) return false;
  return true;
}

inline bool io_dtype_ok(int dt) { return dt == CSA_F32 || dt == CSA_BF16; }
inline bool mixed_ok(const csa_geom* g) { return g->c == 512 && g->rope_dims == 64; }

inline bool out_dtype_ok(const csa_geom* g, int dt) {
  return io_dtype_ok(dt) || (dt == CSA_FP8_MIXED && mixed_ok(g));
}

}  // namespace

extern "C" {

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    case CSA_ERR_TOO_LARGE: return "CSA_ERR_TOO_LARGE";
  }
  return "CSA_ERR_UNKNOWN";
}

const char* csa_version(void) { return "libcsa 0.1 (sm_100a)"; }

uint64_t csa_kernel_launches(void) { return csa::g_launches.load(std::memory_order_relaxed); }

csa_status csa_sync_status(csa_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int host_err = 0;
  if (cudaMemcpyFromSymbolAsync(&host_err, csa::g_device_error, sizeof(int), 0,
                                cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CSA_ERR_CUDA;
  if (host_err != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(csa::g_device_error, &zero, sizeof(int)) != cudaSuccess)
      return CSA_ERR_CUDA;
    return host_err == CSA_ERR_TIMEOUT ? CSA_ERR_TIMEOUT : CSA_ERR_CUDA;
  }
  return CSA_OK;
}

csa_status csa_rmsnorm_rope(const csa_geom* g, csa_dtype in_dtype, csa_dtype out_dtype,
                            const void* x, int64_t rows, const int64_t* pos, int64_t pos0,
                            int64_t pos_step, const float* gain, void* out,
                            const int64_t* out_row, csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(in_dtype) || !out_dtype_ok(g, out_dtype)) return CSA_ERR_INVALID_ARG;
  if (rows < 0 || (rows > 0 && (!x || !out))) return CSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned16(gain) || !aligned16(pos) || !aligned16(out_row))
    return CSA_ERR_INVALID_ARG;
  return cuda_status(csa::launch_rmsnorm_rope(*g, in_dtype, out_dtype, x, rows, pos, pos0,
                                              pos_step, gain, out, out_row,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_quantize_mixed(csa_dtype in_dtype, const void* x, int64_t rows, void* out,
                              csa_stream_t stream) {
  if (!io_dtype_ok(in_dtype) || rows < 0 || (rows > 0 && (!x || !out))) return CSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return CSA_ERR_INVALID_ARG;
  return cuda_status(csa::launch_quantize_mixed(in_dtype, x, rows, out,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

size_t csa_compress_workspace_size(const csa_geom* g, csa_dtype dtype, int64_t T, int d) {
  if (!g || T < 0 || g->c <= 0 || g->m < 1) return 0;
  if (csa::proj_tc_supported(*g, dtype, d)) return csa::proj_pool_workspace(*g, T);
  const int nW = g->overlap ? 4 : 2;
  return (size_t)T * nW * g->c * sizeof(float);
}

csa_status csa_compress(const csa_geom* g, csa_dtype dtype, const void* H, int64_t T, int d,
                        const void* W_aKV, const void* W_bKV, const void* W_aZ,
                        const void* W_bZ, const float* bias, const float* gain,
                        csa_dtype out_dtype, void* E_out, void* workspace, size_t ws_bytes,
                        csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(dtype) || !out_dtype_ok(g, out_dtype)) return CSA_ERR_INVALID_ARG;
  if (T < 0 || d < 1) return CSA_ERR_INVALID_ARG;
  if (!H || !W_aKV || !W_aZ || !bias || !E_out) return CSA_ERR_INVALID_ARG;
  if (g->overlap ? (!W_bKV || !W_bZ) : (W_bKV || W_bZ)) return CSA_ERR_INVALID_ARG;
  const void* ptrs[] = {H, W_aKV, W_bKV, W_aZ, W_bZ, bias, gain, E_out, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSA_ERR_INVALID_ARG;
  if (T / g->m == 0) return CSA_OK;
  if (!workspace || ws_bytes < csa_compress_workspace_size(g, dtype, T, d)) return CSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* P = reinterpret_cast<float*>(workspace);
  const int nW = g->overlap ? 4 : 2;
  // projections in the order [C^a | Z^a | C^b | Z^b]
  const void* W[4] = {W_aKV, W_aZ, W_bKV, W_bZ};
  if (csa::proj_tc_supported(*g, dtype, d)) {
    // tensor-core projection with the pool fused, then RMSNorm + RoPE at i*m
    cudaError_t e = csa::launch_compress_tc(*g, H, T, d, W, bias, P, s);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    return cuda_status(csa::launch_rmsnorm_rope(*g, CSA_F32, out_dtype, P, T / g->m, nullptr, 0,
                                                g->m, gain, E_out, nullptr, s));
  }
  const int64_t Tc = (T / g->m) * g->m;  // tokens after the last complete block are unused
  cudaError_t e = csa::launch_proj_simt(dtype, H, Tc, d, g->c, nW, W, P, s);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  return cuda_status(csa::launch_pool_prefill(*g, P, Tc, bias, gain, out_dtype, E_out, s));
}

int64_t csa_compress_decode_state_floats(const csa_geom* g) {
  if (!g || g->m < 1 || g->c < 1) return 0;
  const int nslot = 1 + (g->overlap ? 1 : 0);
  const int nW = g->overlap ? 4 : 2;
  return (int64_t)nslot * g->m * nW * g->c;
}

size_t csa_compress_decode_workspace_size(const csa_geom* g, csa_dtype dtype, int B, int d) {
  if (!g || B <= 0 || d < 1 || g->c <= 0) return 0;
  return csa::proj_decode_supported(*g, dtype, d) ? csa::proj_decode_workspace(*g, B, d) : 0;
}

csa_status csa_compress_decode(const csa_geom* g, csa_dtype dtype, const void* h,
                               const int64_t* pos, int B, int d, const void* W_aKV,
                               const void* W_bKV, const void* W_aZ, const void* W_bZ,
                               const float* bias, const float* gain, float* state,
                               csa_dtype out_dtype, void* E_cache, int64_t ldE, void* workspace,
                               size_t ws_bytes, csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(dtype) || !out_dtype_ok(g, out_dtype)) return CSA_ERR_INVALID_ARG;
  if (B < 0 || d < 1 || ldE < 0) return CSA_ERR_INVALID_ARG;
  if (B == 0) return CSA_OK;
  if (!h || !pos || !W_aKV || !W_aZ || !bias || !state || !E_cache) return CSA_ERR_INVALID_ARG;
  if (g->overlap ? (!W_bKV || !W_bZ) : (W_bKV || W_bZ)) return CSA_ERR_INVALID_ARG;
  const void* ptrs[] = {h, pos, W_aKV, W_bKV, W_aZ, W_bZ, bias, gain, state, E_cache, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nW = g->overlap ? 4 : 2;
  const void* W[4] = {W_aKV, W_aZ, W_bKV, W_bZ};
  const size_t need = csa_compress_decode_workspace_size(g, dtype, B, d);
  if (need > 0 && (!workspace || ws_bytes < need)) return CSA_ERR_INVALID_ARG;
  cudaError_t e = need > 0 ? csa::launch_decode_proj_tc(*g, h, pos, B, d, W,
                                                        reinterpret_cast<float*>(workspace), state, s)
                           : csa::launch_decode_proj(*g, dtype, h, pos, B, d, W, nW, state, s);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  return cuda_status(csa::launch_decode_pool(*g, pos, B, bias, gain, state, out_dtype, E_cache,
                                             ldE, s));
}

// workspace of csa_index_topk: FP32 scores [Q, ldK], then the top-k
// chunk candidates (256-byte aligned)
static size_t scores_bytes(int Q, int64_t ldK) {
  return ((size_t)Q * (size_t)ldK * sizeof(float) + 255) / 256 * 256;
}

size_t csa_index_topk_workspace_size(int Q, int64_t ldK, int k) {
  if (Q < 0 || ldK < 0 || k < 1) return 0;
  return scores_bytes(Q, ldK) + csa::topk_workspace(Q, ldK, k);
}

csa_status csa_index_topk(const csa_geom* g, csa_dtype dtype, const void* qI, const float* w,
                          const void* KI, int64_t ldK, int nseq, const int32_t* seq_of_q,
                          const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                          int c_I, int k, int32_t* idx_out, float* scores_dbg,
                          void* workspace, size_t ws_bytes, csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(dtype)) return CSA_ERR_INVALID_ARG;
  if (Q < 0 || H_I < 1 || H_I > 128 || c_I < 16 || (c_I % 16) != 0 || c_I > 256) return CSA_ERR_INVALID_ARG;
  if (k < 1 || k > CSA_MAX_TOPK || ldK < 0 || nseq < 0) return CSA_ERR_INVALID_ARG;
  if (!csa::topk_supported(ldK, k)) return CSA_ERR_UNSUPPORTED;
  if (Q == 0) return CSA_OK;
  if (!qI || !w || !KI || !seq_of_q || !pos || !n_entries || !idx_out) return CSA_ERR_INVALID_ARG;
  const void* ptrs[] = {qI, w, KI, seq_of_q, pos, n_entries, idx_out, scores_dbg, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSA_ERR_INVALID_ARG;
  if (ldK > 0 && (!workspace || ws_bytes < csa_index_topk_workspace_size(Q, ldK, k)))
    return CSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* scores = reinterpret_cast<float*>(workspace);
  if (ldK > 0 && nseq > 0) {
    cudaError_t e = csa::index_tc_supported(dtype, H_I, c_I)
                        ? csa::launch_index_scores_tc(*g, qI, w, KI, ldK, nseq, seq_of_q, pos,
                                                      n_entries, Q, H_I, c_I, scores, ldK, s)
                        : csa::launch_index_scores_simt(*g, dtype, qI, w, KI, ldK, nseq, seq_of_q,
                                                        pos, n_entries, Q, H_I, c_I, scores, ldK,
                                                        s);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  void* cand = reinterpret_cast<uint8_t*>(workspace) + scores_bytes(Q, ldK);
  return cuda_status(csa::launch_topk(*g, scores, ldK, nseq, seq_of_q, pos, n_entries, Q, k,
                                      idx_out, scores_dbg, ldK, cand, s));
}

csa_status csa_index_scores(const csa_geom* g, csa_dtype dtype, const void* qI, const float* w,
                            const void* KI, int64_t ldK, int nseq, const int32_t* seq_of_q,
                            const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                            int c_I, float* scores, int64_t ld_scores, csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(dtype)) return CSA_ERR_INVALID_ARG;
  if (Q < 0 || H_I < 1 || H_I > 128 || c_I < 16 || (c_I % 16) != 0 || c_I > 256) return CSA_ERR_INVALID_ARG;
  if (ldK < 0 || nseq < 0 || ld_scores < ldK) return CSA_ERR_INVALID_ARG;
  if (Q == 0 || ldK == 0 || nseq == 0) return CSA_OK;
  if (!qI || !w || !KI || !seq_of_q || !pos || !n_entries || !scores) return CSA_ERR_INVALID_ARG;
  const void* ptrs[] = {qI, w, KI, seq_of_q, pos, n_entries, scores};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = csa::index_tc_supported(dtype, H_I, c_I)
                      ? csa::launch_index_scores_tc(*g, qI, w, KI, ldK, nseq, seq_of_q, pos,
                                                    n_entries, Q, H_I, c_I, scores, ld_scores, s)
                      : csa::launch_index_scores_simt(*g, dtype, qI, w, KI, ldK, nseq, seq_of_q,
                                                      pos, n_entries, Q, H_I, c_I, scores,
                                                      ld_scores, s);
  return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

size_t csa_attend_workspace_size(int Q, int H_q, int c, int k, int n_win) {
  (void)Q, (void)H_q, (void)c, (void)k, (void)n_win;
  return 0;
}

static csa_status attend_common(const csa_geom* g, csa_dtype q_dtype, csa_dtype kv_dtype,
                                const void* q, const float* q_gain, const float* sink,
                                const void* E, int64_t ldE, int nseq, const int64_t* n_entries,
                                const int32_t* idx, int k, int dense, const void* win,
                                int64_t ldW, const int32_t* seq_of_q, const int64_t* pos, int Q,
                                int H_q, void* O, void* workspace, size_t ws_bytes,
                                csa_stream_t stream) {
  if (!geom_ok(g) || !io_dtype_ok(q_dtype)) return CSA_ERR_INVALID_ARG;
  if (!(io_dtype_ok(kv_dtype) || (kv_dtype == CSA_FP8_MIXED && mixed_ok(g)))) return CSA_ERR_INVALID_ARG;
  if (Q < 0 || H_q < 1 || ldE < 0 || ldW < 0 || nseq < 0) return CSA_ERR_INVALID_ARG;
  if (!dense && (k < 0 || k > CSA_MAX_TOPK)) return CSA_ERR_INVALID_ARG;
  if (Q == 0) return CSA_OK;
  if (!q || !sink || !seq_of_q || !pos || !O || !n_entries) return CSA_ERR_INVALID_ARG;
  if (!dense && k > 0 && !idx) return CSA_ERR_INVALID_ARG;
  if (g->n_win > 0 && !win) return CSA_ERR_INVALID_ARG;
  if (g->win_ring && ldW < g->n_win) return CSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, q_gain, sink, E, n_entries, idx, win, seq_of_q, pos, O};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return CSA_ERR_INVALID_ARG;
  (void)workspace, (void)ws_bytes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int kk = dense ? 0 : k;
  // small batches: one cluster per query (batch-invariant); large batches:
  // one CTA per query
  const bool tc_big = csa::attend_tc_supported(q_dtype, kv_dtype, g->c, H_q, kk, g->rope_dims);
  if (csa::attend_cluster_supported(q_dtype, kv_dtype, g->c, H_q, kk, g->rope_dims) &&
      (Q < CSA_ATTEND_INVARIANT_Q || !tc_big))
    return cuda_status(csa::launch_attend_cluster(*g, kv_dtype, q, q_gain, sink, E, ldE, nseq,
                                                  n_entries, idx, kk, dense, win, ldW, seq_of_q,
                                                  pos, Q, O, s));
  if (tc_big)
    return cuda_status(csa::launch_attend_tc(*g, kv_dtype, q, q_gain, sink, E, ldE, nseq, n_entries,
                                             idx, kk, dense, win, ldW, seq_of_q, pos, Q, O, s));
  if (!csa::attend_simt_supported(g->c, H_q)) return CSA_ERR_UNSUPPORTED;
  return cuda_status(launch_attend_simt(*g, q_dtype, kv_dtype, q, q_gain, sink, E, ldE, nseq,
                                        n_entries, idx, k, dense, win, ldW, seq_of_q, pos, Q, H_q, O,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_attend(const csa_geom* g, csa_dtype q_dtype, csa_dtype kv_dtype, const void* q,
                      const float* q_gain, const float* sink, const void* E, int64_t ldE,
                      int nseq, const int64_t* n_entries, const int32_t* idx, int k,
                      const void* win, int64_t ldW, const int32_t* seq_of_q, const int64_t* pos,
                      int Q, int H_q, void* O, void* workspace, size_t ws_bytes,
                      csa_stream_t stream) {
  return attend_common(g, q_dtype, kv_dtype, q, q_gain, sink, E, ldE, nseq, n_entries, idx, k, 0,
                       win, ldW, seq_of_q, pos, Q, H_q, O, workspace, ws_bytes, stream);
}

size_t hca_attend_workspace_size(int Q, int H_q, int c, int64_t ldE, int n_win) {
  (void)Q, (void)H_q, (void)c, (void)ldE, (void)n_win;
  return 0;
}

csa_status hca_attend(const csa_geom* g, csa_dtype q_dtype, csa_dtype kv_dtype, const void* q,
                      const float* q_gain, const float* sink, const void* E, int64_t ldE,
                      int nseq, const int64_t* n_entries, const void* win, int64_t ldW,
                      const int32_t* seq_of_q, const int64_t* pos, int Q, int H_q, void* O,
                      void* workspace, size_t ws_bytes, csa_stream_t stream) {
  return attend_common(g, q_dtype, kv_dtype, q, q_gain, sink, E, ldE, nseq, n_entries, nullptr, 0,
                       1, win, ldW, seq_of_q, pos, Q, H_q, O, workspace, ws_bytes, stream);
}

}  // extern "C"
