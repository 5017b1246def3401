// internal.h - launchers shared between the C-ABI layer and the kernels.
// Host-side declarations only; arguments are validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// Device address of the library error word on the current device.
int* device_error_ptr();

// Counts one kernel launch (csa_kernel_launches()).
void count_launches(int n = 1);

// Launch with programmatic dependent launch allowed: the kernel may be
// scheduled while the previous kernel of the stream finishes. Every kernel
// launched this way calls pdl_wait() (common.cuh) before its first access to
// global memory, so it still observes everything that kernel wrote and
// writes nothing that kernel still reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- SIMT kernels (simt.cu): every dtype, every shape the ABI accepts ----
cudaError_t launch_rmsnorm_rope(const csa_geom& g, int in_dt, int out_dt, const void* x,
                                int64_t rows, const int64_t* pos, int64_t pos0, int64_t pos_step,
                                const float* gain, void* out, const int64_t* out_row,
                                cudaStream_t s);
cudaError_t launch_quantize_mixed(int in_dt, const void* x, int64_t rows, void* out,
                                  cudaStream_t s);
// P[T, nW*c] (FP32) = H[T,d] @ [W_0 | ... | W_{nW-1}], each W_i [d, c].
cudaError_t launch_proj_simt(int dt, const void* H, int64_t T, int d, int c, int nW,
                             const void* const* W, float* P, cudaStream_t s);
// Pool + RMSNorm + RoPE of every complete block from projections P.
cudaError_t launch_pool_prefill(const csa_geom& g, const float* P, int64_t T, const float* bias,
                                const float* gain, int out_dt, void* E, cudaStream_t s);
cudaError_t launch_decode_proj(const csa_geom& g, int dt, const void* h, const int64_t* pos,
                               int B, int d, const void* const* W, int nW, float* state,
                               cudaStream_t s);
cudaError_t launch_decode_pool(const csa_geom& g, const int64_t* pos, int B, const float* bias,
                               const float* gain, const float* state, int out_dt, void* E,
                               int64_t ldE, cudaStream_t s);
cudaError_t launch_index_scores_simt(const csa_geom& g, int dt, const void* qI, const float* w,
                                     const void* KI, int64_t ldK, int nseq,
                                     const int32_t* seq_of_q,
                                     const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                                     int c_I, float* scores, int64_t ld_scores, cudaStream_t s);
// Exact top-k of per-query scores [Q, ld_scores] (topk.cu).
bool topk_supported(int64_t ld_scores, int k);
size_t topk_workspace(int Q, int64_t ld_scores, int k);
cudaError_t launch_topk(const csa_geom& g, const float* scores, int64_t ld_scores, int nseq,
                        const int32_t* seq_of_q, const int64_t* pos, const int64_t* n_entries,
                        int Q, int k, int32_t* idx_out, float* scores_dbg, int64_t ld_dbg,
                        void* cand_ws, cudaStream_t s);
// ---- tensor-core kernels (tc_*.cu) ----
bool index_tc_supported(int dt, int H_I, int c_I);
cudaError_t launch_index_scores_tc(const csa_geom& g, const void* qI, const float* w,
                                   const void* KI, int64_t ldK, int nseq,
                                   const int32_t* seq_of_q, const int64_t* pos,
                                   const int64_t* n_entries, int Q, int H_I, int c_I,
                                   float* scores, int64_t ld_scores, cudaStream_t s);
bool proj_tc_supported(const csa_geom& g, int dt, int d);
bool proj_decode_supported(const csa_geom& g, int dt, int d);
size_t proj_pool_workspace(const csa_geom& g, int64_t T);
size_t proj_decode_workspace(const csa_geom& g, int B, int d);
// pooled [T/m, c] FP32 (before RMSNorm/RoPE) of a prefill sequence
cudaError_t launch_compress_tc(const csa_geom& g, const void* H, int64_t T, int d,
                               const void* const* W, const float* bias, float* pooled,
                               cudaStream_t s);
// projections of one new token per sequence into the decode state
cudaError_t launch_decode_proj_tc(const csa_geom& g, const void* h, const int64_t* pos, int B,
                                  int d, const void* const* W, float* part, float* state,
                                  cudaStream_t s);
// Shared-KV attention, one thread-block cluster per query (tc_attend_cluster.cu).
int attend_cluster_size(int64_t max_slots);
bool attend_cluster_supported(int q_dt, int kv_dt, int c, int H_q, int k, int rope_dims);
cudaError_t launch_attend_cluster(const csa_geom& g, int kv_dt, const void* q, const float* q_gain,
                                  const float* sink, const void* E, int64_t ldE, int nseq,
                                  const int64_t* n_entries, const int32_t* idx, int k, int dense,
                                  const void* win, int64_t ldW, const int32_t* seq_of_q,
                                  const int64_t* pos, int Q, void* O, cudaStream_t s);
bool attend_tc_supported(int q_dt, int kv_dt, int c, int H_q, int k, int rope_dims);
cudaError_t launch_attend_tc(const csa_geom& g, int kv_dt, const void* q, const float* q_gain,
                             const float* sink, const void* E, int64_t ldE, int nseq,
                             const int64_t* n_entries, const int32_t* idx, int k, int dense,
                             const void* win, int64_t ldW, const int32_t* seq_of_q,
                             const int64_t* pos, int Q, void* O, cudaStream_t s);
// dense != 0: HCA (all visible entries); else CSA with idx [Q, k].
cudaError_t launch_attend_simt(const csa_geom& g, int q_dt, int kv_dt, const void* q,
                               const float* q_gain, const float* sink, const void* E,
                               int64_t ldE, int nseq, const int64_t* n_entries,
                               const int32_t* idx, int k,
                               int dense, const void* win, int64_t ldW, const int32_t* seq_of_q,
                               const int64_t* pos, int Q, int H_q, void* O, cudaStream_t s);
bool attend_simt_supported(int c, int H_q);

}  // namespace csa
