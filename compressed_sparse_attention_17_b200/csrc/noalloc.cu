// noalloc.cu - csa_index_topk for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) around a
// call: code running inside a memory pool or arena that forbids outside
// allocations, and runtimes that must not allocate on their serving path.
// This entry point takes the scratch that csa_index_topk needs (the FP32
// scores and the top-k chunk candidates) from one fixed buffer compiled
// into the library instead of from a caller-provided workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/csa.h"

namespace {

// The shared scratch: every GPU that loads the library holds it until the
// process exits.
constexpr size_t kScratchBytes = CSA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void* g_ptr[kMaxDevices];
cudaError_t g_rc[kMaxDevices];

// Device address of the scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_once[dev], [dev] {
    void* p = nullptr;
    g_rc[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_ptr[dev] = g_rc[dev] == cudaSuccess ? p : nullptr;
  });
  return g_ptr[dev];
}

}  // namespace

extern "C" csa_status csa_index_topk_noalloc(const csa_geom* g, csa_dtype dtype, const void* qI,
                                             const float* w, const void* KI, int64_t ldK, int nseq,
                                             const int32_t* seq_of_q, const int64_t* pos,
                                             const int64_t* n_entries, int Q, int H_I, int c_I,
                                             int k, int32_t* idx_out, float* scores_dbg,
                                             csa_stream_t stream) {
  if (Q < 0 || ldK < 0 || k < 1) return CSA_ERR_INVALID_ARG;
  if (csa_index_topk_workspace_size(Q, ldK, k) > kScratchBytes) return CSA_ERR_TOO_LARGE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return CSA_ERR_CUDA;
  return csa_index_topk(g, dtype, qI, w, KI, ldK, nseq, seq_of_q, pos, n_entries, Q, H_I, c_I, k,
                        idx_out, scores_dbg, scratch, kScratchBytes, stream);
}
