// common.cuh - device helpers shared by the libcsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// ---------------------------------------------------------------- errors
// Programmatic dependent launch: a kernel launched with launch_pdl()
// (internal.h) is scheduled as soon as the previous kernel's blocks have all
// exited, and runs its setup while that kernel's writes drain. pdl_wait()
// returns once that kernel has completed and its writes are visible (a no-op
// for ordinary launches). No kernel signals its successor early: measured on
// the decode step, successors that were scheduled while a persistent kernel
// still ran slowed it down.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bounded device-side waits that give up record a status code in the
// library's device error word (defined in api.cu, passed to kernels as a
// pointer); csa_sync_status() reads and clears it.
__device__ __forceinline__ void record_device_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- dtype helpers
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// BF16 pairs packed in 32-bit words (low half = first element), handled in
// registers: taking the address of a local array to reinterpret it would put
// the array in local memory.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint8_t byte_of(uint32_t u, int i) { return (uint8_t)(u >> (8 * i)); }

// E4M3 code -> float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __nv_fp8_e4m3 v;
  v.__x = code;
  return float(v);
}

// float -> E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// Mixed compressed-entry row: 448 E4M3 codes, 64 BF16, FP32 scale.
constexpr int kMixedRowBytes = CSA_MIXED_ROW_BYTES;
constexpr int kMixedFp8Dims = 448;
constexpr int kMixedScaleOffset = 576;

// Value i of a row stored as dtype `dt`. `row` points at the row start.
__device__ __forceinline__ float load_elem(const void* row, int i, int dt) {
  if (dt == CSA_F32) return reinterpret_cast<const float*>(row)[i];
  if (dt == CSA_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(row)[i]);
  const uint8_t* b = reinterpret_cast<const uint8_t*>(row);
  if (i < kMixedFp8Dims) {
    float s = *reinterpret_cast<const float*>(b + kMixedScaleOffset);
    return e4m3_to_f32(b[i]) * s;
  }
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(b + kMixedFp8Dims)[i - kMixedFp8Dims]);
}

__host__ __device__ __forceinline__ int64_t row_bytes(int dt, int c) {
  return dt == CSA_F32 ? 4LL * c : (dt == CSA_BF16 ? 2LL * c : (int64_t)kMixedRowBytes);
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------- visibility
// Compressed entries visible at position p: floor((p + vis_offset)/m),
// clipped to [0, n_entries].
__device__ __forceinline__ int64_t n_visible(int64_t p, int m, int vis_offset, int64_t n_entries) {
  int64_t t = p + vis_offset;
  int64_t v = t < 0 ? 0 : t / m;
  return v > n_entries ? n_entries : v;
}

// ---------------------------------------------------------------- RoPE angle
// cos/sin of pos * base^(-2i/r), evaluated in FP64 so that positions up to
// 2^20 and beyond keep full FP32 accuracy of the rotation.
__device__ __forceinline__ void rope_cs(int64_t pos, int i, int r, double base, float* cs,
                                        float* sn) {
  const double theta = exp(-2.0 * (double)i / (double)r * log(base));
  // angle / pi in FP64 (absolute error ~1e-10 for angles up to 2^20);
  // sincospi reduces its argument modulo 2 exactly, so large positions cost
  // no long argument reduction
  const double x = (double)pos * theta * (1.0 / 3.141592653589793238462643383279502884);
  double s, c;
  sincospi(x, &s, &c);
  *cs = (float)c;
  *sn = (float)s;
}

}  // namespace csa
