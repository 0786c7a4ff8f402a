// fd_common.cuh — types and small device helpers shared by every kernel of
// the FlashDecoder streaming step.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flashdec.h"

namespace fd {

typedef __nv_bfloat16 bf16;

// Longest head the kernels support (RoPE tables are sized from it).
constexpr int kMaxHeadDim = 64;
constexpr int kMaxTemporalPairs = kMaxHeadDim / 8;   // D_h/4 dims -> D_h/8 pairs
constexpr int kMaxStreams = 64;                      // video streams per handle

// Per-frame state, written once per frame by the step_begin kernel from the
// device frame counter and read by every later kernel of the frame.
struct FrameState {
  long long t;          // absolute index of the frame being decoded
  int slot;             // ring slot that receives this frame: t mod (ring slots)
  int n_valid;          // frames attended to: min(t, window - 1) + 1
  int win;              // first ring row (in frames) of the attended keys: 0, or
                        // for a mirrored ring (slot - n_valid + 1) mod slots
  float2 rope_t[kMaxTemporalPairs];  // (cos, sin) of t * theta^(-2m/d_t), m < d_t/2
};

// ---------------------------------------------------------------- storage
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Store n (multiple of 8) consecutive floats as T with 16-byte vector stores.
template <typename T, int n>
__device__ __forceinline__ void store_row(T* dst, const float* v);

template <>
__device__ __forceinline__ void store_row<float, 8>(float* dst, const float* v) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store_row<bf16, 8>(bf16* dst, const float* v) {
  __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 p3 = __floats2bfloat162_rn(v[6], v[7]);
  uint4 u;
  u.x = *reinterpret_cast<uint32_t*>(&p0);
  u.y = *reinterpret_cast<uint32_t*>(&p1);
  u.z = *reinterpret_cast<uint32_t*>(&p2);
  u.w = *reinterpret_cast<uint32_t*>(&p3);
  *reinterpret_cast<uint4*>(dst) = u;
}

// Four consecutive values as T (one 16-byte or 8-byte store).
template <typename T> __device__ __forceinline__ void store_quad(T* dst, const float* v);
template <>
__device__ __forceinline__ void store_quad<float>(float* dst, const float* v) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store_quad<bf16>(bf16* dst, const float* v) {
  __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&p0);
  u.y = *reinterpret_cast<uint32_t*>(&p1);
  *reinterpret_cast<uint2*>(dst) = u;
}

template <typename T, int n>
__device__ __forceinline__ void store_vec(T* dst, const float* v) {
#pragma unroll
  for (int i = 0; i < n; i += 8) store_row<T, 8>(dst + i, v + i);
}

// Device status word: first failure wins.
__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Bounds checks of the bounds-checked build (-DFD_DEBUG, libflashdec_debug.so):
// every computed ring row, slot, V^T column, split-partial index and pixel
// offset is tested before the access; a failed test records FD_ERR_BOUNDS in
// the device status word and the access is skipped (no trap, the kernel runs
// on). In the normal build FD_IN_BOUNDS is the constant true and costs nothing.
__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
  if (!ok) report_status(status, FD_ERR_BOUNDS);
  return ok;
}
#ifdef FD_DEBUG
#define FD_IN_BOUNDS(cond, status) (::fd::in_bounds((cond), (status)))
#else
#define FD_IN_BOUNDS(cond, status) true
#endif

}  // namespace fd
