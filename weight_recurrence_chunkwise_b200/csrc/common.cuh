// common.cuh -- shared definitions of the CUDA side of the delta-rule library.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace dr {

enum : int { MODE_ABSENT = 0, MODE_SCALAR = 1, MODE_CHANNEL = 2 };

// Bits of the device status word kept in the caller's workspace.
enum : uint32_t { STATUS_RANGE = 1u, STATUS_TIMEOUT = 2u };

// Smallest cumulative decay exp(sum log alpha) over one chunk that the
// factorised WY/UT form accepts: its reciprocal must stay finite in fp32/bf16
// with head-room for the key and strength factors.
constexpr float kMinChunkDecay = 1e-30f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Per-token gate value: mode ABSENT -> 1, SCALAR -> g[th], CHANNEL -> g[th*width + i].
__device__ __forceinline__ float gate_at(const float *g, int mode, size_t th, int width, int i) {
  if (mode == MODE_ABSENT) return 1.0f;
  if (mode == MODE_SCALAR) return __ldg(g + th);
  return __ldg(g + th * static_cast<size_t>(width) + i);
}

__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace dr
