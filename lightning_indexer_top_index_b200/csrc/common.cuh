// Device helpers shared by the lidx kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "../../include/lidx.h"

#define LIDX_WS_HEADER 256  // bytes at the start of every workspace: status word + counters

namespace lidx {

// ----------------------------------------------------------------------------
// Storage decoding.
// ----------------------------------------------------------------------------

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// OCP E4M3FN byte -> bf16 bits, exact (every E4M3 value is a bf16 value).
// Normal codes move the 4-bit exponent (bias 7) into the 8-bit field (bias
// 127) and the 3 mantissa bits to the top of the 7-bit field; subnormal codes
// m * 2^-9 are normalised; S.1111.111 (NaN) becomes a bf16 NaN.
__device__ __forceinline__ uint16_t e4m3_to_bf16_bits(uint32_t c) {
  uint32_t s = (c & 0x80u) << 8;
  uint32_t e = (c >> 3) & 0xFu;
  uint32_t m = c & 0x7u;
  if (e == 0xFu && m == 0x7u) return static_cast<uint16_t>(s | 0x7FC0u);
  if (e != 0) return static_cast<uint16_t>(s | ((e + 120u) << 7) | (m << 4));
  if (m == 0) return static_cast<uint16_t>(s);
  // subnormal: value m * 2^-9; leading one of m at bit p (0..2)
  uint32_t p = 31u - __clz(m);
  uint32_t frac = (m << (3u - p)) & 0x7u;  // bits below the leading one, left-aligned to 3 bits
  uint32_t ex = 127u - 9u + p;             // biased exponent of 2^(p-9)
  return static_cast<uint16_t>(s | (ex << 7) | (frac << 4));
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t c) { return bf16_to_f32(e4m3_to_bf16_bits(c)); }

// Two E4M3 codes (bits 0-7 and 8-15 of `codes`) -> two bf16 (low and high
// half of the result), each multiplied by `scale`, a power of two.  Every
// step is exact: the hardware E4M3 -> f16 conversion (all E4M3 values are f16
// normals or zero), f16 -> f32, the power-of-two product while it stays in
// the f32 normal range, and the final rounding to bf16 of a value with at
// most four significant bits.  NaN codes stay NaN.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t codes, float scale = 1.f) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(codes & 0xFFFFu)));
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  lo *= scale;
  hi *= scale;
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// E8M0 scale byte -> 2^(c-127) as float (c = 0 gives 2^-127, a subnormal;
// 255 is NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t c) {
  if (c == 0xFFu) return __uint_as_float(0x7FC00000u);
  if (c == 0) return __uint_as_float(0x00400000u);
  return __uint_as_float(c << 23);
}

// ----------------------------------------------------------------------------
// Order-preserving 32-bit key of a score: larger float -> larger key.  -0 is
// folded onto +0 so that equal values compare equal; NaN and excluded entries
// map to 0, which no number reaches (-inf maps to 0x007FFFFF).
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0u;  // NaN
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ bool is_nan_bits(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu);
}

// ----------------------------------------------------------------------------
// Warp / block helpers.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Inclusive prefix sum within a warp.
template <typename T>
__device__ __forceinline__ T warp_inclusive_scan(T v) {
  uint32_t lane = lane_id();
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= static_cast<uint32_t>(o)) v += n;
  }
  return v;
}

// ----------------------------------------------------------------------------
// Programmatic dependent launch.  pdl_trigger lets the next kernel on the
// stream start its prologue; pdl_wait blocks until the previous kernel has
// completed and its writes are visible.  Both are no-ops for a kernel that
// was not launched as a programmatic dependent.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kern` on `st`, as a programmatic dependent of the previous kernel
// when `pdl` is set.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                          Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Device status word at the start of a workspace.
__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t flag) {
  if (status) atomicOr(status, flag);
}

}  // namespace lidx
