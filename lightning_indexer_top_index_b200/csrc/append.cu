// The cache write side: new compressed rows (or sliding-window rows) are
// quantised into the storage format and appended (DeepSeek-V4-Flash
// architecture post, "why quantising the KV does not save memory", point 1:
// non-RoPE dims as E4M3 with one power-of-two scale per 64 elements, the 64
// RoPE dims as bf16).
//
// One row per group of dim/8 threads; thread t of the group owns the eight
// values [8t, 8t+8).  For an E4M3 cache the eight threads of a 64-element
// block find its largest finite magnitude with three shuffles, pick the
// finest power-of-two scale 2^e with amax <= 448 * 2^e (e in [-127, 127];
// e = 0 for an all-zero block), and convert x * 2^-e with the hardware
// E4M3 conversion (round to nearest even) after clamping to +-448 (so values
// above 448, infinities included, saturate) and mapping NaN to 0x7F.  The
// RoPE dims and bf16 caches round to nearest even.
#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// E4M3 code of v already divided by its block scale: NaN -> 0x7F, |v| > 448
// saturates, else the nearest code (ties to even).
__device__ __forceinline__ float e4m3_prep(float v) {
  return fabsf(v) > 448.f ? copysignf(448.f, v) : v;  // NaN compares false and stays NaN
}

__device__ __forceinline__ uint32_t pack4_e4m3(const float *v) {
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; i++) c[i] = is_nan_bits(v[i]) ? 0x7Fu : 0u;
  const uint32_t lo = e4m3x2(e4m3_prep(v[1]), e4m3_prep(v[0]));
  const uint32_t hi = e4m3x2(e4m3_prep(v[3]), e4m3_prep(v[2]));
  uint32_t r = lo | (hi << 16);
#pragma unroll
  for (int i = 0; i < 4; i++)
    if (c[i]) r = (r & ~(0xFFu << (8 * i))) | (0x7Fu << (8 * i));
  return r;
}

// bf16 bits of x, nearest even; NaN keeps its payload's top bits, quieted
__device__ __forceinline__ uint32_t bf16_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  if (is_nan_bits(x)) return (u >> 16) | 0x40u;
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint4 pack8_bf16(const float *v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; i++) w[i] = bf16_bits(v[2 * i]) | (bf16_bits(v[2 * i + 1]) << 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// smallest e in [-127, 127] with amax <= 448 * 2^e (amax finite, > 0)
__device__ __forceinline__ int block_exponent(float amax) {
  int ex;
  frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
  int e = max(-127, min(127, ex - 9));
  while (e < 127 && amax > ldexpf(448.f, e)) e++;
  while (e > -127 && amax <= ldexpf(448.f, e - 1)) e--;
  return e;
}

__global__ void __launch_bounds__(kThreads) append_kernel(const lidx_append_args a, uint32_t *status) {
  const int dim = a.cache.dim;
  const int tpr = dim / 8;  // threads per row
  const int grp = threadIdx.x / tpr, t = threadIdx.x % tpr;
  const int64_t row_id = static_cast<int64_t>(blockIdx.x) * (kThreads / tpr) + grp;  // (b, r) pair
  pdl_trigger();
  pdl_wait();  // the new rows and positions may come from the previous kernel
  const bool active = row_id < static_cast<int64_t>(a.B) * a.R;
  const int b = active ? static_cast<int>(row_id / a.R) : 0, r = active ? static_cast<int>(row_id % a.R) : 0;
  float v[8];
  if (active) {
    const float4 *src = reinterpret_cast<const float4 *>(a.x + row_id * dim + 8 * t);
    const float4 p0 = __ldg(src), p1 = __ldg(src + 1);
    v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
    v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = 0.f;
  }
  bool nonfinite = false;
#pragma unroll
  for (int i = 0; i < 8; i++) nonfinite |= !isfinite(v[i]);
  // the destination row
  int64_t dst = -1;
  if (active) {
    const int64_t p = static_cast<int64_t>(__ldg(a.pos + b)) + r;
    const int64_t idx = a.ring > 0 ? (p >= 0 ? p % a.ring : -1) : p;
    if (idx >= 0 && idx < a.capacity) dst = static_cast<int64_t>(b) * a.cache.batch_rows + idx;
    else if (t == 0) raise_status(status, LIDX_DEV_BOUNDS);
  }
  if (active && nonfinite) raise_status(status, LIDX_DEV_NAN);
  const int d0 = 8 * t;
  // largest finite magnitude over each 64-element block: eight threads, whose
  // lanes are aligned groups of eight (dim/8 is a multiple of 8); every lane
  // takes part in the shuffles, whatever its row or dims
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const float x = fabsf(v[i]);
    am = isfinite(x) ? fmaxf(am, x) : am;
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
  if (a.cache.dtype == LIDX_E4M3 && d0 < dim - 64) {
    const int e = am > 0.f ? block_exponent(am) : 0;
    const float inv = ldexpf(1.f, -e);  // exact power of two (e <= 120 for finite fp32 amax)
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; i++) s[i] = v[i] * inv;
    if (dst >= 0) {
      uint8_t *codes = static_cast<uint8_t *>(const_cast<void *>(a.cache.data)) + dst * a.cache.ld + d0;
      *reinterpret_cast<uint2 *>(codes) = make_uint2(pack4_e4m3(s), pack4_e4m3(s + 4));
      if ((t & 7) == 0)
        const_cast<uint8_t *>(a.cache.scale)[dst * a.cache.ld_scale + d0 / 64] = static_cast<uint8_t>(e + 127);
    }
  } else if (a.cache.dtype == LIDX_E4M3) {
    if (dst >= 0) {
      uint16_t *rope = static_cast<uint16_t *>(const_cast<void *>(a.cache.rope)) + dst * a.cache.ld_rope + (d0 - (dim - 64));
      *reinterpret_cast<uint4 *>(rope) = pack8_bf16(v);
    }
  } else if (a.cache.dtype == LIDX_BF16) {
    if (dst >= 0) {
      uint16_t *p = static_cast<uint16_t *>(const_cast<void *>(a.cache.data)) + dst * a.cache.ld + d0;
      *reinterpret_cast<uint4 *>(p) = pack8_bf16(v);
    }
  } else {
    if (dst >= 0) {
      float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(const_cast<void *>(a.cache.data)) + dst * a.cache.ld + d0);
      p[0] = make_float4(v[0], v[1], v[2], v[3]);
      p[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

}  // namespace

cudaError_t launch_append(const lidx_append_args &a, void *ws, cudaStream_t st) {
  const int tpr = a.cache.dim / 8;
  const int per_block = kThreads / tpr;
  const int64_t rows = static_cast<int64_t>(a.B) * a.R;
  const int grid = static_cast<int>((rows + per_block - 1) / per_block);
  return launch_kernel(append_kernel, dim3(grid), dim3(kThreads), 0, st, (a.flags & LIDX_LAUNCH_PDL) != 0, a,
                       static_cast<uint32_t *>(ws));
}

}  // namespace lidx
