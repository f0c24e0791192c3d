// Lightning-indexer scores on CUDA cores (fp32 FMA), any head count.
//
//   s[b,t,j] = sum_h w[b,t,h] * max(q[b,t,h,:] . k[b,j,:], 0)
//
// (DeepSeek-V4-Flash architecture post, section (B): the indexer scores
// every compressed entry with its 128-d index key; head-weighted ReLU-MQA
// form of the FlashMemory deep-dive write-up, reply #2.)
//
// One thread owns one key row and accumulates all heads of a head group in
// registers; the query block of (b,t) sits in shared memory and every warp
// reads it by broadcast.  This kernel serves fp32 keys (tiny configuration)
// and any shape the tensor-core scorer does not take.
#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 128;
constexpr int kD = 128;

// Load 8 consecutive logical dims [d0, d0+8) of key row `row` as fp32.
template <int KT>
__device__ __forceinline__ void load8(const lidx_kv &k, int64_t row, int d0, float *v) {
  if constexpr (KT == LIDX_F32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(k.data) + row * k.ld + d0);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if constexpr (KT == LIDX_BF16) {
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(k.data) + row * k.ld + d0));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    if (d0 < kD - 64) {
      uint2 a = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(k.data) + row * k.ld + d0));
      float sc = e8m0_to_f32(__ldg(k.scale + row * k.ld_scale + d0 / 64));
      const uint32_t w[2] = {a.x, a.y};
#pragma unroll
      for (int i = 0; i < 8; i++) v[i] = e4m3_to_f32((w[i / 4] >> (8 * (i % 4))) & 0xFFu) * sc;
    } else {
      uint4 a = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(k.rope) + row * k.ld_rope +
                                                       (d0 - (kD - 64))));
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  }
}

template <int KT, int HG>
__global__ void __launch_bounds__(kThreads) score_cc_kernel(lidx_score_args a, int Hp) {
  extern __shared__ float4 smem4[];
  float *q_s = reinterpret_cast<float *>(smem4);  // [Hp][128], zero-padded heads
  float *w_s = q_s + Hp * kD;                      // [Hp]
  const int bt = blockIdx.y;
  const int b = bt / a.Q;
  const size_t qoff = static_cast<size_t>(bt) * a.H * kD;
  for (int i = threadIdx.x; i < Hp * kD; i += kThreads) {
    float v = 0.f;
    if (i < a.H * kD)
      v = a.q_dtype == LIDX_F32 ? static_cast<const float *>(a.q)[qoff + i]
                                : bf16_to_f32(static_cast<const uint16_t *>(a.q)[qoff + i]);
    q_s[i] = v;
  }
  for (int i = threadIdx.x; i < Hp; i += kThreads) w_s[i] = i < a.H ? a.w[static_cast<size_t>(bt) * a.H + i] : 0.f;
  __syncthreads();
  const int j = blockIdx.x * kThreads + threadIdx.x;
  const bool valid = j < a.N;
  float score = 0.f;
  if (valid) {
    const int64_t row = static_cast<int64_t>(b) * a.keys.batch_rows + j;
    for (int h0 = 0; h0 < Hp; h0 += HG) {
      float acc[HG];
#pragma unroll
      for (int i = 0; i < HG; i++) acc[i] = 0.f;
#pragma unroll 1
      for (int d0 = 0; d0 < kD; d0 += 8) {
        float kv[8];
        load8<KT>(a.keys, row, d0, kv);
#pragma unroll
        for (int hh = 0; hh < HG; hh++) {
          const float4 *qp = reinterpret_cast<const float4 *>(q_s + (h0 + hh) * kD + d0);
          float4 x = qp[0], y = qp[1];
          float s = acc[hh];
          s = fmaf(x.x, kv[0], s); s = fmaf(x.y, kv[1], s); s = fmaf(x.z, kv[2], s); s = fmaf(x.w, kv[3], s);
          s = fmaf(y.x, kv[4], s); s = fmaf(y.y, kv[5], s); s = fmaf(y.z, kv[6], s); s = fmaf(y.w, kv[7], s);
          acc[hh] = s;
        }
      }
#pragma unroll
      for (int hh = 0; hh < HG; hh++) score = fmaf(w_s[h0 + hh], fmaxf(acc[hh], 0.f), score);
    }
    if (a.n_visible && j >= __ldg(a.n_visible + bt)) score = -INFINITY;  // causal entry mask
    a.scores[static_cast<size_t>(bt) * a.ld_scores + j] = score;
  }
  if (a.tile_stats) {  // score bounds of this warp's span of 32 entries (whole warps)
    const uint32_t kk = valid ? order_key(score) : 0u;
    const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, kk);
    const uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, kk ? kk : 0xFFFFFFFFu);
    const int j0 = j & ~31;
    const int n_spans = (a.N + LIDX_STATS_SPAN - 1) / LIDX_STATS_SPAN;
    if ((threadIdx.x & 31) == 0 && j0 < a.N)
      reinterpret_cast<uint2 *>(a.tile_stats)[static_cast<size_t>(bt) * n_spans + j0 / 32] = make_uint2(mx, mn);
  }
}

template <int KT>
cudaError_t launch_kt(const lidx_score_args &a, cudaStream_t st) {
  const int HG = a.H <= 16 ? 16 : 32;
  const int Hp = (a.H + HG - 1) / HG * HG;
  const size_t smem = (static_cast<size_t>(Hp) * kD + Hp) * sizeof(float);
  dim3 grid((a.N + kThreads - 1) / kThreads, a.B * a.Q);
  if (HG == 16) {
    auto k = score_cc_kernel<KT, 16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<grid, kThreads, smem, st>>>(a, Hp);
  } else {
    auto k = score_cc_kernel<KT, 32>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<grid, kThreads, smem, st>>>(a, Hp);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_cc(const lidx_score_args &a, cudaStream_t st) {
  switch (a.keys.dtype) {
    case LIDX_F32: return launch_kt<LIDX_F32>(a, st);
    case LIDX_BF16: return launch_kt<LIDX_BF16>(a, st);
    default: return launch_kt<LIDX_E4M3>(a, st);
  }
}

}  // namespace lidx
