// Sparse MQA decode attention over the selected compressed rows plus the
// sliding window (DeepSeek-V4-Flash architecture post, sections (A)-(B):
// attention reads the top-k attn_comp_kv rows, 512 wide, and a 128-token SWA
// window).  K = V = the full row.
//
// Split-K over rows: CTA (split, b) takes rows [split*RC, split*RC+RC) of the
// sequence's row list (selected ids first, then the window), writes an
// unnormalised partial (m, l, O) in base-2 units, and a merge kernel combines
// the partials with the usual log-sum-exp rescaling.
//
// This is the CUDA-core path (fp32 FMA, rows dequantised to fp32 in shared
// memory); it serves fp32 rows and any head count up to 64.
#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kD = 512;
constexpr int kRC = 32;          // rows per CTA
constexpr int kThreads = 256;
constexpr int kXs = kD + 4;      // padded row stride (floats): conflict-free float4 row reads
constexpr float kLog2e = 1.4426950408889634f;

// Load dims [d0, d0+8) of a 512-wide row as fp32.
template <int KT>
__device__ __forceinline__ void load_row8(const lidx_kv &k, int64_t row, int d0, float *v) {
  if constexpr (KT == LIDX_F32) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(k.data) + row * k.ld + d0);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint16_t *src = nullptr;
    if constexpr (KT == LIDX_BF16) {
      src = static_cast<const uint16_t *>(k.data) + row * k.ld + d0;
    } else {
      if (d0 < kD - 64) {
        uint2 a = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(k.data) + row * k.ld + d0));
        float sc = e8m0_to_f32(__ldg(k.scale + row * k.ld_scale + d0 / 64));
        const uint32_t w[2] = {a.x, a.y};
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = e4m3_to_f32((w[i / 4] >> (8 * (i % 4))) & 0xFFu) * sc;
        return;
      }
      src = static_cast<const uint16_t *>(k.rope) + row * k.ld_rope + (d0 - (kD - 64));
    }
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(src));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <int KT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_cc_kernel(lidx_attn_args a, float *part_o, float2 *part_ml, int n_split, uint32_t *status) {
  extern __shared__ float4 sm4[];
  const int H = a.H;
  float *q_s = reinterpret_cast<float *>(sm4);  // [H][512], pre-scaled by scale*log2(e)
  float *x_s = q_s + H * kD;                     // [RC][kXs]
  float *p_s = x_s + kRC * kXs;                  // [H][RC]
  __shared__ int64_t row_of[kRC];
  __shared__ int kind_of[kRC];                   // 0 none, 1 selected row, 2 window row

  const int split = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  int n_b = a.n_ids;
  if (a.n_sel) n_b = min(max(a.n_sel[b], 0), a.n_ids);
  const int total = n_b + a.swa_len;
  const int i0 = split * kRC;

  if (tid < kRC) {
    const int i = i0 + tid;
    int kind = 0;
    int64_t r = 0;
    if (i < n_b) {
      const int id = a.ids ? a.ids[static_cast<int64_t>(b) * a.ld_ids + i] : i;  // no ids: dense rows
      if (id >= 0 && id < a.N) {
        kind = 1;
        r = static_cast<int64_t>(b) * a.kv.batch_rows + id;
      } else if (id != -1) {
        raise_status(status, LIDX_DEV_BOUNDS);
      }
    } else if (i < total) {
      kind = 2;
      r = static_cast<int64_t>(b) * a.swa.batch_rows + (i - n_b);
    }
    kind_of[tid] = kind;
    row_of[tid] = r;
  }
  const float qscale = a.scale * kLog2e;
  const size_t qoff = static_cast<size_t>(b) * H * kD;
  for (int i = tid; i < H * kD; i += kThreads) {
    float v = a.q_dtype == LIDX_F32 ? static_cast<const float *>(a.q)[qoff + i]
                                    : bf16_to_f32(static_cast<const uint16_t *>(a.q)[qoff + i]);
    q_s[i] = v * qscale;
  }
  __syncthreads();
  // stage the rows (dequantised)
  for (int c = tid; c < kRC * (kD / 8); c += kThreads) {
    const int r = c / (kD / 8), d0 = (c % (kD / 8)) * 8;
    float v[8];
    if (kind_of[r] == 1)
      load_row8<KT>(a.kv, row_of[r], d0, v);
    else if (kind_of[r] == 2)
      load_row8<KT>(a.swa, row_of[r], d0, v);
    else
#pragma unroll
      for (int i = 0; i < 8; i++) v[i] = 0.f;
    float4 *dst = reinterpret_cast<float4 *>(x_s + r * kXs + d0);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();

  // logits: warp w takes heads w, w+8, ...; lane = row
  const int warp = tid >> 5, lane = tid & 31;
  const bool valid = kind_of[lane] != 0;
  for (int h0 = warp; h0 < H; h0 += 8 * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; i++) acc[i] = 0.f;
    const float4 *xr = reinterpret_cast<const float4 *>(x_s + lane * kXs);
#pragma unroll 2
    for (int d4 = 0; d4 < kD / 4; d4++) {
      const float4 x = xr[d4];
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int h = h0 + 8 * i;
        if (h < H) {
          const float4 q = reinterpret_cast<const float4 *>(q_s + h * kD)[d4];
          acc[i] = fmaf(q.x, x.x, fmaf(q.y, x.y, fmaf(q.z, x.z, fmaf(q.w, x.w, acc[i]))));
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int h = h0 + 8 * i;
      if (h < H) {
        const float lg = valid ? acc[i] : -INFINITY;
        const float m = warp_max(lg);
        const float p = valid ? exp2f(lg - m) : 0.f;
        const float l = warp_sum(p);
        p_s[h * kRC + lane] = p;
        if (lane == 0) part_ml[(static_cast<size_t>(b) * n_split + split) * H + h] = make_float2(m, l);
      }
    }
  }
  __syncthreads();

  // O[h][d] = sum_r p[h][r] x[r][d]; thread owns d = tid and tid + 256
  float *po = part_o + (static_cast<size_t>(b) * n_split + split) * H * kD;
  for (int h0 = 0; h0 < H; h0 += 16) {
    float acc0[16], acc1[16];
#pragma unroll
    for (int i = 0; i < 16; i++) acc0[i] = acc1[i] = 0.f;
#pragma unroll 4
    for (int r = 0; r < kRC; r++) {
      const float x0 = x_s[r * kXs + tid], x1 = x_s[r * kXs + tid + 256];
#pragma unroll
      for (int i = 0; i < 16; i++) {
        if (h0 + i < H) {
          const float p = p_s[(h0 + i) * kRC + r];
          acc0[i] = fmaf(p, x0, acc0[i]);
          acc1[i] = fmaf(p, x1, acc1[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      if (h0 + i < H) {
        po[(h0 + i) * kD + tid] = acc0[i];
        po[(h0 + i) * kD + tid + 256] = acc1[i];
      }
    }
  }
}

// Combine the split partials of one (b, h): base-2 log-sum-exp rescaling.
// Thread t owns dims [4t, 4t+4).  Each batch of up to 16 splits issues its
// partial-O loads and its (m, l) loads together, then folds them in with a
// running maximum, so a merge of <= 16 splits costs one memory round trip.
__global__ void __launch_bounds__(128) attn_merge_kernel(lidx_attn_args a, const float *part_o,
                                                          const float2 *part_ml, int n_split) {
  pdl_trigger();
  pdl_wait();  // the partials come from the previous kernel
  const int h = blockIdx.x, b = blockIdx.y, H = a.H;
  const float2 *ml = part_ml + static_cast<size_t>(b) * n_split * H + h;
  const float4 *po = reinterpret_cast<const float4 *>(part_o + (static_cast<size_t>(b) * n_split * H + h) * kD) + threadIdx.x;
  const size_t stride4 = static_cast<size_t>(H) * kD / 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -INFINITY, L = 0.f;
  for (int s0 = 0; s0 < n_split; s0 += 16) {
    float4 v[16];
    float2 w[16];
#pragma unroll
    for (int i = 0; i < 16; i++) {
      if (s0 + i < n_split) {
        w[i] = ml[static_cast<size_t>(s0 + i) * H];
        v[i] = po[(s0 + i) * stride4];
      }
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      if (s0 + i < n_split && w[i].x != -INFINITY) {
        const float mn = fmaxf(M, w[i].x);
        const float c = exp2f(M - mn);  // 0 while M is -inf
        const float e = exp2f(w[i].x - mn);
        L = fmaf(L, c, e * w[i].y);
        acc.x = fmaf(acc.x, c, e * v[i].x);
        acc.y = fmaf(acc.y, c, e * v[i].y);
        acc.z = fmaf(acc.z, c, e * v[i].z);
        acc.w = fmaf(acc.w, c, e * v[i].w);
        M = mn;
      }
    }
  }
  const float il = L > 0.f ? 1.f / L : 0.f;
  reinterpret_cast<float4 *>(a.out + (static_cast<size_t>(b) * H + h) * kD)[threadIdx.x] =
      make_float4(acc.x * il, acc.y * il, acc.z * il, acc.w * il);
  if (threadIdx.x == 0 && a.lse)
    a.lse[static_cast<size_t>(b) * H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

int n_splits(const lidx_attn_args &a) {
  const int rows = a.n_ids + a.swa_len;
  return rows > 0 ? (rows + kRC - 1) / kRC : 1;
}

}  // namespace

bool attn_tc_supported(const lidx_attn_args &a);
int attn_tc_splits(const lidx_attn_args &a);
cudaError_t launch_attn_tc(const lidx_attn_args &a, float *part_o, float2 *part_ml, int n_split, uint32_t *status,
                           cudaStream_t st);

cudaError_t launch_attn_merge(const lidx_attn_args &a, const float *part_o, const float2 *part_ml, int n_split,
                              cudaStream_t st) {
  return launch_kernel(attn_merge_kernel, dim3(a.H, a.B), dim3(128), 0, st,
                       (a.flags & LIDX_LAUNCH_PDL) != 0, a, part_o, part_ml, n_split);
}

namespace {

int splits_for(const lidx_attn_args &a) { return attn_tc_supported(a) ? attn_tc_splits(a) : n_splits(a); }

size_t part_o_bytes(const lidx_attn_args &a, int ns) {
  return ((static_cast<size_t>(ns) * a.B * a.H * kD * sizeof(float) + 255) / 256) * 256;
}

}  // namespace

size_t attn_workspace(const lidx_attn_args &a) {
  const int ns = splits_for(a);
  return LIDX_WS_HEADER + part_o_bytes(a, ns) + static_cast<size_t>(ns) * a.B * a.H * sizeof(float2);
}

int attn_launches(const lidx_attn_args &) { return 2; }  // split kernel + merge kernel

cudaError_t launch_attn(const lidx_attn_args &a, void *ws, cudaStream_t st) {
  uint32_t *status = static_cast<uint32_t *>(ws);
  const int ns = splits_for(a);
  float *part_o = reinterpret_cast<float *>(static_cast<char *>(ws) + LIDX_WS_HEADER);
  float2 *part_ml = reinterpret_cast<float2 *>(static_cast<char *>(ws) + LIDX_WS_HEADER + part_o_bytes(a, ns));
  if (attn_tc_supported(a)) return launch_attn_tc(a, part_o, part_ml, ns, status, st);
  const size_t smem = (static_cast<size_t>(a.H) * kD + kRC * kXs + a.H * kRC) * sizeof(float);
  dim3 grid(ns, a.B);
  switch (a.kv.dtype) {
    case LIDX_F32:
      cudaFuncSetAttribute(attn_cc_kernel<LIDX_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      attn_cc_kernel<LIDX_F32><<<grid, kThreads, smem, st>>>(a, part_o, part_ml, ns, status);
      break;
    case LIDX_BF16:
      cudaFuncSetAttribute(attn_cc_kernel<LIDX_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      attn_cc_kernel<LIDX_BF16><<<grid, kThreads, smem, st>>>(a, part_o, part_ml, ns, status);
      break;
    default:
      cudaFuncSetAttribute(attn_cc_kernel<LIDX_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      attn_cc_kernel<LIDX_E4M3><<<grid, kThreads, smem, st>>>(a, part_o, part_ml, ns, status);
      break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_merge(a, part_o, part_ml, ns, st);
}

}  // namespace lidx
