// Sparse MQA decode attention on tcgen05 (DeepSeek-V4-Flash architecture
// post, sections (A)-(B): attention over the selected 512-wide attn_comp_kv
// rows plus the 128-row sliding window; K = V = the full row).
//
// One CTA takes 128 rows of one sequence's row list (the window rows, then
// the selected ids) and produces the split partial (m_h, l_h, O_h) in base-2
// units for the 64 heads:
//   1. Q [64 heads][512] arrives by TMA.  A chunk made only of window rows
//      (contiguous in memory) arrives as eight 128-row TMA boxes before the
//      top-k kernel has finished; gathered bf16 rows are copied with
//      cp.async, one warp per row, straight into the 128-byte-swizzled
//      K-major layout; E4M3 rows are converted in registers (the
//      power-of-two block scale added to the bf16 exponent; RoPE dims copied).
//   2. MMA 1: S^T[row][head] = X . Q^T (M = 128 rows, N = 64 heads,
//      K = 512) into TMEM.
//   3. Softmax: 16 warps; thread = one row and 16 heads (warp w: TMEM lane
//      quarter w&3, heads 16*(w>>2)..); per-head max and sum over rows by
//      butterfly shuffles and a 4-warp exchange; P^T is written to shared
//      memory as bf16 hi and lo parts (p = hi + lo to ~16 bits) in the
//      swizzled MN-major layout.
//   4. MMA 2: O^T[d][head] = X^T . P^T, reading the same X tile as an
//      MN-major operand (K = V), four 128-wide d tiles into TMEM.
//   5. Warp w stores d tile w>>2, lanes = consecutive d: coalesced stores.
// The partials are combined by the split-K merge kernel.
#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

cudaError_t launch_attn_merge(const lidx_attn_args &a, const float *part_o, const float2 *part_ml, int n_split,
                              cudaStream_t st);

namespace {

constexpr int kD = 512;
constexpr int kH = 64;
constexpr int kRows = 128;
constexpr int kThreads = 512;
constexpr int kQBytes = kH * kD * 2;         // 64 KB: 8 panels of [64][128 B]
constexpr int kQPanel = kH * 128;            // 8 KB
constexpr int kXBytes = kRows * kD * 2;      // 128 KB: 8 panels of [128][128 B]
constexpr int kXPanel = kRows * 128;         // 16 KB
constexpr int kPBytes = kRows * kH * 2;      // 16 KB: one bf16 P^T [128 rows][64 heads]
constexpr float kLog2e = 1.4426950408889634f;

struct __align__(8) AttnTcSmem {
  uint64_t q_full;
  uint64_t s_full;
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
  int64_t row_src[kRows];  // byte offset of the row in its plane set; -1 when empty
  int32_t row_kind[kRows]; // 0 none, 1 selected, 2 window
  float red[4][4][16];     // per head group, per lane quarter: max, then sum
};

// Q is dead once MMA 1 has completed; P^T (hi and lo bf16 parts) reuses it.
constexpr size_t smem_bytes() { return 1024 + kQBytes + kXBytes + sizeof(AttnTcSmem); }
static_assert(2 * kPBytes <= kQBytes, "P^T hi/lo must fit in the Q buffer");

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

// byte offset of dims [8c, 8c+8) of row r inside a 128-row K-major swizzled tile
__device__ __forceinline__ uint32_t x_off(int r, int c) {
  return (c >> 3) * kXPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_win,
                   const lidx_attn_args a, float *part_o, float2 *part_ml, int n_split, uint32_t *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sX = sQ + kQBytes;
  uint8_t *sP = sQ;  // P^T hi at +0, lo at +kPBytes (after MMA 1 is done with Q)
  AttnTcSmem *sm = reinterpret_cast<AttnTcSmem *>(sX + kXBytes);
  volatile uint32_t *abort_flag = &sm->abort;

  const int split = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // Row list of a sequence: the window rows first (known before top-k has
  // run), then the selected ids.  This CTA takes list entries [i0, i0+128).
  const int swa_len = a.swa_len;
  const int i0 = split * kRows;
  const bool pure_window = i0 + kRows <= swa_len;

  const bool tma_window = !kFp8 && pure_window;  // 128 contiguous window rows
  if (tid == 0) {
    tc::mbar_init(&sm->q_full, 1);
    tc::mbar_init(&sm->s_full, 1);
    tc::mbar_init(&sm->o_full, 1);
    sm->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_q);
    tc::mbar_arrive_expect_tx(&sm->q_full, kQBytes + (tma_window ? kXBytes : 0));
#pragma unroll
    for (int p = 0; p < 8; p++) tc::tma_load_2d(sQ + p * kQPanel, &tm_q, &sm->q_full, 64 * p, b * kH);
    if (tma_window) {
      const int y = static_cast<int>(static_cast<int64_t>(b) * a.swa.batch_rows + i0);
#pragma unroll
      for (int p = 0; p < 8; p++) tc::tma_load_2d(sX + p * kXPanel, &tm_win, &sm->q_full, 64 * p, y);
    }
  }
  if (tid < kRows) {
    const int i = i0 + tid;
    const bool win = i < swa_len;
    sm->row_kind[tid] = win ? 2 : 0;
    sm->row_src[tid] = win ? static_cast<int64_t>(b) * a.swa.batch_rows + i : -1;
  }
  if (warp == 1) tc::tmem_alloc(&sm->tmem_base, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t xs = tc::smem_u32(sX);

  // ---- 1. operands: `pass` 0 loads the window rows, pass 1 the selected rows
  // and zero-fills the empty ones
  auto load_rows = [&](int pass) {
    if (!kFp8) {
      if (pass == 0 && tma_window) return;
      const int warp_ = tid >> 5, lane_ = tid & 31;
      for (int r = warp_; r < kRows; r += kThreads / 32) {
        const int kind = sm->row_kind[r];
        if (pass == 0 ? kind != 2 : kind == 2) continue;
        if (kind != 0) {
          const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
          const uint16_t *src = static_cast<const uint16_t *>(kv.data) + sm->row_src[r] * kv.ld;
          cp_async16(xs + x_off(r, lane_), src + lane_ * 8);
          cp_async16(xs + x_off(r, lane_ + 32), src + (lane_ + 32) * 8);
        } else {
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane_)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane_ + 32)) = make_uint4(0, 0, 0, 0);
        }
      }
      return;
    }
    // RoPE dims [448, 512) as they are
    for (int idx = tid; idx < kRows * 8; idx += kThreads) {
      const int r = idx >> 3, c = 56 + (idx & 7);
      const int kind = sm->row_kind[r];
      if (pass == 0 ? kind != 2 : kind == 2) continue;
      if (kind != 0) {
        const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
        cp_async16(xs + x_off(r, c), static_cast<const uint16_t *>(kv.rope) + sm->row_src[r] * kv.ld_rope + (c - 56) * 8);
      } else {
        *reinterpret_cast<uint4 *>(sX + x_off(r, c)) = make_uint4(0, 0, 0, 0);
      }
    }
    // non-RoPE dims: 16 E4M3 codes per step, block scale folded into the exponent
    for (int idx = tid; idx < kRows * 28; idx += kThreads) {
      const int r = idx / 28, c16 = idx % 28;
      const int kind = sm->row_kind[r];
      if (pass == 0 ? kind != 2 : kind == 2) continue;
      uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
      if (kind != 0) {
        const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
        const int64_t row = sm->row_src[r];
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(kv.data) + row * kv.ld + c16 * 16));
        const int e = static_cast<int>(__ldg(kv.scale + row * kv.ld_scale + (c16 >> 2))) - 127;
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
          uint32_t pair = 0;
#pragma unroll
          for (int h = 0; h < 2; h++) {
            const uint32_t code = (w[i / 2] >> (16 * (i & 1) + 8 * h)) & 0xFFu;
            uint32_t bits = e4m3_to_bf16_bits(code);
            // exact while the scaled value stays a normal bf16
            if ((bits & 0x7F80u) != 0 && (bits & 0x7F80u) != 0x7F80u) bits += static_cast<uint32_t>(e) << 7;
            pair |= (bits & 0xFFFFu) << (16 * h);
          }
          o[i] = pair;
        }
        lo = make_uint4(o[0], o[1], o[2], o[3]);
        hi = make_uint4(o[4], o[5], o[6], o[7]);
      }
      *reinterpret_cast<uint4 *>(sX + x_off(r, 2 * c16)) = lo;
      *reinterpret_cast<uint4 *>(sX + x_off(r, 2 * c16 + 1)) = hi;
    }
  };
  load_rows(0);
  if (!pure_window) {
    pdl_wait();  // ids and n_sel come from the top-k kernel
    int n_b = a.n_ids;
    if (a.n_sel) n_b = min(max(a.n_sel[b], 0), a.n_ids);
    if (tid < kRows) {
      const int i = i0 + tid - swa_len;
      if (i >= 0 && i < n_b) {
        const int id = a.ids[static_cast<int64_t>(b) * a.ld_ids + i];
        if (id >= 0 && id < a.N) {
          sm->row_kind[tid] = 1;
          sm->row_src[tid] = static_cast<int64_t>(b) * a.kv.batch_rows + id;
        } else if (id != -1) {
          raise_status(status, LIDX_DEV_BOUNDS);
        }
      }
    }
    __syncthreads();
    load_rows(1);
  }
  cp_async_wait_all();
  tc::fence_proxy_async_smem();
  __syncthreads();

  // ---- 2. S^T = X . Q^T
  if (tid == 0) {
    if (tc::mbar_wait(&sm->q_full, 0, abort_flag)) {
      tc::tc_fence_after();
      const uint32_t idesc = tc::idesc_bf16(kRows, kH);
      const uint32_t qs = tc::smem_u32(sQ);
#pragma unroll
      for (int k = 0; k < 32; k++) {
        const uint32_t ao = (k >> 2) * kXPanel + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * kQPanel + (k & 3) * 32;
        tc::mma_bf16(tmem, tc::desc_kmajor_sw128(xs + ao), tc::desc_kmajor_sw128(qs + bo), idesc, k > 0);
      }
      tc::mma_commit(&sm->s_full);
    }
  }

  // ---- 3. softmax over the 128 rows, per head: warp w covers TMEM lane
  // quarter w&3 (rows) and heads [16g, 16g+16), g = w>>2
  const int quarter = warp & 3, g = warp >> 2;
  const int r = quarter * 32 + lane;
  const bool valid = sm->row_kind[r] != 0;
  bool ready = false;
  if (lane == 0) ready = tc::mbar_wait(&sm->s_full, 0, abort_flag);
  ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
  float s[32];
  if (ready) {
    tc::tc_fence_after();
    tc::tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + (g >> 1) * 32, s);
  }
  const bool upper = (g & 1) != 0;  // this group's heads: columns 16..31 of the load
  const float c2 = a.scale * kLog2e;
  float mx[16];
#pragma unroll
  for (int h = 0; h < 16; h++) {
    const float x = upper ? s[16 + h] : s[h];
    s[h] = valid && ready ? x * c2 : -INFINITY;
    mx[h] = s[h];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < 16; h++) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], o));
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < 16; h++) sm->red[g][quarter][h] = mx[h];
  named_sync(1 + g, 128);
  float pv[16];
#pragma unroll
  for (int h = 0; h < 16; h++) {
    const float m = fmaxf(fmaxf(sm->red[g][0][h], sm->red[g][1][h]), fmaxf(sm->red[g][2][h], sm->red[g][3][h]));
    mx[h] = m;
    pv[h] = (m == -INFINITY || s[h] == -INFINITY) ? 0.f : exp2f(s[h] - m);
  }
  // P^T row r, heads [16g, 16g+16): two 16-byte chunks of 8 bf16, as
  // hi = bf16(p) and lo = bf16(p - hi) so the PV product keeps ~16 bits
  {
    uint8_t *prow = sP + r * 128;
#pragma unroll
    for (int cc = 0; cc < 2; cc++) {
      uint32_t oh[4], ol[4];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float p0 = pv[cc * 8 + 2 * i], p1 = pv[cc * 8 + 2 * i + 1];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        const float2 hf = __bfloat1622float2(h2);
        const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
        oh[i] = *reinterpret_cast<const uint32_t *>(&h2);
        ol[i] = *reinterpret_cast<const uint32_t *>(&l2);
      }
      const int chunk = g * 2 + cc;
      const int off = (chunk ^ (r & 7)) << 4;
      *reinterpret_cast<uint4 *>(prow + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
      *reinterpret_cast<uint4 *>(prow + kPBytes + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    }
  }
  float sum[16];
#pragma unroll
  for (int h = 0; h < 16; h++) sum[h] = pv[h];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < 16; h++) sum[h] += __shfl_xor_sync(0xFFFFFFFFu, sum[h], o);
  named_sync(1 + g, 128);  // everyone has read the maxima
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < 16; h++) sm->red[g][quarter][h] = sum[h];
  named_sync(1 + g, 128);
  if (pure_window) pdl_wait();  // no global write before the previous kernel is done
  if (quarter == 0 && lane < 16) {
    const int h = lane;
    const float l = sm->red[g][0][h] + sm->red[g][1][h] + sm->red[g][2][h] + sm->red[g][3][h];
    float m = mx[0];
#pragma unroll
    for (int i = 1; i < 16; i++)
      if (i == h) m = mx[i];
    part_ml[(static_cast<size_t>(b) * n_split + split) * kH + g * 16 + h] = make_float2(m, l);
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();

  // ---- 4. O^T = X^T . (P_hi + P_lo)^T
  if (tid == 0 && ready && !*abort_flag) {
    tc::tc_fence_after();
    const uint32_t idesc = tc::idesc_bf16(128, kH, true, true);
    const uint32_t ps = tc::smem_u32(sP);
#pragma unroll
    for (int dt = 0; dt < 4; dt++) {
#pragma unroll
      for (int part = 0; part < 2; part++) {
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {
          const uint64_t adesc = tc::desc_mnmajor_sw128(xs + 2 * dt * kXPanel + kk * 2048, kXPanel, 1024);
          const uint64_t bdesc = tc::desc_mnmajor_sw128(ps + part * kPBytes + kk * 2048, kPBytes, 1024);
          tc::mma_bf16(tmem + 64 + 64 * dt, adesc, bdesc, idesc, (part | kk) != 0);
        }
      }
    }
    tc::mma_commit(&sm->o_full);
  }

  // ---- 5. partial O out: warp w stores d tile w>>2, lanes = consecutive d
  bool oready = false;
  if (lane == 0) oready = ready && tc::mbar_wait(&sm->o_full, 0, abort_flag);
  oready = __shfl_sync(0xFFFFFFFFu, oready, 0);
  if (oready) {
    tc::tc_fence_after();
    float *po = part_o + (static_cast<size_t>(b) * n_split + split) * kH * kD;
    const int d = g * 128 + quarter * 32 + lane;
#pragma unroll
    for (int h0 = 0; h0 < kH; h0 += 32) {
      float v[32];
      tc::tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64 + 64 * g + h0, v);
#pragma unroll
      for (int h = 0; h < 32; h++) po[(h0 + h) * kD + d] = v[h];
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && sm->abort) raise_status(status, LIDX_DEV_TIMEOUT);
}

}  // namespace

bool attn_tc_supported(const lidx_attn_args &a) {
  if (a.H != kH || a.q_dtype != LIDX_BF16) return false;
  const int dt = a.n_ids > 0 ? a.kv.dtype : a.swa.dtype;
  return dt == LIDX_BF16 || dt == LIDX_E4M3;
}

int attn_tc_splits(const lidx_attn_args &a) {
  const int rows = a.n_ids + a.swa_len;
  return rows > 0 ? (rows + kRows - 1) / kRows : 1;
}

cudaError_t launch_attn_tc(const lidx_attn_args &a, float *part_o, float2 *part_ml, int n_split, uint32_t *status,
                           cudaStream_t st) {
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, static_cast<uint64_t>(a.B) * kH, kD * 2, 64, kH,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int dt = a.n_ids > 0 ? a.kv.dtype : a.swa.dtype;
  // window rows of one chunk as one 128-row box per 64-dim panel
  CUtensorMap tm_win = tm_q;
  if (dt == LIDX_BF16 && a.swa_len >= kRows) {
    const uint64_t rows = static_cast<uint64_t>(a.B - 1) * (a.B > 1 ? a.swa.batch_rows : 0) + a.swa_len;
    if (!make_tmap_2d(&tm_win, a.swa.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, rows, a.swa.ld * 2, 64, kRows,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const size_t smem = smem_bytes();
  dim3 grid(n_split, a.B);
  const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
  cudaError_t e;
  if (dt == LIDX_E4M3) {
    cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    e = launch_kernel(attn_tc_kernel<true>, grid, dim3(kThreads), smem, st, pdl, tm_q, tm_win, a, part_o, part_ml, n_split,
                      status);
  } else {
    cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    e = launch_kernel(attn_tc_kernel<false>, grid, dim3(kThreads), smem, st, pdl, tm_q, tm_win, a, part_o, part_ml, n_split,
                      status);
  }
  if (e != cudaSuccess) return e;
  return launch_attn_merge(a, part_o, part_ml, n_split, st);
}

}  // namespace lidx
