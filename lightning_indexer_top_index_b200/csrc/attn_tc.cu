// Sparse MQA decode attention on tcgen05 (DeepSeek-V4-Flash architecture
// post, sections (A)-(B): attention over the selected 512-wide attn_comp_kv
// rows plus the 128-row sliding window; K = V = the full row).
//
// Grid (row chunk, head group, sequence).  One CTA takes 64 entries of one
// sequence's row list (the window rows first, then the selected ids) and 16
// of the 64 query heads, and produces the split partial (m_h, l_h, O_h) in
// base-2 units for those heads.  Small CTAs (about 90 KB of shared memory,
// 128 TMEM columns) let a single decode sequence spread over 40 SMs and two
// CTAs share an SM.
//   1. Q [16 heads][512] arrives by TMA.  A chunk made only of window rows
//      (contiguous in memory) arrives as eight 64-row TMA boxes before the
//      top-k kernel has finished; gathered bf16 rows are copied with
//      cp.async, one warp per row, straight into the 128-byte-swizzled
//      K-major layout; E4M3 rows are converted in registers (times their
//      power-of-two block scale; RoPE dims copied).
//   2. MMA 1: S^T[row][head] = X . Q^T (M = 64, N = 16, K = 512) into TMEM.
//   3. Softmax: 8 warps; warp w takes rows 16(w&3).. (its TMEM lanes 0-15)
//      and heads 8(w>>2)..; per-head max and sum over the 64 rows by
//      butterfly shuffles and a 4-warp exchange.  P^T is written to shared
//      memory as bf16 hi and lo parts (p = hi + lo to ~16 bits), K-major: one
//      128-byte swizzled line of 64 rows per head, hi heads then lo heads.
//   4. MMA 2: [O_hi | O_lo]^T[d][.] = X^T . [P_hi | P_lo]^T (N = 32),
//      reading the same X tile as an MN-major operand (K = V), four 128-wide
//      d tiles into TMEM; the epilogue adds the two parts.
//   5. Each warp stores two d tiles, lanes = consecutive d: coalesced stores.
// The partials are combined by the split-K merge kernel.  Batches whose
// grid would need more than one wave of the GPU go to the wide kernel
// (attn_wide.cu) instead: all 64 heads and several chunks per CTA.
#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

cudaError_t launch_attn_merge(const lidx_attn_args &a, const float *part_o, const float2 *part_ml, int n_split,
                              cudaStream_t st);
cudaError_t launch_attn_wide(const lidx_attn_args &a, float *part_o, float2 *part_ml, int n_chunks, uint32_t *status,
                             cudaStream_t st);

namespace {

constexpr int kD = 512;
constexpr int kH = 64;                       // query heads of the supported layout
constexpr int kHG = 16;                      // heads per CTA
constexpr int kGroups = kH / kHG;
constexpr int kRows = 64;                    // row-list entries per CTA
constexpr int kThreads = 256;
constexpr int kXBytes = kRows * kD * 2;      // 64 KB: 8 panels of [64 rows][128 B]
constexpr int kXPanel = kRows * 128;         // 8 KB
constexpr int kQBytes = kHG * kD * 2;        // 16 KB: 8 panels of [16 heads][128 B]
constexpr int kQPanel = kHG * 128;           // 2 KB
constexpr int kPBytes = kHG * kRows * 2;     // 2 KB: one bf16 P^T [16 heads][64 rows]
// TMEM: S^T as kS1 partial sums over K at columns [16i, 16i + 16) (M = 64:
// row 16q + r in lane 32q + r), O^T tile t at [64 + 32t, 96 + 32t) as the
// P_hi part (16 columns) then the P_lo part.  These MMAs are tiny, and each
// costs its issuing thread a roughly fixed time: so MMA 1 is issued by kS1
// threads over K quarters into separate partial sums, MMA 2 by four threads
// (one d tile each) multiplying X^T by P_hi and P_lo at once (N = 32).
constexpr int kS1 = 4;
constexpr uint32_t kOCol = 64;
constexpr uint32_t kTmemCols = 256;
constexpr float kLog2e = 1.4426950408889634f;

struct __align__(8) AttnTcSmem {
  uint64_t q_full;
  uint64_t s_full;
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
  int64_t row_src[kRows];  // row index in its cache; -1 when empty
  int32_t row_kind[kRows]; // 0 none, 1 selected, 2 window
  float red[2][4][8];      // per head half, per row quarter
};

// smem: X (64 KB) | Q (16 KB) | P^T hi, lo (2 x 2 KB) | bookkeeping.  Q
// follows X so that MMA 1's padding rows stay inside the allocation.
constexpr size_t smem_bytes() { return 1024 + kXBytes + kQBytes + 2 * kPBytes + sizeof(AttnTcSmem); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

// byte offset of dims [8c, 8c+8) of row r inside the 64-row K-major swizzled tile
__device__ __forceinline__ uint32_t x_off(int r, int c) {
  return (c >> 3) * kXPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_win,
                   const lidx_attn_args a, float *part_o, float2 *part_ml, int n_split, uint32_t *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem;
  uint8_t *sQ = sX + kXBytes;
  uint8_t *sP = sQ + kQBytes;  // P^T hi at +0, lo at +kPBytes
  AttnTcSmem *sm = reinterpret_cast<AttnTcSmem *>(sP + 2 * kPBytes);
  volatile uint32_t *abort_flag = &sm->abort;

  const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // Row list of a sequence: the window rows first (known before top-k has
  // run), then the selected ids.  This CTA takes list entries [i0, i0+64).
  const int swa_len = a.swa_len;
  const int i0 = split * kRows;
  const bool pure_window = i0 + kRows <= swa_len;

  const bool tma_window = !kFp8 && pure_window;  // 64 contiguous window rows
  if (tid == 0) {
    tc::mbar_init(&sm->q_full, 1);
    tc::mbar_init(&sm->s_full, kS1);
    tc::mbar_init(&sm->o_full, 4);
    sm->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_q);
    tc::mbar_arrive_expect_tx(&sm->q_full, kQBytes + (tma_window ? kXBytes : 0));
#pragma unroll
    for (int p = 0; p < 8; p++) tc::tma_load_2d(sQ + p * kQPanel, &tm_q, &sm->q_full, 64 * p, b * kH + hg * kHG);
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
  if (warp == 1) tc::tmem_alloc(&sm->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t xs = tc::smem_u32(sX);

  // ---- 1. operands: `pass` 0 loads the window rows, pass 1 the selected rows
  // and zero-fills the empty ones
  auto load_rows = [&](int pass) {
    if constexpr (!kFp8) {
      if (pass == 0 && tma_window) return;
      for (int r = warp; r < kRows; r += kThreads / 32) {
        const int kind = sm->row_kind[r];
        if (pass == 0 ? kind != 2 : kind == 2) continue;
        if (kind != 0) {
          const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
          const uint16_t *src = static_cast<const uint16_t *>(kv.data) + sm->row_src[r] * kv.ld;
          cp_async16(xs + x_off(r, lane), src + lane * 8);
          cp_async16(xs + x_off(r, lane + 32), src + (lane + 32) * 8);
        } else {
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane + 32)) = make_uint4(0, 0, 0, 0);
        }
      }
    } else {
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
      // non-RoPE dims: 16 E4M3 codes per step, times their power-of-two block
      // scale (exact while the product is a bf16 value)
      for (int idx = tid; idx < kRows * 28; idx += kThreads) {
        const int r = idx / 28, c16 = idx % 28;
        const int kind = sm->row_kind[r];
        if (pass == 0 ? kind != 2 : kind == 2) continue;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
        if (kind != 0) {
          const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
          const int64_t row = sm->row_src[r];
          const uint4 x = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(kv.data) + row * kv.ld + c16 * 16));
          const float sc = e8m0_to_f32(__ldg(kv.scale + row * kv.ld_scale + (c16 >> 2)));
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 8; i++) o[i] = e4m3x2_to_bf16x2(w[i >> 1] >> (16 * (i & 1)), sc);
          lo = make_uint4(o[0], o[1], o[2], o[3]);
          hi = make_uint4(o[4], o[5], o[6], o[7]);
        }
        *reinterpret_cast<uint4 *>(sX + x_off(r, 2 * c16)) = lo;
        *reinterpret_cast<uint4 *>(sX + x_off(r, 2 * c16 + 1)) = hi;
      }
    }
  };
  load_rows(0);
  if (!pure_window) {
    pdl_wait();  // ids and n_sel come from the top-k kernel
    int n_b = a.n_ids;
    if (a.n_sel) n_b = min(max(a.n_sel[b], 0), a.n_ids);
    // resolve the selected row of list entry i0 + r (row r of the chunk)
    auto resolve_row = [&](int r, int &kind, int64_t &src) {
      const int i = i0 + r - swa_len;
      if (i >= 0 && i < n_b) {
        const int id = a.ids ? a.ids[static_cast<int64_t>(b) * a.ld_ids + i] : i;  // no ids: dense rows
        if (id >= 0 && id < a.N) {
          kind = 1;
          src = static_cast<int64_t>(b) * a.kv.batch_rows + id;
          sm->row_kind[r] = 1;
          sm->row_src[r] = src;
        } else if (id != -1) {
          raise_status(status, LIDX_DEV_BOUNDS);
        }
      }
    };
    if (kFp8) {
      if (tid < kRows) {
        int kind;
        int64_t src;
        resolve_row(tid, kind, src);
      }
      __syncthreads();
      load_rows(1);
    } else {
      // bf16: warp w gathers rows w + 8j; lane j resolves row w + 8j, so no
      // block barrier stands between the ids and the gather
      constexpr int kPerWarp = kRows / (kThreads / 32);
      int kind = 0;
      int64_t src = -1;
      if (lane < kPerWarp) {
        const int r = warp + (kThreads / 32) * lane;
        kind = sm->row_kind[r];
        src = sm->row_src[r];
        resolve_row(r, kind, src);
      }
#pragma unroll
      for (int j = 0; j < kPerWarp; j++) {
        const int kj = __shfl_sync(0xFFFFFFFFu, kind, j);
        const int64_t sj = __shfl_sync(0xFFFFFFFFu, src, j);
        const int r = warp + (kThreads / 32) * j;
        if (kj == 2) continue;  // window row: loaded in pass 0
        if (kj == 1) {
          const uint16_t *row = static_cast<const uint16_t *>(a.kv.data) + sj * a.kv.ld;
          cp_async16(xs + x_off(r, lane), row + lane * 8);
          cp_async16(xs + x_off(r, lane + 32), row + (lane + 32) * 8);
        } else {
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(sX + x_off(r, lane + 32)) = make_uint4(0, 0, 0, 0);
        }
      }
    }
  }
  cp_async_wait_all();
  tc::fence_proxy_async_smem();
  __syncthreads();

  // ---- 2. S^T = X . Q^T: lane 0 of warp i < kS1 issues K steps [8i, 8i + 8)
  // into partial sum i
  if (warp < kS1 && lane == 0) {
    if (tc::mbar_wait(&sm->q_full, 0, abort_flag)) {
      tc::tc_fence_after();
      const uint32_t idesc = tc::idesc_bf16(kRows, kHG);
      const uint32_t qs = tc::smem_u32(sQ);
#pragma unroll
      for (int kk = 0; kk < 32 / kS1; kk++) {
        const int k = warp * (32 / kS1) + kk;
        const uint32_t ao = (k >> 2) * kXPanel + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * kQPanel + (k & 3) * 32;
        tc::mma_bf16(tmem + 16 * warp, tc::desc_kmajor_sw128(xs + ao), tc::desc_kmajor_sw128(qs + bo), idesc, kk > 0);
      }
      tc::mma_commit(&sm->s_full);
    }
  }

  // ---- 3. softmax over the 64 rows, per head: warp w takes row quarter
  // q = w&3 (rows 16q + lane, lanes 0-15; M = 64 puts them in TMEM lanes
  // 32q..32q+15) and heads 8h.. with h = w>>2
  const int quarter = warp & 3, half = warp >> 2;
  bool ready = false;
  if (lane == 0) ready = tc::mbar_wait(&sm->s_full, 0, abort_flag);
  ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
  float mx[8];
  {
    const int r = quarter * 16 + (lane & 15);
    const bool valid = lane < 16 && sm->row_kind[r] != 0;
    float s[8];
    if (ready) {
      tc::tc_fence_after();
      const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 8;
      tc::tmem_ld8(ta, s);
#pragma unroll
      for (int i = 1; i < kS1; i++) {
        float t8[8];
        tc::tmem_ld8(ta + 16 * i, t8);
#pragma unroll
        for (int h = 0; h < 8; h++) s[h] += t8[h];
      }
    }
    const float c2 = a.scale * kLog2e;
#pragma unroll
    for (int h = 0; h < 8; h++) {
      s[h] = valid && ready ? s[h] * c2 : -INFINITY;
      mx[h] = s[h];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)  // lanes 16-31 hold -inf copies: reduce within 16
#pragma unroll
      for (int h = 0; h < 8; h++) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], o));
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < 8; h++) sm->red[half][quarter][h] = mx[h];
    named_sync(1 + half, 128);
    float pv[8];
#pragma unroll
    for (int h = 0; h < 8; h++) {
      const float m = fmaxf(fmaxf(sm->red[half][0][h], sm->red[half][1][h]),
                            fmaxf(sm->red[half][2][h], sm->red[half][3][h]));
      mx[h] = m;
      pv[h] = (m == -INFINITY || s[h] == -INFINITY) ? 0.f : exp2f(s[h] - m);
    }
    // P^T[head][row] as hi = bf16(p), lo = bf16(p - hi): head line h holds
    // rows in 16-byte chunks of 8, chunk index swizzled with h & 7
    if (lane < 16) {
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int h = half * 8 + i;
        const __nv_bfloat16 ph = __float2bfloat16_rn(pv[i]);
        const __nv_bfloat16 pl = __float2bfloat16_rn(pv[i] - __bfloat162float(ph));
        const int off = h * 128 + ((((r >> 3) ^ (h & 7))) << 4) + (r & 7) * 2;
        *reinterpret_cast<__nv_bfloat16 *>(sP + off) = ph;
        *reinterpret_cast<__nv_bfloat16 *>(sP + kPBytes + off) = pl;
      }
    }
    float sum[8];
#pragma unroll
    for (int h = 0; h < 8; h++) sum[h] = lane < 16 ? pv[h] : 0.f;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int h = 0; h < 8; h++) sum[h] += __shfl_xor_sync(0xFFFFFFFFu, sum[h], o);
    named_sync(1 + half, 128);  // the four warps have read the maxima
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < 8; h++) sm->red[half][quarter][h] = sum[h];
    named_sync(1 + half, 128);
  }
  if (pure_window) pdl_wait();  // no global write before the previous kernel is done
  if (quarter == 0 && lane < 8) {
    const float l = (sm->red[half][0][lane] + sm->red[half][1][lane]) + (sm->red[half][2][lane] + sm->red[half][3][lane]);
    float m = mx[0];
#pragma unroll
    for (int i = 1; i < 8; i++)
      if (i == lane) m = mx[i];
    part_ml[(static_cast<size_t>(b) * n_split + split) * kH + hg * kHG + half * 8 + lane] = make_float2(m, l);
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();

  // ---- 4. O^T = X^T . (P_hi + P_lo)^T: lane 0 of warp dt < 4 issues d tile dt
  if (warp < 4 && lane == 0 && !*abort_flag) {
    tc::tc_fence_after();
    const uint32_t idesc = tc::idesc_bf16(128, 2 * kHG, true, false);
    const uint32_t ps = tc::smem_u32(sP);
    const int dt = warp;
#pragma unroll
    for (int kk = 0; kk < kRows / 16; kk++) {
      const uint64_t adesc = tc::desc_mnmajor_sw128(xs + 2 * dt * kXPanel + kk * 2048, kXPanel, 1024);
      const uint64_t bdesc = tc::desc_kmajor_sw128(ps + kk * 32);  // 32 lines: hi heads, then lo heads
      tc::mma_bf16(tmem + kOCol + 32 * dt, adesc, bdesc, idesc, kk > 0);
    }
    tc::mma_commit(&sm->o_full);
  }

  // ---- 5. partial O out: warp w stores d tiles (w>>2) and (w>>2)+2 of its
  // TMEM lane quarter; lanes = consecutive d
  bool oready = false;
  if (lane == 0) oready = !*abort_flag && tc::mbar_wait(&sm->o_full, 0, abort_flag);
  oready = __shfl_sync(0xFFFFFFFFu, oready, 0);
  if (oready) {
    tc::tc_fence_after();
    float *po = part_o + ((static_cast<size_t>(b) * n_split + split) * kH + hg * kHG) * kD;
#pragma unroll
    for (int j = 0; j < 2; j++) {
      const int dt = (warp >> 2) + 2 * j;
      const int d = dt * 128 + quarter * 32 + lane;
      float v[32];
      tc::tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kOCol + 32 * dt, v);
#pragma unroll
      for (int h = 0; h < kHG; h++) po[h * kD + d] = v[h] + v[kHG + h];
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
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

namespace {

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

// The wide kernel once this kernel's grid (four head-group CTAs per row
// chunk, two CTAs per SM) would need more than one wave of the GPU.
bool attn_tc_wide(const lidx_attn_args &a) {
  return static_cast<int64_t>(a.B) * attn_tc_splits(a) * kGroups > 2ll * sm_count();
}

cudaError_t launch_attn_tc(const lidx_attn_args &a, float *part_o, float2 *part_ml, int n_split, uint32_t *status,
                           cudaStream_t st) {
  if (attn_tc_wide(a)) return launch_attn_wide(a, part_o, part_ml, n_split, status, st);
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, static_cast<uint64_t>(a.B) * kH, kD * 2, 64, kHG,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int dt = a.n_ids > 0 ? a.kv.dtype : a.swa.dtype;
  // window rows of one chunk as one 64-row box per 64-dim panel
  CUtensorMap tm_win = tm_q;
  if (dt == LIDX_BF16 && a.swa_len >= kRows) {
    const uint64_t rows = static_cast<uint64_t>(a.B - 1) * (a.B > 1 ? a.swa.batch_rows : 0) + a.swa_len;
    if (!make_tmap_2d(&tm_win, a.swa.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, rows, a.swa.ld * 2, 64, kRows,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const size_t smem = smem_bytes();
  dim3 grid(n_split, kGroups, a.B);
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
