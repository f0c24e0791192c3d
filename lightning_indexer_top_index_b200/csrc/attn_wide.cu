// Sparse MQA decode attention for many sequences (DeepSeek-V4-Flash
// architecture post, sections (A)-(B): attention over the selected 512-wide
// attn_comp_kv rows plus the sliding window; K = V = the full row).
//
// The split kernel of attn_tc.cu gives every CTA one 64-row chunk of a
// sequence's row list, which suits few sequences: many small CTAs.  With many
// sequences its grid needs several waves, every chunk writes a 64-head
// partial O (128 KB of fp32) that the merge kernel reads back, and those
// partials outweigh the rows themselves.  Here one CTA takes all 64 heads
// and a run of consecutive chunks of one sequence, sized so that the grid is
// one wave, and folds the chunks together with an online softmax:
//   * S[head][row] = Q . X^T (M = 64 heads, N = 64 rows, K = 512) into TMEM,
//     issued by four threads over K quarters into partial sums; with the
//     heads on M, each softmax thread owns one head and 16 of the rows.
//   * The running reference maximum M_h and sum L_h live in shared memory;
//     when a chunk raises the maximum by more than 8 (base 2), M_h moves and
//     the O accumulated so far is rescaled by 2^(M_old - M_new) in TMEM
//     (read, scale, write back) before the chunk's MMA adds to it; smaller
//     rises keep M_h, so probabilities stay below 2^8 and the rescale is rare.
//   * O^T[d][head] += X^T . P^T (M = 128 d, N = 64 heads, K = 64 rows), P
//     carried as bf16 hi + lo parts accumulated into the same columns.
//   * The next chunk's rows are gathered into a second buffer while the
//     current one is computed.
// Each CTA writes one split partial (m, l, O) in the split kernel's format,
// so the same merge kernel combines the CTAs of a sequence.
#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

cudaError_t launch_attn_merge(const lidx_attn_args &a, const float *part_o, const float2 *part_ml, int n_split,
                              cudaStream_t st);

namespace {

constexpr int kD = 512;
constexpr int kH = 64;
constexpr int kRows = 64;                // rows per chunk
constexpr int kThreads = 512;
constexpr int kXBytes = kRows * kD * 2;  // 8 panels of [64 rows][128 B]
constexpr int kPanel = 64 * 128;         // one 64-line panel of X or Q
constexpr int kQBytes = kH * kD * 2;
constexpr int kPBytes = kH * kRows * 2;  // one bf16 P^T [64 heads][64 rows]
constexpr int kS1 = 4;                   // K-split partial sums of S
constexpr uint32_t kOCol = kS1 * 64;     // O^T tile t at columns kOCol + 64 t
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.f;             // base-2 headroom of the reference maximum

struct __align__(8) WideSmem {
  uint64_t q_full;
  uint64_t s_full;
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t rescale;           // this chunk raised some head's maximum
  int32_t row_kind[2][kRows]; // per buffer: 0 none, 1 selected, 2 window
  float red_m[4][kH];         // per row part, per head
  float red_l[4][kH];
  float run_m[kH];            // running maximum (base 2) and sum per head
  float run_l[kH];
  float alpha[kH];            // this chunk's rescale factor per head
};

// smem: Q | X[2] | P^T hi, lo | bookkeeping (all panels 1024-aligned)
constexpr size_t smem_bytes() { return 1024 + kQBytes + 2 * kXBytes + 2 * kPBytes + sizeof(WideSmem); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

// byte offset of dims [8c, 8c+8) of row r inside the 64-row K-major swizzled tile
__device__ __forceinline__ uint32_t x_off(int r, int c) {
  return (c >> 3) * kPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// 32 consecutive fp32 columns of this thread's TMEM lane, written back.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's TMEM lane, without waiting;
// tmem_ld16_pin (after tcgen05.wait::ld) keeps their uses after the wait.
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16_pin(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const lidx_attn_args a, float *part_o,
                     float2 *part_ml, int n_split, int n_chunks, uint32_t *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sX = sQ + kQBytes;  // buffer i at sX + i * kXBytes
  uint8_t *sP = sX + 2 * kXBytes;
  WideSmem *sm = reinterpret_cast<WideSmem *>(sP + 2 * kPBytes);
  volatile uint32_t *abort_flag = &sm->abort;

  const int split = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // this CTA's chunks [c0, c1) of the sequence's row list (window rows first)
  const int c0 = static_cast<int>(static_cast<int64_t>(split) * n_chunks / n_split);
  const int c1 = static_cast<int>(static_cast<int64_t>(split + 1) * n_chunks / n_split);
  const int swa_len = a.swa_len;

  if (tid == 0) {
    tc::mbar_init(&sm->q_full, 1);
    tc::mbar_init(&sm->s_full, kS1);
    tc::mbar_init(&sm->o_full, 4);
    sm->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_q);
    tc::mbar_arrive_expect_tx(&sm->q_full, kQBytes);
#pragma unroll
    for (int p = 0; p < 8; p++) tc::tma_load_2d(sQ + p * kPanel, &tm_q, &sm->q_full, 64 * p, b * kH);
  }
  if (tid < kH) {
    sm->run_m[tid] = -INFINITY;
    sm->run_l[tid] = 0.f;
  }
  if (warp == 1) tc::tmem_alloc(&sm->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = sm->tmem_base;
  pdl_wait();  // ids and n_sel come from the top-k kernel; no global write before it is done

  int n_b = a.n_ids;
  if (a.n_sel) n_b = min(max(a.n_sel[b], 0), a.n_ids);

  // Gather chunk c into buffer `buf`: warp w takes rows w, w + 16, ...; bf16
  // rows by cp.async (one warp per 1 KB row), E4M3 rows converted in
  // registers times their power-of-two block scale (RoPE dims as they are).
  auto load_chunk = [&](int c, int buf) {
    uint8_t *x = sX + buf * kXBytes;
    const uint32_t xs = tc::smem_u32(x);
    for (int r = warp; r < kRows; r += kThreads / 32) {
      const int e = c * kRows + r;  // list entry
      int kind = 0;
      int64_t src = -1;
      if (e < swa_len) {
        kind = 2;
        src = static_cast<int64_t>(b) * a.swa.batch_rows + e;
      } else if (e - swa_len < n_b) {
        const int i = e - swa_len;
        const int id = a.ids ? a.ids[static_cast<int64_t>(b) * a.ld_ids + i] : i;  // no ids: dense rows
        if (id >= 0 && id < a.N) {
          kind = 1;
          src = static_cast<int64_t>(b) * a.kv.batch_rows + id;
        } else if (id != -1 && lane == 0) {
          raise_status(status, LIDX_DEV_BOUNDS);
        }
      }
      if (lane == 0) sm->row_kind[buf][r] = kind;
      if (kind == 0) {
        *reinterpret_cast<uint4 *>(x + x_off(r, lane)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(x + x_off(r, lane + 32)) = make_uint4(0, 0, 0, 0);
        continue;
      }
      const lidx_kv &kv = kind == 1 ? a.kv : a.swa;
      if (!kFp8) {
        const uint16_t *row = static_cast<const uint16_t *>(kv.data) + src * kv.ld;
        cp_async16(xs + x_off(r, lane), row + lane * 8);
        cp_async16(xs + x_off(r, lane + 32), row + (lane + 32) * 8);
      } else {
        // lanes 0-27: 16 codes each (dims 16 l .. 16 l + 15); lanes 28-31:
        // RoPE dims 448 + 16 (l - 28) .. by two 16-byte copies
        if (lane < 28) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(kv.data) + src * kv.ld +
                                                                lane * 16));
          const float sc = e8m0_to_f32(__ldg(kv.scale + src * kv.ld_scale + (lane >> 2)));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 8; i++) o[i] = e4m3x2_to_bf16x2(w4[i >> 1] >> (16 * (i & 1)), sc);
          *reinterpret_cast<uint4 *>(x + x_off(r, 2 * lane)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4 *>(x + x_off(r, 2 * lane + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
          const uint16_t *rope = static_cast<const uint16_t *>(kv.rope) + src * kv.ld_rope;
          const int c8 = 56 + 2 * (lane - 28);
          cp_async16(xs + x_off(r, c8), rope + (c8 - 56) * 8);
          cp_async16(xs + x_off(r, c8 + 1), rope + (c8 + 1 - 56) * 8);
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  if (c0 < c1) load_chunk(c0, 0);
  const int quarter = warp & 3, rp = warp >> 2;  // softmax: heads 16q.., rows 16 rp..
  const int head = quarter * 16 + (lane & 15);
  const float c2 = a.scale * kLog2e;
  for (int c = c0; c < c1; c++) {
    const int buf = (c - c0) & 1;
    const uint32_t par = static_cast<uint32_t>((c - c0) & 1);
    // this chunk's rows (gathered one iteration earlier) are in
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // (every thread read the previous chunk's flag before that chunk's
    // rescale barrier, or it was already clear)
    if (tid == 0) sm->rescale = 0u;
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- S[head][row] = Q . X^T: lane 0 of warp 4 + i (i < kS1) issues K
    // steps [8i, 8i + 8).  Other threads than MMA 2's, so that the commit of
    // S does not also wait for the previous chunk's O.
    const uint32_t xs = tc::smem_u32(sX + buf * kXBytes);
    if (warp >= 4 && warp < 4 + kS1 && lane == 0 && !*abort_flag) {
      if (c > c0 || tc::mbar_wait(&sm->q_full, 0, abort_flag)) {
        tc::tc_fence_after();
        const uint32_t idesc = tc::idesc_bf16(64, 64);
        const uint32_t qs = tc::smem_u32(sQ);
        const int part = warp - 4;
#pragma unroll
        for (int kk = 0; kk < 32 / kS1; kk++) {
          const int k = part * (32 / kS1) + kk;
          const uint32_t off = (k >> 2) * kPanel + (k & 3) * 32;
          tc::mma_bf16(tmem + 64 * part, tc::desc_kmajor_sw128(qs + off), tc::desc_kmajor_sw128(xs + off), idesc,
                       kk > 0);
        }
        tc::mma_commit(&sm->s_full);
      }
    }

    // MMA 1 touches nothing MMA 2 of the previous chunk uses; once that has
    // finished, its X buffer, P and O are free: gather the next chunk
    if (c > c0 && lane == 0) tc::mbar_wait(&sm->o_full, par ^ 1u, abort_flag);
    __syncwarp();
    tc::tc_fence_after();
    if (c + 1 < c1) load_chunk(c + 1, buf ^ 1);

    // ---- online softmax: thread (quarter q, lane l < 16) owns head 16q + l
    // and rows 16 rp .. 16 rp + 15 (TMEM lane 32q + l, M = 64)
    bool ready = false;
    if (lane == 0) ready = !*abort_flag && tc::mbar_wait(&sm->s_full, par, abort_flag);
    ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
    float s[16];
    if (ready) {
      tc::tc_fence_after();
      const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 16 * rp;
      uint32_t t[kS1][16];
#pragma unroll
      for (int i = 0; i < kS1; i++) tmem_ld16_issue(ta + 64 * i, t[i]);
      tc::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < kS1; i++) tmem_ld16_pin(t[i]);
#pragma unroll
      for (int j = 0; j < 16; j++)
        s[j] = (__uint_as_float(t[0][j]) + __uint_as_float(t[1][j])) + (__uint_as_float(t[2][j]) + __uint_as_float(t[3][j]));
    }
    float mloc = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const bool valid = ready && sm->row_kind[buf][16 * rp + j] != 0;
      s[j] = valid ? s[j] * c2 : -INFINITY;
      mloc = fmaxf(mloc, s[j]);
    }
    if (lane < 16) sm->red_m[rp][head] = mloc;
    named_sync(1 + quarter, 128);
    // The reference maximum moves only when the chunk raises it by more than
    // kLazy (so p stays below 2^kLazy and O is rescaled rarely); (m, l, O)
    // stay consistent with it, which is all the merge needs.
    const float m_old = sm->run_m[head];
    const float m_hi = fmaxf(m_old, fmaxf(fmaxf(sm->red_m[0][head], sm->red_m[1][head]),
                                          fmaxf(sm->red_m[2][head], sm->red_m[3][head])));
    const float m_new = (m_old != -INFINITY && m_hi - m_old <= kLazy) ? m_old : m_hi;
    float lsum = 0.f;
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float p0 = (m_new == -INFINITY || s[j] == -INFINITY) ? 0.f : exp2f(s[j] - m_new);
      const float p1 = (m_new == -INFINITY || s[j + 1] == -INFINITY) ? 0.f : exp2f(s[j + 1] - m_new);
      lsum += p0 + p1;
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
      hi[j >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
      lo[j >> 1] = *reinterpret_cast<const uint32_t *>(&l2);
    }
    if (lane < 16) {
      // P^T line `head`: rows in 16-byte chunks of 8, chunk index swizzled with head & 7
#pragma unroll
      for (int h2 = 0; h2 < 2; h2++) {
        const int off = head * 128 + (((2 * rp + h2) ^ (head & 7)) << 4);
        *reinterpret_cast<uint4 *>(sP + off) = make_uint4(hi[4 * h2], hi[4 * h2 + 1], hi[4 * h2 + 2], hi[4 * h2 + 3]);
        *reinterpret_cast<uint4 *>(sP + kPBytes + off) =
            make_uint4(lo[4 * h2], lo[4 * h2 + 1], lo[4 * h2 + 2], lo[4 * h2 + 3]);
      }
      sm->red_l[rp][head] = lsum;
    }
    named_sync(1 + quarter, 128);  // the quarter's sums are in; every max read
    if (rp == 0 && lane < 16) {
      const float al = m_old == m_new ? 1.f : (m_old == -INFINITY ? 0.f : exp2f(m_old - m_new));
      const float l_new = (sm->red_l[0][head] + sm->red_l[1][head]) + (sm->red_l[2][head] + sm->red_l[3][head]);
      sm->run_l[head] = fmaf(sm->run_l[head], al, l_new);
      sm->run_m[head] = m_new;
      sm->alpha[head] = al;
      if (al != 1.f && c > c0) sm->rescale = 1u;
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ---- rescale the O accumulated so far where a head's maximum rose:
    // warp (quarter q, d tile rp) scales its lane's 64 head columns
    if (sm->rescale) {
      tc::tc_fence_after();
      const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kOCol + 64 * rp;
#pragma unroll
      for (int h0 = 0; h0 < 64; h0 += 32) {
        uint32_t v[32];
        tc::tmem_ld32_issue(ta + h0, v);
        tc::tmem_ld_wait();
        tc::tmem_ld32_pin(v);
#pragma unroll
        for (int h = 0; h < 32; h++) v[h] = __float_as_uint(__uint_as_float(v[h]) * sm->alpha[h0 + h]);
        tmem_st32(ta + h0, v);
      }
      tmem_st_wait();
      tc::tc_fence_before();
      __syncthreads();
    }

    // ---- O^T += X^T . (P_hi + P_lo)^T: lane 0 of warp dt < 4 issues d tile dt
    if (warp < 4 && lane == 0 && !*abort_flag) {
      tc::tc_fence_after();
      const uint32_t idesc = tc::idesc_bf16(128, 64, true, false);
      const uint32_t ps = tc::smem_u32(sP);
      const int dt = warp;
#pragma unroll
      for (int part = 0; part < 2; part++)
#pragma unroll
        for (int kk = 0; kk < kRows / 16; kk++) {
          const uint64_t adesc = tc::desc_mnmajor_sw128(xs + 2 * dt * kPanel + kk * 2048, kPanel, 1024);
          const uint64_t bdesc = tc::desc_kmajor_sw128(ps + part * kPBytes + kk * 32);
          tc::mma_bf16(tmem + kOCol + 64 * dt, adesc, bdesc, idesc, c > c0 || part > 0 || kk > 0);
        }
      tc::mma_commit(&sm->o_full);
    }
  }

  // ---- the partial (m, l, O) of this CTA's chunks
  bool oready = false;
  if (lane == 0 && c0 < c1)
    oready = !*abort_flag && tc::mbar_wait(&sm->o_full, static_cast<uint32_t>((c1 - 1 - c0) & 1), abort_flag);
  oready = __shfl_sync(0xFFFFFFFFu, oready, 0);
  if (tid < kH) {
    const bool any = c0 < c1;
    part_ml[(static_cast<size_t>(b) * n_split + split) * kH + tid] =
        make_float2(any ? sm->run_m[tid] : -INFINITY, any ? sm->run_l[tid] : 0.f);
  }
  if (oready) {
    tc::tc_fence_after();
    float *po = part_o + (static_cast<size_t>(b) * n_split + split) * kH * kD;
    const int dt = rp, d = dt * 128 + quarter * 32 + lane;
    const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kOCol + 64 * dt;
#pragma unroll
    for (int h0 = 0; h0 < 64; h0 += 32) {
      float v[32];
      tc::tmem_ld32(ta + h0, v);
#pragma unroll
      for (int h = 0; h < 32; h++) po[(h0 + h) * kD + d] = v[h];
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

// CTAs per sequence: as many as keep the grid to one wave, at most one per
// chunk.
int attn_wide_splits(const lidx_attn_args &a, int n_chunks) {
  return std::max(1, std::min(n_chunks, sm_count() / std::max(1, a.B)));
}

cudaError_t launch_attn_wide(const lidx_attn_args &a, float *part_o, float2 *part_ml, int n_chunks, uint32_t *status,
                             cudaStream_t st) {
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, static_cast<uint64_t>(a.B) * kH, kD * 2, 64, kH,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int n_split = attn_wide_splits(a, n_chunks);
  const bool fp8 = (a.n_ids > 0 ? a.kv.dtype : a.swa.dtype) == LIDX_E4M3;
  const size_t smem = smem_bytes();
  const dim3 grid(n_split, a.B);
  const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
  cudaError_t e;
  if (fp8) {
    cudaFuncSetAttribute(attn_wide_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    e = launch_kernel(attn_wide_kernel<true>, grid, dim3(kThreads), smem, st, pdl, tm_q, a, part_o, part_ml, n_split,
                      n_chunks, status);
  } else {
    cudaFuncSetAttribute(attn_wide_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    e = launch_kernel(attn_wide_kernel<false>, grid, dim3(kThreads), smem, st, pdl, tm_q, a, part_o, part_ml, n_split,
                      n_chunks, status);
  }
  if (e != cudaSuccess) return e;
  return launch_attn_merge(a, part_o, part_ml, n_split, st);
}

}  // namespace lidx
