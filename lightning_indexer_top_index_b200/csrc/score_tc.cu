// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05).
//
//   s[b,t,j] = sum_h w[b,t,h] * max(q[b,t,h,:] . k[b,j,:], 0)
//
// (DeepSeek-V4-Flash architecture post, section (B); head-weighted ReLU-MQA
// of the FlashMemory deep-dive write-up, reply #2.)
//
// Layout: keys on the MMA's M side (128 entries per tile), query heads on N
// (QG queries x H heads, <= 256 columns).  One work unit is (sequence b,
// query group g, key tile t); each CTA walks a contiguous range of units.
//   warp 0      TMA producer: the query tile of (b,g) once, then key tiles
//               through a kStages-deep ring of shared-memory stages
//   warp 1      allocates TMEM; one lane issues the MMAs (K = 128 in steps of
//               16) into one of two TMEM accumulators and commits
//   warps 2-9   epilogue, two groups of four warps taking alternate tiles
//               (group k reduces accumulator k): each thread owns one key row
//               (its TMEM lane), loads the H head dots of each query and
//               reduces sum_h w_h max(x,0) in registers; 128 consecutive
//               scores per query are stored.  Two groups keep the reduction,
//               which one warp per SM sub-partition cannot hide, off the
//               critical path.
//   warps 10-13 (E4M3 keys only) convert the FP8 non-RoPE half of each key
//               tile to bf16 in the 128-byte-swizzled layout the MMA reads;
//               the RoPE half arrives by TMA directly.  The power-of-two
//               block scale is applied in the epilogue to a separate
//               accumulator, so the FP8 path is exact.
// One query group per (b,g): for decode (Q = 1) the query tile stays resident
// and the kernel streams the keys once at HBM speed; for many queries
// (prefill / evaluation) each key tile is reused by QG queries per MMA.
#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

namespace {

constexpr int kStages = 4;
constexpr int kTileM = 128;
constexpr int kTileBytes = kTileM * 128 * 2;  // bf16 [128][128] as two 64-wide swizzled panels
constexpr int kPanelBytes = kTileBytes / 2;
constexpr int kF8Bytes = kTileM * 64;         // raw E4M3 half-tile
constexpr int kMaxGroups = 4;                 // epilogue groups of four warps (at most)
// bf16 keys: four groups, each with its own TMEM accumulator of <= 128
// columns; E4M3 keys: two groups (the converter warps need the registers)
template <bool kFp8>
struct Roles {
  static constexpr int kGroups = kFp8 ? 2 : 4;
  static constexpr int kConv0 = 2 + 4 * kGroups;  // first FP8 converter warp
  static constexpr int kThreads = 32 * kConv0 + (kFp8 ? 128 : 0);
};

struct TcParams {
  int B, Q, H, N;
  int QG, n_groups, n_tiles;
  int NM;             // MMA N = QG*H
  int cols_per_acc;   // TMEM columns per accumulator
  int n_acc;          // accumulators = epilogue groups in use (2 or 4)
  uint32_t tmem_cols;
  long long units;
  int64_t key_batch_rows;
  float *scores;
  int64_t ld_scores;
  const float *w;
  const uint8_t *scale;
  int64_t ld_scale;
  uint32_t *stats;    // optional score bounds per span of 32 entries
  int n_spans;
  const int32_t *n_visible;  // optional causal entry mask [B][Q]
  uint32_t *status;
};

struct __align__(8) TcBarriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t conv[kStages];
  uint64_t tfull[kMaxGroups];
  uint64_t tempty[kMaxGroups];
  uint64_t bfull;
  uint64_t bempty;
  uint32_t tmem_base;
  uint32_t abort;
};

__host__ __device__ constexpr size_t tc_smem_bytes(int NM, bool fp8) {
  return 1024 + static_cast<size_t>(kStages) * kTileBytes + 2ull * NM * 128 + (fp8 ? kStages * kF8Bytes : 0) +
         kMaxGroups * 256 * sizeof(float) + sizeof(TcBarriers);
}

// Coordinates (sequence b, query group g, key tile t; bg = b * n_groups + g)
// of consecutive units, t fastest.  Only `init` divides: 64-bit divisions are
// long software sequences, too slow to repeat per tile in the pipeline roles.
struct UnitCursor {
  int b, g, t;
  long long bg;
  __device__ __forceinline__ void init(const TcParams &p, long long u) {
    bg = u / p.n_tiles;
    t = static_cast<int>(u % p.n_tiles);
    b = static_cast<int>(bg / p.n_groups);
    g = static_cast<int>(bg % p.n_groups);
  }
  __device__ __forceinline__ void next(const TcParams &p) {
    if (++t == p.n_tiles) {
      t = 0;
      ++bg;
      if (++g == p.n_groups) {
        g = 0;
        ++b;
      }
    }
  }
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

template <bool kFp8>
__global__ void __launch_bounds__(Roles<kFp8>::kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_rope,
                    const __grid_constant__ CUtensorMap tm_q, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + kStages * kTileBytes;
  uint8_t *sF8 = sB + 2 * p.NM * 128;
  float *sW = reinterpret_cast<float *>(sF8 + (kFp8 ? kStages * kF8Bytes : 0));
  TcBarriers *bar = reinterpret_cast<TcBarriers *>(sW + kMaxGroups * 256);
  volatile uint32_t *abort_flag = &bar->abort;
  constexpr int kConvWarp0 = Roles<kFp8>::kConv0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long u0 = blockIdx.x * p.units / gridDim.x, u1 = (blockIdx.x + 1) * p.units / gridDim.x;

  // Key tiles of the first kStages units: cache-side data, issued before the
  // block sync and before waiting for the previous kernel on the stream.
  const long long n_pre = min(static_cast<long long>(kStages), u1 - u0);
  auto issue_a = [&](const UnitCursor &c, int stage) {
    const int row = static_cast<int>(c.b * p.key_batch_rows + static_cast<int64_t>(c.t) * kTileM);
    uint8_t *a = sA + stage * kTileBytes;
    if (kFp8) {
      tc::mbar_arrive_expect_tx(&bar->full[stage], kF8Bytes + kPanelBytes);
      tc::tma_load_2d(sF8 + stage * kF8Bytes, &tm_a, &bar->full[stage], 0, row);
      tc::tma_load_2d(a + kPanelBytes, &tm_rope, &bar->full[stage], 0, row);
    } else {
      tc::mbar_arrive_expect_tx(&bar->full[stage], kTileBytes);
      tc::tma_load_2d(a, &tm_a, &bar->full[stage], 0, row);
      tc::tma_load_2d(a + kPanelBytes, &tm_a, &bar->full[stage], 64, row);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; s++) {
      tc::mbar_init(&bar->full[s], 1);
      tc::mbar_init(&bar->empty[s], 1);
      tc::mbar_init(&bar->conv[s], 128);
    }
    for (int a = 0; a < kMaxGroups; a++) {
      tc::mbar_init(&bar->tfull[a], 1);
      tc::mbar_init(&bar->tempty[a], 4);
    }
    tc::mbar_init(&bar->bfull, 1);
    tc::mbar_init(&bar->bempty, 1);
    bar->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_a);
    tc::tma_prefetch_desc(&tm_q);
    if (kFp8) tc::tma_prefetch_desc(&tm_rope);
    UnitCursor c;
    c.init(p, u0);
    for (long long i = 0; i < n_pre; i++, c.next(p)) issue_a(c, static_cast<int>(i));
  }
  if (warp == 1) tc::tmem_alloc(&bar->tmem_base, p.tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t bempty_par = 0;
      uint32_t last_par[kStages];
      bool used[kStages] = {};
      for (long long i = 0; i < n_pre; i++) {
        last_par[i] = 0;
        used[i] = true;
      }
      int stage = static_cast<int>(n_pre % kStages);
      uint32_t phase = n_pre == kStages ? 1u : 0u;
      bool b_loaded = false;
      uint32_t bfull_last = 0;
      long long prev_bg = -1;
      pdl_wait();  // queries and weights may come from the previous kernel
      UnitCursor c;
      c.init(p, u0);
      for (long long u = u0; u < u1; u++, c.next(p)) {
        const int b = c.b, g = c.g;
        const long long bg = c.bg;
        if (bg != prev_bg) {
          if (prev_bg != -1) {
            if (!tc::mbar_wait(&bar->bempty, bempty_par, abort_flag)) break;
            bempty_par ^= 1;
            bfull_last ^= 1;
          }
          const int qrow = (b * p.Q + g * p.QG) * p.H;
          tc::mbar_arrive_expect_tx(&bar->bfull, 2 * p.NM * 128);
          tc::tma_load_2d(sB, &tm_q, &bar->bfull, 0, qrow);
          tc::tma_load_2d(sB + p.NM * 128, &tm_q, &bar->bfull, 64, qrow);
          b_loaded = true;
          prev_bg = bg;
        }
        if (u - u0 < n_pre) continue;  // key tile already in flight
        if (!tc::mbar_wait(&bar->empty[stage], phase ^ 1, abort_flag)) break;
        issue_a(c, stage);
        last_par[stage] = phase;
        used[stage] = true;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      // never leave with copies in flight: wait (bounded) for every issued load
      volatile uint32_t no_abort = 0;
      for (int s = 0; s < kStages; s++)
        if (used[s]) tc::mbar_wait(&bar->full[s], last_par[s], &no_abort);
      if (b_loaded) tc::mbar_wait(&bar->bfull, bfull_last, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_par = 0, bfull_par = 0;
      long long prev_bg = -1;
      const uint32_t idesc = tc::idesc_bf16(kTileM, kFp8 ? p.H : p.NM);
      const uint32_t a_base = tc::smem_u32(sA), b_base = tc::smem_u32(sB);
      UnitCursor c;
      c.init(p, u0);
      for (long long u = u0; u < u1; u++, c.next(p)) {
        const long long bg = c.bg;
        if (bg != prev_bg) {
          if (prev_bg != -1) tc::mma_commit(&bar->bempty);
          if (!tc::mbar_wait(&bar->bfull, bfull_par, abort_flag)) break;
          bfull_par ^= 1;
          prev_bg = bg;
        }
        if (!tc::mbar_wait(kFp8 ? &bar->conv[stage] : &bar->full[stage], phase, abort_flag)) break;
        if (!tc::mbar_wait(&bar->tempty[acc], acc_par ^ 1, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + acc * p.cols_per_acc;
        const uint32_t a = a_base + stage * kTileBytes;
        if (kFp8) {
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            tc::mma_bf16(d, tc::desc_kmajor_sw128(a + kk * 32), tc::desc_kmajor_sw128(b_base + kk * 32), idesc, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            tc::mma_bf16(d + p.H, tc::desc_kmajor_sw128(a + kPanelBytes + kk * 32),
                         tc::desc_kmajor_sw128(b_base + p.NM * 128 + kk * 32), idesc, kk > 0);
        } else {
#pragma unroll
          for (int k = 0; k < 8; k++) {
            const uint32_t ao = (k >> 2) * kPanelBytes + (k & 3) * 32;
            const uint32_t bo = (k >> 2) * p.NM * 128 + (k & 3) * 32;
            tc::mma_bf16(d, tc::desc_kmajor_sw128(a + ao), tc::desc_kmajor_sw128(b_base + bo), idesc, k > 0);
          }
        }
        tc::mma_commit(&bar->empty[stage]);
        tc::mma_commit(&bar->tfull[acc]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (++acc == p.n_acc) {
          acc = 0;
          acc_par ^= 1;
        }
      }
    }
  } else if (warp < kConvWarp0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int grp = (warp - 2) >> 2;             // takes units u0 + grp, u0 + grp + n_acc, ...
    const int etid = threadIdx.x - 64 - 128 * grp;
    const int G = p.n_acc;
    float *gW = sW + grp * 256;                   // this group's head weights
    pdl_wait();  // head weights may come from the previous kernel
    const int acc = grp;
    uint32_t acc_par = 0;
    long long prev_bg = -1;
    // E4M3 block scales of this thread's key row, loaded two units ahead so
    // that their latency hides behind the tiles in between
    auto load_scale = [&](const UnitCursor &cu, bool valid) -> float {
      if (!kFp8 || !valid) return 0.f;
      const int j = cu.t * kTileM + row;
      return j < p.N ? e8m0_to_f32(p.scale[(cu.b * p.key_batch_rows + j) * p.ld_scale]) : 0.f;
    };
    auto step = [&](UnitCursor &cu) {
      for (int i = 0; i < G; i++) cu.next(p);
    };
    UnitCursor cs;  // runs two of this group's units ahead of the tile being reduced
    cs.init(p, u0 + grp);
    float sc_next0 = load_scale(cs, u0 + grp < u1);
    step(cs);
    float sc_next1 = load_scale(cs, u0 + grp + G < u1);
    step(cs);
    // Score bounds of this warp's 32 keys of a tile (one span record), for the
    // top-k: the largest and the smallest non-NaN order key.  Called by whole
    // warps.
    auto span_stats = [&](float sv, bool valid, int srow, int t) {
      const uint32_t kk = valid ? order_key(sv) : 0u;
      const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, kk);
      const uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, kk ? kk : 0xFFFFFFFFu);
      const int j0 = t * kTileM + quarter * 32;
      if (lane == 0 && j0 < p.N)
        reinterpret_cast<uint2 *>(p.stats)[static_cast<size_t>(srow) * p.n_spans + j0 / 32] = make_uint2(mx, mn);
    };
    UnitCursor c;
    c.init(p, u0 + grp);
    if (grp >= G) c.init(p, u1);  // an idle group (two accumulators in use)
    for (long long u = u0 + grp; grp < G && u < u1; u += G, step(c)) {
      const int b = c.b, g = c.g, t = c.t;
      const long long bg = c.bg;
      const float sc = sc_next0;
      sc_next0 = sc_next1;
      sc_next1 = load_scale(cs, u + 2 * G < u1);
      step(cs);
      if (bg != prev_bg) {
        named_sync(2 + grp, 128);
        const int nq = min(p.QG, p.Q - g * p.QG);
        for (int i = etid; i < p.QG * p.H; i += 128)
          gW[i] = (i / p.H) < nq ? p.w[static_cast<int64_t>(b * p.Q + g * p.QG) * p.H + i] : 0.f;
        named_sync(2 + grp, 128);
        prev_bg = bg;
      }
      // lane 0 waits, the warp follows its verdict; after a give-up the
      // warp keeps walking the units (skipping the work) so the named
      // barriers above stay matched
      bool ready = false;
      if (lane == 0) ready = tc::mbar_wait(&bar->tfull[acc], acc_par, abort_flag);
      ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
      if (ready) {
        tc::tc_fence_after();
        const uint32_t base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * p.cols_per_acc;
        const int j = t * kTileM + row;
        float v[32], r[32];
        if (kFp8) {
          float s = 0.f;
          for (int c0 = 0; c0 < p.H; c0 += 32) {
            tc::tmem_ld32(base + c0, v);
            tc::tmem_ld32(base + p.H + c0, r);
#pragma unroll
            for (int i = 0; i < 32; i++) s = fmaf(gW[c0 + i], fmaxf(fmaf(sc, v[i], r[i]), 0.f), s);
          }
          if (p.n_visible && j >= __ldg(p.n_visible + b * p.Q + g)) s = -INFINITY;
          if (j < p.N) p.scores[static_cast<int64_t>(b * p.Q + g) * p.ld_scores + j] = s;
          if (p.stats) span_stats(s, j < p.N, b * p.Q + g, t);
        } else {
          // The QG x H accumulator columns in chunks of 32, two register
          // buffers deep: chunk c+1 loads from TMEM while chunk c is reduced.
          // A query's score is complete after its last chunk.
          const int nch = (p.QG * p.H) >> 5;
          uint32_t ra[32], rb[32];
          float s = 0.f;
          auto reduce = [&](const uint32_t (&rr)[32], int c) {
            const float4 *w4 = reinterpret_cast<const float4 *>(gW + 32 * c);
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const float4 wv = w4[i];
              s4[0] = fmaf(wv.x, fmaxf(__uint_as_float(rr[4 * i + 0]), 0.f), s4[0]);
              s4[1] = fmaf(wv.y, fmaxf(__uint_as_float(rr[4 * i + 1]), 0.f), s4[1]);
              s4[2] = fmaf(wv.z, fmaxf(__uint_as_float(rr[4 * i + 2]), 0.f), s4[2]);
              s4[3] = fmaf(wv.w, fmaxf(__uint_as_float(rr[4 * i + 3]), 0.f), s4[3]);
            }
            s += (s4[0] + s4[1]) + (s4[2] + s4[3]);
            if (((c + 1) << 5) % p.H == 0) {  // last chunk of query qi
              const int qq = g * p.QG + ((c << 5) / p.H);
              if (p.n_visible && qq < p.Q && j >= __ldg(p.n_visible + b * p.Q + qq)) s = -INFINITY;
              if (j < p.N && qq < p.Q) p.scores[static_cast<int64_t>(b * p.Q + qq) * p.ld_scores + j] = s;
              if (p.stats && qq < p.Q) span_stats(s, j < p.N, b * p.Q + qq, t);
              s = 0.f;
            }
          };
          // the accumulator is free once its last chunk is in registers:
          // hand it back to the MMA before that chunk is reduced
          auto release = [&]() {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar->tempty[acc]);
          };
          tc::tmem_ld32_issue(base, ra);
          for (int c = 0; c < nch; c += 2) {
            tc::tmem_ld_wait();
            tc::tmem_ld32_pin(ra);
            if (c + 1 < nch) tc::tmem_ld32_issue(base + 32 * (c + 1), rb);
            else release();
            reduce(ra, c);
            if (c + 1 < nch) {
              tc::tmem_ld_wait();
              tc::tmem_ld32_pin(rb);
              if (c + 2 < nch) tc::tmem_ld32_issue(base + 32 * (c + 2), ra);
              else release();
              reduce(rb, c + 1);
            }
          }
        }
      }
      if (kFp8 || !ready) {  // (the bf16 path released the accumulator above)
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0 && ready) tc::mbar_arrive(&bar->tempty[acc]);
      }
      acc_par ^= 1;
    }
  } else if (kFp8) {
    // ------------------------------------------------------------ FP8 -> bf16
    // Pass i: thread t converts codes [16(t%4), +16) of row 32i + t/4, so
    // each 8-lane phase reads 128 contiguous bytes of the raw half-tile and
    // writes 8 distinct 16-byte slots of the swizzled panel (no bank
    // conflicts either way).
    const int t = threadIdx.x - 32 * kConvWarp0;
    int stage = 0;
    uint32_t phase = 0;
    for (long long u = u0; u < u1; u++) {
      if (!tc::mbar_wait(&bar->full[stage], phase, abort_flag)) break;
      const uint8_t *src = sF8 + stage * kF8Bytes;
      uint8_t *dst = sA + stage * kTileBytes;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int r = 32 * i + (t >> 2), c = t & 3;
        const uint4 x = *reinterpret_cast<const uint4 *>(src + r * 64 + c * 16);
        const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; k++) o[k] = e4m3x2_to_bf16x2(wv[k >> 1] >> (16 * (k & 1)));
        uint8_t *drow = dst + r * 128;
        *reinterpret_cast<uint4 *>(drow + (((2 * c) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(drow + (((2 * c + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar->conv[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, p.tmem_cols);
  }
  if (threadIdx.x == 0 && bar->abort) raise_status(p.status, LIDX_DEV_TIMEOUT);
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

int choose_qg(const lidx_score_args &a) {
  if (a.keys.dtype == LIDX_E4M3) return 1;
  return std::max(1, std::min(a.Q, 128 / a.H));  // <= 128 columns: four accumulators fit TMEM
}

}  // namespace

bool score_tc_supported(const lidx_score_args &a) {
  if (a.q_dtype != LIDX_BF16) return false;
  if (a.keys.dtype != LIDX_BF16 && a.keys.dtype != LIDX_E4M3) return false;
  if (a.H % 32 != 0) return false;
  if (a.keys.dtype == LIDX_E4M3 ? a.H > 128 : a.H > 256) return false;
  const int64_t rows = static_cast<int64_t>(a.B - 1) * a.keys.batch_rows + a.N;
  if (rows >= (1ll << 31) || static_cast<int64_t>(a.B) * a.Q * a.H >= (1ll << 31)) return false;
  return true;
}

cudaError_t launch_score_tc(const lidx_score_args &a, cudaStream_t st) {
  const bool fp8 = a.keys.dtype == LIDX_E4M3;
  TcParams p{};
  p.B = a.B;
  p.Q = a.Q;
  p.H = a.H;
  p.N = a.N;
  p.QG = choose_qg(a);
  p.n_groups = (a.Q + p.QG - 1) / p.QG;
  p.n_tiles = (a.N + kTileM - 1) / kTileM;
  p.NM = p.QG * a.H;
  p.cols_per_acc = fp8 ? 2 * a.H : p.NM;
  p.n_acc = (!fp8 && p.cols_per_acc <= 128) ? 4 : 2;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.n_acc * p.cols_per_acc)) cols <<= 1;
  p.tmem_cols = cols;
  p.units = static_cast<long long>(a.B) * p.n_groups * p.n_tiles;
  p.key_batch_rows = a.B > 1 ? a.keys.batch_rows : a.N;
  p.scores = a.scores;
  p.ld_scores = a.ld_scores;
  p.w = a.w;
  p.scale = a.keys.scale;
  p.ld_scale = a.keys.ld_scale;
  p.stats = a.tile_stats;
  p.n_spans = (a.N + LIDX_STATS_SPAN - 1) / LIDX_STATS_SPAN;
  p.n_visible = a.n_visible;
  p.status = nullptr;

  const uint64_t rows = static_cast<uint64_t>(a.B - 1) * p.key_batch_rows + a.N;
  CUtensorMap tm_a, tm_rope, tm_q;
  bool ok;
  if (fp8) {
    ok = make_tmap_2d(&tm_a, a.keys.data, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, rows, a.keys.ld, 64, kTileM,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_tmap_2d(&tm_rope, a.keys.rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, rows, a.keys.ld_rope * 2, 64,
                      kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    ok = make_tmap_2d(&tm_a, a.keys.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, rows, a.keys.ld * 2, 64, kTileM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    tm_rope = tm_a;
  }
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.Q * a.H;
  ok = ok && make_tmap_2d(&tm_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, qrows, 256, 64, p.NM,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;

  const size_t smem = tc_smem_bytes(p.NM, fp8);
  const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
  const int grid = static_cast<int>(std::min<long long>(p.units, sm_count()));
  if (fp8) {
    cudaFuncSetAttribute(score_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    return launch_kernel(score_tc_kernel<true>, dim3(grid), dim3(Roles<true>::kThreads), smem, st, pdl, tm_a,
                         tm_rope, tm_q, p);
  } else {
    cudaFuncSetAttribute(score_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    return launch_kernel(score_tc_kernel<false>, dim3(grid), dim3(Roles<false>::kThreads), smem, st, pdl, tm_a,
                         tm_rope, tm_q, p);
  }
}

}  // namespace lidx
