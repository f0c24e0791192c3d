// One CSA decode layer in a single persistent launch (DeepSeek-V4-Flash
// architecture post, section (B)): the lightning indexer scores every
// compressed entry, the top k are kept, and MQA attention reads those 512-wide
// rows plus the sliding window.  The three steps are chained inside one grid
// of at most one CTA per SM, so a layer costs one launch instead of four and
// no step waits for a kernel boundary.
//
// Work units, in one global order (unit u runs on CTA u mod G, each CTA takes
// its units in increasing u, and a unit only ever waits for units before it
// or, in the merge, for units of its own attention group, which all run at
// once because every CTA holds at most one attention unit):
//   score  (b, tile)    128 keys x H heads on tcgen05 (M = 128 keys, N = H,
//                       K = 128), TMA key and query tiles; the epilogue
//                       reduces sum_h w_h max(x, 0) per key, stores the
//                       scores, folds the row's largest and smallest
//                       order-preserving key into two words by atomics, and
//                       counts the tile done (release)
//   select (b)          waits for the row's tiles (acquire), copies the
//                       row into shared memory with one bulk copy, then
//                       selects the k largest exactly in one CTA: a 2048-bin
//                       histogram linear in value over the row's [min, max],
//                       a suffix scan to the bin holding the k-th key, rank
//                       counting among that bin's keys (or key-space
//                       histogram levels, and an index scan for ties), and a
//                       prefix scan that writes
//                       the ids in ascending order (and starts an L2 prefetch
//                       of each selected row); then it raises the row's
//                       ready flag (release)
//   attn   (b, c, hg)   64 entries of the row list (window rows first, then
//                       the selected ids) x 16 of the 64 heads: rows by TMA
//                       (window) or cp.async gather (selected, after the
//                       ready flag), S^T = X Q^T and O^T = X^T P^T on tcgen05
//                       with P carried as bf16 hi + lo, a split partial
//                       (m, l, O); then the group's CTAs wait for each other
//                       and each merges a slice of the 16 x 512 outputs.
// Score CTAs that finish early pull the next layer's cache-side inputs
// (index keys, window rows) into L2.  Every cross-CTA wait is bounded by
// %globaltimer and sets LIDX_DEV_TIMEOUT when it gives up; the last CTA to
// leave zeroes the control words, so the workspace is ready for the next
// call.
#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kTileM = 128;                    // keys per score tile
constexpr int kKeyStage = kTileM * 128 * 2;    // bf16 [128][128] as two swizzled 64-dim panels
constexpr int kKeyPanel = kKeyStage / 2;
constexpr int kNB = 2048;                      // selector histogram bins
constexpr int kCandMax = 1024;                 // candidates resolved by rank counting
// attention
constexpr int kD = 512;
constexpr int kHA = 64;                        // attention heads
constexpr int kHG = 16;                        // heads per attention unit
constexpr int kRows = 64;                      // row-list entries per attention unit
constexpr int kXBytes = kRows * kD * 2;        // 64 KB: 8 panels of [64 rows][128 B]
constexpr int kXPanel = kRows * 128;
constexpr int kQBytes = kHG * kD * 2;          // 16 KB
constexpr int kQPanel = kHG * 128;
constexpr int kPBytes = kHG * kRows * 2;       // 2 KB per P^T part
constexpr int kS1 = 4;                         // MMA 1 issuers (K quarters)
constexpr uint32_t kOCol = 64;
constexpr uint32_t kTmemCols = 256;
constexpr float kLog2e = 1.4426950408889634f;
// control words of sequence b: ctl[b * kCtlStride + ...]
constexpr int kCtlStride = 16;
constexpr int kCtlTiles = 2, kCtlReady = 3, kCtlAttn = 4;  // kCtlAttn + hg
constexpr int kCtlCand = 9;   // score units that published their candidates
constexpr int kCtlCandN = 10; // candidates in the row's list
constexpr int kCtlMode = 11;  // kModeSplit: the score units select; kModeOneCta: the selector unit does
constexpr int kCtlNeed = 12;  // rank (1-based) of the last taken candidate
constexpr int kCtlAll = 13;   // at most k keys are eligible: all are taken
constexpr uint32_t kModeSplit = 1, kModeOneCta = 2;
constexpr int kMaxOwnTiles = 4;   // score units per CTA
constexpr int kCandSplit = 512;   // largest fine bin the split selection ranks
constexpr int kNB1 = 256;         // coarse histogram bins (top 8 key bits)
constexpr int kNB2 = 65536;       // fine histogram bins (top 16 key bits): 256 under each coarse bin
// smem map (offsets from the 1024-aligned base)
constexpr int kSmKeys = 0;                     // score: two key stages
constexpr int kSmQidx = 2 * kKeyStage;         // score: query tile, up to 128 heads
constexpr int kSelItems = 32;                 // row positions per selector thread
constexpr int kSmRowMax = kSelItems * kThreads * 4 / 32 * 36;  // the staged row, 4 pad words per 32 scores
constexpr int kSmX = 0, kSmQa = kXBytes, kSmP = kXBytes + kQBytes;  // attention
constexpr int kSmHist = 0, kSmCand = kNB * 4, kSmRow = kSmCand + kCandMax * 8;  // select: the row at kSmRow
constexpr int kSmData = (kSmQidx + 128 * 256) > (kSmRow + kSmRowMax) ? (kSmQidx + 128 * 256) : (kSmRow + kSmRowMax);

struct __align__(8) Ctl {
  uint64_t key_full[2];
  uint64_t q_full;
  uint64_t mma_done;
  uint64_t a_full;
  uint64_t s_full;
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t bc[8];         // values broadcast through shared memory
  uint32_t wsum[kWarps];  // per-warp partial sums of the block scans
  uint32_t wlo[kWarps], whi[kWarps];  // per-warp key bounds of the selector
  float tile_x[kMaxOwnTiles][kTileM];  // this CTA's score units: their scores (NaN: none)
  uint32_t h1[kNB1];                   // a tile's coarse histogram, added to the row's in one go
  uint32_t ctile[kTileM];              // split view: per tile, candidates taken
  uint32_t toff[kTileM + 1];           // split view: per tile, offset in the id list
  int32_t chunk_id[kRows];             // attention: the ids of the chunk's selected rows
  float w[128];           // head weights of the query tile
  int64_t row_src[kRows];
  int32_t row_kind[kRows];
  float red[2][4][8];
};

constexpr size_t smem_bytes() { return 1024 + kSmData + sizeof(Ctl); }
static_assert(kSmP + 2 * kPBytes <= kSmData, "attention operands fit the data region");
constexpr int kSmSplit = kSmP + 2 * kPBytes;  // split view: the candidates (beside the attention operands)
static_assert(kSmSplit + kCandSplit * 8 <= kSmData, "split view scratch fits the data region");
static_assert(kSmRow + kSmRowMax <= kSmData, "selector buffers and the staged row fit the data region");

struct FusedParams {
  int B, H, N, k, swa_len;
  int n_tiles, n_chunks, n_score, n_attn, G;
  int64_t key_batch_rows;
  const float *w;
  const uint16_t *kv;     // bf16 rows
  int64_t kv_ld, kv_batch_rows;
  const uint16_t *swa;
  int64_t swa_ld, swa_batch_rows;
  float scale;
  float *out, *lse;
  float *scores_user;
  int64_t ld_user;
  int32_t *ids_user, *n_sel_user;
  uint32_t *status, *ctl;
  float *scores;          // workspace copy, row stride ld_ws
  uint32_t *hist2;        // per sequence: kNB2-bin fine histogram (cleared by the score units)
  uint32_t *above;        // per score tile: its scores taken without ranking
  uint2 *gcand;           // per sequence: kCandSplit (key, position) candidates of the threshold bin
  uint32_t *hist;         // per sequence: kNB1-bin coarse histogram of the score keys (cleared by the score units)
  int64_t ld_ws;
  int32_t *sel_ids, *sel_n;
  float *part_o;
  float2 *part_ml;
  const uint8_t *pf[2];
  uint64_t pf_bytes[2];
  uint64_t wait_ns;
  uint32_t lost_arrival;  // test hook: score unit 0 withholds its count
};

// ------------------------------------------------------------ sync helpers
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Count one arrival after the whole CTA's prior writes (called by one thread
// after a block barrier: the fence is cumulative over what the barrier ordered).
__device__ __forceinline__ void arrive_release(uint32_t *p, uint32_t n = 1u) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(n) : "memory");
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait until *p >= target (acquire); false when `limit_ns` passed first.
// Polls with a short sleep and reads the clock every 16 polls, so that many
// waiting CTAs put little load on the memory system.
__device__ __noinline__ bool wait_geq(const uint32_t *p, uint32_t target, uint64_t limit_ns) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; i++) {
    __nanosleep(32);
    if (ld_acquire(p) >= target) return true;
    if ((i & 15u) == 0 && globaltimer() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint32_t x_off(int r, int c) {
  return (c >> 3) * kXPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Exclusive prefix over the block of one count per thread; also returns the
// block total.  Every thread must call it (two block barriers).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t &total, Ctl *c) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t incl = warp_inclusive_scan(v);
  if (lane == 31) c->wsum[warp] = incl;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kWarps; i++) {
    const uint32_t x = c->wsum[i];
    base += i < warp ? x : 0u;
    tot += x;
  }
  __syncthreads();  // wsum is reused by the next scan
  total = tot;
  return base + incl - v;
}

// ------------------------------------------------------------------ score
__device__ void issue_key_tile(const FusedParams &p, const CUtensorMap *tm, uint8_t *sm, Ctl *c, int u, int stage) {
  const int b = u / p.n_tiles, t = u % p.n_tiles;
  const int row = static_cast<int>(b * p.key_batch_rows + static_cast<int64_t>(t) * kTileM);
  uint8_t *dst = sm + kSmKeys + stage * kKeyStage;
  tc::mbar_arrive_expect_tx(&c->key_full[stage], kKeyStage);
  tc::tma_load_2d(dst, tm, &c->key_full[stage], 0, row);
  tc::tma_load_2d(dst + kKeyPanel, tm, &c->key_full[stage], 64, row);
}

// Bounded wait for the phase with `parity` of a barrier whose copies may still
// be in flight (used before shared memory is reused after a give-up).
__device__ __forceinline__ void drain(uint64_t *bar, uint32_t parity) {
  volatile uint32_t no_abort = 0;
  tc::mbar_wait(bar, parity, &no_abort);
}

__device__ void score_units(const FusedParams &p, const CUtensorMap *tm_keys, const CUtensorMap *tm_q, uint8_t *sm,
                            Ctl *c, uint32_t tmem, bool &abort) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  // key tiles thread 0 has issued per stage (two in the prologue)
  uint32_t issued[2] = {blockIdx.x < static_cast<unsigned>(p.n_score) ? 1u : 0u,
                        blockIdx.x + p.G < static_cast<unsigned>(p.n_score) ? 1u : 0u};
  uint32_t q_loads = 0;
  int q_b = -1;
  for (int i = 0;; i++) {
    const int u = blockIdx.x + i * p.G;
    if (u >= p.n_score) break;
    const int b = u / p.n_tiles, t = u % p.n_tiles;
    const int stage = i & 1;
    if (b != q_b) {  // query tile and head weights of sequence b
      if (tid == 0) {
        tc::mbar_arrive_expect_tx(&c->q_full, H * 256);
        tc::tma_load_2d(sm + kSmQidx, tm_q, &c->q_full, 0, b * H);
        tc::tma_load_2d(sm + kSmQidx + H * 128, tm_q, &c->q_full, 64, b * H);
      }
      for (int h = tid; h < H; h += kThreads) c->w[h] = p.w[static_cast<int64_t>(b) * H + h];
      q_b = b;
      q_loads++;
      __syncthreads();
    }
    if (tid == 32) {
      volatile uint32_t *ab = &c->abort;
      if (tc::mbar_wait(&c->key_full[stage], (i >> 1) & 1, ab) && tc::mbar_wait(&c->q_full, (q_loads - 1) & 1, ab)) {
        tc::tc_fence_after();
        const uint32_t idesc = tc::idesc_bf16(kTileM, H);
        const uint32_t a = tc::smem_u32(sm + kSmKeys + stage * kKeyStage), bq = tc::smem_u32(sm + kSmQidx);
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t ao = (k >> 2) * kKeyPanel + (k & 3) * 32;
          const uint32_t bo = (k >> 2) * H * 128 + (k & 3) * 32;
          tc::mma_bf16(tmem, tc::desc_kmajor_sw128(a + ao), tc::desc_kmajor_sw128(bq + bo), idesc, k > 0);
        }
      }
      tc::mma_commit(&c->mma_done);  // arrives even when nothing was issued
    }
    if (warp >= 4 && warp < 8) {
      const int quarter = warp & 3, row = quarter * 32 + lane;
      const int j = t * kTileM + row;
      bool ready = false;
      if (lane == 0) ready = tc::mbar_wait(&c->mma_done, i & 1, &c->abort);
      ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
      float s = 0.f;
      if (ready) {
        tc::tc_fence_after();
        const uint32_t base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        // per 32 heads four partial sums, folded into s chunk by chunk: the
        // same order as lidx_index_score, so both give identical scores
        for (int c0 = 0; c0 < H; c0 += 32) {
          float v[32];
          tc::tmem_ld32(base + c0, v);
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 32; h++) s4[h & 3] = fmaf(c->w[c0 + h], fmaxf(v[h], 0.f), s4[h & 3]);
          s += (s4[0] + s4[1]) + (s4[2] + s4[3]);
        }
      }
      const bool in = j < p.N;
      if (in) {
        p.scores[static_cast<int64_t>(b) * p.ld_ws + j] = s;
        if (p.scores_user) p.scores_user[static_cast<int64_t>(b) * p.ld_user + j] = s;
      }
      // the row's two key histograms (0 = no score: NaN, or past N)
      const uint32_t kk = in ? order_key(s) : 0u;
      if (__any_sync(0xFFFFFFFFu, in && kk == 0u) && lane == 0) raise_status(p.status, LIDX_DEV_NAN);
      {  // one add per distinct bin of the warp (the scores crowd a few bins)
        const uint32_t m1 = __match_any_sync(0xFFFFFFFFu, kk ? kk >> 24 : 0xFFFFFFFFu);
        const uint32_t m2 = __match_any_sync(0xFFFFFFFFu, kk ? kk >> 16 : 0xFFFFFFFFu);
        if (kk && lane == __ffs(m1) - 1) atomicAdd(&c->h1[kk >> 24], static_cast<uint32_t>(__popc(m1)));
        if (kk && lane == __ffs(m2) - 1)
          atomicAdd(p.hist2 + static_cast<int64_t>(b) * kNB2 + (kk >> 16), static_cast<uint32_t>(__popc(m2)));
      }
      if (i < kMaxOwnTiles) c->tile_x[i][row] = in ? s : NAN;
    }
    tc::tc_fence_before();
    __syncthreads();
    if (c->abort) abort = true;
    // the tile's coarse histogram into the row's (every tile crowds the same
    // few coarse bins: one add per bin and tile)
    if (tid < kNB1) {
      const uint32_t n = c->h1[tid];
      if (n) {
        atomicAdd(p.hist + b * kNB1 + tid, n);
        c->h1[tid] = 0u;
      }
    }
    __syncthreads();
    if (tid == 0) {
      const int un = u + 2 * p.G;  // the stage is free: fetch the unit after next
      if (un < p.n_score) {
        issue_key_tile(p, tm_keys, sm, c, un, stage);
        issued[stage]++;
      }
      if (!(p.lost_arrival && u == 0)) arrive_release(p.ctl + b * kCtlStride + kCtlTiles);
    }
  }
  if (tid == 0 && c->abort) {  // a wait gave up: let every issued copy land first
    for (int st = 0; st < 2; st++)
      if (issued[st]) drain(&c->key_full[st], (issued[st] - 1) & 1);
    if (q_loads) drain(&c->q_full, (q_loads - 1) & 1);
  }
  __syncthreads();
}

// ----------------------------------------------------------------- select
// The k largest scores of a row are found by the score units together, with
// one wait between them:
//  * each score unit adds its tile's scores to two histograms of the row, of
//    the order-preserving keys' top 11 bits (kNB bins) and top 16 bits
//    (kNB2 bins; 32 fine bins under each coarse one), as it stores them;
//  * once every tile is scored, each unit finds the same fine bin f holding
//    the k-th largest key (coarse bin by a scan of the coarse histogram, then
//    the fine bin among its 32), publishes how many of its keys lie above f,
//    and appends its keys in f to the row's candidate list;
//  * once every unit has published, anyone who needs the selection ranks the
//    few candidates (key desc, index asc): the one of rank need-1 is the last
//    taken, (T_key, T_idx).  Entry j with key kk is taken iff kk > T_key or
//    (kk == T_key and j <= T_idx): keys above f exceed T_key, keys below f
//    fall short of it.  The per-tile counts give each tile's offset in the
//    ascending id list, so the attention units build their own chunks of it
//    and the score units write the caller's ids, with no further wait.
// When at most k keys are eligible all are taken.  A fine bin of more than
// kCandSplit keys (long runs of ties) leaves the row to the selector unit,
// which selects it alone (kModeOneCta).

// Bounded wait of the whole CTA for *w >= target; false (and abort) on expiry.
__device__ __forceinline__ bool block_wait(const FusedParams &p, const uint32_t *w, uint32_t target, Ctl *c,
                                           bool &abort) {
  if (threadIdx.x == 0) c->bc[0] = wait_geq(w, target, p.wait_ns) ? 1u : 0u;
  __syncthreads();
  const bool ok = c->bc[0] != 0;
  __syncthreads();  // bc[0] is reused
  if (!ok) {
    abort = true;
    if (threadIdx.x == 0) raise_status(p.status, LIDX_DEV_TIMEOUT);
  }
  return ok;
}

// block-wide min and max of (lo, hi) through the per-warp slots
__device__ __forceinline__ void block_minmax(uint32_t &lo, uint32_t &hi, Ctl *c) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  if (lane == 0) {
    c->wlo[warp] = lo;
    c->whi[warp] = hi;
  }
  __syncthreads();
  lo = __reduce_min_sync(0xFFFFFFFFu, c->wlo[lane & (kWarps - 1)]);
  hi = __reduce_max_sync(0xFFFFFFFFu, c->whi[lane & (kWarps - 1)]);
  __syncthreads();  // the slots are reused
}

// Suffix scan of hist (thread t holds bins kNB-1-4t .. kNB-4-4t) to the bin
// holding the need-th largest key: bc[2] = that bin, bc[3] = keys above it,
// bc[4] = keys in it; returns the histogram's total.
__device__ __forceinline__ uint32_t find_bin(const uint32_t *hist, uint32_t need, Ctl *c) {
  const int tid = threadIdx.x;
  uint32_t cnt[4], ct = 0;
#pragma unroll
  for (int j = 0; j < 4; j++) {
    cnt[j] = hist[kNB - 1 - (4 * tid + j)];
    ct += cnt[j];
  }
  uint32_t tot;
  uint32_t e = block_excl_scan(ct, tot, c);
  if (e < need && need <= e + ct) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
      if (e < need && need <= e + cnt[j]) {
        c->bc[2] = kNB - 1 - (4 * tid + j);
        c->bc[3] = e;
        c->bc[4] = cnt[j];
      }
      e += cnt[j];
    }
  }
  __syncthreads();
  return tot;
}

// Rank the nc candidates (key desc, index asc): bc[5], bc[6] = the key and
// index of rank need-1, the last selected entry.  g threads (a power of two,
// within a warp) share a candidate, each comparing it with every g-th other.
__device__ __forceinline__ void rank_pick(const uint2 *cand, uint32_t nc, uint32_t need, Ctl *c) {
  const int tid = threadIdx.x;
  uint32_t g = 1;
  while (g < 32 && 2 * g * nc <= static_cast<uint32_t>(kThreads)) g *= 2;
  const uint32_t per = static_cast<uint32_t>(kThreads) / g, sub = static_cast<uint32_t>(tid) % g;
  for (uint32_t c0 = 0; c0 < nc; c0 += per) {
    const uint32_t ci = c0 + static_cast<uint32_t>(tid) / g;
    uint32_t rank = 0;
    uint2 me = make_uint2(0u, 0u);
    if (ci < nc) {
      me = cand[ci];
      for (uint32_t cj = sub; cj < nc; cj += g) {
        const uint2 o = cand[cj];
        rank += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1u : 0u;
      }
    }
    for (uint32_t o = g / 2; o; o >>= 1) rank += __shfl_xor_sync(0xFFFFFFFFu, rank, o);
    if (ci < nc && sub == 0 && rank == need - 1) {
      c->bc[5] = me.x;
      c->bc[6] = me.y;
    }
  }
  __syncthreads();
}

// One warp: lane l holds the counts of bins [8l, 8l + 8) of a 256-bin
// histogram (h, ascending).  Finds the bin holding the need-th largest key:
// returns it, with the keys above it in `above` and in it in `in_bin`; the
// histogram's total in `total` (the search needs need <= total).
__device__ __forceinline__ uint32_t warp_find_bin(const uint32_t (&h)[8], uint32_t need, uint32_t &above,
                                                  uint32_t &in_bin, uint32_t &total) {
  const int lane = threadIdx.x & 31;
  uint32_t ls = 0;
#pragma unroll
  for (int j = 0; j < 8; j++) ls += h[j];
  uint32_t sfx = ls;  // keys in lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, sfx, o);
    if (lane + o < 32) sfx += y;
  }
  uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, sfx, 1);
  if (lane == 31) nxt = 0u;
  total = __shfl_sync(0xFFFFFFFFu, sfx, 0);
  uint32_t bin = 0, ab = nxt, in = 0;
  bool hit = false;
#pragma unroll
  for (int j = 7; j >= 0; j--) {
    if (!hit && ab + h[j] >= need) {
      hit = true;
      bin = 8 * lane + j;
      in = h[j];
    } else if (!hit) {
      ab += h[j];
    }
  }
  const uint32_t src = __ffs(__ballot_sync(0xFFFFFFFFu, sfx >= need && nxt < need)) - 1;
  above = __shfl_sync(0xFFFFFFFFu, ab, src);
  in_bin = __shfl_sync(0xFFFFFFFFu, in, src);
  return __shfl_sync(0xFFFFFFFFu, bin, src);
}

// The candidate step, for each score unit of this CTA once every tile of its
// row is scored (run after the CTA's last score unit, so the wait cannot hold
// back a tile; every CTA takes its units in the same order).  Warp 0 finds
// the coarse bin, then the fine bin f among the 256 under it.  The unit of
// tile 0 also publishes the row's mode, need and "all taken" flag.  A unit
// whose wait gave up still counts itself.
__device__ void cand_units(const FusedParams &p, uint8_t *sm, Ctl *c, bool &abort) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  (void)sm;
  for (int i = 0, u = blockIdx.x; u < p.n_score; i++, u += p.G) {
    const int b = u / p.n_tiles, t = u % p.n_tiles;
    uint32_t *ctl = p.ctl + b * kCtlStride;
    const bool ok = block_wait(p, ctl + kCtlTiles, p.n_tiles, c, abort);
    const uint32_t k = static_cast<uint32_t>(p.k);
    if (warp == 0) {
      uint32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.hist + b * kNB1 + 8 * lane);
        const uint4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
        h[0] = x0.x, h[1] = x0.y, h[2] = x0.z, h[3] = x0.w, h[4] = x1.x, h[5] = x1.y, h[6] = x1.z, h[7] = x1.w;
      }
      uint32_t above1, in1, total;
      uint32_t tot;
      uint32_t lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; j++) lsum += h[j];
      tot = __reduce_add_sync(0xFFFFFFFFu, lsum);
      const bool all = tot <= k;
      uint32_t f = 0, need = 0, in2 = 0;
      if (!all) {
        const uint32_t cb = warp_find_bin(h, k, above1, in1, total);
        const uint4 *src = reinterpret_cast<const uint4 *>(p.hist2 + static_cast<int64_t>(b) * kNB2 + cb * 256 + 8 * lane);
        const uint4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
        uint32_t g[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t above2, t2;
        const uint32_t need1 = k - above1;
        f = cb * 256 + warp_find_bin(g, need1, above2, in2, t2);
        need = need1 - above2;
      }
      if (lane == 0) {
        c->bc[1] = all ? 1u : 0u;
        c->bc[5] = f;
        c->bc[6] = need;
        c->bc[7] = in2;
      }
    }
    __syncthreads();
    const bool all = c->bc[1] != 0u;
    const uint32_t f = c->bc[5], need = c->bc[6];
    const bool split = all || c->bc[7] <= static_cast<uint32_t>(kCandSplit);
    if (split) {
      const float v = tid < kTileM ? c->tile_x[i][tid] : NAN;
      const uint32_t kk = tid < kTileM ? order_key(v) : 0u;
      const uint32_t fb = kk >> 16;
      const bool up = kk != 0u && (all || fb > f), cd = !all && kk != 0u && fb == f;
      // candidates: one slot range per warp
      const uint32_t cm = __ballot_sync(0xFFFFFFFFu, cd);
      uint32_t base = 0;
      if (lane == 0 && cm) base = atomicAdd(ctl + kCtlCandN, static_cast<uint32_t>(__popc(cm)));
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
      if (cd) {
        const uint32_t slot = base + __popc(cm & ((1u << lane) - 1u));
        if (slot < static_cast<uint32_t>(kCandSplit))
          p.gcand[b * kCandSplit + slot] = make_uint2(kk, static_cast<uint32_t>(t * kTileM + tid));
      }
      const uint32_t um = __ballot_sync(0xFFFFFFFFu, up);
      if (lane == 0) c->wsum[warp] = __popc(um);
    }
    __syncthreads();
    if (tid == 0) {
      if (split) {
        uint32_t n = 0;
        for (int w = 0; w < kTileM / 32; w++) n += c->wsum[w];
        p.above[u] = n;
      }
      if (t == 0) {  // ordered before the count by its fence
        ctl[kCtlMode] = split ? kModeSplit : kModeOneCta;
        ctl[kCtlNeed] = need;
        ctl[kCtlAll] = all ? 1u : 0u;
      }
      arrive_release(ctl + kCtlCand);
    }
    __syncthreads();
  }
}

// After the candidate step of row b (split mode): the threshold (T_key,
// T_idx), and per tile the offset of its first taken entry in the ascending
// id list (c->toff[0 .. n_tiles], the last being the number taken).  Every
// thread of the CTA calls it; the control words, the tiles' counts and the
// candidate slots are read in one round trip.  It uses the split scratch
// area of shared memory.
__device__ void split_view(const FusedParams &p, int b, uint8_t *sm, Ctl *c, uint32_t &T_key, uint32_t &T_idx) {
  const int tid = threadIdx.x;
  uint2 *cand = reinterpret_cast<uint2 *>(sm + kSmSplit);
  const uint32_t *ctl = p.ctl + b * kCtlStride;
  if (tid == 0) {
    const uint4 w8 = __ldcg(reinterpret_cast<const uint4 *>(ctl + 8)), w12 = __ldcg(reinterpret_cast<const uint4 *>(ctl + 12));
    c->bc[1] = min(w8.z, static_cast<uint32_t>(kCandSplit));  // kCtlCandN
    c->bc[2] = w12.x;                                          // kCtlNeed
    c->bc[3] = w12.y;                                          // kCtlAll
  }
  const uint32_t av = tid < p.n_tiles ? __ldcg(p.above + b * p.n_tiles + tid) : 0u;
  if (tid < kCandSplit) cand[tid] = __ldcg(p.gcand + b * kCandSplit + tid);  // slots past the count are unused
  // the row's scores into L1 while the candidates are ranked (chunk_rows reads its tiles)
  for (int q = 32 * tid; q < p.N; q += 32 * kThreads)
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p.scores + static_cast<int64_t>(b) * p.ld_ws + q));
  for (int q = tid; q < p.n_tiles; q += kThreads) c->ctile[q] = 0u;
  __syncthreads();
  const bool all = c->bc[3] != 0u;
  const uint32_t nc = all ? 0u : c->bc[1];
  T_key = 1u;  // all taken: every eligible key
  T_idx = 0xFFFFFFFFu;
  if (!all) {
    rank_pick(cand, nc, c->bc[2], c);
    T_key = c->bc[5];
    T_idx = c->bc[6];
    if (tid < static_cast<int>(nc)) {
      const uint2 cd = cand[tid];
      if (cd.x > T_key || (cd.x == T_key && cd.y <= T_idx)) atomicAdd(&c->ctile[cd.y / kTileM], 1u);
    }
    __syncthreads();
  }
  const uint32_t cnt = tid < p.n_tiles ? av + c->ctile[tid] : 0u;
  uint32_t total;
  const uint32_t off = block_excl_scan(cnt, total, c);
  if (tid < p.n_tiles) c->toff[tid] = off;
  if (tid == 0) c->toff[p.n_tiles] = total;
  __syncthreads();
}

// Entry j with key kk is taken
__device__ __forceinline__ bool taken_key(uint32_t kk, uint32_t j, uint32_t T_key, uint32_t T_idx) {
  return kk != 0u && (kk > T_key || (kk == T_key && j <= T_idx));
}

// The selector unit clears the row's histogram bins for the next call, once
// every score unit has read them (the candidate step is complete): it reads
// the row's scores back and zeroes the bins of their keys.
__device__ void clear_row(const FusedParams &p, int b) {
  const float *row = p.scores + static_cast<int64_t>(b) * p.ld_ws;
  for (int q = 4 * threadIdx.x; q < p.N; q += 4 * kThreads) {
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(row + q));  // the row is padded to 4 scores
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const uint32_t kk = q + e < p.N ? order_key(f[e]) : 0u;
      if (kk) {
        p.hist[b * kNB1 + (kk >> 24)] = 0u;
        p.hist2[static_cast<int64_t>(b) * kNB2 + (kk >> 16)] = 0u;
      }
    }
  }
}

// Key-space threshold search of the selector unit over its register keys x
// (NaN = not eligible), starting from the row's key range [a, b]: 11 bits a
// level until the interval is small enough to rank or holds one key value,
// which then takes its first entries by index.  Every branch is uniform over
// the block.
__device__ __forceinline__ void find_threshold(const float (&x)[kSelItems], uint32_t a, uint32_t b, int k,
                                               uint32_t *hist, uint2 *cand, Ctl *c, uint32_t &T_key,
                                               uint32_t &T_idx) {
  const int tid = threadIdx.x;
  const int pos0 = tid * kSelItems;
  uint32_t need = static_cast<uint32_t>(k), in_bin = 0;
  T_key = 1u;  // every eligible key (when at most k are)
  T_idx = 0xFFFFFFFFu;
  {
    uint32_t n = 0;
#pragma unroll
    for (int i = 0; i < kSelItems; i++) n += order_key(x[i]) ? 1u : 0u;
    block_excl_scan(n, in_bin, c);
    if (in_bin <= need) return;
  }
  uint32_t s = (b - a) < kNB ? 0u : static_cast<uint32_t>(32 - __clz(b - a) - 11);
  for (int level = 0; level < 3 && in_bin > static_cast<uint32_t>(kCandMax) && b > a; level++) {
    for (int i = tid; i < kNB; i += kThreads) hist[i] = 0u;
    __syncthreads();
    const uint32_t base = a;
#pragma unroll
    for (int i = 0; i < kSelItems; i++) {
      const uint32_t kk = order_key(x[i]);
      if (kk >= a && kk <= b) atomicAdd(&hist[(kk - base) >> s], 1u);
    }
    __syncthreads();
    find_bin(hist, need, c);
    need -= c->bc[3];
    in_bin = c->bc[4];
    const uint32_t nb_lo = base + (c->bc[2] << s);
    a = max(a, nb_lo);
    b = min(b, nb_lo + ((1u << s) - 1u));
    s = s > 11 ? s - 11 : 0u;
  }
  if (in_bin > static_cast<uint32_t>(kCandMax)) {
    // one key value: take its first `need` entries by index
    uint32_t tie = 0;
#pragma unroll
    for (int i = 0; i < kSelItems; i++) tie += order_key(x[i]) == a ? 1u : 0u;
    uint32_t tt;
    uint32_t te = block_excl_scan(tie, tt, c);
#pragma unroll
    for (int i = 0; i < kSelItems; i++) {
      if (order_key(x[i]) == a) {
        if (te == need - 1) c->bc[6] = static_cast<uint32_t>(pos0 + i);
        te++;
      }
    }
    __syncthreads();
    T_key = a;
    T_idx = c->bc[6];
    return;
  }
  if (tid == 0) c->bc[1] = 0u;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kSelItems; i++) {
    const uint32_t kk = order_key(x[i]);
    if (kk >= a && kk <= b && kk) {
      const uint32_t slot = atomicAdd(&c->bc[1], 1u);
      if (slot < kCandMax) cand[slot] = make_uint2(kk, static_cast<uint32_t>(pos0 + i));
    }
  }
  __syncthreads();
  rank_pick(cand, min(c->bc[1], static_cast<uint32_t>(kCandMax)), need, c);
  T_key = c->bc[5];
  T_idx = c->bc[6];
}

// padded shared-memory word of row position q
__device__ __forceinline__ int sel_pad(int q) { return q + (q >> 5) * 4; }

// The selector unit of row b: waits for the candidate step; in split mode
// the row is the score units' already.  Otherwise it selects the row alone:
// thread t owns positions [t*kSelItems, +kSelItems) and keeps their scores
// in registers.  The row is staged through shared memory by coalesced
// 16-byte loads, stored with 4 pad words after every 32 scores, so each
// thread then reads its 32 consecutive scores as 8 conflict-free loads.
__device__ __noinline__ void select_unit(const FusedParams &p, int b, uint8_t *sm, Ctl *c, bool &abort) {
  const int tid = threadIdx.x;
  uint32_t *hist = reinterpret_cast<uint32_t *>(sm + kSmHist);
  uint2 *cand = reinterpret_cast<uint2 *>(sm + kSmCand);
  float *srow = reinterpret_cast<float *>(sm + kSmRow);
  uint32_t *ctl = p.ctl + b * kCtlStride;
  const bool ok = block_wait(p, ctl + kCtlCand, p.n_tiles, c, abort);
  clear_row(p, b);
  if (ok && __ldcg(ctl + kCtlMode) == kModeSplit) return;
  // stage the row: chunk j*kThreads + tid holds positions 4*chunk .. +3 (the
  // workspace row is padded to a multiple of 4 scores)
  const float *row = p.scores + static_cast<int64_t>(b) * p.ld_ws;
  {
    float4 v[kSelItems / 4];
#pragma unroll
    for (int j = 0; j < kSelItems / 4; j++) {
      const int q = 4 * (j * kThreads + tid);
      v[j] = ok && q < p.N ? __ldcg(reinterpret_cast<const float4 *>(row + q)) : make_float4(NAN, NAN, NAN, NAN);
    }
#pragma unroll
    for (int j = 0; j < kSelItems / 4; j++) {
      const int q = 4 * (j * kThreads + tid);
      *reinterpret_cast<float4 *>(srow + sel_pad(q)) = v[j];
    }
  }
  __syncthreads();
  // this thread's scores; positions beyond N become NaN (never selected)
  const int pos0 = tid * kSelItems;
  float x[kSelItems];
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int q = 0; q < kSelItems / 4; q++) {
    const float4 v = *reinterpret_cast<const float4 *>(srow + sel_pad(pos0 + 4 * q));
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      x[4 * q + e] = pos0 + 4 * q + e < p.N ? f[e] : NAN;
      const uint32_t kk = order_key(x[4 * q + e]);
      hi = max(hi, kk);
      lo = kk ? min(lo, kk) : lo;
    }
  }
  block_minmax(lo, hi, c);
  uint32_t T_key = 0xFFFFFFFFu, T_idx = 0u;  // no eligible key: nothing is taken
  if (hi) find_threshold(x, lo, hi, p.k, hist, cand, c, T_key, T_idx);
  // emit ids ascending
  uint32_t mask = 0;
#pragma unroll
  for (int i = 0; i < kSelItems; i++)
    mask |= (taken_key(order_key(x[i]), static_cast<uint32_t>(pos0 + i), T_key, T_idx) ? 1u : 0u) << i;
  uint32_t n_out;
  uint32_t pos = block_excl_scan(__popc(mask), n_out, c);
  const int k = p.k;
  int32_t *sel = p.sel_ids + static_cast<int64_t>(b) * k;
  int32_t *uid = p.ids_user ? p.ids_user + static_cast<int64_t>(b) * k : nullptr;
  for (; mask && pos < static_cast<uint32_t>(k); pos++) {
    const int j = pos0 + __ffs(mask) - 1;
    mask &= mask - 1u;
    sel[pos] = j;
    if (uid) uid[pos] = j;
  }
  const int n_sel = static_cast<int>(min(n_out, static_cast<uint32_t>(k)));
  if (uid)
    for (int i = n_sel + tid; i < k; i += kThreads) uid[i] = -1;
  if (tid == 0) {
    p.sel_n[b] = n_sel;
    if (p.n_sel_user) p.n_sel_user[b] = n_sel;
  }
  __syncthreads();
  if (tid == 0) arrive_release(ctl + kCtlReady, static_cast<uint32_t>(p.n_tiles));
}

// -------------------------------------------------------------- attention
// The ids at positions [s0, s1) of row b's ascending selected list (split
// mode, after split_view): the tiles holding them are read back from the
// workspace scores, one tile per warp, and their taken entries ranked in
// position order.  c->chunk_id[q - s0] = the id at position q.
__device__ void chunk_rows(const FusedParams &p, int b, int s0, int s1, uint32_t T_key, uint32_t T_idx, Ctl *c) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (s0 < s1) {
    // the tiles holding positions s0 and s1 - 1
    for (int t = tid; t < p.n_tiles; t += kThreads) {
      const uint32_t a = c->toff[t], e = c->toff[t + 1];
      if (a <= static_cast<uint32_t>(s0) && static_cast<uint32_t>(s0) < e) c->bc[1] = t;
      if (a < static_cast<uint32_t>(s1) && static_cast<uint32_t>(s1) <= e) c->bc[2] = t;
    }
    __syncthreads();
    const int t0 = static_cast<int>(c->bc[1]), t1 = static_cast<int>(c->bc[2]);
    const float *row = p.scores + static_cast<int64_t>(b) * p.ld_ws;
    for (int t = t0 + warp; t <= t1; t += kWarps) {
      const int j0 = t * kTileM + 4 * lane;
      float4 v = make_float4(NAN, NAN, NAN, NAN);
      if (j0 < p.N) v = *reinterpret_cast<const float4 *>(row + j0);  // the row is padded to 4 scores; in L1
      const float f[4] = {v.x, v.y, v.z, v.w};
      uint32_t bits = 0;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const uint32_t kk = j0 + e < p.N ? order_key(f[e]) : 0u;
        bits |= (taken_key(kk, static_cast<uint32_t>(j0 + e), T_key, T_idx) ? 1u : 0u) << e;
      }
      const uint32_t n = __popc(bits);
      uint32_t x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
      }
      uint32_t g = c->toff[t] + x - n;  // this lane's first position
#pragma unroll
      for (int e = 0; e < 4; e++) {
        if (bits >> e & 1u) {
          if (g >= static_cast<uint32_t>(s0) && g < static_cast<uint32_t>(s1)) c->chunk_id[g - s0] = j0 + e;
          g++;
        }
      }
    }
  }
  __syncthreads();
}

__device__ void attn_unit(const FusedParams &p, int a, const CUtensorMap *tm_qa, const CUtensorMap *tm_win,
                          uint8_t *sm, Ctl *c, uint32_t tmem, bool &abort) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per_b = p.n_chunks * 4;
  const int b = a / per_b, ch = (a % per_b) / 4, hg = a % 4;
  const int swa_len = p.swa_len;
  const int i0 = ch * kRows;
  const bool pure_window = i0 + kRows <= swa_len;
  uint8_t *sX = sm + kSmX, *sQ = sm + kSmQa, *sP = sm + kSmP;
  const uint32_t xs = tc::smem_u32(sX);
  if (tid == 0) {
    tc::fence_proxy_async_smem();
    tc::mbar_arrive_expect_tx(&c->a_full, kQBytes + (pure_window ? kXBytes : 0));
#pragma unroll
    for (int q = 0; q < 8; q++) tc::tma_load_2d(sQ + q * kQPanel, tm_qa, &c->a_full, 64 * q, b * kHA + hg * kHG);
    if (pure_window) {
      const int y = static_cast<int>(static_cast<int64_t>(b) * p.swa_batch_rows + i0);
#pragma unroll
      for (int q = 0; q < 8; q++) tc::tma_load_2d(sX + q * kXPanel, tm_win, &c->a_full, 64 * q, y);
    }
  }
  if (tid < kRows) {
    const int i = i0 + tid;
    const bool win = i < swa_len;
    c->row_kind[tid] = win ? 2 : 0;
    c->row_src[tid] = win ? static_cast<int64_t>(b) * p.swa_batch_rows + i : -1;
  }
  __syncthreads();
  if (!pure_window) {
    // window rows of a mixed chunk, then the selected rows once they are known
    for (int r = warp; r < kRows; r += kWarps) {
      if (c->row_kind[r] != 2) continue;
      const uint16_t *src = p.swa + c->row_src[r] * p.swa_ld;
      cp_async16(xs + x_off(r, lane), src + lane * 8);
      cp_async16(xs + x_off(r, lane + 32), src + (lane + 32) * 8);
    }
    const uint32_t *ctl = p.ctl + b * kCtlStride;
    const bool ok = block_wait(p, ctl + kCtlCand, p.n_tiles, c, abort);
    const bool split = ok && __ldcg(ctl + kCtlMode) == kModeSplit;  // uniform over the CTA
    int n_b = 0;
    const int s0 = max(0, i0 - swa_len);  // the chunk's first position in the selected list
    if (split) {
      uint32_t T_key, T_idx;
      split_view(p, b, sm, c, T_key, T_idx);
      n_b = static_cast<int>(min(c->toff[p.n_tiles], static_cast<uint32_t>(p.k)));
      chunk_rows(p, b, s0, min(n_b, i0 + kRows - swa_len), T_key, T_idx, c);
      if (hg == 0) {  // the caller's ids at this chunk's list positions (-1 past the count)
        const int q1 = min(p.k, i0 + kRows - swa_len);
        if (p.ids_user)
          for (int q = s0 + tid; q < q1; q += kThreads)
            p.ids_user[static_cast<int64_t>(b) * p.k + q] = q < n_b ? c->chunk_id[q - s0] : -1;
        if (s0 == 0 && tid == 0) {
          p.sel_n[b] = n_b;
          if (p.n_sel_user) p.n_sel_user[b] = n_b;
        }
      }
    } else if (ok && block_wait(p, ctl + kCtlReady, static_cast<uint32_t>(p.n_tiles), c, abort)) {
      n_b = __ldcg(p.sel_n + b);  // the selector unit's list
    }
    // warp w gathers rows w + 16j; lane j resolves row w + 16j
    constexpr int kPerWarp = kRows / kWarps;
    int kind = 0;
    int64_t src = -1;
    if (lane < kPerWarp) {
      const int r = warp + kWarps * lane;
      kind = c->row_kind[r];
      src = c->row_src[r];
      const int i = i0 + r - swa_len;
      if (kind == 0 && i >= 0 && i < n_b) {
        const int id = split ? c->chunk_id[i - s0] : __ldcg(p.sel_ids + static_cast<int64_t>(b) * p.k + i);
        if (id >= 0 && id < p.N) {
          kind = 1;
          src = static_cast<int64_t>(b) * p.kv_batch_rows + id;
        }
      }
      c->row_kind[r] = kind;
    }
#pragma unroll
    for (int j = 0; j < kPerWarp; j++) {
      const int kj = __shfl_sync(0xFFFFFFFFu, kind, j);
      const int64_t sj = __shfl_sync(0xFFFFFFFFu, src, j);
      const int r = warp + kWarps * j;
      if (kj == 2) continue;
      if (kj == 1) {
        const uint16_t *rowp = p.kv + sj * p.kv_ld;
        cp_async16(xs + x_off(r, lane), rowp + lane * 8);
        cp_async16(xs + x_off(r, lane + 32), rowp + (lane + 32) * 8);
      } else {
        *reinterpret_cast<uint4 *>(sX + x_off(r, lane)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sX + x_off(r, lane + 32)) = make_uint4(0, 0, 0, 0);
      }
    }
  }
  cp_async_wait_all();
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  // S^T = X . Q^T: lane 0 of warp i < kS1 issues K steps [8i, 8i + 8) into partial sum i
  if (warp < kS1 && lane == 0) {
    if (tc::mbar_wait(&c->a_full, 0, &c->abort)) {
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
    }
    tc::mma_commit(&c->s_full);
  }
  // softmax: warps 0-7; warp w takes row quarter w&3 and heads 8(w>>2)..
  const int quarter = warp & 3, half = (warp >> 2) & 1;
  float mx[8];
  if (warp < 8) {
    bool ready = false;
    if (lane == 0) ready = tc::mbar_wait(&c->s_full, 0, &c->abort) && !c->abort;
    ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
    const int r = quarter * 16 + (lane & 15);
    const bool valid = lane < 16 && c->row_kind[r] != 0;
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
    const float c2 = p.scale * kLog2e;
#pragma unroll
    for (int h = 0; h < 8; h++) {
      s[h] = valid && ready ? s[h] * c2 : -INFINITY;
      mx[h] = s[h];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int h = 0; h < 8; h++) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], o));
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < 8; h++) c->red[half][quarter][h] = mx[h];
    named_sync(1 + half, 128);
    float pv[8];
#pragma unroll
    for (int h = 0; h < 8; h++) {
      const float m = fmaxf(fmaxf(c->red[half][0][h], c->red[half][1][h]), fmaxf(c->red[half][2][h], c->red[half][3][h]));
      mx[h] = m;
      pv[h] = (m == -INFINITY || s[h] == -INFINITY) ? 0.f : exp2f(s[h] - m);
    }
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
    named_sync(1 + half, 128);
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < 8; h++) c->red[half][quarter][h] = sum[h];
    named_sync(1 + half, 128);
    if (quarter == 0 && lane < 8) {
      const float l = (c->red[half][0][lane] + c->red[half][1][lane]) + (c->red[half][2][lane] + c->red[half][3][lane]);
      float m = mx[0];
#pragma unroll
      for (int i = 1; i < 8; i++)
        if (i == lane) m = mx[i];
      p.part_ml[(static_cast<size_t>(b) * p.n_chunks + ch) * kHA + hg * kHG + half * 8 + lane] = make_float2(m, l);
    }
  }
  if (tid == 0 && c->abort) drain(&c->a_full, 0);  // never leave with the Q / window copies in flight
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  // O^T = X^T . (P_hi + P_lo)^T: lane 0 of warp dt < 4 issues d tile dt
  if (warp < 4 && lane == 0) {
    if (!c->abort) {
      tc::tc_fence_after();
      const uint32_t idesc = tc::idesc_bf16(128, 2 * kHG, true, false);
      const uint32_t ps = tc::smem_u32(sP);
      const int dt = warp;
#pragma unroll
      for (int kk = 0; kk < kRows / 16; kk++) {
        const uint64_t adesc = tc::desc_mnmajor_sw128(xs + 2 * dt * kXPanel + kk * 2048, kXPanel, 1024);
        const uint64_t bdesc = tc::desc_kmajor_sw128(ps + kk * 32);
        tc::mma_bf16(tmem + kOCol + 32 * dt, adesc, bdesc, idesc, kk > 0);
      }
    }
    tc::mma_commit(&c->o_full);
  }
  // partial O out: warp w stores d tile w>>2 of its TMEM lane quarter
  {
    bool oready = false;
    if (lane == 0) oready = tc::mbar_wait(&c->o_full, 0, &c->abort) && !c->abort;
    oready = __shfl_sync(0xFFFFFFFFu, oready, 0);
    if (oready) {
      tc::tc_fence_after();
      float *po = p.part_o + ((static_cast<size_t>(b) * p.n_chunks + ch) * kHA + hg * kHG) * kD;
      const int dt = warp >> 2;
      const int d = dt * 128 + quarter * 32 + lane;
      float v[32];
      tc::tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kOCol + 32 * dt, v);
#pragma unroll
      for (int h = 0; h < kHG; h++) po[h * kD + d] = v[h] + v[kHG + h];
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (c->abort) abort = true;
  // the group's units wait for each other, then each merges a slice
  uint32_t *cnt = p.ctl + b * kCtlStride + kCtlAttn + hg;
  if (tid == 0) {
    arrive_release(cnt);
    c->bc[0] = wait_geq(cnt, static_cast<uint32_t>(p.n_chunks), p.wait_ns) ? 1u : 0u;
  }
  __syncthreads();
  if (!c->bc[0]) {
    abort = true;
    if (tid == 0) raise_status(p.status, LIDX_DEV_TIMEOUT);
    return;
  }
  constexpr int kF4 = kHG * kD / 4;  // float4 outputs of the group
  const int f0 = ch * kF4 / p.n_chunks, f1 = (ch + 1) * kF4 / p.n_chunks;
  // two threads per output: each folds every other partial (all of its loads
  // in one round for up to 16 chunks), then the pair combines
  const int par = tid & 1;
  for (int fb = f0; fb < f1; fb += kThreads / 2) {
    const int f = fb + tid / 2;
    const bool act = f < f1;
    const int h = f / (kD / 4), d4 = f % (kD / 4);
    const int head = hg * kHG + h;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float M = -INFINITY, L = 0.f;
    for (int s0 = par; act && s0 < p.n_chunks; s0 += 16) {
      float2 ml[8];
      float4 v[8];
#pragma unroll
      for (int q = 0; q < 8; q++) {
        ml[q] = make_float2(-INFINITY, 0.f);
        if (s0 + 2 * q < p.n_chunks) {
          const size_t base = (static_cast<size_t>(b) * p.n_chunks + s0 + 2 * q) * kHA + head;
          ml[q] = __ldcg(p.part_ml + base);
          v[q] = __ldcg(reinterpret_cast<const float4 *>(p.part_o + base * kD) + d4);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; q++) {
        if (ml[q].x != -INFINITY) {
          const float mn = fmaxf(M, ml[q].x);
          const float cf = exp2f(M - mn);
          const float e = exp2f(ml[q].x - mn);
          L = fmaf(L, cf, e * ml[q].y);
          acc.x = fmaf(acc.x, cf, e * v[q].x);
          acc.y = fmaf(acc.y, cf, e * v[q].y);
          acc.z = fmaf(acc.z, cf, e * v[q].z);
          acc.w = fmaf(acc.w, cf, e * v[q].w);
          M = mn;
        }
      }
    }
    // the pair's two folds
    const float Mo = __shfl_xor_sync(0xFFFFFFFFu, M, 1), Lo = __shfl_xor_sync(0xFFFFFFFFu, L, 1);
    const float ax = __shfl_xor_sync(0xFFFFFFFFu, acc.x, 1), ay = __shfl_xor_sync(0xFFFFFFFFu, acc.y, 1);
    const float az = __shfl_xor_sync(0xFFFFFFFFu, acc.z, 1), aw = __shfl_xor_sync(0xFFFFFFFFu, acc.w, 1);
    if (!act || par) continue;
    const float mn = fmaxf(M, Mo);
    const float c0 = M == -INFINITY ? 0.f : exp2f(M - mn), c1 = Mo == -INFINITY ? 0.f : exp2f(Mo - mn);
    L = L * c0 + Lo * c1;
    acc = make_float4(acc.x * c0 + ax * c1, acc.y * c0 + ay * c1, acc.z * c0 + az * c1, acc.w * c0 + aw * c1);
    M = mn;
    const float il = L > 0.f ? 1.f / L : 0.f;
    reinterpret_cast<float4 *>(p.out + (static_cast<size_t>(b) * kHA + head) * kD)[d4] =
        make_float4(acc.x * il, acc.y * il, acc.z * il, acc.w * il);
    if (d4 == 0 && p.lse)
      p.lse[static_cast<size_t>(b) * kHA + head] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
  }
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_keys, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_qa, const __grid_constant__ CUtensorMap tm_win,
                        const __grid_constant__ FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl *c = reinterpret_cast<Ctl *>(sm + kSmData);
  const int tid = threadIdx.x, warp = tid >> 5;
  bool abort = false;

  if (tid == 0) {
    tc::mbar_init(&c->key_full[0], 1);
    tc::mbar_init(&c->key_full[1], 1);
    tc::mbar_init(&c->q_full, 1);
    tc::mbar_init(&c->mma_done, 1);
    tc::mbar_init(&c->a_full, 1);
    tc::mbar_init(&c->s_full, kS1);
    tc::mbar_init(&c->o_full, 4);
    c->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_keys);
    tc::tma_prefetch_desc(&tm_q);
    tc::tma_prefetch_desc(&tm_qa);
    tc::tma_prefetch_desc(&tm_win);
    // the first two key tiles are cache-side: fetched before waiting for the
    // previous kernel on the stream
    for (int i = 0; i < 2; i++) {
      const int u = blockIdx.x + i * p.G;
      if (u < p.n_score) issue_key_tile(p, &tm_keys, sm, c, u, i);
    }
  }
  if (warp == 1) tc::tmem_alloc(&c->tmem_base, kTmemCols);
  for (int i = tid; i < kNB1; i += kThreads) c->h1[i] = 0u;
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_trigger();
  pdl_wait();
  const uint32_t tmem = c->tmem_base;

  score_units(p, &tm_keys, &tm_q, sm, c, tmem, abort);
  // CTAs done with scoring pull the next layer's cache-side inputs into L2
  {
    for (int r = 0; r < 2; r++) {
      const uint64_t nb = p.pf_bytes[r];
      if (!p.pf[r] || !nb) continue;
      const uint64_t per = ((nb + p.G - 1) / p.G + 15) & ~uint64_t(15);
      const uint64_t s0 = blockIdx.x * per, s1 = min(nb, s0 + per);
      for (uint64_t o = s0 + static_cast<uint64_t>(tid) * 4096; o < s1; o += static_cast<uint64_t>(kThreads) * 4096)
        prefetch_l2(p.pf[r] + o, static_cast<uint32_t>(s1 - o < 4096 ? s1 - o : 4096));
    }
  }
  cand_units(p, sm, c, abort);
  // select units
  for (int u = blockIdx.x + ((p.n_score - static_cast<int>(blockIdx.x) + p.G - 1) / p.G) * p.G;
       u < p.n_score + p.B; u += p.G) {
    tc::fence_proxy_async_smem();
    __syncthreads();
    select_unit(p, u - p.n_score, sm, c, abort);
  }
  // the attention unit (at most one per CTA)
  {
    const int base = p.n_score + p.B;
    const int first = blockIdx.x + ((base - static_cast<int>(blockIdx.x) + p.G - 1) / p.G) * p.G;
    if (first < base + p.n_attn) {
      __syncthreads();
      attn_unit(p, first - base, &tm_qa, &tm_win, sm, c, tmem, abort);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  // the last CTA to leave zeroes the control words for the next call
  if (tid == 0) {
    if (c->abort) raise_status(p.status, LIDX_DEV_TIMEOUT);
    uint32_t prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(p.ctl + p.B * kCtlStride) : "memory");
    c->bc[0] = prev == static_cast<uint32_t>(p.G - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (c->bc[0]) {
    for (int i = tid; i < p.B * kCtlStride; i += kThreads) p.ctl[i] = 0u;
    // after a wait gave up, a histogram may hold counts nobody cleared
    if (ld_acquire(p.status) & LIDX_DEV_TIMEOUT) {
      for (int i = tid; i < p.B * kNB1; i += kThreads) p.hist[i] = 0u;
      for (int64_t i = tid; i < static_cast<int64_t>(p.B) * kNB2; i += kThreads) p.hist2[i] = 0u;
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      p.ctl[p.B * kCtlStride] = 0u;
    }
  }
  (void)abort;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int n_chunks(const lidx_decode_args &a) {
  const int rows = a.k + a.swa_len;
  return rows > 0 ? (rows + kRows - 1) / kRows : 1;
}

struct WsLayout {
  size_t ctl, sel_ids, sel_n, part_ml, part_o, scores, hist, hist2, above, gcand, total;
  int64_t ld_ws;
};

WsLayout ws_layout(const lidx_decode_args &a) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  WsLayout l{};
  const int nc = n_chunks(a);
  l.ld_ws = (a.N + 3) & ~3;
  size_t o = LIDX_WS_HEADER;
  l.ctl = o;
  o += up(static_cast<size_t>(a.B + 1) * kCtlStride * 4);
  l.sel_ids = o;
  o += up(static_cast<size_t>(a.B) * a.k * 4);
  l.sel_n = o;
  o += up(static_cast<size_t>(a.B) * 4);
  l.part_ml = o;
  o += up(static_cast<size_t>(a.B) * nc * kHA * sizeof(float2));
  l.part_o = o;
  o += up(static_cast<size_t>(a.B) * nc * kHA * kD * 4);
  l.scores = o;
  o += up(static_cast<size_t>(a.B) * l.ld_ws * 4);
  l.hist = o;
  o += up(static_cast<size_t>(a.B) * kNB1 * 4);
  l.hist2 = o;
  o += up(static_cast<size_t>(a.B) * kNB2 * 4);
  l.above = o;
  o += up(static_cast<size_t>(a.B) * ((a.N + kTileM - 1) / kTileM) * 4);
  l.gcand = o;
  o += up(static_cast<size_t>(a.B) * kCandSplit * 8);
  l.total = o;
  return l;
}

}  // namespace

bool decode_fused_supported(const lidx_decode_args &a) {
  if (a.keys.dtype != LIDX_BF16 || a.kv.dtype != LIDX_BF16) return false;
  if (a.swa_len > 0 && a.swa.dtype != LIDX_BF16) return false;
  if (a.H % 32 != 0 || a.H > 128 || a.H_attn != kHA) return false;
  if (a.N > kSelItems * kThreads) return false;
  if (static_cast<int64_t>(a.B) * n_chunks(a) * 4 > sm_count()) return false;
  const int64_t n_score = static_cast<int64_t>(a.B) * ((a.N + kTileM - 1) / kTileM);
  const int64_t G = std::min<int64_t>(sm_count(), n_score + a.B + static_cast<int64_t>(a.B) * n_chunks(a) * 4);
  if (n_score > kMaxOwnTiles * G) return false;
  const int64_t rows = static_cast<int64_t>(a.B - 1) * (a.B > 1 ? a.keys.batch_rows : a.N) + a.N;
  return rows < (1ll << 31);
}

size_t decode_fused_workspace(const lidx_decode_args &a) { return ws_layout(a).total; }

cudaError_t launch_decode_fused(const lidx_decode_args &a, void *ws, cudaStream_t st) {
  const WsLayout l = ws_layout(a);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  FusedParams p{};
  p.B = a.B;
  p.H = a.H;
  p.N = a.N;
  p.k = a.k;
  p.swa_len = a.swa_len;
  p.n_tiles = (a.N + kTileM - 1) / kTileM;
  p.n_chunks = n_chunks(a);
  p.n_score = a.B * p.n_tiles;
  p.n_attn = a.B * p.n_chunks * 4;
  p.G = std::min(sm_count(), p.n_score + a.B + p.n_attn);
  p.key_batch_rows = a.B > 1 ? a.keys.batch_rows : a.N;
  p.w = a.w;
  p.kv = static_cast<const uint16_t *>(a.kv.data);
  p.kv_ld = a.kv.ld;
  p.kv_batch_rows = a.B > 1 ? a.kv.batch_rows : a.N;
  p.swa = static_cast<const uint16_t *>(a.swa.data);
  p.swa_ld = a.swa.ld;
  p.swa_batch_rows = a.B > 1 ? a.swa.batch_rows : a.swa_len;
  p.scale = a.scale;
  p.out = a.out;
  p.lse = a.lse;
  p.scores_user = a.scores;
  p.ld_user = a.ld_scores;
  p.ids_user = a.ids;
  p.n_sel_user = a.n_sel;
  p.status = reinterpret_cast<uint32_t *>(w8);
  p.ctl = reinterpret_cast<uint32_t *>(w8 + l.ctl);
  p.sel_ids = reinterpret_cast<int32_t *>(w8 + l.sel_ids);
  p.sel_n = reinterpret_cast<int32_t *>(w8 + l.sel_n);
  p.part_ml = reinterpret_cast<float2 *>(w8 + l.part_ml);
  p.part_o = reinterpret_cast<float *>(w8 + l.part_o);
  p.scores = reinterpret_cast<float *>(w8 + l.scores);
  p.ld_ws = l.ld_ws;
  p.hist2 = reinterpret_cast<uint32_t *>(w8 + l.hist2);
  p.hist = reinterpret_cast<uint32_t *>(w8 + l.hist);
  p.above = reinterpret_cast<uint32_t *>(w8 + l.above);
  p.gcand = reinterpret_cast<uint2 *>(w8 + l.gcand);
  for (int r = 0; r < 2; r++) {
    p.pf[r] = static_cast<const uint8_t *>(a.prefetch[r]);
    p.pf_bytes[r] = a.prefetch[r] ? a.prefetch_bytes[r] : 0;
  }
  const bool test_lost = (a.flags & LIDX_LAUNCH_TEST_LOST_ARRIVAL) != 0;
  p.lost_arrival = test_lost ? 1u : 0u;
  p.wait_ns = test_lost ? 2000000ull : 2000000000ull;  // 2 ms in the test hook, else 2 s

  const uint64_t key_rows = static_cast<uint64_t>(a.B - 1) * p.key_batch_rows + a.N;
  CUtensorMap tm_keys, tm_q, tm_qa, tm_win;
  bool ok = make_tmap_2d(&tm_keys, a.keys.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, key_rows, a.keys.ld * 2, 64,
                         kTileM, CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_tmap_2d(&tm_q, a.q_idx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 128, static_cast<uint64_t>(a.B) * a.H, 256,
                         64, a.H, CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_tmap_2d(&tm_qa, a.q_attn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, static_cast<uint64_t>(a.B) * kHA,
                         kD * 2, 64, kHG, CU_TENSOR_MAP_SWIZZLE_128B);
  tm_win = tm_qa;
  if (ok && a.swa_len >= kRows) {
    const uint64_t rows = static_cast<uint64_t>(a.B - 1) * p.swa_batch_rows + a.swa_len;
    ok = make_tmap_2d(&tm_win, a.swa.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, rows, a.swa.ld * 2, 64, kRows,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = smem_bytes();
  const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
  cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  return launch_kernel(decode_fused_kernel, dim3(p.G), dim3(kThreads), smem, st, pdl, tm_keys, tm_q, tm_qa, tm_win, p);
}

}  // namespace lidx
