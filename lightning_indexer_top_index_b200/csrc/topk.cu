// Top-k row ids by exact selection (DeepSeek-V4-Flash architecture post,
// section (B): keep the n_indexer_top_k highest-scoring compressed entries
// and hand their row ids, or the comp_allowed mask, to attention).
//
// Scores become order-preserving 32-bit keys (order_key: larger score ->
// larger key, -0 folded onto +0, NaN and disallowed entries -> 0).
//
// A row is served by a thread-block cluster of G CTAs (G = 1 when there are
// many rows; up to 8 when a few long rows must use many SMs).  CTA r owns
// the contiguous slice [r*S, r*S + S) of the row and thread t of it the
// positions [t*C, (t+1)*C) of the slice, loaded by one bulk copy and held in
// registers.  The CTAs exchange small summaries through distributed shared
// memory; each exchange pushes (remote stores into a slot per sender) before
// a cluster barrier, so nobody waits on remote loads after it:
//   1. the row's minimum and maximum key: read from the scorer's score
//      bounds when the caller passes them, else exchanged (with the count of
//      eligible keys);
//   2. a histogram over 256 linear value bins between the row's minimum and
//      maximum (the bin is a monotone function of the score, so the bin
//      holding the k-th largest key, and the count above it, are exact; for
//      score-like data that bin holds a few dozen keys);
//   3. the keys of that bin, with each CTA's count of keys above it: every
//      CTA resolves the k-th key T and how many keys equal to T are taken
//      (rank counting, or a radix over the candidates' differing bits when
//      there are many; a bin too full to gather is refined by cluster-wide
//      radix levels), and knows every CTA's count of keys > T and == T;
//   4. those counts' prefix gives every thread its output offset: ids come
//      out ascending, ties to the lower index.
#include <algorithm>

#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxItems = 32;
constexpr int kMaxCluster = 16;  // 16-CTA clusters (a non-portable size) where the device schedules them
constexpr int kSlot = 512;                       // candidates a CTA pushes to every CTA of its cluster
constexpr int kGatherMax = kSlot * kMaxCluster;  // candidates every CTA can gather
constexpr int kRankMax = 96;       // candidates resolved by direct rank counting (quadratic work)

// Values other CTAs of the cluster read.
struct Pub {
  uint32_t kmin, kmax, elig, nan;
  uint32_t cmin, cmax;
  uint32_t gt, eq;
  uint32_t hist[2][256];
};

struct SelSmem {
  Pub pub;
  uint32_t whist[8][256];     // histograms shared by groups of four warps
  uint32_t hist[256];         // cluster-wide histogram
  // written by the other CTAs of the cluster (remote stores before a cluster
  // barrier), slot r by CTA r
  uint32_t hist_in[kMaxCluster][256];
  uint32_t landing[kMaxCluster][kSlot];
  uint32_t cnt_in[kMaxCluster], above_in[kMaxCluster];
  uint32_t gathered[kGatherMax];
  uint32_t red_a[kWarps], red_b[kWarps], red_c[kWarps], red_d[kWarps];
  uint32_t scan[2][kWarps];
  uint32_t cand_count;
  uint32_t red_tot;
  uint32_t digit, above, total;
  uint32_t T, need;
  uint32_t g[4];                       // cluster-wide values broadcast to the CTA
  uint32_t cand_off[kMaxCluster + 1];  // prefix of the CTAs' candidate counts
  uint32_t above_r[kMaxCluster];       // every CTA's count above the threshold bin
  uint32_t cnt_gt[kMaxCluster], cnt_eq[kMaxCluster];  // every CTA's keys > T and == T
  uint64_t bar;
};

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_hw() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Start barrier: every CTA arrives when it starts (after zeroing the slots
// others add into; arrive releases, wait acquires) and waits before its first
// access to another CTA's shared memory, which is only valid once all CTAs of
// the cluster run.
__device__ __forceinline__ void cluster_arrive_start() {
  if (gridDim.x > 1) asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_start() {
  if (gridDim.x > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Cluster barrier; a cluster of one CTA needs only the CTA barrier (no
// cluster-scope fence).
__device__ __forceinline__ void cluster_sync() {
  if (gridDim.x == 1)
    __syncthreads();
  else
    cluster_sync_hw();
}

// Store a 32-bit word into CTA `rank`'s shared memory at the local address `p`
// (the push side of an exchange: a cluster barrier makes it visible).
__device__ __forceinline__ void st_remote(uint32_t *p, uint32_t rank, uint32_t v) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(tc::smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Add to a 32-bit word of CTA `rank`'s shared memory.
__device__ __forceinline__ void add_remote(uint32_t *p, uint32_t rank, uint32_t v) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(tc::smem_u32(p)), "r"(rank));
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Load a 32-bit word of CTA `rank`'s shared memory at the local address `p`.
// Callers issue independent loads back to back (the round trip is long) and
// only read remote words a cluster barrier has published.
__device__ __forceinline__ uint32_t ld_remote(const uint32_t *p, uint32_t rank) {
  uint32_t a, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(tc::smem_u32(p)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Monotone 8-bit bin of a key inside [flo, flo + 256/scale]: round((x-flo)*scale)
// read off the mantissa of x*scale + 2^23 (no float-to-int conversion).
__device__ __forceinline__ uint32_t lin_bin(uint32_t kk, float flo, float scale) {
  const float t = fmaf(key_value(kk) - flo, scale, 8388608.f);
  return min(__float_as_uint(t) - 0x4B000000u, 255u);
}

// CTA-wide reductions (results valid in every thread after the call).
__device__ __forceinline__ uint32_t cta_min(SelSmem &sm, uint32_t v) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  __syncthreads();
  if (lane == 0) sm.red_a[warp] = v;
  __syncthreads();
  v = sm.red_a[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t cta_max(SelSmem &sm, uint32_t v) { return ~cta_min(sm, ~v); }

// Exclusive CTA scan of 32-bit values; *total gets the CTA sum.
// One barrier: every warp scans the 32 warp totals itself.  `buf` alternates
// between two scratch rows, so a scan never overwrites totals the previous
// scan's slower warps may still read (two scans apart there is a barrier).
__device__ __forceinline__ uint32_t cta_exclusive_scan(SelSmem &sm, uint32_t v, uint32_t &total, int &buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t inc = warp_inclusive_scan(v);
  if (lane == 31) sm.scan[buf][warp] = inc;
  __syncthreads();
  const uint32_t x = sm.scan[buf][lane];
  const uint32_t xi = warp_inclusive_scan(x);
  total = __shfl_sync(0xFFFFFFFFu, xi, 31);
  const uint32_t before = __shfl_sync(0xFFFFFFFFu, xi - x, warp);
  buf ^= 1;
  return before + inc - v;
}

// Merge the per-group histograms into pub.hist[buf].
__device__ __forceinline__ void publish_hist(SelSmem &sm, int buf) {
  __syncthreads();
  if (threadIdx.x < 256) {
    uint32_t v = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) v += sm.whist[w][threadIdx.x];
    sm.pub.hist[buf][threadIdx.x] = v;
  }
}

__device__ __forceinline__ void clear_whist(SelSmem &sm) {
  uint32_t *h = &sm.whist[0][0];
  for (int i = threadIdx.x; i < 8 * 256; i += kThreads) h[i] = 0u;
}

// Find, in sm.hist (bins < nbins), the bin holding the rem-th largest key from
// the top: sm.digit, and the count above it: sm.above.
__device__ __forceinline__ void find_bin(SelSmem &sm, int nbins, uint32_t rem) {
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int d = nbins - 1 - 8 * lane - i;
      c[i] = d >= 0 ? sm.hist[d] : 0u;
      sum += c[i];
    }
    const uint32_t inc = warp_inclusive_scan(sum);
    const uint32_t before = inc - sum;
    if (lane == 31) sm.total = inc;
    if (before < rem && inc >= rem) {
      uint32_t acc = before;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        if (acc < rem && acc + c[i] >= rem) {
          sm.digit = static_cast<uint32_t>(nbins - 1 - 8 * lane - i);
          sm.above = acc;
        }
        acc += c[i];
      }
    }
  }
  __syncthreads();
}

// After a cluster barrier: sum pub.hist[buf] over the cluster, then find_bin.
__device__ __forceinline__ void cluster_find(SelSmem &sm, int buf, int nbins, uint32_t rem, uint32_t G) {
  if (threadIdx.x < 256) {
    uint32_t v = 0;
    if (static_cast<int>(threadIdx.x) < nbins) {
      uint32_t x[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) x[r] = r < static_cast<int>(G) ? ld_remote(&sm.pub.hist[buf][threadIdx.x], r) : 0u;
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) v += x[r];
    }
    sm.hist[threadIdx.x] = v;
  }
  find_bin(sm, nbins, rem);
}

// Push this CTA's histogram (the sum of its group histograms) into slot
// `rank` of every CTA of the cluster; a cluster barrier must follow.
__device__ __forceinline__ void push_hist(SelSmem &sm, uint32_t G, uint32_t rank) {
  __syncthreads();
  const int bin = threadIdx.x & 255;
  uint32_t v = 0;
#pragma unroll
  for (int w = 0; w < 8; w++) v += sm.whist[w][bin];
  for (uint32_t r = threadIdx.x >> 8; r < G; r += kThreads / 256) st_remote(&sm.hist_in[rank][bin], r, v);
}

// After the barrier: the cluster-wide histogram from the pushed slots, then find_bin.
__device__ __forceinline__ void sum_pushed_hist(SelSmem &sm, uint32_t G, int nbins, uint32_t rem) {
  if (threadIdx.x < 256) {
    uint32_t v = 0;
    for (uint32_t r = 0; r < G; r++) v += sm.hist_in[r][threadIdx.x];
    sm.hist[threadIdx.x] = v;
  }
  find_bin(sm, nbins, rem);
}

struct SelParams {
  lidx_topk_args a;
  uint32_t *status;
  int slice;    // positions per CTA (C * kThreads)
  int n_seg;    // segments per row: grid row y is segment y % n_seg of row y / n_seg
  int seg_len;  // positions per segment (a.N when n_seg == 1)
};

template <int C>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) uint8_t dyn_smem[];
  SelSmem &sm = *reinterpret_cast<SelSmem *>(dyn_smem);
  float *rowbuf = reinterpret_cast<float *>(dyn_smem + ((sizeof(SelSmem) + 15) & ~size_t(15)));
  const lidx_topk_args &a = p.a;
  const int tid = threadIdx.x;
  const int hg = (tid >> 5) & 7;
  const uint32_t G = gridDim.x;  // the cluster spans the x dimension
  const uint32_t rank = cluster_rank();
  const int grow = blockIdx.y;                       // this CTA's row of the grid
  const int row = grow / p.n_seg;                    // the caller's row (b, t)
  const int seg0 = (grow % p.n_seg) * p.seg_len;     // first position of its segment in that row
  const int Nr = min(p.seg_len, a.N - seg0);         // positions of the segment
  const int k = a.k;
  const int s0 = static_cast<int>(rank) * p.slice;  // first position of this CTA's slice
  const int p0 = tid * C;                           // first position of this thread, within the slice

  if (tid < kMaxCluster) {
    sm.cnt_in[tid] = 0u;
    sm.above_in[tid] = 0u;
  }
  if (tid == 0) sm.cand_count = 0u;
  cluster_arrive_start();
  pdl_trigger();
  pdl_wait();  // the scores come from the previous kernel

  // The scorer's score bounds of the row, if given (one span record per
  // thread now; longer rows read the rest later).
  const int n_spans = (a.N + LIDX_STATS_SPAN - 1) / LIDX_STATS_SPAN;
  const uint2 *stp =
      a.tile_stats ? reinterpret_cast<const uint2 *>(a.tile_stats) + static_cast<size_t>(row) * n_spans : nullptr;
  uint2 st0 = make_uint2(0u, 0xFFFFFFFFu);
  if (stp && tid < n_spans) st0 = stp[tid];

  // ---- 0. this CTA's slice: one bulk copy into shared memory, then thread t
  // takes positions [t*C, t*C + C) of the slice into registers
  const int len = max(0, min(p.slice, Nr - s0));
  const float *s = a.scores + static_cast<size_t>(row) * a.ld_scores + seg0 + s0;
  const uint8_t *al = a.allowed ? a.allowed + static_cast<size_t>(row / a.Q) * a.ld_allowed + seg0 + s0 : nullptr;
  const uint32_t *alb = a.allowed_bits ? a.allowed_bits + static_cast<size_t>(row / a.Q) * a.ld_allowed_bits : nullptr;
  const int n_valid = a.n_valid ? __ldg(a.n_valid + row) : a.N;  // eligible prefix of this row
  float val[C];
  {
    const int head = len > 0 ? static_cast<int>(((16u - (reinterpret_cast<uintptr_t>(s) & 15u)) & 15u) / 4u) : 0;
    const int body = max(0, len - head) & ~3;
    float *sv = rowbuf + ((4 - head) & 3);  // the body lands 16-byte aligned
    if (tid == 0) {
      tc::mbar_init(&sm.bar, 1);
      tc::fence_barrier_init();
    }
    clear_whist(sm);  // for the value histogram, off the critical path
    __syncthreads();
    if (tid == 0 && body > 0) {
      tc::mbar_arrive_expect_tx(&sm.bar, body * 4);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       tc::smem_u32(sv + head)),
                   "l"(s + head), "r"(body * 4), "r"(tc::smem_u32(&sm.bar))
                   : "memory");
    }
    for (int j = tid; j < len; j += kThreads)
      if (j < head || j >= head + body) sv[j] = s[j];
    if (body > 0) {
      volatile uint32_t no_abort = 0;
      if (!tc::mbar_wait(&sm.bar, 0, &no_abort)) raise_status(p.status, LIDX_DEV_TIMEOUT);
    }
    __syncthreads();
    if (C >= 4 && head == 0 && p0 + C <= len) {
      // float4 reads; step j of thread t reads its float4 number
      // (j + t*n/8) mod n (n = C/4), so that the 8 lanes of each phase hit 8
      // different 16-byte bank groups
      constexpr int n = C / 4 > 0 ? C / 4 : 1;
      const int rot = (tid * n / 8) % n;
      const float4 *src = reinterpret_cast<const float4 *>(sv + p0);
#pragma unroll
      for (int j = 0; j < n; j++) {
        const int jj = (j + rot) % n;
        const float4 v = src[jj];
#pragma unroll
        for (int q = 0; q < n; q++)
          if (q == jj) {
            val[4 * q] = v.x;
            val[4 * q + 1] = v.y;
            val[4 * q + 2] = v.z;
            val[4 * q + 3] = v.w;
          }
      }
    } else {
#pragma unroll
      for (int i = 0; i < C; i++) val[i] = p0 + i < len ? sv[p0 + i] : 0.f;
    }
  }
  uint32_t key[C];
  uint32_t nanf = 0, elig = 0, lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int i = 0; i < C; i++) {
    const int pos = p0 + i;
    const bool in = pos < len;
    const int j = seg0 + s0 + pos;  // position in the caller's row
    const bool ok = in && j < n_valid && !(al && !al[pos]) && !(alb && !((__ldg(alb + (j >> 5)) >> (j & 31)) & 1u));
    uint32_t kk = in ? order_key(val[i]) : 0u;
    nanf |= (ok && kk == 0u) ? 1u : 0u;
    kk = ok ? kk : 0u;
    key[i] = kk;
    elig += kk != 0u;
    lo = kk ? min(lo, kk) : lo;
    hi = max(hi, kk);
  }
  // Exact k-th key T (and the number `need` of keys equal to T to take) among
  // the keys in_bin(i) selects, given that `rem` of the k are still to be
  // taken from that bin.
  uint32_t T = 0u, need = 0u;  // T = 0: take every eligible key
  // fast: the candidates were gathered, so every CTA knows every CTA's counts
  // of keys > T and == T (sm.cnt_gt / cnt_eq) and the emission needs no
  // exchange; this CTA has arrived on the final cluster barrier
  bool fast = false;
  auto resolve = [&](auto in_bin, auto above_bin, uint32_t rem) {
    // push this CTA's keys of the threshold bin into slot `rank` of every CTA
    // (positions from a CTA counter: order within a slot does not matter),
    // and add its counts of those keys and of keys above the bin into every
    // CTA's slot; the cluster barrier publishes both, no block barrier needed
    const int lane = tid & 31;
    uint32_t w_in = 0, w_above = 0;
#pragma unroll
    for (int i = 0; i < C; i++) {
      const bool in = in_bin(i);
      w_above += __popc(__ballot_sync(0xFFFFFFFFu, !in && above_bin(i)));
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
      if (m == 0u) continue;
      uint32_t base = 0;
      if (lane == 0) base = atomicAdd(&sm.cand_count, static_cast<uint32_t>(__popc(m)));
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
      w_in += __popc(m);
      if (in) {
        const uint32_t pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < static_cast<uint32_t>(kSlot))
          for (uint32_t r = 0; r < G; r++) st_remote(&sm.landing[rank][pos], r, key[i]);
      }
    }
    if (static_cast<uint32_t>(lane) < G) {
      if (w_in) add_remote(&sm.cnt_in[rank], lane, w_in);
      if (w_above) add_remote(&sm.above_in[rank], lane, w_above);
    }
    cluster_sync();
    if (tid < 32) {  // every CTA's counts, now local
      const uint32_t n = static_cast<uint32_t>(tid) < G ? sm.cnt_in[tid] : 0u;
      if (static_cast<uint32_t>(tid) < G) sm.above_r[tid] = sm.above_in[tid];
      const uint32_t inc = warp_inclusive_scan(n);
      const uint32_t big = __ballot_sync(0xFFFFFFFFu, n > static_cast<uint32_t>(kSlot));
      if (static_cast<uint32_t>(tid) < G) sm.cand_off[tid] = inc - n;
      if (tid == 31) {
        sm.cand_off[kMaxCluster] = inc;
        sm.g[0] = big;
      }
    }
    __syncthreads();
    const uint32_t n_cand = sm.cand_off[kMaxCluster];
    const bool too_many = sm.g[0] != 0u;
    if (!too_many) {
      // the same candidate list in every CTA: warp r compacts slot r
      {
        const int warp = tid >> 5, lane = tid & 31;
        if (static_cast<uint32_t>(warp) < G) {
          const uint32_t off = sm.cand_off[warp];
          const uint32_t n = (warp + 1 < static_cast<int>(G) ? sm.cand_off[warp + 1] : n_cand) - off;
          for (uint32_t i = lane; i < n; i += 32) sm.gathered[off + i] = sm.landing[warp][i];
        }
      }
      __syncthreads();
      fast = true;  // no cluster traffic from here on
      if (n_cand <= static_cast<uint32_t>(kRankMax)) {
        if (tid < static_cast<int>(n_cand)) {
          const uint32_t mine = sm.gathered[tid];
          uint32_t gt = 0, eq = 0;
          for (uint32_t j = 0; j < n_cand; j++) {
            const uint32_t o = sm.gathered[j];
            gt += o > mine;
            eq += o == mine;
          }
          if (gt < rem && gt + eq >= rem) {
            sm.T = mine;
            sm.need = rem - gt;
          }
        }
        __syncthreads();
        T = sm.T;
        need = sm.need;
      } else {
        // radix over the gathered candidates' differing bits (identical in every CTA)
        uint32_t clo = 0xFFFFFFFFu, chi = 0u;
        for (uint32_t i = tid; i < n_cand; i += kThreads) {
          clo = min(clo, sm.gathered[i]);
          chi = max(chi, sm.gathered[i]);
        }
        clo = cta_min(sm, clo);
        chi = cta_max(sm, chi);
        if (clo == chi) {
          T = clo;
          need = rem;
        } else {
          int bits_left = 32 - __clz(clo ^ chi);
          uint32_t pmask = bits_left == 32 ? 0u : ~((1u << bits_left) - 1u);
          uint32_t prefix = clo & pmask;
          while (bits_left > 0) {
            const int w = min(8, bits_left);
            const int shift = bits_left - w;
            const uint32_t dmask = (1u << w) - 1u;
            __syncthreads();
            if (tid < 256) sm.hist[tid] = 0u;
            __syncthreads();
            for (uint32_t i = tid; i < n_cand; i += kThreads) {
              const uint32_t kk = sm.gathered[i];
              if ((kk & pmask) == prefix) atomicAdd(&sm.hist[(kk >> shift) & dmask], 1u);
            }
            find_bin(sm, 1 << w, rem);
            prefix |= sm.digit << shift;
            pmask |= dmask << shift;
            rem -= sm.above;
            bits_left -= w;
          }
          T = prefix;
          need = rem;
        }
      }
      // every CTA's keys > T and == T: its count above the bin plus its
      // candidates (gathered segment r is CTA r's list)
      {
        const int warp = tid >> 5, lane = tid & 31;
        if (static_cast<uint32_t>(warp) < G) {
          const uint32_t off = sm.cand_off[warp];
          const uint32_t n = (warp + 1 < static_cast<int>(G) ? sm.cand_off[warp + 1] : n_cand) - off;
          uint32_t gt = 0, eq = 0;
          for (uint32_t i = lane; i < n; i += 32) {
            const uint32_t kk = sm.gathered[off + i];
            gt += kk > T;
            eq += kk == T;
          }
          gt = warp_sum(gt);
          eq = warp_sum(eq);
          if (lane == 0) {
            sm.cnt_gt[warp] = sm.above_r[warp] + gt;
            sm.cnt_eq[warp] = eq;
          }
        }
      }
      __syncthreads();
    } else {
      // a bin too full to gather: cluster-wide radix levels over the
      // candidates' differing bits, each level one exchange of histograms
      uint32_t clo = 0xFFFFFFFFu, chi = 0u;
#pragma unroll
      for (int i = 0; i < C; i++)
        if (in_bin(i)) {
          clo = min(clo, key[i]);
          chi = max(chi, key[i]);
        }
      clo = cta_min(sm, clo);
      chi = cta_max(sm, chi);
      if (tid == 0) {
        sm.pub.cmin = clo;
        sm.pub.cmax = chi;
      }
      cluster_sync();
      uint32_t cmin = 0xFFFFFFFFu, cmax = 0u;
      for (uint32_t r = 0; r < G; r++) {
        cmin = min(cmin, ld_remote(&sm.pub.cmin, r));
        cmax = max(cmax, ld_remote(&sm.pub.cmax, r));
      }
      if (cmin == cmax) {
        T = cmin;
        need = rem;
      } else {
        int bits_left = 32 - __clz(cmin ^ cmax);
        uint32_t pmask = bits_left == 32 ? 0u : ~((1u << bits_left) - 1u);
        uint32_t prefix = cmin & pmask;
        int buf = 1;
        while (bits_left > 0) {
          const int w = min(8, bits_left);
          const int shift = bits_left - w;
          const uint32_t dmask = (1u << w) - 1u;
          __syncthreads();
          clear_whist(sm);
          __syncthreads();
#pragma unroll
          for (int i = 0; i < C; i++)
            if (in_bin(i) && (key[i] & pmask) == prefix) atomicAdd(&sm.whist[hg][(key[i] >> shift) & dmask], 1u);
          publish_hist(sm, buf);
          cluster_sync();
          cluster_find(sm, buf, 1 << w, rem, G);
          prefix |= sm.digit << shift;
          pmask |= dmask << shift;
          rem -= sm.above;
          bits_left -= w;
          buf ^= 1;
        }
        T = prefix;
        need = rem;
      }
    }
  };

  // ---- 1. the row's key range (and eligible count): from the scorer's score
  // bounds when given (the count then comes with the histogram), else a
  // cluster-wide min / max / eligible count / NaN exchange
  uint32_t kmin, kmax, n_elig = 0;
  const bool elig_known = stp == nullptr;
  cluster_wait_start();
  if (stp) {
    uint32_t bmax = st0.x, bmin = st0.y;
    for (int i = tid + kThreads; i < n_spans; i += kThreads) {
      const uint2 v = stp[i];
      bmax = max(bmax, v.x);
      bmin = min(bmin, v.y);
    }
    // one block reduction for both bounds
    {
      const int lane = tid & 31, warp = tid >> 5;
      bmax = __reduce_max_sync(0xFFFFFFFFu, bmax);
      bmin = __reduce_min_sync(0xFFFFFFFFu, bmin);
      if (lane == 0) {
        sm.red_a[warp] = bmax;
        sm.red_b[warp] = bmin;
      }
      __syncthreads();
      kmax = __reduce_max_sync(0xFFFFFFFFu, sm.red_a[lane]);
      kmin = __reduce_min_sync(0xFFFFFFFFu, sm.red_b[lane]);
    }
    if (nanf) raise_status(p.status, LIDX_DEV_NAN);
  } else {
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
      elig += __shfl_xor_sync(0xFFFFFFFFu, elig, o);
      nanf |= __shfl_xor_sync(0xFFFFFFFFu, nanf, o);
    }
    if (lane == 0) {
      sm.red_a[warp] = lo;
      sm.red_b[warp] = hi;
      sm.red_c[warp] = elig;
      sm.red_d[warp] = nanf;
    }
    __syncthreads();
    if (warp == 0) {
      lo = sm.red_a[lane];
      hi = sm.red_b[lane];
      elig = sm.red_c[lane];
      nanf = sm.red_d[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        elig += __shfl_xor_sync(0xFFFFFFFFu, elig, o);
        nanf |= __shfl_xor_sync(0xFFFFFFFFu, nanf, o);
      }
      if (lane == 0) {
        sm.pub.kmin = lo;
        sm.pub.kmax = hi;
        sm.pub.elig = elig;
        sm.pub.nan = nanf;
      }
    }
    cluster_sync();
    if (warp == 0) {  // lane r reads CTA r
      uint32_t a0 = 0xFFFFFFFFu, a1 = 0u, a2 = 0u, a3 = 0u;
      if (static_cast<uint32_t>(lane) < G) {
        a0 = ld_remote(&sm.pub.kmin, lane);
        a1 = ld_remote(&sm.pub.kmax, lane);
        a2 = ld_remote(&sm.pub.elig, lane);
        a3 = ld_remote(&sm.pub.nan, lane);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a0 = min(a0, __shfl_xor_sync(0xFFFFFFFFu, a0, o));
        a1 = max(a1, __shfl_xor_sync(0xFFFFFFFFu, a1, o));
        a2 += __shfl_xor_sync(0xFFFFFFFFu, a2, o);
        a3 |= __shfl_xor_sync(0xFFFFFFFFu, a3, o);
      }
      if (lane == 0) {
        sm.g[0] = a0;
        sm.g[1] = a1;
        sm.g[2] = a2;
        sm.g[3] = a3;
      }
    }
    __syncthreads();
    kmin = sm.g[0];
    kmax = sm.g[1];
    n_elig = sm.g[2];
    if (rank == 0 && tid == 0 && sm.g[3]) raise_status(p.status, LIDX_DEV_NAN);
  }

  // ---- 2./3. exact k-th key T and the number `need` of keys equal to T to take
  if (elig_known ? n_elig > static_cast<uint32_t>(k) : kmax != 0u) {
    uint32_t rem = static_cast<uint32_t>(k);
    if (elig_known && kmin == kmax) {
      T = kmax;
      need = rem;
    } else {
      const float flo = key_value(kmin), fhi = key_value(kmax);
      const float range = fhi - flo;
      const float scale0 = 256.f / range;
      const bool linear = isfinite(range) && range > 0.f && isfinite(scale0);
      const float scale = linear ? scale0 : 0.f;
      uint32_t pbin[(C + 3) / 4];
#pragma unroll
      for (int i = 0; i < (C + 3) / 4; i++) pbin[i] = 0u;
#pragma unroll
      for (int i = 0; i < C; i++) {
        uint32_t b = 0u;
        if (key[i]) {
          b = linear ? lin_bin(key[i], flo, scale) : (key[i] >> 24);
          atomicAdd(&sm.whist[hg][b], 1u);
        }
        pbin[i / 4] |= b << (8 * (i % 4));
      }
      auto in_lin_bin = [&](int i, uint32_t d) { return key[i] != 0u && ((pbin[i / 4] >> (8 * (i % 4))) & 0xFFu) == d; };
      push_hist(sm, G, rank);
      cluster_sync();
      sum_pushed_hist(sm, G, 256, rem);
      if (!elig_known && sm.total <= static_cast<uint32_t>(k)) {
        // at most k eligible keys: take them all (T = 0)
      } else if (!elig_known && kmin == kmax) {
        T = kmax;  // every eligible key equals the row's only value
        need = rem;
      } else {
        const uint32_t dbin = sm.digit;
        rem -= sm.above;
        resolve([&](int i) { return in_lin_bin(i, dbin); },
                [&](int i) { return key[i] != 0u && ((pbin[i / 4] >> (8 * (i % 4))) & 0xFFu) > dbin; }, rem);
      }
    }
  }

  // ---- 4. ordered emission
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < C; i++) {
    n_gt += T == 0u ? (key[i] != 0u) : (key[i] > T);
    n_eq += T != 0u && key[i] == T;
  }
  uint32_t cta_tot;
  int scan_buf = 0;
  const uint32_t ex = cta_exclusive_scan(sm, (n_gt << 16) | n_eq, cta_tot, scan_buf);  // at most 32768 each
  uint32_t gt_before = 0, eq_before = 0, gt_total = 0, eq_total = 0;
  if (fast) {
    for (uint32_t r = 0; r < G; r++) {
      const uint32_t g = sm.cnt_gt[r], e = sm.cnt_eq[r];
      if (r < rank) {
        gt_before += g;
        eq_before += e;
      }
      gt_total += g;
      eq_total += e;
    }
  } else {
    if (tid == 0) {
      sm.pub.gt = cta_tot >> 16;
      sm.pub.eq = cta_tot & 0xFFFFu;
    }
    cluster_sync();
    if (tid < 32) {  // lane r reads CTA r's counts
      const bool in = static_cast<uint32_t>(tid) < G;
      const uint32_t g = in ? ld_remote(&sm.pub.gt, tid) : 0u, e = in ? ld_remote(&sm.pub.eq, tid) : 0u;
      const uint32_t gi = warp_inclusive_scan(g), ei = warp_inclusive_scan(e);
      if (static_cast<uint32_t>(tid) == rank) {
        sm.g[0] = gi - g;
        sm.g[1] = ei - e;
      }
      if (tid == 31) {
        sm.g[2] = gi;
        sm.g[3] = ei;
      }
    }
    __syncthreads();
    gt_before = sm.g[0];
    eq_before = sm.g[1];
    gt_total = sm.g[2];
    eq_total = sm.g[3];
  }
  gt_before += ex >> 16;
  eq_before += ex & 0xFFFFu;
  uint32_t out = gt_before + min(eq_before, need);
  uint32_t eq_rank = eq_before;
  // never more than k ids, whatever the counts above say
  const uint32_t n_out = min(gt_total + min(eq_total, need), static_cast<uint32_t>(a.k));
  int32_t *ids = a.ids + static_cast<size_t>(grow) * a.k;
  uint32_t selbits = 0;
#pragma unroll
  for (int i = 0; i < C; i++) {
    const uint32_t kk = key[i];
    bool sel;
    if (T == 0u) {
      sel = kk != 0u;
    } else {
      sel = kk > T;
      if (kk == T) {
        sel = eq_rank < need;
        eq_rank++;
      }
    }
    if (sel) {
      if (out < static_cast<uint32_t>(a.k)) ids[out] = seg0 + s0 + p0 + i;
      out++;
      selbits |= 1u << i;
    }
  }
  if (rank == 0) {
    for (int i = static_cast<int>(n_out) + tid; i < a.k; i += kThreads) ids[i] = -1;
    if (tid == 0 && a.n_sel) a.n_sel[grow] = static_cast<int32_t>(n_out);
  }
  const int N = a.N;
  if (a.mask) {
    uint8_t *m = a.mask + static_cast<size_t>(row) * N + s0;
#pragma unroll
    for (int i = 0; i < C; i++)
      if (p0 + i < len) m[p0 + i] = static_cast<uint8_t>((selbits >> i) & 1u);
  }
  if (a.mask_bits) {
    const int Wn = (N + 31) / 32;
    const int w0 = s0 / 32;  // slices are multiples of 32 positions
    uint32_t *bw = a.mask_bits + static_cast<size_t>(row) * Wn + w0;
    const int wmax = Wn - w0;
    if (C == 32) {
      if (tid < wmax) bw[tid] = selbits;
    } else {
      uint32_t word = selbits << (p0 & 31);
#pragma unroll
      for (int o = 1; o < 32 / C; o <<= 1) word |= __shfl_xor_sync(0xFFFFFFFFu, word, o);
      const int wi = p0 >> 5;
      if ((p0 & 31) == 0 && wi < wmax) bw[wi] = word;
    }
  }
  // keep this CTA's shared memory alive until every CTA has read it (the
  // fast path reads no remote memory after its last barrier)
  if (!fast) cluster_sync();
}

template <int C>
size_t select_smem() {
  return ((sizeof(SelSmem) + 15) & ~size_t(15)) + (static_cast<size_t>(C) * kThreads + 4) * sizeof(float);
}

template <int C>
cudaError_t launch_c(int G, int rows, const SelParams &p, cudaStream_t st, bool pdl) {
  const size_t smem = select_smem<C>();
  cudaFuncSetAttribute(select_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  cudaFuncSetAttribute(select_kernel<C>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G, rows);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeClusterDimension;
  attr[n].val.clusterDim.x = G;
  attr[n].val.clusterDim.y = 1;
  attr[n].val.clusterDim.z = 1;
  n++;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    n++;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, select_kernel<C>, p);
}

// Whether the device schedules a 16-CTA cluster of the select kernel (a
// non-portable size), found once per device.
bool cluster16_ok() {
  static int cache[64] = {};  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return false;
  if (!cache[dev]) {
    cudaFuncSetAttribute(select_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(select_smem<32>()));
    cudaFuncSetAttribute(select_kernel<32>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = select_smem<32>();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, select_kernel<32>, &cfg);
    cudaGetLastError();
    cache[dev] = e == cudaSuccess && n >= 1 ? 1 : 2;
  }
  return cache[dev] == 1;
}

// Cluster size and items per thread for rows of N entries.
void plan(int N, int rows, int &G, int &C) {
  const int gmax = cluster16_ok() ? 16 : 8;
  G = 1;
  if (rows < 148) {
    G = 148 / rows;
    G = G >= gmax ? gmax : G >= 8 ? 8 : G >= 4 ? 4 : G >= 2 ? 2 : 1;
    while (G > 1 && (N + G - 1) / G < 2048) G >>= 1;  // keep slices worth a CTA
  }
  while ((N + G - 1) / G > kThreads * kMaxItems && G < gmax) G <<= 1;
  const int per = (N + G - 1) / G;
  C = 1;
  while (C * kThreads < per) C <<= 1;
}

cudaError_t launch_select(const SelParams &p, int grid_rows, int N, cudaStream_t st, bool pdl) {
  int G, C;
  plan(N, grid_rows, G, C);
  SelParams q = p;
  q.slice = C * kThreads;
  switch (C) {
    case 1: return launch_c<1>(G, grid_rows, q, st, pdl);
    case 2: return launch_c<2>(G, grid_rows, q, st, pdl);
    case 4: return launch_c<4>(G, grid_rows, q, st, pdl);
    case 8: return launch_c<8>(G, grid_rows, q, st, pdl);
    case 16: return launch_c<16>(G, grid_rows, q, st, pdl);
    default: return launch_c<32>(G, grid_rows, q, st, pdl);
  }
}

// ---- rows longer than one cluster holds: each segment's own top-k first
// (the row's top-k lies in the union of its segments' top-k: an entry with
// fewer than k entries ranked above it in the row has fewer than k above it
// in its segment), then the top-k of that union, whose candidates keep the
// row's index order so ties still go to the lower index.
// Longest row one cluster holds, and the segment length of longer rows (half
// a cluster's capacity): 524288 and 262144 positions with 16-CTA clusters,
// 262144 and 131072 with 8.
int max_row() { return (cluster16_ok() ? 16 : 8) * kThreads * kMaxItems; }
int seg_len() { return (cluster16_ok() ? 16 : 8) * kThreads * 16; }

struct BigRowWs {
  size_t seg_ids, seg_n, cand_s, cand_ok, ids2, total;
};

BigRowWs big_row_ws(const lidx_topk_args &a) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = static_cast<size_t>(a.B) * a.Q, n_seg = (a.N + seg_len() - 1) / seg_len();
  const size_t nc = n_seg * a.k;
  BigRowWs w{};
  size_t o = LIDX_WS_HEADER;
  w.seg_ids = o;
  o += up(rows * nc * 4);
  w.seg_n = o;
  o += up(rows * n_seg * 4);
  w.cand_s = o;
  o += up(rows * nc * 4);
  w.cand_ok = o;
  o += up(rows * nc);
  w.ids2 = o;
  o += up(rows * a.k * 4);
  w.total = o;
  return w;
}

// candidate c of row r: segment c / k, its i = c % k-th selected id
__global__ void __launch_bounds__(256) gather_candidates_kernel(const lidx_topk_args a, int n_seg,
                                                                const int32_t *seg_ids, const int32_t *seg_n,
                                                                float *cand_s, uint8_t *cand_ok) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.y, nc = n_seg * a.k;
  for (int c = blockIdx.x * 256 + threadIdx.x; c < nc; c += gridDim.x * 256) {
    const int sg = c / a.k, i = c % a.k;
    const size_t sr = static_cast<size_t>(r) * n_seg + sg;
    const int id = seg_ids[sr * a.k + i];
    const bool ok = i < seg_n[sr] && id >= 0 && id < a.N;
    cand_s[static_cast<size_t>(r) * nc + c] = ok ? a.scores[static_cast<size_t>(r) * a.ld_scores + id] : 0.f;
    cand_ok[static_cast<size_t>(r) * nc + c] = ok ? 1 : 0;
  }
}

// final ids: candidate positions back to row positions (still ascending);
// the optional mask and bit set of the row (cleared before this kernel)
__global__ void __launch_bounds__(256) map_candidates_kernel(const lidx_topk_args a, int n_seg,
                                                             const int32_t *seg_ids, const int32_t *ids2) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.y, nc = n_seg * a.k;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < a.k; i += gridDim.x * 256) {
    const int c = ids2[static_cast<size_t>(r) * a.k + i];
    int id = -1;
    if (c >= 0 && c < nc) id = seg_ids[(static_cast<size_t>(r) * n_seg + c / a.k) * a.k + c % a.k];
    a.ids[static_cast<size_t>(r) * a.k + i] = id;
    if (id >= 0) {
      if (a.mask) a.mask[static_cast<size_t>(r) * a.N + id] = 1;
      if (a.mask_bits) atomicOr(a.mask_bits + static_cast<size_t>(r) * ((a.N + 31) / 32) + id / 32, 1u << (id % 32));
    }
  }
}

cudaError_t launch_big_row(const lidx_topk_args &a, void *ws, cudaStream_t st, bool pdl) {
  const BigRowWs w = big_row_ws(a);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  int32_t *seg_ids = reinterpret_cast<int32_t *>(w8 + w.seg_ids), *seg_n = reinterpret_cast<int32_t *>(w8 + w.seg_n);
  float *cand_s = reinterpret_cast<float *>(w8 + w.cand_s);
  uint8_t *cand_ok = w8 + w.cand_ok;
  int32_t *ids2 = reinterpret_cast<int32_t *>(w8 + w.ids2);
  const int rows = a.B * a.Q, n_seg = (a.N + seg_len() - 1) / seg_len(), nc = n_seg * a.k;
  // 1. every segment's top-k, ids in row positions
  SelParams p1{};
  p1.a = a;
  p1.a.ids = seg_ids;
  p1.a.n_sel = seg_n;
  p1.a.mask = nullptr;
  p1.a.mask_bits = nullptr;
  p1.a.tile_stats = nullptr;
  p1.status = static_cast<uint32_t *>(ws);
  p1.n_seg = n_seg;
  p1.seg_len = seg_len();
  cudaError_t e = launch_select(p1, rows * n_seg, seg_len(), st, pdl);
  if (e != cudaSuccess) return e;
  // 2. their scores in row order, with an eligibility flag
  const dim3 g2((nc + 255) / 256 < 64 ? (nc + 255) / 256 : 64, rows);
  e = launch_kernel(gather_candidates_kernel, g2, dim3(256), 0, st, true, a, n_seg, seg_ids, seg_n, cand_s, cand_ok);
  if (e != cudaSuccess) return e;
  // 3. the top-k of the union
  SelParams p2{};
  p2.a = a;
  p2.a.B = rows;
  p2.a.Q = 1;
  p2.a.N = nc;
  p2.a.scores = cand_s;
  p2.a.ld_scores = nc;
  p2.a.allowed = cand_ok;
  p2.a.ld_allowed = nc;
  p2.a.allowed_bits = nullptr;
  p2.a.n_valid = nullptr;
  p2.a.ids = ids2;
  p2.a.mask = nullptr;
  p2.a.mask_bits = nullptr;
  p2.a.tile_stats = nullptr;
  p2.status = static_cast<uint32_t *>(ws);
  p2.n_seg = 1;
  p2.seg_len = nc;
  e = launch_select(p2, rows, nc, st, true);
  if (e != cudaSuccess) return e;
  // 4. back to row positions
  if (a.mask && (e = cudaMemsetAsync(a.mask, 0, static_cast<size_t>(rows) * a.N, st)) != cudaSuccess) return e;
  if (a.mask_bits &&
      (e = cudaMemsetAsync(a.mask_bits, 0, static_cast<size_t>(rows) * ((a.N + 31) / 32) * 4, st)) != cudaSuccess)
    return e;
  return launch_kernel(map_candidates_kernel, dim3((a.k + 255) / 256, rows), dim3(256), 0, st, true, a, n_seg,
                       seg_ids, ids2);
}

}  // namespace

bool topk_supported(const lidx_topk_args &a) {
  if (a.N <= max_row()) return true;
  const int64_t n_seg = (static_cast<int64_t>(a.N) + seg_len() - 1) / seg_len();
  return n_seg * a.k <= max_row();
}

size_t topk_workspace(const lidx_topk_args &a) { return a.N <= max_row() ? LIDX_WS_HEADER : big_row_ws(a).total; }

// one cluster select, or: segment selects, candidate gather, candidate select,
// map back (the mask clears are memsets, not kernels)
int topk_launches(const lidx_topk_args &a) { return a.N <= max_row() ? 1 : 4; }

cudaError_t launch_topk(const lidx_topk_args &a, void *ws, cudaStream_t st) {
  const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
  if (a.N > max_row()) return launch_big_row(a, ws, st, pdl);
  SelParams p{};
  p.a = a;
  p.status = static_cast<uint32_t *>(ws);
  p.n_seg = 1;
  p.seg_len = a.N;
  return launch_select(p, a.B * a.Q, a.N, st, pdl);
}

}  // namespace lidx
