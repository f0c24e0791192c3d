// Top-k row ids by exact radix select (DeepSeek-V4-Flash architecture post,
// section (B): keep the n_indexer_top_k highest-scoring compressed entries
// and hand their row ids, or the comp_allowed mask, to attention).
//
// One CTA of 1024 threads per (b,t) row.  Scores become order-preserving
// 32-bit keys (see order_key); four 8-bit digit passes, each a shared-memory
// histogram built with warp-aggregated atomics (__match_any_sync), pin the
// exact k-th key T and how many entries equal to T are taken.  A final pass
// in index order emits ids ascending with a ballot/prefix compaction: every
// key > T, and the lowest-index entries == T until k are reached.  When the
// row fits, keys are staged in shared memory once; otherwise each pass
// re-reads the scores (L2-resident right after scoring).
#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kT = 1024;
constexpr int kWarps = kT / 32;
constexpr int kMaxSmemKeys = 50 * 1024;  // 200 KB of keys

struct TopkSmem {
  uint32_t hist[256];
  uint32_t warp_a[kWarps];
  uint32_t warp_b[kWarps];
  uint32_t n_elig;
  uint32_t nan_seen;
  uint32_t digit;
  uint32_t above;
  uint32_t tot_a, tot_b;
};

__device__ __forceinline__ uint32_t key_of(const float *s, const uint8_t *al, int j, uint32_t *nan_flag) {
  if (al && !al[j]) return 0u;
  float x = s[j];
  uint32_t k = order_key(x);
  if (k == 0u) *nan_flag = 1u;
  return k;
}

// Exclusive block scan of two 0/1 predicates in index order; returns the
// thread's exclusive offsets and (through smem) the block totals.
__device__ __forceinline__ void block_scan2(TopkSmem &sm, bool pa, bool pb, uint32_t &oa, uint32_t &ob) {
  const uint32_t lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t ba = __ballot_sync(0xFFFFFFFFu, pa), bb = __ballot_sync(0xFFFFFFFFu, pb);
  const uint32_t lt = (1u << lane) - 1u;
  if (lane == 0) {
    sm.warp_a[warp] = __popc(ba);
    sm.warp_b[warp] = __popc(bb);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t va = sm.warp_a[lane], vb = sm.warp_b[lane];
    uint32_t ia = warp_inclusive_scan(va), ib = warp_inclusive_scan(vb);
    sm.warp_a[lane] = ia - va;
    sm.warp_b[lane] = ib - vb;
    if (lane == 31) {
      sm.tot_a = ia;
      sm.tot_b = ib;
    }
  }
  __syncthreads();
  oa = sm.warp_a[warp] + __popc(ba & lt);
  ob = sm.warp_b[warp] + __popc(bb & lt);
}

template <bool kSmem>
__global__ void __launch_bounds__(kT, 1) topk_kernel(lidx_topk_args a, uint32_t *status) {
  extern __shared__ uint32_t skeys[];
  __shared__ TopkSmem sm;
  const int row = blockIdx.x;
  const int b = row / a.Q;
  const int N = a.N;
  const float *s = a.scores + static_cast<size_t>(row) * a.ld_scores;
  const uint8_t *al = a.allowed ? a.allowed + static_cast<size_t>(b) * a.ld_allowed : nullptr;
  const int tid = threadIdx.x;
  const uint32_t lane = lane_id();

  if (tid == 0) {
    sm.n_elig = 0;
    sm.nan_seen = 0;
  }
  __syncthreads();
  uint32_t nan_flag = 0, elig = 0;
  for (int j = tid; j < N; j += kT) {
    uint32_t k = key_of(s, al, j, &nan_flag);
    if (kSmem) skeys[j] = k;
    elig += (k != 0u);
  }
  elig = warp_sum(elig);
  if (lane == 0 && elig) atomicAdd(&sm.n_elig, elig);
  if (nan_flag) sm.nan_seen = 1u;
  __syncthreads();
  const uint32_t n_elig = sm.n_elig;
  if (tid == 0 && sm.nan_seen) raise_status(status, LIDX_DEV_NAN);

  auto get = [&](int j) -> uint32_t {
    if (kSmem) return skeys[j];
    uint32_t dummy;
    return key_of(s, al, j, &dummy);
  };

  // ---- radix descent to the exact k-th key
  uint32_t T = 0u, need = 0u;  // T = 0: take every eligible entry
  if (n_elig > static_cast<uint32_t>(a.k)) {
    uint32_t prefix = 0u, pmask = 0u, rem = static_cast<uint32_t>(a.k);
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) sm.hist[tid] = 0u;
      __syncthreads();
      for (int base = 0; base < N; base += kT) {
        const int j = base + tid;
        uint32_t d = 0xFFFFFFFFu;
        if (j < N) {
          uint32_t k = get(j);
          if (k != 0u && (k & pmask) == prefix) d = (k >> shift) & 0xFFu;
        }
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, d);
        if (d != 0xFFFFFFFFu && lane == static_cast<uint32_t>(__ffs(peers) - 1))
          atomicAdd(&sm.hist[d], static_cast<uint32_t>(__popc(peers)));
      }
      __syncthreads();
      // suffix counts from the top digit down: thread i looks at digit 255-i
      if (tid < 256) {
        const uint32_t v = sm.hist[255 - tid];
        uint32_t inc = warp_inclusive_scan(v);
        if (lane == 31) sm.warp_a[tid >> 5] = inc;
        __syncwarp();
        // wait for the 8 warp totals
        asm volatile("bar.sync 1, 256;");
        uint32_t before = 0;
        for (int w = 0; w < (tid >> 5); w++) before += sm.warp_a[w];
        inc += before;
        if (inc >= rem && inc - v < rem) {
          sm.digit = 255u - tid;
          sm.above = inc - v;
        }
      }
      __syncthreads();
      prefix |= sm.digit << shift;
      pmask |= 0xFFu << shift;
      rem -= sm.above;
      __syncthreads();
    }
    T = prefix;
    need = rem;
  }

  // ---- ordered compaction: ids ascending, mask, bit set
  int32_t *ids = a.ids + static_cast<size_t>(row) * a.k;
  uint32_t out_base = 0, eq_seen = 0;
  const int Wn = (N + 31) / 32;
  for (int base = 0; base < N; base += kT) {
    const int j = base + tid;
    const uint32_t k = j < N ? get(j) : 0u;
    const bool gt = k > T;
    const bool eq = (k == T) && (k != 0u);
    uint32_t o_eq, o_dummy;
    block_scan2(sm, eq, false, o_eq, o_dummy);
    const uint32_t tot_eq = sm.tot_a;
    const bool sel = gt || (eq && eq_seen + o_eq < need);
    uint32_t o_sel;
    __syncthreads();
    block_scan2(sm, sel, false, o_sel, o_dummy);
    const uint32_t tot_sel = sm.tot_a;
    if (sel) ids[out_base + o_sel] = j;
    if (a.mask && j < N) a.mask[static_cast<size_t>(row) * N + j] = sel ? 1 : 0;
    if (a.mask_bits) {
      const uint32_t word = __ballot_sync(0xFFFFFFFFu, sel);
      const int wi = (base >> 5) + static_cast<int>(threadIdx.x >> 5);
      if (lane == 0 && wi < Wn) a.mask_bits[static_cast<size_t>(row) * Wn + wi] = word;
    }
    out_base += tot_sel;
    eq_seen += tot_eq;
    __syncthreads();
  }
  for (int i = static_cast<int>(out_base) + tid; i < a.k; i += kT) ids[i] = -1;
  if (tid == 0 && a.n_sel) a.n_sel[row] = static_cast<int32_t>(out_base);
}

}  // namespace

size_t topk_workspace(const lidx_topk_args &) { return LIDX_WS_HEADER; }

cudaError_t launch_topk(const lidx_topk_args &a, void *ws, cudaStream_t st) {
  uint32_t *status = static_cast<uint32_t *>(ws);
  const int rows = a.B * a.Q;
  if (a.N <= kMaxSmemKeys) {
    const size_t smem = static_cast<size_t>(a.N) * sizeof(uint32_t);
    cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    topk_kernel<true><<<rows, kT, smem, st>>>(a, status);
  } else {
    topk_kernel<false><<<rows, kT, 0, st>>>(a, status);
  }
  return cudaGetLastError();
}

}  // namespace lidx
