// Top-k row ids by exact selection (DeepSeek-V4-Flash architecture post,
// section (B): keep the n_indexer_top_k highest-scoring compressed entries
// and hand their row ids, or the comp_allowed mask, to attention).
//
// Scores become order-preserving 32-bit keys (order_key: larger score ->
// larger key, -0 folded onto +0, NaN and disallowed entries -> 0).  One CTA of
// 512 threads selects within up to 32768 keys held in registers: thread t owns
// the contiguous positions [t*ITEMS, (t+1)*ITEMS).
//   1. One histogram pass over 256 linear value bins between the row's
//      minimum and maximum.  The bin is a monotone function of the score, so
//      the bin holding the k-th largest key, and the count above it, are
//      exact; for score-like distributions that bin holds a few dozen keys.
//   2. Those keys are compacted into shared memory and an exact radix select
//      over only their differing bits (8-bit digits, per-warp histograms)
//      pins the k-th key T and how many keys equal to T are taken.
//      Degenerate rows (a bin too full to compact) run the same radix over
//      the register-resident keys of that bin.
//   3. One packed 64-bit block scan of (#keys > T, #keys == T) per thread gives
//      each thread its output offset: ids come out ascending, ties resolved
//      toward the lower index.
//
// Rows longer than 32768 entries take two levels: chunks of 8192 keep their
// own top-k (the global top-k is a subset of the union, under the same total
// order), written as (key, index) candidates in index order, and one CTA per
// row selects from the candidates.
#include <algorithm>

#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxItems = 64;
constexpr int kSingleMax = kThreads * kMaxItems;  // 32768
constexpr int kChunk = 8192;

enum Mode { kRowFinal = 0, kRowCandidates = 1, kMergeFinal = 2 };

struct SelParams {
  lidx_topk_args a;
  uint32_t *status;
  int n_chunks;
  uint32_t *cand_key;  // [rows][n_chunks][k]
  int32_t *cand_idx;   // [rows][n_chunks][k]
  int32_t *cand_n;     // [rows][n_chunks]
  int kc;              // candidate slots per chunk = min(k, kChunk)
};

constexpr int kCandMax = 4096;

struct SelSmem {
  uint32_t whist[kWarps][256];  // per-warp histograms
  uint32_t hist[256];
  uint32_t cand[kCandMax];      // keys of the threshold bin
  unsigned long long warp_tot[kWarps];
  uint32_t red_a[kWarps], red_b[kWarps];
  uint32_t n_elig;
  uint32_t nan_seen;
  uint32_t n_cand;
  uint32_t digit;
  uint32_t above;
  uint32_t kmin, kmax;
  int32_t chunk_off[130];
};

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Block-wide min and max of per-thread values (results in sm.kmin / sm.kmax).
__device__ __forceinline__ void block_minmax(SelSmem &sm, uint32_t lo, uint32_t hi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  if (lane == 0) {
    sm.red_a[warp] = lo;
    sm.red_b[warp] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0xFFFFFFFFu, b = 0u;
    for (int w = 0; w < kWarps; w++) {
      a = min(a, sm.red_a[w]);
      b = max(b, sm.red_b[w]);
    }
    sm.kmin = a;
    sm.kmax = b;
  }
  __syncthreads();
}

__device__ __forceinline__ void whist_clear(SelSmem &sm) {
  uint32_t *h = &sm.whist[0][0];
  for (int i = threadIdx.x; i < kWarps * 256; i += kThreads) h[i] = 0u;
}

// Merge the per-warp histograms of `nbins` bins and find the bin holding the
// rem-th largest key counting from the top: sm.digit, sm.above (keys above it).
__device__ __forceinline__ void whist_find(SelSmem &sm, int nbins, uint32_t rem) {
  __syncthreads();
  if (threadIdx.x < 256) {
    uint32_t v = 0;
    if (static_cast<int>(threadIdx.x) < nbins)
#pragma unroll
      for (int w = 0; w < kWarps; w++) v += sm.whist[w][threadIdx.x];
    sm.hist[threadIdx.x] = v;
  }
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

__device__ __forceinline__ unsigned long long block_exclusive_scan_u64(SelSmem &sm, unsigned long long v,
                                                                        unsigned long long &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) sm.warp_tot[warp] = inc;
  __syncthreads();
  unsigned long long before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; w++) {
    const unsigned long long x = sm.warp_tot[w];
    before += (w < warp) ? x : 0ull;
    tot += x;
  }
  total = tot;
  return before + inc - v;
}

template <int ITEMS, int MODE>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelParams p) {
  __shared__ SelSmem sm;
  const lidx_topk_args &a = p.a;
  const int tid = threadIdx.x, lane = tid & 31;
  const int row = blockIdx.y;
  const int chunk = blockIdx.x;
  const int k = MODE == kRowCandidates ? p.kc : a.k;

  uint32_t key[ITEMS];
  int len;  // number of positions this CTA selects from
  pdl_trigger();
  pdl_wait();  // the scores / candidates come from the previous kernel
  if (tid == 0) {
    sm.n_elig = 0;
    sm.nan_seen = 0;
  }
  if (MODE == kMergeFinal) {
    if (tid == 0) {
      int off = 0;
      for (int c = 0; c < p.n_chunks; c++) {
        sm.chunk_off[c] = off;
        off += p.cand_n[row * p.n_chunks + c];
      }
      sm.chunk_off[p.n_chunks] = off;
    }
  }
  __syncthreads();
  if (MODE == kMergeFinal) {
    len = sm.chunk_off[p.n_chunks];
    int c = 0;
#pragma unroll
    for (int i = 0; i < ITEMS; i++) {
      const int pos = tid * ITEMS + i;
      key[i] = 0u;
      if (pos < len) {
        while (pos >= sm.chunk_off[c + 1]) c++;
        key[i] = p.cand_key[(static_cast<size_t>(row) * p.n_chunks + c) * p.kc + (pos - sm.chunk_off[c])];
      }
    }
  } else {
    const int j0 = MODE == kRowCandidates ? chunk * kChunk : 0;
    len = MODE == kRowCandidates ? min(kChunk, a.N - j0) : a.N;
    const float *s = a.scores + static_cast<size_t>(row) * a.ld_scores + j0;
    const uint8_t *al = a.allowed ? a.allowed + static_cast<size_t>(row / a.Q) * a.ld_allowed + j0 : nullptr;
    uint32_t nanf = 0;
    if (ITEMS % 4 == 0 && ((reinterpret_cast<uintptr_t>(s) & 15u) == 0) && (tid + 1) * ITEMS <= len) {
#pragma unroll
      for (int i = 0; i < ITEMS; i += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(s + tid * ITEMS + i);
        key[i] = order_key(v.x);
        key[i + 1] = order_key(v.y);
        key[i + 2] = order_key(v.z);
        key[i + 3] = order_key(v.w);
      }
    } else {
#pragma unroll
      for (int i = 0; i < ITEMS; i++) {
        const int pos = tid * ITEMS + i;
        key[i] = pos < len ? order_key(s[pos]) : 0u;
      }
    }
#pragma unroll
    for (int i = 0; i < ITEMS; i++) {
      const int pos = tid * ITEMS + i;
      if (pos < len) {
        if (key[i] == 0u && !(al && !al[pos])) nanf = 1u;
        if (al && !al[pos]) key[i] = 0u;
      }
    }
    if (nanf) sm.nan_seen = 1u;
  }
  uint32_t elig = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; i++) elig += key[i] != 0u;
  elig = warp_sum(elig);
  if (lane == 0 && elig) atomicAdd(&sm.n_elig, elig);
  __syncthreads();
  const uint32_t n_elig = sm.n_elig;
  if (MODE != kMergeFinal && tid == 0 && sm.nan_seen) raise_status(p.status, LIDX_DEV_NAN);

  // ---- exact k-th key T and the number `need` of keys equal to T to take
  uint32_t T = 0u, need = 0u;  // T = 0: take every eligible key
  if (n_elig > static_cast<uint32_t>(k)) {
    const int warp = tid >> 5;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int i = 0; i < ITEMS; i++)
      if (key[i]) {
        lo = min(lo, key[i]);
        hi = max(hi, key[i]);
      }
    block_minmax(sm, lo, hi);
    const uint32_t kmin = sm.kmin, kmax = sm.kmax;
    uint32_t rem = static_cast<uint32_t>(k);
    if (kmin == kmax) {
      T = kmax;
      need = rem;
    } else {
      // 1. linear value bins (monotone in the key)
      const float flo = key_value(kmin), fhi = key_value(kmax);
      const float range = fhi - flo;
      const float scale0 = 256.f / range;
      const bool linear = isfinite(range) && range > 0.f && isfinite(scale0);
      const float scale = linear ? scale0 : 0.f;
      auto bin_of = [&](uint32_t kk) -> uint32_t {
        if (!linear) return kk >> 24;
        const float t = (key_value(kk) - flo) * scale;
        return t >= 255.f ? 255u : static_cast<uint32_t>(t);
      };
      whist_clear(sm);
      if (tid == 0) sm.n_cand = 0;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < ITEMS; i++)
        if (key[i]) atomicAdd(&sm.whist[warp][bin_of(key[i])], 1u);
      whist_find(sm, 256, rem);
      const uint32_t dbin = sm.digit;
      rem -= sm.above;
      // 2. compact the threshold bin
#pragma unroll
      for (int i = 0; i < ITEMS; i++) {
        const bool c = key[i] != 0u && bin_of(key[i]) == dbin;
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, c);
        uint32_t base = 0;
        if (lane == 0 && bal) base = atomicAdd(&sm.n_cand, static_cast<uint32_t>(__popc(bal)));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
        if (c && pos < kCandMax) sm.cand[pos] = key[i];
      }
      __syncthreads();
      const uint32_t n_cand = sm.n_cand;
      const bool in_smem = n_cand <= static_cast<uint32_t>(kCandMax);
      // candidate source: the compacted list, or the register keys of the bin
      auto for_each_cand = [&](auto &&fn) {
        if (in_smem) {
          for (uint32_t i = tid; i < n_cand; i += kThreads) fn(sm.cand[i]);
        } else {
#pragma unroll
          for (int i = 0; i < ITEMS; i++)
            if (key[i] && bin_of(key[i]) == dbin) fn(key[i]);
        }
      };
      uint32_t clo = 0xFFFFFFFFu, chi = 0u;
      for_each_cand([&](uint32_t kk) {
        clo = min(clo, kk);
        chi = max(chi, kk);
      });
      block_minmax(sm, clo, chi);
      const uint32_t cmin = sm.kmin, cmax = sm.kmax;
      if (cmin == cmax) {
        T = cmin;
        need = rem;
      } else {
        // 3. radix over the differing bits of the candidates
        int bits_left = 32 - __clz(cmin ^ cmax);
        uint32_t prefix = cmin & (bits_left == 32 ? 0u : ~((1u << bits_left) - 1u));
        uint32_t pmask = bits_left == 32 ? 0u : ~((1u << bits_left) - 1u);
        while (bits_left > 0) {
          const int w = min(8, bits_left);
          const int shift = bits_left - w;
          const uint32_t dmask = (1u << w) - 1u;
          whist_clear(sm);
          __syncthreads();
          for_each_cand([&](uint32_t kk) {
            if ((kk & pmask) == prefix) atomicAdd(&sm.whist[warp][(kk >> shift) & dmask], 1u);
          });
          whist_find(sm, 1 << w, rem);
          prefix |= sm.digit << shift;
          pmask |= dmask << shift;
          rem -= sm.above;
          bits_left -= w;
        }
        T = prefix;
        need = rem;
      }
    }
  }

  // ---- ordered emission
  uint32_t n_gt = 0, n_eq = 0;
  if (T != 0u) {
#pragma unroll
    for (int i = 0; i < ITEMS; i++) {
      n_gt += key[i] > T;
      n_eq += key[i] == T;
    }
  } else {
#pragma unroll
    for (int i = 0; i < ITEMS; i++) n_gt += key[i] != 0u;
  }
  unsigned long long total;
  const unsigned long long ex = block_exclusive_scan_u64(sm, (static_cast<unsigned long long>(n_gt) << 32) | n_eq, total);
  const uint32_t gt_before = static_cast<uint32_t>(ex >> 32), eq_before = static_cast<uint32_t>(ex);
  uint32_t out = gt_before + min(eq_before, need);
  uint32_t eq_rank = eq_before;
  const uint32_t n_out = static_cast<uint32_t>(total >> 32) + min(static_cast<uint32_t>(total), need);

  uint64_t selbits = 0;
  int32_t *ids = nullptr;
  uint32_t *ckey = nullptr;
  int32_t *cidx = nullptr;
  if (MODE == kRowCandidates) {
    ckey = p.cand_key + (static_cast<size_t>(row) * p.n_chunks + chunk) * p.kc;
    cidx = p.cand_idx + (static_cast<size_t>(row) * p.n_chunks + chunk) * p.kc;
  } else {
    ids = a.ids + static_cast<size_t>(row) * a.k;
  }
  int c = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; i++) {
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
      const int pos = tid * ITEMS + i;
      if (MODE == kRowCandidates) {
        ckey[out] = kk;
        cidx[out] = chunk * kChunk + pos;
      } else if (MODE == kRowFinal) {
        ids[out] = pos;
      } else {
        while (pos >= sm.chunk_off[c + 1]) c++;
        ids[out] = p.cand_idx[(static_cast<size_t>(row) * p.n_chunks + c) * p.kc + (pos - sm.chunk_off[c])];
      }
      out++;
      if (ITEMS <= 64) selbits |= 1ull << i;
    }
  }
  if (MODE == kRowCandidates) {
    if (tid == 0) p.cand_n[row * p.n_chunks + chunk] = static_cast<int32_t>(n_out);
    return;
  }
  for (int i = static_cast<int>(n_out) + tid; i < a.k; i += kThreads) ids[i] = -1;
  if (tid == 0 && a.n_sel) a.n_sel[row] = static_cast<int32_t>(n_out);
  if (MODE == kRowFinal) {
    const int N = a.N;
    if (a.mask) {
      uint8_t *m = a.mask + static_cast<size_t>(row) * N;
#pragma unroll
      for (int i = 0; i < ITEMS; i++) {
        const int pos = tid * ITEMS + i;
        if (pos < N) m[pos] = static_cast<uint8_t>((selbits >> i) & 1u);
      }
    }
    if (a.mask_bits) {
      const int Wn = (N + 31) / 32;
      uint32_t *bw = a.mask_bits + static_cast<size_t>(row) * Wn;
      if (ITEMS >= 32) {
#pragma unroll
        for (int w = 0; w < ITEMS / 32; w++) {
          const int wi = tid * (ITEMS / 32) + w;
          if (wi < Wn) bw[wi] = static_cast<uint32_t>(selbits >> (32 * w));
        }
      } else {
        uint32_t word = static_cast<uint32_t>(selbits) << ((tid * ITEMS) & 31);
#pragma unroll
        for (int o = 1; o < 32 / ITEMS; o <<= 1) word |= __shfl_xor_sync(0xFFFFFFFFu, word, o);
        const int wi = (tid * ITEMS) >> 5;
        if (((tid * ITEMS) & 31) == 0 && wi < Wn) bw[wi] = word;
      }
    }
  }
}

// mask / bit set from final ids (two-level path)
__global__ void mask_from_ids_kernel(lidx_topk_args a) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.y;
  const int N = a.N, Wn = (N + 31) / 32;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < N; j += gridDim.x * blockDim.x) {
    if (a.mask) a.mask[static_cast<size_t>(row) * N + j] = 0;
  }
  if (a.mask_bits)
    for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < Wn; w += gridDim.x * blockDim.x)
      a.mask_bits[static_cast<size_t>(row) * Wn + w] = 0u;
}

__global__ void mask_scatter_kernel(lidx_topk_args a) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.y;
  const int N = a.N, Wn = (N + 31) / 32;
  const int32_t *ids = a.ids + static_cast<size_t>(row) * a.k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.k; i += gridDim.x * blockDim.x) {
    const int j = ids[i];
    if (j < 0 || j >= N) continue;
    if (a.mask) a.mask[static_cast<size_t>(row) * N + j] = 1;
    if (a.mask_bits) atomicOr(&a.mask_bits[static_cast<size_t>(row) * Wn + (j >> 5)], 1u << (j & 31));
  }
}

template <int MODE>
cudaError_t launch_items(int items, dim3 grid, const SelParams &p, cudaStream_t st) {
  const bool pdl = (p.a.flags & LIDX_LAUNCH_PDL) != 0;
  const dim3 blk(kThreads);
  switch (items) {
    case 1: return launch_kernel(select_kernel<1, MODE>, grid, blk, 0, st, pdl, p);
    case 2: return launch_kernel(select_kernel<2, MODE>, grid, blk, 0, st, pdl, p);
    case 4: return launch_kernel(select_kernel<4, MODE>, grid, blk, 0, st, pdl, p);
    case 8: return launch_kernel(select_kernel<8, MODE>, grid, blk, 0, st, pdl, p);
    case 16: return launch_kernel(select_kernel<16, MODE>, grid, blk, 0, st, pdl, p);
    case 32: return launch_kernel(select_kernel<32, MODE>, grid, blk, 0, st, pdl, p);
    default: return launch_kernel(select_kernel<64, MODE>, grid, blk, 0, st, pdl, p);
  }
}

int items_for(int len) {
  int it = 1;
  while (it * kThreads < len) it <<= 1;
  return it;
}

bool two_level(const lidx_topk_args &a) { return a.N > kSingleMax; }

int n_chunks_of(const lidx_topk_args &a) { return (a.N + kChunk - 1) / kChunk; }

size_t cand_bytes(const lidx_topk_args &a) {
  const size_t rows = static_cast<size_t>(a.B) * a.Q;
  const size_t slots = rows * n_chunks_of(a) * std::min(a.k, kChunk);
  return ((slots * 4 + 255) / 256) * 256 * 2 + ((rows * n_chunks_of(a) * 4 + 255) / 256) * 256;
}

}  // namespace

bool topk_supported(const lidx_topk_args &a) {
  if (!two_level(a)) return true;
  return static_cast<long long>(n_chunks_of(a)) * std::min(a.k, kChunk) <= kSingleMax && n_chunks_of(a) <= 128;
}

size_t topk_workspace(const lidx_topk_args &a) {
  return LIDX_WS_HEADER + (two_level(a) ? cand_bytes(a) : 0);
}

cudaError_t launch_topk(const lidx_topk_args &a, void *ws, cudaStream_t st) {
  SelParams p{};
  p.a = a;
  p.status = static_cast<uint32_t *>(ws);
  const int rows = a.B * a.Q;
  if (!two_level(a)) {
    return launch_items<kRowFinal>(items_for(a.N), dim3(1, rows), p, st);
  }
  p.n_chunks = n_chunks_of(a);
  p.kc = std::min(a.k, kChunk);
  const size_t rows_s = static_cast<size_t>(rows);
  const size_t slots = rows_s * p.n_chunks * p.kc;
  char *cur = static_cast<char *>(ws) + LIDX_WS_HEADER;
  p.cand_key = reinterpret_cast<uint32_t *>(cur);
  cur += ((slots * 4 + 255) / 256) * 256;
  p.cand_idx = reinterpret_cast<int32_t *>(cur);
  cur += ((slots * 4 + 255) / 256) * 256;
  p.cand_n = reinterpret_cast<int32_t *>(cur);
  cudaError_t e = launch_items<kRowCandidates>(kChunk / kThreads, dim3(p.n_chunks, rows), p, st);
  if (e != cudaSuccess) return e;
  e = launch_items<kMergeFinal>(items_for(p.n_chunks * p.kc), dim3(1, rows), p, st);
  if (e != cudaSuccess) return e;
  if (a.mask || a.mask_bits) {
    const bool pdl = (a.flags & LIDX_LAUNCH_PDL) != 0;
    e = launch_kernel(mask_from_ids_kernel, dim3(32, rows), dim3(256), 0, st, pdl, a);
    if (e == cudaSuccess) e = launch_kernel(mask_scatter_kernel, dim3(1, rows), dim3(256), 0, st, pdl, a);
  }
  return e;
}

}  // namespace lidx
