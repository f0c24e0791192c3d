// Top-k row ids by exact selection (DeepSeek-V4-Flash architecture post,
// section (B): keep the n_indexer_top_k highest-scoring compressed entries
// and hand their row ids, or the comp_allowed mask, to attention).
//
// Scores become order-preserving 32-bit keys (order_key: larger score ->
// larger key, -0 folded onto +0, NaN and disallowed entries -> 0).  One CTA of
// 1024 threads selects within up to 32768 keys held in registers: thread t
// owns the contiguous positions [t*C, (t+1)*C), all loaded up front.
//   1. One histogram pass over 256 linear value bins between the row's
//      minimum and maximum (found during the load).  The bin is a monotone
//      function of the score, so the bin holding the k-th largest key, and
//      the count above it, are exact; for score-like distributions that bin
//      holds a few dozen keys.
//   2. A block scan compacts that bin into shared memory; each candidate
//      counts the candidates above and equal to it, which pins the k-th key
//      T and how many keys equal to T are taken.  A bin too full for this
//      runs an exact radix over the candidates' differing bits instead.
//   3. One packed 64-bit block scan of (#keys > T, #keys == T) per thread gives
//      each thread its output offset: ids come out ascending, ties resolved
//      toward the lower index.
// Every phase costs a few instructions per key; the few block barriers are
// the floor.
//
// Rows longer than 32768 entries take two levels: chunks of 8192 keep their
// own top-k (the global top-k is a subset of the union, under the same total
// order), written as (key, index) candidates in index order, and one CTA per
// row selects from the candidates.
#include <algorithm>

#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxItems = 32;
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
constexpr int kRankMax = 1024;  // candidates resolved by direct rank counting

struct SelSmem {
  uint32_t whist[8][256];       // histograms shared by groups of four warps
  uint32_t hist[256];
  uint32_t cand[kCandMax];      // keys of the threshold bin
  uint32_t red_a[kWarps], red_b[kWarps];
  uint32_t red_tot;
  uint32_t n_elig;
  uint32_t nan_seen;
  uint32_t n_cand;
  uint32_t digit;
  uint32_t above;
  uint32_t kmin, kmax;
  int32_t chunk_off[130];
  uint64_t bar;
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
  for (int i = threadIdx.x; i < 8 * 256; i += kThreads) h[i] = 0u;
}

// Merge the per-warp histograms of `nbins` bins and find the bin holding the
// rem-th largest key counting from the top: sm.digit, sm.above (keys above it).
__device__ __forceinline__ void whist_find(SelSmem &sm, int nbins, uint32_t rem) {
  __syncthreads();
  if (threadIdx.x < 256) {
    uint32_t v = 0;
    if (static_cast<int>(threadIdx.x) < nbins)
#pragma unroll
      for (int w = 0; w < 8; w++) v += sm.whist[w][threadIdx.x];
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

// Exclusive block scan of 32-bit values; warp totals are scanned by one warp.
// Returns the thread's exclusive prefix; *total gets the block sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(SelSmem &sm, uint32_t v, uint32_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t inc = warp_inclusive_scan(v);
  if (lane == 31) sm.red_a[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = sm.red_a[lane];
    const uint32_t xi = warp_inclusive_scan(x);
    sm.red_b[lane] = xi - x;
    if (lane == 31) sm.red_tot = xi;
  }
  __syncthreads();
  total = sm.red_tot;
  return sm.red_b[warp] + inc - v;
}

// Monotone 8-bit bin of a key inside [flo, flo + 256/scale]: round((x-flo)*scale)
// read off the mantissa of x*scale + 2^23 (no float-to-int conversion).
__device__ __forceinline__ uint32_t lin_bin(uint32_t kk, float flo, float scale) {
  const float t = fmaf(key_value(kk) - flo, scale, 8388608.f);
  return min(__float_as_uint(t) - 0x4B000000u, 255u);
}

template <int C, int MODE>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) float rowbuf[];  // the row's scores (row modes)
  __shared__ SelSmem sm;
  const lidx_topk_args &a = p.a;
  const int tid = threadIdx.x, lane = tid & 31;
  const int hg = (tid >> 5) & 7;  // histogram group
  const int row = blockIdx.y;
  const int chunk = blockIdx.x;
  const int k = MODE == kRowCandidates ? p.kc : a.k;
  const int p0 = tid * C;

  pdl_trigger();
  pdl_wait();  // the scores / candidates come from the previous kernel
  if (tid == 0) {
    sm.n_elig = 0;
    sm.nan_seen = 0;
    sm.n_cand = 0;
    if (MODE == kMergeFinal) {
      int off = 0;
      for (int c = 0; c < p.n_chunks; c++) {
        sm.chunk_off[c] = off;
        off += p.cand_n[row * p.n_chunks + c];
      }
      sm.chunk_off[p.n_chunks] = off;
    }
  }
  whist_clear(sm);
  __syncthreads();

  // ---- keys into registers
  uint32_t key[C];
  int len;
  if (MODE == kMergeFinal) {
    len = sm.chunk_off[p.n_chunks];
    int c = 0;
#pragma unroll
    for (int i = 0; i < C; i++) {
      const int pos = p0 + i;
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
    // one bulk copy of the 16-byte-aligned body of the row into shared memory
    const int head = static_cast<int>(((16u - (reinterpret_cast<uintptr_t>(s) & 15u)) & 15u) / 4u);
    const int body = max(0, (len - head)) & ~3;
    // shift the buffer so the body lands 16-byte aligned in shared memory too
    float *sv = rowbuf + ((4 - head) & 3);
    if (tid == 0) {
      tc::mbar_init(&sm.bar, 1);
      tc::fence_barrier_init();
    }
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
    uint32_t nanf = 0;
#pragma unroll
    for (int i = 0; i < C; i++) {
      const int pos = p0 + i;
      uint32_t kk = pos < len ? order_key(sv[pos]) : 0u;
      if (pos < len && kk == 0u && !(al && !al[pos])) nanf = 1u;
      if (al && pos < len && !al[pos]) kk = 0u;
      key[i] = kk;
    }
    if (nanf) sm.nan_seen = 1u;
  }
  uint32_t elig = 0, lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int i = 0; i < C; i++) {
    if (key[i]) {
      elig++;
      lo = min(lo, key[i]);
      hi = max(hi, key[i]);
    }
  }
  elig = warp_sum(elig);
  if (lane == 0 && elig) atomicAdd(&sm.n_elig, elig);
  block_minmax(sm, lo, hi);  // includes the barrier that publishes n_elig
  const uint32_t n_elig = sm.n_elig;
  const uint32_t kmin = sm.kmin, kmax = sm.kmax;
  if (MODE != kMergeFinal && tid == 0 && sm.nan_seen) raise_status(p.status, LIDX_DEV_NAN);

  // ---- exact k-th key T and the number `need` of keys equal to T to take
  uint32_t T = 0u, need = 0u;  // T = 0: take every eligible key
  if (n_elig > static_cast<uint32_t>(k)) {
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
      // bins computed once, four per register; 0xFF..: no key (bins are 0..255)
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
      auto bin_at = [&](int i) -> uint32_t { return (pbin[i / 4] >> (8 * (i % 4))) & 0xFFu; };
      whist_find(sm, 256, rem);
      const uint32_t dbin = sm.digit;
      rem -= sm.above;
      // 2. compact the threshold bin (index order, by block scan)
      uint32_t nc = 0;
#pragma unroll
      for (int i = 0; i < C; i++) nc += key[i] != 0u && bin_at(i) == dbin;
      uint32_t n_cand;
      uint32_t cpos = block_exclusive_scan(sm, nc, n_cand);
#pragma unroll
      for (int i = 0; i < C; i++)
        if (key[i] != 0u && bin_at(i) == dbin) {
          if (cpos < kCandMax) sm.cand[cpos] = key[i];
          cpos++;
        }
      __syncthreads();
      if (n_cand <= static_cast<uint32_t>(kRankMax)) {
        // 3a. each candidate counts the candidates above / equal to it
        if (tid < static_cast<int>(n_cand)) {
          const uint32_t mine = sm.cand[tid];
          uint32_t gt = 0, eq = 0;
          for (uint32_t j = 0; j < n_cand; j++) {
            const uint32_t o = sm.cand[j];
            gt += o > mine;
            eq += o == mine;
          }
          if (gt < rem && gt + eq >= rem) {
            sm.kmin = mine;        // T
            sm.kmax = rem - gt;    // need
          }
        }
        __syncthreads();
        T = sm.kmin;
        need = sm.kmax;
      } else {
        // 3b. radix over the differing bits of the candidates
        const bool in_list = n_cand <= static_cast<uint32_t>(kCandMax);
        auto for_each_cand = [&](auto &&fn) {
          if (in_list) {
            for (uint32_t i = tid; i < n_cand; i += kThreads) fn(sm.cand[i]);
          } else {
#pragma unroll
            for (int i = 0; i < C; i++)
              if (key[i] != 0u && bin_at(i) == dbin) fn(key[i]);
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
          int bits_left = 32 - __clz(cmin ^ cmax);
          uint32_t pmask = bits_left == 32 ? 0u : ~((1u << bits_left) - 1u);
          uint32_t prefix = cmin & pmask;
          while (bits_left > 0) {
            const int w = min(8, bits_left);
            const int shift = bits_left - w;
            const uint32_t dmask = (1u << w) - 1u;
            __syncthreads();
            whist_clear(sm);
            __syncthreads();
            for_each_cand([&](uint32_t kk) {
              if ((kk & pmask) == prefix) atomicAdd(&sm.whist[hg][(kk >> shift) & dmask], 1u);
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
  }

  // ---- ordered emission
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < C; i++) {
    if (T == 0u) {
      n_gt += key[i] != 0u;
    } else {
      n_gt += key[i] > T;
      n_eq += key[i] == T;
    }
  }
  uint32_t total;
  __syncthreads();
  // (#gt << 16) | #eq: both at most 32768 per CTA
  const uint32_t ex = block_exclusive_scan(sm, (n_gt << 16) | n_eq, total);
  const uint32_t gt_before = ex >> 16, eq_before = ex & 0xFFFFu;
  uint32_t out = gt_before + min(eq_before, need);
  uint32_t eq_rank = eq_before;
  const uint32_t n_out = (total >> 16) + min(total & 0xFFFFu, need);

  uint32_t selbits = 0;
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
  for (int i = 0; i < C; i++) {
    const int pos = p0 + i;
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
      selbits |= 1u << i;
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
      for (int i = 0; i < C; i++)
        if (p0 + i < N) m[p0 + i] = static_cast<uint8_t>((selbits >> i) & 1u);
    }
    if (a.mask_bits) {
      const int Wn = (N + 31) / 32;
      uint32_t *bw = a.mask_bits + static_cast<size_t>(row) * Wn;
      if (C == 32) {
        if (tid < Wn) bw[tid] = selbits;
      } else {
        uint32_t word = selbits << (p0 & 31);
#pragma unroll
        for (int o = 1; o < 32 / C; o <<= 1) word |= __shfl_xor_sync(0xFFFFFFFFu, word, o);
        const int wi = p0 >> 5;
        if ((p0 & 31) == 0 && wi < Wn) bw[wi] = word;
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

template <int C, int MODE>
cudaError_t launch_c(dim3 grid, const SelParams &p, cudaStream_t st, bool pdl) {
  const size_t smem = MODE == kMergeFinal ? 0 : (static_cast<size_t>(C) * kThreads + 4) * sizeof(float);
  // static + dynamic shared memory exceeds the default 48 KB window
  cudaFuncSetAttribute(select_kernel<C, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  return launch_kernel(select_kernel<C, MODE>, grid, dim3(kThreads), smem, st, pdl, p);
}

template <int MODE>
cudaError_t launch_items(int items, dim3 grid, const SelParams &p, cudaStream_t st) {
  const bool pdl = (p.a.flags & LIDX_LAUNCH_PDL) != 0;
  switch (items) {
    case 1: return launch_c<1, MODE>(grid, p, st, pdl);
    case 2: return launch_c<2, MODE>(grid, p, st, pdl);
    case 4: return launch_c<4, MODE>(grid, p, st, pdl);
    case 8: return launch_c<8, MODE>(grid, p, st, pdl);
    case 16: return launch_c<16, MODE>(grid, p, st, pdl);
    default: return launch_c<32, MODE>(grid, p, st, pdl);
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
