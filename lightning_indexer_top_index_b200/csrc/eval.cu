// Selection evaluation over a tau-window.
//
//  GOLDEN  dense-attention ground truth (FlashMemory-vs-native post, Act 3;
//          FlashMemory deep-dive write-up, section 3.2 step 1):
//          p[l,t,j] = (1/H) sum_h softmax_j(scale * qa[l,t,h] . x_l[j]).
//          Pass 1 gives the per-(l,t,h) log-sum-exp, pass 2 the head mean.
//  TOPP    nucleus set per (l,t) (write-up 3.2 step 2), exact in fixed point.
//  VOTE    >= min_votes of the L layers (write-up 3.2 step 3), union over t.
//  LSA     sigmoid(logit + bias) >= 0.5, OR over gate layers (write-up 2.2,
//          4.1).
//  OVERLAP |A & B|, |A|, |B| (FlashMemory-vs-native post, Acts 1 and 3).
#include "kernels.cuh"

namespace lidx {

namespace {

constexpr int kD = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int KT>
__device__ __forceinline__ float row_elem(const lidx_kv &k, int64_t row, int d) {
  if constexpr (KT == LIDX_F32) return static_cast<const float *>(k.data)[row * k.ld + d];
  if constexpr (KT == LIDX_BF16) return bf16_to_f32(static_cast<const uint16_t *>(k.data)[row * k.ld + d]);
  if (d < k.dim - 64)
    return e4m3_to_f32(static_cast<const uint8_t *>(k.data)[row * k.ld + d]) *
           e8m0_to_f32(k.scale[row * k.ld_scale + d / 64]);
  return bf16_to_f32(static_cast<const uint16_t *>(k.rope)[row * k.ld_rope + d - (k.dim - 64)]);
}

__device__ __forceinline__ float q_elem(const void *q, int dt, size_t i) {
  return dt == LIDX_F32 ? static_cast<const float *>(q)[i] : bf16_to_f32(static_cast<const uint16_t *>(q)[i]);
}

// ---- GOLDEN pass 1: lse2[l,t,h] = log2 sum_j 2^(c * qa . x_j), c = scale*log2(e)
template <int KT>
__global__ void __launch_bounds__(256) golden_lse_kernel(lidx_eval_args a, float *lse2) {
  __shared__ float q_s[kD];
  __shared__ float red_m[8], red_s[8];
  const int lth = blockIdx.x;  // (l*T + t)*H + h
  const int l = lth / (a.T * a.H);
  const float c = a.scale * kLog2e;
  for (int d = threadIdx.x; d < kD; d += 256) q_s[d] = q_elem(a.qa, a.qa_dtype, static_cast<size_t>(lth) * kD + d) * c;
  __syncthreads();
  float m = -INFINITY, s = 0.f;
  for (int j = threadIdx.x; j < a.N; j += 256) {
    const int64_t row = static_cast<int64_t>(l) * a.kv.batch_rows + j;
    float acc = 0.f;
    for (int d = 0; d < kD; d++) acc = fmaf(q_s[d], row_elem<KT>(a.kv, row, d), acc);
    const float mn = fmaxf(m, acc);
    s = s * exp2f(m - mn) + exp2f(acc - mn);
    m = mn;
  }
  // combine (m, s) pairs
  const float M = warp_max(m);
  s = (m == -INFINITY) ? 0.f : s * exp2f(m - M);
  s = warp_sum(s);
  if (lane_id() == 0) {
    red_m[threadIdx.x >> 5] = M;
    red_s[threadIdx.x >> 5] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float MM = -INFINITY;
    for (int w = 0; w < 8; w++) MM = fmaxf(MM, red_m[w]);
    float S = 0.f;
    for (int w = 0; w < 8; w++) S += red_m[w] == -INFINITY ? 0.f : red_s[w] * exp2f(red_m[w] - MM);
    lse2[lth] = MM + log2f(S);
  }
}

// ---- GOLDEN pass 2: p[l,t,j] = (1/H) sum_h 2^(c * qa_h . x_j - lse2_h)
template <int KT>
__global__ void __launch_bounds__(128) golden_prob_kernel(lidx_eval_args a, const float *lse2) {
  extern __shared__ float gsm[];
  float *q_s = gsm;               // [H][512] scaled
  float *l_s = gsm + a.H * kD;    // [H]
  const int lt = blockIdx.y;      // l*T + t
  const int l = lt / a.T;
  const float c = a.scale * kLog2e;
  for (int i = threadIdx.x; i < a.H * kD; i += 128) q_s[i] = q_elem(a.qa, a.qa_dtype, static_cast<size_t>(lt) * a.H * kD + i) * c;
  for (int i = threadIdx.x; i < a.H; i += 128) l_s[i] = lse2[static_cast<size_t>(lt) * a.H + i];
  __syncthreads();
  const int j = blockIdx.x * 128 + threadIdx.x;
  if (j >= a.N) return;
  const int64_t row = static_cast<int64_t>(l) * a.kv.batch_rows + j;
  float p = 0.f;
  for (int h0 = 0; h0 < a.H; h0 += 16) {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; i++) acc[i] = 0.f;
    for (int d = 0; d < kD; d++) {
      const float x = row_elem<KT>(a.kv, row, d);
#pragma unroll
      for (int i = 0; i < 16; i++)
        if (h0 + i < a.H) acc[i] = fmaf(q_s[(h0 + i) * kD + d], x, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; i++)
      if (h0 + i < a.H) p += exp2f(acc[i] - l_s[h0 + i]);
  }
  a.probs[static_cast<size_t>(lt) * a.N + j] = p / static_cast<float>(a.H);
}

// ---- TOPP: one CTA per (l,t) row.
constexpr int kT = 1024;

__device__ __forceinline__ uint64_t mass_of(float p) {
  // floor(p * 2^40): the product is exact in fp32 for p in [0, 1]
  return __float2ull_rd(p * 1099511627776.0f);
}

// Digit masses are kept as two 32-bit sums, mass = hi * 2^kLoBits + lo, which
// the shared-memory atomic units add natively.  Exact whenever the row's total
// mass is below 2^(32 + kLoBits) (every hi sum is at most total >> kLoBits)
// and N < 2^(32 - kLoBits) (every lo sum is below 2^kLoBits per run); other
// rows take 64-bit adds.
constexpr int kLoBits = 11;

struct ToppSmem {
  unsigned long long hist[256];
  uint32_t hist_hi[256], hist_lo[256];
  unsigned long long warp_m[32];
  uint32_t warp_a[32];
  unsigned long long total;
  uint32_t digit;
  unsigned long long above;
  uint32_t tot_a;
  uint32_t bad;
};

// The row is staged in shared memory once when it fits (kStage); every pass
// then reads it from there.  The radix starts at the highest bit in which the
// row's keys differ, and each thread folds runs of equal digits before its
// atomic add, so rows whose probabilities share an exponent (one hot bin)
// do not serialise on a single shared-memory address.
template <bool kStage>
__global__ void __launch_bounds__(kT, 1) topp_kernel(lidx_eval_args a, uint32_t *status) {
  extern __shared__ float prow[];  // [N] when staged
  __shared__ ToppSmem sm;
  __shared__ uint32_t red_lo[32], red_hi[32];
  const int row = blockIdx.x;
  const float *gp = a.probs + static_cast<size_t>(row) * a.N;
  const int N = a.N, tid = threadIdx.x;
  const uint32_t lane = lane_id(), warp = tid >> 5;
  if (tid == 0) {
    sm.total = 0;
    sm.bad = 0;
  }
  if (kStage)
    for (int j = tid; j < N; j += kT) prow[j] = gp[j];
  __syncthreads();
  const float *p = kStage ? prow : gp;
  auto key_mass = [&](int j, uint32_t &key, uint64_t &m) {
    const float x = p[j];
    if (!(x >= 0.f) || x > 1.f) {  // negative, > 1 or NaN: excluded
      key = 0u;
      m = 0;
      sm.bad = 1u;
      return;
    }
    key = order_key(x);
    m = mass_of(x);
  };
  // total mass, and the range of keys that carry mass
  unsigned long long tot = 0;
  uint32_t klo = 0xFFFFFFFFu, khi = 0u;
  for (int j = tid; j < N; j += kT) {
    uint32_t k;
    uint64_t m;
    key_mass(j, k, m);
    tot += m;
    if (m) {
      klo = min(klo, k);
      khi = max(khi, k);
    }
  }
  tot = warp_sum(tot);
  klo = __reduce_min_sync(0xFFFFFFFFu, klo);
  khi = __reduce_max_sync(0xFFFFFFFFu, khi);
  if (lane == 0) {
    atomicAdd(&sm.total, tot);
    red_lo[warp] = klo;
    red_hi[warp] = khi;
  }
  __syncthreads();
  if (tid == 0 && sm.bad) raise_status(status, LIDX_DEV_NAN);
  klo = __reduce_min_sync(0xFFFFFFFFu, red_lo[lane]);
  khi = __reduce_max_sync(0xFFFFFFFFu, red_hi[lane]);
  const uint64_t M = sm.total;
  const bool split = M < (1ull << (32 + kLoBits)) && N < (1 << (32 - kLoBits));
  auto add_mass = [&](uint32_t d, unsigned long long m) {
    if (split) {
      atomicAdd(&sm.hist_hi[d], static_cast<uint32_t>(m >> kLoBits));
      atomicAdd(&sm.hist_lo[d], static_cast<uint32_t>(m & ((1u << kLoBits) - 1u)));
    } else {
      atomicAdd(&sm.hist[d], m);
    }
  };
  const uint64_t q1 = M / a.top_p_den, r1 = M % a.top_p_den;
  const uint64_t rr = r1 * a.top_p_num;
  const uint64_t Tm = q1 * a.top_p_num + rr / a.top_p_den + (rr % a.top_p_den != 0);

  uint32_t T = 0xFFFFFFFFu;  // threshold key; nothing selected when Tm == 0
  uint32_t take_eq = 0;
  if (Tm > 0) {
    // keys with mass share the bits above the highest differing one
    const int bits_left = khi == klo ? 0 : 32 - __clz(klo ^ khi);
    uint32_t pmask = bits_left >= 32 ? 0u : ~((1u << bits_left) - 1u);
    uint32_t prefix = khi & pmask;
    uint64_t rem = Tm;
    for (int hi = bits_left; hi > 0; hi -= 8) {
      const int w = min(8, hi), shift = hi - w;
      const uint32_t dmask = (1u << w) - 1u;
      if (tid < 256) {
        sm.hist[tid] = 0ull;
        sm.hist_hi[tid] = 0u;
        sm.hist_lo[tid] = 0u;
      }
      __syncthreads();
      uint32_t run_d = 0xFFFFFFFFu;
      unsigned long long run_m = 0;
      for (int j = tid; j < N; j += kT) {
        uint32_t k;
        uint64_t m;
        key_mass(j, k, m);
        if (m && (k & pmask) == prefix) {
          const uint32_t d = (k >> shift) & dmask;
          if (d != run_d) {
            if (run_m) add_mass(run_d, run_m);
            run_d = d;
            run_m = 0;
          }
          run_m += m;
        }
      }
      if (run_m) add_mass(run_d, run_m);
      __syncthreads();
      const int nb = 1 << w;
      if (tid < 256) {
        const int x = nb - 1 - tid;
        const unsigned long long v =
            tid >= nb ? 0ull
            : split   ? (static_cast<unsigned long long>(sm.hist_hi[x]) << kLoBits) + sm.hist_lo[x]
                      : sm.hist[x];
        unsigned long long inc = warp_inclusive_scan(v);
        if (lane == 31) sm.warp_m[warp] = inc;
        asm volatile("bar.sync 1, 256;");
        unsigned long long before = 0;
        for (int ww = 0; ww < static_cast<int>(warp); ww++) before += sm.warp_m[ww];
        inc += before;
        if (tid < nb && inc >= rem && inc - v < rem) {
          sm.digit = static_cast<uint32_t>(nb - 1 - tid);
          sm.above = inc - v;
        }
      }
      __syncthreads();
      prefix |= sm.digit << shift;
      pmask |= dmask << shift;
      rem -= sm.above;
      __syncthreads();
    }
    T = prefix;
    // every entry with key T carries the same mass: take the first ceil(rem / m*)
    const float pv = (T & 0x80000000u) ? __uint_as_float(T & 0x7FFFFFFFu) : 0.f;
    const uint64_t mstar = mass_of(pv);
    take_eq = static_cast<uint32_t>((rem + mstar - 1) / mstar);
  }

  // ordered emission of the bit set
  const int Wn = (N + 31) / 32;
  uint32_t *bits = a.topp_bits + static_cast<size_t>(row) * Wn;
  uint32_t eq_seen = 0;
  for (int base = 0; base < Wn * 32; base += kT) {
    const int j = base + tid;
    uint32_t k = 0u;
    uint64_t m = 0;
    if (j < N) key_mass(j, k, m);
    const bool gt = k != 0u && T != 0xFFFFFFFFu && k > T && m;
    const bool eq = k != 0u && k == T;
    const uint32_t be = __ballot_sync(0xFFFFFFFFu, eq);
    if (lane == 0) sm.warp_a[warp] = __popc(be);
    __syncthreads();
    if (warp == 0) {
      const uint32_t v = sm.warp_a[lane];
      const uint32_t inc = warp_inclusive_scan(v);
      sm.warp_a[lane] = inc - v;
      if (lane == 31) sm.tot_a = inc;
    }
    __syncthreads();
    const uint32_t rank = eq_seen + sm.warp_a[warp] + __popc(be & ((1u << lane) - 1u));
    const bool sel = gt || (eq && rank < take_eq);
    const uint32_t word = __ballot_sync(0xFFFFFFFFu, sel);
    const int wi = (base >> 5) + static_cast<int>(warp);
    if (lane == 0 && wi < Wn) bits[wi] = word;
    eq_seen += sm.tot_a;
    __syncthreads();
  }
}

// ---- VOTE: per (t, word) count over layers; then union over t.
__global__ void vote_kernel(lidx_eval_args a, uint32_t *vote_out) {
  const int Wn = (a.N + 31) / 32;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.T * Wn) return;
  const int t = idx / Wn, w = idx % Wn;
  uint32_t out = 0;
  for (int bit = 0; bit < 32; bit++) {
    int c = 0;
    for (int l = 0; l < a.L; l++) c += (a.topp_bits[(static_cast<size_t>(l) * a.T + t) * Wn + w] >> bit) & 1u;
    if (c >= a.min_votes) out |= 1u << bit;
  }
  if (w == Wn - 1 && (a.N & 31)) out &= (1u << (a.N & 31)) - 1u;
  vote_out[static_cast<size_t>(t) * Wn + w] = out;
}

__global__ void union_kernel(int T, int Wn, const uint32_t *sets, uint32_t *out) {
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= Wn) return;
  uint32_t u = 0;
  for (int t = 0; t < T; t++) u |= sets[static_cast<size_t>(t) * Wn + w];
  out[w] = u;
}

// ---- LSA gate: thread per entry, warp ballot forms the word.
__global__ void lsa_kernel(lidx_eval_args a) {
  const int Wn = (a.N + 31) / 32;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  bool f = false;
  if (j < a.N)
    for (int g = 0; g < a.n_gate; g++) f |= (a.gate_logits[static_cast<size_t>(g) * a.N + j] + a.gate_bias) >= 0.f;
  const uint32_t word = __ballot_sync(0xFFFFFFFFu, f);
  if (lane_id() == 0 && (j >> 5) < Wn) a.fetched_bits[j >> 5] = word;
}

// ---- OVERLAP: one CTA per pair.
__global__ void __launch_bounds__(256) overlap_kernel(lidx_eval_args a) {
  const int pr = blockIdx.x;
  const int Wn = (a.N + 31) / 32;
  const uint32_t *A = a.set_a + static_cast<size_t>(pr) * a.ld_a;
  const uint32_t *B = a.set_b + static_cast<size_t>(pr) * a.ld_b;
  const uint32_t last = (a.N & 31) ? (1u << (a.N & 31)) - 1u : 0xFFFFFFFFu;
  unsigned long long c0 = 0, c1 = 0, c2 = 0;
  for (int w = threadIdx.x; w < Wn; w += 256) {
    uint32_t x = A[w], y = B[w];
    if (w == Wn - 1) {
      x &= last;
      y &= last;
    }
    c0 += __popc(x & y);
    c1 += __popc(x);
    c2 += __popc(y);
  }
  __shared__ unsigned long long r[3][8];
  c0 = warp_sum(c0);
  c1 = warp_sum(c1);
  c2 = warp_sum(c2);
  if (lane_id() == 0) {
    r[0][threadIdx.x >> 5] = c0;
    r[1][threadIdx.x >> 5] = c1;
    r[2][threadIdx.x >> 5] = c2;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    unsigned long long s = 0;
    for (int w = 0; w < 8; w++) s += r[threadIdx.x][w];
    a.counts[static_cast<size_t>(pr) * 3 + threadIdx.x] = static_cast<int64_t>(s);
  }
}

size_t lse_bytes(const lidx_eval_args &a) {
  return (static_cast<size_t>(a.L) * a.T * a.H * sizeof(float) + 255) / 256 * 256;
}
size_t vote_bytes(const lidx_eval_args &a) {
  return (static_cast<size_t>(a.T) * ((a.N + 31) / 32) * sizeof(uint32_t) + 255) / 256 * 256;
}

}  // namespace

// Softmax of one score row per CTA over its N entries (the golden step read
// as a softmax of the indexer logits): the row's largest non-NaN score m,
// l = sum exp(s - m) over the non-NaN scores, then p = exp(s - m) / l.
// NaN scores get p = 0 (and LIDX_DEV_NAN); -inf ones get 0 by exp; a row
// without a finite score (m = -inf) is all zeros.
__global__ void __launch_bounds__(256) golden_index_kernel(lidx_eval_args a, uint32_t *status) {
  __shared__ float red[8];
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *s = a.index_scores + static_cast<size_t>(r) * a.ld_index_scores;
  float *p = a.probs + static_cast<size_t>(r) * a.N;
  float m = -INFINITY;
  bool nan = false;
  for (int j = tid; j < a.N; j += 256) {
    const float v = s[j];
    nan |= v != v;
    m = fmaxf(m, v);  // fmaxf skips NaN
  }
  if (nan) raise_status(status, LIDX_DEV_NAN);
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < 8; w++) m = fmaxf(m, red[w]);
  __syncthreads();
  if (m == -INFINITY) {
    for (int j = tid; j < a.N; j += 256) p[j] = 0.f;
    return;
  }
  float l = 0.f;
  for (int j = tid; j < a.N; j += 256) {
    const float v = s[j];
    if (v == v) l += expf(v - m);
  }
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.f;
  for (int w = 0; w < 8; w++) l += red[w];
  const float il = 1.f / l;
  for (int j = tid; j < a.N; j += 256) {
    const float v = s[j];
    p[j] = v == v ? expf(v - m) * il : 0.f;
  }
}

size_t eval_workspace(const lidx_eval_args &a) {
  size_t n = LIDX_WS_HEADER;
  if (a.ops & LIDX_EVAL_GOLDEN) n += golden_tc_supported(a) ? golden_tc_workspace(a) : lse_bytes(a);
  if ((a.ops & LIDX_EVAL_VOTE) && !a.vote_bits) n += vote_bytes(a);
  return n;
}

// Kernels launch_eval launches for a.ops, in its order: golden (two tensor-core
// passes around the lse merge, or the lse and probability kernels), golden
// from the index logits, top-p, vote + union, gate, overlap.
int eval_launches(const lidx_eval_args &a) {
  int n = 0;
  if (a.ops & LIDX_EVAL_GOLDEN) n += golden_tc_supported(a) ? 3 : 2;
  if (a.ops & LIDX_EVAL_GOLDEN_INDEX) n += 1;
  if (a.ops & LIDX_EVAL_TOPP) n += 1;
  if (a.ops & LIDX_EVAL_VOTE) n += 2;
  if (a.ops & LIDX_EVAL_LSA) n += 1;
  if (a.ops & LIDX_EVAL_OVERLAP) n += 1;
  return n;
}

cudaError_t launch_eval(const lidx_eval_args &a, void *ws, cudaStream_t st) {
  uint32_t *status = static_cast<uint32_t *>(ws);
  char *cur = static_cast<char *>(ws) + LIDX_WS_HEADER;
  cudaError_t e;
  if ((a.ops & LIDX_EVAL_GOLDEN) && golden_tc_supported(a)) {
    if ((e = launch_golden_tc(a, cur, status, st)) != cudaSuccess) return e;
    cur += golden_tc_workspace(a);
  } else if (a.ops & LIDX_EVAL_GOLDEN) {
    float *lse2 = reinterpret_cast<float *>(cur);
    cur += lse_bytes(a);
    const size_t smem = (static_cast<size_t>(a.H) * kD + a.H) * sizeof(float);
    dim3 g2((a.N + 127) / 128, a.L * a.T);
    switch (a.kv.dtype) {
      case LIDX_F32:
        golden_lse_kernel<LIDX_F32><<<a.L * a.T * a.H, 256, 0, st>>>(a, lse2);
        cudaFuncSetAttribute(golden_prob_kernel<LIDX_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        golden_prob_kernel<LIDX_F32><<<g2, 128, smem, st>>>(a, lse2);
        break;
      case LIDX_BF16:
        golden_lse_kernel<LIDX_BF16><<<a.L * a.T * a.H, 256, 0, st>>>(a, lse2);
        cudaFuncSetAttribute(golden_prob_kernel<LIDX_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        golden_prob_kernel<LIDX_BF16><<<g2, 128, smem, st>>>(a, lse2);
        break;
      default:
        golden_lse_kernel<LIDX_E4M3><<<a.L * a.T * a.H, 256, 0, st>>>(a, lse2);
        cudaFuncSetAttribute(golden_prob_kernel<LIDX_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        golden_prob_kernel<LIDX_E4M3><<<g2, 128, smem, st>>>(a, lse2);
        break;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.ops & LIDX_EVAL_GOLDEN_INDEX) {
    golden_index_kernel<<<a.L * a.T, 256, 0, st>>>(a, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.ops & LIDX_EVAL_TOPP) {
    const size_t row_bytes = static_cast<size_t>(a.N) * sizeof(float);
    if (row_bytes <= 200u * 1024u) {
      cudaFuncSetAttribute(topp_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(row_bytes));
      topp_kernel<true><<<a.L * a.T, kT, row_bytes, st>>>(a, status);
    } else {
      topp_kernel<false><<<a.L * a.T, kT, 0, st>>>(a, status);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int Wn = (a.N + 31) / 32;
  if (a.ops & LIDX_EVAL_VOTE) {
    uint32_t *vb = a.vote_bits;
    if (!vb) {
      vb = reinterpret_cast<uint32_t *>(cur);
      cur += vote_bytes(a);
    }
    const int n = a.T * Wn;
    vote_kernel<<<(n + 255) / 256, 256, 0, st>>>(a, vb);
    union_kernel<<<(Wn + 255) / 256, 256, 0, st>>>(a.T, Wn, vb, a.window_bits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.ops & LIDX_EVAL_LSA) {
    lsa_kernel<<<(Wn * 32 + 255) / 256, 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.ops & LIDX_EVAL_OVERLAP) {
    overlap_kernel<<<a.n_pairs, 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lidx
