// Golden dense-attention probabilities on tcgen05 (FlashMemory-vs-native
// post, Act 3: unmasked dense attention as the ground truth; FlashMemory
// deep-dive write-up, section 3.2 step 1):
//
//   p[l,t,j] = (1/H) sum_h softmax_j(scale * qa[l,t,h] . x_l[j])
//
// The logits are one GEMM per layer, (T*H rows) x (N keys) x 512, run twice:
//   pass 1  per row the base-2 log-sum-exp over all N keys: each 256-key
//           block leaves a partial (max, sum) per row, a small kernel merges
//           them;
//   pass 2  2^(c*logit - lse2) per element, then the mean over the H = 64
//           heads of each query.
// Tile: 128 rows (two queries x 64 heads) x 256 keys, K = 512 in eight
// 64-wide panels.  Persistent CTAs take the (layer, key block, row block)
// units round-robin, row block fastest: at any time all CTAs work on one
// layer and a few key blocks, so each 256-key block is fetched from HBM once
// and reused from L2 by the layer's row blocks (ranges per CTA would spread
// the CTAs over every layer and re-read the keys once per row block):
//   warp 0      TMA producer: per panel the 128 x 64 query box and the
//               256 x 64 key box (128-byte swizzled) into a 4-stage ring
//   warp 1      TMEM allocation; one lane issues 4 MMAs per panel
//               (M = 128, N = 256) into one of two TMEM accumulators
//   warps 2-17  epilogue: warp w reads TMEM lane quarter w&3 (32 rows) and
//               64 of the 256 columns, thread = one row; four warps per
//               quarter keep the exponentials (one SFU op per element) and
//               their latencies spread over the SM
// Pass 2 sums over the 64 rows of a query with a transposed warp reduction
// (each lane ends with one column's sum over the warp's 32 rows) and one
// shared-memory exchange between the two warps of the query that share the
// columns.
#include <algorithm>

#include "kernels.cuh"
#include "tc.cuh"

namespace lidx {

namespace {

constexpr int kD = 512;
constexpr int kHeads = 64;          // rows of a query
constexpr int kTM = 128;            // rows per tile (two queries)
constexpr int kTN = 256;            // keys per tile
constexpr int kPanels = kD / 64;
constexpr int kStages = 4;
constexpr int kABytes = kTM * 128;  // one 64-wide panel of the query rows
constexpr int kBBytes = kTN * 128;  // one 64-wide panel of the keys
constexpr int kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
constexpr int kEpiWarps = 16;        // 4 lane quarters x 4 column groups
constexpr int kCG = kTN / 4;         // columns per epilogue warp
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr float kLog2e = 1.4426950408889634f;

struct GoldenParams {
  int L, T, N;
  int rows;          // T * 64 per layer
  int n_rb, n_kb;    // row blocks, key blocks per layer
  long long units;
  int64_t key_rows;  // rows between layers in the key tensor map
  float c;           // scale * log2(e)
  float2 *part;      // pass 1: [L][rows][n_kb][4 column groups]
  const float *lse2; // pass 2: [L][rows]
  float *probs;      // pass 2: [L][T][N]
};

struct __align__(8) GoldenBars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  uint32_t abort;
};

constexpr size_t golden_smem_bytes() {
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + 2 * kTN * sizeof(float) + sizeof(GoldenBars);
}

// 32-bit arithmetic (units < 2^31 is checked at launch): a 64-bit division
// is a long software sequence.
__device__ __forceinline__ void unit_coords(const GoldenParams &p, long long u, int &l, int &rb, int &kb) {
  const uint32_t uu = static_cast<uint32_t>(u), nrb = static_cast<uint32_t>(p.n_rb), nkb = static_cast<uint32_t>(p.n_kb);
  rb = static_cast<int>(uu % nrb);
  const uint32_t r = uu / nrb;
  kb = static_cast<int>(r % nkb);
  l = static_cast<int>(r / nkb);
}

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

// Each lane holds v[0..31] (columns of a 32-wide chunk); afterwards lane i
// holds the sum over the warp's 32 lanes of column i.
__device__ __forceinline__ float transpose_sum32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; i++) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, s);
    }
  }
  return v[0];
}

template <int kPass>
__global__ void __launch_bounds__(kThreads, 1)
    golden_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const GoldenParams p, uint32_t *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *sRed = reinterpret_cast<float *>(smem + kStages * kStageBytes);  // [2][256]: partner warps' column sums
  GoldenBars *bar = reinterpret_cast<GoldenBars *>(sRed + 2 * kTN);
  volatile uint32_t *abort_flag = &bar->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long u0 = blockIdx.x, ustep = gridDim.x;  // units u0, u0 + ustep, ...

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; s++) {
      tc::mbar_init(&bar->full[s], 1);
      tc::mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; a++) {
      tc::mbar_init(&bar->tfull[a], 1);
      tc::mbar_init(&bar->tempty[a], kEpiWarps);
    }
    bar->abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_q);
    tc::tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) tc::tmem_alloc(&bar->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t last_par[kStages] = {};
      bool used[kStages] = {};
      for (long long u = u0; u < p.units && !*abort_flag; u += ustep) {
        int l, rb, kb;
        unit_coords(p, u, l, rb, kb);
        const int qrow = l * p.rows + rb * kTM;
        const int krow = static_cast<int>(l * p.key_rows + static_cast<int64_t>(kb) * kTN);
        for (int pn = 0; pn < kPanels; pn++) {
          if (!tc::mbar_wait(&bar->empty[stage], phase ^ 1, abort_flag)) break;
          uint8_t *st = smem + stage * kStageBytes;
          tc::mbar_arrive_expect_tx(&bar->full[stage], kStageBytes);
          tc::tma_load_2d(st, &tm_q, &bar->full[stage], 64 * pn, qrow);
          tc::tma_load_2d(st + kABytes, &tm_k, &bar->full[stage], 64 * pn, krow);
          last_par[stage] = phase;
          used[stage] = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // never leave with copies in flight
      volatile uint32_t no_abort = 0;
      for (int s = 0; s < kStages; s++)
        if (used[s]) tc::mbar_wait(&bar->full[s], last_par[s], &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_par = 0;
      const uint32_t idesc = tc::idesc_bf16(kTM, kTN);
      const uint32_t base = tc::smem_u32(smem);
      for (long long u = u0; u < p.units; u += ustep) {
        if (!tc::mbar_wait(&bar->tempty[acc], acc_par ^ 1, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + acc * kTN;
        bool ok = true;
        for (int pn = 0; pn < kPanels; pn++) {
          if (!tc::mbar_wait(&bar->full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t a = base + stage * kStageBytes, b = a + kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            tc::mma_bf16(d, tc::desc_kmajor_sw128(a + kk * 32), tc::desc_kmajor_sw128(b + kk * 32), idesc,
                         (pn | kk) != 0);
          tc::mma_commit(&bar->empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc::mma_commit(&bar->tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_par ^= 1;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lane quarter = rows [32q, 32q+32) of the tile
    const int cg = (warp - 2) >> 2;  // column group: columns [64cg, 64cg + 64)
    const int trow = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_par = 0;
    for (long long u = u0; u < p.units; u += ustep) {
      int l, rb, kb;
      unit_coords(p, u, l, rb, kb);
      const int row = rb * kTM + trow;  // row of the layer: t * 64 + h
      const bool row_ok = row < p.rows;
      bool ready = false;
      if (lane == 0) ready = tc::mbar_wait(&bar->tfull[acc], acc_par, abort_flag);
      ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
      if (ready) {
        tc::tc_fence_after();
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kTN + cg * kCG;
        const int j0 = kb * kTN + cg * kCG;
        if (kPass == 1) {
          float m = -INFINITY, s = 0.f;
          for (int c0 = 0; c0 < kCG; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tbase + c0, v);
            float cm = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; i++) {
              v[i] = j0 + c0 + i < p.N ? v[i] * p.c : -INFINITY;
              cm = fmaxf(cm, v[i]);
            }
            const float mn = fmaxf(m, cm);
            if (mn != -INFINITY) {
              float cs = 0.f;
#pragma unroll
              for (int i = 0; i < 32; i++) cs += exp2f(v[i] - mn);
              s = s * exp2f(m - mn) + cs;
              m = mn;
            }
          }
          if (row_ok) p.part[((static_cast<size_t>(l) * p.rows + row) * p.n_kb + kb) * 4 + cg] = make_float2(m, s);
        } else {
          const float lse = row_ok ? p.lse2[static_cast<size_t>(l) * p.rows + row] : INFINITY;
          const int q = quarter >> 1;       // query of the tile
          const int t = rb * 2 + q;         // query of the layer
          const int bar_id = 1 + q * 4 + cg;  // the two warps of query q on these columns
          for (int c0 = 0; c0 < kCG; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tbase + c0, v);
#pragma unroll
            for (int i = 0; i < 32; i++) v[i] = row_ok ? exp2f(v[i] * p.c - lse) : 0.f;
            const float colsum = transpose_sum32(v);  // column c0 + lane, this warp's 32 heads
            float *red = sRed + q * kTN + cg * kCG + c0;
            if (quarter & 1) red[lane] = colsum;
            named_sync(bar_id, 64);
            if (!(quarter & 1)) {
              const int j = j0 + c0 + lane;
              const float tot = colsum + red[lane];
              if (t < p.T && j < p.N)
                p.probs[(static_cast<size_t>(l) * p.T + t) * p.N + j] = tot * (1.f / kHeads);
            }
            named_sync(bar_id, 64);  // the partner may overwrite sRed
          }
        }
      } else if (kPass == 2) {
        // keep the named barriers of the pair matched on a give-up
        const int bar_id = 1 + (quarter >> 1) * 4 + cg;
        for (int c0 = 0; c0 < kCG; c0 += 32) {
          named_sync(bar_id, 64);
          named_sync(bar_id, 64);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0 && ready) tc::mbar_arrive(&bar->tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_par ^= 1;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bar->abort) raise_status(status, LIDX_DEV_TIMEOUT);
}

// lse2[l][row] = log2 sum over the partials (key blocks x column groups).
// One warp per row: the lanes read the row's (max, sum) pairs two at a time
// with coalesced 16-byte loads in a single pass, keep an online (max, sum),
// and fold the 32 lane states with shuffles.  n_kb is a multiple of 4 and
// the partials are 16-byte aligned.
__device__ __forceinline__ void lse_fold(float &M, float &S, float m, float s) {
  if (m == -INFINITY) return;
  if (m > M) {
    S = S * exp2f(M - m) + s;
    M = m;
  } else {
    S += s * exp2f(m - M);
  }
}

__global__ void golden_lse_merge_kernel(const float2 *part, int n, int n_kb, float *lse2) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= n) return;
  const float4 *pp = reinterpret_cast<const float4 *>(part + static_cast<size_t>(i) * n_kb);
  float M = -INFINITY, S = 0.f;
  for (int b = lane; b < (n_kb >> 1); b += 32) {
    const float4 v = __ldcs(pp + b);
    lse_fold(M, S, v.x, v.y);
    lse_fold(M, S, v.z, v.w);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, M, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, S, o);
    lse_fold(M, S, m2, s2);
  }
  if (lane == 0) lse2[i] = M + log2f(S);
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

bool golden_tc_supported(const lidx_eval_args &a) {
  if (a.H != kHeads || a.qa_dtype != LIDX_BF16 || a.kv.dtype != LIDX_BF16) return false;
  if ((a.kv.ld * 2) % 16 != 0) return false;
  const int64_t qrows = static_cast<int64_t>(a.L) * a.T * a.H;
  const int64_t krows = static_cast<int64_t>(a.L - 1) * (a.L > 1 ? a.kv.batch_rows : 0) + a.N;
  const int64_t units = static_cast<int64_t>(a.L) * ((a.T * kHeads + kTM - 1) / kTM) * ((a.N + kTN - 1) / kTN);
  return qrows < (1ll << 31) && krows < (1ll << 31) && units < (1ll << 31);
}

size_t golden_tc_workspace(const lidx_eval_args &a) {
  const size_t rows = static_cast<size_t>(a.L) * a.T * a.H;
  const size_t n_kb = (a.N + kTN - 1) / kTN;
  return ((rows * n_kb * 4 * sizeof(float2) + 255) / 256) * 256 + ((rows * sizeof(float) + 255) / 256) * 256;
}

cudaError_t launch_golden_tc(const lidx_eval_args &a, void *scratch, uint32_t *status, cudaStream_t st) {
  GoldenParams p{};
  p.L = a.L;
  p.T = a.T;
  p.N = a.N;
  p.rows = a.T * kHeads;
  p.n_rb = (p.rows + kTM - 1) / kTM;
  p.n_kb = (a.N + kTN - 1) / kTN;
  p.units = static_cast<long long>(a.L) * p.n_rb * p.n_kb;
  p.key_rows = a.L > 1 ? a.kv.batch_rows : a.N;
  p.c = a.scale * kLog2e;
  const size_t rows = static_cast<size_t>(a.L) * p.rows;
  p.part = static_cast<float2 *>(scratch);
  float *lse2 = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                          ((rows * p.n_kb * 4 * sizeof(float2) + 255) / 256) * 256);
  p.lse2 = lse2;
  p.probs = a.probs;

  CUtensorMap tm_q, tm_k;
  const uint64_t krows = static_cast<uint64_t>(a.L - 1) * p.key_rows + a.N;
  if (!make_tmap_2d(&tm_q, a.qa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, rows, kD * 2, 64, kTM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_k, a.kv.data, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kD, krows, a.kv.ld * 2, 64, kTN,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = golden_smem_bytes();
  const int grid = static_cast<int>(std::min<long long>(p.units, sm_count()));
  cudaFuncSetAttribute(golden_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  cudaFuncSetAttribute(golden_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  golden_tc_kernel<1><<<grid, kThreads, smem, st>>>(tm_q, tm_k, p, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n = static_cast<int>(rows);
  golden_lse_merge_kernel<<<(n + 7) / 8, 256, 0, st>>>(p.part, n, p.n_kb * 4, lse2);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  golden_tc_kernel<2><<<grid, kThreads, smem, st>>>(tm_q, tm_k, p, status);
  return cudaGetLastError();
}

}  // namespace lidx
