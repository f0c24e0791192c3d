/*
 * lidx -- lightning indexer, top-k selection and sparse MQA decode for
 * NVIDIA B200 (sm_100a).  C ABI of liblidx.so.
 *
 * The path (DeepSeek-V4-Flash architecture post, "Part 6", section (B)):
 * in every CSA layer the lightning indexer scores each 4:1-compressed entry
 * with its own 128-d index key (index_comp_kv), keeps the top 512 entries
 * (n_indexer_top_k; 1024 for the Pro variant), and attention reads the
 * selected 512-wide rows (attn_comp_kv, section (A)) plus a 128-row sliding
 * window.  The evaluation side (FlashMemory-vs-native post, Act 3; FlashMemory
 * deep-dive write-up, sections 2.2, 3.2 and 4.1) builds golden labels from
 * dense attention (softmax, top-p 0.6, >= 3-of-21 layer vote), applies the
 * memory-indexer gate (sigmoid >= 0.5, OR over layers 10/12/20) and measures
 * set overlap.
 *
 * Conventions for every call:
 *  - All pointers in the argument structs are DEVICE pointers unless noted.
 *    The caller owns all memory; the library allocates and frees nothing.
 *    Scratch memory is a caller-provided workspace whose size
 *    lidx_workspace_size() reports; it must be 256-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work on it: no host synchronisation.
 *  - Synchronous argument errors are returned as lidx_status before anything
 *    is enqueued.  Data-dependent problems found on the device (an id outside
 *    [0, N), a NaN score, a device wait that gave up) are OR-ed as bit flags
 *    into a status word at the start of the workspace; read it with
 *    lidx_read_device_status().  The kernels never trap.
 *  - The library keeps no mutable global state besides cached device
 *    properties, so concurrent calls on different streams with different
 *    workspaces are safe.
 */
#ifndef LIDX_H
#define LIDX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LIDX_ABI_VERSION 6

#if defined(__GNUC__)
#define LIDX_API __attribute__((visibility("default")))
#else
#define LIDX_API
#endif

typedef enum lidx_status {
    LIDX_OK = 0,
    LIDX_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer */
    LIDX_ERR_UNSUPPORTED = 2, /* format/shape not implemented (e.g. f16 comp KV), or not sm_100 */
    LIDX_ERR_CUDA = 3,        /* a CUDA runtime call failed */
    LIDX_ERR_WORKSPACE = 4    /* workspace missing or smaller than lidx_workspace_size() */
} lidx_status;

/* Bit flags of the device status word (asynchronous). */
#define LIDX_DEV_BOUNDS 0x1u  /* an id outside [0, N) was skipped */
#define LIDX_DEV_NAN 0x2u     /* a NaN score / negative or NaN probability was excluded */
#define LIDX_DEV_TIMEOUT 0x4u /* a bounded device wait gave up */

/* Launch flags (the `flags` field of the score, top-k and attention args). */
#define LIDX_LAUNCH_PDL 0x1u /* programmatic dependent launch: the kernels may start while the previous
                              * kernel on the stream still runs.  Before waiting for it they only set up
                              * and read cache-side inputs (index keys, compressed KV and window rows,
                              * E8M0 scales, attention queries); everything else is read, and every
                              * global write is made, after the wait.  So with this flag the cache-side
                              * inputs must not be written by kernels that may still be running. */

#define LIDX_LAUNCH_TEST_LOST_ARRIVAL 0x80000000u /* test hook of lidx_decode_layer: one score CTA
                              * withholds its arrival and the cross-CTA waits give up after about 2 ms;
                              * the call must then finish and report LIDX_DEV_TIMEOUT */

/* Storage formats. */
#define LIDX_F32 0
#define LIDX_BF16 1
#define LIDX_E4M3 2 /* OCP E4M3FN non-RoPE dims + E8M0 scale per 64 + bf16 RoPE dims */
#define LIDX_F16 3  /* recognised and refused (LIDX_ERR_UNSUPPORTED), as the ds4 CUDA path refuses f16 comp KV */

/*
 * Rows of a cache (index keys, compressed KV or sliding-window rows).
 *
 * Logical row (width `dim`): for LIDX_F32 / LIDX_BF16 the `dim` stored
 * values.  For LIDX_E4M3 (architecture post, "why quantising the KV does not
 * save memory"): dims [0, dim-64) are E4M3 codes in `data`, scaled by
 * 2^(e-127) where e is the E8M0 byte scale[(d)/64] of the row; dims
 * [dim-64, dim) are the bf16 RoPE dims in `rope`.
 *
 * Row j of batch entry b is row b*batch_rows + j of every plane; row r of a
 * plane starts at plane + r*ld (ld in elements of that plane).  Planes must
 * be 16-byte aligned and ld*elem_size a multiple of 16 (scale plane: any ld).
 */
typedef struct lidx_kv {
    int32_t dtype;        /* LIDX_F32 | LIDX_BF16 | LIDX_E4M3 */
    int32_t dim;          /* 128 for index keys, 512 for attention rows */
    const void *data;     /* F32: float, BF16: bf16, E4M3: uint8 codes */
    const uint8_t *scale; /* E4M3 only: E8M0 codes, (dim-64)/64 per row */
    const void *rope;     /* E4M3 only: bf16, 64 per row */
    int64_t ld;           /* elements between rows of `data` */
    int64_t ld_scale;     /* bytes between rows of `scale` */
    int64_t ld_rope;      /* elements between rows of `rope` */
    int64_t batch_rows;   /* rows between consecutive batch entries (>= N) */
} lidx_kv;

/* ------------------------------------------------------------------------
 * lidx_index_score -- lightning indexer scores.
 *
 *   scores[b,t,j] = sum_h w[b,t,h] * max(q[b,t,h,:] . keys[b,j,:], 0)
 *
 * (head-weighted ReLU of MQA dot products; the ReLU-MQA indexer of the
 * FlashMemory deep-dive write-up, reply #2, with the head weights applied
 * outside the ReLU).  Accumulation is fp32.
 *
 *   q       [B][Q][H][128], q_dtype LIDX_F32 (with F32 keys) or LIDX_BF16
 *           (with BF16 or E4M3 keys)
 *   w       [B][Q][H] fp32 (any sign)
 *   keys    dim 128
 *   scores  [B][Q][ld_scores] fp32, ld_scores >= N; entries j >= N untouched
 *   tile_stats  optional [B][Q][ceil(N/LIDX_STATS_SPAN)][2] uint32, 8-byte
 *           aligned: the score bounds lidx_topk_select can start from (see
 *           LIDX_STATS_SPAN)
 *   n_visible optional [B][Q] int32: causal entry mask for prefill, where the
 *           queries sit at different positions: entry j is visible to query
 *           (b,t) only when j < n_visible[b][t] (the compressed entries formed
 *           before its token); the scores of the others are written as -inf.
 *           Pass the same counts as n_valid to lidx_topk_select.
 * Returns INVALID_ARG for null pointers / non-positive sizes / misaligned
 * planes, UNSUPPORTED for other format combinations.
 * ------------------------------------------------------------------------ */

/* Score bounds per span of 32 entries (optional side output of
 * lidx_index_score, input of lidx_topk_select).  For score row (b,t) and span
 * i, entry [i][0] is the largest and [i][1] the smallest order-preserving key
 * of the non-NaN scores j in [32i, min(32i+32, N)), or (0, 0xFFFFFFFF) when
 * the span has none.  The key of a score s with IEEE bits u (-0 taken as +0)
 * is u | 0x80000000 for s >= 0 and ~u for s < 0, so larger scores have larger
 * keys.  With them the top-k reads the row's score range instead of
 * exchanging it among its CTAs. */
#define LIDX_STATS_SPAN 32
typedef struct lidx_score_args {
    int32_t B, Q, H, N;
    int32_t q_dtype;
    const void *q;
    const float *w;
    lidx_kv keys;
    float *scores;
    int64_t ld_scores;
    uint32_t flags;       /* LIDX_LAUNCH_* */
    uint32_t *tile_stats; /* optional score bounds, see LIDX_STATS_SPAN */
    const int32_t *n_visible; /* optional causal entry mask, [B][Q] */
} lidx_score_args;

LIDX_API lidx_status lidx_index_score(const lidx_score_args *args, void *stream);

/* ------------------------------------------------------------------------
 * lidx_topk_select -- top-k row ids (architecture post, section (B):
 * n_indexer_top_k, and the comp_allowed row set).
 *
 * For each (b,t): the k largest scores[b,t,0..N) among the eligible
 * entries: those with allowed[b][j] != 0 when `allowed` is given, and with
 * bit j%32 of allowed_bits[b][j/32] set when `allowed_bits` is given (all
 * entries when neither is).  allowed_bits takes the fetched set of the
 * memory-indexer gate (lidx_selection_eval, LIDX_EVAL_LSA) as it is: the
 * native indexer then keeps its top-k inside the fetched set
 * (FlashMemory-vs-native post, "The setup"; write-up, reply #2).  Equal scores
 * (+0 and -0 included) are ranked by index, lower first; NaN scores are
 * never selected and set LIDX_DEV_NAN.
 *
 *   ids     [B][Q][k] int32: selected indices in ascending order, then -1
 *   n_sel   [B][Q] int32 (optional): min(k, #eligible)
 *   mask    [B][Q][N] uint8 (optional): 1 for selected entries (comp_allowed)
 *   mask_bits [B][Q][ceil(N/32)] uint32 (optional): bit j%32 of word j/32
 *   n_valid [B][Q] int32 (optional): only entries j < n_valid[b][t] are
 *           eligible (the causal prefix of a prefill query; see n_visible of
 *           lidx_index_score)
 *   tile_stats optional: the score bounds lidx_index_score wrote for exactly
 *           these scores (LIDX_STATS_SPAN).  Bounds that do not hold give
 *           wrong ids but never a write outside ids[b][t][0..k).
 * Needs a workspace of lidx_workspace_size(LIDX_OP_TOPK).
 * ------------------------------------------------------------------------ */
typedef struct lidx_topk_args {
    int32_t B, Q, N, k;
    const float *scores;
    int64_t ld_scores;
    const uint8_t *allowed; /* optional [B][ld_allowed], shared by the Q queries */
    int64_t ld_allowed;
    int32_t *ids;
    int32_t *n_sel;
    uint8_t *mask;
    uint32_t *mask_bits;
    uint32_t flags;             /* LIDX_LAUNCH_* */
    const uint32_t *tile_stats; /* optional score bounds, see LIDX_STATS_SPAN */
    const uint32_t *allowed_bits; /* optional [B][ld_allowed_bits] bit set, shared by the Q queries */
    int64_t ld_allowed_bits;      /* words between sequences, >= ceil(N/32) */
    const int32_t *n_valid;       /* optional per-row eligible prefix, [B][Q] */
} lidx_topk_args;

LIDX_API lidx_status lidx_topk_select(const lidx_topk_args *args, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * lidx_sparse_attn_decode -- MQA attention of one decode token over the
 * selected compressed rows plus the sliding window (architecture post,
 * sections (A)-(B)).  K = V = the full 512-wide row.
 *
 *   R_b  = { kv row ids[b][i] : i < n_b, ids[b][i] >= 0 } U { swa rows 0..swa_len-1 }
 *          with n_b = n_sel[b] if n_sel is given, else n_ids.
 *          ids NULL means ids[b][i] = i: the rows 0..n_b-1 are read whole, with
 *          no top-k (the HCA layers of the architecture post, section (A):
 *          128:1 compression, every entry attended); n_ids <= N then.
 *   out[b,h,:] = sum_{r in R_b} softmax_r(scale * q[b,h,:] . x_r) x_r
 *   lse[b,h]   = log sum_{r in R_b} exp(scale * q[b,h,:] . x_r)   (optional)
 *
 *   q     [B][H][512], LIDX_F32 (with F32 rows) or LIDX_BF16
 *   kv    comp_kv rows, dim 512, N entries per sequence
 *   ids   [B][ld_ids] int32 (ascending not required; duplicates count twice),
 *         or NULL for the dense rows 0..n_b-1
 * The rows of the B queries may overlap: kv.batch_rows and swa.batch_rows
 * may be smaller than the rows one query reads (0: every query reads the
 * same rows).  So the T queries of a prefill attend through one call: B = T,
 * kv.batch_rows = 0 (one shared compressed cache, each query with its own
 * ids), swa rows of query t starting at row t of the raw-token window buffer
 * (swa.batch_rows = 1).
 *   swa   sliding-window rows, dim 512, same dtype as kv (swa_len may be 0)
 *   out   [B][H][512] fp32
 * Ids outside [-1, N) are skipped and set LIDX_DEV_BOUNDS.  Empty R gives
 * out = 0 and lse = -inf.  Needs lidx_workspace_size(LIDX_OP_ATTN) bytes
 * (split-K partial results).
 * ------------------------------------------------------------------------ */
typedef struct lidx_attn_args {
    int32_t B, H;
    int32_t q_dtype;
    const void *q;
    lidx_kv kv;
    int32_t N;
    const int32_t *ids;
    int32_t n_ids;
    int64_t ld_ids;
    const int32_t *n_sel;
    lidx_kv swa;
    int32_t swa_len;
    float scale;
    float *out;
    float *lse;
    uint32_t flags; /* LIDX_LAUNCH_* */
} lidx_attn_args;

LIDX_API lidx_status lidx_sparse_attn_decode(const lidx_attn_args *args, void *ws, size_t ws_bytes,
                                    void *stream);

/* ------------------------------------------------------------------------
 * lidx_decode_layer -- one CSA layer of decode in a single launch: index
 * scores -> top-k -> sparse MQA attention over the selected rows plus the
 * window (architecture post, section (B): the indexer scores every compressed
 * entry, keeps the top k, and attention reads those attn_comp_kv rows and the
 * 128-row window).  Same results as lidx_index_score, lidx_topk_select (on
 * the scores it computes) and lidx_sparse_attn_decode (on those ids) in
 * sequence, with Q = 1 query per sequence.
 *
 *   q_idx [B][H][128] bf16, w [B][H] fp32, keys bf16 dim 128
 *   q_attn [B][64][512] bf16, kv and swa bf16 dim 512 (64 query heads)
 *   out [B][64][512] fp32, lse [B][64] (optional)
 *   scores [B][ld_scores] fp32 (optional), ids [B][k] int32 ascending with -1
 *           padding (optional), n_sel [B] (optional): the intermediate
 *           results, written when given
 *   prefetch[i], prefetch_bytes[i] (optional): device ranges to pull into L2
 *           while this layer runs, e.g. the next layer's index keys and window
 *           rows, which are known before its query is (a hint; no result
 *           depends on it).  16-byte aligned, sizes multiples of 16.
 *
 * Supported: bf16 keys, rows and queries, H a multiple of 32 up to 128,
 * N <= 16384, and B * ceil((swa_len + k) / 64) * 4 <= the device's SM count
 * (every attention unit runs concurrently); otherwise LIDX_ERR_UNSUPPORTED
 * (use the three calls).  The workspace (lidx_workspace_size(LIDX_OP_DECODE))
 * must be zeroed before its first use; every call leaves its control words
 * zeroed again.  One workspace serves one call at a time.
 * ------------------------------------------------------------------------ */
typedef struct lidx_decode_args {
    int32_t B, H, N, k;
    const void *q_idx;
    const float *w;
    lidx_kv keys;
    int32_t H_attn;        /* must be 64 */
    const void *q_attn;
    lidx_kv kv;
    lidx_kv swa;
    int32_t swa_len;
    float scale;
    float *out;
    float *lse;
    float *scores;
    int64_t ld_scores;
    int32_t *ids;
    int32_t *n_sel;
    const void *prefetch[2];
    uint64_t prefetch_bytes[2];
    uint32_t flags;        /* LIDX_LAUNCH_* */
} lidx_decode_args;

LIDX_API lidx_status lidx_decode_layer(const lidx_decode_args *args, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * lidx_sparse_attn_decode_noalloc -- lidx_sparse_attn_decode without a
 * caller workspace.  The pages have no counterpart: this exists for callers
 * that cannot allocate device memory when they call, such as a plugin hosted
 * by another runtime that provides no scratch allocator, or a serving loop
 * that forbids cudaMalloc after start-up (it can synchronise the device and
 * fragments a fixed memory budget).
 *
 * Same arguments and results as lidx_sparse_attn_decode.  The split-K
 * scratch lives in a device array of LIDX_NOALLOC_SCRATCH_BYTES owned by the
 * library; every GPU that loads the library holds it until the process exits.
 * The call allocates nothing.
 *  - Requests whose workspace (lidx_workspace_size(LIDX_OP_ATTN)) exceeds
 *    LIDX_NOALLOC_SCRATCH_BYTES are rejected with LIDX_ERR_WORKSPACE before
 *    anything is enqueued; use lidx_sparse_attn_decode for them.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls share the array and it keeps the last call's contents; the
 *    call clears the status word itself.  Calls whose work overlaps on the
 *    GPU (e.g. on two streams) race on the array: serialise them.
 *  - dev_status (optional, DEVICE pointer): receives this call's device
 *    status word (LIDX_DEV_* flags) when the call's work completes.
 * ------------------------------------------------------------------------ */
#define LIDX_NOALLOC_SCRATCH_BYTES (16u << 20)

LIDX_API lidx_status lidx_sparse_attn_decode_noalloc(const lidx_attn_args *args, uint32_t *dev_status,
                                                     void *stream);

/* ------------------------------------------------------------------------
 * lidx_cache_append -- the cache write side: quantise new rows into the
 * storage format and append them (architecture post, "why quantising the KV
 * does not save memory", point 1: non-RoPE dims as E4M3 with one
 * power-of-two scale per 64 elements, RoPE dims as bf16).
 *
 *   x      [B][R][dim] fp32, 16-byte aligned: the R new rows of each
 *          sequence (new compressed entries, or new window rows)
 *   cache  destination rows (dim 128 or 512; LIDX_F32 | LIDX_BF16 |
 *          LIDX_E4M3); its planes are WRITTEN.  Sequence b's region is rows
 *          b*batch_rows .. b*batch_rows + capacity - 1.
 *   pos    [B] int32 (device): new row r of sequence b goes to row
 *          pos[b] + r of its region, or to (pos[b] + r) mod ring when ring > 0
 *          (the sliding window as a ring of `ring` rows)
 * E4M3: for each 64-element block the scale is 2^e with e the smallest
 * integer in [-127, 127] such that the block's largest finite magnitude is
 * <= 448 * 2^e (the finest scale that fits; e = 0 for an all-zero block),
 * stored as the E8M0 byte e + 127; codes are x / 2^e rounded to the nearest
 * E4M3FN value, ties to even, magnitudes above 448 saturating; NaN is stored
 * as 0x7F.  bf16 values (RoPE dims, bf16 caches) round to nearest even.
 * A destination outside [0, capacity) is skipped and sets LIDX_DEV_BOUNDS;
 * a non-finite input sets LIDX_DEV_NAN.  Needs
 * lidx_workspace_size(LIDX_OP_APPEND) bytes (the status word).
 * ------------------------------------------------------------------------ */
typedef struct lidx_append_args {
    int32_t B, R;
    const float *x;
    lidx_kv cache;
    int64_t capacity;
    const int32_t *pos;
    int32_t ring;
    uint32_t flags; /* LIDX_LAUNCH_* */
} lidx_append_args;

LIDX_API lidx_status lidx_cache_append(const lidx_append_args *args, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * lidx_selection_eval -- selection evaluation over a tau-window.
 * `ops` is a bit mask; the requested steps run in this order:
 *
 *  LIDX_EVAL_GOLDEN  (FlashMemory-vs-native post, Act 3; write-up 3.2 step 1)
 *     probs[l][t][j] = (1/H) sum_h softmax_j(scale * qa[l][t][h] . kv_l[j])
 *     over the N entries of layer l (kv rows l*kv.batch_rows + j).
 *  LIDX_EVAL_GOLDEN_INDEX (write-up 3.2 step 1, which applies the softmax
 *     to the indexer logits: the other reading of the golden step)
 *     probs[l][t][j] = softmax_j(index_scores[l*T + t][j]) over the N
 *     entries, row r of index_scores at index_scores + r * ld_index_scores
 *     (>= N).  NaN and -inf scores carry no mass (a NaN sets LIDX_DEV_NAN);
 *     a row without a finite score is all zeros.  Excludes LIDX_EVAL_GOLDEN
 *     (both write probs).
 *  LIDX_EVAL_TOPP    (write-up 3.2 step 2)
 *     per row (l,t): with m_j = floor(probs_j * 2^40) and M = sum m_j, the
 *     shortest prefix of the ranking (probs descending, ties to the lower
 *     index) whose mass reaches ceil(M * top_p_num / top_p_den)
 *     -> topp_bits[l][t][W].  Rows need not sum to 1; a value outside
 *     [0, 1] or NaN carries no mass and sets LIDX_DEV_NAN.  N above 2^23
 *     (where the masses could overflow 64 bits) is LIDX_ERR_UNSUPPORTED.
 *  LIDX_EVAL_VOTE    (write-up 3.2 step 3)
 *     vote_bits[t] = { j : #{l : j in topp_bits[l][t]} >= min_votes },
 *     window_bits = union over t of vote_bits[t].
 *  LIDX_EVAL_LSA     (write-up sections 2.2 and 4.1)
 *     fetched_bits = { j : exists g, gate_logits[g][j] + gate_bias >= 0 }
 *     (sigmoid(z) >= 0.5 <=> z >= 0; the sum is rounded to fp32).
 *  LIDX_EVAL_OVERLAP (FlashMemory-vs-native post, Acts 1 and 3)
 *     counts[p] = { |A_p & B_p|, |A_p|, |B_p| } with A_p = set_a + p*ld_a,
 *     B_p = set_b + p*ld_b (ld 0 reuses one set for all pairs).
 *
 * Bit sets are uint32 [.][W], W = ceil(N/32), bit j%32 of word j/32; bits at
 * and beyond N are written as 0 and must be 0 on input.  Inputs of a step
 * may be the outputs of an earlier step in the same call.
 * Needs lidx_workspace_size(LIDX_OP_EVAL) bytes.
 * ------------------------------------------------------------------------ */
#define LIDX_EVAL_GOLDEN 0x1u
#define LIDX_EVAL_TOPP 0x2u
#define LIDX_EVAL_VOTE 0x4u
#define LIDX_EVAL_LSA 0x8u
#define LIDX_EVAL_OVERLAP 0x10u
#define LIDX_EVAL_GOLDEN_INDEX 0x20u

typedef struct lidx_eval_args {
    uint32_t ops;
    int32_t L, T, H, N;
    /* GOLDEN */
    int32_t qa_dtype;      /* LIDX_BF16 (LIDX_F32 with F32 rows) */
    const void *qa;        /* [L][T][H][512] */
    lidx_kv kv;            /* dim 512 */
    float scale;
    float *probs;          /* [L][T][N]: GOLDEN output, TOPP input */
    /* TOPP */
    uint32_t top_p_num, top_p_den;
    uint32_t *topp_bits;   /* [L][T][W]: TOPP output, VOTE input */
    /* VOTE */
    int32_t min_votes;
    uint32_t *vote_bits;   /* [T][W] (optional) */
    uint32_t *window_bits; /* [W] */
    /* LSA */
    int32_t n_gate;
    const float *gate_logits; /* [n_gate][N] */
    float gate_bias;
    uint32_t *fetched_bits;   /* [W] */
    /* OVERLAP */
    int32_t n_pairs;
    const uint32_t *set_a;
    int64_t ld_a;
    const uint32_t *set_b;
    int64_t ld_b;
    int64_t *counts;          /* [n_pairs][3] */
    /* GOLDEN_INDEX */
    const float *index_scores; /* [L*T][ld_index_scores] */
    int64_t ld_index_scores;
} lidx_eval_args;

LIDX_API lidx_status lidx_selection_eval(const lidx_eval_args *args, void *ws, size_t ws_bytes,
                                void *stream);

/* ------------------------------------------------------------------------
 * Workspace sizes, status, introspection.
 * ------------------------------------------------------------------------ */
#define LIDX_OP_SCORE 0
#define LIDX_OP_TOPK 1
#define LIDX_OP_ATTN 2
#define LIDX_OP_EVAL 3
#define LIDX_OP_DECODE 4
#define LIDX_OP_APPEND 5

/* Bytes of workspace call `op` needs for `args` (a pointer to the matching
 * *_args struct, host memory).  Score needs none (0). */
LIDX_API lidx_status lidx_workspace_size(int op, const void *args, size_t *bytes);

/* Number of kernels call `op` launches for `args` (host memory), after the
 * same argument checks as the call (their status on failure): 1 for the
 * scorer, the decode layer and the append; 1 for lidx_topk_select on rows
 * one cluster holds, 4 beyond (segment selects, candidate gather, candidate
 * select, map back); 2 for lidx_sparse_attn_decode (split kernel, merge);
 * for lidx_selection_eval the sum over the requested ops.  Memsets and
 * copies a call enqueues are not counted.  For launch accounting and for
 * checking a captured graph. */
LIDX_API lidx_status lidx_launch_count(int op, const void *args, int *count);

/* Synchronises `stream`, copies the status word at the start of `ws` into
 * *status (host) and clears it on the device. */
LIDX_API lidx_status lidx_read_device_status(void *ws, uint32_t *status, void *stream);

/* Static description of a status code. */
LIDX_API const char *lidx_status_string(lidx_status s);

/* LIDX_ABI_VERSION of the loaded library. */
LIDX_API int lidx_abi_version(void);

/* sizeof() of the argument structs as compiled into the library, for binding
 * checks: which = 0 lidx_kv, 1 score, 2 topk, 3 attn, 4 eval, 5 decode,
 * 6 append. */
LIDX_API size_t lidx_struct_size(int which);

#ifdef __cplusplus
}
#endif

#endif /* LIDX_H */
