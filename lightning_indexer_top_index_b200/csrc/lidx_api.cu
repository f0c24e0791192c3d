// C ABI of liblidx.so: argument validation, dispatch to the kernels,
// workspace sizing and the device status word.  See include/lidx.h.
#include <mutex>

#include "kernels.cuh"

using namespace lidx;

namespace {

constexpr int kMaxDevices = 64;
int g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other
std::mutex g_dev_mu;

lidx_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LIDX_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LIDX_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev_ok[dev] == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return LIDX_ERR_CUDA;
    }
    g_dev_ok[dev] = major == 10 ? 1 : 2;
  }
  return g_dev_ok[dev] == 1 ? LIDX_OK : LIDX_ERR_UNSUPPORTED;
}

bool aligned(const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

size_t elem_size(int dt) { return dt == LIDX_F32 ? 4 : dt == LIDX_BF16 ? 2 : 1; }

// Layout checks of a row set; `rows_per_batch` is the largest row index used + 1
// within one batch entry.
lidx_status check_kv(const lidx_kv &k, int dim, int B, int64_t rows_per_batch, bool overlap_ok = false) {
  if (k.dtype == LIDX_F16) return LIDX_ERR_UNSUPPORTED;
  if (k.dtype != LIDX_F32 && k.dtype != LIDX_BF16 && k.dtype != LIDX_E4M3) return LIDX_ERR_INVALID_ARG;
  if (k.dim != dim) return LIDX_ERR_UNSUPPORTED;
  if (!k.data) return LIDX_ERR_INVALID_ARG;
  const int64_t stored = k.dtype == LIDX_E4M3 ? dim - 64 : dim;
  if (k.ld < stored) return LIDX_ERR_INVALID_ARG;
  if (!aligned(k.data, 16) || (k.ld * static_cast<int64_t>(elem_size(k.dtype))) % 16 != 0) return LIDX_ERR_INVALID_ARG;
  if (k.dtype == LIDX_E4M3) {
    if (!k.scale || !k.rope) return LIDX_ERR_INVALID_ARG;
    if (k.ld_scale < (dim - 64) / 64 || k.ld_rope < 64) return LIDX_ERR_INVALID_ARG;
    if (!aligned(k.rope, 16) || (k.ld_rope * 2) % 16 != 0) return LIDX_ERR_INVALID_ARG;
  }
  if (B > 1 && (overlap_ok ? k.batch_rows < 0 : k.batch_rows < rows_per_batch)) return LIDX_ERR_INVALID_ARG;
  return LIDX_OK;
}

lidx_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LIDX_OK : LIDX_ERR_CUDA; }

lidx_status check_score(const lidx_score_args *a) {
  if (!a || !a->q || !a->w || !a->scores) return LIDX_ERR_INVALID_ARG;
  if (a->B < 1 || a->Q < 1 || a->H < 1 || a->H > 128 || a->N < 1 || a->ld_scores < a->N) return LIDX_ERR_INVALID_ARG;
  lidx_status s = check_kv(a->keys, 128, a->B, a->N);
  if (s != LIDX_OK) return s;
  if (a->keys.dtype == LIDX_F32 && a->q_dtype != LIDX_F32) return LIDX_ERR_UNSUPPORTED;
  if (a->keys.dtype != LIDX_F32 && a->q_dtype != LIDX_BF16) return LIDX_ERR_UNSUPPORTED;
  if (!aligned(a->q, 4) || !aligned(a->w, 4) || !aligned(a->scores, 4)) return LIDX_ERR_INVALID_ARG;
  if (a->tile_stats && !aligned(a->tile_stats, 8)) return LIDX_ERR_INVALID_ARG;
  if (a->n_visible && !aligned(a->n_visible, 4)) return LIDX_ERR_INVALID_ARG;
  return LIDX_OK;
}

lidx_status check_topk(const lidx_topk_args *a) {
  if (!a || !a->scores || !a->ids) return LIDX_ERR_INVALID_ARG;
  if (a->B < 1 || a->Q < 1 || a->N < 1 || a->k < 1 || a->ld_scores < a->N) return LIDX_ERR_INVALID_ARG;
  if (a->allowed && a->ld_allowed < a->N) return LIDX_ERR_INVALID_ARG;
  if (a->allowed_bits && (a->ld_allowed_bits < (a->N + 31) / 32 || !aligned(a->allowed_bits, 4)))
    return LIDX_ERR_INVALID_ARG;
  if (!aligned(a->scores, 4) || !aligned(a->ids, 4) || (a->mask_bits && !aligned(a->mask_bits, 4)))
    return LIDX_ERR_INVALID_ARG;
  if (a->tile_stats && !aligned(a->tile_stats, 8)) return LIDX_ERR_INVALID_ARG;
  if (a->n_valid && !aligned(a->n_valid, 4)) return LIDX_ERR_INVALID_ARG;
  if (!topk_supported(*a)) return LIDX_ERR_UNSUPPORTED;
  return LIDX_OK;
}

lidx_status check_attn(const lidx_attn_args *a) {
  if (!a || !a->q || !a->out) return LIDX_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->H > 64 || a->n_ids < 0 || a->swa_len < 0) return LIDX_ERR_INVALID_ARG;
  if (a->n_ids > 0 && a->N < 1) return LIDX_ERR_INVALID_ARG;
  if (a->n_ids > 0 && a->ids && a->ld_ids < a->n_ids) return LIDX_ERR_INVALID_ARG;
  if (a->n_ids > a->N && !a->ids) return LIDX_ERR_INVALID_ARG;  // dense rows 0..n_ids-1 must exist
  if (!(a->scale == a->scale) || a->scale == INFINITY || a->scale == -INFINITY) return LIDX_ERR_INVALID_ARG;
  if (a->n_ids > 0) {
    lidx_status s = check_kv(a->kv, 512, a->B, a->N, true);
    if (s != LIDX_OK) return s;
  } else if (a->kv.dtype == LIDX_F16) {
    return LIDX_ERR_UNSUPPORTED;
  }
  if (a->swa_len > 0) {
    lidx_status s = check_kv(a->swa, 512, a->B, a->swa_len, true);
    if (s != LIDX_OK) return s;
    if (a->n_ids > 0 && a->swa.dtype != a->kv.dtype) return LIDX_ERR_UNSUPPORTED;
  }
  const int rows_dt = a->n_ids > 0 ? a->kv.dtype : a->swa.dtype;
  if (rows_dt == LIDX_F32 && a->q_dtype != LIDX_F32) return LIDX_ERR_UNSUPPORTED;
  if (rows_dt != LIDX_F32 && a->q_dtype != LIDX_BF16) return LIDX_ERR_UNSUPPORTED;
  if (!aligned(a->q, 4) || !aligned(a->out, 4)) return LIDX_ERR_INVALID_ARG;
  return LIDX_OK;
}

lidx_status check_eval(const lidx_eval_args *a) {
  if (!a || a->ops == 0 || (a->ops & ~0x3Fu)) return LIDX_ERR_INVALID_ARG;
  if ((a->ops & LIDX_EVAL_GOLDEN) && (a->ops & LIDX_EVAL_GOLDEN_INDEX)) return LIDX_ERR_INVALID_ARG;
  if (a->N < 1) return LIDX_ERR_INVALID_ARG;
  if (a->ops & LIDX_EVAL_GOLDEN) {
    if (!a->qa || !a->probs || a->L < 1 || a->T < 1 || a->H < 1 || a->H > 64) return LIDX_ERR_INVALID_ARG;
    lidx_status s = check_kv(a->kv, 512, a->L, a->N);
    if (s != LIDX_OK) return s;
    if (a->kv.dtype == LIDX_F32 ? a->qa_dtype != LIDX_F32 : a->qa_dtype != LIDX_BF16) return LIDX_ERR_UNSUPPORTED;
  }
  if (a->ops & LIDX_EVAL_GOLDEN_INDEX) {
    if (!a->index_scores || !a->probs || a->L < 1 || a->T < 1 || a->ld_index_scores < a->N) return LIDX_ERR_INVALID_ARG;
    if (!aligned(a->index_scores, 4) || !aligned(a->probs, 4)) return LIDX_ERR_INVALID_ARG;
  }
  if (a->ops & LIDX_EVAL_TOPP) {
    if (!a->probs || !a->topp_bits || a->L < 1 || a->T < 1) return LIDX_ERR_INVALID_ARG;
    if (a->top_p_den == 0 || a->top_p_num > a->top_p_den) return LIDX_ERR_INVALID_ARG;
    if (a->N > (1 << 23)) return LIDX_ERR_UNSUPPORTED;  // fixed-point mass must fit 64 bits
  }
  if (a->ops & LIDX_EVAL_VOTE) {
    if (!a->topp_bits || !a->window_bits || a->L < 1 || a->T < 1 || a->min_votes < 0) return LIDX_ERR_INVALID_ARG;
  }
  if (a->ops & LIDX_EVAL_LSA) {
    if (!a->gate_logits || !a->fetched_bits || a->n_gate < 1) return LIDX_ERR_INVALID_ARG;
  }
  if (a->ops & LIDX_EVAL_OVERLAP) {
    if (!a->set_a || !a->set_b || !a->counts || a->n_pairs < 1 || a->ld_a < 0 || a->ld_b < 0) return LIDX_ERR_INVALID_ARG;
  }
  return LIDX_OK;
}

lidx_status check_decode(const lidx_decode_args *a) {
  if (!a || !a->q_idx || !a->w || !a->q_attn || !a->out) return LIDX_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->N < 1 || a->k < 1 || a->swa_len < 0 || a->H_attn < 1) return LIDX_ERR_INVALID_ARG;
  if (!(a->scale == a->scale) || a->scale == INFINITY || a->scale == -INFINITY) return LIDX_ERR_INVALID_ARG;
  lidx_status s = check_kv(a->keys, 128, a->B, a->N);
  if (s != LIDX_OK) return s;
  if ((s = check_kv(a->kv, 512, a->B, a->N)) != LIDX_OK) return s;
  if (a->swa_len > 0 && (s = check_kv(a->swa, 512, a->B, a->swa_len)) != LIDX_OK) return s;
  if (a->scores && a->ld_scores < a->N) return LIDX_ERR_INVALID_ARG;
  if (!aligned(a->q_idx, 16) || !aligned(a->q_attn, 16) || !aligned(a->w, 4) || !aligned(a->out, 16))
    return LIDX_ERR_INVALID_ARG;
  if ((a->scores && !aligned(a->scores, 4)) || (a->ids && !aligned(a->ids, 4)) || (a->n_sel && !aligned(a->n_sel, 4)) ||
      (a->lse && !aligned(a->lse, 4)))
    return LIDX_ERR_INVALID_ARG;
  for (int r = 0; r < 2; r++)
    if (a->prefetch[r] && (!aligned(a->prefetch[r], 16) || a->prefetch_bytes[r] % 16 != 0)) return LIDX_ERR_INVALID_ARG;
  if (!decode_fused_supported(*a)) return LIDX_ERR_UNSUPPORTED;
  return LIDX_OK;
}

lidx_status check_append(const lidx_append_args *a) {
  if (!a || !a->x || !a->pos) return LIDX_ERR_INVALID_ARG;
  if (a->B < 1 || a->R < 1 || a->capacity < 1 || a->ring < 0 || a->ring > a->capacity) return LIDX_ERR_INVALID_ARG;
  if (a->cache.dim != 128 && a->cache.dim != 512) return LIDX_ERR_UNSUPPORTED;
  lidx_status s = check_kv(a->cache, a->cache.dim, a->B, a->capacity);
  if (s != LIDX_OK) return s;
  if (!aligned(a->x, 16) || !aligned(a->pos, 4)) return LIDX_ERR_INVALID_ARG;
  if (a->cache.dtype == LIDX_E4M3 && (a->cache.ld % 8 != 0)) return LIDX_ERR_INVALID_ARG;
  return LIDX_OK;
}

lidx_status check_ws(void *ws, size_t have, size_t need) {
  if (!ws || !aligned(ws, 256)) return need ? LIDX_ERR_WORKSPACE : LIDX_OK;
  return have >= need ? LIDX_OK : LIDX_ERR_WORKSPACE;
}

}  // namespace

namespace lidx {
lidx_status check_device_sm100() { return check_device(); }
}  // namespace lidx

extern "C" {

lidx_status lidx_index_score(const lidx_score_args *args, void *stream) {
  lidx_status s = check_score(args);
  if (s != LIDX_OK) return s;
  if ((s = check_device()) != LIDX_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (score_tc_supported(*args)) return from_cuda(launch_score_tc(*args, st));
  return from_cuda(launch_score_cc(*args, st));
}

lidx_status lidx_topk_select(const lidx_topk_args *args, void *ws, size_t ws_bytes, void *stream) {
  lidx_status s = check_topk(args);
  if (s != LIDX_OK) return s;
  if ((s = check_ws(ws, ws_bytes, topk_workspace(*args))) != LIDX_OK) return s;
  if ((s = check_device()) != LIDX_OK) return s;
  return from_cuda(launch_topk(*args, ws, static_cast<cudaStream_t>(stream)));
}

lidx_status lidx_sparse_attn_decode(const lidx_attn_args *args, void *ws, size_t ws_bytes, void *stream) {
  lidx_status s = check_attn(args);
  if (s != LIDX_OK) return s;
  if ((s = check_ws(ws, ws_bytes, attn_workspace(*args))) != LIDX_OK) return s;
  if ((s = check_device()) != LIDX_OK) return s;
  return from_cuda(launch_attn(*args, ws, static_cast<cudaStream_t>(stream)));
}

lidx_status lidx_selection_eval(const lidx_eval_args *args, void *ws, size_t ws_bytes, void *stream) {
  lidx_status s = check_eval(args);
  if (s != LIDX_OK) return s;
  if ((s = check_ws(ws, ws_bytes, eval_workspace(*args))) != LIDX_OK) return s;
  if ((s = check_device()) != LIDX_OK) return s;
  return from_cuda(launch_eval(*args, ws, static_cast<cudaStream_t>(stream)));
}

lidx_status lidx_decode_layer(const lidx_decode_args *args, void *ws, size_t ws_bytes, void *stream) {
  lidx_status s = check_device();
  if (s != LIDX_OK) return s;
  if ((s = check_decode(args)) != LIDX_OK) return s;
  if ((s = check_ws(ws, ws_bytes, decode_fused_workspace(*args))) != LIDX_OK) return s;
  return from_cuda(launch_decode_fused(*args, ws, static_cast<cudaStream_t>(stream)));
}

lidx_status lidx_cache_append(const lidx_append_args *args, void *ws, size_t ws_bytes, void *stream) {
  lidx_status s = check_append(args);
  if (s != LIDX_OK) return s;
  if ((s = check_ws(ws, ws_bytes, LIDX_WS_HEADER)) != LIDX_OK) return s;
  if ((s = check_device()) != LIDX_OK) return s;
  return from_cuda(launch_append(*args, ws, static_cast<cudaStream_t>(stream)));
}

lidx_status lidx_workspace_size(int op, const void *args, size_t *bytes) {
  if (!args || !bytes) return LIDX_ERR_INVALID_ARG;
  lidx_status s = LIDX_OK;
  switch (op) {
    case LIDX_OP_SCORE:
      s = check_score(static_cast<const lidx_score_args *>(args));
      *bytes = 0;
      break;
    case LIDX_OP_TOPK:
      s = check_topk(static_cast<const lidx_topk_args *>(args));
      if (s == LIDX_OK) *bytes = topk_workspace(*static_cast<const lidx_topk_args *>(args));
      break;
    case LIDX_OP_ATTN:
      s = check_attn(static_cast<const lidx_attn_args *>(args));
      if (s == LIDX_OK) *bytes = attn_workspace(*static_cast<const lidx_attn_args *>(args));
      break;
    case LIDX_OP_EVAL:
      s = check_eval(static_cast<const lidx_eval_args *>(args));
      if (s == LIDX_OK) *bytes = eval_workspace(*static_cast<const lidx_eval_args *>(args));
      break;
    case LIDX_OP_APPEND:
      s = check_append(static_cast<const lidx_append_args *>(args));
      if (s == LIDX_OK) *bytes = LIDX_WS_HEADER;
      break;
    case LIDX_OP_DECODE:
      s = check_decode(static_cast<const lidx_decode_args *>(args));
      if (s == LIDX_OK) *bytes = decode_fused_workspace(*static_cast<const lidx_decode_args *>(args));
      break;
    default:
      return LIDX_ERR_INVALID_ARG;
  }
  return s;
}

lidx_status lidx_launch_count(int op, const void *args, int *count) {
  if (!args || !count) return LIDX_ERR_INVALID_ARG;
  lidx_status s = LIDX_OK;
  switch (op) {
    case LIDX_OP_SCORE:
      s = check_score(static_cast<const lidx_score_args *>(args));
      if (s == LIDX_OK) *count = 1;
      break;
    case LIDX_OP_TOPK:
      s = check_topk(static_cast<const lidx_topk_args *>(args));
      if (s == LIDX_OK) *count = topk_launches(*static_cast<const lidx_topk_args *>(args));
      break;
    case LIDX_OP_ATTN:
      s = check_attn(static_cast<const lidx_attn_args *>(args));
      if (s == LIDX_OK) *count = attn_launches(*static_cast<const lidx_attn_args *>(args));
      break;
    case LIDX_OP_EVAL:
      s = check_eval(static_cast<const lidx_eval_args *>(args));
      if (s == LIDX_OK) *count = eval_launches(*static_cast<const lidx_eval_args *>(args));
      break;
    case LIDX_OP_APPEND:
      s = check_append(static_cast<const lidx_append_args *>(args));
      if (s == LIDX_OK) *count = 1;
      break;
    case LIDX_OP_DECODE:
      s = check_decode(static_cast<const lidx_decode_args *>(args));
      if (s == LIDX_OK) *count = 1;
      break;
    default:
      return LIDX_ERR_INVALID_ARG;
  }
  return s;
}

lidx_status lidx_read_device_status(void *ws, uint32_t *status, void *stream) {
  if (!ws || !status) return LIDX_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess) return LIDX_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return LIDX_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LIDX_ERR_CUDA;
  return LIDX_OK;
}

const char *lidx_status_string(lidx_status s) {
  switch (s) {
    case LIDX_OK: return "ok";
    case LIDX_ERR_INVALID_ARG: return "invalid argument";
    case LIDX_ERR_UNSUPPORTED: return "unsupported format, shape or device";
    case LIDX_ERR_CUDA: return "CUDA runtime error";
    case LIDX_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int lidx_abi_version(void) { return LIDX_ABI_VERSION; }

size_t lidx_struct_size(int which) {
  switch (which) {
    case 0: return sizeof(lidx_kv);
    case 1: return sizeof(lidx_score_args);
    case 2: return sizeof(lidx_topk_args);
    case 3: return sizeof(lidx_attn_args);
    case 4: return sizeof(lidx_eval_args);
    case 5: return sizeof(lidx_decode_args);
    case 6: return sizeof(lidx_append_args);
  }
  return 0;
}

}  // extern "C"
