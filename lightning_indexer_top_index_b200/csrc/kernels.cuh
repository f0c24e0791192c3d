// Internal launchers of the lidx kernels.  Every launcher only enqueues work
// on `st` and returns the launch error; arguments were validated by the C-ABI
// layer (lidx_api.cu).
#pragma once

#include "common.cuh"

namespace lidx {

// Scratch layout inside a caller workspace: a 256-byte header whose first
// word is the device status word, then the op's own region.
struct WsHeader {
  uint32_t status;
  uint32_t pad[63];
};

// LIDX_OK when the current device is an sm_100 part, else UNSUPPORTED (or
// CUDA when the device cannot be queried); leaves no pending CUDA error.
lidx_status check_device_sm100();

// ---- index score
cudaError_t launch_score_cc(const lidx_score_args &a, cudaStream_t st);
// tcgen05 scorer; returns cudaErrorNotSupported when the shape is not covered.
cudaError_t launch_score_tc(const lidx_score_args &a, cudaStream_t st);
bool score_tc_supported(const lidx_score_args &a);

// ---- top-k
bool topk_supported(const lidx_topk_args &a);
size_t topk_workspace(const lidx_topk_args &a);
int topk_launches(const lidx_topk_args &a);  // kernels one call launches
cudaError_t launch_topk(const lidx_topk_args &a, void *ws, cudaStream_t st);

// ---- sparse attention decode
size_t attn_workspace(const lidx_attn_args &a);
int attn_launches(const lidx_attn_args &a);  // kernels one call launches
cudaError_t launch_attn(const lidx_attn_args &a, void *ws, cudaStream_t st);

// ---- fused decode layer (score -> top-k -> attention in one launch)
bool decode_fused_supported(const lidx_decode_args &a);
size_t decode_fused_workspace(const lidx_decode_args &a);
cudaError_t launch_decode_fused(const lidx_decode_args &a, void *ws, cudaStream_t st);

// ---- cache write side
cudaError_t launch_append(const lidx_append_args &a, void *ws, cudaStream_t st);

// ---- selection evaluation
bool golden_tc_supported(const lidx_eval_args &a);
size_t golden_tc_workspace(const lidx_eval_args &a);
cudaError_t launch_golden_tc(const lidx_eval_args &a, void *scratch, uint32_t *status, cudaStream_t st);
size_t eval_workspace(const lidx_eval_args &a);
int eval_launches(const lidx_eval_args &a);
cudaError_t launch_eval(const lidx_eval_args &a, void *ws, cudaStream_t st);

}  // namespace lidx
