// Allocation-free variant of the sparse decode attention.
//
// Some callers cannot hand the library a workspace: a plugin hosted by
// another runtime that gives it no scratch allocator, or a serving loop that
// forbids device allocation once it has started (cudaMalloc can synchronise
// the device and fragments a fixed memory budget).  For them this entry point
// keeps the split-K scratch in a fixed device array that belongs to the
// library and runs the same kernels as lidx_sparse_attn_decode.
//
// The array is LIDX_NOALLOC_SCRATCH_BYTES long and every GPU that loads the
// library holds it until the process exits.  All calls share it, so calls
// whose work overlaps on the GPU (for example on two streams) race on it.
#include <cuda.h>

#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LIDX_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx_id;  // driver context the address belongs to (0: none yet)
  void *addr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrent = CUresult (*)(CUcontext *);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the current driver context (ids are never reused within a
// process, unlike context handles); false when it cannot be read.
bool current_ctx_id(unsigned long long *id) {
  static CtxGetCurrent get_current = nullptr;
  static CtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetId>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the array in the current device's context.  In host code
// the array's name is only a host-side stand-in; the kernels must receive the
// address the runtime reports.  The address is looked up on the first call in
// each context and again whenever the device's context has changed (after a
// cudaDeviceReset the module is loaded anew and the array may move).
lidx_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LIDX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LIDX_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchAddr &e = g_scratch_addr[dev];
  if (!have_id || !e.addr || e.ctx_id != id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // leave no pending error behind
      return LIDX_ERR_CUDA;
    }
    e.addr = p;
    e.ctx_id = have_id ? id : 0;
    if (!have_id) {  // no context id to key on: look the address up on every call
      *out = p;
      e.addr = nullptr;
      return LIDX_OK;
    }
  }
  *out = e.addr;
  return LIDX_OK;
}

}  // namespace

extern "C" LIDX_API lidx_status lidx_sparse_attn_decode_noalloc(const lidx_attn_args *args, uint32_t *dev_status,
                                                                 void *stream) {
  size_t need = 0;
  lidx_status s = lidx_workspace_size(LIDX_OP_ATTN, args, &need);
  if (s != LIDX_OK) return s;
  if (need > LIDX_NOALLOC_SCRATCH_BYTES) return LIDX_ERR_WORKSPACE;
  // an unsupported device has no kernel image, so the symbol lookup below
  // would fail with a CUDA error: report it as unsupported instead
  if ((s = lidx::check_device_sm100()) != LIDX_OK) return s;
  void *scratch = nullptr;
  if ((s = scratch_address(&scratch)) != LIDX_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word is the only scratch that must start at zero
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), st) != cudaSuccess) return LIDX_ERR_CUDA;
  s = lidx_sparse_attn_decode(args, scratch, LIDX_NOALLOC_SCRATCH_BYTES, stream);
  if (s != LIDX_OK) return s;
  if (dev_status && cudaMemcpyAsync(dev_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return LIDX_ERR_CUDA;
  return LIDX_OK;
}
