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
#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LIDX_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the array on the current device, looked up once per
// device.  In host code the array's name is only a host-side stand-in; the
// kernels must receive the address the runtime reports.
lidx_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LIDX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LIDX_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LIDX_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LIDX_OK;
}

}  // namespace

extern "C" LIDX_API lidx_status lidx_sparse_attn_decode_noalloc(const lidx_attn_args *args, uint32_t *dev_status,
                                                                 void *stream) {
  size_t need = 0;
  lidx_status s = lidx_workspace_size(LIDX_OP_ATTN, args, &need);
  if (s != LIDX_OK) return s;
  if (need > LIDX_NOALLOC_SCRATCH_BYTES) return LIDX_ERR_WORKSPACE;
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
