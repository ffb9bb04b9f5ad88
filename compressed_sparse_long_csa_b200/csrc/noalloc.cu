// sparse_attn_decode_noalloc: the sparse decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot hand the library a workspace.  Examples: code that runs
// under an allocator it does not control, such as a plugin inside another
// framework's memory pool; a real-time path that must not call cudaMalloc, which
// can synchronise the device and take milliseconds; and environments where every
// device allocation must be budgeted up front.  For them, the split-KV partials of
// the decode attention live in a fixed buffer that the library itself owns: a
// file-scope __device__ array of CSA_NOALLOC_SCRATCH_BYTES.  Every GPU that loads
// the library holds this buffer until the process exits.
//
// The array's name, used in host code, is only a host-side handle, not a device
// address.  Passing it to a kernel would fault, or, where the GPU can reach host
// memory, silently use the wrong memory.  The device address is therefore looked
// up once per device with cudaGetSymbolAddress, with that device current, and the
// result is cached.
#include <mutex>

#include "../../include/csa.h"
#include <cuda_runtime.h>

// 32 MiB of fp32 split partials.
static __device__ __align__(256) float g_csa_noalloc_scratch[CSA_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up on first use).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_csa_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" csa_status sparse_attn_decode_noalloc(const void* q, const void* cache, const int32_t* idx,
                                                 const void* win, const int32_t* win_len, const float* sink,
                                                 int B, int H, int d_k, int d_v, int64_t n_max, int k, int W,
                                                 float sm_scale, int dtype, void* out, float* lse, void* stream) {
  // The partials this call needs must fit the fixed buffer; larger requests are
  // refused before any device work.
  if (B < 1 || H < 1 || d_v < 1 || k < 0 || W < 0) return CSA_ERR_SHAPE;
  const size_t need = attn_decode_workspace_size(B, H, d_v, (int64_t)k + W);
  if (need > (size_t)CSA_NOALLOC_SCRATCH_BYTES) return CSA_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return CSA_ERR_CUDA;
  // Every partial record is rewritten by the kernels of each call, so nothing in the
  // buffer has to start at zero.
  return sparse_attn_decode(q, cache, idx, win, win_len, sink, B, H, d_k, d_v, n_max, k, W, sm_scale, dtype, out, lse,
                            scratch, (size_t)CSA_NOALLOC_SCRATCH_BYTES, stream);
}
