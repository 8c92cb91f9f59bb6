// prefill_static.cu -- gdn_chunk_prefill_static_ws: the chunked prefill with its scratch in a
// fixed device array owned by this library, for callers that cannot allocate device memory.
//
// The scratch is a file-scope __device__ array of GDN_STATIC_WORKSPACE_BYTES.  Every GPU that
// loads this library holds it until the process exits.  In host code the array's name is only
// a host-side stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached; kernels always receive that
// address.  The entry point itself allocates nothing.
#include <cuda_runtime.h>

#include <mutex>

#include "args.cuh"
#include "common.cuh"

namespace gdn_host {
size_t prefill_tc_workspace(int N, int T, int Hk, int Hv);
}

static __device__ __align__(256) uint8_t g_static_workspace[GDN_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device (set-up on first use).
cudaError_t static_workspace_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int gdn_chunk_prefill_static_ws(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                                           const void* conv_w, const float* beta, const float* g,
                                           const void* z, const void* norm_w,
                                           const int32_t* cu_seqlens, int32_t num_seqs,
                                           int32_t num_tokens, const float* S0, float* SN,
                                           const void* conv0, void* convN, void* out,
                                           int32_t* dev_status, void* stream) {
  const size_t need = gdn_chunk_prefill_workspace_size(dims, dtype, num_seqs, num_tokens);
  if (need == 0)  // invalid shape: let the regular entry point report which status applies
    return gdn_chunk_prefill(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                             num_tokens, S0, SN, conv0, convN, out, nullptr, 0, dev_status, stream);
  if (need > (size_t)GDN_STATIC_WORKSPACE_BYTES) return GDN_ERR_WORKSPACE;
  void* ws = nullptr;
  if (static_workspace_address(&ws) != cudaSuccess) return GDN_ERR_CUDA;
  // Nothing in the scratch has to start at zero: every byte a kernel reads was written earlier
  // in the same call.  Calls that overlap on the GPU share the array and therefore race.
  return gdn_chunk_prefill(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                           num_tokens, S0, SN, conv0, convN, out, ws,
                           (size_t)GDN_STATIC_WORKSPACE_BYTES, dev_status, stream);
}
