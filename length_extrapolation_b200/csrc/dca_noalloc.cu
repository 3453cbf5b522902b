// dca_noalloc.cu -- one-shot DCA prefill that allocates no device memory.
//
// Some callers cannot call cudaMalloc: a serving process that reserved all
// free HBM for its own pool at start-up (where a late cudaMalloc fails or
// stalls the device), or a plugin whose host framework owns every device
// allocation.  For them this entry point uses a fixed scratch area that is
// part of the library image (a file-scope __device__ array), so the caller
// passes only its inputs and outputs.  The array exists on a GPU once the
// library's device code is loaded there (at its first use on that device
// under lazy module loading; dca_noalloc_prepare forces it), until the
// process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dca.h"
#include "dca_internal.h"

// The scratch: RoPE table, rotated keys and the status word of one call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DCA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current and kept (stale after cudaDeviceReset).
// The lookup also loads the module on the device under lazy loading.
int scratch_on_current_device(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DCA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return DCA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return DCA_OK;
}

}  // namespace

extern "C" int dca_noalloc_prepare(void) {
  void* scratch = nullptr;
  return scratch_on_current_device(&scratch);
}

extern "C" int dca_noalloc_device_status(void* cuda_stream) {
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != DCA_OK) return rc;
  return dca_device_status(scratch, cuda_stream);
}

extern "C" int dca_prefill_noalloc(const void* q, const void* k, const void* v, void* out,
                                   int64_t L, int Hq, int Hkv, int d, int64_t chunk_size,
                                   int64_t local_window, int64_t pretrain_window,
                                   double rope_base, double yarn_scale, int dtype,
                                   void* cuda_stream) {
  const size_t need = dca_workspace_size(L, Hq, Hkv, d, chunk_size, local_window,
                                         pretrain_window, dtype);
  if (need == 0) return DCA_ERR_ARG;
  if (need > DCA_NOALLOC_SCRATCH_BYTES) return DCA_ERR_WORKSPACE;  // problem too large
  void* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != DCA_OK) return rc;
  // every argument is checked before the shared scratch is touched, so a
  // rejected call leaves the status word of an earlier call alone
  rc = dca::check_prefill_args(q, k, v, out, L, Hq, Hkv, d, chunk_size, local_window,
                               pretrain_window, rope_base, yarn_scale, dtype, scratch,
                               DCA_NOALLOC_SCRATCH_BYTES);
  if (rc != DCA_OK || L == 0) return rc;
  // the previous call's status word must not leak into this one
  rc = dca_workspace_init(scratch, DCA_NOALLOC_SCRATCH_BYTES, cuda_stream);
  if (rc != DCA_OK) return rc;
  return dca_prefill(q, k, v, out, L, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                     rope_base, yarn_scale, dtype, scratch, DCA_NOALLOC_SCRATCH_BYTES,
                     cuda_stream);
}
