// Ring forward for callers that cannot allocate device memory.
//
// cbv_zigzag_ring_fwd needs a caller-provided workspace (the device status word and
// the tile schedule it uploads).  Some callers cannot call cudaMalloc at the point
// where they run attention: code inside an allocation-free serving loop whose memory
// budget was fixed at start-up, foreign runtimes that own every device buffer through
// their own allocator and hand out none for scratch, or plain C hosts with no device
// allocator of their own.  For them this file keeps the scratch in a file-scope
// __device__ array of fixed size that lives as long as the library is loaded, and
// runs the same fused ring forward out of it.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/cbv.h"

namespace cbv {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kScratchBytes = (size_t)1 << 20;  // 1 MiB: status word + tile schedule
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

thread_local char g_msg[256];

int fail(int code) {
  cbv::set_last_error(g_msg);
  return code;
}

// Device address of g_scratch on the current device; looked up once per device.
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof g_msg, "cudaGetDevice: %s", cudaGetErrorString(e));
    return fail(CBV_ERR_CUDA);
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(g_msg, sizeof g_msg, "device %d is beyond the %d devices this library tracks", dev, kMaxDevices);
    return fail(CBV_ERR_BAD_ARG);
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(g_msg, sizeof g_msg, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
      return fail(CBV_ERR_CUDA);
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return CBV_OK;
}

}  // namespace

extern "C" {

size_t cbv_noalloc_scratch_bytes(void) { return kScratchBytes; }

int cbv_zigzag_ring_fwd_noalloc(const cbv_ring_args* a, void* stream) {
  if (!a) {
    snprintf(g_msg, sizeof g_msg, "args is NULL");
    return fail(CBV_ERR_BAD_ARG);
  }
  const size_t need = cbv_zigzag_ring_fwd_workspace_size(a);
  if (need == 0) return cbv_zigzag_ring_fwd(a, stream);  // invalid arguments: same status and message
  if (need > kScratchBytes) {
    snprintf(g_msg, sizeof g_msg,
             "this problem needs %zu bytes of scratch; the static scratch holds %zu (use cbv_zigzag_ring_fwd "
             "with a caller-provided workspace)",
             need, kScratchBytes);
    return fail(CBV_ERR_WORKSPACE_TOO_SMALL);
  }
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != CBV_OK) return rc;
  cbv_ring_args b = *a;
  b.workspace = scratch;
  b.workspace_bytes = kScratchBytes;
  return cbv_zigzag_ring_fwd(&b, stream);
}

}  // extern "C"
