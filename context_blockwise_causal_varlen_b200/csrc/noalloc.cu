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

#include "api_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)1 << 20;  // 1 MiB: status word + tile schedule
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

thread_local char g_msg[256];

int fail(int code) {
  cbv::set_last_error(g_msg);
  return code;
}

// Device address of g_scratch in the current device's context.  Looked up on every call (the
// lookup allocates nothing), so a context torn down and created again (cudaDeviceReset) never
// leaves a stale address behind.  The first lookup on a device loads the library's module
// into that device's context, which must not happen inside a stream capture.
int scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess || !p) {
    snprintf(g_msg, sizeof g_msg, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
    return fail(CBV_ERR_CUDA);
  }
  *out = p;
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
  cbv_ring_args b = *a;
  b.schedule = CBV_SCHEDULE_FUSED;  // the stepwise schedule's fp32 running output does not fit
  cbv::RingFwdLayout L;
  int rc = cbv::ring_fwd_plan(&b, &L);  // argument errors: the status and message of cbv_zigzag_ring_fwd
  if (rc != CBV_OK || b.total == 0) return rc;
  if (L.bytes > kScratchBytes) {
    snprintf(g_msg, sizeof g_msg,
             "this problem needs %zu bytes of scratch; the static scratch holds %zu (use cbv_zigzag_ring_fwd "
             "with a caller-provided workspace)",
             L.bytes, kScratchBytes);
    return fail(CBV_ERR_WORKSPACE_TOO_SMALL);
  }
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != CBV_OK) return rc;
  b.workspace = scratch;
  b.workspace_bytes = kScratchBytes;
  return cbv::ring_fwd_run(&b, L, scratch, static_cast<cudaStream_t>(stream));
}

int cbv_noalloc_read_status(int* status_out, void* stream) {
  if (!status_out) {
    snprintf(g_msg, sizeof g_msg, "status_out is NULL");
    return fail(CBV_ERR_BAD_ARG);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof g_msg, "reading the static scratch's status word: %s", cudaGetErrorString(e));
    return fail(CBV_ERR_CUDA);
  }
  *status_out = v;
  if (v != 0) {
    snprintf(g_msg, sizeof g_msg, "a kernel gave up a wait (code 0x%x)", v);
    return fail(CBV_ERR_TIMEOUT);
  }
  return CBV_OK;
}

}  // extern "C"
