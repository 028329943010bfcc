// noalloc.cu -- a forward entry point for callers that cannot allocate
// device memory.
//
// relpos_attn_fwd needs a caller-provided workspace (tables and the Z^Q/Z^K
// projections).  Some callers have no way to obtain one: code that runs
// while another runtime or a memory pool owns the whole device and forbids
// outside allocations, plugins whose enqueue step must not allocate, or
// host code where a blocking cudaMalloc is not acceptable.  For them the
// forward below runs in a fixed scratch array that is part of the library's
// device image, so the call itself never allocates.
//
// The array is kScratchBytes (32 MiB) of global memory on every GPU that
// loads this library, held until the process exits.  It lives in this file's
// own module, which CUDA loads lazily by default: the first call on a device
// (its cudaGetSymbolAddress) loads the module and commits the 32 MiB, and the
// first launch of each kernel loads that kernel's module.  A caller that must
// not allocate later makes one small call on each device early, before a pool
// claims the memory, or runs with CUDA_MODULE_LOADING=EAGER.
#include <mutex>

#include "kernels.cuh"

#define RELPOS_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kScratchBytes = 32u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

// Device address of g_fwd_scratch per device, looked up once (host code
// cannot use the symbol itself: it names a host-side shadow, not device memory).
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess) return (int)e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return 0;
}

}  // namespace

RELPOS_EXPORT int relpos_attn_fwd_noalloc(const relpos_fwd_args* a, relpos_stream_t stream) {
  size_t fwd_bytes = 0, bwd_bytes = 0;
  int st = relpos_workspace_size(a, &fwd_bytes, &bwd_bytes);
  if (st) return st;
  if (fwd_bytes > kScratchBytes) return RELPOS_ERR_WORKSPACE;
  void* ws = nullptr;
  const int e = scratch_for_current_device(&ws);
  if (e) return relpos::cuda_status((cudaError_t)e);
  // the caller's stream only: forks would create events (and a stream on first use)
  relpos::set_single_stream(true);
  const int st2 = relpos_attn_fwd(a, ws, kScratchBytes, stream);
  relpos::set_single_stream(false);
  return st2;
}

RELPOS_EXPORT int relpos_check_noalloc(relpos_stream_t stream, int32_t* device_status) {
  void* ws = nullptr;
  const int e = scratch_for_current_device(&ws);
  if (e) return relpos::cuda_status((cudaError_t)e);
  // the status word sits at the start of the forward's workspace layout
  return relpos_check_workspace(ws, stream, device_status);
}
