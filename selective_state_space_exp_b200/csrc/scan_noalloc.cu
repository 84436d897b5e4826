// scan_noalloc.cu -- m3_scan_fwd_noalloc: the prefill scan with its scratch
// memory in a fixed, library-owned device array, for callers that cannot
// allocate device memory (no cudaMalloc, no allocator of their own).
//
// The scratch is a file-scope static __device__ array of
// M3_NOALLOC_SCRATCH_BYTES.  Every GPU that loads this library holds it until
// the process exits.  Host code cannot use the array's name as a device
// address (on the host it is only a stand-in symbol), so the first call on
// each device looks up the real address with cudaGetSymbolAddress while that
// device is current, caches it with the identity of the device's context, and
// every call hands that address to the scan as its workspace.  A new context
// on the device (after a cudaDeviceReset) triggers a fresh lookup, since the
// reloaded module may put the array elsewhere.
//
// All calls on a device share the one array.  The scan writes every scratch
// element before it reads it (chunk states and chunk summaries), so nothing
// left by an earlier call is read and nothing has to be cleared.  Two calls
// whose kernels overlap on the GPU (different streams, or different host
// threads, without ordering between them) race on the array and corrupt each
// other's results: order them on one stream.
#include <mutex>

#include "m3_internal.cuh"

namespace m3 {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[M3_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device and context).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return M3_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return M3_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the lookup made a context current if none was
  }
  *out = g_scratch_addr[dev];
  return M3_OK;
}

}  // namespace
}  // namespace m3

extern "C" M3_API int m3_scan_fwd_noalloc(const m3_shape* s, const void* x, const float* dt,
                                          const float* A, const float* lam,
                                          const float* theta, const void* B, const void* C,
                                          const float* h0, const void* B_prev,
                                          const void* x_prev, void* y, float* final_state,
                                          m3_stream_t stream) {
  size_t need = 0;  // (m3_scan_fwd below opens this call's NVTX range)
  const int st = m3_scan_workspace_size(s, &need);
  if (st != M3_OK) return st;
  if (need > (size_t)M3_NOALLOC_SCRATCH_BYTES) return M3_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (m3::scratch_address(&scratch) != M3_OK) return M3_ERR_CUDA;
  return m3_scan_fwd(s, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, y, final_state, scratch,
                     (size_t)M3_NOALLOC_SCRATCH_BYTES, stream);
}
