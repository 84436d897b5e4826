// m3_api.cu -- the C ABI declared in include/m3.h: argument checks, workspace
// sizing, dispatch to the kernels, and the device-side error word.
#include <cuda.h>  // CUcontext (the driver calls are reached through the runtime)
#include <nvtx3/nvToolsExt.h>  // header-only; ranges cost a pointer check with no tool attached

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "m3_internal.cuh"

namespace m3 {

// An NVTX range named after the C-ABI call for the duration of the call (host
// side: argument checks and launches), so a timeline tool attached to the
// process shows each call around its kernels.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// First device-side error raised by a kernel (M3_ERR_*), 0 if none.
__device__ int g_device_status = 0;

unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c ||
      get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int check_common(const m3_shape* s) {
  if (!s) return M3_ERR_INVALID_ARGUMENT;
  if (s->batch < 1 || s->nheads < 1 || s->ngroups < 1 || s->headdim < 1 ||
      s->dstate < 2 || s->rank < 1 || s->seqlen < 0 || s->chunk < 1)
    return M3_ERR_INVALID_ARGUMENT;
  if (s->dstate % 2 != 0 || s->nheads % s->ngroups != 0) return M3_ERR_INVALID_ARGUMENT;
  if (s->io_dtype != M3_F32 && s->io_dtype != M3_BF16) return M3_ERR_INVALID_ARGUMENT;
  if ((s->flags & ~(M3_FLAG_SIMT | M3_FLAG_TEST_TIMEOUT | M3_FLAG_THETA_PER_HEAD |
                    M3_FLAG_DY_F32)) != 0)
    return M3_ERR_INVALID_ARGUMENT;
  // supported set
  if (!is_pow2(s->dstate) || s->dstate < 16 || s->dstate > 256) return M3_ERR_UNSUPPORTED;
  if (!is_pow2(s->headdim) || s->headdim < 16 || s->headdim > 128) return M3_ERR_UNSUPPORTED;
  if (s->dstate * s->headdim > 16384) return M3_ERR_UNSUPPORTED;
  if (!(s->rank == 1 || s->rank == 2 || s->rank == 4 || s->rank == 8)) return M3_ERR_UNSUPPORTED;
  if (!(s->chunk == 16 || s->chunk == 32 || s->chunk == 64)) return M3_ERR_UNSUPPORTED;
  if (s->batch > 65535 || s->nheads > 65535) return M3_ERR_UNSUPPORTED;
  if (s->batch * s->nheads > (int64_t)1 << 30) return M3_ERR_UNSUPPORTED;
  return M3_OK;
}

ScanArgs make_scan_args(const m3_shape* s) {
  ScanArgs a;
  memset(&a, 0, sizeof(a));
  a.batch = s->batch;
  a.seqlen = s->seqlen;
  a.nheads = s->nheads;
  a.ngroups = s->ngroups;
  a.P = s->headdim;
  a.N = s->dstate;
  a.R = s->rank;
  a.Q = s->chunk;
  a.nchunks = (s->seqlen + s->chunk - 1) / s->chunk;
  a.bf16 = s->io_dtype == M3_BF16;
  a.test_timeout = (s->flags & M3_FLAG_TEST_TIMEOUT) != 0;
  a.tgroups = (s->flags & M3_FLAG_THETA_PER_HEAD) ? s->nheads : s->ngroups;
  return a;
}

int status_word(int** out) {
  // Device address of g_device_status, looked up once per device and context.
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static int* cache[kMaxDevices] = {};
  static unsigned long long cache_ctx[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return M3_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (!cache[dev] || ctx == 0 || ctx != cache_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return M3_ERR_CUDA;
    cache[dev] = static_cast<int*>(p);
    cache_ctx[dev] = current_context_id();  // the lookup made a context current if none was
  }
  *out = cache[dev];
  return M3_OK;
}

bool use_tc(const m3_shape* s, const ScanArgs& a) {
  return (s->flags & M3_FLAG_SIMT) == 0 && tc_scan_supported(a);
}

size_t scan_workspace(const m3_shape* s, const ScanArgs& a) {
  return use_tc(s, a) ? tc_scan_workspace(a) : simt_scan_workspace(a);
}

}  // namespace
}  // namespace m3

using namespace m3;

extern "C" {

M3_API const char* m3_version(void) { return "m3 0.1.0 (sm_100a)"; }

M3_API const char* m3_status_string(int st) {
  switch (st) {
    case M3_OK: return "M3_OK";
    case M3_ERR_INVALID_ARGUMENT: return "M3_ERR_INVALID_ARGUMENT";
    case M3_ERR_UNSUPPORTED: return "M3_ERR_UNSUPPORTED";
    case M3_ERR_ALIGNMENT: return "M3_ERR_ALIGNMENT";
    case M3_ERR_WORKSPACE: return "M3_ERR_WORKSPACE";
    case M3_ERR_CUDA: return "M3_ERR_CUDA";
    case M3_ERR_TIMEOUT: return "M3_ERR_TIMEOUT";
    case M3_ERR_BOUNDS: return "M3_ERR_BOUNDS";
    default: return "M3_ERR_UNKNOWN";
  }
}

M3_API int m3_check_shape(const m3_shape* s) { return check_common(s); }

namespace {

int workspace_query(const m3_shape* s, size_t* bytes, bool state_only) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  if (!bytes) return M3_ERR_INVALID_ARGUMENT;
  if (s->seqlen == 0) {
    *bytes = 0;
    return M3_OK;
  }
  ScanArgs a = make_scan_args(s);
  a.state_only = state_only;
  *bytes = scan_workspace(s, a);
  return M3_OK;
}

}  // namespace

M3_API int m3_scan_workspace_size(const m3_shape* s, size_t* bytes) {
  return workspace_query(s, bytes, false);
}

M3_API size_t m3_scan_workspace_bytes(const m3_shape* s) {
  size_t n = 0;
  return workspace_query(s, &n, false) == M3_OK ? n : SIZE_MAX;
}

M3_API int m3_scan_state_workspace_size(const m3_shape* s, size_t* bytes) {
  return workspace_query(s, bytes, true);
}

extern "C++" {
namespace m3 {
// Kernel launches of one tensor-core scan call (scan_tc.cu).
int tc_scan_launches(const ScanArgs& a);
}  // namespace m3
}

M3_API int m3_scan_plan(const m3_shape* s, int* tensor_core, int64_t* segments, int* launches) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  ScanArgs a = make_scan_args(s);
  const bool tc = use_tc(s, a);
  const int64_t nseg = (tc && s->seqlen > 0) ? tc_scan_segments(a) : 1;
  if (tensor_core) *tensor_core = tc ? 1 : 0;
  if (segments) *segments = nseg;
  if (launches) *launches = s->seqlen == 0 ? 0 : (tc ? tc_scan_launches(a) : 3);
  return M3_OK;
}

namespace {

// m3_scan_fwd and m3_scan_state: state_only skips y (and needs final_state).
int scan_call(const m3_shape* s, const void* x, const float* dt, const float* A,
              const float* lam, const float* theta, const void* B, const void* C,
              const float* h0, const void* B_prev, const void* x_prev, void* y,
              float* final_state, void* workspace, size_t workspace_bytes, m3_stream_t stream,
              bool state_only, const int32_t* cu_seqlens = nullptr, int64_t total_tokens = 0) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen && (total_tokens < 0 || !aligned(cu_seqlens, 4))) return M3_ERR_INVALID_ARGUMENT;
  // tokens of the call: none when L == 0 (or a packed batch holds none)
  const bool empty = s->seqlen == 0 || (varlen && total_tokens == 0);
  if ((B_prev == nullptr) != (x_prev == nullptr)) return M3_ERR_INVALID_ARGUMENT;
  if (state_only && !final_state) return M3_ERR_INVALID_ARGUMENT;
  const bool bf16 = s->io_dtype == M3_BF16;
  if (bf16 && s->headdim % 8 != 0) return M3_ERR_UNSUPPORTED;
  if (!empty && (!x || !dt || !A || !lam || !theta || !B || !C || (!y && !state_only)))
    return M3_ERR_INVALID_ARGUMENT;
  const void* v16[] = {x, B, C, state_only ? nullptr : y, h0, final_state, B_prev, x_prev, theta};
  for (const void* p : v16)
    if (p && !aligned(p, 16)) return M3_ERR_ALIGNMENT;
  const void* v4[] = {dt, A, lam};
  for (const void* p : v4)
    if (p && !aligned(p, 4)) return M3_ERR_ALIGNMENT;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  if (empty) {  // no token: the state is h0 (the left term waits for a token)
    if (!final_state) return M3_OK;
    const size_t nb = sizeof(float) * s->batch * s->nheads * s->dstate * s->headdim;
    cudaError_t e = h0 ? cudaMemcpyAsync(final_state, h0, nb, cudaMemcpyDeviceToDevice, cs)
                       : cudaMemsetAsync(final_state, 0, nb, cs);
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
  }

  ScanArgs a = make_scan_args(s);
  a.state_only = state_only;
  const size_t need = scan_workspace(s, a);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
    return M3_ERR_WORKSPACE;
  a.x = x; a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.B = B; a.C = C;
  a.h0 = h0; a.B_prev = B_prev; a.x_prev = x_prev; a.y = state_only ? nullptr : y;
  a.final_state = final_state;
  a.ws = static_cast<char*>(workspace);
  a.ws_bytes = workspace_bytes;
  a.cu_seqlens = cu_seqlens;
  a.total_tokens = varlen ? total_tokens : s->batch * s->seqlen;
  if (status_word(&a.status) != M3_OK) return M3_ERR_CUDA;
  cudaError_t e = use_tc(s, a) ? tc_scan_launch(a, cs) : simt_scan_launch(a, cs);
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // namespace

M3_API int m3_scan_fwd(const m3_shape* s, const void* x, const float* dt, const float* A,
                       const float* lam, const float* theta, const void* B, const void* C,
                       const float* h0, const void* B_prev, const void* x_prev, void* y,
                       float* final_state, void* workspace, size_t workspace_bytes,
                       m3_stream_t stream) {
  m3::CallRange range_("m3_scan_fwd");
  return scan_call(s, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, y, final_state, workspace,
                   workspace_bytes, stream, false);
}

M3_API int m3_scan_fwd_varlen(const m3_shape* s, const int32_t* cu_seqlens,
                              int64_t total_tokens, const void* x, const float* dt,
                              const float* A, const float* lam, const float* theta,
                              const void* B, const void* C, const float* h0,
                              const void* B_prev, const void* x_prev, void* y,
                              float* final_state, void* workspace, size_t workspace_bytes,
                              m3_stream_t stream) {
  m3::CallRange range_("m3_scan_fwd_varlen");
  if (!cu_seqlens) return M3_ERR_INVALID_ARGUMENT;
  return scan_call(s, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, y, final_state, workspace,
                   workspace_bytes, stream, false, cu_seqlens, total_tokens);
}

M3_API int m3_scan_bwd_workspace_size(const m3_shape* s, size_t* bytes) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  if (!bytes) return M3_ERR_INVALID_ARGUMENT;
  ScanArgs a = make_scan_args(s);
  if (!bwd_supported(a)) return M3_ERR_UNSUPPORTED;
  *bytes = s->seqlen == 0 ? 0 : bwd_workspace(a, (s->flags & M3_FLAG_SIMT) == 0);
  return M3_OK;
}

namespace {

int bwd_call(const m3_shape* s, const int32_t* cu_seqlens, int64_t total_tokens, const void* x,
             const float* dt, const float* A, const float* lam, const float* theta,
             const void* B, const void* C, const float* h0, const void* B_prev,
             const void* x_prev, const void* dy, const float* d_final, float* dx, float* ddt,
             float* dA, float* dlam, float* dtheta, float* dB, float* dC, float* dh0,
             float* dB_prev, float* dx_prev, void* workspace, size_t workspace_bytes,
             m3_stream_t stream) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen && (total_tokens < 0 || !aligned(cu_seqlens, 4))) return M3_ERR_INVALID_ARGUMENT;
  if ((B_prev == nullptr) != (x_prev == nullptr)) return M3_ERR_INVALID_ARGUMENT;
  if ((dB_prev == nullptr) != (dx_prev == nullptr)) return M3_ERR_INVALID_ARGUMENT;
  const bool bf16 = s->io_dtype == M3_BF16;
  if (bf16 && s->headdim % 8 != 0) return M3_ERR_UNSUPPORTED;
  ScanArgs a = make_scan_args(s);
  if (!bwd_supported(a)) return M3_ERR_UNSUPPORTED;
  const bool empty = s->seqlen == 0 || (varlen && total_tokens == 0);
  if (!empty && (!x || !dt || !A || !lam || !theta || !B || !C || !dy || !dx || !ddt ||
                 !dA || !dlam || !dtheta || !dB || !dC))
    return M3_ERR_INVALID_ARGUMENT;
  const void* v16[] = {x, B, C, dy, h0, d_final, B_prev, x_prev, theta, dx, dtheta, dB, dC,
                       dh0, dB_prev, dx_prev};
  for (const void* p : v16)
    if (p && !aligned(p, 16)) return M3_ERR_ALIGNMENT;
  const void* v4[] = {dt, A, lam, ddt, dA, dlam};
  for (const void* p : v4)
    if (p && !aligned(p, 4)) return M3_ERR_ALIGNMENT;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const size_t sb = sizeof(float) * s->batch * s->nheads * s->dstate * s->headdim;

  if (empty) {  // no token: the state is h0, so dh0 = d_final; nothing else
    if (dh0) {
      cudaError_t e = d_final ? cudaMemcpyAsync(dh0, d_final, sb, cudaMemcpyDeviceToDevice, cs)
                              : cudaMemsetAsync(dh0, 0, sb, cs);
      if (e != cudaSuccess) return M3_ERR_CUDA;
    }
    if (dB_prev) {
      const size_t nb = sizeof(float) * s->batch * s->ngroups * s->rank * s->dstate;
      const size_t nx = sizeof(float) * s->batch * s->nheads * s->rank * s->headdim;
      if (cudaMemsetAsync(dB_prev, 0, nb, cs) != cudaSuccess ||
          cudaMemsetAsync(dx_prev, 0, nx, cs) != cudaSuccess)
        return M3_ERR_CUDA;
    }
    return M3_OK;
  }
  const bool tc = (s->flags & M3_FLAG_SIMT) == 0;
  const size_t need = bwd_workspace(a, tc);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return M3_ERR_WORKSPACE;
  a.x = x; a.dt = dt; a.A = A; a.lam = lam; a.theta = theta; a.B = B; a.C = C;
  a.h0 = h0; a.B_prev = B_prev; a.x_prev = x_prev;
  a.ws = static_cast<char*>(workspace);
  a.ws_bytes = workspace_bytes;
  a.cu_seqlens = cu_seqlens;
  a.total_tokens = varlen ? total_tokens : s->batch * s->seqlen;
  if (status_word(&a.status) != M3_OK) return M3_ERR_CUDA;
  BwdArgs g;
  g.dy = dy; g.dy_f32 = (s->flags & M3_FLAG_DY_F32) != 0;
  g.d_final = d_final; g.dx = dx; g.ddt = ddt; g.dA = dA; g.dlam = dlam;
  g.dtheta = dtheta; g.dB = dB; g.dC = dC; g.dh0 = dh0;
  g.dB_prev = B_prev ? dB_prev : nullptr;
  g.dx_prev = B_prev ? dx_prev : nullptr;
  if (dB_prev && !B_prev) {  // no previous token: its gradients are zero
    const size_t nb = sizeof(float) * s->batch * s->ngroups * s->rank * s->dstate;
    const size_t nx = sizeof(float) * s->batch * s->nheads * s->rank * s->headdim;
    if (cudaMemsetAsync(dB_prev, 0, nb, cs) != cudaSuccess ||
        cudaMemsetAsync(dx_prev, 0, nx, cs) != cudaSuccess)
      return M3_ERR_CUDA;
  }
  cudaError_t e = bwd_launch(a, g, tc, cs);
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // namespace

M3_API int m3_scan_bwd(const m3_shape* s, const void* x, const float* dt, const float* A,
                       const float* lam, const float* theta, const void* B, const void* C,
                       const float* h0, const void* B_prev, const void* x_prev, const void* dy,
                       const float* d_final, float* dx, float* ddt, float* dA, float* dlam,
                       float* dtheta, float* dB, float* dC, float* dh0, float* dB_prev,
                       float* dx_prev, void* workspace, size_t workspace_bytes,
                       m3_stream_t stream) {
  m3::CallRange range_("m3_scan_bwd");
  return bwd_call(s, nullptr, 0, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, dy, d_final,
                  dx, ddt, dA, dlam, dtheta, dB, dC, dh0, dB_prev, dx_prev, workspace,
                  workspace_bytes, stream);
}

M3_API int m3_scan_bwd_varlen(const m3_shape* s, const int32_t* cu_seqlens, int64_t total_tokens,
                              const void* x, const float* dt, const float* A, const float* lam,
                              const float* theta, const void* B, const void* C, const float* h0,
                              const void* B_prev, const void* x_prev, const void* dy,
                              const float* d_final, float* dx, float* ddt, float* dA,
                              float* dlam, float* dtheta, float* dB, float* dC, float* dh0,
                              float* dB_prev, float* dx_prev, void* workspace,
                              size_t workspace_bytes, m3_stream_t stream) {
  m3::CallRange range_("m3_scan_bwd_varlen");
  if (!cu_seqlens) return M3_ERR_INVALID_ARGUMENT;
  return bwd_call(s, cu_seqlens, total_tokens, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev,
                  dy, d_final, dx, ddt, dA, dlam, dtheta, dB, dC, dh0, dB_prev, dx_prev,
                  workspace, workspace_bytes, stream);
}

M3_API int m3_bc_prep(const m3_shape* s, const void* B_raw, const void* C_raw,
                      const float* B_weight, const float* B_bias, const float* C_weight,
                      const float* C_bias, float eps, void* B, void* C, m3_stream_t stream) {
  m3::CallRange range_("m3_bc_prep");
  int st = check_common(s);
  if (st != M3_OK) return st;
  if ((B_raw == nullptr) != (B == nullptr) || (C_raw == nullptr) != (C == nullptr))
    return M3_ERR_INVALID_ARGUMENT;
  if (!(eps >= 0.f) || !(eps < 1e30f)) return M3_ERR_INVALID_ARGUMENT;
  const void* v16[] = {B_raw, C_raw, B_weight, B_bias, C_weight, C_bias, B, C};
  for (const void* p : v16)
    if (p && !aligned(p, 16)) return M3_ERR_ALIGNMENT;
  // an output may be its own input (in place); other overlaps are not allowed
  const size_t esz = s->io_dtype == M3_BF16 ? 2 : 4;
  const int64_t rows = s->batch * s->seqlen * s->ngroups * s->rank;
  const size_t nb = esz * (size_t)rows * (size_t)s->dstate;
  auto overlap = [&](const void* a, const void* b) {
    const char* x = static_cast<const char*>(a);
    const char* y = static_cast<const char*>(b);
    return a && b && x != y && x < y + nb && y < x + nb;
  };
  if (overlap(B, B_raw) || overlap(C, C_raw) || overlap(B, C) || overlap(B, C_raw) ||
      overlap(C, B_raw) || (B && B == C))
    return M3_ERR_INVALID_ARGUMENT;
  cudaError_t e = bc_prep_launch(s->batch * s->seqlen, s->dstate, s->ngroups * s->rank,
                                 s->io_dtype == M3_BF16, B_raw, C_raw, B_weight, B_bias, C_weight,
                                 C_bias, eps, B, C, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_linear(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                     const float* bias, void* out, int32_t out_dtype, m3_stream_t stream) {
  m3::CallRange range_("m3_linear");
  if (out_dtype != M3_BF16 && out_dtype != M3_F32) return M3_ERR_INVALID_ARGUMENT;
  const bool f32 = out_dtype == M3_F32;
  if (M < 0 || N < 1 || K < 8) return M3_ERR_INVALID_ARGUMENT;
  if (K % 8 != 0 || N % (f32 ? 4 : 8) != 0) return M3_ERR_UNSUPPORTED;
  if (M >= ((int64_t)1 << 31) - 256 || N >= ((int64_t)1 << 31) - 256) return M3_ERR_UNSUPPORTED;
  if (M == 0) return M3_OK;
  if (!A || !W || !out) return M3_ERR_INVALID_ARGUMENT;
  if (!aligned(A, 16) || !aligned(W, 16) || !aligned(out, 16) || (bias && !aligned(bias, 4)))
    return M3_ERR_ALIGNMENT;
  const size_t nout = (size_t)M * (size_t)N * (f32 ? 4 : 2);
  auto overlaps = [&](const void* p, size_t n) {
    const char* c = static_cast<const char*>(p);
    const char* o = static_cast<const char*>(out);
    return p && c < o + nout && o < c + n;
  };
  if (overlaps(A, (size_t)M * K * 2) || overlaps(W, (size_t)N * K * 2) ||
      overlaps(bias, (size_t)N * 4))
    return M3_ERR_INVALID_ARGUMENT;
  int* status = nullptr;
  if (status_word(&status) != M3_OK) return M3_ERR_CUDA;
  cudaError_t e = gemm_launch(M, N, K, A, W, bias, out, f32, status,
                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

namespace {
int mimo_check(const m3_shape* s, const void* in, const float* w, const void* extra,
               const void* out) {
  int st = check_common(s);
  if (st != M3_OK) return st;
  const bool bf16 = s->io_dtype == M3_BF16;
  if (s->headdim % (bf16 ? 8 : 4) != 0) return M3_ERR_UNSUPPORTED;
  if (s->batch * s->seqlen == 0) return M3_OK;
  if (!in || !w || !out) return M3_ERR_INVALID_ARGUMENT;
  if (!aligned(in, 16) || !aligned(out, 16) || (extra && !aligned(extra, 16)) || !aligned(w, 16))
    return M3_ERR_ALIGNMENT;
  return M3_OK;
}
}  // namespace

M3_API int m3_mimo_up(const m3_shape* s, const void* x, const float* w_up, void* X,
                      m3_stream_t stream) {
  m3::CallRange range_("m3_mimo_up");
  int st = mimo_check(s, x, w_up, nullptr, X);
  if (st != M3_OK || s->batch * s->seqlen == 0) return st;
  const size_t es = s->io_dtype == M3_BF16 ? 2 : 4;
  const int64_t T = s->batch * s->seqlen;
  const char* xi = static_cast<const char*>(x);
  const char* xo = static_cast<const char*>(X);
  const size_t nin = es * T * s->nheads * s->headdim, nout = nin * s->rank;
  if (xi < xo + nout && xo < xi + nin) return M3_ERR_INVALID_ARGUMENT;  // no overlap
  cudaError_t e = mimo_up_launch(T, s->nheads, s->rank, s->headdim, s->io_dtype == M3_BF16, x,
                                 w_up, X, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_mimo_down_gate(const m3_shape* s, const void* Y, const float* w_down,
                             const void* z, void* out, m3_stream_t stream) {
  m3::CallRange range_("m3_mimo_down_gate");
  int st = mimo_check(s, Y, w_down, z, out);
  if (st != M3_OK || s->batch * s->seqlen == 0) return st;
  const size_t es = s->io_dtype == M3_BF16 ? 2 : 4;
  const int64_t T = s->batch * s->seqlen;
  const size_t nout = es * T * s->nheads * s->headdim, nY = nout * s->rank;
  auto overlaps = [&](const void* p, size_t n) {
    const char* c = static_cast<const char*>(p);
    const char* o = static_cast<const char*>(out);
    return p && c < o + nout && o < c + n;
  };
  if (overlaps(Y, nY) || overlaps(z, nout)) return M3_ERR_INVALID_ARGUMENT;
  cudaError_t e = mimo_down_gate_launch(T, s->nheads, s->rank, s->headdim,
                                        s->io_dtype == M3_BF16, Y, w_down, z, out,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_scan_state(const m3_shape* s, const void* x, const float* dt, const float* A,
                         const float* lam, const float* theta, const void* B, const void* C,
                         const float* h0, const void* B_prev, const void* x_prev,
                         float* final_state, void* workspace, size_t workspace_bytes,
                         m3_stream_t stream) {
  m3::CallRange range_("m3_scan_state");
  return scan_call(s, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, nullptr, final_state,
                   workspace, workspace_bytes, stream, true);
}

M3_API int m3_segment_totals(const m3_shape* s, const float* dt, const float* A,
                             const float* theta, float* lam_tot, float* phi_tot,
                             m3_stream_t stream) {
  m3::CallRange range_("m3_segment_totals");
  int st = check_common(s);
  if (st != M3_OK) return st;
  if (!lam_tot || !phi_tot) return M3_ERR_INVALID_ARGUMENT;
  if (s->seqlen > 0 && (!dt || !A || !theta)) return M3_ERR_INVALID_ARGUMENT;
  const void* v4[] = {dt, A, theta, lam_tot, phi_tot};
  for (const void* p : v4)
    if (p && !aligned(p, 4)) return M3_ERR_ALIGNMENT;
  ScanArgs a = make_scan_args(s);
  a.dt = dt; a.A = A; a.theta = theta;
  cudaError_t e = segment_totals_launch(a, lam_tot, phi_tot, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_state_fold(const m3_shape* s, int64_t nseg, const float* h0, const float* T,
                         const float* lam_tot, const float* phi_tot, float* out,
                         m3_stream_t stream) {
  m3::CallRange range_("m3_state_fold");
  int st = check_common(s);
  if (st != M3_OK) return st;
  if (nseg < 0 || !out || (nseg > 0 && (!T || !lam_tot || !phi_tot))) return M3_ERR_INVALID_ARGUMENT;
  const void* v16[] = {h0, T, out};
  for (const void* p : v16)
    if (p && !aligned(p, 16)) return M3_ERR_ALIGNMENT;
  const void* v4[] = {lam_tot, phi_tot};
  for (const void* p : v4)
    if (p && !aligned(p, 4)) return M3_ERR_ALIGNMENT;
  // out must not overlap the inputs
  const size_t sb = sizeof(float) * s->batch * s->nheads * s->dstate * s->headdim;
  const char* o0 = reinterpret_cast<const char*>(out);
  auto overlaps = [&](const void* p, size_t n) {
    const char* c = reinterpret_cast<const char*>(p);
    return p && c < o0 + sb && o0 < c + n;
  };
  if (overlaps(h0, sb) || overlaps(T, sb * (size_t)nseg)) return M3_ERR_INVALID_ARGUMENT;
  cudaError_t e = state_fold_launch(nseg, s->batch, s->nheads, s->dstate, s->headdim, h0, T,
                                    lam_tot, phi_tot, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_decode_step(const m3_shape* s, const float* state_in, float* state_out,
                          const void* x_t, const float* dt_t, const float* A_t,
                          const float* lam_t, const float* theta_t, const void* B_t,
                          const void* C_t, const void* B_prev, const void* x_prev, void* y_t,
                          m3_stream_t stream) {
  m3::CallRange range_("m3_decode_step");
  int st = check_common(s);
  if (st != M3_OK) return st;
  if ((B_prev == nullptr) != (x_prev == nullptr)) return M3_ERR_INVALID_ARGUMENT;
  if (!state_in || !state_out || !x_t || !dt_t || !A_t || !lam_t || !theta_t || !B_t || !C_t ||
      !y_t)
    return M3_ERR_INVALID_ARGUMENT;
  const bool bf16 = s->io_dtype == M3_BF16;
  if (bf16 && s->headdim % 8 != 0) return M3_ERR_UNSUPPORTED;
  const void* v16[] = {state_in, state_out, x_t, B_t, C_t, y_t, B_prev, x_prev};
  for (const void* p : v16)
    if (p && !aligned(p, 16)) return M3_ERR_ALIGNMENT;
  const void* v4[] = {dt_t, A_t, lam_t, theta_t};
  for (const void* p : v4)
    if (!aligned(p, 4)) return M3_ERR_ALIGNMENT;
  // in-place is allowed; a partial overlap is not
  const size_t sb = sizeof(float) * s->batch * s->nheads * s->dstate * s->headdim;
  const char* i0 = reinterpret_cast<const char*>(state_in);
  const char* o0 = reinterpret_cast<const char*>(state_out);
  if (i0 != o0 && i0 < o0 + sb && o0 < i0 + sb) return M3_ERR_INVALID_ARGUMENT;

  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.batch = s->batch; a.nheads = s->nheads; a.ngroups = s->ngroups;
  a.P = s->headdim; a.N = s->dstate; a.R = s->rank; a.bf16 = bf16;
  a.tgroups = (s->flags & M3_FLAG_THETA_PER_HEAD) ? s->nheads : s->ngroups;
  a.state_in = state_in; a.state_out = state_out; a.x = x_t; a.dt = dt_t; a.A = A_t;
  a.lam = lam_t; a.theta = theta_t; a.B = B_t; a.C = C_t; a.B_prev = B_prev;
  a.x_prev = x_prev; a.y = y_t;
  if (status_word(&a.status) != M3_OK) return M3_ERR_CUDA;
  cudaError_t e = decode_launch(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

M3_API int m3_stream_status(m3_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return M3_ERR_CUDA;
  int* p = nullptr;
  if (status_word(&p) != M3_OK) return M3_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return M3_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return M3_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
