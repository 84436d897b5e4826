// m3_internal.cuh -- internal declarations shared by the library's .cu files.
// Not part of the public ABI (include/m3.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/m3.h"

namespace m3 {

// Bounds-checked builds (compiled with -DM3_DEBUG_BOUNDS; `_build.build(debug=True)`
// writes lib/libm3_debug.so): the kernels' global writes, and their reads of
// tensors and the workspace at computed indices, first test the index against
// the extent of the tensor it addresses (elements, from the call's shape);
// an index outside records M3_ERR_BOUNDS in the device status word and the
// access is skipped.  In normal builds the test is the constant true.
#ifdef M3_DEBUG_BOUNDS
static __device__ __noinline__ void bounds_fail(int* status) {
  if (status) atomicCAS(status, 0, (int)M3_ERR_BOUNDS);
}
#define M3_IN(i, n, st) \
  (((int64_t)(i) >= 0 && (int64_t)(i) < (int64_t)(n)) ? true : (::m3::bounds_fail(st), false))
#else
#define M3_IN(i, n, st) true
#endif

// Element access for the io dtype (fp32 or bf16).
__device__ __forceinline__ float io_load(const void* p, int64_t i, bool bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void io_store(void* p, int64_t i, float v, bool bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[i] = v;
}

// Everything a prefill scan launch needs; pointers are device pointers.
struct ScanArgs {
  int64_t batch, seqlen, nheads, ngroups, P, N, R, Q, nchunks;
  bool bf16;
  const void* x;
  const float* dt;
  const float* A;
  const float* lam;
  const float* theta;
  const void* B;
  const void* C;
  const float* h0;
  const void* B_prev;
  const void* x_prev;
  void* y;
  float* final_state;
  char* ws;
  size_t ws_bytes;
  int* status;        // device-side error word
  bool test_timeout;  // M3_FLAG_TEST_TIMEOUT
  int64_t tgroups;    // theta groups: ngroups, or nheads (M3_FLAG_THETA_PER_HEAD)
  bool state_only;    // m3_scan_state: the final state only, no y
  // Packed variable-length batch (m3_scan_fwd_varlen): sequence i is tokens
  // [cu_seqlens[i], cu_seqlens[i+1]) of tensors with total_tokens rows, and
  // seqlen is the longest sequence.  nullptr: batch x seqlen, fixed length.
  const int32_t* cu_seqlens;
  int64_t total_tokens;
};

// Token range of chain b's sequence in the token dimension of its tensors.
struct Chain {
  int64_t base, len;
};

// Sequence b's first token and length.  Packed batches are read from
// cu_seqlens and checked: an offset pair outside [0, total_tokens], a
// decreasing pair or a sequence longer than seqlen records
// M3_ERR_INVALID_ARGUMENT and yields an empty sequence (nothing is read).
__device__ __forceinline__ Chain chain_of(const ScanArgs& a, int64_t b) {
  if (!a.cu_seqlens) return Chain{b * a.seqlen, a.seqlen};
  const int64_t s0 = __ldg(a.cu_seqlens + b), s1 = __ldg(a.cu_seqlens + b + 1);
  if (s0 >= 0 && s1 >= s0 && s1 <= a.total_tokens && s1 - s0 <= a.seqlen) return Chain{s0, s1 - s0};
  if (a.status) atomicCAS(a.status, 0, (int)M3_ERR_INVALID_ARGUMENT);
  return Chain{0, 0};
}

struct DecodeArgs {
  int64_t batch, nheads, ngroups, P, N, R;
  bool bf16;
  const float* state_in;
  float* state_out;
  const void* x;
  const float* dt;
  const float* A;
  const float* lam;
  const float* theta;
  const void* B;
  const void* C;
  const void* B_prev;
  const void* x_prev;
  void* y;
  int* status;  // device status word (timeouts)
  int64_t tgroups;  // theta groups: ngroups, or nheads (M3_FLAG_THETA_PER_HEAD)
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A process-unique identity of the calling thread's current CUDA context
// (0 when there is none yet or the driver cannot say).  Device addresses of
// the library's __device__ variables are cached with it: a device reset
// replaces the context and reloads the module, which may move them.
unsigned long long current_context_id();

// CUDA-core fp32 scan (chunk state -> state passing -> chunk output).
size_t simt_scan_workspace(const ScanArgs& a);
cudaError_t simt_scan_launch(const ScanArgs& a, cudaStream_t s);

// Tensor-core (tcgen05) scan for bf16 io, N = 128, P = 64, Q*R in {64, 128, 256}.
bool tc_scan_supported(const ScanArgs& a);
size_t tc_scan_workspace(const ScanArgs& a);
int64_t tc_scan_segments(const ScanArgs& a);
cudaError_t tc_scan_launch(const ScanArgs& a, cudaStream_t s);

// Where the CUDA-core pass keeps its chunk states (one N x P fp32 matrix per
// chunk-head, [b][H][nc][N][P]; the chunk-start states once state passing has
// run) and its chunk totals ([b][H][nc][1 + N/2]: Lam_end, Phi_end).
void simt_state_views(const ScanArgs& a, float** states, float** sums);

// Backward pass of the scan (CUDA cores, fp32): outputs and incoming adjoints.
struct BwdArgs {
  const void* dy;         // [b][L][H][R][P] io dtype (fp32 when dy_f32)
  bool dy_f32;            // M3_FLAG_DY_F32
  const float* d_final;   // [b][H][N][P] or nullptr
  float* dx;              // [b][L][H][R][P]
  float* ddt;             // [b][L][H]
  float* dA;              // [b][L][H]
  float* dlam;            // [b][L][H]
  float* dtheta;          // [b][L][Gt][N/2]
  float* dB;              // [b][L][G][R][N]
  float* dC;              // [b][L][G][R][N]
  float* dh0;             // [b][H][N][P] or nullptr
  float* dB_prev;         // [b][G][R][N] or nullptr (with dx_prev)
  float* dx_prev;         // [b][H][R][P] or nullptr
};
// tc: the tensor-core form where the shape allows it (bf16 io, N = 128,
// P = 64), else the CUDA-core one; the workspace depends on the form.
size_t bwd_workspace(const ScanArgs& a, bool tc);
bool bwd_supported(const ScanArgs& a);
bool bwd_use_tc(const ScanArgs& a, bool allow);
cudaError_t bwd_launch(const ScanArgs& a, const BwdArgs& g, bool tc, cudaStream_t s);

// B / C prep: QK-norm, per-channel scale and bias over rows of N values,
// tensors [tokens][gr][N] with gr = G * R channel rows.
cudaError_t bc_prep_launch(int64_t tokens, int64_t N, int64_t gr, bool bf16, const void* Braw,
                           const void* Craw, const float* wB, const float* bB, const float* wC,
                           const float* bC, float eps, void* Bo, void* Co, cudaStream_t s);

// Block projections: out = A W^T (+ bias) on the tensor cores; the MIMO up-
// projection; the MIMO down-projection with the output gate.
cudaError_t gemm_launch(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                        const float* bias, void* out, bool out_f32, int* status, cudaStream_t st);
cudaError_t mimo_up_launch(int64_t T, int64_t H, int64_t R, int64_t P, bool bf16, const void* x,
                           const float* w, void* X, cudaStream_t s);
cudaError_t mimo_down_gate_launch(int64_t T, int64_t H, int64_t R, int64_t P, bool bf16,
                                  const void* Y, const float* w, const void* z, void* out,
                                  cudaStream_t s);

// Decode step.
cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t s);

// Sequence split across ranks: segment totals and the fold of summaries.
cudaError_t segment_totals_launch(const ScanArgs& a, float* lam_tot, float* phi_tot,
                                  cudaStream_t s);
cudaError_t state_fold_launch(int64_t nseg, int64_t batch, int64_t nheads, int64_t N, int64_t P,
                              const float* h0, const float* T, const float* lam_tot,
                              const float* phi_tot, float* out, cudaStream_t s);

}  // namespace m3
