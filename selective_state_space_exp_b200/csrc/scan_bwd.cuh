// scan_bwd.cuh -- pieces of the backward pass shared by its CUDA-core and
// tensor-core forms: the workspace views, the backward's own chunking and the
// state-pass launch.
#pragma once

#include "m3_internal.cuh"

namespace m3 {

struct BwdWs {
  float* G;     // [b][H][nc][N][P] chunk-start states (forward)
  float* sums;  // [b][H][nc][1 + N] chunk factors: exp(Lam_end), (cos, sin) of Phi_end per pair
  float* D;     // [b][H][nc][N][P] D_c, then (CUDA-core form) the adjoint of chunk c's
                // outgoing state
  float* fin;   // [b][H][N][P] final state (forward)
  // tensor-core form only (nullptr otherwise), written by the state pass:
  uint8_t* Gb;  // [b][H][nc + 1] blocks of 16 KB: G_c in bf16 (block nc: the final
                // state), the MMA operand layout (rows n of 128 bytes, the 16-byte
                // chunk index XORed with n mod 8)
  uint8_t* Hb;  // [b][H][nc] blocks: dGhat_c = Rot(-Phi_end) dG_c+1, the same layout
};

// Forward args of the backward's own chunking (chunk Qb, state only).
ScanArgs bwd_fwd_args(const ScanArgs& a, int64_t Qb);
// The workspace views of chunking f (tc: with the tensor-core form's buffers).
BwdWs bwd_carve(const ScanArgs& f, bool tc);
// Workspace bytes of chunking f.
size_t bwd_ws_bytes(const ScanArgs& f, bool tc);
// Zero the gradients that are accumulated with atomic adds.
cudaError_t bwd_zero_outputs(const ScanArgs& a, const BwdArgs& g, cudaStream_t st);
// Step 2, both state passes, over chunking f (S_c, D_c and the chunk factors
// written by step 1); with w.Gb set, the tensor-core form's outputs.
cudaError_t bwd_pass_launch(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st);

// Tensor-core steps 1 and 3 (bf16 io, N = 128, P = 64, chunks of 64 rows).
constexpr int64_t kBwdTcRows = 64;
bool bwd_tc_shape(const ScanArgs& a);
cudaError_t bwd_tc_sums_launch(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st);
cudaError_t bwd_tc_chunk_launch(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st);

}  // namespace m3
