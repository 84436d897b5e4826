// seqpar.cu -- the pieces a sequence split across ranks (context parallel)
// needs besides the scan itself.
//
// Unrolling the recurrence over a segment of tokens (the exponential-
// trapezoidal step, PaperWeekly page section 2.2, with the rotation of
// section 2.1) gives, per (batch, head),
//   h_end = exp(Lam_seg) Rot(Phi_seg) h_start + T,
// where Lam_seg = sum_t dt_t A_t, Phi_seg,k = sum_t dt_t theta_{t,k} and T is
// the segment's end state from a zero start (its first token's left
// endpoint, B_prev x_prev, included).  Each rank computes T for its segment
// (m3_scan_state with h0 = NULL) and the totals (segment_totals_kernel); after
// one exchange, each rank folds the earlier segments' summaries into its
// incoming state (state_fold_kernel) and scans its segment from it.
#include "m3_internal.cuh"

namespace m3 {
namespace {

// Lam_seg[b][H] and Phi_seg[b][H][N/2], accumulated in fp64 over the segment;
// the angle is stored reduced to [-pi, pi] (it only enters through its sine and
// cosine, and a long segment's total reaches thousands of radians, where an
// fp32 value would have lost its fraction).
// Block (b, h); thread k < K sums pair k's angles, thread K the log-decay.
__global__ void segment_totals_kernel(const float* dt, const float* A, const float* theta,
                                      int64_t L, int64_t H, int64_t tgroups, int K,
                                      float* lam_tot, float* phi_tot) {
  const int64_t b = blockIdx.y, h = blockIdx.x;
  const int64_t tg = h / (H / tgroups);
  for (int k = threadIdx.x; k <= K; k += blockDim.x) {
    double acc = 0.0;
    if (k < K) {
      for (int64_t t = 0; t < L; ++t)
        acc += (double)dt[(b * L + t) * H + h] * (double)theta[((b * L + t) * tgroups + tg) * K + k];
      phi_tot[(b * H + h) * K + k] = (float)remainder(acc, 6.283185307179586);
    } else {
      for (int64_t t = 0; t < L; ++t)
        acc += (double)dt[(b * L + t) * H + h] * (double)A[(b * L + t) * H + h];
      lam_tot[b * H + h] = (float)acc;
    }
  }
}

// out = fold of nseg summaries from h0: h <- Rot(Phi_s) exp(Lam_s) h + T_s.
// Thread (b, h, k, p) holds the pair (2k, 2k+1) of column p.
__global__ void state_fold_kernel(int64_t nseg, int64_t batch, int64_t H, int N, int P,
                                  const float* h0, const float* T, const float* lam_tot,
                                  const float* phi_tot, float* out) {
  const int K = N / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per_chain = (int64_t)K * P;
  if (idx >= batch * H * per_chain) return;
  const int64_t bh = idx / per_chain;
  const int k = (int)((idx % per_chain) / P), p = (int)(idx % P);
  const int64_t i0 = (bh * N + 2 * k) * P + p, i1 = i0 + P;
  float g0 = h0 ? h0[i0] : 0.f, g1 = h0 ? h0[i1] : 0.f;
  const int64_t chains = batch * H;
  for (int64_t s = 0; s < nseg; ++s) {
    const float e = expf(lam_tot[s * chains + bh]);
    float sn, cs;
    sincosf(phi_tot[(s * chains + bh) * K + k], &sn, &cs);
    const float u0 = e * g0, u1 = e * g1;
    const float* Ts = T + s * chains * (int64_t)N * P;
    g0 = cs * u0 - sn * u1 + Ts[i0];
    g1 = sn * u0 + cs * u1 + Ts[i1];
  }
  out[i0] = g0;
  out[i1] = g1;
}

}  // namespace

cudaError_t segment_totals_launch(const ScanArgs& a, float* lam_tot, float* phi_tot,
                                  cudaStream_t s) {
  const int K = (int)(a.N / 2);
  dim3 grid((unsigned)a.nheads, (unsigned)a.batch);
  const int threads = K + 1 < 256 ? ((K + 1 + 31) / 32) * 32 : 256;
  segment_totals_kernel<<<grid, threads, 0, s>>>(a.dt, a.A, a.theta, a.seqlen, a.nheads,
                                                 a.tgroups, K, lam_tot, phi_tot);
  return cudaGetLastError();
}

cudaError_t state_fold_launch(int64_t nseg, int64_t batch, int64_t nheads, int64_t N, int64_t P,
                              const float* h0, const float* T, const float* lam_tot,
                              const float* phi_tot, float* out, cudaStream_t s) {
  const int64_t n = batch * nheads * (N / 2) * P;
  if (n == 0) return cudaSuccess;
  state_fold_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      nseg, batch, nheads, (int)N, (int)P, h0, T, lam_tot, phi_tot, out);
  return cudaGetLastError();
}

}  // namespace m3
