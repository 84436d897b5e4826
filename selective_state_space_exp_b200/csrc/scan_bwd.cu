// scan_bwd.cu -- backward pass of the chunked prefill scan (CUDA cores, fp32).
//
// Gradients of a scalar loss through y and the final state, for every input:
// x, dt, A, lam, theta, B, C, h0 and the previous token (B_prev, x_prev).
// The forward is the chunked form of the exponential-trapezoidal recurrence
// with the rotation folded into B and C (PaperWeekly page sections 2.1-2.3):
// per chunk of a (b, h) chain, with chunk-local prefix sums Lam, Phi,
//   y_t   = sum_{s<=t} M_ts (Ct_t . Bt_s) x_s + exp(Lam_t) Ct_t^T G_c
//   G_c+1 = Rot(Phi_end) Ghat,  Ghat = sum_s w_s Bt_s x_s^T + exp(Lam_end) G_c
// with M_ts = exp(Lam_t - Lam_s) (s == t ? gamma_t : delta_s),
// w_s = exp(Lam_end - Lam_s) delta_s, Bt = Rot(-Phi) B, Ct = Rot(-Phi) C and
// G_c the state entering chunk c (its first token's left endpoint included).
//
// Steps (one launch each):
//  1. the forward's chunk-start states G_c and chunk totals (the CUDA-core
//     forward pass run without its output step);
//  2. D_c = sum_t exp(Lam_t) Ct_t dy_t^T, the adjoint y sends to G_c;
//  3. reverse state passing: dG_c = D_c + exp(Lam_end) Rot(-Phi_end) dG_c+1,
//     from dG_nc = d_final; each chunk keeps dG_c+1, the adjoint of its
//     outgoing state; dG_0 gives dh0 and the previous token's gradients;
//  4. per chunk: dCt = (M o dY X^T) Bt + diag(exp Lam) dY G_c^T,
//     dBt = (M o dY X^T)^T Ct + diag(w) X dGhat^T,
//     dX = (M o Ct Bt^T)^T dY + diag(w) Bt dGhat  (dGhat = Rot(-Phi_end) dG_c+1),
//     the gradients of Lam (mask decay, exp(Lam_t) term, w_s), of Phi (the
//     rotations of B, C and of the outgoing state), gamma and delta, and
//     from them, through the prefix sums, dt, A, lam and theta.
// B, C and theta are shared by the heads of a group, and a token's dt and
// lam also receive the next chunk's left-endpoint term, so those gradients
// are accumulated with atomic adds into zeroed outputs.
#include "m3_internal.cuh"
#include "simt_chunk.cuh"

namespace m3 {
namespace {

using simt::chunk_geo;
using simt::chunk_prep;
using simt::Geo;

constexpr int kThreads = 256;
constexpr int kTileRows = 64;  // (token, rank) rows staged per pass of step 2
constexpr int kMaxPairs = 16;  // accumulator pairs per thread in step 4 (N/2 * M <= 4096)
constexpr int kMaxCols = 32;   // dX columns per thread in step 4 (P * M <= 8192)

struct BwdWs {
  float* G;     // [b][H][nc][N][P] chunk-start states (forward)
  float* sums;  // [b][H][nc][1 + K] chunk totals (forward)
  float* D;     // [b][H][nc][N][P] D_c, then the adjoint of chunk c's outgoing state
  float* fin;   // [b][H][N][P] final state (forward)
};

// Forward args of the backward's own chunking (chunk Qb, state only).
ScanArgs fwd_args(const ScanArgs& a, int64_t Qb) {
  ScanArgs f = a;
  f.Q = Qb;
  f.nchunks = (a.seqlen + Qb - 1) / Qb;
  f.state_only = true;
  f.y = nullptr;
  return f;
}

// ---- step 2: D_c -------------------------------------------------------------
template <int R, int OPT>
__global__ void __launch_bounds__(kThreads) bwd_dstate_kernel(const ScanArgs a, const BwdArgs g,
                                                              const BwdWs w) {
  const Geo q = chunk_geo(a, blockIdx.x);
  const int N = (int)a.N, P = (int)a.P, K = N / 2, Q = (int)a.Q;
  extern __shared__ float sm[];
  float* lcum = sm;
  float* gam = lcum + Q;
  float* del = gam + Q;
  float* dts = del + Q;
  float* phi = dts + Q;
  float* Cs = phi + Q * K;          // [kTileRows][N] exp(Lam_t) Rot(-Phi_t) C_t
  float* Ys = Cs + kTileRows * N;   // [kTileRows][P] dy
  chunk_prep(a, q, lcum, gam, del, dts, phi);

  const int p = threadIdx.x % P, n0 = threadIdx.x / P, NS = kThreads / P;
  float acc[OPT];
#pragma unroll
  for (int i = 0; i < OPT; ++i) acc[i] = 0.f;
  const int TS = kTileRows / R;
  for (int s0 = 0; s0 < q.nt; s0 += TS) {
    for (int e = threadIdx.x; e < kTileRows * K; e += blockDim.x) {
      const int ri = e / K, k = e % K, s = s0 + ri / R, r = ri % R;
      float v0 = 0.f, v1 = 0.f;
      if (s < q.nt) {
        const int64_t base = ((q.base + q.t0 + s) * a.ngroups + q.g) * R * N + (int64_t)r * N;
        const float c0 = io_load(a.C, base + 2 * k, a.bf16), c1 = io_load(a.C, base + 2 * k + 1, a.bf16);
        float sn, cs;
        sincosf(phi[s * K + k], &sn, &cs);
        const float el = expf(lcum[s]);
        v0 = el * (cs * c0 + sn * c1);
        v1 = el * (-sn * c0 + cs * c1);
      }
      Cs[ri * N + 2 * k] = v0;
      Cs[ri * N + 2 * k + 1] = v1;
    }
    for (int e = threadIdx.x; e < kTileRows * P; e += blockDim.x) {
      const int ri = e / P, pp = e % P, s = s0 + ri / R, r = ri % R;
      Ys[ri * P + pp] = (s < q.nt) ? io_load(g.dy, ((q.base + q.t0 + s) * a.nheads + q.h) * R * P +
                                                        (int64_t)r * P + pp, a.bf16)
                                   : 0.f;
    }
    __syncthreads();
    const int rows = min(kTileRows, (q.nt - s0) * R);
    for (int ri = 0; ri < rows; ++ri) {
      const float yv = Ys[ri * P + p];
#pragma unroll
      for (int i = 0; i < OPT; ++i) {
        const int n = n0 + i * NS;
        if (n < N) acc[i] = fmaf(Cs[ri * N + n], yv, acc[i]);
      }
    }
    __syncthreads();
  }
  float* D = w.D + ((q.b * a.nheads + q.h) * a.nchunks + q.c) * (int64_t)N * P;
#pragma unroll
  for (int i = 0; i < OPT; ++i) {
    const int n = n0 + i * NS;
    if (n < N) D[n * P + p] = acc[i];
  }
}

// ---- step 3: reverse state passing ------------------------------------------
__global__ void __launch_bounds__(kThreads) bwd_state_pass_kernel(const ScanArgs a, const BwdArgs g,
                                                                  const BwdWs w) {
  const int N = (int)a.N, P = (int)a.P, K = N / 2, R = (int)a.R;
  const int64_t b = blockIdx.z, h = blockIdx.y, H = a.nheads;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= K * P) return;  // K * P is a multiple of 32: whole warps leave
  const int k = idx / P, p = idx % P;
  const int64_t so = (b * H + h) * (int64_t)N * P;
  float d0 = g.d_final ? g.d_final[so + (2 * k) * P + p] : 0.f;
  float d1 = g.d_final ? g.d_final[so + (2 * k + 1) * P + p] : 0.f;
  for (int64_t c = a.nchunks - 1; c >= 0; --c) {
    const int64_t cidx = (b * H + h) * a.nchunks + c;
    float* Dc = w.D + cidx * (int64_t)N * P;
    const float* su = w.sums + cidx * (1 + K);
    const float e0 = Dc[(2 * k) * P + p], e1 = Dc[(2 * k + 1) * P + p];
    Dc[(2 * k) * P + p] = d0;  // adjoint of chunk c's outgoing state
    Dc[(2 * k + 1) * P + p] = d1;
    const float dec = expf(su[0]);
    float sn, cs;
    sincosf(su[1 + k], &sn, &cs);
    const float n0 = fmaf(dec, cs * d0 + sn * d1, e0);  // D_c + exp(Lam) Rot(-Phi) dG
    const float n1 = fmaf(dec, -sn * d0 + cs * d1, e1);
    d0 = n0;
    d1 = n1;
  }
  if (g.dh0) {
    g.dh0[so + (2 * k) * P + p] = d0;
    g.dh0[so + (2 * k + 1) * P + p] = d1;
  }
  if (a.B_prev && a.seqlen > 0) {  // G_0 = h0 + eps_0 B_prev x_prev^T
    const int64_t grp = h / (H / a.ngroups);
    const int64_t t0 = (b * a.seqlen) * H + h;  // token 0 of this chain
    const float lam0 = a.lam[t0], dt0 = a.dt[t0], eps0 = (1.f - lam0) * dt0;
    float part = 0.f;
    for (int r = 0; r < R; ++r) {
      const int64_t bb = ((b * a.ngroups + grp) * R + r) * N;
      const float bp0 = io_load(a.B_prev, bb + 2 * k, a.bf16);
      const float bp1 = io_load(a.B_prev, bb + 2 * k + 1, a.bf16);
      const int64_t xo = ((b * H + h) * R + r) * P + p;
      const float xv = io_load(a.x_prev, xo, a.bf16);
      const float gb = d0 * bp0 + d1 * bp1;
      part = fmaf(gb, xv, part);
      if (g.dB_prev) {
        atomicAdd(g.dB_prev + bb + 2 * k, eps0 * d0 * xv);
        atomicAdd(g.dB_prev + bb + 2 * k + 1, eps0 * d1 * xv);
        atomicAdd(g.dx_prev + xo, eps0 * gb);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if ((threadIdx.x & 31) == 0) {  // d eps_0 = <dG_0, B_prev x_prev^T>
      atomicAdd(g.ddt + t0, (1.f - lam0) * part);
      atomicAdd(g.dlam + t0, -dt0 * part);
    }
  }
}

// ---- step 4: per-chunk gradients ---------------------------------------------
// Shared memory (floats), M = Q * R rows, rows of Ct / Bt padded to N + 1 and
// of X / dY to P + 1 (conflict-free column walks).
struct ChunkSmem {
  int lcum, gam, del, dts, phi, Ct, Bt, X, dY, S, DX, dMt, dPhi, dLam, dgam, ddel, beta, wv, ecs,
      thT, red, total;
  __host__ __device__ ChunkSmem(int M, int N, int P, int Q) {
    const int K = N / 2;
    int o = 0;
    lcum = o; o += Q;
    gam = o; o += Q;
    del = o; o += Q;
    dts = o; o += Q;
    phi = o; o += Q * K;  // chunk_prep's layout ends here
    Ct = o; o += M * (N + 1);
    Bt = o; o += M * (N + 1);
    X = o; o += M * (P + 1);
    dY = o; o += M * (P + 1);
    S = o; o += M * M;
    DX = o; o += M * M;
    dMt = o; o += Q * Q;
    dPhi = o; o += Q * K;
    dLam = o; o += Q;
    dgam = o; o += Q;
    ddel = o; o += Q;
    beta = o; o += Q;
    wv = o; o += Q;
    ecs = o; o += 2 * K;
    thT = o; o += Q;
    red = o; o += 32;
    total = o;
  }
};

template <int R>
__global__ void __launch_bounds__(kThreads) bwd_chunk_kernel(const ScanArgs a, const BwdArgs g,
                                                             const BwdWs w) {
  const Geo q = chunk_geo(a, blockIdx.x);
  const int N = (int)a.N, P = (int)a.P, K = N / 2, Q = (int)a.Q, M = Q * R;
  const int ldn = N + 1, ldp = P + 1;
  const int64_t H = a.nheads;
  const ChunkSmem L(M, N, P, Q);
  extern __shared__ float sm[];
  float* lcum = sm + L.lcum;
  float* gam = sm + L.gam;
  float* del = sm + L.del;
  float* dts = sm + L.dts;
  float* phi = sm + L.phi;
  float* Ct = sm + L.Ct;
  float* Bt = sm + L.Bt;
  float* X = sm + L.X;
  float* dY = sm + L.dY;
  float* S = sm + L.S;
  float* DX = sm + L.DX;
  float* dMt = sm + L.dMt;
  float* dPhi = sm + L.dPhi;
  float* dLam = sm + L.dLam;
  float* dgam = sm + L.dgam;
  float* ddel = sm + L.ddel;
  float* beta = sm + L.beta;
  float* wv = sm + L.wv;
  float* ecs = sm + L.ecs;
  float* thT = sm + L.thT;
  float* red = sm + L.red;
  const int tid = threadIdx.x;
  const int nt = q.nt;
  if (nt <= 0) return;  // uniform over the block

  chunk_prep(a, q, lcum, gam, del, dts, phi);
  const int t1 = nt - 1;
  const float lam_end = lcum[t1];
  for (int i = tid; i < Q; i += kThreads) {
    wv[i] = (i < nt) ? expf(lam_end - lcum[i]) * del[i] : 0.f;
    dLam[i] = 0.f; dgam[i] = 0.f; ddel[i] = 0.f; beta[i] = 0.f; thT[i] = 0.f;
  }
  for (int i = tid; i < Q * K; i += kThreads) dPhi[i] = 0.f;
  for (int k = tid; k < K; k += kThreads) {
    float sn, cs;
    sincosf(phi[t1 * K + k], &sn, &cs);
    ecs[2 * k] = cs;
    ecs[2 * k + 1] = sn;
  }
  // rotated operands and the row data; rows past the chunk end are zero
  for (int e = tid; e < M * K; e += kThreads) {
    const int ri = e / K, k = e % K, s = ri / R, r = ri % R;
    float c0 = 0.f, c1 = 0.f, b0 = 0.f, b1 = 0.f;
    if (s < nt) {
      const int64_t base = ((q.base + q.t0 + s) * a.ngroups + q.g) * R * N + (int64_t)r * N;
      const float cr0 = io_load(a.C, base + 2 * k, a.bf16), cr1 = io_load(a.C, base + 2 * k + 1, a.bf16);
      const float br0 = io_load(a.B, base + 2 * k, a.bf16), br1 = io_load(a.B, base + 2 * k + 1, a.bf16);
      float sn, cs;
      sincosf(phi[s * K + k], &sn, &cs);
      c0 = cs * cr0 + sn * cr1; c1 = -sn * cr0 + cs * cr1;
      b0 = cs * br0 + sn * br1; b1 = -sn * br0 + cs * br1;
    }
    Ct[ri * ldn + 2 * k] = c0; Ct[ri * ldn + 2 * k + 1] = c1;
    Bt[ri * ldn + 2 * k] = b0; Bt[ri * ldn + 2 * k + 1] = b1;
  }
  for (int e = tid; e < M * P; e += kThreads) {
    const int ri = e / P, p = e % P, s = ri / R, r = ri % R;
    float xv = 0.f, yv = 0.f;
    if (s < nt) {
      const int64_t o = ((q.base + q.t0 + s) * H + q.h) * R * P + (int64_t)r * P + p;
      xv = io_load(a.x, o, a.bf16);
      yv = io_load(g.dy, o, a.bf16);
    }
    X[ri * ldp + p] = xv;
    dY[ri * ldp + p] = yv;
  }
  __syncthreads();

  // scores S = Ct Bt^T and DX = dY X^T on the causal token blocks
  for (int e = tid; e < M * M; e += kThreads) {
    const int i = e / M, j = e % M;
    float sv = 0.f, dv = 0.f;
    if (j / R <= i / R && i / R < nt) {
      for (int n = 0; n < N; ++n) sv = fmaf(Ct[i * ldn + n], Bt[j * ldn + n], sv);
      for (int p = 0; p < P; ++p) dv = fmaf(dY[i * ldp + p], X[j * ldp + p], dv);
    }
    S[e] = sv;
    DX[e] = dv;
  }
  __syncthreads();
  // dL/dM per token pair, summed over the ranks of both tokens
  for (int e = tid; e < Q * Q; e += kThreads) {
    const int t = e / Q, s = e % Q;
    float v = 0.f;
    if (s <= t && t < nt)
      for (int r = 0; r < R; ++r)
        for (int r2 = 0; r2 < R; ++r2) {
          const int o = (t * R + r) * M + s * R + r2;
          v = fmaf(S[o], DX[o], v);
        }
    dMt[e] = v;
  }
  __syncthreads();
  auto mtok = [&](int t, int s) {  // mask entry M_ts, s <= t < nt
    return s == t ? gam[t] : expf(lcum[t] - lcum[s]) * del[s];
  };
  // S <- M o S,  DX <- M o DX
  for (int e = tid; e < M * M; e += kThreads) {
    const int t = (e / M) / R, s = (e % M) / R;
    const float m = (s <= t && t < nt) ? mtok(t, s) : 0.f;
    S[e] *= m;
    DX[e] *= m;
  }
  // the mask's own gradients: Lam (row minus column), gamma, delta
  for (int u = tid; u < nt; u += kThreads) {
    float dl = 0.f, dd = 0.f;
    for (int s = 0; s <= u; ++s) dl = fmaf(dMt[u * Q + s], mtok(u, s), dl);
    for (int t = u; t < nt; ++t) dl -= dMt[t * Q + u] * mtok(t, u);
    for (int t = u + 1; t < nt; ++t) dd = fmaf(dMt[t * Q + u], expf(lcum[t] - lcum[u]), dd);
    dLam[u] += dl;
    dgam[u] += dMt[u * Q + u];
    ddel[u] += dd;
  }
  __syncthreads();

  const int TPR = kThreads / M;  // threads per row
  const int row = tid / TPR, qq = tid % TPR;
  const int64_t cidx = (q.b * H + q.h) * a.nchunks + q.c;
  const float* Gc = w.G + cidx * (int64_t)N * P;  // state entering the chunk
  const float* Do = w.D + cidx * (int64_t)N * P;  // adjoint of the state leaving it
  const int np = (K - qq + TPR - 1) / TPR;        // pairs of this thread: k = qq + TPR * m

  // dCt rows -> dC, dPhi (C's rotation), dLam (the exp(Lam_t) term)
  if (row < M && row / R < nt) {
    const int i = row, t = i / R, r = i % R;
    float acc[2 * kMaxPairs];
#pragma unroll
    for (int m = 0; m < 2 * kMaxPairs; ++m) acc[m] = 0.f;
    for (int j = 0; j < (t + 1) * R; ++j) {
      const float pij = DX[i * M + j];
#pragma unroll
      for (int m = 0; m < kMaxPairs; ++m)
        if (m < np) {
          const int k = qq + TPR * m;
          acc[2 * m] = fmaf(pij, Bt[j * ldn + 2 * k], acc[2 * m]);
          acc[2 * m + 1] = fmaf(pij, Bt[j * ldn + 2 * k + 1], acc[2 * m + 1]);
        }
    }
    const float el = expf(lcum[t]);
    float dl = 0.f;
    const int64_t base = ((q.base + q.t0 + t) * a.ngroups + q.g) * R * N + (int64_t)r * N;
#pragma unroll
    for (int m = 0; m < kMaxPairs; ++m)
      if (m < np) {
        const int k = qq + TPR * m;
        float g0 = 0.f, g1 = 0.f;
        for (int p = 0; p < P; ++p) {
          const float yv = dY[i * ldp + p];
          g0 = fmaf(yv, __ldg(Gc + (2 * k) * P + p), g0);
          g1 = fmaf(yv, __ldg(Gc + (2 * k + 1) * P + p), g1);
        }
        const float c0 = Ct[i * ldn + 2 * k], c1 = Ct[i * ldn + 2 * k + 1];
        dl = fmaf(c0, g0, fmaf(c1, g1, dl));
        const float d0 = fmaf(el, g0, acc[2 * m]), d1 = fmaf(el, g1, acc[2 * m + 1]);
        atomicAdd(dPhi + t * K + k, d0 * c1 - d1 * c0);
        float sn, cs;
        sincosf(phi[t * K + k], &sn, &cs);
        atomicAdd(g.dC + base + 2 * k, cs * d0 - sn * d1);  // Rot(Phi_t) dCt
        atomicAdd(g.dC + base + 2 * k + 1, sn * d0 + cs * d1);
      }
    atomicAdd(dLam + t, el * dl);
  }

  // dBt rows -> dB, dPhi (B's rotation), beta_s = Bt_s^T dGhat x_s
  if (row < M && row / R < nt) {
    const int j = row, s = j / R, r = j % R;
    float acc[2 * kMaxPairs];
#pragma unroll
    for (int m = 0; m < 2 * kMaxPairs; ++m) acc[m] = 0.f;
    for (int i = s * R; i < nt * R; ++i) {
      const float pij = DX[i * M + j];
#pragma unroll
      for (int m = 0; m < kMaxPairs; ++m)
        if (m < np) {
          const int k = qq + TPR * m;
          acc[2 * m] = fmaf(pij, Ct[i * ldn + 2 * k], acc[2 * m]);
          acc[2 * m + 1] = fmaf(pij, Ct[i * ldn + 2 * k + 1], acc[2 * m + 1]);
        }
    }
    const float ws = wv[s];
    float bt = 0.f;
    const int64_t base = ((q.base + q.t0 + s) * a.ngroups + q.g) * R * N + (int64_t)r * N;
#pragma unroll
    for (int m = 0; m < kMaxPairs; ++m)
      if (m < np) {
        const int k = qq + TPR * m;
        float a0 = 0.f, a1 = 0.f;
        for (int p = 0; p < P; ++p) {
          const float xv = X[j * ldp + p];
          a0 = fmaf(__ldg(Do + (2 * k) * P + p), xv, a0);
          a1 = fmaf(__ldg(Do + (2 * k + 1) * P + p), xv, a1);
        }
        const float ce = ecs[2 * k], se = ecs[2 * k + 1];
        const float v0 = ce * a0 + se * a1, v1 = -se * a0 + ce * a1;  // (dGhat x_j) pair
        const float b0 = Bt[j * ldn + 2 * k], b1 = Bt[j * ldn + 2 * k + 1];
        bt = fmaf(b0, v0, fmaf(b1, v1, bt));
        const float d0 = fmaf(ws, v0, acc[2 * m]), d1 = fmaf(ws, v1, acc[2 * m + 1]);
        atomicAdd(dPhi + s * K + k, d0 * b1 - d1 * b0);
        float sn, cs;
        sincosf(phi[s * K + k], &sn, &cs);
        atomicAdd(g.dB + base + 2 * k, cs * d0 - sn * d1);  // Rot(Phi_s) dBt
        atomicAdd(g.dB + base + 2 * k + 1, sn * d0 + cs * d1);
      }
    atomicAdd(beta + s, bt);
  }

  // dX rows
  if (row < M && row / R < nt) {
    const int j = row, s = j / R, r = j % R;
    const int nc = (P - qq + TPR - 1) / TPR;  // columns p = qq + TPR * m
    float acc[kMaxCols];
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) acc[m] = 0.f;
    for (int i = s * R; i < nt * R; ++i) {
      const float pij = S[i * M + j];
#pragma unroll
      for (int m = 0; m < kMaxCols; ++m)
        if (m < nc) acc[m] = fmaf(pij, dY[i * ldp + qq + TPR * m], acc[m]);
    }
    const float ws = wv[s];
    float* dxo = g.dx + ((q.base + q.t0 + s) * H + q.h) * R * P + (int64_t)r * P;
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m)
      if (m < nc) {
        const int p = qq + TPR * m;
        float v = 0.f;  // (dGhat^T Bt_j)_p = sum_k Do_pair . Rot(Phi_end) Bt_pair
        for (int k = 0; k < K; ++k) {
          const float b0 = Bt[j * ldn + 2 * k], b1 = Bt[j * ldn + 2 * k + 1];
          const float ce = ecs[2 * k], se = ecs[2 * k + 1];
          v = fmaf(__ldg(Do + (2 * k) * P + p), ce * b0 - se * b1,
                   fmaf(__ldg(Do + (2 * k + 1) * P + p), se * b0 + ce * b1, v));
        }
        dxo[p] = fmaf(ws, v, acc[m]);
      }
  }

  // <dGhat, G_c> and the outgoing rotation's angle gradient
  {
    const float* Gn = (q.c + 1 < a.nchunks) ? Gc + (int64_t)N * P   // next chunk's start state
                                            : w.fin + (q.b * H + q.h) * (int64_t)N * P;
    float part = 0.f;
    for (int e = tid; e < K * P; e += kThreads) {
      const int k = e / P, p = e % P;
      const float o0 = __ldg(Do + (2 * k) * P + p), o1 = __ldg(Do + (2 * k + 1) * P + p);
      const float ce = ecs[2 * k], se = ecs[2 * k + 1];
      const float h0v = ce * o0 + se * o1, h1v = -se * o0 + ce * o1;  // dGhat pair
      part = fmaf(h0v, __ldg(Gc + (2 * k) * P + p), fmaf(h1v, __ldg(Gc + (2 * k + 1) * P + p), part));
      atomicAdd(dPhi + t1 * K + k,
                o1 * __ldg(Gn + (2 * k) * P + p) - o0 * __ldg(Gn + (2 * k + 1) * P + p));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if ((tid & 31) == 0) red[tid >> 5] = part;
  }
  __syncthreads();
  // w_s = exp(Lam_end - Lam_s) delta_s and the exp(Lam_end) G_c term of Ghat
  for (int u = tid; u < nt; u += kThreads) {
    float dl = -wv[u] * beta[u];
    if (u == t1) {
      float dgg = 0.f, wb = 0.f;
      for (int i = 0; i < kThreads / 32; ++i) dgg += red[i];
      for (int s = 0; s < nt; ++s) wb = fmaf(wv[s], beta[s], wb);
      dl += wb + expf(lam_end) * dgg;
    }
    dLam[u] += dl;
    ddel[u] = fmaf(expf(lam_end - lcum[u]), beta[u], ddel[u]);
  }
  __syncthreads();

  // through the prefix sums: d(dt theta) and theta's gradient, per pair
  for (int k = tid; k < K; k += kThreads) {
    float run = 0.f;
    for (int u = nt - 1; u >= 0; --u) {
      run += dPhi[u * K + k];
      const int64_t to = ((q.base + q.t0 + u) * a.tgroups + q.tg) * K + k;
      atomicAdd(g.dtheta + to, dts[u] * run);
      atomicAdd(thT + u, __ldg(a.theta + to) * run);
    }
  }
  __syncthreads();
  // per token: dt, A, lam (gamma = lam dt, eps = (1 - lam) dt, delta_s = gamma_s + eps_s+1)
  for (int u = tid; u < nt; u += kThreads) {
    float run = 0.f;
    for (int t = u; t < nt; ++t) run += dLam[t];
    const int64_t o = (q.base + q.t0 + u) * H + q.h;
    const float dt = dts[u], lam = __ldg(a.lam + o), Av = __ldg(a.A + o);
    const float dg = dgam[u] + ddel[u];
    const float de = (u > 0) ? ddel[u - 1] : 0.f;  // eps_u through delta_u-1 (this chunk)
    g.dA[o] = dt * run;
    atomicAdd(g.ddt + o, Av * run + thT[u] + lam * dg + (1.f - lam) * de);
    atomicAdd(g.dlam + o, dt * (dg - de));
    if (u == t1 && q.t0 + nt < q.len) {  // the next token's eps, through delta_end
      const int64_t on = o + H;
      const float lamn = __ldg(a.lam + on), dtn = __ldg(a.dt + on);
      atomicAdd(g.ddt + on, (1.f - lamn) * ddel[u]);
      atomicAdd(g.dlam + on, -dtn * ddel[u]);
    }
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

constexpr size_t kSmemMax = 227 * 1024;

// Rows per chunk of the backward (M = Qb * R): the largest of 64, 32, 16 whose
// shared memory and per-thread accumulators fit.
int64_t bwd_rows(const ScanArgs& a) {
  for (int64_t M = 64; M >= 16; M /= 2) {
    if (M < a.R || M % a.R != 0) continue;
    const int64_t Qb = M / a.R;
    const ChunkSmem L((int)M, (int)a.N, (int)a.P, (int)Qb);
    const int64_t tpr = kThreads / M;
    if ((size_t)L.total * 4 <= kSmemMax && (a.N / 2) <= kMaxPairs * tpr &&
        a.P <= kMaxCols * tpr)
      return M;
  }
  return 0;
}

size_t dstate_smem(const ScanArgs& f) {
  return sizeof(float) * (4 * f.Q + f.Q * (f.N / 2) + kTileRows * (f.N + f.P));
}

template <int R>
cudaError_t launch_r(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st) {
  cudaError_t e;
  const int64_t opt = (f.N * f.P + kThreads - 1) / kThreads;
  const size_t sm1 = dstate_smem(f);
  dim3 grid((unsigned)f.nchunks, (unsigned)f.nheads, (unsigned)f.batch);
#define M3_DSTATE(O)                                                  \
  do {                                                                \
    e = set_smem(bwd_dstate_kernel<R, O>, sm1);                       \
    if (e != cudaSuccess) return e;                                   \
    bwd_dstate_kernel<R, O><<<grid, kThreads, sm1, st>>>(f, g, w);    \
  } while (0)
  if (opt <= 8) M3_DSTATE(8);
  else if (opt <= 16) M3_DSTATE(16);
  else if (opt <= 32) M3_DSTATE(32);
  else M3_DSTATE(64);
#undef M3_DSTATE
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  dim3 pgrid((unsigned)(((f.N / 2) * f.P + kThreads - 1) / kThreads), (unsigned)f.nheads,
             (unsigned)f.batch);
  bwd_state_pass_kernel<<<pgrid, kThreads, 0, st>>>(f, g, w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const ChunkSmem L((int)(f.Q * R), (int)f.N, (int)f.P, (int)f.Q);
  const size_t sm3 = sizeof(float) * (size_t)L.total;
  e = set_smem(bwd_chunk_kernel<R>, sm3);
  if (e != cudaSuccess) return e;
  bwd_chunk_kernel<R><<<grid, kThreads, sm3, st>>>(f, g, w);
  return cudaGetLastError();
}

BwdWs carve(const ScanArgs& f) {
  BwdWs w;
  simt_state_views(f, &w.G, &w.sums);
  const size_t fwd = simt_scan_workspace(f);
  const size_t dbytes = align_up(sizeof(float) * f.batch * f.nheads * f.nchunks * f.N * f.P, 256);
  w.D = reinterpret_cast<float*>(f.ws + fwd);
  w.fin = reinterpret_cast<float*>(f.ws + fwd + dbytes);
  return w;
}

}  // namespace

bool bwd_supported(const ScanArgs& a) { return bwd_rows(a) > 0 && a.cu_seqlens == nullptr; }

size_t bwd_workspace(const ScanArgs& a) {
  const int64_t M = bwd_rows(a);
  if (M == 0 || a.seqlen == 0) return 0;
  const ScanArgs f = fwd_args(a, M / a.R);
  return simt_scan_workspace(f) +
         align_up(sizeof(float) * f.batch * f.nheads * f.nchunks * f.N * f.P, 256) +
         align_up(sizeof(float) * f.batch * f.nheads * f.N * f.P, 256);
}

cudaError_t bwd_launch(const ScanArgs& a, const BwdArgs& g, cudaStream_t st) {
  const int64_t M = bwd_rows(a);
  if (M == 0) return cudaErrorInvalidValue;
  ScanArgs f = fwd_args(a, M / a.R);
  BwdWs w = carve(f);
  f.final_state = w.fin;
  // outputs accumulated with atomic adds start from zero
  const int64_t tok = a.batch * a.seqlen;
  const int64_t K = a.N / 2;
  struct Z { float* p; int64_t n; } zs[] = {
      {g.ddt, tok * a.nheads}, {g.dlam, tok * a.nheads}, {g.dtheta, tok * a.tgroups * K},
      {g.dB, tok * a.ngroups * a.R * a.N}, {g.dC, tok * a.ngroups * a.R * a.N},
      {g.dB_prev, a.batch * a.ngroups * a.R * a.N}, {g.dx_prev, a.batch * a.nheads * a.R * a.P}};
  for (const Z& z : zs)
    if (z.p && z.n > 0) {
      cudaError_t e = cudaMemsetAsync(z.p, 0, sizeof(float) * z.n, st);
      if (e != cudaSuccess) return e;
    }
  cudaError_t e = simt_scan_launch(f, st);  // chunk-start states, totals, final state
  if (e != cudaSuccess) return e;
  switch (a.R) {
    case 1: return launch_r<1>(f, g, w, st);
    case 2: return launch_r<2>(f, g, w, st);
    case 4: return launch_r<4>(f, g, w, st);
    case 8: return launch_r<8>(f, g, w, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
