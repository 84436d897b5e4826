// scan_simt.cu -- CUDA-core fp32 chunked prefill scan of the Mamba-3 layer.
//
// This is the exact-fp32 path (fp32 io at 1e-4) and the debugging twin of the
// tensor-core path.  It evaluates the chunked form of the recurrence:
//
// Per (b, h), chunk c = tokens [c0, c0 + nt), chunk-local inclusive sums
//   Lam_t = sum_{c0<=u<=t} dt_u A_u,  Phi_{t,k} = sum_{c0<=u<=t} dt_u theta_{u,k},
// rotated operands (data-dependent RoPE, paper section 2.2)
//   Bt_s = Rot(-Phi_s) B_s,  Ct_t = Rot(-Phi_t) C_t,
// and the trapezoid weights (section 2.2: the mask is decay x width-2 conv)
//   gamma_t = lam_t dt_t,  delta_s = gamma_s + (1 - lam_{s+1}) dt_{s+1}
//   (delta_{L-1} = gamma_{L-1}: no token follows the last one).
//
//   1. chunk state  S_c = sum_s exp(Lam_end - Lam_s) delta_s Bt_s x_s^T   (N x P)
//   2. state pass   G_c = state carried into chunk c (true frame);
//                   G_0 = h0 + (1 - lam_0) dt_0 B_prev x_prev^T,
//                   G_{c+1} = Rot(Phi_end) (exp(Lam_end) G_c + S_c);
//                   the last G is h_{L-1} (final_state).
//   3. chunk output y_t = exp(Lam_t) Ct_t^T G_c
//                   + sum_{s<=t} exp(Lam_t - Lam_s) w_{t,s} (Ct_t . Bt_s) x_s,
//                   w_{t,t} = gamma_t, w_{t,s<t} = delta_s.
//
// Workspace: S / G [b][H][nc][N][P] fp32 (G overwrites S in place) and the
// chunk summaries [b][H][nc][1 + N/2] fp32 (Lam_end, Phi_end[k]).
#include "m3_internal.cuh"
#include "simt_chunk.cuh"

namespace m3 {
namespace {

using simt::Geo;
using simt::chunk_geo;
using simt::chunk_prep;

constexpr int kThreads = 256;
constexpr int kTileRows = 64;  // (token, rank) rows of B / x per staged tile
constexpr int kOutRows = 32;   // (token, rank) output rows per chunk-output CTA

// Stage rows (s, r) of Rot(-Phi_s) B_s (scaled per token by wts[s] if given)
// and of x_s for tokens [s0, s0 + kTileRows / R) into shared memory.
// Rows past the chunk end are zero.
template <int R>
__device__ void stage_tile(const ScanArgs& a, const Geo& q, int s0, const float* phi,
                           const float* wts, float* Bs, int ldb, float* Xs) {
  const int K = (int)(a.N / 2), N = (int)a.N, P = (int)a.P;
  for (int e = threadIdx.x; e < kTileRows * K; e += blockDim.x) {
    const int ri = e / K, k = e % K;
    const int s = s0 + ri / R, r = ri % R;
    float v0 = 0.f, v1 = 0.f;
    if (s < q.nt) {
      const int64_t base = ((q.base + q.t0 + s) * a.ngroups + q.g) * R * N + (int64_t)r * N;
      const float b0 = io_load(a.B, base + 2 * k, a.bf16);
      const float b1 = io_load(a.B, base + 2 * k + 1, a.bf16);
      float sn, cs;
      sincosf(phi[s * K + k], &sn, &cs);
      const float w = wts ? wts[s] : 1.f;
      v0 = w * (cs * b0 + sn * b1);
      v1 = w * (-sn * b0 + cs * b1);
    }
    Bs[ri * ldb + 2 * k] = v0;
    Bs[ri * ldb + 2 * k + 1] = v1;
  }
  for (int e = threadIdx.x; e < kTileRows * P; e += blockDim.x) {
    const int ri = e / P, p = e % P;
    const int s = s0 + ri / R, r = ri % R;
    float v = 0.f;
    if (s < q.nt)
      v = io_load(a.x, ((q.base + q.t0 + s) * a.nheads + q.h) * R * P + (int64_t)r * P + p,
                  a.bf16);
    Xs[ri * P + p] = v;
  }
}

struct WsView {
  float* S;    // [b][H][nc][N][P]
  float* sum;  // [b][H][nc][1 + K]
};

__host__ __device__ __forceinline__ WsView ws_view(const ScanArgs& a) {
  WsView w;
  const size_t sbytes = align_up(sizeof(float) * a.batch * a.nheads * a.nchunks * a.N * a.P, 256);
  w.S = reinterpret_cast<float*>(a.ws);
  w.sum = reinterpret_cast<float*>(a.ws + sbytes);
  return w;
}

// ---- 1. chunk state ---------------------------------------------------------
// Thread tiles of 4 x 4 (n, p) outputs; per staged row a thread reads one float4
// of the rotated B row and one of x (TPT tiles per thread).
template <int R, int TPT>
__global__ void __launch_bounds__(kThreads) chunk_state_kernel(const ScanArgs a) {
  const Geo q = chunk_geo(a, blockIdx.x);
  if (!simt::geo_ok(a, q)) return;  // uniform over the block
  const int N = (int)a.N, P = (int)a.P, K = N / 2, Q = (int)a.Q;
  extern __shared__ __align__(16) float sm[];
  float* lcum = sm;
  float* gam = lcum + Q;
  float* del = gam + Q;
  float* dts = del + Q;
  float* wts = dts + Q;
  float* phi = wts + Q;
  float* Bs = phi + Q * K;           // [kTileRows][N]
  float* Xs = Bs + kTileRows * N;    // [kTileRows][P]

  chunk_prep(a, q, lcum, gam, del, dts, phi);
  for (int i = threadIdx.x; i < q.nt; i += blockDim.x)
    wts[i] = expf(lcum[q.nt - 1] - lcum[i]) * del[i];
  __syncthreads();

  const int PG = P / 4, ntiles = (N / 4) * PG;
  float acc[TPT][4][4];
#pragma unroll
  for (int m = 0; m < TPT; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[m][u][v] = 0.f;

  const int TS = kTileRows / R;
  for (int s0 = 0; s0 < q.nt; s0 += TS) {
    stage_tile<R>(a, q, s0, phi, wts, Bs, N, Xs);
    __syncthreads();
    const int rows = min(kTileRows, (q.nt - s0) * R);
    for (int ri = 0; ri < rows; ++ri) {
#pragma unroll
      for (int m = 0; m < TPT; ++m) {
        const int ti = threadIdx.x + kThreads * m;
        if (ti < ntiles) {
          const float4 bv = *reinterpret_cast<const float4*>(Bs + ri * N + 4 * (ti / PG));
          const float4 xv = *reinterpret_cast<const float4*>(Xs + ri * P + 4 * (ti % PG));
          const float b4[4] = {bv.x, bv.y, bv.z, bv.w}, x4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[m][u][v] = fmaf(b4[u], x4[v], acc[m][u][v]);
        }
      }
    }
    __syncthreads();
  }
  const WsView w = ws_view(a);
  const int64_t cidx = (q.b * a.nheads + q.h) * a.nchunks + q.c;
  float* S = w.S + cidx * N * P;
#pragma unroll
  for (int m = 0; m < TPT; ++m) {
    const int ti = threadIdx.x + kThreads * m;
    if (ti < ntiles) {
      const int n0 = 4 * (ti / PG), p0 = 4 * (ti % PG);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(S + (n0 + u) * P + p0) =
            make_float4(acc[m][u][0], acc[m][u][1], acc[m][u][2], acc[m][u][3]);
    }
  }
  // an empty chunk (past a short packed sequence) passes the state unchanged
  float* sm_out = w.sum + cidx * (1 + K);
  if (threadIdx.x == 0) sm_out[0] = q.nt > 0 ? lcum[q.nt - 1] : 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    sm_out[1 + k] = q.nt > 0 ? phi[(q.nt - 1) * K + k] : 0.f;
}

// ---- 2. state passing -------------------------------------------------------
__global__ void __launch_bounds__(kThreads) state_pass_kernel(const ScanArgs a) {
  const int N = (int)a.N, P = (int)a.P, K = N / 2;
  const int64_t b = blockIdx.z, h = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= K * P) return;
  const int k = idx / P, p = idx % P;
  const int64_t H = a.nheads, R = a.R;
  const int64_t g = h / (H / a.ngroups);
  const Chain ch = chain_of(a, b);
  float g0 = 0.f, g1 = 0.f;
  const int64_t so = ((b * H + h) * N) * P;
  if (!M3_IN(b, a.batch, a.status) || !M3_IN(h, a.nheads, a.status)) return;
  if (a.h0) {
    g0 = a.h0[so + (2 * k) * P + p];
    g1 = a.h0[so + (2 * k + 1) * P + p];
  }
  if (a.B_prev && ch.len > 0) {  // the left endpoint term waits for a token
    const float eps = (1.f - a.lam[ch.base * H + h]) * a.dt[ch.base * H + h];
    for (int r = 0; r < R; ++r) {
      const int64_t bb = ((b * a.ngroups + g) * R + r) * N;
      const float xv = io_load(a.x_prev, ((b * H + h) * R + r) * P + p, a.bf16);
      g0 = fmaf(eps * io_load(a.B_prev, bb + 2 * k, a.bf16), xv, g0);
      g1 = fmaf(eps * io_load(a.B_prev, bb + 2 * k + 1, a.bf16), xv, g1);
    }
  }
  const WsView w = ws_view(a);
  // chunks in batches of kPipe, all of a batch's loads issued before its
  // dependent updates (the chain waits on arithmetic, not on each load)
  constexpr int kPipe = 8;
  for (int64_t c0 = 0; c0 < a.nchunks; c0 += kPipe) {
    float s0[kPipe], s1[kPipe], dec[kPipe], sn[kPipe], cs[kPipe];
#pragma unroll
    for (int j = 0; j < kPipe; ++j) {
      const int64_t c = c0 + j;
      if (c >= a.nchunks) break;
      const int64_t cidx = (b * H + h) * a.nchunks + c;
      const float* S = w.S + cidx * N * P;
      const float* su = w.sum + cidx * (1 + K);
      s0[j] = S[(2 * k) * P + p];
      s1[j] = S[(2 * k + 1) * P + p];
      dec[j] = expf(su[0]);
      sincosf(su[1 + k], &sn[j], &cs[j]);
    }
#pragma unroll
    for (int j = 0; j < kPipe; ++j) {
      const int64_t c = c0 + j;
      if (c >= a.nchunks) break;
      float* S = w.S + ((b * H + h) * a.nchunks + c) * N * P;
      S[(2 * k) * P + p] = g0;  // chunk-start state, true frame
      S[(2 * k + 1) * P + p] = g1;
      const float v0 = fmaf(dec[j], g0, s0[j]), v1 = fmaf(dec[j], g1, s1[j]);
      g0 = cs[j] * v0 - sn[j] * v1;
      g1 = sn[j] * v0 + cs[j] * v1;
    }
  }
  if (a.final_state && M3_IN(so + (2 * k + 1) * P + p, a.batch * H * N * P, a.status)) {
    a.final_state[so + (2 * k) * P + p] = g0;
    a.final_state[so + (2 * k + 1) * P + p] = g1;
  }
}

// ---- 3. chunk output --------------------------------------------------------
template <int R, int YPT>
__global__ void __launch_bounds__(kThreads) chunk_output_kernel(const ScanArgs a) {
  const int N = (int)a.N, P = (int)a.P, K = N / 2, Q = (int)a.Q;
  const int tiles_per_chunk = (Q * R + kOutRows - 1) / kOutRows;
  const int64_t c = blockIdx.x / tiles_per_chunk;
  const int tile = blockIdx.x % tiles_per_chunk;
  const Geo q = chunk_geo(a, c);
  if (!simt::geo_ok(a, q)) return;  // uniform over the block
  const int TT = kOutRows / R;          // tokens per output tile
  const int tt0 = tile * TT;            // first token (chunk-local) of the tile
  if (tt0 >= q.nt) return;
  const int tt1 = min(tt0 + TT, q.nt);  // one past the last valid token

  extern __shared__ __align__(16) float sm[];
  float* lcum = sm;
  float* gam = lcum + Q;
  float* del = gam + Q;
  float* dts = del + Q;
  float* phi = dts + Q;
  const int ldc = N + 1;
  float* Cs = phi + Q * K;               // [kOutRows][N+1]  Rot(-Phi_t) C_t
  float* Bs = Cs + kOutRows * ldc;       // [kTileRows][N+1] Rot(-Phi_s) B_s, or a G tile [64][P]
  float* Xs = Bs + kTileRows * max(ldc, P);  // [kTileRows][P]
  float* Sc = Xs + kTileRows * P;        // [kOutRows][kTileRows+1] masked scores

  chunk_prep(a, q, lcum, gam, del, dts, phi);
  for (int e = threadIdx.x; e < kOutRows * K; e += blockDim.x) {
    const int ro = e / K, k = e % K;
    const int t = tt0 + ro / R, r = ro % R;
    float v0 = 0.f, v1 = 0.f;
    if (t < tt1) {
      const int64_t base = ((q.base + q.t0 + t) * a.ngroups + q.g) * R * N + (int64_t)r * N;
      const float c0 = io_load(a.C, base + 2 * k, a.bf16);
      const float c1 = io_load(a.C, base + 2 * k + 1, a.bf16);
      float sn, cs;
      sincosf(phi[t * K + k], &sn, &cs);
      v0 = cs * c0 + sn * c1;
      v1 = -sn * c0 + cs * c1;
    }
    Cs[ro * ldc + 2 * k] = v0;
    Cs[ro * ldc + 2 * k + 1] = v1;
  }
  __syncthreads();

  const int p = threadIdx.x % P, ro0 = threadIdx.x / P, RS = kThreads / P;
  float acc[YPT];
#pragma unroll
  for (int i = 0; i < YPT; ++i) acc[i] = 0.f;

  // inter-chunk term: exp(Lam_t) Ct_t^T G_c, G_c staged 64 rows at a time
  const WsView w = ws_view(a);
  const int64_t cidx = (q.b * a.nheads + q.h) * a.nchunks + q.c;
  const float* G = w.S + cidx * N * P;
  for (int n0 = 0; n0 < N; n0 += kTileRows) {
    const int nr = min(kTileRows, N - n0);
    for (int e = threadIdx.x; e < nr * P; e += blockDim.x) Bs[e] = G[(int64_t)n0 * P + e];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < YPT; ++i) {
      const int ro = ro0 + i * RS;
      float s = acc[i];
      for (int n = 0; n < nr; ++n) s = fmaf(Cs[ro * ldc + n0 + n], Bs[n * P + p], s);
      acc[i] = s;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < YPT; ++i) {
    const int t = tt0 + (ro0 + i * RS) / R;
    acc[i] *= (t < tt1) ? expf(lcum[t]) : 0.f;
  }

  // intra-chunk term over source tiles s <= t
  const int TS = kTileRows / R;
  for (int s0 = 0; s0 < tt1; s0 += TS) {
    stage_tile<R>(a, q, s0, phi, nullptr, Bs, ldc, Xs);
    __syncthreads();
    for (int e = threadIdx.x; e < kOutRows * kTileRows; e += blockDim.x) {
      const int ro = e / kTileRows, ci = e % kTileRows;
      const int t = tt0 + ro / R, s = s0 + ci / R;
      float v = 0.f;
      if (t < tt1 && s <= t) {
        float d = 0.f;
        for (int n = 0; n < N; ++n) d = fmaf(Cs[ro * ldc + n], Bs[ci * ldc + n], d);
        const float wgt = (s == t) ? gam[t] : del[s];
        v = expf(lcum[t] - lcum[s]) * wgt * d;
      }
      Sc[ro * (kTileRows + 1) + ci] = v;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < YPT; ++i) {
      const int ro = ro0 + i * RS;
      float s = acc[i];
      for (int ci = 0; ci < kTileRows; ++ci)
        s = fmaf(Sc[ro * (kTileRows + 1) + ci], Xs[ci * P + p], s);
      acc[i] = s;
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < YPT; ++i) {
    const int ro = ro0 + i * RS;
    const int t = tt0 + ro / R, r = ro % R;
    const int64_t yo = ((q.base + q.t0 + t) * a.nheads + q.h) * R * P + (int64_t)r * P + p;
    if (t < tt1 && M3_IN(yo, a.total_tokens * a.nheads * R * P, a.status))
      io_store(a.y, yo, acc[i], a.bf16);
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

template <int R, int TPT>
cudaError_t launch_state(const ScanArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (5 * a.Q + a.Q * (a.N / 2) + kTileRows * (a.N + a.P));
  cudaError_t e = set_smem(chunk_state_kernel<R, TPT>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.nchunks, (unsigned)a.nheads, (unsigned)a.batch);
  chunk_state_kernel<R, TPT><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int R, int YPT>
cudaError_t launch_output(const ScanArgs& a, cudaStream_t st) {
  const size_t ldc = a.N + 1;
  const size_t ldb = ldc > (size_t)a.P ? ldc : (size_t)a.P;
  const size_t smem = sizeof(float) * (4 * a.Q + a.Q * (a.N / 2) + kOutRows * ldc +
                                       kTileRows * ldb + kTileRows * a.P +
                                       kOutRows * (kTileRows + 1));
  cudaError_t e = set_smem(chunk_output_kernel<R, YPT>, smem);
  if (e != cudaSuccess) return e;
  const unsigned tiles = (unsigned)((a.Q * R + kOutRows - 1) / kOutRows);
  dim3 grid((unsigned)a.nchunks * tiles, (unsigned)a.nheads, (unsigned)a.batch);
  chunk_output_kernel<R, YPT><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_all(const ScanArgs& a, cudaStream_t st) {
  cudaError_t e;
  const int64_t tiles = (a.N / 4) * (a.P / 4);  // 4 x 4 output tiles
  if (tiles <= kThreads) e = launch_state<R, 1>(a, st);
  else if (tiles <= 2 * kThreads) e = launch_state<R, 2>(a, st);
  else e = launch_state<R, 4>(a, st);
  if (e != cudaSuccess) return e;

  const int K = (int)(a.N / 2);
  dim3 pgrid((unsigned)((K * a.P + kThreads - 1) / kThreads), (unsigned)a.nheads,
             (unsigned)a.batch);
  state_pass_kernel<<<pgrid, kThreads, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.state_only) return e;

  const int64_t ypt = (kOutRows * a.P) / kThreads;  // P / 8
  if (ypt <= 2) return launch_output<R, 2>(a, st);
  if (ypt <= 4) return launch_output<R, 4>(a, st);
  if (ypt <= 8) return launch_output<R, 8>(a, st);
  return launch_output<R, 16>(a, st);
}

}  // namespace

size_t simt_scan_workspace(const ScanArgs& a) {
  const size_t sbytes = align_up(sizeof(float) * a.batch * a.nheads * a.nchunks * a.N * a.P, 256);
  const size_t mbytes =
      align_up(sizeof(float) * a.batch * a.nheads * a.nchunks * (1 + a.N / 2), 256);
  return sbytes + mbytes;
}

void simt_state_views(const ScanArgs& a, float** states, float** sums) {
  const WsView w = ws_view(a);
  *states = w.S;
  *sums = w.sum;
}

cudaError_t simt_scan_launch(const ScanArgs& a, cudaStream_t st) {
  switch (a.R) {
    case 1: return launch_all<1>(a, st);
    case 2: return launch_all<2>(a, st);
    case 4: return launch_all<4>(a, st);
    case 8: return launch_all<8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
