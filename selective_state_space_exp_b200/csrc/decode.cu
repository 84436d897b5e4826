// decode.cu -- single-token decode step of the Mamba-3 SSM layer.
//
// Per (batch, head) the fp32 state h (N x P) is read once and written once:
//   g      = h + (1 - lam) dt B_prev x_prev^T          (left endpoint, rank R)
//   h'     = alpha Rot(dt theta) g + lam dt B_t x_t^T   (pairs (2k, 2k+1))
//   y_t    = C_t^T h'                                   (R x P)
// This is the exponential-trapezoidal step of the paper (PaperWeekly page
// section 2.2) with the complex transition as 2x2 rotations (section 2.1) and
// the rank-R MIMO update (section 2.3).  The step is HBM-bound (section 3.3:
// decode is limited by state IO, not FLOPs): 2 * 4 * N * P bytes per head.
//
// Layout: one CTA of 128 threads per (b, h) (whole state rows).
// Thread (kslot, pv) owns float4 column pv of the block and the pairs
// k = kslot, kslot + nslots, ...; a block row is read by consecutive threads
// as float4 (a contiguous 128-byte segment per row).  The per-head operands
// (B, C, B_prev, x, x_prev, the cos/sin table) are staged in shared memory;
// y is reduced over kslots through shared memory.
#include "m3_internal.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

constexpr int kMaxCols = 128;  // state columns per CTA (whole rows: P <= 128)
constexpr int kPairsInFlight = 4;  // pairs whose state rows are loaded before any is computed

// CTA (b, h, column block): columns [cb*CB, cb*CB + CB) of the head's state
// and of y (columns are independent: y[r][p] only reads column p of h').
// Whole rows per CTA (CB = P) read best: splitting a 256-byte state row
// between CTAs that run at different times costs HBM locality.
// Resident CTAs per SM the register budget is sized for (more state bytes in
// flight for small R, room for the rank-R operands for large R).
// 128 threads per CTA; the register budget is sized for the resident CTAs
// per SM (more state bytes in flight for small R, room for the rank-R
// operands for large R).
template <int R>
struct DecodeCfg {
  static constexpr int threads = 128;
  static constexpr int occupancy = R == 1 ? 7 : (R == 2 ? 5 : (R == 4 ? 4 : 3));
};

template <int R>
__global__ void __launch_bounds__(DecodeCfg<R>::threads, DecodeCfg<R>::occupancy)
decode_kernel(const DecodeArgs a) {
  constexpr int kDecodeThreads = DecodeCfg<R>::threads;
  const int P = (int)a.P, N = (int)a.N, K = N / 2;
  const int CB = P < kMaxCols ? P : kMaxCols;
  const int nblk = P / CB;
  const int64_t bh = blockIdx.x / nblk;
  const int cb = blockIdx.x % nblk;
  const int64_t h = bh % a.nheads, b = bh / a.nheads;
  const int64_t g = h / (a.nheads / a.ngroups);
  const int64_t bg = b * a.ngroups + g;
  const int tid = threadIdx.x;

  extern __shared__ float sm[];
  float* s_ac = sm;               // alpha cos(dt theta_k)          [K]
  float* s_as = s_ac + K;         // alpha sin(dt theta_k)          [K]
  float* s_Bp = s_as + K;         // B_prev, transposed             [N][R]
  float* s_Bt = s_Bp + R * N;     // B_t, transposed                [N][R]
  float* s_Ct = s_Bt + R * N;     // C_t, transposed                [N][R]
  float* s_xe = s_Ct + R * N;     // (1-lam) dt x_prev              [R][CB]
  float* s_xg = s_xe + R * CB;    // lam dt x_t                     [R][CB]
  float* s_red = s_xg + R * CB;   // partial y per kslot            [nslots][R][CB]

  const float dt = a.dt[bh], lamv = a.lam[bh];
  const float alpha = expf(dt * a.A[bh]);
  const float gamma = lamv * dt, eps = (1.f - lamv) * dt;
  const bool prev = a.B_prev != nullptr;

  const int PV = CB / 4;  // float4 columns per state row in this block
  const int nslots = kDecodeThreads / PV;
  const int pv = tid % PV, kslot = tid / PV;
  const int p0 = pv * 4;
  const float4* src = reinterpret_cast<const float4*>(a.state_in + bh * (int64_t)N * P + cb * CB);
  float4* dst = reinterpret_cast<float4*>(a.state_out + bh * (int64_t)N * P + cb * CB);
  const int rowq = P / 4;  // float4 stride between state rows

  // Issue the first pairs' state loads before staging the per-head operands.
  float4 r0[kPairsInFlight], r1[kPairsInFlight];
#pragma unroll
  for (int u = 0; u < kPairsInFlight; ++u) {
    const int k = kslot + u * nslots;
    if (k < K) {
      r0[u] = __ldcs(src + (2 * k) * rowq + pv);
      r1[u] = __ldcs(src + (2 * k + 1) * rowq + pv);
    }
  }

  for (int k = tid; k < K; k += kDecodeThreads) {
    float sn, cs;
    sincosf(dt * a.theta[bg * K + k], &sn, &cs);
    s_ac[k] = alpha * cs;
    s_as[k] = alpha * sn;
  }
  for (int i = tid; i < R * N; i += kDecodeThreads) {  // i = r * N + n -> [n][r]
    const int r = i / N, nn = i % N, ti = nn * R + r;
    s_Bt[ti] = io_load(a.B, bg * R * N + i, a.bf16);
    s_Ct[ti] = io_load(a.C, bg * R * N + i, a.bf16);
    s_Bp[ti] = prev ? io_load(a.B_prev, bg * R * N + i, a.bf16) : 0.f;
  }
  for (int i = tid; i < R * CB; i += kDecodeThreads) {
    const int r = i / CB, c = i % CB;
    const int64_t xi = bh * R * P + r * P + cb * CB + c;
    s_xg[i] = gamma * io_load(a.x, xi, a.bf16);
    s_xe[i] = prev ? eps * io_load(a.x_prev, xi, a.bf16) : 0.f;
  }
  __syncthreads();

  // column pairs (p0, p0+1) and (p0+2, p0+3) as packed fp32x2 operands
  float2 xg[R][2], xe[R][2], yacc[R][2];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      xg[r][j] = make_float2(s_xg[r * CB + p0 + 2 * j], s_xg[r * CB + p0 + 2 * j + 1]);
      xe[r][j] = make_float2(s_xe[r * CB + p0 + 2 * j], s_xe[r * CB + p0 + 2 * j + 1]);
      yacc[r][j] = make_float2(0.f, 0.f);
    }

  for (int kb = kslot; kb < K; kb += kPairsInFlight * nslots) {
    if (kb != kslot) {
#pragma unroll
      for (int u = 0; u < kPairsInFlight; ++u) {
        const int k = kb + u * nslots;
        if (k < K) {
          r0[u] = __ldcs(src + (2 * k) * rowq + pv);
          r1[u] = __ldcs(src + (2 * k + 1) * rowq + pv);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPairsInFlight; ++u) {
      const int k = kb + u * nslots;
      if (k < K) {
        const float ac = s_ac[k], as = s_as[k];
        float bp0[R], bp1[R], bt0[R], bt1[R], c0[R], c1[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {  // rows 2k and 2k+1 are adjacent R-vectors
          bp0[r] = s_Bp[(2 * k) * R + r]; bp1[r] = s_Bp[(2 * k + 1) * R + r];
          bt0[r] = s_Bt[(2 * k) * R + r]; bt1[r] = s_Bt[(2 * k + 1) * R + r];
          c0[r] = s_Ct[(2 * k) * R + r]; c1[r] = s_Ct[(2 * k + 1) * R + r];
        }
        const float2 in0[2] = {make_float2(r0[u].x, r0[u].y), make_float2(r0[u].z, r0[u].w)};
        const float2 in1[2] = {make_float2(r1[u].x, r1[u].y), make_float2(r1[u].z, r1[u].w)};
        float o0[4], o1[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float2 g0 = in0[j], g1 = in1[j], u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            g0 = tc::ffma2(make_float2(bp0[r], bp0[r]), xe[r][j], g0);
            g1 = tc::ffma2(make_float2(bp1[r], bp1[r]), xe[r][j], g1);
            u0 = tc::ffma2(make_float2(bt0[r], bt0[r]), xg[r][j], u0);
            u1 = tc::ffma2(make_float2(bt1[r], bt1[r]), xg[r][j], u1);
          }
          // (h'_{2k}, h'_{2k+1}) = alpha Rot(phi) (g_{2k}, g_{2k+1}) + (u_{2k}, u_{2k+1})
          const float2 w0 = tc::ffma2(make_float2(ac, ac), g0,
                                      tc::ffma2(make_float2(-as, -as), g1, u0));
          const float2 w1 = tc::ffma2(make_float2(as, as), g0,
                                      tc::ffma2(make_float2(ac, ac), g1, u1));
#pragma unroll
          for (int r = 0; r < R; ++r)
            yacc[r][j] = tc::ffma2(make_float2(c0[r], c0[r]), w0,
                                   tc::ffma2(make_float2(c1[r], c1[r]), w1, yacc[r][j]));
          o0[2 * j] = w0.x; o0[2 * j + 1] = w0.y;
          o1[2 * j] = w1.x; o1[2 * j + 1] = w1.y;
        }
        __stcs(dst + (2 * k) * rowq + pv, make_float4(o0[0], o0[1], o0[2], o0[3]));
        __stcs(dst + (2 * k + 1) * rowq + pv, make_float4(o1[0], o1[1], o1[2], o1[3]));
      }
    }
  }

#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      s_red[(kslot * R + r) * CB + p0 + 2 * j] = yacc[r][j].x;
      s_red[(kslot * R + r) * CB + p0 + 2 * j + 1] = yacc[r][j].y;
    }
  __syncthreads();
  for (int i = tid; i < R * CB; i += kDecodeThreads) {
    float acc = 0.f;
    for (int q = 0; q < nslots; ++q) acc += s_red[q * R * CB + i];
    const int r = i / CB, c = i % CB;
    io_store(a.y, bh * R * P + r * P + cb * CB + c, acc, a.bf16);
  }
}

template <int R>
cudaError_t launch_r(const DecodeArgs& a, cudaStream_t s) {
  const int P = (int)a.P, N = (int)a.N;
  const int CB = P < kMaxCols ? P : kMaxCols;
  constexpr int kDecodeThreads = DecodeCfg<R>::threads;
  const int nslots = kDecodeThreads / (CB / 4);
  const size_t smem = sizeof(float) * (N + 3 * R * N + 2 * R * CB + (size_t)nslots * R * CB);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = a.batch * a.nheads * (P / CB);
  decode_kernel<R><<<(unsigned)blocks, kDecodeThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t s) {
  switch (a.R) {
    case 1: return launch_r<1>(a, s);
    case 2: return launch_r<2>(a, s);
    case 4: return launch_r<4>(a, s);
    case 8: return launch_r<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
