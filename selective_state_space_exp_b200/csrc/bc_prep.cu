// bc_prep.cu -- QK-norm, per-channel scale and bias of the B and C projections.
//
// The block normalises each (token, group, rank) row of B and C after their
// projections and adds a learnable bias (PaperWeekly page section 2.4,
// "normalisation and bias"; Figure 4):
//   out[n] = raw[n] * rsqrt(mean_m raw[m]^2 + eps) * weight[n] + bias[n].
// One pass over both tensors: a row of N values is held by N/8 lanes, 16 bytes
// each for bf16 (8 values), the mean square is a shuffle sum over those lanes,
// and the result is rounded to the io dtype.  HBM-bound: every raw value is
// read once and every output written once.
#include "m3_internal.cuh"

namespace m3 {
namespace {

constexpr int kThreads = 256;

struct Vec8 {
  float v[8];
};

template <bool BF16>
__device__ __forceinline__ Vec8 load8(const void* base, int64_t i) {
  Vec8 r;
  if constexpr (BF16) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + i));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      r.v[2 * j] = __uint_as_float(w[j] << 16);
      r.v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + i);
    const float4 a = __ldcs(p), b = __ldcs(p + 1);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  }
  return r;
}

template <bool BF16>
__device__ __forceinline__ void store8(void* base, int64_t i, const Vec8& r) {
  if constexpr (BF16) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(r.v[2 * j], r.v[2 * j + 1]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + i),
           make_uint4(w[0], w[1], w[2], w[3]));
  } else {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + i);
    __stcs(p, make_float4(r.v[0], r.v[1], r.v[2], r.v[3]));
    __stcs(p + 1, make_float4(r.v[4], r.v[5], r.v[6], r.v[7]));
  }
}

__device__ __forceinline__ Vec8 ld_param8(const float* p, int64_t i, float dflt) {
  Vec8 r;
  if (!p) {
#pragma unroll
    for (int j = 0; j < 8; ++j) r.v[j] = dflt;
    return r;
  }
  const float4 a = __ldg(reinterpret_cast<const float4*>(p + i));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + i) + 1);
  r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
  r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  return r;
}

// Rows [0, rows) of B then [rows, 2 rows) of C (a NULL tensor's rows are
// skipped).  Lane group j of a warp (LPR = N / 8 lanes) takes row
// r0 + u * RPW + j of pass u; kU passes' loads are issued before any
// reduction.  Whole warps iterate together so the shuffles see every lane.
// Rows stay contiguous in memory across a warp (streaming order); the weight
// and bias of a row's channels come through L1 / L2.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) bc_prep_kernel(int64_t rows, int N, int64_t grn,
                                                           const void* Braw, const void* Craw,
                                                           const float* wB, const float* bB,
                                                           const float* wC, const float* bC,
                                                           float eps, void* Bo, void* Co) {
  const int LPR = N / 8, RPW = 32 / LPR;  // lanes per row, rows per warp pass
  const int lane = threadIdx.x & 31, sub = lane % LPR;
  const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  const float inv_n = 1.f / (float)N;
  constexpr int kU = 4;
  const int64_t step = RPW * kU;
  for (int64_t r0 = warp * step; r0 < 2 * rows; r0 += nwarps * step) {
    Vec8 x[kU];
    float ss[kU];
    bool live[kU], isC[kU];
    int64_t off[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t row = r0 + u * RPW + lane / LPR;
      isC[u] = row >= rows;
      const int64_t rr = isC[u] ? row - rows : row;
      live[u] = row < 2 * rows && (isC[u] ? Craw : Braw) != nullptr;
      off[u] = rr * N + 8 * sub;
      ss[u] = 0.f;
      if (live[u]) x[u] = load8<BF16>(isC[u] ? Craw : Braw, off[u]);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (live[u]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) ss[u] = fmaf(x[u].v[j], x[u].v[j], ss[u]);
      }
      for (int o = LPR / 2; o > 0; o >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
      if (live[u]) {
        const float sc = rsqrtf(ss[u] * inv_n + eps);
        const int64_t ch = off[u] % grn;  // (group, rank, n) of the first value
        const Vec8 w = ld_param8(isC[u] ? wC : wB, ch, 1.f);
        const Vec8 b = ld_param8(isC[u] ? bC : bB, ch, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) x[u].v[j] = fmaf(x[u].v[j] * sc, w.v[j], b.v[j]);
        store8<BF16>(isC[u] ? Co : Bo, off[u], x[u]);
      }
    }
  }
}

}  // namespace

cudaError_t bc_prep_launch(int64_t tokens, int64_t N, int64_t gr, bool bf16, const void* Braw,
                           const void* Craw, const float* wB, const float* bB, const float* wC,
                           const float* bC, float eps, void* Bo, void* Co, cudaStream_t st) {
  const int64_t rows = tokens * gr;
  if (rows == 0) return cudaSuccess;
  const int64_t threads_needed = (2 * rows * (N / 8) + 3) / 4;  // four row groups per pass
  int64_t blocks = (threads_needed + kThreads - 1) / kThreads;
  const int64_t cap = 148 * 8;  // resident CTAs of 256 threads: 8 per SM
  if (blocks > cap) blocks = cap;
  if (bf16)
    bc_prep_kernel<true><<<(unsigned)blocks, kThreads, 0, st>>>(rows, (int)N, gr * N, Braw, Craw,
                                                                wB, bB, wC, bC, eps, Bo, Co);
  else
    bc_prep_kernel<false><<<(unsigned)blocks, kThreads, 0, st>>>(rows, (int)N, gr * N, Braw, Craw,
                                                                 wB, bB, wC, bC, eps, Bo, Co);
  return cudaGetLastError();
}

}  // namespace m3
