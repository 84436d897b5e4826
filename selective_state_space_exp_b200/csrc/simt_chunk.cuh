// simt_chunk.cuh -- per-chunk geometry and the chunk-local prefix sums shared
// by the CUDA-core forward scan and the backward pass.
#pragma once

#include "m3_internal.cuh"

namespace m3 {
namespace simt {

struct Geo {
  int64_t b, h, g, tg, c, t0;  // g: B/C group, tg: theta group, t0: first token of the chunk
  int64_t base, len;           // the sequence's first token (token dimension) and length
  int nt;                      // valid tokens in the chunk (0 past a short packed sequence)
};

__device__ __forceinline__ Geo chunk_geo(const ScanArgs& a, int64_t c) {
  Geo q;
  q.b = blockIdx.z;
  q.h = blockIdx.y;
  q.g = q.h / (a.nheads / a.ngroups);
  q.tg = q.h / (a.nheads / a.tgroups);
  q.c = c;
  q.t0 = c * a.Q;
  const Chain ch = chain_of(a, q.b);
  q.base = ch.base;
  q.len = ch.len;
  int64_t rem = ch.len - q.t0;
  q.nt = (int)(rem < 0 ? 0 : rem < a.Q ? rem : a.Q);
  return q;
}

// Bounds-checked builds: the chunk's batch, head and chunk indices and its
// token range lie inside the call's tensors (always true otherwise).
__device__ __forceinline__ bool geo_ok(const ScanArgs& a, const Geo& q) {
  return M3_IN(q.b, a.batch, a.status) && M3_IN(q.h, a.nheads, a.status) &&
         M3_IN(q.c, a.nchunks, a.status) &&
         (q.nt <= 0 || M3_IN(q.base + q.t0 + q.nt - 1, a.total_tokens, a.status));
}

// Chunk-local prefix sums and trapezoid weights into shared memory:
// lcum[Q], gam[Q], del[Q], dts[Q], phi[Q][K].
__device__ __forceinline__ void chunk_prep(const ScanArgs& a, const Geo& q, float* lcum, float* gam,
                           float* del, float* dts, float* phi) {
  const int K = (int)(a.N / 2);
  const int64_t H = a.nheads;
  for (int i = threadIdx.x; i < q.nt; i += blockDim.x) {
    const int64_t bt = q.base + q.t0 + i;
    const float dt = a.dt[bt * H + q.h], lam = a.lam[bt * H + q.h];
    float nxt = 0.f;
    if (q.t0 + i + 1 < q.len) nxt = (1.f - a.lam[(bt + 1) * H + q.h]) * a.dt[(bt + 1) * H + q.h];
    dts[i] = dt;
    gam[i] = lam * dt;
    del[i] = lam * dt + nxt;
    lcum[i] = dt * a.A[bt * H + q.h];
  }
  // the chunk's angle rates, one coalesced pass (the scan below reads them
  // from shared memory)
  for (int e = threadIdx.x; e < q.nt * K; e += blockDim.x) {
    const int i = e / K, k = e % K;
    phi[e] = a.theta[((q.base + q.t0 + i) * a.tgroups + q.tg) * K + k];
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // <= 64 sequential adds: the plain prefix sum
    float acc = 0.f;
    for (int i = 0; i < q.nt; ++i) {
      acc += lcum[i];
      lcum[i] = acc;
    }
  }
  // angle prefix sums, one pair per thread (threads from the second warp on,
  // beside thread 0's decay sum)
  const int first = blockDim.x > 32 ? 32 : 0;
  for (int k = (int)threadIdx.x - first; k < K; k += (int)blockDim.x - first) {
    if (k < 0) break;
    float acc = 0.f;
    for (int i = 0; i < q.nt; ++i) {
      acc = fmaf(dts[i], phi[i * K + k], acc);
      phi[i * K + k] = acc;
    }
  }
  __syncthreads();
}

}  // namespace simt
}  // namespace m3
