// scan_bwd_tc.cu -- steps 1 and 3 of the backward pass on the tensor cores
// (tcgen05.mma kind::f16: bf16 operands in 128-byte-swizzled shared memory,
// fp32 accumulators in TMEM), for the layer's shape: bf16 io, N = 128,
// P = 64, chunks of M = Q R = 64 rows (token, rank).
//
// The quantities and notation are those of the CUDA-core backward
// (scan_bwd.cu), which follows the chunked form of the exponential-
// trapezoidal recurrence (PaperWeekly page sections 2.1-2.3):
//   Bt = Rot(-Phi) B, Ct = Rot(-Phi) C        (chunk-local angles Phi)
//   M_ts = exp(Lam_t - Lam_s) delta_s (s < t), gamma_t (s = t), 0 (s > t)
//   w_s  = exp(Lam_end - Lam_s) delta_s
//   G_c  = the state entering chunk c,  dGhat = Rot(-Phi_end) dG_c+1.
//
// Step 1, per chunk: S_c = (w Bt)^T X and D_c = (exp(Lam) Ct)^T dY, two
// N x P products with K = M, each one MMA chain (M = 128 state rows).
//
// Step 3, per chunk, in two MMA phases around the mask:
//   phase A   S  = Ct Bt^T,  DX = dY X^T          (M x M, K = N and P)
//             AX = Bt dGhat                       (M x P, K = N)
//             AC = dY G_c^T, AB = X dGhat^T       (M x N, K = P)
//   between   the masked scores M o S, M o DX (bf16, to shared memory); the
//             mask's gradients (token pair t, s: dL/dM_ts summed over both
//             ranks, F_ts = dL/dM_ts exp(Lam_t - Lam_s)); beta_s = x_s . AX_s;
//             the exp(Lam_t) term of dLam, Ct_t . AC_t exp(Lam_t); then AC,
//             AB, AX scaled in TMEM by exp(Lam_t), w_s, w_s
//   phase B   AC += (M o DX) Bt      -> dCt = exp(Lam) dY G^T + (M o DX) Bt
//             AB += (M o DX)^T Ct    -> dBt = (M o DX)^T Ct + w X dGhat^T
//             AX += (M o S)^T dY     -> dX  = (M o S)^T dY + w Bt dGhat
// then the rotations back to B and C, the angle gradients and the backward
// of the chunk-local prefix sums, as on the CUDA cores.  G_c, dGhat and
// G_c+1 arrive as bf16 blocks in the MMA operand layout written by step 2
// (the first two by bulk copy into shared memory).  TMEM holds 448 of its
// 512 columns; the global loads of a chunk are staged before its TMEM is
// allocated, so a second CTA on the SM prepares its chunk while the first
// one computes.  Step 1 is persistent: three CTAs per SM walk the chunks.
#include <cuda_bf16.h>

#include "m3_internal.cuh"
#include "scan_bwd.cuh"
#include "simt_chunk.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

using namespace tc;
using simt::chunk_geo;
using simt::Geo;

constexpr int kN = 128;                 // dstate
constexpr int kP = 64;                  // headdim
constexpr int kK = kN / 2;              // rotation pairs
constexpr int kKP = kK + 1;             // row stride of the per-token angle arrays (odd:
                                        // 16 rows of one pair fall on 16 banks)
constexpr int kM = (int)kBwdTcRows;     // rows per chunk
constexpr int kTh = 256;
constexpr int kOPB = kM * 128;          // one [64 rows][128 B] operand block
constexpr float kL2E = 1.4426950408889634f;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier wait (2 s)

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Polls an mbarrier (one thread); false after recording M3_ERR_TIMEOUT.
__device__ bool wait_mma(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (now_ns() - t0 > kWaitNs) {
      if (status) atomicCAS(status, 0, (int)M3_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) {
  return d + (uint64_t)(bytes >> 4);
}

// 16 consecutive bf16 values of row `row` from column c0 (a multiple of 16)
// of a [rows][64] swizzled block, as floats.
__device__ __forceinline__ void ld16_sw(const uint8_t* blk, int row, int c0, float (&v)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 u = *reinterpret_cast<const uint4*>(blk + sw128_off(row, c0 / 8 + h));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16(w[j]);
      v[8 * h + 2 * j] = f.x;
      v[8 * h + 2 * j + 1] = f.y;
    }
  }
}

// Chunk-local prefix sums into shared memory: lcum[Q] (Lam), phi[Q][kKP]
// (Phi, padded rows), and the per-token gamma, delta, dt.  Each prefix sum
// (the decay and the K angle pairs) is one warp's inclusive scan over the
// chunk's tokens, Q / 32 tokens per lane.
template <int Q>
__device__ void prep_tc(const ScanArgs& a, const Geo& q, float* lcum, float* gam, float* del,
                        float* dts, float* phi) {
  const int64_t H = a.nheads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < q.nt; i += kTh) {
    const int64_t bt = q.base + q.t0 + i;
    const float dt = __ldg(a.dt + bt * H + q.h), lam = __ldg(a.lam + bt * H + q.h);
    float nxt = 0.f;
    if (q.t0 + i + 1 < q.len)
      nxt = (1.f - __ldg(a.lam + (bt + 1) * H + q.h)) * __ldg(a.dt + (bt + 1) * H + q.h);
    dts[i] = dt;
    gam[i] = lam * dt;
    del[i] = lam * dt + nxt;
    lcum[i] = dt * __ldg(a.A + bt * H + q.h);
  }
  {  // the chunk's angle rates: every load issued before the first store
    constexpr int PER = (Q * kK + kTh - 1) / kTh;
    float th[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = tid + j * kTh, i = e / kK, k = e % kK;
      th[j] = (e < q.nt * kK) ? __ldg(a.theta + ((q.base + q.t0 + i) * a.tgroups + q.tg) * kK + k)
                              : 0.f;
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = tid + j * kTh;
      if (e < q.nt * kK) phi[(e / kK) * kKP + e % kK] = th[j];
    }
  }
  __syncthreads();
  // column c of warp w: c = w + 8 j; the warp's columns are scanned together
  constexpr int TPL = Q > 32 ? Q / 32 : 1;  // tokens per lane
  constexpr int NW = kTh / 32, CPW = (kK + NW) / NW;  // columns 0..kK (kK: the decay)
  float v[CPW][TPL], run[CPW], incl[CPW];
#pragma unroll
  for (int j = 0; j < CPW; ++j) {
    const int col = warp + NW * j;
    run[j] = 0.f;
#pragma unroll
    for (int u = 0; u < TPL; ++u) {
      const int t = lane * TPL + u;
      float x = 0.f;
      if (col <= kK && t < q.nt) x = col < kK ? dts[t] * phi[t * kKP + col] : lcum[t];
      run[j] += x;
      v[j][u] = run[j];
    }
    incl[j] = run[j];
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1)
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const float y = __shfl_up_sync(0xffffffffu, incl[j], off);
      if (lane >= off) incl[j] += y;
    }
#pragma unroll
  for (int j = 0; j < CPW; ++j) {
    const int col = warp + NW * j;
    const float excl = incl[j] - run[j];
#pragma unroll
    for (int u = 0; u < TPL; ++u) {
      const int t = lane * TPL + u;
      if (col <= kK && t < q.nt) {
        if (col < kK) phi[t * kKP + col] = v[j][u] + excl;
        else lcum[t] = v[j][u] + excl;
      }
    }
  }
  __syncthreads();
}

// Sine and cosine of an angle of any size (reduced to about [-pi, pi] first).
__device__ __forceinline__ void sincos_r(float x, float* s, float* c) {
  __sincosf(reduce_2pi(x), s, c);
}

// Rows (token, rank) of a chunk: row i is token i / R, rank i % R.  Stages
// Rot(-Phi_t) of B and C (times the per-token scales sb, sc) for rows i with
// token t < nt, zeros beyond, as 2 K-major blocks of [64 rows][64 columns].
template <int R>
__device__ __forceinline__ void stage_bc(const ScanArgs& a, const Geo& q, const float* phi,
                                         const float* sb, const float* sc, uint8_t* bt,
                                         uint8_t* ct) {
  constexpr int PER = kM * 16 / kTh;
  uint4 rb[PER], rc[PER];  // every load issued before the first use
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = (int)threadIdx.x + j * kTh, i = e >> 4, c16 = e & 15, t = i / R, r = i % R;
    rb[j] = rc[j] = make_uint4(0u, 0u, 0u, 0u);
    if (t < q.nt) {
      const int64_t base = ((q.base + q.t0 + t) * a.ngroups + q.g) * R * kN + (int64_t)r * kN + 8 * c16;
      rb[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.B) + base));
      rc[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.C) + base));
    }
  }
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = (int)threadIdx.x + j * kTh, i = e >> 4, c16 = e & 15, t = i / R;
    uint32_t ob[4] = {0u, 0u, 0u, 0u}, oc[4] = {0u, 0u, 0u, 0u};
    if (t < q.nt) {
      const uint32_t wb[4] = {rb[j].x, rb[j].y, rb[j].z, rb[j].w};
      const uint32_t wc[4] = {rc[j].x, rc[j].y, rc[j].z, rc[j].w};
      const float fb = sb ? sb[t] : 1.f, fc = sc ? sc[t] : 1.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float sn, cs;
        sincos_r(phi[t * kKP + 4 * c16 + u], &sn, &cs);
        const float2 b = unpack_bf16(wb[u]), c = unpack_bf16(wc[u]);
        ob[u] = pack_bf16(fb * (cs * b.x + sn * b.y), fb * (-sn * b.x + cs * b.y));
        oc[u] = pack_bf16(fc * (cs * c.x + sn * c.y), fc * (-sn * c.x + cs * c.y));
      }
    }
    const uint32_t off = (c16 >> 3) * kOPB + sw128_off(i, c16 & 7);
    *reinterpret_cast<uint4*>(bt + off) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    *reinterpret_cast<uint4*>(ct + off) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
  }
}

// x and dy rows as one K-major [64 rows][64 columns] block each.
template <int R>
__device__ __forceinline__ void stage_xdy(const ScanArgs& a, const BwdArgs& g, const Geo& q,
                                          uint8_t* xs, uint8_t* dys) {
  constexpr int PER = kM * 8 / kTh;
  uint4 rx[PER], ry[PER], ry2[PER];  // ry2: the second half of an fp32 dy row piece
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = (int)threadIdx.x + j * kTh, i = e >> 3, c8 = e & 7, t = i / R, r = i % R;
    rx[j] = ry[j] = ry2[j] = make_uint4(0u, 0u, 0u, 0u);
    if (t < q.nt) {
      const int64_t o = ((q.base + q.t0 + t) * a.nheads + q.h) * R * kP + (int64_t)r * kP + 8 * c8;
      rx[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.x) + o));
      if (g.dy_f32) {
        const uint4* py = reinterpret_cast<const uint4*>(static_cast<const float*>(g.dy) + o);
        ry[j] = __ldg(py);
        ry2[j] = __ldg(py + 1);
      } else {
        ry[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g.dy) + o));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = (int)threadIdx.x + j * kTh, i = e >> 3, c8 = e & 7;
    uint4 yv = ry[j];
    if (g.dy_f32)  // eight fp32 values -> bf16
      yv = make_uint4(pack_bf16(__uint_as_float(ry[j].x), __uint_as_float(ry[j].y)),
                      pack_bf16(__uint_as_float(ry[j].z), __uint_as_float(ry[j].w)),
                      pack_bf16(__uint_as_float(ry2[j].x), __uint_as_float(ry2[j].y)),
                      pack_bf16(__uint_as_float(ry2[j].z), __uint_as_float(ry2[j].w)));
    *reinterpret_cast<uint4*>(xs + sw128_off(i, c8)) = rx[j];
    *reinterpret_cast<uint4*>(dys + sw128_off(i, c8)) = yv;
  }
}

// A chunk's raw B, C, x and dy pieces in registers, loaded ahead of their use
// (the loads of a chunk are in flight while its prefix sums run), then
// rotated and staged as stage_bc and stage_xdy do.
template <int R>
struct RawChunk {
  static constexpr int PB = kM * 16 / kTh, PX = kM * 8 / kTh;
  uint4 b[PB], c[PB], x[PX], y[PX], y2[PX];

  __device__ __forceinline__ void load(const ScanArgs& a, const BwdArgs& g, const Geo& q) {
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      const int e = (int)threadIdx.x + j * kTh, i = e >> 4, c16 = e & 15, t = i / R, r = i % R;
      b[j] = c[j] = make_uint4(0u, 0u, 0u, 0u);
      if (t < q.nt) {
        const int64_t base =
            ((q.base + q.t0 + t) * a.ngroups + q.g) * R * kN + (int64_t)r * kN + 8 * c16;
        b[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.B) + base));
        c[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.C) + base));
      }
    }
#pragma unroll
    for (int j = 0; j < PX; ++j) {
      const int e = (int)threadIdx.x + j * kTh, i = e >> 3, c8 = e & 7, t = i / R, r = i % R;
      x[j] = y[j] = y2[j] = make_uint4(0u, 0u, 0u, 0u);
      if (t < q.nt) {
        const int64_t o = ((q.base + q.t0 + t) * a.nheads + q.h) * R * kP + (int64_t)r * kP + 8 * c8;
        x[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.x) + o));
        if (g.dy_f32) {
          const uint4* py = reinterpret_cast<const uint4*>(static_cast<const float*>(g.dy) + o);
          y[j] = __ldg(py);
          y2[j] = __ldg(py + 1);
        } else {
          y[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g.dy) + o));
        }
      }
    }
  }

  // Rot(-Phi_t) B and C (unscaled) into 2 K-major blocks each; x, dy into one.
  __device__ __forceinline__ void stage(const BwdArgs& g, const Geo& q, const float* phi,
                                        uint8_t* bt, uint8_t* ct, uint8_t* xs, uint8_t* dys) const {
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      const int e = (int)threadIdx.x + j * kTh, i = e >> 4, c16 = e & 15, t = i / R;
      uint32_t ob[4] = {0u, 0u, 0u, 0u}, oc[4] = {0u, 0u, 0u, 0u};
      if (t < q.nt) {
        const uint32_t wb[4] = {b[j].x, b[j].y, b[j].z, b[j].w};
        const uint32_t wc[4] = {c[j].x, c[j].y, c[j].z, c[j].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float sn, cs;
          sincos_r(phi[t * kKP + 4 * c16 + u], &sn, &cs);
          const float2 bf = unpack_bf16(wb[u]), cf = unpack_bf16(wc[u]);
          ob[u] = pack_bf16(cs * bf.x + sn * bf.y, -sn * bf.x + cs * bf.y);
          oc[u] = pack_bf16(cs * cf.x + sn * cf.y, -sn * cf.x + cs * cf.y);
        }
      }
      const uint32_t off = (c16 >> 3) * kOPB + sw128_off(i, c16 & 7);
      *reinterpret_cast<uint4*>(bt + off) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
      *reinterpret_cast<uint4*>(ct + off) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
    }
#pragma unroll
    for (int j = 0; j < PX; ++j) {
      const int e = (int)threadIdx.x + j * kTh, i = e >> 3, c8 = e & 7;
      uint4 yv = y[j];
      if (g.dy_f32)  // eight fp32 values -> bf16
        yv = make_uint4(pack_bf16(__uint_as_float(y[j].x), __uint_as_float(y[j].y)),
                        pack_bf16(__uint_as_float(y[j].z), __uint_as_float(y[j].w)),
                        pack_bf16(__uint_as_float(y2[j].x), __uint_as_float(y2[j].y)),
                        pack_bf16(__uint_as_float(y2[j].z), __uint_as_float(y2[j].w)));
      *reinterpret_cast<uint4*>(xs + sw128_off(i, c8)) = x[j];
      *reinterpret_cast<uint4*>(dys + sw128_off(i, c8)) = yv;
    }
  }
};

// ---- step 1: S_c and D_c ----------------------------------------------------
// Shared memory: w Bt (2 blocks), exp(Lam) Ct (2 blocks), x, dy (1 block
// each), then the prefix sums.  TMEM: S_c in columns 0-63, D_c in 64-127,
// lane n = state row n.
struct SumsSmem {
  static constexpr int WB = 0, EC = 2 * kOPB, XS = 4 * kOPB, DYS = 5 * kOPB;
  static constexpr int SMALL = 6 * kOPB;
  static constexpr int bytes(int Q) { return SMALL + (Q * kKP + 6 * Q) * 4 + 32; }
};

// Chunk c of chain (b, h): its tokens and groups.
__device__ __forceinline__ Geo geo_at(const ScanArgs& a, int64_t b, int64_t h, int64_t c) {
  Geo q;
  q.b = b;
  q.h = h;
  q.g = h / (a.nheads / a.ngroups);
  q.tg = h / (a.nheads / a.tgroups);
  q.c = c;
  q.t0 = c * a.Q;
  const Chain ch = chain_of(a, b);
  q.base = ch.base;
  q.len = ch.len;
  const int64_t rem = ch.len - q.t0;
  q.nt = (int)(rem < 0 ? 0 : rem < a.Q ? rem : a.Q);
  return q;
}

// Persistent: CTA i takes chunks i, i + gridDim.x, ... of all chains (index
// (b H + h) nc + c), keeping its TMEM columns for the whole run.
template <int R>
__global__ void __launch_bounds__(kTh, 3) bwd_tc_sums_kernel(const ScanArgs a, const BwdArgs g,
                                                             const BwdWs w) {
  constexpr int Q = kM / R;
  using L = SumsSmem;
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {
    if (tid == 0 && a.status) atomicCAS(a.status, 0, (int)M3_ERR_CUDA);
    return;
  }
  float* phi = reinterpret_cast<float*>(sm + L::SMALL);
  float* lcum = phi + Q * kKP;
  float* gam = lcum + Q;
  float* del = gam + Q;
  float* dts = del + Q;
  float* s_w = dts + Q;  // w_s, the row scale of Bt
  float* s_e = s_w + Q;  // exp(Lam_t), the row scale of Ct
  // 8-byte aligned: 71 Q floats (Q even) before it
  uint64_t* bar = reinterpret_cast<uint64_t*>(s_e + Q);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar + 1);
  if (warp == 0) {
    tmem_alloc(s_tmem, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const uint64_t dWB = sw128_desc(sbase + L::WB, kOPB, 1024);
  const uint64_t dEC = sw128_desc(sbase + L::EC, kOPB, 1024);
  const uint64_t dXS = sw128_desc(sbase + L::XS, kOPB, 1024);
  const uint64_t dDY = sw128_desc(sbase + L::DYS, kOPB, 1024);
  const int64_t total = a.batch * a.nheads * a.nchunks;
  uint32_t phase = 0;
  bool aborted = false;
  for (int64_t it = blockIdx.x; it < total && !aborted; it += gridDim.x) {
    const int64_t bh = it / a.nchunks;
    const Geo q = geo_at(a, bh / a.nheads, bh % a.nheads, it % a.nchunks);
    if (!simt::geo_ok(a, q)) continue;  // uniform over the block
    float* S = w.G + it * (int64_t)kN * kP;  // turned into G_c by the state pass
    float* D = w.D + it * (int64_t)kN * kP;
    float* su = w.sums + it * (1 + kN);
    if (q.nt <= 0) {  // past a short packed sequence: both states pass unchanged
      for (int e = tid; e < kN * kP / 4; e += kTh) {
        reinterpret_cast<float4*>(S)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(D)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int k = tid; k < 1 + kN; k += kTh) su[k] = (k == 0 || (k & 1)) ? 1.f : 0.f;
      continue;  // uniform over the block
    }
    prep_tc<Q>(a, q, lcum, gam, del, dts, phi);
    const float lend = lcum[q.nt - 1];
    for (int i = tid; i < Q; i += kTh) {
      s_w[i] = i < q.nt ? expf(lend - lcum[i]) * del[i] : 0.f;
      s_e[i] = i < q.nt ? expf(lcum[i]) : 0.f;
    }
    __syncthreads();
    stage_bc<R>(a, q, phi, s_w, s_e, sm + L::WB, sm + L::EC);
    stage_xdy<R>(a, g, q, sm + L::XS, sm + L::DYS);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      // M = 128 state rows (MN-major A: rows i of the chunk are K), N = 64
      const uint32_t id = idesc_bf16(kN, kP, 1, 1);
#pragma unroll
      for (int ks = 0; ks < kM / 16; ++ks)
        mma_bf16_ss(tm, dadd(dWB, ks * 2048), dadd(dXS, ks * 2048), id, ks != 0);
#pragma unroll
      for (int ks = 0; ks < kM / 16; ++ks)
        mma_bf16_ss(tm + kP, dadd(dEC, ks * 2048), dadd(dDY, ks * 2048), id, ks != 0);
      mma_commit(bar);
    }
    const bool ok = (tid == 0) ? wait_mma(bar, phase, a.status) : true;
    phase ^= 1;
    aborted = __syncthreads_or(!ok);
    tc_fence_after();
    if (!aborted) {
      // S_c, then D_c, through a 32 KB staging block over the consumed operands:
      // thread row n = 32 (warp % 4) + lane, column half warp / 4; float4 j of
      // row n sits in slot (j + n) mod 16 of the row (no bank conflicts either
      // way), then all threads write the matrix out in contiguous 16-byte pieces.
      const int qd = warp & 3, hf = warp >> 2;
      const int n = 32 * qd + lane;
      float* stg = reinterpret_cast<float*>(sm + L::WB);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        uint32_t v[32];
        tmem_ld32(tm + ((uint32_t)(32 * qd) << 16) + which * kP + 32 * hf, v);
        tmem_ld_wait();
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const int j = 8 * hf + j4;
          *reinterpret_cast<float4*>(stg + n * kP + ((j + n) & 15) * 4) =
              make_float4(__uint_as_float(v[4 * j4]), __uint_as_float(v[4 * j4 + 1]),
                          __uint_as_float(v[4 * j4 + 2]), __uint_as_float(v[4 * j4 + 3]));
        }
        __syncthreads();
        float4* dst = reinterpret_cast<float4*>(which ? D : S);
#pragma unroll
        for (int it = 0; it < kN * kP / 4 / kTh; ++it) {
          const int e = tid + it * kTh, r = e >> 4, j = e & 15;
          dst[e] = *reinterpret_cast<const float4*>(stg + r * kP + ((j + r) & 15) * 4);
        }
        __syncthreads();
      }
      if (tid == 0) su[0] = expf(lend);
      for (int k = tid; k < kK; k += kTh) {
        float sn, cs;
        sincosf(phi[(q.nt - 1) * kKP + k], &sn, &cs);
        su[1 + 2 * k] = cs;
        su[2 + 2 * k] = sn;
      }
    }
    // TMEM read and shared memory free before the next chunk
    tc_fence_before();
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 128);
}

// ---- step 3: per-chunk gradients ---------------------------------------------
// Shared memory (bytes):
//   CT, BT   Ct, Bt: 2 K-major blocks each
//   XS, DYS  x, dy: 1 block each
//   GM       G_c in bf16, [128 rows n][64 p]; after phase A: M o S, M o DX
//   DG       dGhat in bf16, [128 rows n][64 p]; after phase A: dPhi, fp32 [Q][kKP]
//   SMALL    Phi [Q][kKP], per-token arrays, end-angle cos / sin, barriers
template <int Q>
struct ChunkTc {
  static constexpr int CT = 0, BT = 2 * kOPB, XS = 4 * kOPB, DYS = 5 * kOPB;
  static constexpr int GM = 6 * kOPB, MS = GM, MD = GM + kOPB;
  static constexpr int DG = GM + kN * 128;
  static constexpr int DG_BYTES =
      ((Q * kKP * 4 > kN * 128 ? Q * kKP * 4 : kN * 128) + 1023) / 1024 * 1024;
  static constexpr int SMALL = DG + DG_BYTES;
  static constexpr int NTOK = 12;  // per-token float arrays
  // the barriers follow 77 Q + 96 floats (Q even): 8-byte aligned
  static constexpr int bytes() {
    return SMALL + (Q * kKP + NTOK * Q + kK + 32) * 4 + 32;
  }
  // TMEM columns
  static constexpr int S_COL = 0, DX_COL = 64, AX_COL = 128, AC_COL = 192, AB_COL = 320;
  static constexpr int TMEM_COLS = 512;
};

template <int R>
__global__ void __launch_bounds__(kTh, 2) bwd_tc_chunk_kernel(const ScanArgs a, const BwdArgs g,
                                                              const BwdWs w) {
  constexpr int Q = kM / R;
  using L = ChunkTc<Q>;
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sbase = smem_u32(sm);
  const Geo q = chunk_geo(a, blockIdx.x);
  const int nt = q.nt;
  if (nt <= 0 || !simt::geo_ok(a, q)) return;  // uniform over the block
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {
    if (tid == 0 && a.status) atomicCAS(a.status, 0, (int)M3_ERR_CUDA);
    return;
  }
  const int64_t H = a.nheads;
  float* phi = reinterpret_cast<float*>(sm + L::SMALL);
  float* lcum = phi + Q * kKP;
  float* gam = lcum + Q;
  float* del = gam + Q;
  float* dts = del + Q;
  float* lg = dts + Q;     // Lam_t log2(e)
  float* wv = lg + Q;      // w_s
  float* beta = wv + Q;    // x_s . (Bt dGhat)_s over the ranks
  float* dLam = beta + Q;
  float* dgam = dLam + Q;
  float* ddel = dgam + Q;
  float* colF = ddel + Q;  // sum over t > s of F_ts
  float* thT = colF + Q;   // sum_k theta_k d(dt theta)_k
  float* s_pe = thT + Q;   // the outgoing rotation's angle gradient, [K]
  float* red = s_pe + kK;
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 32);  // phase A, phase B, G / dGhat copy
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 3);
  float* dPhi = reinterpret_cast<float*>(sm + L::DG);  // after phase A
  const int64_t cidx = (q.b * H + q.h) * a.nchunks + q.c;
  const int64_t gbi = (q.b * H + q.h) * (a.nchunks + 1) + q.c;  // G_c's block

  // ---- prologue: operand blocks of the state pass in flight, prefix sums,
  // rotated operands (all before TMEM is taken) --------------------------------
  if (tid == 0) {
    mbar_init(bars, 1);
    mbar_init(bars + 1, 1);
    mbar_init(bars + 2, 1);
    fence_mbar_init();
    mbar_expect_tx(bars + 2, 2 * kN * kP * 2);
    bulk_load(sm + L::GM, w.Gb + gbi * kN * kP * 2, kN * kP * 2, bars + 2);
    bulk_load(sm + L::DG, w.Hb + cidx * (int64_t)kN * kP * 2, kN * kP * 2, bars + 2);
  }
  // G_c+1 (the next block of the chain: the next chunk's start state, or the
  // final state), for the outgoing rotation's angle gradient.  Item e = (pair
  // k, logical 16-byte chunk u of P): rows 2k and 2k + 1 at u's swizzled place.
  constexpr int kItems = kK * 8 / kTh;
  uint4 gn[kItems][2];
#pragma unroll
  for (int j = 0; j < kItems; ++j) {
    const int e = tid + j * kTh, k = e >> 3, u = e & 7;
    const uint8_t* nb = w.Gb + (gbi + 1) * kN * kP * 2;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = 2 * k + r;
      gn[j][r] = __ldg(reinterpret_cast<const uint4*>(nb + sw128_off(row, u)));
    }
  }
  RawChunk<R> raw;
  raw.load(a, g, q);  // in flight during the prefix sums
  prep_tc<Q>(a, q, lcum, gam, del, dts, phi);
  const int t1 = nt - 1;
  const float lam_end = lcum[t1];
  for (int i = tid; i < Q; i += kTh) {
    wv[i] = (i < nt) ? expf(lam_end - lcum[i]) * del[i] : 0.f;
    lg[i] = (i < nt) ? lcum[i] * kL2E : 0.f;
    beta[i] = dLam[i] = dgam[i] = ddel[i] = colF[i] = thT[i] = 0.f;
  }
  __syncthreads();
  raw.stage(g, q, phi, sm + L::BT, sm + L::CT, sm + L::XS, sm + L::DYS);
  fence_async_smem();
  const bool okc = (tid == 0) ? wait_mma(bars + 2, 0, a.status) : true;
  if (warp == 0) {
    tmem_alloc(s_tmem, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  bool aborted = __syncthreads_or(!okc);
  tc_fence_after();
  {
    // <dGhat, G_c> and, per pair k, sum_p (dG1 G'0 - dG0 G'1) with dG =
    // Rot(Phi_end) dGhat and G' = G_c+1 (the angle gradient of the chunk's
    // outgoing rotation), from the bf16 blocks
    float dgg = 0.f;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int e = tid + j * kTh, k = e >> 3, u = e & 7;
      float sn, cs;
      sincos_r(phi[t1 * kKP + k], &sn, &cs);
      float gv[2][8], hv[2][8], nv[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint32_t off = sw128_off(2 * k + r, u);
        const uint4 gu = *reinterpret_cast<const uint4*>(sm + L::GM + off);
        const uint4 hu = *reinterpret_cast<const uint4*>(sm + L::DG + off);
        const uint32_t gw[4] = {gu.x, gu.y, gu.z, gu.w}, hw[4] = {hu.x, hu.y, hu.z, hu.w};
        const uint32_t nw[4] = {gn[j][r].x, gn[j][r].y, gn[j][r].z, gn[j][r].w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float2 gf = unpack_bf16(gw[v]), hf = unpack_bf16(hw[v]), nf = unpack_bf16(nw[v]);
          gv[r][2 * v] = gf.x; gv[r][2 * v + 1] = gf.y;
          hv[r][2 * v] = hf.x; hv[r][2 * v + 1] = hf.y;
          nv[r][2 * v] = nf.x; nv[r][2 * v + 1] = nf.y;
        }
      }
      float cr = 0.f;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        dgg = fmaf(hv[0][v], gv[0][v], fmaf(hv[1][v], gv[1][v], dgg));
        const float o0 = cs * hv[0][v] - sn * hv[1][v], o1 = sn * hv[0][v] + cs * hv[1][v];
        cr = fmaf(o1, nv[0][v], fmaf(-o0, nv[1][v], cr));
      }
      // the 8 chunks of pair k are 8 consecutive lanes
      cr += __shfl_xor_sync(0xffffffffu, cr, 1);
      cr += __shfl_xor_sync(0xffffffffu, cr, 2);
      cr += __shfl_xor_sync(0xffffffffu, cr, 4);
      if (u == 0) s_pe[k] = cr;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dgg += __shfl_xor_sync(0xffffffffu, dgg, off);
    if (lane == 0) red[warp] = dgg;
  }
  const uint32_t tm = *s_tmem;

  const uint64_t kCT = sw128_desc(sbase + L::CT, 16, 1024), mCT = sw128_desc(sbase + L::CT, kOPB, 1024);
  const uint64_t kBT = sw128_desc(sbase + L::BT, 16, 1024), mBT = sw128_desc(sbase + L::BT, kOPB, 1024);
  const uint64_t kXS = sw128_desc(sbase + L::XS, 16, 1024);
  const uint64_t kDY = sw128_desc(sbase + L::DYS, 16, 1024), mDY = sw128_desc(sbase + L::DYS, kOPB, 1024);
  const uint64_t kGM = sw128_desc(sbase + L::GM, 16, 1024);
  const uint64_t kDG = sw128_desc(sbase + L::DG, 16, 1024), mDG = sw128_desc(sbase + L::DG, kN * 128, 1024);
  const uint64_t kMD = sw128_desc(sbase + L::MD, 16, 1024), mMD = sw128_desc(sbase + L::MD, kOPB, 1024);
  const uint64_t mMS = sw128_desc(sbase + L::MS, kOPB, 1024);

  // ---- phase A ----------------------------------------------------------------
  if (!aborted && tid == 0) {
    const uint32_t id64 = idesc_bf16(kM, 64, 0, 0), id128 = idesc_bf16(kM, 128, 0, 0);
    const uint32_t idAX = idesc_bf16(kM, kP, 0, 1);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {  // S = Ct Bt^T, K = N
        const uint32_t o = kb * kOPB + k4 * 32;
        mma_bf16_ss(tm + L::S_COL, dadd(kCT, o), dadd(kBT, o), id64, (kb | k4) != 0);
      }
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4)  // DX = dY X^T, K = P
      mma_bf16_ss(tm + L::DX_COL, dadd(kDY, k4 * 32), dadd(kXS, k4 * 32), id64, k4 != 0);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)  // AX = Bt dGhat, K = N (dGhat MN-major)
        mma_bf16_ss(tm + L::AX_COL, dadd(kBT, kb * kOPB + k4 * 32), dadd(mDG, (kb * 4 + k4) * 2048),
                    idAX, (kb | k4) != 0);
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {  // AC = dY G^T, AB = X dGhat^T, K = P
      mma_bf16_ss(tm + L::AC_COL, dadd(kDY, k4 * 32), dadd(kGM, k4 * 32), id128, k4 != 0);
      mma_bf16_ss(tm + L::AB_COL, dadd(kXS, k4 * 32), dadd(kDG, k4 * 32), id128, k4 != 0);
    }
    mma_commit(bars);
  }
  bool ok = (!aborted && tid == 0) ? wait_mma(bars, 0, a.status) : true;
  aborted = __syncthreads_or(aborted || !ok);
  tc_fence_after();

  // Thread layout over 64-row accumulators: warp w reads TMEM lanes
  // 32 (w % 4) .. +15 (rows 16 (w % 4) .. +15); warps w and w + 4 split the
  // columns (hh = w / 4), and the half-warps split a warp's columns again.
  const int qd = warp & 3, hh = warp >> 2, hl = lane >> 4;
  const int rho = 16 * qd + (lane & 15);
  const int tr = rho / R, rr = rho % R;
  const bool trow = tr < nt;
  const uint32_t lb = tm + ((uint32_t)(32 * qd) << 16);
  const int c64 = 32 * hh + 16 * hl;  // this thread's 16 columns of a 64-column accumulator

  if (!aborted) {
    // (1) the mask, its gradients and the masked scores
    {
      uint32_t sv[16], dv[16];
      tmem_ld16x2<16>(lb + L::S_COL + 32 * hh, sv);
      tmem_ld16x2<16>(lb + L::DX_COL + 32 * hh, dv);
      tmem_ld_wait();
      const float lgt = trow ? lg[tr] : 0.f;
      float rowacc = 0.f, dg = 0.f, colv[16];
      uint32_t pks[8], pkd[8];
#pragma unroll
      for (int jj = 0; jj < 16; jj += 2) {
        float msv[2], mdv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int s = (c64 + jj + u) / R;
          const float sv_ = __uint_as_float(sv[jj + u]), dv_ = __uint_as_float(dv[jj + u]);
          const float p = sv_ * dv_;
          float m = 0.f, F = 0.f;
          if (trow) {
            if (s < tr) {
              const float e = ex2(lgt - lg[s]);
              F = p * e;
              rowacc = fmaf(F, del[s], rowacc);
              m = e * del[s];
            } else if (s == tr) {
              dg += p;
              m = gam[tr];
            }
          }
          colv[jj + u] = F;
          msv[u] = sv_ * m;
          mdv[u] = dv_ * m;
        }
        pks[jj / 2] = pack_bf16(msv[0], msv[1]);
        pkd[jj / 2] = pack_bf16(mdv[0], mdv[1]);
      }
      *reinterpret_cast<uint4*>(sm + L::MS + sw128_off(rho, c64 / 8)) = make_uint4(pks[0], pks[1], pks[2], pks[3]);
      *reinterpret_cast<uint4*>(sm + L::MS + sw128_off(rho, c64 / 8 + 1)) = make_uint4(pks[4], pks[5], pks[6], pks[7]);
      *reinterpret_cast<uint4*>(sm + L::MD + sw128_off(rho, c64 / 8)) = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
      *reinterpret_cast<uint4*>(sm + L::MD + sw128_off(rho, c64 / 8 + 1)) = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
      // row terms: the two half-warps hold the same rows
      rowacc += __shfl_xor_sync(0xffffffffu, rowacc, 16);
      dg += __shfl_xor_sync(0xffffffffu, dg, 16);
      if (hl == 0 && trow) {
        if (rowacc != 0.f) atomicAdd(dLam + tr, rowacc);
        if (dg != 0.f) atomicAdd(dgam + tr, dg);
      }
      // column terms: reduce the 16 rows of a half-warp, one column per lane
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
          const float send = up ? colv[i] : colv[i + off];
          const float keep = up ? colv[i + off] : colv[i];
          colv[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      const int sc_ = (c64 + (lane & 15)) / R;
      if (sc_ < nt && colv[0] != 0.f) atomicAdd(colF + sc_, colv[0]);
    }
    // (2) beta from AX = Bt dGhat; AX *= w_s
    {
      uint32_t v[16];
      tmem_ld16x2<16>(lb + L::AX_COL + 32 * hh, v);
      tmem_ld_wait();
      float xr[16];
      ld16_sw(sm + L::XS, rho, c64, xr);
      float bt = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) bt = fmaf(xr[j], __uint_as_float(v[j]), bt);
      bt += __shfl_xor_sync(0xffffffffu, bt, 16);
      if (hl == 0 && trow) atomicAdd(beta + tr, bt);
      const float ws = trow ? wv[tr] : 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * ws);
      tmem_st16x2<16>(lb + L::AX_COL + 32 * hh, v);
    }
    // (3) AC = dY G^T: the exp(Lam_t) term of dLam; AC *= exp(Lam_t).
    // (4) AB = X dGhat^T: AB *= w_s.  128 columns: two 32-column loads per warp.
    {
      const float el = trow ? ex2(lg[tr]) : 0.f;
      const float ws = trow ? wv[tr] : 0.f;
      float cdot = 0.f;
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        const int col = 64 * hh + 32 * pc;  // the warp's 32 columns; this thread's 16 from col + 16 hl
        const int n0 = col + 16 * hl;
        uint32_t v[16];
        tmem_ld16x2<16>(lb + L::AC_COL + col, v);
        tmem_ld_wait();
        float cr[16];
        ld16_sw(sm + L::CT + (n0 >> 6) * kOPB, rho, n0 & 63, cr);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float x = __uint_as_float(v[j]);
          cdot = fmaf(cr[j], x, cdot);
          v[j] = __float_as_uint(x * el);
        }
        tmem_st16x2<16>(lb + L::AC_COL + col, v);
        uint32_t u[16];
        tmem_ld16x2<16>(lb + L::AB_COL + col, u);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * ws);
        tmem_st16x2<16>(lb + L::AB_COL + col, u);
      }
      cdot += __shfl_xor_sync(0xffffffffu, cdot, 16);
      if (hl == 0 && trow) atomicAdd(dLam + tr, el * cdot);
    }
    // dPhi goes over dGhat, which phase A has read
    for (int i = tid; i < Q * kKP; i += kTh) dPhi[i] = 0.f;
    tmem_st_wait();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- phase B ----------------------------------------------------------------
  if (!aborted && tid == 0) {
    const uint32_t idC = idesc_bf16(kM, 128, 0, 1), idB = idesc_bf16(kM, 128, 1, 1);
    const uint32_t idX = idesc_bf16(kM, kP, 1, 1);
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {  // K = the chunk's 64 rows
      // AC += (M o DX) Bt: A K-major [t][s], B MN-major (rows s, N = n)
      mma_bf16_ss(tm + L::AC_COL, dadd(kMD, k4 * 32), dadd(mBT, k4 * 2048), idC, 1);
      // AB += (M o DX)^T Ct: A MN-major (rows t, M = s), B MN-major (rows t, N = n)
      mma_bf16_ss(tm + L::AB_COL, dadd(mMD, k4 * 2048), dadd(mCT, k4 * 2048), idB, 1);
      // AX += (M o S)^T dY
      mma_bf16_ss(tm + L::AX_COL, dadd(mMS, k4 * 2048), dadd(mDY, k4 * 2048), idX, 1);
    }
    mma_commit(bars + 1);
  }
  if (!aborted) {
    ok = (tid == 0) ? wait_mma(bars + 1, 0, a.status) : true;
    aborted = __syncthreads_or(!ok);
    tc_fence_after();
  }

  // ---- epilogue: dC, dB (rotated back), their angle gradients, dx ----------------
  if (!aborted) {
    const int64_t tok = q.base + q.t0 + tr;
    const int64_t bcb = (tok * a.ngroups + q.g) * R * kN + (int64_t)rr * kN;
#pragma unroll
    for (int pc = 0; pc < 2; ++pc) {
      const int col = 64 * hh + 32 * pc;  // the warp's 32 columns; this thread's 16 from n0
      const int n0 = col + 16 * hl;
      uint32_t vc[16], vb[16];
      tmem_ld16x2<16>(lb + L::AC_COL + col, vc);
      tmem_ld16x2<16>(lb + L::AB_COL + col, vb);
      tmem_ld_wait();
      float dph[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) dph[j] = 0.f;
      if (trow) {
        float oc[16], ob[16], rc[16], rb[16];
        ld16_sw(sm + L::CT + (n0 >> 6) * kOPB, rho, n0 & 63, oc);
        ld16_sw(sm + L::BT + (n0 >> 6) * kOPB, rho, n0 & 63, ob);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float c0 = __uint_as_float(vc[2 * j]), c1 = __uint_as_float(vc[2 * j + 1]);
          const float b0 = __uint_as_float(vb[2 * j]), b1 = __uint_as_float(vb[2 * j + 1]);
          // angle gradient of the rotations of C and B (pair n0 / 2 + j)
          dph[j] = c0 * oc[2 * j + 1] - c1 * oc[2 * j] + b0 * ob[2 * j + 1] - b1 * ob[2 * j];
          float sn, cs;
          sincos_r(phi[tr * kKP + n0 / 2 + j], &sn, &cs);
          rc[2 * j] = cs * c0 - sn * c1;  // Rot(Phi_t) of the rotated-frame gradients
          rc[2 * j + 1] = sn * c0 + cs * c1;
          rb[2 * j] = cs * b0 - sn * b1;
          rb[2 * j + 1] = sn * b0 + cs * b1;
        }
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          atomicAdd(reinterpret_cast<float4*>(g.dC + bcb + n0 + j),
                    make_float4(rc[j], rc[j + 1], rc[j + 2], rc[j + 3]));
          atomicAdd(reinterpret_cast<float4*>(g.dB + bcb + n0 + j),
                    make_float4(rb[j], rb[j + 1], rb[j + 2], rb[j + 3]));
        }
      }
      // the R rows of a token are R consecutive lanes: one shared-memory add
      // per token and pair
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = dph[j];
#pragma unroll
        for (int off = 1; off < R; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (trow && (lane % R) == 0) atomicAdd(dPhi + tr * kKP + n0 / 2 + j, v);
      }
    }
    {  // dX, staged over the masked scores (phase B has read them): float4 j of
       // row i in slot (j + i) mod 16, written out once TMEM is released
      uint32_t v[16];
      tmem_ld16x2<16>(lb + L::AX_COL + 32 * hh, v);
      tmem_ld_wait();
      float* stg = reinterpret_cast<float*>(sm + L::GM);
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const int j = c64 / 4 + j4;
        *reinterpret_cast<float4*>(stg + rho * kP + ((j + rho) & 15) * 4) =
            make_float4(__uint_as_float(v[4 * j4]), __uint_as_float(v[4 * j4 + 1]),
                        __uint_as_float(v[4 * j4 + 2]), __uint_as_float(v[4 * j4 + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, L::TMEM_COLS);
  if (aborted) return;
  {  // dx of the chunk's tokens: a token's R rows are contiguous, 16-byte pieces
    const float* stg = reinterpret_cast<const float*>(sm + L::GM);
#pragma unroll
    for (int e0 = 0; e0 < kM * 16; e0 += kTh) {
      const int e = e0 + tid, i = e >> 4, j = e & 15, t = i / R, r = i % R;
      if (t < nt) {
        float* dxo = g.dx + ((q.base + q.t0 + t) * H + q.h) * R * kP + (int64_t)r * kP + 4 * j;
        *reinterpret_cast<float4*>(dxo) =
            *reinterpret_cast<const float4*>(stg + i * kP + ((j + i) & 15) * 4);
      }
    }
  }

  // ---- the scalar gradients (as on the CUDA cores) ----------------------------
  for (int k = tid; k < kK; k += kTh) dPhi[t1 * kKP + k] += s_pe[k];
  for (int u = tid; u < nt; u += kTh) {
    float dl = -wv[u] * beta[u] - del[u] * colF[u];
    if (u == t1) {
      float dsum = 0.f, wb = 0.f;
      for (int i = 0; i < kTh / 32; ++i) dsum += red[i];
      for (int s = 0; s < nt; ++s) wb = fmaf(wv[s], beta[s], wb);
      dl += wb + expf(lam_end) * dsum;
    }
    dLam[u] += dl;
    ddel[u] += expf(lam_end - lcum[u]) * beta[u] + colF[u];
  }
  __syncthreads();
  // Suffix sums over the chunk's tokens, one warp's scan per column: of dPhi
  // (they are d(dt theta)) and of dLam (column kK; the gradient of a token's
  // dt A term collects every later Lam of the chunk).
  {
    constexpr int TPL = Q > 32 ? Q / 32 : 1;
    constexpr int NW = kTh / 32, CPW = (kK + NW) / NW;  // column c = warp + 8 j
    float x[CPW][TPL], run[CPW], incl[CPW];
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int col = warp + NW * j;
      run[j] = 0.f;
#pragma unroll
      for (int u = 0; u < TPL; ++u) {
        const int t = lane * TPL + u;
        x[j][u] = 0.f;
        if (col <= kK && t < nt) x[j][u] = col < kK ? dPhi[t * kKP + col] : dLam[t];
        run[j] += x[j][u];
      }
      incl[j] = run[j];
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1)
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const float y = __shfl_up_sync(0xffffffffu, incl[j], off);
        if (lane >= off) incl[j] += y;
      }
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int col = warp + NW * j;
      const float total = __shfl_sync(0xffffffffu, incl[j], 31);
      float pre = incl[j] - run[j];  // sum over the tokens before this lane's
#pragma unroll
      for (int u = 0; u < TPL; ++u) {
        const int t = lane * TPL + u;
        if (col <= kK && t < nt) {
          if (col < kK) dPhi[t * kKP + col] = total - pre;
          else dLam[t] = total - pre;
        }
        pre += x[j][u];
      }
    }
  }
  __syncthreads();
  {
    constexpr int K4 = kK / 4;  // 16 float4 groups per token
    constexpr int PER = (Q * K4 + kTh - 1) / kTh;
    float4 th[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {  // every theta load issued first
      const int e = tid + j * kTh, u = e / K4, k4 = e % K4;
      th[j] = e < nt * K4
                  ? __ldg(reinterpret_cast<const float4*>(
                        a.theta + ((q.base + q.t0 + u) * a.tgroups + q.tg) * kK + 4 * k4))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = tid + j * kTh, u = e / K4, k4 = e % K4;
      float part = 0.f;
      if (e < nt * K4) {
        const int64_t to = ((q.base + q.t0 + u) * a.tgroups + q.tg) * kK + 4 * k4;
        const float* dpr = dPhi + u * kKP + 4 * k4;
        const float4 dp = make_float4(dpr[0], dpr[1], dpr[2], dpr[3]);
        const float d = dts[u];
        atomicAdd(reinterpret_cast<float4*>(g.dtheta + to),
                  make_float4(d * dp.x, d * dp.y, d * dp.z, d * dp.w));
        part = th[j].x * dp.x + th[j].y * dp.y + th[j].z * dp.z + th[j].w * dp.w;
      }
#pragma unroll
      for (int off = 1; off < K4; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (e < nt * K4 && (tid & (K4 - 1)) == 0) atomicAdd(thT + u, part);
    }
  }
  __syncthreads();
  // per token: dt, A, lam (gamma = lam dt, eps = (1 - lam) dt, delta_s = gamma_s + eps_s+1)
  for (int u = tid; u < nt; u += kTh) {
    const float run = dLam[u];  // sum over t >= u of dLam_t
    const int64_t o = (q.base + q.t0 + u) * H + q.h;
    const float dt = dts[u], lam = __ldg(a.lam + o), Av = __ldg(a.A + o);
    const float dgv = dgam[u] + ddel[u];
    const float de = (u > 0) ? ddel[u - 1] : 0.f;  // eps_u through delta_u-1 (this chunk)
    g.dA[o] = dt * run;
    atomicAdd(g.ddt + o, Av * run + thT[u] + lam * dgv + (1.f - lam) * de);
    atomicAdd(g.dlam + o, dt * (dgv - de));
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
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

template <int R>
cudaError_t sums_r(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st) {
  const size_t smem = SumsSmem::bytes(kM / R);
  cudaError_t e = set_smem(bwd_tc_sums_kernel<R>, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  // three CTAs per SM: shared memory (under 75 KB each), registers (at most
  // 85 per thread, the launch bounds) and TMEM (3 x 128 of 512 columns)
  static_assert(3 * (SumsSmem::bytes(kM) + 1024) <= 232448, "three CTAs per SM");
  const int64_t total = f.batch * f.nheads * f.nchunks;
  const int64_t slots = 3 * (int64_t)sms;
  bwd_tc_sums_kernel<R><<<(unsigned)(total < slots ? total : slots), kTh, smem, st>>>(f, g, w);
  return cudaGetLastError();
}

template <int R>
cudaError_t chunk_r(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st) {
  const size_t smem = ChunkTc<kM / R>::bytes();
  cudaError_t e = set_smem(bwd_tc_chunk_kernel<R>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)f.nchunks, (unsigned)f.nheads, (unsigned)f.batch);
  bwd_tc_chunk_kernel<R><<<grid, kTh, smem, st>>>(f, g, w);
  return cudaGetLastError();
}

}  // namespace

bool bwd_tc_shape(const ScanArgs& a) {
  return a.bf16 && a.N == kN && a.P == kP &&
         (a.R == 1 || a.R == 2 || a.R == 4 || a.R == 8);
}

cudaError_t bwd_tc_sums_launch(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st) {
  switch (f.R) {
    case 1: return sums_r<1>(f, g, w, st);
    case 2: return sums_r<2>(f, g, w, st);
    case 4: return sums_r<4>(f, g, w, st);
    case 8: return sums_r<8>(f, g, w, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t bwd_tc_chunk_launch(const ScanArgs& f, const BwdArgs& g, const BwdWs& w, cudaStream_t st) {
  switch (f.R) {
    case 1: return chunk_r<1>(f, g, w, st);
    case 2: return chunk_r<2>(f, g, w, st);
    case 4: return chunk_r<4>(f, g, w, st);
    case 8: return chunk_r<8>(f, g, w, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
