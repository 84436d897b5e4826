// scan_tc.cu -- tensor-core (tcgen05 / TMEM) chunked prefill scan, bf16 io.
//
// The chunked form of the Mamba-3 recurrence (paper: PaperWeekly page
// section 2.2 -- the trapezoid rule makes the mask "decay x width-2
// convolution", and the complex transition is data-dependent RoPE on B, C;
// section 2.3 -- rank-R MIMO), per (batch b, head h) and chunk of Q tokens
// with M = Q*R rows (token, rank):
//
//   S   = Ct Bt^T                       M x M,  K = N     (MMA1, tcgen05)
//   P   = S o mask,  mask[(t,r),(s,r')] = [s<=t] exp(Lam_t - Lam_s) (s==t ? gamma_t : delta_s)
//   Y   = P X  +  diag(exp(Lam_t)) Ct G  M x P            (MMA2 + MMA4)
//   Sc  = Bt^T diag(w) X,  w_s = exp(Lam_end - Lam_s) delta_s   (MMA3)
//   G  <- Rot(Phi_end) (exp(Lam_end) G + Sc)                     (fp32, registers)
//
// with Bt = Rot(-Phi) B, Ct = Rot(-Phi) C rotated in the chunk-local frame.
// One CTA owns a run of consecutive chunks ("segment") of one (b, h) and
// carries the fp32 state G across them in registers (thread n holds state
// row n).  When there are too few (b, h) chains to fill the GPU, each chain is
// cut into segments: a first pass (MODE_STATE) computes every segment's local
// end state from a zero start, a small pass combines them into each segment's
// incoming state, and the full pass runs every segment with its true state.
//
// Operands live in shared memory in the 128-byte-swizzled canonical layout
// and are read by tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) issued by one
// thread; accumulators live in TMEM and are read back with tcgen05.ld.
// Supported: N = 128, P = 64, M = Q*R in {64, 128, 256}.
#include "m3_internal.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

using namespace tc;

constexpr int kN = 128;       // dstate
constexpr int kP = 64;        // headdim
constexpr int kPairs = kN / 2;
constexpr int kThreads = 128;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier wait (2 s)

enum { MODE_FULL = 0, MODE_STATE = 1 };

template <int R, int Q>
struct Cfg {
  static constexpr int M = Q * R;
  static constexpr int MT = M < 128 ? M : 128;  // rows per MMA tile
  static constexpr int NT = M / MT;             // tiles per chunk
  static constexpr int OPB = M * 128;           // bytes of one [M][128 B] operand block
  // shared memory regions (1024-byte aligned)
  static constexpr int C_OFF = 0;               // Ct: K = N split in 2 blocks of 64
  static constexpr int X_OFF = C_OFF + 2 * OPB;
  static constexpr int B_OFF = X_OFF + OPB;     // Bt: 2 blocks
  static constexpr int XW_OFF = B_OFF + 2 * OPB;
  static constexpr int P_OFF = B_OFF;           // masked scores reuse Bt + Xw
  static constexpr int G_OFF = XW_OFF + OPB;    // state, bf16 [N][128 B]
  static constexpr int SMALL_OFF = G_OFF + kN * 128;
  static constexpr int SMALL_BYTES = 8 * Q * 4 + 2 * kPairs * 4 + 64;
  // + alignment slack; at least 80 KB so that no more than two CTAs (2 x 256
  // TMEM columns) share an SM
  static constexpr int SMEM_RAW = SMALL_OFF + SMALL_BYTES + 1024;
  static constexpr int SMEM = SMEM_RAW < 80 * 1024 ? 80 * 1024 : SMEM_RAW;
  // P tile mt: ((mt + 1) * MT / 64) blocks of [MT][128 B]
  __host__ __device__ static constexpr int p_tile_off(int mt) {
    return mt == 0 ? 0 : (MT / 64) * MT * 128;
  }
  static constexpr int P_BYTES = p_tile_off(NT - 1) + (NT * MT / 64) * MT * 128;
  static_assert(P_BYTES <= 3 * OPB, "masked scores must fit over Bt + Xw");
  // TMEM columns
  static constexpr int S_COL1 = 0;                  // tile 1 scores (M = 256 only)
  static constexpr int S_COL0 = (NT == 2) ? 256 : 0;
  static constexpr int SC_COL = (NT == 2) ? 384 : 128;  // chunk state N x P
  static constexpr int TMEM_COLS = (NT == 2) ? 512 : 256;
  __host__ __device__ static constexpr int s_col(int mt) { return mt == 0 ? S_COL0 : S_COL1; }
  __host__ __device__ static constexpr int y_col(int mt) { return 64 * mt; }
  __host__ __device__ static constexpr int y2_col(int mt) { return 64 * (NT + mt); }
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct TcPlan {
  int64_t nseg;  // segments per (b, h) chain
  int64_t cps;   // chunks per segment
  float* wsT;    // [b][H][nseg-1][N][P]: local end states, then incoming states
  float* wsSum;  // [b][H][nseg-1][1 + N/2]: segment log-decay and angles
};

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Every thread polls; returns false on timeout (after recording it).
__device__ bool wait_bar(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitNs) {
      if (status) atomicCAS(status, 0, (int)M3_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

template <int R, int Q, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_scan_kernel(const ScanArgs a, const TcPlan pl) {
  using C = Cfg<R, Q>;
  constexpr int M = C::M, MT = C::MT, NT = C::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* s_lam = reinterpret_cast<float*>(sm + C::SMALL_OFF);  // chunk-local Lam_t
  float* s_gam = s_lam + Q;
  float* s_del = s_gam + Q;
  float* s_w = s_del + Q;
  float* s_dt = s_w + Q;
  float* s_ph = s_dt + 3 * Q;                  // [2][kPairs] half-chunk angle sums
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(s_ph + 2 * kPairs);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_bar + 1);
  float* s_lend = reinterpret_cast<float*>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t L = a.seqlen, H = a.nheads, G = a.ngroups;
  const int64_t g = h / (H / G);
  const int64_t nseg = (MODE == MODE_FULL) ? pl.nseg : pl.nseg - 1;
  (void)nseg;

  if (warp == 0) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(s_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  uint32_t phase = 0;
  bool aborted = false;

  // ---- incoming state: thread n = tid owns state row n ---------------------
  const int n = tid;
  float gst[kP];
  if (MODE == MODE_STATE) {
#pragma unroll
    for (int p = 0; p < kP; ++p) gst[p] = 0.f;
  } else if (seg == 0) {
    const int64_t so = ((b * H + h) * kN + n) * kP;
#pragma unroll
    for (int p = 0; p < kP; ++p) gst[p] = a.h0 ? a.h0[so + p] : 0.f;
    if (a.B_prev) {
      const float eps0 = (1.f - a.lam[(b * L) * H + h]) * a.dt[(b * L) * H + h];
      for (int r = 0; r < R; ++r) {
        const float bp = eps0 * io_load(a.B_prev, ((b * G + g) * R + r) * kN + n, true);
        const int64_t xo = ((b * H + h) * R + r) * kP;
#pragma unroll
        for (int p = 0; p < kP; ++p) gst[p] = fmaf(bp, io_load(a.x_prev, xo + p, true), gst[p]);
      }
    }
  } else {
    const float* src = pl.wsT + (((b * H + h) * (pl.nseg - 1) + (seg - 1)) * kN + n) * kP;
#pragma unroll
    for (int p = 0; p < kP; p += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + p);
      gst[p] = v.x; gst[p + 1] = v.y; gst[p + 2] = v.z; gst[p + 3] = v.w;
    }
  }
  auto store_state_bf16 = [&]() {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint4 v;
      v.x = pack_bf16(gst[8 * ch + 0], gst[8 * ch + 1]);
      v.y = pack_bf16(gst[8 * ch + 2], gst[8 * ch + 3]);
      v.z = pack_bf16(gst[8 * ch + 4], gst[8 * ch + 5]);
      v.w = pack_bf16(gst[8 * ch + 6], gst[8 * ch + 7]);
      *reinterpret_cast<uint4*>(sm + C::G_OFF + sw128_off(n, ch)) = v;
    }
  };
  if (MODE == MODE_FULL) store_state_bf16();

  float lam_seg = 0.f, phi_seg = 0.f;  // MODE_STATE summaries (pair k = n / 2)
  const int64_t c_begin = seg * pl.cps;
  const int64_t c_end = min(c_begin + pl.cps, a.nchunks);

  for (int64_t c = c_begin; c < c_end && !aborted; ++c) {
    const int64_t c0 = c * Q;
    const int nt = (int)min((int64_t)Q, L - c0);

    // ---- gates: dt, lam, gamma, delta, chunk-local Lam ----------------------
    for (int t = tid; t < Q; t += kThreads) {
      float dt = 0.f, lm = 0.f, av = 0.f, nx = 0.f;
      if (t < nt) {
        const int64_t bt = b * L + c0 + t;
        dt = a.dt[bt * H + h];
        lm = a.lam[bt * H + h];
        av = a.A[bt * H + h];
        if (c0 + t + 1 < L) nx = (1.f - a.lam[(bt + 1) * H + h]) * a.dt[(bt + 1) * H + h];
      }
      s_dt[t] = dt;
      s_gam[t] = lm * dt;
      s_del[t] = lm * dt + nx;
      s_lam[t] = dt * av;
    }
    __syncthreads();
    {  // half-chunk sums of the step angles, pair k = tid % 64, half = tid / 64
      const int k = tid & (kPairs - 1), half = tid >> 6;
      float acc = 0.f;
      const int t1 = min(nt, (half + 1) * (Q / 2));
      for (int t = half * (Q / 2); t < t1; ++t)
        acc = fmaf(s_dt[t], a.theta[((b * L + c0 + t) * G + g) * kPairs + k], acc);
      s_ph[half * kPairs + k] = acc;
    }
    if (tid == 0) {
      float acc = 0.f;
      for (int t = 0; t < nt; ++t) {
        acc += s_lam[t];
        s_lam[t] = acc;
      }
      *s_lend = acc;
    }
    __syncthreads();
    const float lend = *s_lend;
    for (int t = tid; t < Q; t += kThreads)
      s_w[t] = (t < nt) ? __expf(lend - s_lam[t]) * s_del[t] : 0.f;
    __syncthreads();

    // ---- operands: Bt (and Ct) rotated by -Phi_t, x and w*x ------------------
    {
      const int k = tid & (kPairs - 1), half = tid >> 6;
      float phi = half ? s_ph[k] : 0.f;
      const int kb = k >> 5;                     // 64-element K block of element 2k
      const int ch = (k & 31) >> 2;              // 16-byte chunk in the 128-byte row
      const int cb = (k & 3) * 4;                // byte in the chunk
      for (int tt = 0; tt < Q / 2; ++tt) {
        const int t = half * (Q / 2) + tt;
        float sn = 0.f, cs = 0.f;
        const bool valid = t < nt;
        if (valid) {
          phi = fmaf(s_dt[t], a.theta[((b * L + c0 + t) * G + g) * kPairs + k], phi);
          sincosf(phi, &sn, &cs);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t row = t * R + r;
          const uint32_t off = kb * C::OPB + sw128_off(row, ch) + cb;
          uint32_t vb = 0, vc = 0;
          if (valid) {
            const int64_t e = (((b * L + c0 + t) * G + g) * R + r) * kN + 2 * k;
            const float2 bb = unpack_bf16(*reinterpret_cast<const uint32_t*>(
                reinterpret_cast<const __nv_bfloat16*>(a.B) + e));
            vb = pack_bf16(cs * bb.x + sn * bb.y, -sn * bb.x + cs * bb.y);
            if (MODE == MODE_FULL) {
              const float2 cc = unpack_bf16(*reinterpret_cast<const uint32_t*>(
                  reinterpret_cast<const __nv_bfloat16*>(a.C) + e));
              vc = pack_bf16(cs * cc.x + sn * cc.y, -sn * cc.x + cs * cc.y);
            }
          }
          *reinterpret_cast<uint32_t*>(sm + C::B_OFF + off) = vb;
          if (MODE == MODE_FULL) *reinterpret_cast<uint32_t*>(sm + C::C_OFF + off) = vc;
        }
      }
    }
    for (int q = tid; q < M * 8; q += kThreads) {
      const int row = q >> 3, ch = q & 7;
      const int t = row / R, r = row % R;
      uint4 v = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
      if (t < nt) {
        const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.x) +
                                   (((b * L + c0 + t) * H + h) * R + r) * kP + ch * 8;
        v = *reinterpret_cast<const uint4*>(src);
        const float w = s_w[t];
        float2 f;
        f = unpack_bf16(v.x); vw.x = pack_bf16(w * f.x, w * f.y);
        f = unpack_bf16(v.y); vw.y = pack_bf16(w * f.x, w * f.y);
        f = unpack_bf16(v.z); vw.z = pack_bf16(w * f.x, w * f.y);
        f = unpack_bf16(v.w); vw.w = pack_bf16(w * f.x, w * f.y);
      }
      if (MODE == MODE_FULL) *reinterpret_cast<uint4*>(sm + C::X_OFF + sw128_off(row, ch)) = v;
      *reinterpret_cast<uint4*>(sm + C::XW_OFF + sw128_off(row, ch)) = vw;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA1 (scores) and MMA3 (chunk state) ---------------------------------
    if (tid == 0) {
      if (MODE == MODE_FULL) {
#pragma unroll
        for (int mt = 0; mt < NT; ++mt) {
          const uint32_t id = idesc_bf16(MT, (mt + 1) * MT, 0, 0);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint64_t ad = sw128_desc(sbase + C::C_OFF + kb * C::OPB + mt * MT * 128 + k4 * 32, 16, 1024);
              const uint64_t bd = sw128_desc(sbase + C::B_OFF + kb * C::OPB + k4 * 32, 16, 1024);
              mma_bf16_ss(tm + C::s_col(mt), ad, bd, id, (kb | k4) != 0);
            }
        }
      }
      const uint32_t id3 = idesc_bf16(kN, kP, 1, 1);
#pragma unroll
      for (int ks = 0; ks < M / 16; ++ks) {
        const uint64_t ad = sw128_desc(sbase + C::B_OFF + ks * 2048, C::OPB, 1024);
        const uint64_t bd = sw128_desc(sbase + C::XW_OFF + ks * 2048, C::OPB, 1024);
        mma_bf16_ss(tm + C::SC_COL, ad, bd, id3, ks != 0);
      }
      mma_commit(s_bar);
    }
    const bool ok1 = wait_bar(s_bar, phase, a.status);
    phase ^= 1;
    if (__syncthreads_or(!ok1)) { aborted = true; break; }
    tc_fence_after();

    if (MODE == MODE_FULL) {
      // ---- mask the scores into P (bf16, K-major, over Bt / Xw) -------------
#pragma unroll
      for (int mt = 0; mt < NT; ++mt) {
        const int rho = (MT == 64) ? 16 * warp + lane : tid;  // row within the tile
        const bool live = (MT == 64) ? lane < 16 : true;
        const int i = mt * MT + rho;
        const int t = i / R;
        const bool trow = live && t < nt;
        const float lt = trow ? s_lam[t] : 0.f;
        const int ncols = (mt + 1) * MT;
        for (int cc = 0; cc < ncols / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tm + lane_base + C::s_col(mt) + cc * 32, v);
          tmem_ld_wait();
          if (!live) continue;
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float o[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int s = (cc * 32 + j + e) / R;
              float m = 0.f;
              if (trow && s <= t)
                m = __expf(lt - s_lam[s]) * ((s == t) ? s_gam[t] : s_del[s]);
              o[e] = __uint_as_float(v[j + e]) * m;
            }
            pk[j / 2] = pack_bf16(o[0], o[1]);
          }
          const int kb = (cc * 32) / 64;
          uint8_t* blk = sm + C::P_OFF + C::p_tile_off(mt) + kb * MT * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = ((cc * 32) % 64) / 8 + q;
            *reinterpret_cast<uint4*>(blk + sw128_off(rho, ch)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();

      // ---- MMA2 (P x) and MMA4 (Ct G) ----------------------------------------
      if (tid == 0) {
        const uint32_t id2 = idesc_bf16(MT, kP, 0, 1);
#pragma unroll
        for (int mt = 0; mt < NT; ++mt) {
          const int kblocks = (mt + 1) * MT / 64;
          for (int kb = 0; kb < kblocks; ++kb)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint64_t ad = sw128_desc(
                  sbase + C::P_OFF + C::p_tile_off(mt) + kb * MT * 128 + k4 * 32, 16, 1024);
              const uint64_t bd = sw128_desc(sbase + C::X_OFF + (kb * 4 + k4) * 2048, C::OPB, 1024);
              mma_bf16_ss(tm + C::y_col(mt), ad, bd, id2, (kb | k4) != 0);
            }
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint64_t ad = sw128_desc(sbase + C::C_OFF + kb * C::OPB + mt * MT * 128 + k4 * 32, 16, 1024);
              const uint64_t bd = sw128_desc(sbase + C::G_OFF + (kb * 4 + k4) * 2048, kN * 128, 1024);
              mma_bf16_ss(tm + C::y2_col(mt), ad, bd, id2, (kb | k4) != 0);
            }
        }
        mma_commit(s_bar);
      }
      const bool ok2 = wait_bar(s_bar, phase, a.status);
      phase ^= 1;
      if (__syncthreads_or(!ok2)) { aborted = true; break; }
      tc_fence_after();

      // ---- epilogue: y = P x + exp(Lam_t) Ct G ---------------------------------
#pragma unroll
      for (int mt = 0; mt < NT; ++mt) {
        const int rho = (MT == 64) ? 16 * warp + lane : tid;
        const bool live = (MT == 64) ? lane < 16 : true;
        const int i = mt * MT + rho;
        const int t = i / R, r = i % R;
        const bool out = live && t < nt;
        const float el = out ? __expf(s_lam[t]) : 0.f;
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.y) +
                             (((b * L + c0 + (out ? t : 0)) * H + h) * R + r) * kP;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t yv[32], zv[32];
          tmem_ld32(tm + lane_base + C::y_col(mt) + 32 * half, yv);
          tmem_ld32(tm + lane_base + C::y2_col(mt) + 32 * half, zv);
          tmem_ld_wait();
          if (out) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = q * 8 + 2 * e;
                w4[e] = pack_bf16(fmaf(el, __uint_as_float(zv[j]), __uint_as_float(yv[j])),
                                  fmaf(el, __uint_as_float(zv[j + 1]), __uint_as_float(yv[j + 1])));
              }
              *reinterpret_cast<uint4*>(dst + 32 * half + q * 8) =
                  make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
      }
    }

    // ---- state update: G <- Rot(Phi_end) (exp(Lam_end) G + Sc) ---------------
    {
      uint32_t s0[32], s1[32];
      tmem_ld32(tm + lane_base + C::SC_COL, s0);
      tmem_ld32(tm + lane_base + C::SC_COL + 32, s1);
      tmem_ld_wait();
      const int k = n >> 1;
      const float phe = s_ph[k] + s_ph[kPairs + k];
      float sn, cs;
      sincosf(phe, &sn, &cs);
      const float el = __expf(lend);
      const bool even = (n & 1) == 0;
#pragma unroll
      for (int p = 0; p < kP; ++p) {
        const float sc = __uint_as_float(p < 32 ? s0[p] : s1[p - 32]);
        const float v = fmaf(el, gst[p], sc);
        const float o = __shfl_xor_sync(0xffffffffu, v, 1);
        gst[p] = even ? (cs * v - sn * o) : (sn * o + cs * v);
      }
      if (MODE == MODE_STATE) {
        lam_seg += lend;
        phi_seg += phe;
      }
    }
    if (MODE == MODE_FULL) store_state_bf16();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (!aborted) {
    if (MODE == MODE_FULL) {
      if (seg == pl.nseg - 1 && a.final_state) {
        float* dst = a.final_state + ((b * H + h) * kN + n) * kP;
#pragma unroll
        for (int p = 0; p < kP; p += 4)
          *reinterpret_cast<float4*>(dst + p) = make_float4(gst[p], gst[p + 1], gst[p + 2], gst[p + 3]);
      }
    } else {
      const int64_t slot = (b * H + h) * (pl.nseg - 1) + seg;
      float* dst = pl.wsT + (slot * kN + n) * kP;
#pragma unroll
      for (int p = 0; p < kP; p += 4)
        *reinterpret_cast<float4*>(dst + p) = make_float4(gst[p], gst[p + 1], gst[p + 2], gst[p + 3]);
      float* su = pl.wsSum + slot * (1 + kPairs);
      if (tid == 0) su[0] = lam_seg;
      if ((n & 1) == 0) su[1 + (n >> 1)] = phi_seg;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, C::TMEM_COLS);
}

// Combine segment summaries into each segment's incoming state (fp32).
// Thread (k, p) of chain (b, h): G_0 = h0 + (1 - lam_0) dt_0 B_prev x_prev^T,
// G_{s+1} = Rot(Phi_s) exp(Lam_s) G_s + T_s, stored over T_s.
__global__ void __launch_bounds__(256) tc_seg_pass_kernel(const ScanArgs a, const TcPlan pl) {
  const int64_t b = blockIdx.z, h = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= kPairs * kP) return;
  const int k = idx / kP, p = idx % kP;
  const int64_t H = a.nheads, L = a.seqlen, R = a.R, G = a.ngroups;
  const int64_t g = h / (H / G);
  const int64_t so = (b * H + h) * kN * kP;
  float g0 = a.h0 ? a.h0[so + (2 * k) * kP + p] : 0.f;
  float g1 = a.h0 ? a.h0[so + (2 * k + 1) * kP + p] : 0.f;
  if (a.B_prev) {
    const float eps = (1.f - a.lam[(b * L) * H + h]) * a.dt[(b * L) * H + h];
    for (int r = 0; r < R; ++r) {
      const int64_t bb = ((b * G + g) * R + r) * kN;
      const float xv = io_load(a.x_prev, ((b * H + h) * R + r) * kP + p, true);
      g0 = fmaf(eps * io_load(a.B_prev, bb + 2 * k, true), xv, g0);
      g1 = fmaf(eps * io_load(a.B_prev, bb + 2 * k + 1, true), xv, g1);
    }
  }
  for (int64_t s = 0; s + 1 < pl.nseg; ++s) {
    const int64_t slot = (b * H + h) * (pl.nseg - 1) + s;
    float* T = pl.wsT + slot * kN * kP;
    const float* su = pl.wsSum + slot * (1 + kPairs);
    const float e = expf(su[0]);
    float sn, cs;
    sincosf(su[1 + k], &sn, &cs);
    const float u0 = e * g0, u1 = e * g1;
    const float n0 = cs * u0 - sn * u1 + T[(2 * k) * kP + p];
    const float n1 = sn * u0 + cs * u1 + T[(2 * k + 1) * kP + p];
    T[(2 * k) * kP + p] = n0;
    T[(2 * k + 1) * kP + p] = n1;
    g0 = n0;
    g1 = n1;
  }
}

TcPlan make_plan(const ScanArgs& a) {
  TcPlan pl{};
  const int64_t chains = a.batch * a.nheads;
  const int64_t target = 2 * 148;  // CTAs for at least two waves of one CTA per SM
  int64_t nseg = chains >= target ? 1 : (target + chains - 1) / chains;
  if (nseg > a.nchunks) nseg = a.nchunks;
  if (nseg < 1) nseg = 1;
  pl.cps = (a.nchunks + nseg - 1) / nseg;
  pl.nseg = (a.nchunks + pl.cps - 1) / pl.cps;
  return pl;
}

template <int R, int Q, int MODE>
cudaError_t launch_kernel(const ScanArgs& a, const TcPlan& pl, int64_t nblocks, cudaStream_t st) {
  using C = Cfg<R, Q>;
  auto kern = tc_scan_kernel<R, Q, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)nblocks, (unsigned)a.nheads, (unsigned)a.batch);
  kern<<<grid, kThreads, C::SMEM, st>>>(a, pl);
  return cudaGetLastError();
}

template <int R, int Q>
cudaError_t launch_rq(const ScanArgs& a, TcPlan pl, cudaStream_t st) {
  if (pl.nseg > 1) {
    cudaError_t e = launch_kernel<R, Q, MODE_STATE>(a, pl, pl.nseg - 1, st);
    if (e != cudaSuccess) return e;
    dim3 pg((kPairs * kP + 255) / 256, (unsigned)a.nheads, (unsigned)a.batch);
    tc_seg_pass_kernel<<<pg, 256, 0, st>>>(a, pl);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_kernel<R, Q, MODE_FULL>(a, pl, pl.nseg, st);
}

}  // namespace

bool tc_scan_supported(const ScanArgs& a) {
  if (!a.bf16 || a.N != kN || a.P != kP) return false;
  const int64_t m = a.Q * a.R;
  return (a.R == 1 || a.R == 2 || a.R == 4) && (m == 64 || m == 128 || m == 256) && a.Q >= 16;
}

size_t tc_scan_workspace(const ScanArgs& a) {
  const TcPlan pl = make_plan(a);
  if (pl.nseg <= 1) return 0;
  const size_t slots = (size_t)a.batch * a.nheads * (pl.nseg - 1);
  return align_up(sizeof(float) * slots * kN * kP, 256) +
         align_up(sizeof(float) * slots * (1 + kPairs), 256);
}

cudaError_t tc_scan_launch(const ScanArgs& a, cudaStream_t st) {
  TcPlan pl = make_plan(a);
  if (pl.nseg > 1) {
    const size_t slots = (size_t)a.batch * a.nheads * (pl.nseg - 1);
    pl.wsT = reinterpret_cast<float*>(a.ws);
    pl.wsSum = reinterpret_cast<float*>(a.ws + align_up(sizeof(float) * slots * kN * kP, 256));
  }
  const int64_t m = a.Q * a.R;
  if (a.R == 1 && a.Q == 64) return launch_rq<1, 64>(a, pl, st);
  if (a.R == 2 && a.Q == 64) return launch_rq<2, 64>(a, pl, st);
  if (a.R == 2 && a.Q == 32) return launch_rq<2, 32>(a, pl, st);
  if (a.R == 4 && a.Q == 64) return launch_rq<4, 64>(a, pl, st);
  if (a.R == 4 && a.Q == 32) return launch_rq<4, 32>(a, pl, st);
  if (a.R == 4 && a.Q == 16) return launch_rq<4, 16>(a, pl, st);
  (void)m;
  return cudaErrorInvalidValue;
}

}  // namespace m3
