// scan_tc.cu -- tensor-core (tcgen05 / TMEM) chunked prefill scan, bf16 io.
//
// The chunked form of the Mamba-3 recurrence (paper: PaperWeekly page
// section 2.2 -- the trapezoid rule makes the mask "decay x width-2
// convolution", and the complex transition is data-dependent RoPE on B, C;
// section 2.3 -- rank-R MIMO), per (batch b, head h) and chunk of Q tokens
// with M = Q*R rows (token, rank):
//
//   y_t = sum_{s<=t} exp(Lam_t - Lam_s) c_ts (Ct_t . Bt_s) x_s + exp(Lam_t) Ct_t G,
//   c_tt = gamma_t, c_ts = delta_s (s < t);   G <- Rot(Phi_end)(exp(Lam_end) G + Sc),
//   Sc = sum_s exp(Lam_end - Lam_s) delta_s Bt_s x_s^T,
//
// with Bt = Rot(-Phi) B, Ct = Rot(-Phi) C rotated in the chunk-local frame.  The
// decay matrix exp(Lam_t - Lam_s) is factored around a reference ref = Lam_end / 2:
// B is staged as Bh_s = u_s Bt_s with u_s = exp(ref - Lam_s) delta_s, so that
//
//   S'  = Ct Bh^T                         M x M,  K = N     (MMA1, tcgen05)
//   P'  = S' o M',  M'[(t,r),(s,r')] = 1 (s < t), gamma_t / delta_t (s = t), 0 (s > t)
//   Y'  = P' X + Ct (exp(ref) G)          M x P, one accumulator (MMA2 + MMA4)
//   y_t = exp(Lam_t - ref) Y'_t                               (epilogue)
//   Sc  = exp(Lam_end - ref) Bh^T X                           (MMA3)
//
// so the mask is a plain causal mask and no weighted copy of x is made.  The
// factors stay inside fp32 / bf16 range while the chunk's total decay does
// (|Lam_end| below about 100 nats, every chunk of the usual inputs); a chunk
// that decays further is done exactly the plain way: Bh_s = delta_s Bt_s for
// the scores, P[t,s] = S'[t,s] exp(Lam_t - Lam_s), a separate Ct G
// accumulator scaled by exp(Lam_t), and Bh rescaled in place to
// exp(Lam_end - Lam_s) delta_s Bt_s before MMA3 reads it.
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
// Independent accumulators are issued as interleaved chains (an MMA waits on
// the previous one into the same tile), and 256-row chunks keep their masked
// scores in TMEM as the A operand of P x.  When one segment per chain leaves
// the last wave of CTAs partly empty, only that wave's chains are cut in two
// (TcPlan's tail split).
// Supported: N = 128, P = 64, M = Q*R in {64, 128, 256}.
#include <cuda.h>  // CUtensorMap (the encoder is reached through the runtime)

#include "m3_internal.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

using namespace tc;

// D (TMEM) [+]= A (TMEM) * B (smem), issued by one thread.  A is M x K with
// row i in TMEM lane i and K along the columns, two bf16 elements per 32-bit
// column (the lower K index in the low half): a K = 16 step reads 8 columns
// from `a_tmem`.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// 8 consecutive 32-bit columns of this thread's TMEM lane (warp-wide store).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}

constexpr int kN = 128;       // dstate
constexpr int kP = 64;        // headdim
constexpr int kPairs = kN / 2;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier wait (2 s)
// A chunk whose total log-decay (log2 units) is at or below this (about -100
// nats) is done in the plain form: the factored one would need factors beyond
// e^+-50, where bf16 state and scaled-B values lose their low-order bits.
constexpr float kPlainL2 = -144.f;

enum { MODE_FULL = 0, MODE_STATE = 1 };

template <int R, int Q>
struct Cfg {
  static constexpr int M = Q * R;
  // 256 threads and two CTAs per SM for 64-row chunks, else 512 threads
  static constexpr int NTH = (Q * R == 64) ? 256 : 512;
  static constexpr int MINB = (Q * R == 64) ? 2 : 1;
  static constexpr int SLOTS_MAX = NTH / 16;    // token slots of the rotation pass
  static constexpr int MT = M < 128 ? M : 128;  // rows per MMA tile
  static constexpr int NT = M / MT;             // tiles per chunk
  static constexpr int OPB = M * 128;           // bytes of one [M][128 B] operand block
  // shared memory regions (1024-byte aligned)
  static constexpr int C_OFF = 0;               // Ct: K = N split in 2 blocks of 64
  static constexpr int X_OFF = C_OFF + 2 * OPB;
  static constexpr int B_OFF = X_OFF + OPB;     // Bt: 2 blocks
  static constexpr int ST_OFF = B_OFF + 2 * OPB;  // staging: masked scores of tile 0, y
  static constexpr int G_OFF = ST_OFF + OPB;    // scaled state, bf16 [N][128 B]
  static constexpr int SMALL_OFF = G_OFF + kN * 128;
  // small region: the chunk's theta [Q][N/2] (a TMA destination, first so it
  // is 1 KB aligned; the slot angle sums go over it once it is read),
  // per-token gamma, delta, w, Lam (log2 units) and the decay factor F,
  // chunk-end angles with their cos / sin, and the mbarriers.
  static constexpr int TH_FLOATS = Q * kPairs;
  // The slot angle sums have their own buffer when shared memory allows (one
  // tile per chunk), else they go over theta once it is read (a barrier more).
  static constexpr bool PART_OWN = NT == 1;
  static constexpr int PART_FLOATS = PART_OWN ? SLOTS_MAX * kPairs : 0;
  static constexpr int SMALL_BYTES =
      (TH_FLOATS + PART_FLOATS + 6 * Q + 3 * kPairs) * 4 + 64;  // + 8 mbarrier slots
  static_assert(((TH_FLOATS + PART_FLOATS + 6 * Q + 3 * kPairs) * 4) % 8 == 0,
                "mbarrier alignment");
  // at least 80 KB so that no more than two CTAs (2 x 256 TMEM columns) share
  // an SM; the dynamic shared memory base is declared 1024-byte aligned
  static constexpr int SMEM_RAW = SMALL_OFF + SMALL_BYTES;
  static constexpr int SMEM = SMEM_RAW < 80 * 1024 ? 80 * 1024 : SMEM_RAW;
  static_assert(MINB * (SMEM + 1024) <= 233472, "CTAs per SM must fit the SM's shared memory");
  // Masked scores P, tile mt: ((mt + 1) * MT / 64) K-blocks of [MT][128 B].
  // One tile: over Bh (MMA1 and MMA3 are done when it is written).  Two
  // tiles: tile 0 in the staging block (tile 1's MMA1 still reads all of Bh),
  // tile 1 over Bh once tile 1's scores and MMA3 are complete.
  __host__ __device__ static constexpr int p_off(int mt) {
    return (NT == 2 && mt == 0) ? ST_OFF : B_OFF;
  }
  static_assert(NT == 1 ? (MT / 64) * MT * 128 <= 2 * OPB
                        : (MT / 64) * MT * 128 <= OPB && 2 * (MT / 64) * MT * 128 <= 2 * OPB,
                "masked scores must fit their regions");
  // TMEM columns
  static constexpr int S_COL1 = 0;                  // tile 1 scores (M = 256 only)
  static constexpr int S_COL0 = (NT == 2) ? 256 : 0;
  // One tile per chunk: scores (MT columns), output accumulator and chunk
  // state side by side, so MMA4 can run with MMA3 before the mask.  Two
  // tiles: the scores take 384 columns, so a tile's MMA2 and MMA4 run after
  // its mask and their accumulators reuse that tile's score columns (tile 0's
  // MMAs then overlap tile 1's mask).  y_col / y2_col: the two accumulators
  // of the plain (large-decay) form; the factored form accumulates both
  // products in acc_col.
  static constexpr bool EARLY4 = NT == 1;
  static constexpr int SC_COL = (NT == 2) ? 384 : MT + 64;  // chunk state N x P
  static constexpr int TMEM_COLS = (NT == 2) ? 512 : 256;
  __host__ __device__ static constexpr int s_col(int mt) { return mt == 0 ? S_COL0 : S_COL1; }
  __host__ __device__ static constexpr int y_col(int mt) {
    return NT == 2 ? (mt == 0 ? 256 : 0) : 0;
  }
  __host__ __device__ static constexpr int y2_col(int mt) {
    return NT == 2 ? (mt == 0 ? 320 : 64) : MT;
  }
  __host__ __device__ static constexpr int acc_col(int mt) { return NT == 2 ? y_col(mt) : MT; }
  static_assert(SC_COL + kP <= TMEM_COLS, "TMEM columns");
  // Two-tile chunks (M = 256) run three MMA chains side by side instead of
  // one dependent chain: the chunk state in two halves over the rows (K),
  // rows 0-127 into SC_COL and rows 128-255 into SC2_COL, interleaved with
  // tile 0's scores; once the state update has read both halves, the output
  // accumulators of tile 0 and tile 1 take their columns (acc2_col: SC2_COL /
  // SC_COL) and both tiles' Ct G products are issued together before the
  // masks; tile 1's scores are issued after the chunk-state wait.  The
  // masked scores stay in TMEM as packed bf16 (each warp's 16-column step
  // over columns it has already read) and are P x's A operand.
  static constexpr int SC2_COL = 448;
  __host__ __device__ static constexpr int acc2_col(int mt) { return mt == 0 ? SC2_COL : SC_COL; }
  static_assert(NT != 2 || SC2_COL + kP <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// TMA descriptors of one call: x, B, C (bf16, 128-byte swizzled boxes of
// {64 elements, R rows, Q tokens}), theta (fp32 boxes {N/2, 1, Q}) and y
// (bf16 stores of {64, R, Q, 1} over [batch][L][H*R][P], so a chunk's rows
// past its sequence's end are clipped).
struct TcMaps {
  CUtensorMap x, b, c, th, y;
};

struct TcPlan {
  int64_t nseg;   // segments per (b, h) chain
  int64_t cps;    // chunks per segment
  int64_t slots;  // segment summaries per chain: nseg - 1, or nseg for the state only
  float* wsT;    // [b][H][nseg-1][N][P]: local end states, then incoming states
  float* wsSum;  // [b][H][nseg-1][1 + N/2]: segment log-decay and angles
  // Tail split (nseg == 1 plans whose last wave of chains is partial): the
  // last `ntail` chains (b * H + h order) run as two halves of cps2 chunks,
  // so that the last wave holds 2 * ntail half chains; their summaries are
  // [ntail][N][P] and [ntail][1 + N/2], indexed by the chain's tail index.
  // Grids are then one-dimensional: the full pass takes the whole chains
  // first, then the halves (tail chain i: blocks 2i and 2i + 1 after them);
  // the state-only pass takes the tail chains' first halves, and the full
  // pass runs as its programmatic dependent: the second halves wait for it
  // and fold its summaries into their incoming state themselves.
  int64_t ntail;
  int64_t cps2;
};

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Polls an mbarrier (called by one thread); returns false on timeout after
// recording it in the device status word.
__device__ bool wait_bar(uint64_t* bar, uint32_t parity, int* status,
                         unsigned long long limit_ns = kWaitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) {
      if (status) atomicCAS(status, 0, (int)M3_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Thread layout (NTH = 256 or 512 threads).
//  - TMEM work: warp w reads TMEM lanes 32*(w%4)..+31 ("quadrant" qd = w % 4)
//    and takes column part cq = w / 4 of NTH / 128 parts; state row n =
//    32*qd + lane is split over NTH / 128 threads.
//  - Rotation: thread (kg = lane % 16, tq = 2*warp + lane / 16) rotates pairs
//    4*kg..4*kg+3 for the TQ tokens of slot tq.  The 16 lanes of a half-warp
//    cover one 256-byte row of B or C (coalesced 16-byte loads, conflict-free
//    16-byte swizzled stores); the cumulative angles cross token slots
//    through a small shared array.
template <int R, int Q, int MODE>
__global__ void __launch_bounds__(Cfg<R, Q>::NTH, Cfg<R, Q>::MINB)
tc_scan_kernel(const ScanArgs a, const TcPlan pl, const __grid_constant__ TcMaps maps) {
  using C = Cfg<R, Q>;
  constexpr int M = C::M, MT = C::MT, NT = C::NT;
  constexpr int NTH = C::NTH;
  constexpr int CQN = NTH / 128;                          // column parts per TMEM lane
  constexpr int TQ = Q >= C::SLOTS_MAX ? Q / C::SLOTS_MAX : 1;  // tokens per rotation slot
  constexpr int SLOTS = Q / TQ;                           // active rotation slots
  constexpr int CW = kP / CQN;                            // state / output columns per thread
  constexpr float kL2E = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const uint32_t sbase = smem_u32(sm);
  if ((sbase & 1023u) != 0) {  // the swizzled operand layout needs 1 KB alignment
    if (threadIdx.x == 0 && a.status) atomicCAS(a.status, 0, (int)M3_ERR_CUDA);
    return;
  }
  float* s_th = reinterpret_cast<float*>(sm + C::SMALL_OFF);  // chunk theta [Q][N/2] (TMA)
  float* s_gam = s_th + C::TH_FLOATS + C::PART_FLOATS;  // gamma_t = lam_t dt_t         [Q]
  float* s_del = s_gam + Q;                     // delta_s, trapezoid weight of token s [Q]
  float* s_u = s_del + Q;                       // row scale u_s of Bh                  [Q]
  float* s_lg = s_u + Q;                        // Lam_t * log2(e)                      [Q]
  float* s_d = s_lg + Q;                        // gamma_t / delta_t (mask diagonal)    [Q]
  float* s_dtv = s_d + Q;                       // dt_t                                 [Q]
  float* s_phe = s_dtv + Q;                     // chunk-end angles                     [kPairs]
  float2* s_pcs = reinterpret_cast<float2*>(s_phe + kPairs);  // their cos, sin        [kPairs]
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(s_pcs + kPairs);  // MMA3+MMA4, MMA2
  uint64_t* s_bar1 = s_bar + 1;                                         // MMA1
  uint64_t* s_tbT = s_bar + 2;                                          // TMA of theta
  uint64_t* s_tbM = s_bar + 3;                                          // TMA of B, C, x
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_bar + 4);
  uint64_t* s_never = s_bar + 5;  // M3_FLAG_TEST_TIMEOUT: a barrier nothing completes
  uint64_t* s_bar1b = s_bar + 6;  // MMA1 of tile 1 (two-tile chunks)
  // [slots][kPairs] slot angle sums: their own buffer, or over the consumed theta rows
  float* s_part = C::PART_OWN ? s_th + C::TH_FLOATS : s_th;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cq = warp >> 2;
  const int kg = lane & 15, tq = (warp << 1) | (lane >> 4);
  // this CTA's chain, segment and segment length (see TcPlan for the tail split)
  int64_t seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z, nseg_c = pl.nseg, cps_c = pl.cps;
  int64_t ti = -1;  // tail index of a split chain
  if (pl.ntail > 0) {
    const int64_t nfull = a.batch * a.nheads - pl.ntail;
    int64_t chain;
    if (MODE == MODE_STATE) {
      ti = blockIdx.x;
      chain = nfull + ti;
      seg = 0;
    } else if ((int64_t)blockIdx.x < nfull) {
      chain = blockIdx.x;
      seg = 0;
    } else {
      const int64_t k = (int64_t)blockIdx.x - nfull;
      ti = k >> 1;
      chain = nfull + ti;
      seg = k & 1;
    }
    nseg_c = ti >= 0 ? 2 : 1;
    cps_c = ti >= 0 ? pl.cps2 : a.nchunks;
    b = chain / a.nheads;
    h = chain % a.nheads;
  }
  const int64_t H = a.nheads, G = a.ngroups;
  // this chain's sequence: tokens [tokb, tokb + L) of the token dimension
  const Chain chn = chain_of(a, b);
  const int64_t L = chn.len, tokb = chn.base;
  const int64_t g = h / (H / G);
  const int64_t tg = h / (H / a.tgroups);  // theta group
  // bounds-checked builds: the CTA's chain and segment, and its tokens
  if (!M3_IN(b, a.batch, a.status) || !M3_IN(h, H, a.status) || !M3_IN(seg, nseg_c, a.status) ||
      (L > 0 && !M3_IN(tokb + L - 1, a.total_tokens, a.status)))
    return;  // uniform over the block

  // a state-only pass lets a programmatically dependent full pass start now:
  // the full pass's CTAs that need this pass's summaries wait for it
  if (MODE == MODE_STATE) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(s_bar, 1);
    mbar_init(s_bar1, 1);
    mbar_init(s_tbT, 1);
    mbar_init(s_tbM, 1);
    mbar_init(s_never, 1);
    mbar_init(s_bar1b, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
  // Operand descriptors at each region's start; an MMA's descriptor adds its
  // byte offset / 16 to the 14-bit start-address field (shared addresses stay
  // below 256 KB, so the field never carries).
  const uint64_t dC = sw128_desc(sbase + C::C_OFF, 16, 1024);         // Ct, K-major
  const uint64_t dB = sw128_desc(sbase + C::B_OFF, 16, 1024);         // Bh, K-major
  const uint64_t dBmn = sw128_desc(sbase + C::B_OFF, C::OPB, 1024);   // Bh, MN-major
  const uint64_t dX = sw128_desc(sbase + C::X_OFF, C::OPB, 1024);     // x, MN-major
  const uint64_t dG = sw128_desc(sbase + C::G_OFF, kN * 128, 1024);   // state, MN-major
  auto dadd = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
  uint32_t phase = 0, phase1 = 0, phase1b = 0, tphT = 0, tphM = 0;
  bool aborted = false;
  bool tpendT = false, tpendM = false;  // thread 0: TMA bytes expected on s_tbT / s_tbM

  // ---- incoming state: thread (n, cq) owns columns [CW*cq, CW*cq + CW) of row n
  const int n = 32 * qd + lane;
  const int p0 = CW * cq;
  float gst[CW];
  if (MODE == MODE_STATE) {
#pragma unroll
    for (int p = 0; p < CW; ++p) gst[p] = 0.f;
  } else if (seg == 0) {
    const int64_t so = ((b * H + h) * kN + n) * kP + p0;
#pragma unroll
    for (int p = 0; p < CW; ++p) gst[p] = a.h0 ? __ldg(a.h0 + so + p) : 0.f;
    if (a.B_prev && L > 0) {  // the left endpoint term waits for a token
      const float eps0 = (1.f - __ldg(a.lam + tokb * H + h)) * __ldg(a.dt + tokb * H + h);
      for (int r = 0; r < R; ++r) {
        const float bp = eps0 * io_load(a.B_prev, ((b * G + g) * R + r) * kN + n, true);
        const int64_t xo = ((b * H + h) * R + r) * kP + p0;
#pragma unroll
        for (int p = 0; p < CW; ++p) gst[p] = fmaf(bp, io_load(a.x_prev, xo + p, true), gst[p]);
      }
    }
  } else if (ti >= 0) {
    // Second half of a tail chain: the state-only pass over the first half
    // may still be running (this grid is its programmatic dependent), so wait
    // for it, then fold its summary here: G_1 = Rot(Phi_0) exp(Lam_0) G_0 + T_0
    // with G_0 the chain's initial state (rows n and n ^ 1 of a pair are
    // adjacent lanes).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t so = ((b * H + h) * kN + n) * kP + p0;
#pragma unroll
    for (int p = 0; p < CW; ++p) gst[p] = a.h0 ? __ldg(a.h0 + so + p) : 0.f;
    if (a.B_prev && L > 0) {
      const float eps0 = (1.f - __ldg(a.lam + tokb * H + h)) * __ldg(a.dt + tokb * H + h);
      for (int r = 0; r < R; ++r) {
        const float bp = eps0 * io_load(a.B_prev, ((b * G + g) * R + r) * kN + n, true);
        const int64_t xo = ((b * H + h) * R + r) * kP + p0;
#pragma unroll
        for (int p = 0; p < CW; ++p) gst[p] = fmaf(bp, io_load(a.x_prev, xo + p, true), gst[p]);
      }
    }
    const float* T = pl.wsT + (ti * kN + n) * kP + p0;
    const float* su = pl.wsSum + ti * (1 + kPairs);
    const float e = expf(su[0]);
    float sn, cs;
    sincosf(su[1 + (n >> 1)], &sn, &cs);
    const float ss = (n & 1) ? sn : -sn;  // even row: c u - s u'; odd row: c u + s u'
#pragma unroll
    for (int p = 0; p < CW; ++p) {
      const float u = e * gst[p];
      const float o = __shfl_xor_sync(0xffffffffu, u, 1);
      gst[p] = fmaf(cs, u, fmaf(ss, o, T[p]));
    }
  } else {
    const int64_t slot_in = (b * H + h) * pl.slots + (seg - 1);
    const float* src = pl.wsT + (slot_in * kN + n) * kP + p0;
#pragma unroll
    for (int p = 0; p < CW; p += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + p);
      gst[p] = v.x; gst[p + 1] = v.y; gst[p + 2] = v.z; gst[p + 3] = v.w;
    }
  }
  // The MMA4 operand: the chunk-start state times `scale`, bf16.
  auto store_state_bf16 = [&](float scale) {
#pragma unroll
    for (int c2 = 0; c2 < CW / 8; ++c2) {
      uint4 v;
      v.x = pack_bf16(scale * gst[8 * c2 + 0], scale * gst[8 * c2 + 1]);
      v.y = pack_bf16(scale * gst[8 * c2 + 2], scale * gst[8 * c2 + 3]);
      v.z = pack_bf16(scale * gst[8 * c2 + 4], scale * gst[8 * c2 + 5]);
      v.w = pack_bf16(scale * gst[8 * c2 + 6], scale * gst[8 * c2 + 7]);
      *reinterpret_cast<uint4*>(sm + C::G_OFF + sw128_off(n, (CW / 8) * cq + c2)) = v;
    }
  };

  // MODE_STATE summaries (pair k = n / 2): log-decay in log2 units, and the
  // angle in fp64 (thousands of radians over a long segment), stored mod 2 pi
  float l2seg = 0.f;
  double phi_seg = 0.0;
  const int64_t c_begin = seg * cps_c;
  const int64_t c_end = min(c_begin + cps_c, (L + Q - 1) / Q);

  // Prefetch of a chunk's inputs in three steps, each as soon as its buffer is
  // free: theta (TMA, on s_tbT) and the gates (cp.async) once the previous
  // chunk's angle prefix has been formed; raw C once MMA1 and MMA4 are done;
  // raw B and x once MMA2 (MODE_FULL) or MMA3 (MODE_STATE) is done.  B and C
  // land straight in the swizzled operand tiles and are rotated in place; x
  // lands in its MMA tile.  C, B and x complete on s_tbM, whose byte count
  // is declared by whichever of their steps comes first.
  constexpr uint32_t kTileBytes = Q * R * 128;  // one {64, R, Q} bf16 box
  constexpr uint32_t kMBytes = kTileBytes * (MODE == MODE_FULL ? 5 : 3);
  auto prefetch_early = [&](int64_t cn) {
    if (cn >= c_end || tid != 0) return;
    mbar_expect_tx(s_tbT, Q * kPairs * 4);
    tpendT = true;
    tma_load_3d(s_th, &maps.th, 0, (int)tg, (int)(tokb + cn * Q), s_tbT);
  };
  // The gates go to registers of the gate threads one chunk ahead (plain
  // loads: the prologue that uses them runs a whole chunk later): token tid's
  // dt, lam, A and the next token's dt, lam.
  float gr_dt = 0.f, gr_lm = 0.f, gr_av = 0.f, gr_dt1 = 0.f, gr_lm1 = 0.f;
  auto load_gates = [&](int64_t cn) {
    const int64_t cn0 = cn * Q;
    if (tid < Q) {
      const int64_t t0 = cn0 + tid, i0 = (tokb + t0) * H + h;
      const bool v0 = cn < c_end && t0 < L, v1 = cn < c_end && t0 + 1 < L;
      gr_dt = v0 ? ldg_early(a.dt + i0) : 0.f;
      gr_lm = v0 ? ldg_early(a.lam + i0) : 0.f;
      gr_av = v0 ? ldg_early(a.A + i0) : 0.f;
      gr_dt1 = v1 ? ldg_early(a.dt + i0 + H) : 0.f;
      gr_lm1 = v1 ? ldg_early(a.lam + i0 + H) : 0.f;
    }
  };
  auto arm_m = [&]() {  // thread 0
    if (!tpendM) {
      mbar_expect_tx(s_tbM, kMBytes);
      tpendM = true;
    }
  };
  auto prefetch_c = [&](int64_t cn) {
    if (MODE != MODE_FULL || cn >= c_end || tid != 0) return;
    arm_m();
    const int tok = (int)(tokb + cn * Q);
    tma_load_3d(sm + C::C_OFF, &maps.c, 0, (int)(g * R), tok, s_tbM);
    tma_load_3d(sm + C::C_OFF + C::OPB, &maps.c, 64, (int)(g * R), tok, s_tbM);
  };
  auto prefetch_bx = [&](int64_t cn) {
    if (cn >= c_end || tid != 0) return;
    arm_m();
    const int tok = (int)(tokb + cn * Q);
    tma_load_3d(sm + C::X_OFF, &maps.x, 0, (int)(h * R), tok, s_tbM);
    tma_load_3d(sm + C::B_OFF, &maps.b, 0, (int)(g * R), tok, s_tbM);
    tma_load_3d(sm + C::B_OFF + C::OPB, &maps.b, 64, (int)(g * R), tok, s_tbM);
  };

  // Chunk prologue: gates, the chunk-local log-decay prefix Lam_t (log2
  // units) and the cumulative angles.  Leaves the angle increments `ang` and
  // the slot prefix `phi` of this thread's rotation tokens in registers,
  // gamma, delta, Lam, u, the diagonal factor and the chunk-end angles in
  // shared memory, and the chunk's total decay in `l2end`.  Needs only theta and the gates, so it
  // runs while the chunk's B, C and x are still in flight.
  float2 ang[TQ][2];
  float phi[4];
  float l2end = 0.f;
  auto prologue = [&](int64_t cc) -> bool {
    const int nt = (int)min((int64_t)Q, L - cc * Q);
    const bool slot_live = tq < SLOTS;
    const bool gate_warp = warp < (Q + 31) / 32;
    if (gate_warp) {  // whole warps take part in the shuffle scan of Lam
      // loaded as zeros past the sequence end
      const float g_dt = gr_dt, g_lm = gr_lm, g_av = gr_av, g_nx = (1.f - gr_lm1) * gr_dt1;
      const bool inq = tid < Q;
      if (inq) {
        s_gam[tid] = g_lm * g_dt;
        s_del[tid] = g_lm * g_dt + g_nx;
        s_dtv[tid] = g_dt;
      }
      float v = g_dt * g_av * kL2E;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      if (inq) s_lg[tid] = v;
    }
    const bool okt = (tid == 0) ? wait_bar(s_tbT, tphT, a.status) : true;
    if (okt && tid == 0) { tpendT = false; tphT ^= 1; }  // on a timeout the phase stays
    if (__syncthreads_or(!okt)) return false;  // theta, gates and each warp's Lam visible
    if (Q > 32 && tid >= 32 && tid < Q) s_lg[tid] += s_lg[31];  // second warp of tokens
    // cumulative angles of pairs 4kg..4kg+3 over this slot's tokens
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < TQ; ++u) {
      const int t = tq * TQ + u;
      const bool live_t = slot_live && t < nt;
      const float d = live_t ? s_dtv[t] : 0.f;
      const float4 th = live_t ? *reinterpret_cast<const float4*>(s_th + t * kPairs + 4 * kg)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      ang[u][0] = make_float2(d * th.x, d * th.y);
      ang[u][1] = make_float2(d * th.z, d * th.w);
      part[0] += ang[u][0].x; part[1] += ang[u][0].y;
      part[2] += ang[u][1].x; part[3] += ang[u][1].y;
    }
    if (!C::PART_OWN) __syncthreads();  // theta read: the slot sums go over it
    // slot sums: row = slot, 16-byte piece kg at position kg ^ (slot % 8)
    auto part_at = [&](int slot, int k4) { return s_part + slot * kPairs + 4 * (k4 ^ (slot & 7)); };
    if (slot_live)
      *reinterpret_cast<float4*>(part_at(tq, kg)) = make_float4(part[0], part[1], part[2], part[3]);
    __syncthreads();  // Lam complete, slot sums written
    {  // exclusive prefix over the slots: warp w scans pieces kg of 32 / SLOTS groups,
       // lane = slot within its group; the chunk-end angles are the group totals
      static_assert(SLOTS == NTH / 16 && SLOTS <= 32, "one scan lane per slot and piece");
      const int sl = lane % SLOTS;
      const int k4 = warp * (32 / SLOTS) + lane / SLOTS;
      float* pp = part_at(sl, k4);
      const float4 o = *reinterpret_cast<const float4*>(pp);
      float v[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int off = 1; off < SLOTS; off <<= 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float u = __shfl_up_sync(0xffffffffu, v[j], off, SLOTS);
          if (sl >= off) v[j] += u;
        }
      }
      *reinterpret_cast<float4*>(pp) = make_float4(v[0] - o.x, v[1] - o.y, v[2] - o.z, v[3] - o.w);
      if (sl == SLOTS - 1) *reinterpret_cast<float4*>(s_phe + 4 * k4) = make_float4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();  // slot prefixes and chunk-end angles written
    if (slot_live) {
      const float4 o = *reinterpret_cast<const float4*>(part_at(tq, kg));
      phi[0] = o.x; phi[1] = o.y; phi[2] = o.z; phi[3] = o.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) phi[j] = 0.f;
    }
    l2end = s_lg[nt - 1];
    // Row scale of Bh: exp(ref - Lam_s) delta_s in the factored form,
    // delta_s in the plain one; a state-only pass has no scores, so its Bh
    // carries the chunk-state weights exp(Lam_end - Lam_s) delta_s directly
    // (a weight that underflows belongs to a negligible term).
    if (tid < Q) {
      const float lg = s_lg[tid], del = s_del[tid];
      float u;
      if (MODE == MODE_STATE) u = ex2(l2end - lg) * del;
      else if (l2end > kPlainL2) u = ex2(0.5f * l2end - lg) * del;
      else u = del;
      s_u[tid] = (tid < nt) ? u : 0.f;
      s_d[tid] = (tid < nt && del > 0.f) ? s_gam[tid] / del : 0.f;
    } else if (tid < Q + kPairs) {  // cos, sin of the chunk-end angles (state update)
      float sn, cs;
      sincosf(s_phe[tid - Q], &sn, &cs);
      s_pcs[tid - Q] = make_float2(cs, sn);
    }
    return true;
  };

  if (a.test_timeout) {  // diagnostics: this wait must end in M3_ERR_TIMEOUT after 1 ms
    const bool okn = (tid == 0) ? wait_bar(s_never, 0, a.status, 1000000ull) : true;
    if (__syncthreads_or(!okn)) aborted = true;
  }
  if (!aborted) {
    prefetch_early(c_begin);
    prefetch_c(c_begin);
    prefetch_bx(c_begin);
    load_gates(c_begin);
    if (c_begin < c_end && !prologue(c_begin)) aborted = true;
  }

  for (int64_t c = c_begin; c < c_end && !aborted; ++c) {
    const int64_t c0 = c * Q;
    const int nt = (int)min((int64_t)Q, L - c0);
    const bool slot_live = tq < SLOTS;
    const float l2ref = 0.5f * l2end;  // the factored form's reference (log2 units)
    const bool plain = MODE == MODE_FULL && l2end <= kPlainL2;  // chunk-uniform

    load_gates(c + 1);  // consumed by the next chunk's prologue, at the end of this one
    // the last chunk's staged y must be read before the staging block is reused
    if (MODE == MODE_FULL && tid == 0) bulk_wait_read0();
    const bool okm = (tid == 0) ? wait_bar(s_tbM, tphM, a.status) : true;
    if (okm && tid == 0) { tpendM = false; tphM ^= 1; }  // on a timeout the phase stays
    if (__syncthreads_or(!okm)) { aborted = true; break; }  // B, C and x of this chunk visible
    // every thread has read theta and the slot sums over it (the prologue): the
    // theta buffer takes the next chunk's
    prefetch_early(c + 1);

    // ---- operands: Bh = u Bt (and Ct) rotated by -Phi_t in place (16-byte pieces)
    if (slot_live) {
      const uint32_t kboff = (uint32_t)(kg >> 3) * C::OPB;
      const uint32_t chk = (uint32_t)(kg & 7);
#pragma unroll
      for (int u = 0; u < TQ; ++u) {
        const int t = tq * TQ + u;
        const bool live_t = t < nt;  // rows past the chunk end become zeros
        phi[0] += ang[u][0].x; phi[1] += ang[u][0].y;
        phi[2] += ang[u][1].x; phi[3] += ang[u][1].y;
        float cs[4], sn[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) __sincosf(reduce_2pi(phi[j]), &sn[j], &cs[j]);
        // two pairs at a time as (even elements, odd elements) fp32x2 vectors:
        // (b0, b1) -> (c b0 + s b1, c b1 - s b0) for each pair; B's rows also
        // take their scale u_t
        const float us = live_t ? s_u[t] : 0.f;
        const float2 c2[2] = {make_float2(cs[0], cs[1]), make_float2(cs[2], cs[3])};
        const float2 s2[2] = {make_float2(sn[0], sn[1]), make_float2(sn[2], sn[3])};
        const float2 n2[2] = {make_float2(-sn[0], -sn[1]), make_float2(-sn[2], -sn[3])};
        const float2 u2 = make_float2(us, us);
        const float2 cb2[2] = {fmul2(u2, c2[0]), fmul2(u2, c2[1])};
        const float2 sb2[2] = {fmul2(u2, s2[0]), fmul2(u2, s2[1])};
        const float2 nb2[2] = {fmul2(u2, n2[0]), fmul2(u2, n2[1])};
        auto rot4 = [&](const uint4 in, uint32_t (&o)[4], const float2 (&cv)[2],
                        const float2 (&sv)[2], const float2 (&nv)[2]) {
          const uint32_t iw[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float2 e = make_float2(__uint_as_float(iw[2 * q] << 16),
                                         __uint_as_float(iw[2 * q + 1] << 16));
            const float2 d = make_float2(__uint_as_float(iw[2 * q] & 0xffff0000u),
                                         __uint_as_float(iw[2 * q + 1] & 0xffff0000u));
            const float2 oe = ffma2(cv[q], e, fmul2(sv[q], d));
            const float2 od = ffma2(cv[q], d, fmul2(nv[q], e));
            o[2 * q] = pack_bf16(oe.x, od.x);
            o[2 * q + 1] = pack_bf16(oe.y, od.y);
          }
        };
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t off = kboff + sw128_off(t * R + r, chk);
          uint32_t ob[4], oc[4];
          uint4 rb = *reinterpret_cast<const uint4*>(sm + C::B_OFF + off);
          uint4 rc = make_uint4(0, 0, 0, 0);
          if (MODE == MODE_FULL) rc = *reinterpret_cast<const uint4*>(sm + C::C_OFF + off);
          if (!live_t) { rb = make_uint4(0, 0, 0, 0); rc = make_uint4(0, 0, 0, 0); }
          rot4(rb, ob, cb2, sb2, nb2);
          if (MODE == MODE_FULL) rot4(rc, oc, c2, s2, n2);
          *reinterpret_cast<uint4*>(sm + C::B_OFF + off) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
          if (MODE == MODE_FULL)
            *reinterpret_cast<uint4*>(sm + C::C_OFF + off) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
        }
      }
    }

    // ---- the MMA4 operand: the chunk-start state, times exp(ref) when factored
    // (every MMA of the previous chunk is complete, so its tile is free)
    if (MODE == MODE_FULL) store_state_bf16(plain ? 1.f : ex2(l2ref));
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA3 (chunk state) and MMA4 (Ct G), then MMA1 (scores) ----------------
    // MMA4: Ct G' for tile mt into TMEM column `col` (one thread); `acc`: add
    // to what the column holds
    auto issue_mma4 = [&](int mt, int col, bool acc) {
      const uint32_t id4 = idesc_bf16(MT, kP, 0, 1);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint64_t ad = dadd(dC, kb * C::OPB + mt * MT * 128 + k4 * 32);
            const uint64_t bd = dadd(dG, (kb * 4 + k4) * 2048);
            mma_bf16_ss(tm + col, ad, bd, id4, acc || (kb | k4) != 0);
          }
    };
    auto issue_mma3 = [&]() {  // Sc' = Bh^T x (one thread)
      const uint32_t id3 = idesc_bf16(kN, kP, 1, 1);
#pragma unroll
      for (int ks = 0; ks < M / 16; ++ks) {
        const uint64_t ad = dadd(dBmn, ks * 2048);
        const uint64_t bd = dadd(dX, ks * 2048);
        if constexpr (NT == 2) {  // two row halves as interleaved chains
          const int hf = ks & 1, kst = (ks >> 1) + 8 * hf;
          mma_bf16_ss(tm + (hf ? C::SC2_COL : C::SC_COL), dadd(dBmn, kst * 2048), dadd(dX, kst * 2048),
                      id3, ks > 1);
        } else
          mma_bf16_ss(tm + C::SC_COL, ad, bd, id3, ks != 0);
      }
    };
    auto issue_mma1 = [&]() {  // S' = Ct Bh^T per tile, each on its own barrier (one thread)
#pragma unroll
      for (int mt = 0; mt < NT; ++mt) {
        const uint32_t id = idesc_bf16(MT, (mt + 1) * MT, 0, 0);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint64_t ad = dadd(dC, kb * C::OPB + mt * MT * 128 + k4 * 32);
            const uint64_t bd = dadd(dB, kb * C::OPB + k4 * 32);
            mma_bf16_ss(tm + C::s_col(mt), ad, bd, id, (kb | k4) != 0);
          }
        mma_commit(mt == 0 ? s_bar1 : s_bar1b);
      }
    };
    if (tid == 0) {
      if (MODE == MODE_STATE) {
        issue_mma3();
        mma_commit(s_bar);
      } else if (NT == 2 && !plain) {  // tile 0's scores and both chunk-state halves interleaved
        const uint32_t id3 = idesc_bf16(kN, kP, 1, 1);
        const uint32_t id0 = idesc_bf16(MT, MT, 0, 0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mma_bf16_ss(tm + C::s_col(0), dadd(dC, (k >> 2) * C::OPB + (k & 3) * 32),
                      dadd(dB, (k >> 2) * C::OPB + (k & 3) * 32), id0, k != 0);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // rows 16 (k + 8 hf) .. of half hf
            const uint32_t kst = (uint32_t)(k + 8 * hf);
            mma_bf16_ss(tm + (hf ? C::SC2_COL : C::SC_COL), dadd(dBmn, kst * 2048), dadd(dX, kst * 2048),
                        id3, k != 0);
          }
        }
        mma_commit(s_bar);
        mma_commit(s_bar1);
        // tile 1's scores follow once the chunk state is done (below), so that
        // they run under the state update instead of ahead of it
      } else if (!plain) {  // one tile: scores, Ct G and the chunk state as three interleaved chains
        static_assert(NT == 2 || M / 16 <= 8, "one-tile chunk state in at most 8 K steps");
        const uint32_t id1 = idesc_bf16(MT, MT, 0, 0);
        const uint32_t id3 = idesc_bf16(kN, kP, 1, 1);
        const uint32_t id4 = idesc_bf16(MT, kP, 0, 1);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t ko = (k >> 2) * C::OPB + (k & 3) * 32;  // K step k of N = 128
          mma_bf16_ss(tm + C::s_col(0), dadd(dC, ko), dadd(dB, ko), id1, k != 0);
          mma_bf16_ss(tm + C::acc_col(0), dadd(dC, ko), dadd(dG, k * 2048), id4, k != 0);
          if (k < M / 16) mma_bf16_ss(tm + C::SC_COL, dadd(dBmn, k * 2048), dadd(dX, k * 2048), id3, k != 0);
        }
        mma_commit(s_bar);
        mma_commit(s_bar1);
      } else {  // plain form: the scores read Bh before it is rescaled for MMA3
        if (C::EARLY4) issue_mma4(0, C::y2_col(0), false);
        issue_mma1();
      }
    }
    if (plain) {  // chunk-uniform branch
      bool okp = true;
      if (tid == 0) {  // both score tiles done (waited again, same phase, below)
        okp = wait_bar(s_bar1, phase1, a.status);
        if (okp && NT == 2) okp = wait_bar(s_bar1b, phase1b, a.status);
      }
      if (__syncthreads_or(!okp)) { aborted = true; break; }
      // Bh_s <- exp(Lam_end - Lam_s) Bh_s = w_s Bt_s, the chunk-state weights
      for (int q = tid; q < M * 16; q += NTH) {
        const int row = q >> 4, t = row / R;
        if (t >= nt) continue;  // rows past the end are zero
        const float f = ex2(l2end - s_lg[t]);
        uint8_t* pq = sm + C::B_OFF + ((q >> 3) & 1) * C::OPB + sw128_off(row, q & 7);
        const uint4 v = *reinterpret_cast<const uint4*>(pq);
        const uint32_t iv[4] = {v.x, v.y, v.z, v.w};
        uint32_t ov[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 g = fmul2(make_float2(f, f), make_float2(__uint_as_float(iv[e] << 16),
                                                                __uint_as_float(iv[e] & 0xffff0000u)));
          ov[e] = pack_bf16(g.x, g.y);
        }
        *reinterpret_cast<uint4*>(pq) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
        if constexpr (NT == 2 && MODE == MODE_FULL) {
          // two-tile chunks: Ct_t <- exp(Lam_t) Ct_t, so that Ct G lands in the
          // one output accumulator already scaled (MMA1 has read Ct)
          const float fc = ex2(s_lg[t]);
          uint8_t* pc = sm + C::C_OFF + ((q >> 3) & 1) * C::OPB + sw128_off(row, q & 7);
          const uint4 w = *reinterpret_cast<const uint4*>(pc);
          const uint32_t iw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 g = fmul2(make_float2(fc, fc), make_float2(__uint_as_float(iw[e] << 16),
                                                                  __uint_as_float(iw[e] & 0xffff0000u)));
            ov[e] = pack_bf16(g.x, g.y);
          }
          *reinterpret_cast<uint4*>(pc) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        issue_mma3();
        mma_commit(s_bar);
      }
    }
    const bool ok3 = (tid == 0) ? wait_bar(s_bar, phase, a.status) : true;
    phase ^= 1;
    if (__syncthreads_or(!ok3)) { aborted = true; break; }
    tc_fence_after();
    if (MODE == MODE_FULL && NT == 2 && !plain && tid == 0) {  // tile 1's scores (N = 256)
      const uint32_t id1 = idesc_bf16(MT, 2 * MT, 0, 0);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ss(tm + C::s_col(1), dadd(dC, (k >> 2) * C::OPB + MT * 128 + (k & 3) * 32),
                    dadd(dB, (k >> 2) * C::OPB + (k & 3) * 32), id1, k != 0);
      mma_commit(s_bar1b);
    }
    if (MODE == MODE_STATE) prefetch_bx(c + 1);  // B and x are free once MMA3 is done

    // ---- state update G <- Rot(Phi_end) (exp(Lam_end) G + Sc), under MMA1 -------
    //      (Sc = exp(Lam_end - ref) Sc' when factored)
    {
      const float phe = s_phe[n >> 1];
      const float2 pcs = s_pcs[n >> 1];
      const float cs = pcs.x, sn = pcs.y;
      const float el = ex2(l2end);
      const float sc = (MODE == MODE_FULL && !plain) ? ex2(l2end - l2ref) : 1.f;
      const float ss = (n & 1) ? sn : -sn;  // even row: c v - s o; odd row: c v + s o
#pragma unroll
      for (int pc = 0; pc < CW / 16; ++pc) {
        uint32_t sv[16];
        tmem_ld16(tm + lane_base + C::SC_COL + CW * cq + 16 * pc, sv);
        if constexpr (NT == 2) {  // the second half of the rows
          uint32_t sw[16];
          tmem_ld16(tm + lane_base + C::SC2_COL + CW * cq + 16 * pc, sw);
          tmem_ld_wait();
#pragma unroll
          for (int p = 0; p < 16; ++p) sv[p] = __float_as_uint(__uint_as_float(sv[p]) + __uint_as_float(sw[p]));
        }
        tmem_ld_wait();
#pragma unroll
        for (int p = 0; p < 16; p += 2) {
          const int pp = 16 * pc + p;
          const float2 v = ffma2(make_float2(el, el), make_float2(gst[pp], gst[pp + 1]),
                                 fmul2(make_float2(sc, sc), make_float2(__uint_as_float(sv[p]),
                                                                        __uint_as_float(sv[p + 1]))));
          const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v.x, 1),
                                       __shfl_xor_sync(0xffffffffu, v.y, 1));
          const float2 w = ffma2(make_float2(cs, cs), v, fmul2(make_float2(ss, ss), o));
          gst[pp] = w.x;
          gst[pp + 1] = w.y;
        }
      }
      if (MODE == MODE_STATE) {
        l2seg += l2end;
        phi_seg += (double)phe;
      }
    }

    if (MODE == MODE_FULL) {
      const bool ok1 = (tid == 0) ? wait_bar(s_bar1, phase1, a.status) : true;
      phase1 ^= 1;
      tc_fence_before();  // the chunk-state columns are read
      if (__syncthreads_or(!ok1)) { aborted = true; break; }
      tc_fence_after();
      if (C::EARLY4) prefetch_c(c + 1);  // MMA1 and MMA4 have read Ct
      if constexpr (NT == 2) {  // Ct G of both tiles, interleaved, into the freed state columns
        if (tid == 0) {
          const uint32_t id4 = idesc_bf16(MT, kP, 0, 1);
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
              mma_bf16_ss(tm + C::acc2_col(mt), dadd(dC, (k >> 2) * C::OPB + mt * MT * 128 + (k & 3) * 32),
                          dadd(dG, k * 2048), id4, k != 0);
        }
      }

      // ---- per score tile: mask into P (bf16, K-major), then its MMA2 (P x) -----
      //   factored: P'[(t,r),(s,r')] = S' * (s < t ? 1 : s == t ? gamma_t / delta_t : 0)
      //   plain:    P [(t,r),(s,r')] = S' * (s < t ? exp(Lam_t - Lam_s) : s == t ? gamma_t / delta_t : 0)
      // With two tiles, tile 1's mask runs while tile 0's MMA2 and MMA4 run.
#pragma unroll
      for (int mt = 0; mt < NT; ++mt) {
        if (mt == 1) {  // tile 1's scores
          const bool okb = (tid == 0) ? wait_bar(s_bar1b, phase1b, a.status) : true;
          phase1b ^= 1;
          if (__syncthreads_or(!okb)) { aborted = true; break; }
          tc_fence_after();
        }
        // 64-row tiles fill lanes 0-15 of each warp's TMEM quadrant: both
        // half-warps take those 16 rows, each half 16 of the warp's columns
        const int rho0 = (MT == 64) ? 16 * qd : 32 * qd;     // the warp's first row
        const int rho = rho0 + ((MT == 64) ? (lane & 15) : lane);
        const int hsel = (MT == 64) ? (lane >> 4) : 0;        // column half (64-row tiles)
        const int t = (mt * MT + rho) / R;
        const bool trow = t < nt;
        const int t_hi = (mt * MT + rho0 + ((MT == 64) ? 15 : 31)) / R;  // the warp's last token
        const float lgt = trow ? s_lg[t] : 0.f;
        const float dgt = trow ? s_d[t] : 0.f;
        const int cpt = (mt + 1) * MT / CQN;  // columns per thread, a multiple of 32
        static_assert((MT / CQN) % 32 == 0, "mask columns per thread");
        // 16 masked columns (16 / R tokens from s0) of v, packed to bf16
        auto mask16 = [&](const uint32_t* v, int s0, uint32_t* pk) {
          if (!plain && s0 + 16 / R - 1 < t) {  // wholly below the diagonal: S' as it is
#pragma unroll
            for (int j = 0; j < 16; j += 2)
              pk[j / 2] = pack_bf16(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            return;
          }
          float mk[16 / R];
#pragma unroll
          for (int q4 = 0; q4 < 16 / R / 4; ++q4) {
            const int sb = s0 + 4 * q4;
            float f[4] = {1.f, 1.f, 1.f, 1.f};
            if (plain) {
              const float4 l4 = *reinterpret_cast<const float4*>(s_lg + sb);
              f[0] = ex2(lgt - l4.x); f[1] = ex2(lgt - l4.y);
              f[2] = ex2(lgt - l4.z); f[3] = ex2(lgt - l4.w);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
              mk[4 * q4 + e] = sb + e < t ? f[e] : (sb + e == t ? dgt : 0.f);
          }
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 fm = fmul2(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                    make_float2(mk[j / R], mk[(j + 1) / R]));
            pk[j / 2] = pack_bf16(fm.x, fm.y);
          }
        };
        if (MT == 64) {  // one 32-column block per warp; each half-warp masks 16 of them
          const int c0 = cq * cpt;             // the warp's first column
          const int cth = c0 + 16 * hsel;      // this thread's first column
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) pk[j] = 0u;
          if (c0 / R <= t_hi) {  // warp-uniform: blocks wholly above the diagonal stay zero
            uint32_t v[16];
            tmem_ld16x2<16>(tm + lane_base + C::s_col(mt) + c0, v);
            tmem_ld_wait();
            if (trow) mask16(v, cth / R, pk);
          }
          uint8_t* blk = sm + C::p_off(mt);  // K = 64: one block
          const int ch0 = cth / 8;
          *reinterpret_cast<uint4*>(blk + sw128_off(rho, ch0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(blk + sw128_off(rho, ch0 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else if constexpr (NT == 2) {
          // P' in TMEM: step st reads the warp's score columns [16 st, +16)
          // and stores their packed bf16 over columns [8 st, +8), which this
          // or an earlier step has read (K step j of the tile: part
          // 16 j / cpt, 8-column step j mod (cpt / 16))
          const uint32_t pbase = tm + lane_base + C::s_col(mt) + cq * cpt;
          for (int st = 0; st < cpt / 16; ++st) {
            const int s0 = (cq * cpt + 16 * st) / R;  // first key token of the step
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[j] = 0u;
            if (s0 <= t_hi) {  // warp-uniform: steps wholly above the diagonal stay zero
              uint32_t v[16];
              tmem_ld16(pbase + 16 * st, v);
              tmem_ld_wait();
              if (trow) mask16(v, s0, pk);
            }
            tmem_st8(pbase + 8 * st, pk);
          }
          tmem_st_wait();
        } else {
          for (int cc = cq * cpt / 16; cc < (cq + 1) * cpt / 16; cc += 2) {
            const int s0 = cc * 16 / R;  // first token of these 32 columns
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = 0u;
            if (s0 <= t_hi) {  // warp-uniform: blocks wholly above the diagonal stay zero
              uint32_t v[32];
              tmem_ld32(tm + lane_base + C::s_col(mt) + cc * 16, v);
              tmem_ld_wait();
              if (trow) {
                mask16(v, s0, pk);
                mask16(v + 16, s0 + 16 / R, pk + 8);
              }
            }
            const int kb = (cc * 16) / 64;
            uint8_t* blk = sm + C::p_off(mt) + kb * MT * 128;
            const int ch0 = ((cc * 16) % 64) / 8;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(blk + sw128_off(rho, ch0 + q)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (NT == 2 && tid == 0) {  // P' x onto Ct G, P' from TMEM
          const uint32_t id2 = idesc_bf16(MT, kP, 0, 1);
          const int cps = cpt / 16;  // K steps per part
#pragma unroll 4
          for (int j = 0; j < (mt + 1) * MT / 16; ++j)
            mma_bf16_ts(tm + C::acc2_col(mt), tm + C::s_col(mt) + cpt * (j / cps) + 8 * (j % cps),
                        dadd(dX, j * 2048), id2, 1);
          if (mt == NT - 1) mma_commit(s_bar);
        } else if (tid == 0) {  // MMA2 for this tile (and MMA4 for two-tile chunks)
          const uint32_t id2 = idesc_bf16(MT, kP, 0, 1);
          const int kblocks = (mt + 1) * MT / 64;
          // factored: one accumulator, Ct G' (MMA4) first; plain: P x alone
          int col = C::y_col(mt);
          bool acc = false;
          if (!plain) {
            col = C::acc_col(mt);
            if (!C::EARLY4) issue_mma4(mt, col, false);
            acc = true;
          }
          for (int kb = 0; kb < kblocks; ++kb)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint64_t ad = dadd(mt == 0 && NT == 2 ? dadd(dC, C::ST_OFF - C::C_OFF) : dB,
                                       kb * MT * 128 + k4 * 32);  // P in the staging block or over Bh
              const uint64_t bd = dadd(dX, (kb * 4 + k4) * 2048);
              mma_bf16_ss(tm + col, ad, bd, id2, acc || (kb | k4) != 0);
            }
          if (plain && !C::EARLY4) issue_mma4(mt, C::y2_col(mt), false);
          if (mt == NT - 1) mma_commit(s_bar);
        }
      }
      if (aborted) break;
      const bool ok2 = (tid == 0) ? wait_bar(s_bar, phase, a.status) : true;
      phase ^= 1;
      if (__syncthreads_or(!ok2)) { aborted = true; break; }
      tc_fence_after();
      prefetch_bx(c + 1);                 // MMA2 has read P (over Bh) and x
      if (!C::EARLY4) prefetch_c(c + 1);  // MMA4 has read Ct

      // ---- epilogue, staged in the staging block: y = exp(Lam_t - ref) Y'
      //      (factored), y = Y + exp(Lam_t) Y2 (plain) --------------------------
#pragma unroll
      for (int mt = 0; mt < NT; ++mt) {
        // 64-row tiles: both half-warps take the warp's 16 rows, each half
        // 16 of the thread group's columns (see the mask)
        const int rho = (MT == 64) ? 16 * qd + (lane & 15) : 32 * qd + lane;
        const int i = mt * MT + rho;  // row (t, r) of the chunk
        const int t = i / R;
        // plain: (1, exp(Lam_t)) on (Y, Y2); factored: exp(Lam_t - ref) on Y'.
        // Two-tile chunks keep one accumulator in both forms (the plain form's
        // Ct G is scaled through Ct), at acc2_col.
        const bool two = plain && NT != 2;
        const float el = (t < nt) ? ((NT == 2 && plain) ? 1.f : ex2(plain ? s_lg[t] : s_lg[t] - l2ref)) : 0.f;
        const int ycol = NT == 2 ? C::acc2_col(mt) : plain ? C::y_col(mt) : C::acc_col(mt);
        constexpr int NPC = (MT == 64) ? CW / 32 : CW / 16;  // 16-column pieces per thread
        static_assert(MT != 64 || CW % 32 == 0, "64-row tiles: 32 columns per thread group");
#pragma unroll
        for (int pc = 0; pc < NPC; ++pc) {
          uint32_t yv[16], zv[16];
          int col;  // this thread's first column
          if (MT == 64) {
            col = CW * cq + 32 * pc + 16 * (lane >> 4);
            tmem_ld16x2<16>(tm + lane_base + ycol + CW * cq + 32 * pc, yv);
            if (two) tmem_ld16x2<16>(tm + lane_base + C::y2_col(mt) + CW * cq + 32 * pc, zv);
          } else {
            col = CW * cq + 16 * pc;
            tmem_ld16(tm + lane_base + ycol + col, yv);
            if (two) tmem_ld16(tm + lane_base + C::y2_col(mt) + col, zv);
          }
          tmem_ld_wait();
          {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = q * 8 + 2 * e;
                const float2 yy = make_float2(__uint_as_float(yv[j]), __uint_as_float(yv[j + 1]));
                const float2 f =
                    two ? ffma2(make_float2(el, el),
                                  make_float2(__uint_as_float(zv[j]), __uint_as_float(zv[j + 1])), yy)
                          : fmul2(make_float2(el, el), yy);
                w4[e] = pack_bf16(f.x, f.y);
              }
              *reinterpret_cast<uint4*>(sm + C::ST_OFF + sw128_off(i, col / 8 + q)) =
                  make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
      }
      fence_async_smem();  // staged y visible to the bulk store
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (MODE == MODE_FULL) {
      if (!a.cu_seqlens) {  // y of this chunk: one bulk tensor store, clipped at the sequence end
        if (tid == 0) {
          tma_store_4d(&maps.y, sm + C::ST_OFF, 0, (int)(h * R), (int)c0, (int)b);
          bulk_commit();
        }
      } else if (nt == Q) {  // packed batch: a whole chunk by the bulk store
        if (tid == 0) {
          tma_store_4d(&maps.y, sm + C::ST_OFF, 0, (int)(h * R), (int)(tokb + c0), 0);
          bulk_commit();
        }
      } else {  // packed batch, a sequence's last partial chunk: the next sequence's rows
                // follow, so only its nt * R rows are written (16-byte pieces)
        const int pieces = nt * R * 8;
        for (int e = tid; e < pieces; e += NTH) {
          const int i = e >> 3, j = e & 7, t = i / R, r = i % R;
          const uint4 v = *reinterpret_cast<const uint4*>(sm + C::ST_OFF + sw128_off(i, j));
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.y) +
                               (((tokb + c0 + t) * H + h) * R + r) * kP + 8 * j;
          *reinterpret_cast<uint4*>(dst) = v;
        }
      }
    }
    // the next chunk's gates and angles overlap its B, C, x loads
    if (c + 1 < c_end && !prologue(c + 1)) { aborted = true; break; }
  }

  if (!aborted) {
    if (MODE == MODE_FULL) {
      if (seg == nseg_c - 1 && a.final_state) {
        float* dst = a.final_state + ((b * H + h) * kN + n) * kP + p0;
#pragma unroll
        for (int p = 0; p < CW; p += 4)
          *reinterpret_cast<float4*>(dst + p) = make_float4(gst[p], gst[p + 1], gst[p + 2], gst[p + 3]);
      }
    } else {
      const int64_t slot = ti >= 0 ? ti : (b * H + h) * pl.slots + seg;
      float* dst = pl.wsT + (slot * kN + n) * kP + p0;
#pragma unroll
      for (int p = 0; p < CW; p += 4)
        *reinterpret_cast<float4*>(dst + p) = make_float4(gst[p], gst[p + 1], gst[p + 2], gst[p + 3]);
      float* su = pl.wsSum + slot * (1 + kPairs);
      if (tid == 0) su[0] = l2seg * kLn2;
      if (cq == 0 && (n & 1) == 0) su[1 + (n >> 1)] = (float)remainder(phi_seg, 6.283185307179586);
    }
  }
  // an aborted run may leave a prefetch in flight: let it land (bounded wait)
  if (tid == 0 && tpendT) wait_bar(s_tbT, tphT, a.status);
  if (tid == 0 && tpendM) wait_bar(s_tbM, tphM, a.status);
  if (MODE == MODE_FULL && tid == 0) bulk_wait0();  // y stores complete
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, C::TMEM_COLS);
}

// Combine segment summaries into each segment's incoming state (fp32).
// Thread (k, p) of chain (b, h): G_0 = h0 + (1 - lam_0) dt_0 B_prev x_prev^T,
// G_{s+1} = Rot(Phi_s) exp(Lam_s) G_s + T_s, stored over T_s.
// TO_FINAL: fold every segment and write the chain's final state (state-only
// calls) instead of the incoming state of each later segment.
template <bool TO_FINAL>
__global__ void __launch_bounds__(256) tc_seg_pass_kernel(const ScanArgs a, const TcPlan pl) {
  const int64_t b = blockIdx.z, h = blockIdx.y;
  const int64_t nsum = TO_FINAL ? pl.nseg : pl.nseg - 1, slot0 = (b * a.nheads + h) * pl.slots;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= kPairs * kP) return;
  const int k = idx / kP, p = idx % kP;
  const int64_t H = a.nheads, R = a.R, G = a.ngroups;
  const int64_t g = h / (H / G);
  const Chain chn = chain_of(a, b);
  const int64_t so = (b * H + h) * kN * kP;
  if (!M3_IN(b, a.batch, a.status) || !M3_IN(h, H, a.status)) return;
  float g0 = a.h0 ? a.h0[so + (2 * k) * kP + p] : 0.f;
  float g1 = a.h0 ? a.h0[so + (2 * k + 1) * kP + p] : 0.f;
  if (a.B_prev && chn.len > 0) {  // the left endpoint term waits for a token
    const float eps = (1.f - a.lam[chn.base * H + h]) * a.dt[chn.base * H + h];
    for (int r = 0; r < R; ++r) {
      const int64_t bb = ((b * G + g) * R + r) * kN;
      const float xv = io_load(a.x_prev, ((b * H + h) * R + r) * kP + p, true);
      g0 = fmaf(eps * io_load(a.B_prev, bb + 2 * k, true), xv, g0);
      g1 = fmaf(eps * io_load(a.B_prev, bb + 2 * k + 1, true), xv, g1);
    }
  }
  for (int64_t s = 0; s < nsum; ++s) {
    const int64_t slot = slot0 + s;
    float* T = pl.wsT + slot * kN * kP;
    const float* su = pl.wsSum + slot * (1 + kPairs);
    const float e = expf(su[0]);
    float sn, cs;
    sincosf(su[1 + k], &sn, &cs);
    const float u0 = e * g0, u1 = e * g1;
    const float n0 = cs * u0 - sn * u1 + T[(2 * k) * kP + p];
    const float n1 = sn * u0 + cs * u1 + T[(2 * k + 1) * kP + p];
    if (!TO_FINAL) {
      T[(2 * k) * kP + p] = n0;
      T[(2 * k + 1) * kP + p] = n1;
    }
    g0 = n0;
    g1 = n1;
  }
  if (TO_FINAL && a.final_state) {
    a.final_state[so + (2 * k) * kP + p] = g0;
    a.final_state[so + (2 * k + 1) * kP + p] = g1;
  }
}

// Segments per chain: minimise the estimated time in chunk steps of one CTA,
//   rounds(full pass) * cps + kStateCost * rounds(state pass) * cps,
// where a round is one wave of CTAs over the SMs (148 SMs x CTAs per SM) and
// the state-only pass costs about kStateCost of a full chunk step.
TcPlan make_plan(const ScanArgs& a) {
  constexpr double kStateCost = 0.4;
  const int64_t chains = a.batch * a.nheads;
  const int64_t slots = 148 * ((a.Q * a.R == 64) ? 2 : 1);
  TcPlan best{};
  double best_cost = 0.0;
  const int64_t max_seg = a.nchunks < 64 ? a.nchunks : 64;
  for (int64_t ns = 1; ns <= (max_seg > 0 ? max_seg : 1); ++ns) {
    const int64_t cps = (a.nchunks + ns - 1) / ns;
    const int64_t nseg = (a.nchunks + cps - 1) / cps;
    if (nseg != ns) continue;
    const int64_t rounds_full = (chains * nseg + slots - 1) / slots;
    const int64_t rounds_state = nseg > 1 ? (chains * (nseg - 1) + slots - 1) / slots : 0;
    const double cost = (double)rounds_full * cps + kStateCost * (double)rounds_state * cps;
    if (ns == 1 || cost < best_cost * 0.97) {  // more segments only for a clear gain
      best_cost = cost;
      best.nseg = nseg;
      best.cps = cps;
    }
  }
  if (best.nseg < 1) {
    best.nseg = 1;
    best.cps = a.nchunks;
  }
  // Tail split: whole chains in the full waves, the chains of a last, partial
  // wave cut in two so that their halves fill one wave (cost: a state-only
  // pass over their first halves, one partial wave).  Fixed-length full
  // scans only.
  best.ntail = 0;
  best.cps2 = 0;
  if (best.nseg == 1 && !a.state_only && !a.cu_seqlens && a.nchunks >= 2) {
    const int64_t rounds = (chains + slots - 1) / slots;
    const int64_t rem = chains - (rounds - 1) * slots;  // chains in the last wave
    const int64_t cps2 = (a.nchunks + 1) / 2;
    if (rounds >= 2 && 2 * rem <= slots) {
      const double split = (double)(rounds - 1) * a.nchunks + (1.0 + kStateCost) * cps2;
      if (split < 0.97 * (double)rounds * a.nchunks) {
        best.ntail = rem;
        best.cps2 = cps2;
      }
    }
  }
  return best;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Map over a row-major tensor of `rank` (<= 4) dimensions, dims[0] innermost,
// of `esize`-byte elements.
bool encode_nd(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base, int rank,
               const uint64_t* d, const uint32_t* bx, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4];
  uint64_t st = esize;
  for (int i = 0; i < rank; ++i) {
    dims[i] = d[i];
    box[i] = bx[i];
    estr[i] = 1;
    if (i > 0) strides[i - 1] = st;
    st *= d[i];
  }
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode3d(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base, uint64_t d0,
              uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2,
              CUtensorMapSwizzle sw) {
  const uint64_t d[3] = {d0, d1, d2};
  const uint32_t bx[3] = {b0, b1, b2};
  return encode_nd(m, dt, esize, base, 3, d, bx, sw);
}

// Rows of the token dimension: batch x seqlen, or a packed batch's total.
int64_t token_rows(const ScanArgs& a) {
  return a.cu_seqlens ? a.total_tokens : a.batch * a.seqlen;
}

bool make_maps(const ScanArgs& a, TcMaps* m) {
  const uint64_t tok = (uint64_t)token_rows(a);
  const uint32_t R = (uint32_t)a.R, Q = (uint32_t)a.Q;
  // y as [batch][L][H*R][P], or a packed batch as [1][total][H*R][P]
  const uint64_t yd[4] = {kP, (uint64_t)(a.nheads * a.R),
                          a.cu_seqlens ? tok : (uint64_t)a.seqlen,
                          a.cu_seqlens ? 1u : (uint64_t)a.batch};
  const uint32_t yb[4] = {64, R, Q, 1};
  return encode3d(&m->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.x, kP, a.nheads * a.R, tok, 64, R,
                  Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode3d(&m->b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, kN, a.ngroups * a.R, tok, 64,
                  R, Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode3d(&m->c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.C, kN, a.ngroups * a.R, tok, 64,
                  R, Q, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode3d(&m->th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.theta, kPairs, a.tgroups, tok,
                  kPairs, 1, Q, CU_TENSOR_MAP_SWIZZLE_NONE) &&
         (a.state_only ||  // no y in a state-only call
          encode_nd(&m->y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.y, 4, yd, yb,
                    CU_TENSOR_MAP_SWIZZLE_128B));
}

// dependent: launched as a programmatic dependent of the kernel before it on
// the stream (it may start once that kernel's CTAs have all signalled).
template <int R, int Q, int MODE>
cudaError_t launch_grid(const ScanArgs& a, const TcPlan& pl, const TcMaps& maps, dim3 grid,
                        cudaStream_t st, bool dependent = false) {
  using C = Cfg<R, Q>;
  auto kern = tc_scan_kernel<R, Q, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  if (!dependent) {
    kern<<<grid, C::NTH, C::SMEM, st>>>(a, pl, maps);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::NTH);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, pl, maps);
}

template <int R, int Q, int MODE>
cudaError_t launch_kernel(const ScanArgs& a, const TcPlan& pl, const TcMaps& maps,
                          int64_t nblocks, cudaStream_t st) {
  return launch_grid<R, Q, MODE>(a, pl, maps,
                                 dim3((unsigned)nblocks, (unsigned)a.nheads, (unsigned)a.batch), st);
}

template <int R, int Q>
cudaError_t launch_rq(const ScanArgs& a, TcPlan pl, cudaStream_t st) {
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_maps(a, &maps)) return cudaErrorInvalidValue;
  dim3 pg((kPairs * kP + 255) / 256, (unsigned)a.nheads, (unsigned)a.batch);
  if (a.state_only) {  // every segment's local end state, then the fold into final_state
    cudaError_t e = launch_kernel<R, Q, MODE_STATE>(a, pl, maps, pl.nseg, st);
    if (e != cudaSuccess) return e;
    tc_seg_pass_kernel<true><<<pg, 256, 0, st>>>(a, pl);
    return cudaGetLastError();
  }
  if (pl.ntail > 0) {
    // tail split: the first halves' local end states, and the full pass over
    // every chain launched as its programmatic dependent (the whole chains
    // start while the state-only pass runs; the second halves wait for it and
    // fold its summaries themselves)
    const int64_t nfull = a.batch * a.nheads - pl.ntail;
    cudaError_t e = launch_grid<R, Q, MODE_STATE>(a, pl, maps, dim3((unsigned)pl.ntail), st);
    if (e != cudaSuccess) return e;
    return launch_grid<R, Q, MODE_FULL>(a, pl, maps, dim3((unsigned)(nfull + 2 * pl.ntail)), st, true);
  }
  if (pl.nseg > 1) {
    cudaError_t e = launch_kernel<R, Q, MODE_STATE>(a, pl, maps, pl.nseg - 1, st);
    if (e != cudaSuccess) return e;
    tc_seg_pass_kernel<false><<<pg, 256, 0, st>>>(a, pl);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_kernel<R, Q, MODE_FULL>(a, pl, maps, pl.nseg, st);
}

}  // namespace

bool tc_scan_supported(const ScanArgs& a) {
  if (!a.bf16 || a.N != kN || a.P != kP) return false;
  const int64_t m = a.Q * a.R;
  // TMA token coordinates are 32-bit
  if (token_rows(a) > (int64_t)0x7fffffff - a.Q) return false;
  return (a.R == 1 || a.R == 2 || a.R == 4) && (m == 64 || m == 128 || m == 256) && a.Q >= 16;
}

int64_t tc_scan_segments(const ScanArgs& a) {
  const TcPlan pl = make_plan(a);
  return pl.ntail > 0 ? 2 : pl.nseg;
}

// Kernel launches of one full scan call: one; three with segments (state-only
// pass, fold, full pass); two with the tail split (the fold is in the full pass).
int tc_scan_launches(const ScanArgs& a) {
  const TcPlan pl = make_plan(a);
  return pl.ntail > 0 ? 2 : pl.nseg > 1 ? 3 : 1;
}

size_t tc_scan_workspace(const ScanArgs& a) {
  const TcPlan pl = make_plan(a);
  const int64_t per = a.state_only ? pl.nseg : pl.nseg - 1;
  if (per <= 0 && pl.ntail == 0) return 0;
  const size_t slots = pl.ntail > 0 ? (size_t)pl.ntail : (size_t)a.batch * a.nheads * per;
  return align_up(sizeof(float) * slots * kN * kP, 256) +
         align_up(sizeof(float) * slots * (1 + kPairs), 256);
}

cudaError_t tc_scan_launch(const ScanArgs& a, cudaStream_t st) {
  TcPlan pl = make_plan(a);
  pl.slots = a.state_only ? pl.nseg : pl.nseg - 1;
  if (pl.slots > 0 || pl.ntail > 0) {
    const size_t slots = pl.ntail > 0 ? (size_t)pl.ntail : (size_t)a.batch * a.nheads * pl.slots;
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
