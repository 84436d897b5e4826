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
// Rank R >= 2 (the arithmetic per element grows with R):
// CTAs of 256 threads, two or more per SM, each walking a contiguous
// range of heads (so consecutive heads mostly share one (batch, group) and
// its B, C, B_prev are converted once).  A head's state and its operands
// arrive in shared memory by bulk async copies issued one head ahead into a
// second buffer, so the state stream never waits on the arithmetic; h'
// leaves by streaming 16-byte stores.
// Thread (kslot, pv) owns float4 column pv of the state and the pairs
// k = kslot, kslot + nslots, ...; y is reduced over kslots with warp
// shuffles and then across warps through shared memory.
// Rank 1: one CTA per head streams the state through registers (see
// stream_decode_kernel below).
#include "m3_internal.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

using namespace tc;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned long long kDecodeWaitNs = 2000000000ull;  // bounded mbarrier wait (2 s)

__device__ __forceinline__ unsigned long long decode_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// One thread polls; false (and the status word set) after the time limit.
__device__ bool decode_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = decode_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (decode_ns() - t0 > kDecodeWaitNs) {
      if (status) atomicCAS(status, 0, (int)M3_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Bulk async copy global -> shared of `bytes` (a multiple of 16, both
// addresses 16-byte aligned), completing on `bar`.
__device__ __forceinline__ void bulk_load(void* smem, const void* gmem, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem)),
      "l"(gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory plan of one CTA (byte offsets, all 128-byte aligned): the
// state and raw operands of up to three heads in flight (one for the largest
// shapes), the fp32 B / C / B_prev of the current (batch, group), the
// per-head rotation and x factors, and the per-warp partial sums of y.
constexpr int kMaxBuf = 3;
struct DecodeSmem {
  int64_t st_bytes, ops_bytes;
  int64_t st_stride, ops_stride;  // buffer i: st at i * st_stride, ops at ops0 + i * ops_stride
  int64_t ops0, bc_off, head_off, red_off, bar_off, total;
  int nbuf;  // heads whose state is resident or in flight; nbuf - 1 stream in during one
};
constexpr int64_t kMaxSmem = 232448;  // dynamic shared memory of one CTA

// want: buffers asked for (three when the arithmetic per head is light and
// more bytes in flight pay, else two); fewer when they do not fit.
__host__ __device__ inline DecodeSmem decode_smem(int64_t N, int64_t P, int64_t R, bool bf16,
                                                  int want) {
  DecodeSmem m;
  const int64_t es = bf16 ? 2 : 4;
  const int64_t K = N / 2;
  m.st_bytes = N * P * 4;
  m.ops_bytes = (3 * R * N + 2 * R * P) * es + K * 4;  // B, C, B_prev, x, x_prev, theta
  const int64_t bc = align_up(3 * R * N * 8, 128);            // [3][n][R] float pairs
  const int64_t head = align_up((6 * K + 2 * R * P) * 4, 128);  // rot, sin pairs, xe, xg
  const int64_t red = align_up(kWarps * R * P * 4, 128);
  const int64_t buf = align_up(m.st_bytes, 128) + align_up(m.ops_bytes, 128);
  m.nbuf = want;
  while (m.nbuf > 1 && m.nbuf * buf + bc + head + red + 32 > kMaxSmem) --m.nbuf;
  m.st_stride = align_up(m.st_bytes, 128);
  m.ops_stride = align_up(m.ops_bytes, 128);
  m.ops0 = m.nbuf * m.st_stride;
  int64_t o = m.ops0 + m.nbuf * m.ops_stride;
  m.bc_off = o; o += bc;
  m.head_off = o; o += head;
  m.red_off = o; o += red;
  m.bar_off = o; o += 32;
  m.total = o;
  return m;
}

// Buffers asked for, and the CTAs per SM the register budget is sized for.
template <int R>
struct DecodeOcc {
  static constexpr int want = 2;
  static constexpr int value = R <= 4 ? 2 : 1;
};

// NC, PC: compile-time N and P (0: taken from the arguments), so that the
// common state shape gets a fully unrolled pair loop.
template <int R, int NC, int PC>
__global__ void __launch_bounds__(kThreads, DecodeOcc<R>::value) decode_kernel(const DecodeArgs a) {
  const int P = PC ? PC : (int)a.P, N = NC ? NC : (int)a.N, K = N / 2;
  const int lgN = __ffs(N) - 1;  // N and P are powers of two
  const int64_t H = a.nheads, G = a.ngroups, total = a.batch * H;
  const int64_t es = a.bf16 ? 2 : 4;
  const DecodeSmem sp = decode_smem(N, P, R, a.bf16, DecodeOcc<R>::want);
  const int nbuf = sp.nbuf;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + sp.bar_off);
  // packed fp32x2 operands are staged with both halves equal, so the pair
  // loop feeds them to the f32x2 FMAs as loaded
  float2* s_Bp = reinterpret_cast<float2*>(sm + sp.bc_off);  // B_prev, [n][R] pairs
  float2* s_Bt = s_Bp + R * N;                                // B_t,    [n][R] pairs
  float2* s_Ct = s_Bt + R * N;                                // C_t,    [n][R] pairs
  float4* s_rot = reinterpret_cast<float4*>(sm + sp.head_off);  // (a cos, a cos, -a sin, -a sin)
  float2* s_as = reinterpret_cast<float2*>(s_rot + K);          // (a sin, a sin)      [K]
  float* s_xe = reinterpret_cast<float*>(s_as + K);  // (1-lam) dt x_prev              [R][P]
  float* s_xg = s_xe + R * P;                        // lam dt x_t                     [R][P]
  float* s_red = reinterpret_cast<float*>(sm + sp.red_off);  // partial y [warps][R][P]

  const bool prev = a.B_prev != nullptr;
  const uint32_t opsB = (uint32_t)(R * N * es), opsX = (uint32_t)(R * P * es);
  // bytes of one head: state, x (and x_prev), theta, plus B, C (and B_prev)
  // whenever its (batch, group) differs from the previous head's
  const uint32_t bytes_head = (uint32_t)sp.st_bytes + (prev ? 2 : 1) * opsX + (uint32_t)(K * 4);
  const uint32_t bytes_bc = (prev ? 3 : 2) * opsB;

  if (tid == 0) {
    for (int i = 0; i < nbuf; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int hpg = (int)(H / G);  // heads per group
  // thread 0: bring head hd's state and operands into buffer bi
  auto issue = [&](int64_t hd, int64_t bg, int bi, bool with_bc) {
    // (a skipped copy leaves its barrier incomplete: the wait then times out
    // after the bounds error is recorded)
    if (!M3_IN(hd, total, a.status) || !M3_IN(bg, a.batch * G, a.status)) return;
    uint8_t* st = sm + bi * sp.st_stride;
    uint8_t* ops = sm + sp.ops0 + bi * sp.ops_stride;
    fence_async_smem();
    mbar_expect_tx(&bars[bi], bytes_head + (with_bc ? bytes_bc : 0u));
    bulk_load(st, a.state_in + hd * (int64_t)N * P, (uint32_t)sp.st_bytes, &bars[bi]);
    if (with_bc) {
      bulk_load(ops, static_cast<const char*>(a.B) + bg * opsB, opsB, &bars[bi]);
      bulk_load(ops + opsB, static_cast<const char*>(a.C) + bg * opsB, opsB, &bars[bi]);
      if (prev) bulk_load(ops + 2 * opsB, static_cast<const char*>(a.B_prev) + bg * opsB, opsB, &bars[bi]);
    }
    bulk_load(ops + 3 * opsB, static_cast<const char*>(a.x) + hd * opsX, opsX, &bars[bi]);
    if (prev) bulk_load(ops + 3 * opsB + opsX, static_cast<const char*>(a.x_prev) + hd * opsX, opsX, &bars[bi]);
    const int64_t tgi = (hd / H) * a.tgroups + (hd % H) / (H / a.tgroups);  // theta group
    bulk_load(ops + 3 * opsB + 2 * opsX, a.theta + tgi * K, (uint32_t)(K * 4), &bars[bi]);
  };

  const int PV = P / 4;                     // float4 columns of a state row
  const int nslots = kThreads / PV;
  const int pv = tid % PV, kslot = tid / PV;
  const int p0 = pv * 4;
  const int rowq = P / 4;

  // this CTA's heads: a contiguous range, so consecutive heads share B and C
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t h_begin = (int64_t)blockIdx.x * per;
  const int64_t h_end = min(total, h_begin + per);
  uint32_t pending = 0u;  // thread 0: bit i = bytes expected on bars[i]
  uint32_t ph = 0u;       // bit i = phase parity of bars[i]
  // issue cursor (thread 0): the next head to bring in, its index within the
  // batch, its (batch, group), the group of the head issued before it, its buffer
  int64_t ihd = h_begin;
  int ihh = (int)(h_begin % H);
  int64_t ibg = (h_begin / H) * G + ihh / hpg, last_bg = -1;
  int islot = 0;
  auto issue_next = [&]() {
    issue(ihd, ibg, islot, ibg != last_bg);
    pending |= 1u << islot;
    last_bg = ibg;
    ++ihd;
    ihh = ihh + 1 == H ? 0 : ihh + 1;
    if (ihh % hpg == 0) ++ibg;
    islot = islot + 1 == nbuf ? 0 : islot + 1;
  };
  if (tid == 0)
    for (int i = 0; i < (nbuf > 1 ? nbuf - 1 : 1) && ihd < h_end; ++i) issue_next();

  int64_t hd = h_begin;
  int hh = (int)(h_begin % H);  // head index within the batch
  // per-head scalars of the current head, loaded one head ahead
  float dt = 0.f, Av = 0.f, lamv = 0.f;
  if (hd < h_end) { dt = a.dt[hd]; Av = a.A[hd]; lamv = a.lam[hd]; }
  bool aborted = false;

  for (int bi = 0; hd < h_end; ++hd, bi = bi + 1 == nbuf ? 0 : bi + 1) {
    const int64_t nhd = hd + 1;
    const bool new_bc = hd == h_begin || hh % hpg == 0;  // first head of its (batch, group)
    // buffer (bi + nbuf - 1) % nbuf was released by the last head
    if (nbuf > 1 && tid == 0 && ihd < h_end) issue_next();
    float ndt = 0.f, nA = 0.f, nlam = 0.f;
    if (nhd < h_end) { ndt = a.dt[nhd]; nA = a.A[nhd]; nlam = a.lam[nhd]; }

    const bool ok = (tid == 0) ? decode_wait(&bars[bi], (ph >> bi) & 1u, a.status) : true;
    if (tid == 0 && ok) {  // on a timeout the phase stays for the exit wait
      pending &= ~(1u << bi);
      ph ^= 1u << bi;
    }
    if (__syncthreads_or(!ok)) { aborted = true; break; }

    const float alpha = expf(dt * Av);
    const float gamma = lamv * dt, eps = (1.f - lamv) * dt;
    const uint8_t* ops = sm + sp.ops0 + bi * sp.ops_stride;
    const void* ox = ops + 3 * opsB;
    const void* oxp = ops + 3 * opsB + opsX;
    const float* oth = reinterpret_cast<const float*>(ops + 3 * opsB + 2 * opsX);
    if (new_bc) {  // fp32 pairs of B, C, B_prev of this (batch, group), [n][r] order
      for (int i = tid; i < R * N; i += kThreads) {
        const int nn = i / R, r = i % R, si = (r << lgN) + nn;
        const float vb = io_load(ops, si, a.bf16), vc = io_load(ops + opsB, si, a.bf16);
        const float vp = prev ? io_load(ops + 2 * opsB, si, a.bf16) : 0.f;
        s_Bt[i] = make_float2(vb, vb);
        s_Ct[i] = make_float2(vc, vc);
        s_Bp[i] = make_float2(vp, vp);
      }
    }
    for (int k = tid; k < K; k += kThreads) {
      float sn, cs;
      sincosf(dt * oth[k], &sn, &cs);
      s_rot[k] = make_float4(alpha * cs, alpha * cs, -alpha * sn, -alpha * sn);
      s_as[k] = make_float2(alpha * sn, alpha * sn);
    }
    for (int i = tid; i < R * P; i += kThreads) {
      s_xg[i] = gamma * io_load(ox, i, a.bf16);
      s_xe[i] = prev ? eps * io_load(oxp, i, a.bf16) : 0.f;
    }
    __syncthreads();

    // column pairs (p0, p0+1) and (p0+2, p0+3) as packed fp32x2 operands
    float2 xg[R][2], xe[R][2], yacc[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        xg[r][jj] = make_float2(s_xg[r * P + p0 + 2 * jj], s_xg[r * P + p0 + 2 * jj + 1]);
        xe[r][jj] = make_float2(s_xe[r * P + p0 + 2 * jj], s_xe[r * P + p0 + 2 * jj + 1]);
        yacc[r][jj] = make_float2(0.f, 0.f);
      }

    const float4* src = reinterpret_cast<const float4*>(sm + bi * sp.st_stride);
    float4* dst = reinterpret_cast<float4*>(a.state_out + hd * (int64_t)N * P);
#pragma unroll
    for (int k = kslot; k < K; k += nslots) {
      const float4 r0 = src[(2 * k) * rowq + pv];
      const float4 r1 = src[(2 * k + 1) * rowq + pv];
      const float4 rot = s_rot[k];
      const float2 AC = make_float2(rot.x, rot.y), NAS = make_float2(rot.z, rot.w);
      const float2 AS = s_as[k];
      float2 bp0[R], bp1[R], bt0[R], bt1[R], c0[R], c1[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {  // rows 2k and 2k+1 are adjacent R-vectors
        bp0[r] = s_Bp[(2 * k) * R + r]; bp1[r] = s_Bp[(2 * k + 1) * R + r];
        bt0[r] = s_Bt[(2 * k) * R + r]; bt1[r] = s_Bt[(2 * k + 1) * R + r];
        c0[r] = s_Ct[(2 * k) * R + r]; c1[r] = s_Ct[(2 * k + 1) * R + r];
      }
      const float2 in0[2] = {make_float2(r0.x, r0.y), make_float2(r0.z, r0.w)};
      const float2 in1[2] = {make_float2(r1.x, r1.y), make_float2(r1.z, r1.w)};
      float o0[4], o1[4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        float2 g0 = in0[jj], g1 = in1[jj], u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          g0 = ffma2(bp0[r], xe[r][jj], g0);
          g1 = ffma2(bp1[r], xe[r][jj], g1);
          u0 = ffma2(bt0[r], xg[r][jj], u0);
          u1 = ffma2(bt1[r], xg[r][jj], u1);
        }
        // (h'_{2k}, h'_{2k+1}) = alpha Rot(phi) (g_{2k}, g_{2k+1}) + (u_{2k}, u_{2k+1})
        const float2 w0 = ffma2(AC, g0, ffma2(NAS, g1, u0));
        const float2 w1 = ffma2(AS, g0, ffma2(AC, g1, u1));
#pragma unroll
        for (int r = 0; r < R; ++r)
          yacc[r][jj] = ffma2(c0[r], w0, ffma2(c1[r], w1, yacc[r][jj]));
        o0[2 * jj] = w0.x; o0[2 * jj + 1] = w0.y;
        o1[2 * jj] = w1.x; o1[2 * jj + 1] = w1.y;
      }
      if (M3_IN(hd * (int64_t)N * P / 4 + (2 * k + 1) * rowq + pv, total * N * P / 4, a.status)) {
        __stcs(dst + (2 * k) * rowq + pv, make_float4(o0[0], o0[1], o0[2], o0[3]));
        __stcs(dst + (2 * k + 1) * rowq + pv, make_float4(o1[0], o1[1], o1[2], o1[3]));
      }
    }

    // y: kslots of one warp share columns every PV lanes; then across warps
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
        for (int off = PV; off < 32; off <<= 1) {
          yacc[r][jj].x += __shfl_xor_sync(0xffffffffu, yacc[r][jj].x, off);
          yacc[r][jj].y += __shfl_xor_sync(0xffffffffu, yacc[r][jj].y, off);
        }
    if (lane < PV) {  // PV = P / 4 <= 32: lanes below PV hold the warp's sums
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          s_red[(warp * R + r) * P + p0 + 2 * jj] = yacc[r][jj].x;
          s_red[(warp * R + r) * P + p0 + 2 * jj + 1] = yacc[r][jj].y;
        }
    }
    __syncthreads();
    for (int i = tid; i < R * P; i += kThreads) {
      float acc = 0.f;
      for (int q = 0; q < kWarps; ++q) acc += s_red[q * R * P + i];
      if (M3_IN(hd * R * P + i, total * R * P, a.status)) io_store(a.y, hd * R * P + i, acc, a.bf16);
    }
    __syncthreads();  // buffer bi, staging and partial sums free
    if (nbuf == 1 && tid == 0 && ihd < h_end) issue_next();  // one buffer: the next head now
    dt = ndt; Av = nA; lamv = nlam;
    hh = hh + 1 == H ? 0 : hh + 1;
  }

  if (aborted && tid == 0) {  // let copies still in flight land (bounded) before exiting
    for (int i = 0; i < nbuf; ++i)
      if ((pending >> i) & 1u) decode_wait(&bars[i], (ph >> i) & 1u, a.status);
  }
}

template <int R, int NC, int PC>
cudaError_t launch_shape(const DecodeArgs& a, cudaStream_t s) {
  const DecodeSmem sp = decode_smem(a.N, a.P, R, a.bf16, DecodeOcc<R>::want);
  const size_t smem = (size_t)sp.total;
  auto kern = decode_kernel<R, NC, PC>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t heads = a.batch * a.nheads;
  const int64_t grid = heads < (int64_t)sms * per_sm ? heads : (int64_t)sms * per_sm;
  kern<<<(unsigned)grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_r(const DecodeArgs& a, cudaStream_t s) {
  if (a.N == 128 && a.P == 64) return launch_shape<R, 128, 64>(a, s);
  return launch_shape<R, 0, 0>(a, s);
}


// ---- rank 1: one CTA per head, state streamed through registers -------------
// With R = 1 the arithmetic per state element is small, and loads issued
// straight into registers (four row pairs per thread in flight, seven CTAs
// of 128 threads per SM) keep more bytes in flight than the shared-memory
// pipeline above.  CTA (b, h); thread (kslot, pv) as above.
constexpr int kStreamThreads = 128;
constexpr int kStreamPairs = 4;  // row pairs whose loads are issued before any is used

__global__ void __launch_bounds__(kStreamThreads, 7) stream_decode_kernel(const DecodeArgs a) {
  const int P = (int)a.P, N = (int)a.N, K = N / 2;
  const int64_t bh = blockIdx.x;
  const int64_t h = bh % a.nheads, b = bh / a.nheads;
  const int64_t bg = b * a.ngroups + h / (a.nheads / a.ngroups);
  const int64_t tgi = b * a.tgroups + h / (a.nheads / a.tgroups);  // theta group
  const int tid = threadIdx.x;

  extern __shared__ float smf[];
  float* s_ac = smf;              // alpha cos(dt theta_k)          [K]
  float* s_as = s_ac + K;         // alpha sin(dt theta_k)          [K]
  float* s_Bp = s_as + K;         // B_prev                         [N]
  float* s_Bt = s_Bp + N;         // B_t                            [N]
  float* s_Ct = s_Bt + N;         // C_t                            [N]
  float* s_xe = s_Ct + N;         // (1-lam) dt x_prev              [P]
  float* s_xg = s_xe + P;         // lam dt x_t                     [P]
  float* s_red = s_xg + P;        // partial y per kslot            [nslots][P]

  const float dt = a.dt[bh], lamv = a.lam[bh];
  const float alpha = expf(dt * a.A[bh]);
  const float gamma = lamv * dt, eps = (1.f - lamv) * dt;
  const bool prev = a.B_prev != nullptr;

  const int PV = P / 4;
  const int nslots = kStreamThreads / PV;
  const int pv = tid % PV, kslot = tid / PV;
  const int p0 = pv * 4;
  const float4* src = reinterpret_cast<const float4*>(a.state_in + bh * (int64_t)N * P);
  float4* dst = reinterpret_cast<float4*>(a.state_out + bh * (int64_t)N * P);
  const int rowq = P / 4;
  // the head's float4 pieces end inside the state tensor
  if (!M3_IN((bh + 1) * (int64_t)N * P / 4 - 1, a.batch * a.nheads * (int64_t)N * P / 4, a.status))
    return;  // uniform over the block

  // the first row pairs' loads go out before the per-head operands are staged
  float4 r0[kStreamPairs], r1[kStreamPairs];
#pragma unroll
  for (int u = 0; u < kStreamPairs; ++u) {
    const int k = kslot + u * nslots;
    if (k < K) {
      r0[u] = __ldcs(src + (2 * k) * rowq + pv);
      r1[u] = __ldcs(src + (2 * k + 1) * rowq + pv);
    }
  }
  for (int k = tid; k < K; k += kStreamThreads) {
    float sn, cs;
    sincosf(dt * a.theta[tgi * K + k], &sn, &cs);
    s_ac[k] = alpha * cs;
    s_as[k] = alpha * sn;
  }
  for (int i = tid; i < N; i += kStreamThreads) {
    s_Bt[i] = io_load(a.B, bg * N + i, a.bf16);
    s_Ct[i] = io_load(a.C, bg * N + i, a.bf16);
    s_Bp[i] = prev ? io_load(a.B_prev, bg * N + i, a.bf16) : 0.f;
  }
  for (int i = tid; i < P; i += kStreamThreads) {
    s_xg[i] = gamma * io_load(a.x, bh * P + i, a.bf16);
    s_xe[i] = prev ? eps * io_load(a.x_prev, bh * P + i, a.bf16) : 0.f;
  }
  __syncthreads();

  float2 xg[2], xe[2], yacc[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    xg[j] = make_float2(s_xg[p0 + 2 * j], s_xg[p0 + 2 * j + 1]);
    xe[j] = make_float2(s_xe[p0 + 2 * j], s_xe[p0 + 2 * j + 1]);
    yacc[j] = make_float2(0.f, 0.f);
  }
  for (int kb = kslot; kb < K; kb += kStreamPairs * nslots) {
    if (kb != kslot) {
#pragma unroll
      for (int u = 0; u < kStreamPairs; ++u) {
        const int k = kb + u * nslots;
        if (k < K) {
          r0[u] = __ldcs(src + (2 * k) * rowq + pv);
          r1[u] = __ldcs(src + (2 * k + 1) * rowq + pv);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kStreamPairs; ++u) {
      const int k = kb + u * nslots;
      if (k < K) {
        const float ac = s_ac[k], as = s_as[k];
        const float bp0 = s_Bp[2 * k], bp1 = s_Bp[2 * k + 1];
        const float bt0 = s_Bt[2 * k], bt1 = s_Bt[2 * k + 1];
        const float c0 = s_Ct[2 * k], c1 = s_Ct[2 * k + 1];
        const float2 in0[2] = {make_float2(r0[u].x, r0[u].y), make_float2(r0[u].z, r0[u].w)};
        const float2 in1[2] = {make_float2(r1[u].x, r1[u].y), make_float2(r1[u].z, r1[u].w)};
        float o0[4], o1[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 g0 = ffma2(make_float2(bp0, bp0), xe[j], in0[j]);
          const float2 g1 = ffma2(make_float2(bp1, bp1), xe[j], in1[j]);
          const float2 u0 = fmul2(make_float2(bt0, bt0), xg[j]);
          const float2 u1 = fmul2(make_float2(bt1, bt1), xg[j]);
          // (h'_{2k}, h'_{2k+1}) = alpha Rot(phi) (g_{2k}, g_{2k+1}) + (u_{2k}, u_{2k+1})
          const float2 w0 = ffma2(make_float2(ac, ac), g0, ffma2(make_float2(-as, -as), g1, u0));
          const float2 w1 = ffma2(make_float2(as, as), g0, ffma2(make_float2(ac, ac), g1, u1));
          yacc[j] = ffma2(make_float2(c0, c0), w0, ffma2(make_float2(c1, c1), w1, yacc[j]));
          o0[2 * j] = w0.x; o0[2 * j + 1] = w0.y;
          o1[2 * j] = w1.x; o1[2 * j + 1] = w1.y;
        }
        __stcs(dst + (2 * k) * rowq + pv, make_float4(o0[0], o0[1], o0[2], o0[3]));
        __stcs(dst + (2 * k + 1) * rowq + pv, make_float4(o1[0], o1[1], o1[2], o1[3]));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    s_red[kslot * P + p0 + 2 * j] = yacc[j].x;
    s_red[kslot * P + p0 + 2 * j + 1] = yacc[j].y;
  }
  __syncthreads();
  for (int i = tid; i < P; i += kStreamThreads) {
    float acc = 0.f;
    for (int q = 0; q < nslots; ++q) acc += s_red[q * P + i];
    if (M3_IN(bh * P + i, a.batch * a.nheads * P, a.status)) io_store(a.y, bh * P + i, acc, a.bf16);
  }
}

cudaError_t launch_stream(const DecodeArgs& a, cudaStream_t s) {
  const int P = (int)a.P, N = (int)a.N;
  const int nslots = kStreamThreads / (P / 4);
  const size_t smem = sizeof(float) * (N + 3 * N + 2 * P + (size_t)nslots * P);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(stream_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  stream_decode_kernel<<<(unsigned)(a.batch * a.nheads), kStreamThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t s) {
  if (a.batch * a.nheads == 0) return cudaSuccess;
  switch (a.R) {
    case 1: return launch_stream(a, s);
    case 2: return launch_r<2>(a, s);
    case 4: return launch_r<4>(a, s);
    case 8: return launch_r<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
