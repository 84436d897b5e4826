// gemm_tc.cu -- the block's linear projections on the tensor cores:
//   out[M][N] = A[M][K] W[N][K]^T (+ bias[N]),  bf16 operands, fp32 accumulation,
// output bf16 or fp32.  These are the dense maps around the SSM layer in a
// Mamba-3 block (PaperWeekly page section 2.4 and Figure 4: the input-side
// projections that give x, the gate z and the data-dependent angle rates
// theta, and the output projection); A holds one token per row.
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0       TMA producer: 128 x 64 tiles of A and BN x 64 tiles of W
//                (128-byte swizzled, K-major) into a ring of kStages stages;
//   warp 1       TMEM allocation and the single MMA-issuing thread:
//                tcgen05.mma kind::f16, M = 128, N = BN, K = 16, fp32
//                accumulators in TMEM, two of them (ping-pong), so one output
//                tile's epilogue overlaps the next tile's main loop;
//   warps 2-5    epilogue: tcgen05.ld of the accumulator (one row per thread),
//                bias, rounding, 16-byte stores.
// Stages and accumulators are handed over on mbarriers; every wait is bounded
// and a wait that runs out records M3_ERR_TIMEOUT and ends the CTA's work.
#include <cuda.h>  // CUtensorMap

#include "m3_internal.cuh"
#include "tc_ptx.cuh"

namespace m3 {
namespace {

using namespace tc;

constexpr int kBM = 128;      // rows of A per tile
constexpr int kBK = 64;       // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int kThreads = 192;  // 6 warps
constexpr unsigned long long kGemmWaitNs = 2000000000ull;

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = kStages * STAGE;
  // full[S], empty[S], acc_full[2], acc_empty[2], fin, tmem holder
  static constexpr int SMEM = BAR_OFF + (2 * kStages + 5) * 8 + 16;
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators
  static_assert(SMEM + 1024 <= 232448, "shared memory");
};

struct GemmArgs {
  int64_t M, N, K;
  const float* bias;  // [N] or nullptr
  void* out;          // [M][N]
  bool out_f32;
  int* status;
};

__device__ __forceinline__ unsigned long long gemm_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ bool gemm_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = gemm_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (gemm_ns() - t0 > kGemmWaitNs) {
      if (status) atomicCAS(status, 0, (int)M3_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// TMA: 2-D tiled bulk tensor load, completing bytes on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

struct GemmMaps {
  CUtensorMap a, w;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const GemmArgs g, const __grid_constant__ GemmMaps maps) {
  using Cf = GemmCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((sbase & 1023u) != 0) {  // the swizzled layout needs 1 KB alignment
    if (tid == 0 && g.status) atomicCAS(g.status, 0, (int)M3_ERR_CUDA);
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Cf::BAR_OFF);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* s_fin = acc_empty + 2;  // every MMA issued, before TMEM is released
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_fin + 1);

  const int64_t mt = (g.M + kBM - 1) / kBM, nt = (g.N + BN - 1) / BN;
  const int64_t tiles = mt * nt;
  const int kb_n = (int)((g.K + kBK - 1) / kBK);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);  // every epilogue thread arrives
    }
    mbar_init(s_fin, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, Cf::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;

  if (warp == 0 && lane == 0) {
    // ---- producer -----------------------------------------------------------
    uint32_t it = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int m0 = (int)((t / nt) * kBM), n0 = (int)((t % nt) * BN);
      for (int kb = 0; kb < kb_n; ++kb, ++it) {
        const int s = (int)(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        if (!gemm_wait(&empty[s], ph ^ 1u, g.status)) { ok = false; break; }
        uint8_t* st = sm + s * Cf::STAGE;
        mbar_expect_tx(&full[s], (uint32_t)Cf::STAGE);
        tma_load_2d(st, &maps.a, kb * kBK, m0, &full[s]);
        tma_load_2d(st + Cf::A_BYTES, &maps.w, kb * kBK, n0, &full[s]);
      }
    }
    // let the last stages' copies land (bounded) before the CTA can exit
    for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
      gemm_wait(&full[j % kStages], (j / kStages) & 1u, g.status);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issue ------------------------------------------------------------
    const uint32_t idesc = idesc_bf16(kBM, BN, 0, 0);
    uint32_t it = 0;
    int j = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
      const int b = j & 1;
      if (!gemm_wait(&acc_empty[b], ((j >> 1) & 1) ^ 1u, g.status)) break;
      tc_fence_after();
      const uint32_t dcol = tm + (uint32_t)(b * BN);
      for (int kb = 0; kb < kb_n; ++kb, ++it) {
        const int s = (int)(it % kStages);
        if (!gemm_wait(&full[s], (it / kStages) & 1u, g.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + (uint32_t)(s * Cf::STAGE);
        const uint64_t ad = sw128_desc(st, 16, 1024);
        const uint64_t bd = sw128_desc(st + Cf::A_BYTES, 16, 1024);
#pragma unroll
        for (int k4 = 0; k4 < kBK / 16; ++k4)
          mma_bf16_ss(dcol, ad + (uint64_t)(k4 * 2), bd + (uint64_t)(k4 * 2), idesc,
                      (kb | k4) != 0);
        mma_commit(&empty[s]);  // the stage is free once these MMAs have read it
      }
      if (ok) mma_commit(&acc_full[b]);
    }
  } else if (warp >= 2) {
    // ---- epilogue -------------------------------------------------------------
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int j = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
      const int b = j & 1;
      if (!gemm_wait(&acc_full[b], (j >> 1) & 1u, g.status)) break;
      tc_fence_after();
      const int64_t m = (t / nt) * kBM + row;
      const int64_t n0 = (t % nt) * BN;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tm + lane_base + (uint32_t)(b * BN + c), v);
        tmem_ld_wait();
        if (m >= g.M) continue;
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int64_t n = n0 + c + e;
          f[e] = __uint_as_float(v[e]) + ((g.bias && n < g.N) ? __ldg(g.bias + n) : 0.f);
        }
        const int64_t nb = n0 + c;
        if (g.out_f32) {
          float* o = reinterpret_cast<float*>(g.out) + m * g.N + nb;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            if (nb + e + 4 <= g.N)
              *reinterpret_cast<float4*>(o + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
        } else {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(g.out) + m * g.N + nb;
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            if (nb + e + 8 <= g.N)
              *reinterpret_cast<uint4*>(o + e) =
                  make_uint4(pack_bf16(f[e], f[e + 1]), pack_bf16(f[e + 2], f[e + 3]),
                             pack_bf16(f[e + 4], f[e + 5]), pack_bf16(f[e + 6], f[e + 7]));
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);  // the accumulator may take the next tile
    }
  }

  // every MMA issued has completed before TMEM is released (bounded)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if (lane == 0) {
      mma_commit(s_fin);  // arrives once all earlier MMAs are done
      gemm_wait(s_fin, 0, g.status);
    }
    __syncwarp();
    tmem_dealloc(tm, Cf::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn gemm_encode_fn() {
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

// [rows][K] bf16, boxes of kBK x box_rows, 128-byte swizzle.
bool encode_kmajor(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = gemm_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t gemm_launch_bn(const GemmArgs& g, const void* A, const void* W, cudaStream_t st) {
  using Cf = GemmCfg<BN>;
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!encode_kmajor(&maps.a, A, g.M, g.K, kBM) || !encode_kmajor(&maps.w, W, g.N, g.K, BN))
    return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((g.M + kBM - 1) / kBM) * ((g.N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  kern<<<grid, kThreads, Cf::SMEM, st>>>(g, maps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_launch(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                        const float* bias, void* out, bool out_f32, int* status,
                        cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  GemmArgs g;
  g.M = M; g.N = N; g.K = K; g.bias = bias; g.out = out; g.out_f32 = out_f32; g.status = status;
  if (N <= 64) return gemm_launch_bn<64>(g, A, W, st);
  return gemm_launch_bn<256>(g, A, W, st);
}

}  // namespace m3
