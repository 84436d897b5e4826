// block_ops.cu -- the MIMO projections and the output gate of a Mamba-3
// block (PaperWeekly page section 2.3, the rank-R MIMO update, and section
// 2.4 / Figure 4, "MIMO projection"; the gate is the block's output gate).
// Element-wise and HBM-bound; each thread moves 16 bytes of io data at a time.
//
//   up:        X[t][h][r][p] = x[t][h][p] * w_up[h][r][p]
//   down+gate: out[t][h][p]  = (sum_r Y[t][h][r][p] * w_down[h][r][p]) * silu(z[t][h][p])
//              (silu(v) = v / (1 + exp(-v)); without z the gate is left out)
#include "m3_internal.cuh"

namespace m3 {
namespace {

constexpr int kThreads = 256;

// V consecutive io elements (8 bf16 or 4 fp32 = 16 bytes) to / from fp32.
template <bool BF16>
struct Vec {
  static constexpr int V = BF16 ? 8 : 4;
  __device__ static void load(const void* p, int64_t i, float (&f)[V]) {
    const uint4 u = *reinterpret_cast<const uint4*>(
        static_cast<const char*>(p) + i * (BF16 ? 2 : 4));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if (BF16) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) f[e] = __uint_as_float(w[e]);
    }
  }
  __device__ static void store(void* p, int64_t i, const float (&f)[V]) {
    uint4 u;
    uint32_t w[4];
    if (BF16) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        w[e] = *reinterpret_cast<const uint32_t*>(&b);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = __float_as_uint(f[e]);
    }
    u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
    *reinterpret_cast<uint4*>(static_cast<char*>(p) + i * (BF16 ? 2 : 4)) = u;
  }
};

// V consecutive fp32 weights (two or one float4 loads through the read-only path).
template <int V>
__device__ __forceinline__ void load_w(const float* w, float (&f)[V]) {
#pragma unroll
  for (int e = 0; e < V; e += 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(w + e));
    f[e] = v.x; f[e + 1] = v.y; f[e + 2] = v.z; f[e + 3] = v.w;
  }
}

// one thread per V-wide piece of x: piece q covers (t, h, p .. p+V-1) and
// writes that piece of all R ranks of X
template <bool BF16, int R>
__global__ void __launch_bounds__(kThreads) mimo_up_kernel(int64_t T, int H, int P, const void* x,
                                                           const float* w, void* X) {
  using Vc = Vec<BF16>;
  constexpr int V = Vc::V;
  const int pv = P / V;
  const int64_t pieces = T * H * pv;
  for (int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x; q < pieces;
       q += (int64_t)gridDim.x * kThreads) {
    const int p = (int)(q % pv) * V;
    const int64_t th = q / pv;  // t * H + h
    const int h = (int)(th % H);
    float xv[V];
    Vc::load(x, th * P + p, xv);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float wv[V], o[V];
      load_w<V>(w + ((int64_t)h * R + r) * P + p, wv);
#pragma unroll
      for (int e = 0; e < V; ++e) o[e] = xv[e] * wv[e];
      Vc::store(X, (th * R + r) * P + p, o);
    }
  }
}

// one thread per V-wide piece of out: piece q covers (t, h, p .. p+V-1); the
// R pieces of Y are all loaded before any is used
template <bool BF16, int R>
__global__ void __launch_bounds__(kThreads) mimo_down_gate_kernel(int64_t T, int H, int P,
                                                                  const void* Y, const float* w,
                                                                  const void* z, void* out) {
  using Vc = Vec<BF16>;
  constexpr int V = Vc::V;
  const int pv = P / V;
  const int64_t pieces = T * H * pv;
  for (int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x; q < pieces;
       q += (int64_t)gridDim.x * kThreads) {
    const int p = (int)(q % pv) * V;
    const int64_t th = q / pv;  // t * H + h
    const int h = (int)(th % H);
    float yv[R][V], zv[V];
#pragma unroll
    for (int r = 0; r < R; ++r) Vc::load(Y, (th * R + r) * P + p, yv[r]);
    if (z) Vc::load(z, th * P + p, zv);
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float wv[V];
      load_w<V>(w + ((int64_t)h * R + r) * P + p, wv);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = fmaf(yv[r][e], wv[e], acc[e]);
    }
    if (z) {
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] *= zv[e] / (1.f + __expf(-zv[e]));
    }
    Vc::store(out, th * P + p, acc);
  }
}

int grid_for(int64_t pieces) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = (pieces + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sms * 8;  // eight CTAs of 256 threads per SM
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <bool BF16, int R>
cudaError_t up_r(int64_t T, int64_t H, int64_t P, const void* x, const float* w, void* X,
                 cudaStream_t s) {
  const int64_t pieces = T * H * (P / Vec<BF16>::V);
  mimo_up_kernel<BF16, R><<<grid_for(pieces), kThreads, 0, s>>>(T, (int)H, (int)P, x, w, X);
  return cudaGetLastError();
}

template <bool BF16, int R>
cudaError_t down_r(int64_t T, int64_t H, int64_t P, const void* Y, const float* w, const void* z,
                   void* out, cudaStream_t s) {
  const int64_t pieces = T * H * (P / Vec<BF16>::V);
  mimo_down_gate_kernel<BF16, R><<<grid_for(pieces), kThreads, 0, s>>>(T, (int)H, (int)P, Y, w,
                                                                        z, out);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t up_dispatch(int64_t T, int64_t H, int64_t R, int64_t P, const void* x, const float* w,
                        void* X, cudaStream_t s) {
  switch (R) {
    case 1: return up_r<BF16, 1>(T, H, P, x, w, X, s);
    case 2: return up_r<BF16, 2>(T, H, P, x, w, X, s);
    case 4: return up_r<BF16, 4>(T, H, P, x, w, X, s);
    case 8: return up_r<BF16, 8>(T, H, P, x, w, X, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool BF16>
cudaError_t down_dispatch(int64_t T, int64_t H, int64_t R, int64_t P, const void* Y,
                          const float* w, const void* z, void* out, cudaStream_t s) {
  switch (R) {
    case 1: return down_r<BF16, 1>(T, H, P, Y, w, z, out, s);
    case 2: return down_r<BF16, 2>(T, H, P, Y, w, z, out, s);
    case 4: return down_r<BF16, 4>(T, H, P, Y, w, z, out, s);
    case 8: return down_r<BF16, 8>(T, H, P, Y, w, z, out, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t mimo_up_launch(int64_t T, int64_t H, int64_t R, int64_t P, bool bf16, const void* x,
                           const float* w, void* X, cudaStream_t s) {
  if (T * H == 0) return cudaSuccess;
  return bf16 ? up_dispatch<true>(T, H, R, P, x, w, X, s)
              : up_dispatch<false>(T, H, R, P, x, w, X, s);
}

cudaError_t mimo_down_gate_launch(int64_t T, int64_t H, int64_t R, int64_t P, bool bf16,
                                  const void* Y, const float* w, const void* z, void* out,
                                  cudaStream_t s) {
  if (T * H == 0) return cudaSuccess;
  return bf16 ? down_dispatch<true>(T, H, R, P, Y, w, z, out, s)
              : down_dispatch<false>(T, H, R, P, Y, w, z, out, s);
}

}  // namespace m3
