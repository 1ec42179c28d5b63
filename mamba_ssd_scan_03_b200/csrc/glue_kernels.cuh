// glue_kernels.cuh -- the steps either side of the SSD layer inside a Mamba block: a short
// causal depthwise convolution with SiLU on the layer's inputs, the step size dt = softplus(raw
// + bias), and the SiLU gate on the output.  "State Space Models (SSM)" (ultralytics.com
// glossary), section "Da S4 a Mamba": every Mamba block wraps the selective SSM with a short
// convolution and a SiLU gate.  All three stream HBM once; float32 arithmetic.
#pragma once
#include "ssd_common.cuh"

namespace ssd {
namespace glue {

__device__ __forceinline__ float silu(float v) { return v / (1.f + expf(-v)); }

// softplus(v) = log(1 + e^v), written so that no exp overflows
__device__ __forceinline__ float softplus(float v) {
  return v > 20.f ? v : log1pf(expf(v));
}

template <typename T> struct vec;  // VW channels per thread, one 16-byte access
template <> struct vec<__nv_bfloat16> {
  static constexpr int VW = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    *reinterpret_cast<uint4*>(p) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                   pack_bf16x2(v[6], v[7]));
  }
};
template <> struct vec<float> {
  static constexpr int VW = 4;
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

// SiLU for the streaming kernels: the hardware exp2-based exponential and the approximate
// divide (a few float32 ulps; v / (1 + inf) gives -0 for v below about -88).
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// out[b,t,c] = silu(bias[c] + sum_{k<K} w[c,k] u[b, t-K+1+k, c]), u = 0 before t = 0.
// One thread per (batch row, 16-byte group of channels, run of kConvTok tokens): its weights
// and bias sit in registers, the last K-1 input rows in a register window, and the run's rows
// are read kConvStep at a time, their 16-byte loads issued together (a warp reads 32
// neighbouring groups: 512 contiguous bytes per row), so that a thread keeps several loads in
// flight.  The K-1 rows before the run are read again by the previous run's thread (K-1 of
// kConvTok).
constexpr int kConvTok = 64, kConvStep = 4;

template <typename T, int K>
__global__ void __launch_bounds__(32) conv_silu_kernel(const T* __restrict__ u,
                                                        const float* __restrict__ w,
                                                        const float* __restrict__ bias,
                                                        T* __restrict__ out, int64_t seqlen,
                                                        int cdim) {
  constexpr int VW = vec<T>::VW;
  constexpr int W = K - 1 + kConvStep;  // window rows: K - 1 before the step, then the step's
  const int cg = blockIdx.x * blockDim.x + threadIdx.x;
  if (cg >= cdim / VW) return;
  const int c0 = cg * VW;
  const int64_t t0 = int64_t(blockIdx.y) * kConvTok;
  const int64_t t1 = t0 + kConvTok < seqlen ? t0 + kConvTok : seqlen;
  const T* ub = u + int64_t(blockIdx.z) * seqlen * cdim + c0;
  T* ob = out + int64_t(blockIdx.z) * seqlen * cdim + c0;

  float wr[VW][K], bv[VW];
  {  // this thread's VW x K weights are contiguous: VW*K/4 float4 loads
    const float4* w4 = reinterpret_cast<const float4*>(w + int64_t(c0) * K);
#pragma unroll
    for (int i = 0; i < VW * K / 4; ++i) {
      const float4 v = __ldg(w4 + i);
      const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) wr[(4 * i + e) / K][(4 * i + e) % K] = f[e];
    }
  }
#pragma unroll
  for (int j = 0; j < VW; ++j) bv[j] = bias ? bias[c0 + j] : 0.f;

  float win[W][VW];  // win[k] = input row t-K+1+k; rows before t = 0 (and past the end) zero
#pragma unroll
  for (int k = 0; k < K - 1; ++k) {
    const int64_t ts = t0 - (K - 1) + k;
    if (ts >= 0) vec<T>::load(ub + ts * cdim, win[k]);
    else {
#pragma unroll
      for (int j = 0; j < VW; ++j) win[k][j] = 0.f;
    }
  }
  for (int64_t t = t0; t < t1; t += kConvStep) {
#pragma unroll
    for (int i = 0; i < kConvStep; ++i) {
      if (t + i < t1) vec<T>::load(ub + (t + i) * cdim, win[K - 1 + i]);
      else {
#pragma unroll
        for (int j = 0; j < VW; ++j) win[K - 1 + i][j] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < kConvStep; ++i) {
      if (t + i < t1) {
        float o[VW];
#pragma unroll
        for (int j = 0; j < VW; ++j) {
          float acc = bv[j];
#pragma unroll
          for (int k = 0; k < K; ++k) acc = fmaf(wr[j][k], win[i + k][j], acc);
          o[j] = silu_fast(acc);
        }
        vec<T>::store(ob + (t + i) * cdim, o);
      }
    }
#pragma unroll
    for (int k = 0; k < K - 1; ++k)
#pragma unroll
      for (int j = 0; j < VW; ++j) win[k][j] = win[k + kConvStep][j];
  }
}

// dt[b,t,h] = softplus(raw[b,t,h] + bias[h]); 8 consecutive elements per thread, read as two
// 16-byte loads when the pointers allow it (enough bytes in flight to stream HBM).
__global__ void __launch_bounds__(256) dt_softplus_kernel(const float* raw,
                                                          const float* __restrict__ bias,
                                                          float* dt, int64_t n, int nheads,
                                                          bool vec4) {
  const int64_t i0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i0 >= n) return;
  int h = int(i0 % nheads);
  float v[8];
  if (vec4 && i0 + 8 <= n) {
    const float4 a = *reinterpret_cast<const float4*>(raw + i0);
    const float4 b = *reinterpret_cast<const float4*>(raw + i0 + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = i0 + j < n ? raw[i0 + j] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = softplus(v[j] + (bias ? bias[h] : 0.f));
    h = h + 1 == nheads ? 0 : h + 1;
  }
  if (vec4 && i0 + 8 <= n) {
    *reinterpret_cast<float4*>(dt + i0) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(dt + i0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j < n) dt[i0 + j] = v[j];
  }
}

// out[i] = y[i] * silu(z[i]); VW elements per thread (the element count is a multiple of VW)
template <typename TZ, typename TO>
__global__ void __launch_bounds__(256) gate_silu_kernel(const float* y,
                                                        const TZ* __restrict__ z,
                                                        TO* out, int64_t n) {
  constexpr int VW = vec<TZ>::VW;
  const int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * VW;
  if (i >= n) return;
  float zv[VW], r[VW];
  vec<TZ>::load(z + i, zv);
#pragma unroll
  for (int j = 0; j < VW; j += 4) {
    const float4 yv = *reinterpret_cast<const float4*>(y + i + j);
    r[j] = yv.x * silu(zv[j]);
    r[j + 1] = yv.y * silu(zv[j + 1]);
    r[j + 2] = yv.z * silu(zv[j + 2]);
    r[j + 3] = yv.w * silu(zv[j + 3]);
  }
  if constexpr (sizeof(TO) == 4) {
#pragma unroll
    for (int j = 0; j < VW; j += 4)
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + i + j) =
          make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < VW; j += 8) {
      float rr[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) rr[q] = r[j + q];
      vec<__nv_bfloat16>::store(reinterpret_cast<__nv_bfloat16*>(out) + i + j, rr);
    }
  }
}

}  // namespace glue
}  // namespace ssd
