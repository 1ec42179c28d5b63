// glue_kernels.cuh -- the steps either side of the SSD layer inside a Mamba block: a short
// causal depthwise convolution with SiLU on the layer's inputs, the step size dt = softplus(raw
// + bias), and the SiLU gate on the output.  "Puntata 205 -- State Space Models e Mamba"
// (aiperbabbani.it), "Da S4 a Mamba": every Mamba block wraps the selective SSM with a short
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

// out[b,t,c] = silu(bias[c] + sum_{k<K} w[c,k] u[b, t-K+1+k, c]), u = 0 before t = 0.
// One thread per (b, t, group of VW channels); the K input rows it reads are shared with the
// neighbouring tokens' threads through L1.
template <typename T>
__global__ void __launch_bounds__(256) conv_silu_kernel(const T* __restrict__ u,
                                                        const float* __restrict__ w,
                                                        const float* __restrict__ bias,
                                                        T* __restrict__ out, int64_t seqlen,
                                                        int64_t ntok, int cdim, int K) {
  constexpr int VW = vec<T>::VW;
  const int ng = cdim / VW;
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= ntok * ng) return;
  const int64_t tok = i / ng;  // b * seqlen + t
  const int c0 = int(i % ng) * VW;
  const int64_t t = tok % seqlen;
  float acc[VW];
#pragma unroll
  for (int j = 0; j < VW; ++j) acc[j] = bias ? bias[c0 + j] : 0.f;
  for (int k = 0; k < K; ++k) {
    const int64_t ts = t - (K - 1) + k;
    if (ts < 0) continue;
    float v[VW];
    vec<T>::load(u + (tok - (K - 1) + k) * cdim + c0, v);
#pragma unroll
    for (int j = 0; j < VW; ++j) acc[j] = fmaf(w[(c0 + j) * K + k], v[j], acc[j]);
  }
#pragma unroll
  for (int j = 0; j < VW; ++j) acc[j] = silu(acc[j]);
  vec<T>::store(out + tok * cdim + c0, acc);
}

// dt[b,t,h] = softplus(raw[b,t,h] + bias[h])
__global__ void __launch_bounds__(256) dt_softplus_kernel(const float* raw,
                                                          const float* __restrict__ bias,
                                                          float* dt, int64_t n,
                                                          int nheads) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  dt[i] = softplus(raw[i] + (bias ? bias[i % nheads] : 0.f));
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
