// step_kernels.cuh -- the single-token recurrent update (decode).
//
//   alpha = exp(dt[b,h] A[h]);  h[p,n] <- alpha h[p,n] + dt x[p] B[n];  y[p] = sum_n C[n] h[p,n] + D x[p]
//
// "State Space Models (SSM)" (ultralytics.com glossary), section "Come funzionano gli SSM":
// the recurrent form, one state update per token.  The state is the only large tensor
// (batch*heads*headdim*dstate float32), so the kernel is an HBM stream: every state element
// is read once and written once with 128-bit streaming accesses, y is reduced from the
// updated registers in the same pass, and nothing else touches HBM in bulk.
#pragma once
#include "ssd_common.cuh"

namespace ssd {

// Fast path: dstate == 128 (one float4 of the row per lane, a warp per row), block of 8 warps
// per (b, h), RPW rows per warp issued back to back so each lane has RPW 16-byte loads in flight.
template <typename T, typename TY, int RPW>
__global__ void __launch_bounds__(256) step_n128_kernel(
    float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
    const float* __restrict__ D, TY* __restrict__ y, int nheads, int heads_per_group,
    int ngroups) {
  constexpr int N = 128;
  constexpr int P = 8 * RPW;
  const int64_t bh = blockIdx.x;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / heads_per_group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const float delta = dt[bh];
  const float alpha = expf(delta * A[h]);
  const float dh = D ? D[h] : 0.0f;
  const int64_t bc = (b * ngroups + g) * N + lane * 4;
  float Bn[4], Cn[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    Bn[i] = io_traits<T>::load(Bm, bc + i);
    Cn[i] = io_traits<T>::load(Cm, bc + i);
  }
  const int p0 = warp * RPW;
  float4* rowp = reinterpret_cast<float4*>(state + (bh * P + p0) * N) + lane;
  float4 s[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) s[r] = __ldcs(rowp + r * (N / 4));
  float xv[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) xv[r] = io_traits<T>::load(x, bh * P + p0 + r);
  float acc[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const float u = delta * xv[r];
    s[r].x = fmaf(alpha, s[r].x, u * Bn[0]);
    s[r].y = fmaf(alpha, s[r].y, u * Bn[1]);
    s[r].z = fmaf(alpha, s[r].z, u * Bn[2]);
    s[r].w = fmaf(alpha, s[r].w, u * Bn[3]);
    __stcs(rowp + r * (N / 4), s[r]);
    acc[r] = Cn[0] * s[r].x + Cn[1] * s[r].y + Cn[2] * s[r].z + Cn[3] * s[r].w;
  }
#pragma unroll
  for (int r = 0; r < RPW; ++r) acc[r] = warp_sum(acc[r]);
  if (lane < RPW) {
    // lane r writes row r's output (select without dynamic register indexing)
    float out = 0.0f, xo = 0.0f;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
      if (lane == r) { out = acc[r]; xo = xv[r]; }
    io_traits<TY>::store(y, bh * P + p0 + lane, out + dh * xo);
  }
}

// General shapes: a warp per (p) row, lanes stride over dstate.
template <typename T, typename TY>
__global__ void __launch_bounds__(256) step_generic_kernel(
    float* __restrict__ state, const T* __restrict__ x, const float* __restrict__ dt,
    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
    const float* __restrict__ D, TY* __restrict__ y, int nheads, int headdim, int dstate,
    int heads_per_group, int ngroups) {
  const int64_t bh = blockIdx.x;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / heads_per_group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float delta = dt[bh];
  const float alpha = expf(delta * A[h]);
  const float dh = D ? D[h] : 0.0f;
  const int64_t bc = (b * ngroups + g) * dstate;
  for (int p = warp; p < headdim; p += blockDim.x / 32) {
    const float xv = io_traits<T>::load(x, bh * headdim + p);
    const float u = delta * xv;
    float* row = state + (bh * headdim + p) * dstate;
    float acc = 0.0f;
    for (int n = lane; n < dstate; n += 32) {
      const float sv = fmaf(alpha, row[n], u * io_traits<T>::load(Bm, bc + n));
      row[n] = sv;
      acc += io_traits<T>::load(Cm, bc + n) * sv;
    }
    acc = warp_sum(acc);
    if (lane == 0) io_traits<TY>::store(y, bh * headdim + p, acc + dh * xv);
  }
}

}  // namespace ssd
