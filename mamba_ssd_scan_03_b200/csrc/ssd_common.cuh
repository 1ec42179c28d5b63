// ssd_common.cuh -- small helpers shared by the SSD kernels (one translation unit: ssd_lib.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// log2(e): decays are evaluated as exp2(a * log2 e) on the MUFU ex2 unit.
constexpr float kLog2e = 1.4426950408889634f;

// Device status word latched by kernels whose bounded waits expire (0 = OK).  Bits:
// low byte = ssd_status code, upper bits = site id of the wait that gave up.
__device__ unsigned int g_status;

__device__ __forceinline__ void latch_status(unsigned code, unsigned site) {
  atomicCAS(&g_status, 0u, code | (site << 8));
}

// Hardware 2^x (MUFU ex2, approximate, flush-to-zero): a PTX instruction, not a library call.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T> struct io_traits;
template <> struct io_traits<float> {
  static __device__ __forceinline__ float load(const float* p, int64_t i) { return p[i]; }
  static __device__ __forceinline__ void store(float* p, int64_t i, float v) { p[i] = v; }
  // four consecutive elements from p + i, 16-byte aligned
  static __device__ __forceinline__ void load4(const float* p, int64_t i, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p + i);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
  }
};
template <> struct io_traits<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
  }
  // four consecutive elements from p + i, 8-byte aligned
  static __device__ __forceinline__ void load4(const __nv_bfloat16* p, int64_t i, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2*>(p + i);
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xffff0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, int64_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_inclusive_scan(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// bf16 helpers on raw 16-bit patterns (round to nearest even via the CUDA intrinsic).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Packed two-lane float32 arithmetic (sm_100 f32x2 instructions).  Each lane is rounded to
// nearest exactly as the scalar operation would round it.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// a * b + c per lane, one rounding (as fmaf)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// ---- register-tiled outer-product sums (float32 CUDA cores) ----------------------------------
// out[p * N + n] = sum over a chunk's tokens s of u_s[p] v_s[n], for a P x N output, by a block
// of kOuterThreads threads, 4 x 4 outputs per thread and tile (two 16-byte shared loads per 16
// FMAs).  stage(s0, ts, us, vs) fills ts = outer_ts(P, N) token rows: us [ts][P4], vs [ts][N4]
// (P4, N4: P and N rounded up to multiples of 4; the padding and rows past the chunk's end
// hold zeros).  Shared memory: outer_smem_floats(P, N).
constexpr int kOuterThreads = 256, kOuterTiles = 2;
__host__ __device__ inline int round4(int v) { return (v + 3) & ~3; }
// token rows per staging step: a whole 64-token chunk for the usual widths (one barrier pair),
// fewer for wide states
__host__ __device__ inline int outer_ts(int P, int N) {
  const int w = round4(P) + round4(N);
  return w <= 192 ? 64 : (w <= 384 ? 32 : 16);
}
__host__ __device__ inline size_t outer_smem_floats(int P, int N) {
  return size_t(outer_ts(P, N)) * (round4(P) + round4(N));
}
// Four consecutive elements (a multiple-of-4 offset i) of a row of `len`: one vector load when
// `vec` (the row length a multiple of 4 and the base aligned), else element by element with
// zeros past the row's end.
template <typename T>
__device__ __forceinline__ void load4_row(const T* p, int64_t i, int col, int len, bool vec,
                                          float (&v)[4]) {
  if (vec) {
    io_traits<T>::load4(p, i, v);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = col + q < len ? io_traits<T>::load(p, i + q) : 0.f;
  }
}
template <typename T>
__device__ __forceinline__ bool vec4_ok(const T* p, int len) {
  return len % 4 == 0 && (reinterpret_cast<uintptr_t>(p) % (4 * sizeof(T))) == 0;
}

template <typename Stage>
__device__ __forceinline__ void outer_sum(const Stage& stage, int ntok, int P, int N,
                                          float* __restrict__ out, float* us, float* vs) {
  const int P4 = round4(P), N4 = round4(N), ts = outer_ts(P, N);
  const int ntn = N4 / 4, ntiles = (P4 / 4) * ntn;
  for (int base = 0; base < ntiles; base += kOuterThreads * kOuterTiles) {
    float acc[kOuterTiles][4][4];
    int tp[kOuterTiles], tn[kOuterTiles];
    bool live[kOuterTiles];
#pragma unroll
    for (int k = 0; k < kOuterTiles; ++k) {
      const int idx = base + k * kOuterThreads + int(threadIdx.x);
      live[k] = idx < ntiles;  // a tile past the end computes tile 0 again and stores nothing
      tp[k] = live[k] ? idx / ntn : 0;
      tn[k] = live[k] ? idx % ntn : 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[k][i][j] = 0.f;
    }
    for (int s0 = 0; s0 < ntok; s0 += ts) {
      __syncthreads();
      stage(s0, ts, us, vs);
      __syncthreads();
#pragma unroll 4
      for (int s = 0; s < ts; ++s) {
#pragma unroll
        for (int k = 0; k < kOuterTiles; ++k) {
          const float4 u = *reinterpret_cast<const float4*>(us + s * P4 + 4 * tp[k]);
          const float4 v = *reinterpret_cast<const float4*>(vs + s * N4 + 4 * tn[k]);
          const float uu[4] = {u.x, u.y, u.z, u.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[k][i][j] = fmaf(uu[i], vv[j], acc[k][i][j]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kOuterTiles; ++k) {
      if (!live[k]) continue;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int p = 4 * tp[k] + i;
        if (p >= P) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n = 4 * tn[k] + j;
          if (n < N) out[int64_t(p) * N + n] = acc[k][i][j];
        }
      }
    }
  }
}

}  // namespace ssd
