// selective_kernels.cuh -- the selective scan with a per-state (diagonal) transition, the first
// Mamba generation's layer.  "Architektury Mamba-2, State Space Models i liniowa atencja"
// (tech.tersel.eu), section "Od S4 do Mamba-1: Wprowadzenie mechanizmu selektywnego": B, C and
// the step dt depend on the input, and the recurrence is scanned on CUDA cores with the state
// held on chip instead of materialised in HBM.  Per batch row b and channel d (group g):
//
//   h_t[n] = exp(dt_t[d] A[d,n]) h_{t-1}[n] + dt_t[d] B_t[g,n] x_t[d]
//   y_t[d] = sum_n C_t[g,n] h_t[n] + D[d] x_t[d]
//
// Unlike the scalar-transition layer there is no matrix form to put on the tensor cores: every
// (token, channel, state) needs its own exp, so the kernel is bound by the MUFU ex2 rate.
//
// Layout of the work: one warp per batch row and 8 channels; four lanes per channel, each lane
// holding 4 of the 16 states in registers for the whole sequence.  The warp streams its inputs
// in chunks of 32 tokens: 16-byte global loads one chunk ahead into registers, unpacked to
// float32 in the warp's own shared-memory tiles; y is staged the same way and written with
// 16-byte stores.  Warps are independent (one-warp CTAs, __syncwarp only), so the grid spreads
// evenly over the SM sub-partitions whose ex2 units bound the kernel.
#pragma once
#include "ssd_common.cuh"

namespace ssd {
namespace sel {

constexpr int kTok = 32;   // tokens per staged chunk
constexpr int kCpw = 8;    // channels per warp
constexpr int kN = 16;     // states per channel
constexpr int kSpl = 4;    // states per lane (kN / lanes per channel)

// A [kTok][W] tile of T from global memory, row stride `ld` elements, moved through registers
// (one chunk ahead) into a float32 shared-memory tile.  Rows at or past `rows` read as zero.
template <typename T, int W>
struct Tile {
  static constexpr int EPV = 16 / int(sizeof(T));  // elements per 16-byte vector
  static constexpr int VPR = W / EPV;              // vectors per row
  static constexpr int NV = kTok * VPR / 32;       // vectors per lane
  static_assert(kTok * VPR % 32 == 0, "tile must split evenly over the warp");
  uint4 r[NV];

  __device__ __forceinline__ void load(const T* base, int64_t ld, int rows, int lane) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int v = lane + 32 * j, row = v / VPR, col = (v % VPR) * EPV;
      r[j] = row < rows ? __ldg(reinterpret_cast<const uint4*>(base + row * ld + col))
                        : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ __forceinline__ void stage(float (*s)[W], int lane) const {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int v = lane + 32 * j, row = v / VPR, col = (v % VPR) * EPV;
      float4* d = reinterpret_cast<float4*>(&s[row][col]);
      if constexpr (sizeof(T) == 4) {
        d[0] = make_float4(__uint_as_float(r[j].x), __uint_as_float(r[j].y),
                           __uint_as_float(r[j].z), __uint_as_float(r[j].w));
      } else {
        d[0] = make_float4(bf16lo(r[j].x), bf16hi(r[j].x), bf16lo(r[j].y), bf16hi(r[j].y));
        d[1] = make_float4(bf16lo(r[j].z), bf16hi(r[j].z), bf16lo(r[j].w), bf16hi(r[j].w));
      }
    }
  }
};

// y tile [kTok][kCpw] float32 in shared memory -> global rows (stride `ld`), rows < `rows`.
template <typename TY>
__device__ __forceinline__ void store_y(const float (*s)[kCpw], TY* base, int64_t ld, int rows,
                                        int lane) {
  if constexpr (sizeof(TY) == 4) {  // 32 rows x 2 float4
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int v = lane + 32 * j, row = v >> 1, col = (v & 1) * 4;
      if (row < rows)
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + row * ld + col) =
            *reinterpret_cast<const float4*>(&s[row][col]);
    }
  } else {  // 32 rows x one 16-byte vector of 8 bf16
    if (lane < rows) {
      const float4 a = *reinterpret_cast<const float4*>(&s[lane][0]);
      const float4 b = *reinterpret_cast<const float4*>(&s[lane][4]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + lane * ld) =
          make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                     pack_bf16x2(b.z, b.w));
    }
  }
}

// One warp per (batch row, 8 channels).  Preconditions (checked on the host): dstate == 16,
// dim % 8 == 0, (dim / ngroups) % 8 == 0, every pointer 16-byte aligned.
template <typename T, typename TY>
__global__ void __launch_bounds__(32) selective_scan_kernel(
    const T* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
    const T* __restrict__ B, const T* __restrict__ C, const float* __restrict__ D,
    const float* __restrict__ init, TY* __restrict__ y, float* __restrict__ fin,
    int64_t seqlen, int dim, int ngroups) {
  __shared__ __align__(16) float xs[kTok][kCpw];
  __shared__ __align__(16) float ds[kTok][kCpw];
  __shared__ __align__(16) float bs[kTok][kN];
  __shared__ __align__(16) float cs[kTok][kN];
  __shared__ __align__(16) float ys[kTok][kCpw];

  const int lane = threadIdx.x;
  const int c = lane >> 2, q = lane & 3;  // channel within the warp, state quarter
  const int wpr = dim / kCpw;             // warps per batch row
  const int64_t b = blockIdx.x / wpr;
  const int d0 = int(blockIdx.x % wpr) * kCpw;
  const int d = d0 + c;
  const int g = d0 / (dim / ngroups);

  // per-lane constants: this lane's 4 decay rates in log2 units, the skip weight
  float2 a2[2];
  {
    const float4 av = *reinterpret_cast<const float4*>(A + int64_t(d) * kN + q * kSpl);
    a2[0] = make_float2(av.x * kLog2e, av.y * kLog2e);
    a2[1] = make_float2(av.z * kLog2e, av.w * kLog2e);
  }
  const float Dd = D ? D[d] : 0.f;
  float2 h[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  const int64_t st = (b * dim + d) * kN + q * kSpl;  // this lane's slice of the state
  if (init) {
    const float4 iv = *reinterpret_cast<const float4*>(init + st);
    h[0] = make_float2(iv.x, iv.y);
    h[1] = make_float2(iv.z, iv.w);
  }

  const int64_t row0 = b * seqlen;  // first token row of this batch row
  const int64_t gld = int64_t(ngroups) * kN;
  Tile<T, kCpw> tx;
  Tile<float, kCpw> td;
  Tile<T, kN> tb, tc;
  auto fetch = [&](int64_t t0) {
    const int rows = int(seqlen - t0 < kTok ? seqlen - t0 : kTok);
    tx.load(x + (row0 + t0) * dim + d0, dim, rows, lane);
    td.load(dt + (row0 + t0) * dim + d0, dim, rows, lane);
    tb.load(B + (row0 + t0) * gld + int64_t(g) * kN, gld, rows, lane);
    tc.load(C + (row0 + t0) * gld + int64_t(g) * kN, gld, rows, lane);
  };

  fetch(0);
  for (int64_t t0 = 0; t0 < seqlen; t0 += kTok) {
    __syncwarp();  // the previous chunk's reads of the tiles (and of ys) are done
    tx.stage(xs, lane);
    td.stage(ds, lane);
    tb.stage(bs, lane);
    tc.stage(cs, lane);
    __syncwarp();
    if (t0 + kTok < seqlen) fetch(t0 + kTok);
    // Rows past the end were staged as zeros: dt = 0 makes them identity steps (decay 1, no
    // input), so the state carried out of the last chunk is exact without a per-token check.
#pragma unroll 4
    for (int t = 0; t < kTok; ++t) {
      const float xv = xs[t][c], dv = ds[t][c];
      const float4 bv = *reinterpret_cast<const float4*>(&bs[t][q * kSpl]);
      const float4 cv = *reinterpret_cast<const float4*>(&cs[t][q * kSpl]);
      const float2 dd = make_float2(dv, dv);
      const float2 l0 = mul2(dd, a2[0]), l1 = mul2(dd, a2[1]);
      const float2 e0 = make_float2(ex2(l0.x), ex2(l0.y)), e1 = make_float2(ex2(l1.x), ex2(l1.y));
      const float u = dv * xv;
      const float2 uu = make_float2(u, u);
      h[0] = fma2(e0, h[0], mul2(uu, make_float2(bv.x, bv.y)));
      h[1] = fma2(e1, h[1], mul2(uu, make_float2(bv.z, bv.w)));
      const float2 acc = fma2(make_float2(cv.z, cv.w), h[1], mul2(make_float2(cv.x, cv.y), h[0]));
      float s = acc.x + acc.y;
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (q == 0) ys[t][c] = fmaf(Dd, xv, s);
    }
    __syncwarp();
    const int rows = int(seqlen - t0 < kTok ? seqlen - t0 : kTok);
    store_y<TY>(ys, y + (row0 + t0) * dim + d0, dim, rows, lane);
  }
  if (fin) {
    *reinterpret_cast<float4*>(fin + st) = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
  }
}

}  // namespace sel
}  // namespace ssd
