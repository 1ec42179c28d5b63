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
// (token, channel, state) needs its own exp, so the kernel is bound by the SFU's ex2 rate.
//
// Layout of the work: a CTA of one warp per batch row and 8 channels; four lanes per channel,
// each lane holding 4 of the 16 states in registers for the whole sequence.  One warp per CTA
// makes the most CTAs (2,560 at 4 x 5,120 channels: 17.3 per SM, so no SM holds much more than
// its share of a grid that runs in one wave); four warps sharing the group's B and C tiles
// measured 8% slower, as 640 CTAs put five on some SMs and four on most.  The inputs arrive as
// TMA tiles of 32 tokens ({8 channels} of x and dt, {16 states} of B and C) in a two-stage ring,
// so the loads cost the SM no per-row cache lookups.  Rows past the end of the sequence
// are zero-filled by the TMA unit: dt = 0 makes them exact identity steps (decay 1, no input).
// Per token a lane updates its four states with packed float32 pairs; every four tokens the four
// lanes of a channel reduce-scatter their partial y sums (three shuffles), so that each lane
// finishes and stores one token's y.  y is staged in shared memory (two buffers) and written by
// TMA stores, which drop rows past the end.  Every wait on a TMA barrier is bounded; on expiry
// the kernel latches the device status word, waits (bounded) for its own copies in flight and
// returns without writing the final state.
#pragma once
#include "tc_prims.cuh"

namespace ssd {
namespace sel {

constexpr int kTok = 32;    // tokens per tile
constexpr int kCpw = 8;     // channels per CTA (one warp)
constexpr int kN = 16;      // states per channel
constexpr int kSpl = 4;     // states per lane
constexpr int kStages = 2;  // input tiles in flight

template <typename T, typename TY>
struct Smem {
  static constexpr int kCw = kCpw;                           // channels per CTA
  static constexpr int kX = kTok * kCw * int(sizeof(T));    // x tile   [32][kCw]
  static constexpr int kDt = kTok * kCw * 4;                // dt tile  [32][kCw] float32
  static constexpr int kBC = kTok * kN * int(sizeof(T));    // B, C tiles [32][16]
  static constexpr int kStage = kX + kDt + 2 * kBC;         // one TMA transaction
  static constexpr int kY = kTok * kCw * int(sizeof(TY));   // y tile   [32][kCw]
  static constexpr int kBars = kStages * kStage + 2 * kY;   // offset of the barriers
  static constexpr int kBytes = kBars + 64 + 128;           // + barriers + alignment slack
  static_assert(kX % 128 == 0 && kDt % 128 == 0 && kBC % 128 == 0 && kY % 128 == 0,
                "tiles must stay 128-byte aligned");
};

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) {
  return __uint_as_float(uint32_t(*reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return bf16_at(p); }
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
}
__device__ __forceinline__ void store1(float* p, float v) { *p = v; }
__device__ __forceinline__ void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Allow the most recent bulk group to be pending; every older one has finished reading smem.
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Bounded wait that ignores the abort flag: used after an abort to let this CTA's own TMA
// loads land before it exits.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_test_sleep(bar, parity, 20000u))
    if (tc::globaltimer() - t0 > 1000000000ull) return;
}

// Preconditions (checked on the host): dstate == 16, (dim / ngroups) % 8 == 0, 16-byte aligned
// pointers; the tensor maps are 3-D {inner, seqlen, batch} with boxes {8, 32, 1} (x, dt, y) and
// {16, 32, 1} (B, C), no swizzle, zero fill.
template <typename T, typename TY>
__global__ void __launch_bounds__(32) selective_scan_kernel(
    const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mdt,
    const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mc,
    const __grid_constant__ CUtensorMap my, const float* __restrict__ A,
    const float* __restrict__ D, const float* __restrict__ init, float* __restrict__ fin,
    int64_t seqlen, int dim, int ngroups) {
  using S = Smem<T, TY>;
  constexpr int CW = S::kCw;
  extern __shared__ uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 127) &
                                           ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S::kBars);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, lane = tid;
  const int c = lane >> 2, q = lane & 3;  // channel within the CTA, state quarter
  const int cw = c;                       // channel within the CTA's tiles
  const int cpr = dim / CW;               // CTAs per batch row
  const int b = int(blockIdx.x / cpr);
  const int d0 = int(blockIdx.x % cpr) * CW;
  const int d = d0 + cw;
  const int g = d0 / (dim / ngroups);
  const int nck = int((seqlen + kTok - 1) / kTok);

  auto issue = [&](int k) {  // thread 0: the four input tiles of chunk k into stage k % kStages
    uint64_t* bar = &full[k % kStages];
    uint8_t* st = sm + (k % kStages) * S::kStage;
    tc::mbar_arrive_expect_tx(bar, uint32_t(S::kStage));
    tc::tma_load_3d(st, &mx, bar, d0, k * kTok, b);
    tc::tma_load_3d(st + S::kX, &mdt, bar, d0, k * kTok, b);
    tc::tma_load_3d(st + S::kX + S::kDt, &mb, bar, g * kN, k * kTok, b);
    tc::tma_load_3d(st + S::kX + S::kDt + S::kBC, &mc, bar, g * kN, k * kTok, b);
  };
  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) tc::mbar_init(&full[s], 1);
    tc::fence_mbar_init();
    for (int k = 0; k < kStages && k < nck; ++k) issue(k);
  }
  __syncthreads();

  // per-lane constants: this lane's 4 decay rates in log2 units, the skip weight, the state
  float2 a01, a23;
  {
    const float4 av = *reinterpret_cast<const float4*>(A + int64_t(d) * kN + q * kSpl);
    a01 = make_float2(av.x * kLog2e, av.y * kLog2e);
    a23 = make_float2(av.z * kLog2e, av.w * kLog2e);
  }
  const float Dd = D ? D[d] : 0.f;
  float2 h01 = make_float2(0.f, 0.f), h23 = make_float2(0.f, 0.f);
  const int64_t st_off = (int64_t(b) * dim + d) * kN + q * kSpl;
  if (init) {
    const float4 iv = *reinterpret_cast<const float4*>(init + st_off);
    h01 = make_float2(iv.x, iv.y);
    h23 = make_float2(iv.z, iv.w);
  }
  const int b0 = q & 1, b1 = q >> 1;

  int k = 0;
  for (; k < nck; ++k) {
    const int s = k % kStages;
    const bool got = tc::mbar_wait(&full[s], uint32_t(k / kStages) & 1u, &abort_flag, 60);
    if (__syncthreads_or(!got)) break;
    // y buffer k & 1 was last handed to the TMA store of chunk k - 2
    if (tid == 0 && k >= 2) bulk_wait_read_all_but_one();
    __syncthreads();
    const uint8_t* stg = sm + s * S::kStage;
    const T* xs = reinterpret_cast<const T*>(stg);
    const float* ds = reinterpret_cast<const float*>(stg + S::kX);
    const T* bs = reinterpret_cast<const T*>(stg + S::kX + S::kDt);
    const T* cs = reinterpret_cast<const T*>(stg + S::kX + S::kDt + S::kBC);
    TY* ys = reinterpret_cast<TY*>(sm + kStages * S::kStage + (k & 1) * S::kY);
#pragma unroll 2
    for (int t0 = 0; t0 < kTok; t0 += 4) {
      float pv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = t0 + i;
        const float xv = load1(xs + t * CW + cw), dv = ds[t * CW + cw];
        const float4 bv = load4(bs + t * kN + q * kSpl);
        const float4 cv = load4(cs + t * kN + q * kSpl);
        const float2 dd = make_float2(dv, dv);
        const float2 l01 = mul2(dd, a01), l23 = mul2(dd, a23);
        const float u = dv * xv;
        const float2 uu = make_float2(u, u);
        h01 = fma2(make_float2(ex2(l01.x), ex2(l01.y)), h01, mul2(uu, make_float2(bv.x, bv.y)));
        h23 = fma2(make_float2(ex2(l23.x), ex2(l23.y)), h23, mul2(uu, make_float2(bv.z, bv.w)));
        const float2 pp = fma2(make_float2(cv.z, cv.w), h23, mul2(make_float2(cv.x, cv.y), h01));
        pv[i] = pp.x + pp.y;
      }
      // reduce-scatter over the channel's four lanes: lane q ends with token t0 + q's sum
      const float r0 = __shfl_xor_sync(0xffffffffu, b0 ? pv[0] : pv[1], 1);
      const float k0 = (b0 ? pv[1] : pv[0]) + r0;  // token t0 + b0
      const float r1 = __shfl_xor_sync(0xffffffffu, b0 ? pv[2] : pv[3], 1);
      const float k1 = (b0 ? pv[3] : pv[2]) + r1;  // token t0 + 2 + b0
      const float r2 = __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
      const float yq = (b1 ? k1 : k0) + r2;        // token t0 + q
      const int tq = t0 + q;
      store1(ys + tq * CW + cw, fmaf(Dd, load1(xs + tq * CW + cw), yq));
    }
    tc::fence_proxy_async_smem();  // this thread's y writes -> visible to the TMA store
    __syncthreads();               // every thread is done with stage s and with ys
    if (tid == 0) {
      tc::tma_store_3d(&my, ys, d0, k * kTok, b);
      tc::bulk_commit();
      if (k + kStages < nck) issue(k + kStages);
    }
  }
  if (k < nck) {
    // aborted at chunk k: chunks k .. min(k + kStages, nck) - 1 may still be landing
    if (tid == 0)
      for (int j = k; j < k + kStages && j < nck; ++j)
        drain_wait(&full[j % kStages], uint32_t(j / kStages) & 1u);
  } else if (fin) {
    *reinterpret_cast<float4*>(fin + st_off) = make_float4(h01.x, h01.y, h23.x, h23.y);
  }
  if (tid == 0) tc::bulk_wait_all();
  __syncthreads();
}

}  // namespace sel
}  // namespace ssd
