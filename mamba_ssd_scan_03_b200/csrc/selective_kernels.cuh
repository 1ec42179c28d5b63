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
// Layout of the work: one warp (one CTA) per batch row and 8 channels; four lanes per channel,
// each lane holding 4 of the 16 states in registers for the whole sequence.  The inputs arrive
// as TMA tiles of 32 tokens ({8 channels} of x and dt, {16 states} of B and C) in a two-stage
// ring, so the loads cost the SM no per-row cache lookups (a plain 16-byte load of a 32-row
// tile takes one L1 lookup per row, and with ~4 warps per scheduler those lookups, not the
// exps, set the pace).  Rows past the end of the sequence are zero-filled by the TMA unit:
// dt = 0 makes them exact identity steps (decay 1, no input).  y goes out the same way: staged
// in shared memory (two buffers) and written by TMA stores, which drop rows past the end.
// Every wait on a TMA barrier is bounded; on expiry the kernel latches the device status word,
// waits (bounded) for its own copies in flight and returns without writing the final state.
#pragma once
#include "tc_prims.cuh"

namespace ssd {
namespace sel {

constexpr int kTok = 32;    // tokens per tile
constexpr int kCpw = 8;     // channels per warp
constexpr int kN = 16;      // states per channel
constexpr int kSpl = 4;     // states per lane
constexpr int kStages = 2;  // input tiles in flight

template <typename T, typename TY>
struct Smem {
  static constexpr int kX = kTok * kCpw * int(sizeof(T));   // x tile   [32][8]
  static constexpr int kDt = kTok * kCpw * 4;               // dt tile  [32][8] float32
  static constexpr int kBC = kTok * kN * int(sizeof(T));    // B, C tiles [32][16]
  static constexpr int kStage = kX + kDt + 2 * kBC;         // one TMA transaction
  static constexpr int kY = kTok * kCpw * int(sizeof(TY));  // y tile   [32][8]
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

// Preconditions (checked on the host): dstate == 16, dim % 8 == 0, (dim / ngroups) % 8 == 0,
// 16-byte aligned pointers; the tensor maps are 3-D {inner, seqlen, batch} with boxes
// {8, 32, 1} (x, dt, y) and {16, 32, 1} (B, C), no swizzle, zero fill.
template <typename T, typename TY>
__global__ void __launch_bounds__(32) selective_scan_kernel(
    const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mdt,
    const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mc,
    const __grid_constant__ CUtensorMap my, const float* __restrict__ A,
    const float* __restrict__ D, const float* __restrict__ init, float* __restrict__ fin,
    int64_t seqlen, int dim, int ngroups) {
  using S = Smem<T, TY>;
  extern __shared__ uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 127) &
                                           ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S::kBars);
  __shared__ int abort_flag;

  const int lane = threadIdx.x;
  const int c = lane >> 2, q = lane & 3;  // channel within the warp, state quarter
  const int wpr = dim / kCpw;             // warps per batch row
  const int b = int(blockIdx.x / wpr);
  const int d0 = int(blockIdx.x % wpr) * kCpw;
  const int d = d0 + c;
  const int g = d0 / (dim / ngroups);
  const int nck = int((seqlen + kTok - 1) / kTok);

  auto issue = [&](int k) {  // lane 0: the four input tiles of chunk k into stage k % kStages
    uint64_t* bar = &full[k % kStages];
    uint8_t* st = sm + (k % kStages) * S::kStage;
    tc::mbar_arrive_expect_tx(bar, uint32_t(S::kStage));
    tc::tma_load_3d(st, &mx, bar, d0, k * kTok, b);
    tc::tma_load_3d(st + S::kX, &mdt, bar, d0, k * kTok, b);
    tc::tma_load_3d(st + S::kX + S::kDt, &mb, bar, g * kN, k * kTok, b);
    tc::tma_load_3d(st + S::kX + S::kDt + S::kBC, &mc, bar, g * kN, k * kTok, b);
  };
  if (lane == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) tc::mbar_init(&full[s], 1);
    tc::fence_mbar_init();
    for (int k = 0; k < kStages && k < nck; ++k) issue(k);
  }
  __syncwarp();

  // per-lane constants: this lane's 4 decay rates in log2 units, the skip weight, the state
  float a2[kSpl];
  {
    const float4 av = *reinterpret_cast<const float4*>(A + int64_t(d) * kN + q * kSpl);
    a2[0] = av.x * kLog2e; a2[1] = av.y * kLog2e; a2[2] = av.z * kLog2e; a2[3] = av.w * kLog2e;
  }
  const float Dd = D ? D[d] : 0.f;
  float h[kSpl] = {0.f, 0.f, 0.f, 0.f};
  const int64_t st_off = (int64_t(b) * dim + d) * kN + q * kSpl;
  if (init) {
    const float4 iv = *reinterpret_cast<const float4*>(init + st_off);
    h[0] = iv.x; h[1] = iv.y; h[2] = iv.z; h[3] = iv.w;
  }

  int k = 0;
  for (; k < nck; ++k) {
    const int s = k % kStages;
    const bool got = tc::mbar_wait(&full[s], uint32_t(k / kStages) & 1u, &abort_flag, 60);
    if (__any_sync(0xffffffffu, !got)) break;
    // y buffer k & 1 was last handed to the TMA store of chunk k - 2
    if (lane == 0 && k >= 2) bulk_wait_read_all_but_one();
    __syncwarp();
    const uint8_t* stg = sm + s * S::kStage;
    const T* xs = reinterpret_cast<const T*>(stg);
    const float* ds = reinterpret_cast<const float*>(stg + S::kX);
    const T* bs = reinterpret_cast<const T*>(stg + S::kX + S::kDt);
    const T* cs = reinterpret_cast<const T*>(stg + S::kX + S::kDt + S::kBC);
    TY* ys = reinterpret_cast<TY*>(sm + kStages * S::kStage + (k & 1) * S::kY);
#pragma unroll 4
    for (int t = 0; t < kTok; ++t) {
      const float xv = load1(xs + t * kCpw + c), dv = ds[t * kCpw + c];
      const float4 bv = load4(bs + t * kN + q * kSpl);
      const float4 cv = load4(cs + t * kN + q * kSpl);
      const float u = dv * xv;
      h[0] = fmaf(ex2(dv * a2[0]), h[0], u * bv.x);
      h[1] = fmaf(ex2(dv * a2[1]), h[1], u * bv.y);
      h[2] = fmaf(ex2(dv * a2[2]), h[2], u * bv.z);
      h[3] = fmaf(ex2(dv * a2[3]), h[3], u * bv.w);
      float p = fmaf(cv.z, h[2], cv.x * h[0]) + fmaf(cv.w, h[3], cv.y * h[1]);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      if (q == 0) store1(ys + t * kCpw + c, fmaf(Dd, xv, p));
    }
    tc::fence_proxy_async_smem();  // this lane's y writes -> visible to the TMA store
    __syncwarp();                  // every lane is done with stage s and with ys
    if (lane == 0) {
      tc::tma_store_3d(&my, ys, d0, k * kTok, b);
      tc::bulk_commit();
      if (k + kStages < nck) issue(k + kStages);
    }
  }
  if (k < nck) {
    // aborted at chunk k: chunks k .. min(k + kStages, nck) - 1 may still be landing
    if (lane == 0)
      for (int j = k; j < k + kStages && j < nck; ++j)
        drain_wait(&full[j % kStages], uint32_t(j / kStages) & 1u);
  } else if (fin) {
    *reinterpret_cast<float4*>(fin + st_off) = make_float4(h[0], h[1], h[2], h[3]);
  }
  if (lane == 0) tc::bulk_wait_all();
  __syncwarp();
}

}  // namespace sel
}  // namespace ssd
