// tc_kernels.cuh -- the chunked scan on sm_100a tensor cores (bf16 io, headdim 64, dstate 128).
//
// The sequence of each (batch row, head) is cut into 128-token blocks (the tcgen05 M=128 tile)
// and the blocks into segments of consecutive blocks.  Three kernels, in stream order:
//
//  seg_state   per (b, segment, head quad): S_seg = sum_{t in seg} exp(sum_{k>t in seg} a_k)
//              dt_t B_t x_t^T, one long-K GEMM on the tensor cores (A = B^T, B = w*x, K =
//              tokens), plus the segment's total log-decay.  Reads x and B once.
//  seg_scan    per state element: H_in(seg) = state entering each segment (the linear state
//              passing between blocks, here at segment granularity), and final_state.
//  chunk_out   per (b, segment, head pair): walks the segment's blocks in order with the
//              running state resident in TMEM.  Per block: G = C B^T (once for both heads),
//              masked diagonal tile (L o G o dt) X, off-diagonal C H, skip term D x, y store,
//              then H <- exp(cs_end) H + B^T (w*x) in place.
//
// "Mamba-2 (2024): SSM e attention sono la stessa cosa" (paithon.it), "Il trucco a blocchi":
// quadratic attention-like form inside blocks, state summary passed between blocks.
// "State Space Model" (book.paithon.it), "Un sistema che riassume il passato": the parallel
// scan fuses steps pairwise by associativity of their composition, which is what lets a
// segment's steps be summarised by (total decay, state) and combined afterwards.
//
// Decays are carried in log2 units (a = dt*A*log2 e) and evaluated with ex2.  Every decay
// factor used is exp of a non-positive number, so nothing overflows: the diagonal tile's
// mask uses exact per-element exps on its 16x16 diagonal sub-blocks and, elsewhere, the
// product of two factors <= 1 split at the sub-block boundary r: exp(cs_t-cs_s) =
// exp(cs_t-cs_r) * exp(cs_r-cs_s) with s <= r <= t.
#pragma once
#include "tc_prims.cuh"

namespace ssd {
namespace tc {

constexpr int kP = 64;     // headdim
constexpr int kN = 128;    // dstate
constexpr int kBlk = 128;  // tokens per block
constexpr uint32_t kTile = 16384;  // one 128-row x 128-byte swizzled region

struct Seg {
  int nblk;      // 128-token blocks per sequence
  int seg_blks;  // blocks per segment
  int nseg;      // segments per sequence
};

// Inclusive scan over the 128 threads of one half of a 256-thread CTA (warps 0-3 form half 0,
// warps 4-7 half 1).  Returns the prefix and writes the half's total to *total.  Every thread
// of the CTA must call it (it synchronises the CTA).
__device__ __forceinline__ float half_scan128(float v, float* scratch8, float* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_inclusive_scan(v);
  if (lane == 31) scratch8[warp] = v;
  __syncthreads();
  const int w0 = warp & ~3;
  float off = 0.f, tot = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float s = scratch8[w0 + w];
    off += (w0 + w < warp) ? s : 0.f;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return v + off;
}

// Wait (bounded) for a phase of an mbarrier; used only on the abort path so that no copy or
// MMA is still writing shared memory or TMEM when the CTA leaves.
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_test(bar, parity)) {
    if (globaltimer() - t0 > 200000000ull) break;
  }
}

// Split a float pair into bf16 high parts and the bf16 rounding of the remainders.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  lo = pack_bf16x2(a - bf16lo(hi), b - bf16hi(hi));
}

// =============================================================================================
// seg_state: grid = batch * nseg * (nheads / 2), block = 256 threads: thread (row = tid % 128,
// head j = tid / 128) owns token row `row` of head j's x tile.  Per stage (two stages):
//   B tile (2 x 16 KB, n halves) | X'hi (2 heads x 16 KB) | X'lo (2 heads x 16 KB)
// X' = w * x is split into a bf16 high part (written over x) and a bf16 low part, and both go
// through the tensor core, so the segment state carries ~16 significant bits of X'.
// TMEM: 128 columns, lane n / column (j, p) = S_seg[n, (j, p)].
// =============================================================================================
constexpr uint32_t kSegStage = 6 * kTile;

__global__ void __launch_bounds__(256, 1) seg_state_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const float* __restrict__ dt, const float* __restrict__ A, float* __restrict__ seg_states,
    float* __restrict__ seg_decay, int64_t seqlen, int nheads, int heads_per_group, Seg sg) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full_bar[2], mma_bar[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ float scan_scratch[8];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int row = tid & 127, j = tid >> 7, warp = tid >> 5;
  const int npair = nheads / 2;
  const int unit = blockIdx.x;
  const int hp = unit % npair;
  const int seg = (unit / npair) % sg.nseg;
  const int b = unit / (npair * sg.nseg);
  const int h0 = hp * 2;
  const int g = h0 / heads_per_group;
  const int blk0 = seg * sg.seg_blks;
  const int nb = min(sg.nblk, blk0 + sg.seg_blks) - blk0;

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < 2; ++i) { mbar_init(&full_bar[i], 1); mbar_init(&mma_bar[i], 1); }
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_b);
  }
  if (warp == 0) tmem_alloc(&tmem_base_sh, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_v = &abort_flag;
  uint32_t n_loads[2] = {0, 0}, n_commits[2] = {0, 0};  // thread 0's issue counts per stage

  auto issue_loads = [&](int i, int stage) {  // block i of the walk (last block first)
    const int blk = blk0 + nb - 1 - i;
    uint8_t* st = smem + stage * kSegStage;
    ++n_loads[stage];
    mbar_arrive_expect_tx(&full_bar[stage], 4 * kTile);
    tma_load_3d(st, &tm_b, &full_bar[stage], g * kN, blk * kBlk, b);
    tma_load_3d(st + kTile, &tm_b, &full_bar[stage], g * kN + 64, blk * kBlk, b);
    tma_load_3d(st + 2 * kTile, &tm_x, &full_bar[stage], h0 * kP, blk * kBlk, b);
    tma_load_3d(st + 3 * kTile, &tm_x, &full_bar[stage], (h0 + 1) * kP, blk * kBlk, b);
  };

  float run = 0.f;  // log2-decay of the blocks after the current one, within the segment
  const float Alog = A[h0 + j] * kLog2e;
  if (tid == 0) issue_loads(0, 0);
  bool ok = true;
  for (int i = 0; i < nb; ++i) {
    const int stage = i & 1;
    const int blk = blk0 + nb - 1 - i;
    if (tid == 0 && i + 1 < nb) {
      // the other stage is free once the MMAs of block i-1 have read it
      if (i >= 1) ok = mbar_wait(&mma_bar[stage ^ 1], ((i - 1) >> 1) & 1, abort_v, 11);
      if (ok) issue_loads(i + 1, stage ^ 1);
    }
    // w_t = exp(sum_{k > t, k in segment} a_k) * dt_t
    const int64_t tok = int64_t(blk) * kBlk + row;
    const float d = tok < seqlen ? dt[(int64_t(b) * seqlen + tok) * nheads + h0 + j] : 0.f;
    float tot;
    const float incl = half_scan128(d * Alog, scan_scratch, &tot);
    const float w = ex2(tot - incl + run) * d;
    run += tot;
    ok = ok && mbar_wait(&full_bar[stage], (i >> 1) & 1, abort_v, 12);
    if (ok) {
      uint8_t* xr = smem + stage * kSegStage + (2 + j) * kTile;
      uint8_t* lr = smem + stage * kSegStage + (4 + j) * kTile;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4* ph = reinterpret_cast<uint4*>(xr + swz(row, c));
        const uint4 v = *ph;
        uint4 hi, lo;
        split2(bf16lo(v.x) * w, bf16hi(v.x) * w, hi.x, lo.x);
        split2(bf16lo(v.y) * w, bf16hi(v.y) * w, hi.y, lo.y);
        split2(bf16lo(v.z) * w, bf16hi(v.z) * w, hi.z, lo.z);
        split2(bf16lo(v.w) * w, bf16hi(v.w) * w, hi.w, lo.w);
        *ph = hi;
        *reinterpret_cast<uint4*>(lr + swz(row, c)) = lo;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sb = smem_u32(smem + stage * kSegStage);
      const uint32_t idesc = idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int k = 0; k < kBlk / 16; ++k) {
        const uint64_t ad = sdesc(sb + k * 2048, kTile, 1024);               // B^T: M = n
        mma_ss(tmem, ad, sdesc(sb + 2 * kTile + k * 2048, kTile, 1024), idesc,
               (i > 0 || k > 0) ? 1u : 0u);                                   // X'hi
        mma_ss(tmem, ad, sdesc(sb + 4 * kTile + k * 2048, kTile, 1024), idesc, 1u);  // X'lo
      }
      mma_commit(&mma_bar[stage]);
      ++n_commits[stage];
    }
  }
  if (ok && nb > 0) {
    const int last = nb - 1;
    ok = mbar_wait(&mma_bar[last & 1], (last >> 1) & 1, abort_v, 13);
  }
  if (__syncthreads_or(!ok || *abort_v)) {
    if (tid == 0) {  // let in-flight copies and MMAs land before the CTA leaves
      for (int i = 0; i < 2; ++i) {
        if (n_loads[i]) drain(&full_bar[i], (n_loads[i] - 1) & 1);
        mma_commit(&mma_bar[i]);  // arrives once every earlier MMA is done
        drain(&mma_bar[i], n_commits[i] & 1);
      }
    }
    __syncthreads();
  } else {
    tc_fence_after();
    // epilogue: lane n = row, columns of head j
    const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16) + j * 64;
    float* out = seg_states + (((int64_t(b) * sg.nseg + seg) * nheads + h0 + j) * kP) * kN + row;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      uint32_t r[16];
      tmem_ld16(lane_addr + pc * 16, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) out[(pc * 16 + e) * kN] = nb > 0 ? __uint_as_float(r[e]) : 0.f;
    }
    if (row == 0) seg_decay[(int64_t(b) * sg.nseg + seg) * nheads + h0 + j] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_free(tmem, 128);
}

// =============================================================================================
// seg_scan: one thread per state element; H_in(0) = init, H_in(s+1) = 2^decay(s) H_in(s) + S(s).
// seg_states is overwritten in place with H_in; final_state receives the state after the last
// segment (it may alias init_state: each element is read before it is written, by one thread).
// Segments are processed eight at a time so that eight independent loads are in flight.
// =============================================================================================
__global__ void __launch_bounds__(256) seg_scan_kernel(float* __restrict__ seg_states,
                                                       const float* __restrict__ seg_decay,
                                                       const float* init_state,
                                                       float* final_state, int batch,
                                                       int nheads, int nseg) {
  const int64_t per_bh = int64_t(kP) * kN;
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= int64_t(batch) * nheads * per_bh) return;
  const int64_t bh = e / per_bh, pn = e % per_bh;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  float run = init_state ? init_state[e] : 0.f;
  const int64_t stride = int64_t(nheads) * per_bh;
  float* base = seg_states + (b * nseg * nheads + h) * per_bh + pn;
  const float* dbase = seg_decay + b * nseg * nheads + h;
  for (int s0 = 0; s0 < nseg; s0 += 8) {
    float v[8], dcy[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (s0 + i < nseg) {
        v[i] = base[(s0 + i) * stride];
        dcy[i] = dbase[(s0 + i) * nheads];
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (s0 + i < nseg) {
        base[(s0 + i) * stride] = run;
        run = fmaf(ex2(dcy[i]), run, v[i]);
      }
    }
  }
  if (final_state) final_state[e] = run;
}

// =============================================================================================
// chunk_out: grid = batch * nseg * (nheads / 2), block = 256 threads.  Thread (row = tid % 128,
// half = tid / 128): token row `row` of a block (and state row n = row for the state passes);
// `half` selects the head (state pass, epilogue) or the 64-column half of G (masks).
// Shared memory (1024-aligned, 10 x 16 KB):
//   sC   2 tiles  C, K-major (rows t), n halves
//   sB   2 tiles  B, rows s, n halves: K-major for G = C B^T, MN-major for B^T X'
//   sX   2 tiles  x of the two heads (rows t, 64 p), MN-major; scaled in place to X'
//   sHh  2 tiles  bf16 high part of the entering state of the two heads (rows n, 64 p)
//   sHl  2 tiles  bf16 low part (the state's rounding remainder), same layout
// TMEM (512 columns): [0,128) running state H (head, p) | [128,256) diagonal accumulators |
//   [256,384) off-diagonal accumulators C H | [384,512) G = C B^T, overwritten in place, one
//   head at a time, by that head's masked tile as bf16 high and low parts, which the diagonal
//   MMAs read as their A operand.
// =============================================================================================
constexpr uint32_t kOffC = 0, kOffB = 2 * kTile, kOffX = 4 * kTile, kOffHh = 6 * kTile,
                   kOffHl = 8 * kTile, kSmemTiles = 10 * kTile;

template <typename TY> struct yout;
template <> struct yout<float> {
  static __device__ __forceinline__ void store16(float* p, const float (&v)[16]) {
    float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
};
template <> struct yout<__nv_bfloat16> {
  static __device__ __forceinline__ void store16(__nv_bfloat16* p, const float (&v)[16]) {
    uint4* q = reinterpret_cast<uint4*>(p);
    q[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
    q[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                      pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
  }
};

template <typename TY>
__global__ void __launch_bounds__(256, 1) chunk_out_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const float* __restrict__ dt,
    const float* __restrict__ A, const float* __restrict__ D, const float* __restrict__ h_in,
    TY* __restrict__ y, int64_t seqlen, int nheads, int heads_per_group, Seg sg) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float cs_sh[2][kBlk], dt_sh[2][kBlk], v_sh[2][kBlk];
  __shared__ float scan_scratch[8];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int row = tid & 127, half = tid >> 7;
  const int npair = nheads / 2;
  const int unit = blockIdx.x;
  const int hp = unit % npair;
  const int seg = (unit / npair) % sg.nseg;
  const int b = unit / (npair * sg.nseg);
  const int h0 = hp * 2;
  const int g = h0 / heads_per_group;
  const int blk0 = seg * sg.seg_blks;
  const int nb = min(sg.nblk, blk0 + sg.seg_blks) - blk0;

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&tma_bar, 1);
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_c);
  }
  if (warp == 0) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tH = tmem, tD = tmem + 128, tO = tmem + 256, tG = tmem + 384;
  const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;  // this warp's TMEM lane quarter
  const uint32_t sbase = smem_u32(smem);

  // entering state of the segment -> TMEM (lane n = row, columns of head `half`)
  {
    const float* src =
        h_in + (((int64_t(b) * sg.nseg + seg) * nheads + h0 + half) * kP) * kN + row;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      uint32_t r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(src[(pc * 16 + e) * kN]);
      tmem_st16(tH + lane_off + half * 64 + pc * 16, r);
    }
    tmem_wait_st();
  }
  const float Alog = A[h0 + half] * kLog2e;
  const float Dh = D ? D[h0 + half] : 0.f;
  uint32_t tma_phase = 0, mma_phase = 0;
  bool ok = true;
  volatile int* abort_v = &abort_flag;

  for (int k = 0; k < nb; ++k) {
    const int blk = blk0 + k;
    const int64_t t0 = int64_t(blk) * kBlk;
    tc_fence_before();
    if (__syncthreads_or(*abort_v)) { ok = false; break; }
    if (tid == 0) {
      mbar_arrive_expect_tx(&tma_bar, 6 * kTile);
      tma_load_3d(smem + kOffC, &tm_c, &tma_bar, g * kN, int(t0), b);
      tma_load_3d(smem + kOffC + kTile, &tm_c, &tma_bar, g * kN + 64, int(t0), b);
      tma_load_3d(smem + kOffB, &tm_b, &tma_bar, g * kN, int(t0), b);
      tma_load_3d(smem + kOffB + kTile, &tm_b, &tma_bar, g * kN + 64, int(t0), b);
      tma_load_3d(smem + kOffX, &tm_x, &tma_bar, h0 * kP, int(t0), b);
      tma_load_3d(smem + kOffX + kTile, &tm_x, &tma_bar, (h0 + 1) * kP, int(t0), b);
    }
    // within-block log2 cumsums of head `half`; v_s = exp(cs_r(s) - cs_s) dt_s, r(s) = s | 15
    const int64_t tok = t0 + row;
    {
      const float d = tok < seqlen ? dt[(int64_t(b) * seqlen + tok) * nheads + h0 + half] : 0.f;
      float tot;
      const float c = half_scan128(d * Alog, scan_scratch, &tot);
      cs_sh[half][row] = c;
      dt_sh[half][row] = d;
      __syncthreads();
      v_sh[half][row] = ex2(cs_sh[half][row | 15] - c) * d;
    }
    ok = mbar_wait(&tma_bar, tma_phase, abort_v, 21);
    tma_phase ^= 1;
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }

    // ---- G = C B^T (M = t, N = s, K = n) ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 128, 0, 0);
#pragma unroll
      for (int kk = 0; kk < kN / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * kTile + (kk & 3) * 32;
        mma_ss(tG, sdesc(sbase + kOffC + koff, 16, 1024), sdesc(sbase + kOffB + koff, 16, 1024),
               idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(&mma_bar);
    }
    // ---- H pass (lane n = row, head = half): hi/lo bf16 copy of H for C H, then
    //      H <- exp(cs_end) H in place ----
    {
      tc_fence_after();
      const float al = ex2(cs_sh[half][kBlk - 1]);
      uint8_t* hh = smem + kOffHh + half * kTile;
      uint8_t* hl = smem + kOffHl + half * kTile;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t r[16];
        tmem_ld16(tH + lane_off + half * 64 + pc * 16, r);
        tmem_wait_ld();
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          split2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]), hi[e], lo[e]);
        *reinterpret_cast<uint4*>(hh + swz(row, pc * 2)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(hh + swz(row, pc * 2 + 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        *reinterpret_cast<uint4*>(hl + swz(row, pc * 2)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(hl + swz(row, pc * 2 + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * al);
        tmem_st16(tH + lane_off + half * 64 + pc * 16, r);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    // ---- Off = C (Hhi + Hlo) (M = t, N = (head, p), K = n) ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int kk = 0; kk < kN / 16; ++kk) {
        const uint64_t ad = sdesc(sbase + kOffC + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024);
        mma_ss(tO, ad, sdesc(sbase + kOffHh + kk * 2048, kTile, 1024), idesc, kk > 0 ? 1u : 0u);
        mma_ss(tO, ad, sdesc(sbase + kOffHl + kk * 2048, kTile, 1024), idesc, 1u);
      }
    }
    ok = mbar_wait(&mma_bar, mma_phase, abort_v, 22);  // G complete
    mma_phase ^= 1;
    tc_fence_after();
    // ---- masked tiles, one head at a time: M_h[t, s] = G[t, s] exp(cs_t - cs_s) dt_s for
    //      s <= t.  Thread (row t, column half c) keeps G[t, 64c .. 64c+64) in registers and
    //      writes head h's mask over those TMEM columns as a bf16 high part (columns
    //      64c .. 64c+32) and the bf16 rounding of the remainder (64c+32 .. 64c+64); the
    //      diagonal MMAs read both as their A operand, so the mask carries ~16 bits. ----
    float gv[64];
    const bool g_live = (warp & 3) * 32 + 31 >= half * 64;  // some row of the warp reaches 64c
    if (ok && g_live) {
      const uint32_t gaddr = tG + lane_off + half * 64;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t r[16];
        tmem_ld16(gaddr + q * 16, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) gv[q * 16 + e] = __uint_as_float(r[e]);
      }
      tmem_wait_ld();
    }
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      if (ok) {
        const int t = row, c = half;
        const uint32_t gaddr = tG + lane_off + c * 64;
        uint32_t hi[32], lo[32];
        if (g_live) {
          const float ct = cs_sh[h][t];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int s0 = c * 64 + q * 16;
            float f[16];
            if (t >= s0 + 15) {  // the whole 16-column sub-block is at or before t
              const float u = ex2(ct - cs_sh[h][s0 + 15]);
#pragma unroll
              for (int e = 0; e < 16; ++e) f[e] = gv[q * 16 + e] * (u * v_sh[h][s0 + e]);
            } else if (t >= s0) {  // diagonal sub-block: exact exps, zero above the diagonal
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int s = s0 + e;
                f[e] = s <= t ? gv[q * 16 + e] * ex2(ct - cs_sh[h][s]) * dt_sh[h][s] : 0.f;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) f[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) split2(f[2 * e], f[2 * e + 1], hi[q * 8 + e], lo[q * 8 + e]);
          }
        } else {  // every row of this warp lies before column 64c: zero masks
#pragma unroll
          for (int e = 0; e < 32; ++e) { hi[e] = 0u; lo[e] = 0u; }
        }
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = hi[e];
        tmem_st16(gaddr, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = hi[16 + e];
        tmem_st16(gaddr + 16, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = lo[e];
        tmem_st16(gaddr + 32, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = lo[16 + e];
        tmem_st16(gaddr + 48, r);
        tmem_wait_st();
      }
      tc_fence_before();
      if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
      // ---- Diag_h = (Mhi_h + Mlo_h) X_h (M = t, N = p, K = s), A from TMEM ----
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint32_t acol = tG + (kk >> 2) * 64 + (kk & 3) * 8;
          const uint64_t bd = sdesc(sbase + kOffX + h * kTile + kk * 2048, kTile, 1024);
          mma_ts(tD + h * 64, acol, bd, idesc, kk > 0 ? 1u : 0u);
          mma_ts(tD + h * 64, acol + 32, bd, idesc, 1u);
        }
        mma_commit(&mma_bar);  // head 0: covers Off as well
      }
      ok = mbar_wait(&mma_bar, mma_phase, abort_v, 23);
      mma_phase ^= 1;
      tc_fence_after();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
    tc_fence_after();
    // ---- epilogue (row t, head = half): y_t = Diag + exp(cs_t) Off + D x_t; then X' = w x ----
    if (ok) {
      const int t = row, j = half;
      const float ej = ex2(cs_sh[j][t]);
      const float wj = ex2(cs_sh[j][kBlk - 1] - cs_sh[j][t]) * dt_sh[j][t];
      uint8_t* xrow = smem + kOffX + j * kTile;
      TY* yrow = y + ((int64_t(b) * seqlen + tok) * nheads + h0 + j) * kP;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t rd[16], ro[16];
        tmem_ld16(tD + lane_off + j * 64 + pc * 16, rd);
        tmem_ld16(tO + lane_off + j * 64 + pc * 16, ro);
        tmem_wait_ld();
        uint4* x0p = reinterpret_cast<uint4*>(xrow + swz(t, pc * 2));
        uint4* x1p = reinterpret_cast<uint4*>(xrow + swz(t, pc * 2 + 1));
        const uint4 xa = *x0p, xb = *x1p;
        const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        float yv[16];
        uint32_t xs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xl = bf16lo(xw[e]), xh = bf16hi(xw[e]);
          yv[2 * e] = __uint_as_float(rd[2 * e]) + ej * __uint_as_float(ro[2 * e]) + Dh * xl;
          yv[2 * e + 1] =
              __uint_as_float(rd[2 * e + 1]) + ej * __uint_as_float(ro[2 * e + 1]) + Dh * xh;
          xs[e] = pack_bf16x2(xl * wj, xh * wj);
        }
        if (tok < seqlen) yout<TY>::store16(yrow + pc * 16, yv);
        *x0p = make_uint4(xs[0], xs[1], xs[2], xs[3]);
        *x1p = make_uint4(xs[4], xs[5], xs[6], xs[7]);
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
    // ---- H += B^T X' (M = n, N = (head, p), K = t) ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk)
        mma_ss(tH, sdesc(sbase + kOffB + kk * 2048, kTile, 1024),
               sdesc(sbase + kOffX + kk * 2048, kTile, 1024), idesc, 1u);
      mma_commit(&mma_bar);
    }
    ok = mbar_wait(&mma_bar, mma_phase, abort_v, 24);
    mma_phase ^= 1;
    tc_fence_after();
  }
  if (__syncthreads_or(!ok || *abort_v)) {
    if (tid == 0) {  // let an in-flight copy and every issued MMA land before leaving
      drain(&tma_bar, tma_phase ^ 1);
      mma_commit(&mma_bar);
      drain(&mma_bar, mma_phase);
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_free(tmem, 512);
}

}  // namespace tc
}  // namespace ssd
