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

// 128-thread inclusive scan; returns the prefix and writes the block total to *total.
__device__ __forceinline__ float block_scan128(float v, float* scratch4, float* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_inclusive_scan(v);
  if (lane == 31) scratch4[warp] = v;
  __syncthreads();
  float off = 0.f, tot = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float s = scratch4[w];
    off += (w < warp) ? s : 0.f;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return v + off;
}

// Wait until every outstanding async op a CTA started has finished (bounded, used only on
// the abort path so that no copy or MMA is still writing when the CTA leaves).
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_test(bar, parity)) {
    if (globaltimer() - t0 > 200000000ull) break;
  }
}

// =============================================================================================
// seg_state: grid = batch * nseg * (nheads / HQ), block = 128 threads.
// Shared memory per stage: B tile (2 x 16 KB, n halves), x tiles (HQ x 16 KB) -- two stages.
// TMEM: 64*HQ columns, lane n / column (h, p) = S_seg[n, (h, p)].
// =============================================================================================
template <int HQ>
__global__ void __launch_bounds__(128, 1) seg_state_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const float* __restrict__ dt, const float* __restrict__ A, float* __restrict__ seg_states,
    float* __restrict__ seg_decay, int64_t seqlen, int nheads, int heads_per_group, Seg sg) {
  constexpr uint32_t kStage = 2 * kTile + HQ * kTile;
  constexpr uint32_t kCols = (64 * HQ < 32) ? 32 : 64 * HQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full_bar[2], mma_bar[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ float scan_scratch[4];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int nq = nheads / HQ;
  const int unit = blockIdx.x;
  const int q = unit % nq;
  const int seg = (unit / nq) % sg.nseg;
  const int b = unit / (nq * sg.nseg);
  const int h0 = q * HQ;
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
  if (tid < 32) tmem_alloc(&tmem_base_sh, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  volatile int* abort_v = &abort_flag;
  uint32_t n_loads[2] = {0, 0}, n_commits[2] = {0, 0};  // thread 0's issue counts per stage
  auto issue_loads = [&](int i, int stage) {  // block i of the walk (reverse order)
    const int blk = blk0 + nb - 1 - i;
    uint8_t* st = smem + stage * kStage;
    ++n_loads[stage];
    mbar_arrive_expect_tx(&full_bar[stage], kStage);
    tma_load_3d(st, &tm_b, &full_bar[stage], g * kN, blk * kBlk, b);
    tma_load_3d(st + kTile, &tm_b, &full_bar[stage], g * kN + 64, blk * kBlk, b);
    for (int j = 0; j < HQ; ++j)
      tma_load_3d(st + (2 + j) * kTile, &tm_x, &full_bar[stage], (h0 + j) * kP, blk * kBlk, b);
  };

  float run[HQ];  // log2-decay of the blocks after the current one, within the segment
#pragma unroll
  for (int j = 0; j < HQ; ++j) run[j] = 0.f;
  float Alog[HQ];
#pragma unroll
  for (int j = 0; j < HQ; ++j) Alog[j] = A[h0 + j] * kLog2e;

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
    // suffix sums within the block: w_t = exp(sum_{k>t, k in segment} a_k) * dt_t
    const int64_t tok = int64_t(blk) * kBlk + tid;
    float w[HQ];
#pragma unroll
    for (int j = 0; j < HQ; ++j) {
      const float d = tok < seqlen ? dt[(int64_t(b) * seqlen + tok) * nheads + h0 + j] : 0.f;
      const float a = d * Alog[j];
      float tot;
      const float incl = block_scan128(a, scan_scratch, &tot);
      w[j] = ex2(tot - incl + run[j]) * d;  // tot - incl = sum over k > t in this block
      run[j] += tot;
    }
    ok = ok && mbar_wait(&full_bar[stage], (i >> 1) & 1, abort_v, 12);
    if (ok) {
      // scale row `tid` of each x tile in place: X' = w * x
      uint8_t* st = smem + stage * kStage;
#pragma unroll
      for (int j = 0; j < HQ; ++j) {
        uint8_t* row = st + (2 + j) * kTile;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* pch = reinterpret_cast<uint4*>(row + swz(tid, c));
          uint4 v = *pch;
          v.x = pack_bf16x2(bf16lo(v.x) * w[j], bf16hi(v.x) * w[j]);
          v.y = pack_bf16x2(bf16lo(v.y) * w[j], bf16hi(v.y) * w[j]);
          v.z = pack_bf16x2(bf16lo(v.z) * w[j], bf16hi(v.z) * w[j]);
          v.w = pack_bf16x2(bf16lo(v.w) * w[j], bf16hi(v.w) * w[j]);
          *pch = v;
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sb = smem_u32(smem + stage * kStage);
      const uint32_t idesc = idesc_bf16(128, 64 * HQ, 1, 1);
#pragma unroll
      for (int k = 0; k < kBlk / 16; ++k) {
        const uint64_t ad = sdesc(sb + k * 2048, kTile, 1024);          // B^T: M = n
        const uint64_t bd = sdesc(sb + 2 * kTile + k * 2048, kTile, 1024);  // X': N = (h,p)
        mma_ss(tmem, ad, bd, idesc, (i > 0 || k > 0) ? 1u : 0u);
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
    // epilogue: lane n = tid, column (j, p)
    const int n = tid;
    const uint32_t lane_addr = tmem + (uint32_t(tid & ~31) << 16);
#pragma unroll
    for (int j = 0; j < HQ; ++j) {
      float* out = seg_states +
                   (((int64_t(b) * sg.nseg + seg) * nheads + h0 + j) * kP) * kN + n;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t r[16];
        tmem_ld16(lane_addr + j * 64 + pc * 16, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) out[(pc * 16 + e) * kN] = nb > 0 ? __uint_as_float(r[e]) : 0.f;
      }
    }
    if (tid < HQ) {
      float v = 0.f;
#pragma unroll
      for (int j = 0; j < HQ; ++j) v = (tid == j) ? run[j] : v;
      seg_decay[(int64_t(b) * sg.nseg + seg) * nheads + h0 + tid] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid < 32) tmem_free(tmem, kCols);
}

// =============================================================================================
// seg_scan: one thread per state element; H_in(0) = init, H_in(s+1) = 2^decay(s) H_in(s) + S(s).
// seg_states is overwritten in place with H_in; final_state receives the state after the last
// segment (it may alias init_state: each element is read before it is written, by one thread).
// =============================================================================================
__global__ void seg_scan_kernel(float* __restrict__ seg_states,
                                const float* __restrict__ seg_decay, const float* init_state,
                                float* final_state, int batch, int nheads, int nseg) {
  const int64_t per_bh = int64_t(kP) * kN;
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= int64_t(batch) * nheads * per_bh) return;
  const int64_t bh = e / per_bh, pn = e % per_bh;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  float run = init_state ? init_state[e] : 0.f;
  for (int s = 0; s < nseg; ++s) {
    float* slot = seg_states + ((b * nseg + s) * nheads + h) * per_bh + pn;
    const float v = *slot;
    *slot = run;
    run = fmaf(ex2(seg_decay[(b * nseg + s) * nheads + h]), run, v);
  }
  if (final_state) final_state[e] = run;
}

// =============================================================================================
// chunk_out: grid = batch * nseg * (nheads / 2), block = 128 threads (thread t <-> token row t
// of a block, and <-> state row n for the state passes).  Shared memory (1024-aligned):
//   sC  2 x 16 KB   C tile, K-major (rows t), n halves
//   sB  2 x 16 KB   B tile, rows s, n halves: K-major for G = C B^T, MN-major for B^T X'
//   sX  2 x 16 KB   x tiles of the two heads (rows t, 64 p): MN-major; scaled in place to X'
//   sM  2 x 32 KB   masked tiles of the two heads, K-major (rows t, s halves)
//   sH  2 x 16 KB   bf16 copy of the entering state of the two heads (rows n, 64 p): MN-major
// TMEM (512 columns): [0,128) running state H (head, p) | [128,256) diagonal accumulators |
//                     [256,384) off-diagonal accumulators C H | [384,512) G = C B^T.
// =============================================================================================
constexpr uint32_t kOffC = 0, kOffB = 2 * kTile, kOffX = 4 * kTile, kOffM = 6 * kTile,
                   kOffH = 10 * kTile, kSmemTiles = 12 * kTile;

__global__ void __launch_bounds__(128, 1) chunk_out_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const float* __restrict__ dt,
    const float* __restrict__ A, const float* __restrict__ D, const float* __restrict__ h_in,
    __nv_bfloat16* __restrict__ y, int64_t seqlen, int nheads, int heads_per_group, Seg sg) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float cs_sh[2][kBlk], dt_sh[2][kBlk], v_sh[2][kBlk];
  __shared__ float scan_scratch[4];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
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
  if (tid < 32) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tH = tmem, tD = tmem + 128, tO = tmem + 256, tG = tmem + 384;
  const uint32_t lane_off = uint32_t(warp * 32) << 16;  // this warp's TMEM lane quarter
  const uint32_t sbase = smem_u32(smem);

  // entering state of the segment -> TMEM (lane n = tid, column (head, p))
  {
    const int n = tid;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float* src = h_in + (((int64_t(b) * sg.nseg + seg) * nheads + h0 + j) * kP) * kN + n;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(src[(pc * 16 + e) * kN]);
        tmem_st16(tH + lane_off + j * 64 + pc * 16, r);
      }
    }
    tmem_wait_st();
  }
  const float Alog0 = A[h0] * kLog2e, Alog1 = A[h0 + 1] * kLog2e;
  const float Dh0 = D ? D[h0] : 0.f, Dh1 = D ? D[h0 + 1] : 0.f;
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
    // within-block log2 cumsums, per head; v_s = exp(cs_r(s) - cs_s) dt_s, r(s) = s | 15
    const int64_t tok = t0 + tid;
    {
      const float d0 = tok < seqlen ? dt[(int64_t(b) * seqlen + tok) * nheads + h0] : 0.f;
      const float d1 = tok < seqlen ? dt[(int64_t(b) * seqlen + tok) * nheads + h0 + 1] : 0.f;
      float tot;
      const float c0 = block_scan128(d0 * Alog0, scan_scratch, &tot);
      const float c1 = block_scan128(d1 * Alog1, scan_scratch, &tot);
      cs_sh[0][tid] = c0; cs_sh[1][tid] = c1;
      dt_sh[0][tid] = d0; dt_sh[1][tid] = d1;
      __syncthreads();
      const int r = tid | 15;
      v_sh[0][tid] = ex2(cs_sh[0][r] - c0) * d0;
      v_sh[1][tid] = ex2(cs_sh[1][r] - c1) * d1;
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
    // ---- H pass: bf16 copy of H for C H, then H <- exp(cs_end) H (lane n = tid) ----
    {
      tc_fence_after();
      const float al0 = ex2(cs_sh[0][kBlk - 1]), al1 = ex2(cs_sh[1][kBlk - 1]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float al = j ? al1 : al0;
        uint8_t* hrow = smem + kOffH + j * kTile;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          uint32_t r[16];
          tmem_ld16(tH + lane_off + j * 64 + pc * 16, r);
          tmem_wait_ld();
          uint4 lo, hi;
          lo.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
          lo.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
          lo.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
          lo.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
          hi.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
          hi.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
          hi.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
          hi.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
          *reinterpret_cast<uint4*>(hrow + swz(tid, pc * 2)) = lo;
          *reinterpret_cast<uint4*>(hrow + swz(tid, pc * 2 + 1)) = hi;
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * al);
          tmem_st16(tH + lane_off + j * 64 + pc * 16, r);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    // ---- Off = C H (M = t, N = (head, p), K = n) ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int kk = 0; kk < kN / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * kTile + (kk & 3) * 32;
        mma_ss(tO, sdesc(sbase + kOffC + koff, 16, 1024),
               sdesc(sbase + kOffH + kk * 2048, kTile, 1024), idesc, kk > 0 ? 1u : 0u);
      }
    }
    ok = mbar_wait(&mma_bar, mma_phase, abort_v, 22);  // G complete
    mma_phase ^= 1;
    tc_fence_after();
    // ---- masked tiles: M_h[t, s] = G[t, s] exp(cs_t - cs_s) dt_s  (s <= t), row t = tid ----
    if (ok) {
      const int t = tid;
      const int jmax = 2 * warp + 1;  // last 16-column block any row of this warp needs
      const float cst0 = cs_sh[0][t], cst1 = cs_sh[1][t];
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        const uint32_t region = (j >> 2) * kTile, c0 = (j & 3) * 2;
        uint4 m0lo = make_uint4(0, 0, 0, 0), m0hi = m0lo, m1lo = m0lo, m1hi = m0lo;
        if (j <= jmax) {
          uint32_t r[16];
          tmem_ld16(tG + lane_off + j * 16, r);
          tmem_wait_ld();
          const int s0 = j * 16;
          float f0[16], f1[16];
          if (t >= s0 + 15) {  // whole sub-block at or before t: split at r = s0 + 15
            const float u0 = ex2(cst0 - cs_sh[0][s0 + 15]);
            const float u1 = ex2(cst1 - cs_sh[1][s0 + 15]);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float gv = __uint_as_float(r[e]);
              f0[e] = gv * (u0 * v_sh[0][s0 + e]);
              f1[e] = gv * (u1 * v_sh[1][s0 + e]);
            }
          } else {  // diagonal sub-block (or beyond): exact exps, zero above the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int s = s0 + e;
              const float gv = __uint_as_float(r[e]);
              f0[e] = s <= t ? gv * ex2(cst0 - cs_sh[0][s]) * dt_sh[0][s] : 0.f;
              f1[e] = s <= t ? gv * ex2(cst1 - cs_sh[1][s]) * dt_sh[1][s] : 0.f;
            }
          }
          m0lo = make_uint4(pack_bf16x2(f0[0], f0[1]), pack_bf16x2(f0[2], f0[3]),
                            pack_bf16x2(f0[4], f0[5]), pack_bf16x2(f0[6], f0[7]));
          m0hi = make_uint4(pack_bf16x2(f0[8], f0[9]), pack_bf16x2(f0[10], f0[11]),
                            pack_bf16x2(f0[12], f0[13]), pack_bf16x2(f0[14], f0[15]));
          m1lo = make_uint4(pack_bf16x2(f1[0], f1[1]), pack_bf16x2(f1[2], f1[3]),
                            pack_bf16x2(f1[4], f1[5]), pack_bf16x2(f1[6], f1[7]));
          m1hi = make_uint4(pack_bf16x2(f1[8], f1[9]), pack_bf16x2(f1[10], f1[11]),
                            pack_bf16x2(f1[12], f1[13]), pack_bf16x2(f1[14], f1[15]));
        }
        uint8_t* m0 = smem + kOffM + region;
        uint8_t* m1 = smem + kOffM + 2 * kTile + region;
        *reinterpret_cast<uint4*>(m0 + swz(t, c0)) = m0lo;
        *reinterpret_cast<uint4*>(m0 + swz(t, c0 + 1)) = m0hi;
        *reinterpret_cast<uint4*>(m1 + swz(t, c0)) = m1lo;
        *reinterpret_cast<uint4*>(m1 + swz(t, c0 + 1)) = m1hi;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || *abort_v)) { ok = false; break; }
    // ---- Diag_h = M_h X_h (M = t, N = p, K = s) ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 64, 0, 1);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kTile + (kk & 3) * 32;
          mma_ss(tD + j * 64, sdesc(sbase + kOffM + j * 2 * kTile + koff, 16, 1024),
                 sdesc(sbase + kOffX + j * kTile + kk * 2048, kTile, 1024), idesc,
                 kk > 0 ? 1u : 0u);
        }
      }
      mma_commit(&mma_bar);  // covers Off and both Diag
    }
    ok = mbar_wait(&mma_bar, mma_phase, abort_v, 23);
    mma_phase ^= 1;
    tc_fence_after();
    // ---- epilogue: y_t = Diag + exp(cs_t) Off + D x_t; then X' = w * x in place ----
    if (ok) {
      const int t = tid;
      const float e0 = ex2(cs_sh[0][t]), e1 = ex2(cs_sh[1][t]);
      const float w0 = ex2(cs_sh[0][kBlk - 1] - cs_sh[0][t]) * dt_sh[0][t];
      const float w1 = ex2(cs_sh[1][kBlk - 1] - cs_sh[1][t]) * dt_sh[1][t];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float ej = j ? e1 : e0, Dj = j ? Dh1 : Dh0, wj = j ? w1 : w0;
        uint8_t* xrow = smem + kOffX + j * kTile;
        __nv_bfloat16* yrow = y + ((int64_t(b) * seqlen + tok) * nheads + h0 + j) * kP;
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
          uint32_t yo[8], xs[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float xl = bf16lo(xw[e]), xh = bf16hi(xw[e]);
            const float yl = __uint_as_float(rd[2 * e]) + ej * __uint_as_float(ro[2 * e]) + Dj * xl;
            const float yh =
                __uint_as_float(rd[2 * e + 1]) + ej * __uint_as_float(ro[2 * e + 1]) + Dj * xh;
            yo[e] = pack_bf16x2(yl, yh);
            xs[e] = pack_bf16x2(xl * wj, xh * wj);
          }
          if (tok < seqlen) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + pc * 16);
            dst[0] = make_uint4(yo[0], yo[1], yo[2], yo[3]);
            dst[1] = make_uint4(yo[4], yo[5], yo[6], yo[7]);
          }
          *x0p = make_uint4(xs[0], xs[1], xs[2], xs[3]);
          *x1p = make_uint4(xs[4], xs[5], xs[6], xs[7]);
        }
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
  if (tid < 32) tmem_free(tmem, 512);
}

}  // namespace tc
}  // namespace ssd
