// tc_kernels.cuh -- the chunked scan on sm_100a tensor cores (bf16 io, headdim 64, dstate 128).
//
// The sequence of each (batch row, head pair) is cut into 128-token blocks (the tcgen05 M=128
// tile).  The output pass, scan_walk, walks blocks in order with the running state resident in
// TMEM.  Per block: G = C B^T (once for both heads), masked diagonal tile (L o G o dt) X,
// off-diagonal C H, skip term D x, y store, then H <- exp(cs_end) H + B^T (w*x) in place.
//
// The walk's work is cut into equal ranges of blocks, one per CTA.  Unless a sequence is much
// longer than every CTA's share of all blocks, a range starting inside a sequence gets its
// entering state from the CTA that walked the sequence's head (published through L2), and
// nothing else runs.  With few, long sequences each is cut into segments first:
//
//  seg_state   per (b, segment, head pair): S_seg = sum_{t in seg} exp(sum_{k>t in seg} a_k)
//              dt_t B_t x_t^T, one long-K GEMM on the tensor cores (A = B^T, B = w*x, K =
//              tokens), plus the segment's total log-decay.  Persistent.
//  seg_pass    per state element: passes the state along the segments: H_in(seg) = state
//              entering each segment.
//  scan_walk   as above, with the segments' entering states from seg_pass.
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
  int nseg;      // segments per sequence (stride of the per-segment state and decay arrays)
  int useg;      // leading segments per sequence that seg_state summarises (<= nseg)
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
  const float2 r = sub2(make_float2(a, b), make_float2(bf16lo(hi), bf16hi(hi)));
  lo = pack_bf16x2(r.x, r.y);
}
// a bf16 pair scaled by w, rounded back to a bf16 pair
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float2 ww) {
  const float2 r = mul2(make_float2(bf16lo(v), bf16hi(v)), ww);
  return pack_bf16x2(r.x, r.y);
}

// =============================================================================================
// seg_state (persistent): grid = min(units, SMs), units = batch * nseg * (nheads / HU) taken in
// turn (u = blockIdx.x, + gridDim.x, ...), HU heads per unit (the library launches HU = 2; HU = 4,
// one B tile for four heads, measured slower at the 2.7B shape).  The rings below run across
// units, so the next unit's loads and MMAs start while the current unit's state is read out.
// HU * 128 + 96 threads:
//   compute    warps 0 .. 4 HU - 1: thread (row = tid % 128, j = tid / 128) scales token row
//              `row` of head j's x tile to X' = w x (for a unit's first walk block also the bf16
//              remainder), and at a unit's end writes the state from TMEM to the workspace.
//   then       TMA producer (lane 0);  MMA issuer (lane 0);  weights: takes each block's dt,
//              writes w_t into a four-slot ring, and each unit's total log2-decay to the
//              workspace.  When nheads % 4 == 0 (and dt is 16-byte aligned) dt arrives with the
//              stage as a TMA box {4 heads, 128 tokens}; otherwise (HU = 2 only) the warp loads
//              it itself, four blocks ahead.
// Stage ring (3 stages of 64 KB for HU = 2, 2 stages of 96 KB for HU = 4):  B tile (2 x 16 KB,
// n halves) | x of the HU heads, scaled in place to X'.  Blocks are numbered g = 0, 1, ... over
// the CTA's units, stage g % S.  Within a unit blocks are walked last to first so that the
// suffix sums of the log-decays are running totals.  A unit's first walk block (the segment's
// last block, which dominates a fast-decaying state) sends both X' parts through the tensor
// core, so those tokens carry ~16 bits of X'; earlier blocks reach the state through at least
// one block's decay and send the high part only.  Its low part goes to the x area of stage
// (g + S - 1) % S: written once block g - 1's MMAs (the previous occupant) are done, and block
// g + S - 1 is loaded there only after block g's MMAs.
// TMEM: 2 x HU*64 columns (unit n in buffer n % 2), lane n / column (j, p) = S_seg[n, (j, p)].
// =============================================================================================
template <int HU>
struct SegCfg {
  static constexpr int kStages = HU == 2 ? 3 : 2;
  static constexpr uint32_t kStage = (2 + HU) * kTile;
  static constexpr uint32_t kDtOff = kStages * kStage;  // dt boxes: [stage][128 tokens][4 heads]
  static constexpr uint32_t kDtBox = kBlk * 4 * 4;
  static constexpr uint32_t kSmem = kStages * (kStage + kDtBox) + 1024;
  static constexpr int kCompute = HU * 128;
  static constexpr int kThreads = kCompute + 96;
  static constexpr uint32_t kAccCols = HU * 64;
};
constexpr int kWtSlots = 4;

// unit u -> (b, seg, head group of HU heads)
struct SegUnit {
  int b, seg, hq, blk0, nb;
};
__device__ __forceinline__ SegUnit seg_unit(int u, int nq, const Seg& sg) {
  SegUnit r;
  r.hq = u % nq;
  r.seg = (u / nq) % sg.useg;
  r.b = u / (nq * sg.useg);
  r.blk0 = r.seg * sg.seg_blks;
  r.nb = min(sg.nblk, r.blk0 + sg.seg_blks) - r.blk0;
  return r;
}

template <int HU>
__global__ void __launch_bounds__(SegCfg<HU>::kThreads, 1) seg_state_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_dt, int dt_tma, const float* __restrict__ dt,
    const float* __restrict__ A, float* __restrict__ seg_states, float* __restrict__ seg_decay,
    int64_t seqlen, int nheads, int heads_per_group, Seg sg, int units) {
  using Cfg = SegCfg<HU>;
  constexpr int S = Cfg::kStages;
  constexpr int kProd = Cfg::kCompute / 32, kMma = kProd + 1, kWts = kProd + 2;  // warp roles
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full_bar[S], ready_bar[S], empty_bar[S];
  __shared__ uint64_t wt_full[kWtSlots], wt_empty[kWtSlots];
  __shared__ uint64_t acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(16) float wt_stage[kWtSlots][HU][kBlk];  // [block % 4][head][row]
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nq = nheads / HU;
  volatile int* abort_v = &abort_flag;
  uint32_t n_loads[S];  // the producer's loads per stage
#pragma unroll
  for (int i = 0; i < S; ++i) n_loads[i] = 0;

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&ready_bar[i], Cfg::kCompute);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < kWtSlots; ++i) {
      mbar_init(&wt_full[i], 32);
      mbar_init(&wt_empty[i], Cfg::kCompute);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], Cfg::kCompute);
    }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base_sh, 2 * Cfg::kAccCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProd) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_b);
      if (dt_tma) prefetch_tmap(&tm_dt);
      int g = 0;
      int g_first = -1;  // block number of the current unit's first walk block
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const SegUnit su = seg_unit(u, nq, sg);
        const int h0 = su.hq * HU;
        const int gh = h0 / heads_per_group;
        for (int i = 0; i < su.nb; ++i, ++g) {  // walk block i = block blk0 + nb - 1 - i
          const int stage = g % S;
          if (i == 0) g_first = g;
          if (g >= S && !mbar_wait(&empty_bar[stage], ((g - S) / S) & 1, abort_v, 11)) {
            ok = false;
            break;
          }
          // this stage's x area held the low part of block g - (S - 1) when that was a first
          if (g - (S - 1) == g_first && i >= S - 1 &&
              !mbar_wait(&empty_bar[(g - (S - 1)) % S], ((g - (S - 1)) / S) & 1, abort_v, 17)) {
            ok = false;
            break;
          }
          const int t0 = (su.blk0 + su.nb - 1 - i) * kBlk;
          uint8_t* st = smem + stage * Cfg::kStage;
          ++n_loads[stage];
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStage + (dt_tma ? Cfg::kDtBox : 0u));
          if (dt_tma)
            tma_load_3d(smem + Cfg::kDtOff + stage * Cfg::kDtBox, &tm_dt, &full_bar[stage],
                        h0 & ~3, t0, su.b);
          tma_load_3d(st, &tm_b, &full_bar[stage], gh * kN, t0, su.b);
          tma_load_3d(st + kTile, &tm_b, &full_bar[stage], gh * kN + 64, t0, su.b);
#pragma unroll
          for (int hh = 0; hh < HU; ++hh)
            tma_load_3d(st + (2 + hh) * kTile, &tm_x, &full_bar[stage], (h0 + hh) * kP, t0, su.b);
        }
        // a unit shorter than S blocks: block g_first + S - 1 is not in this unit, so wait for
        // the low part's MMA before any later load reuses its stage
        if (ok && su.nb < S && g_first >= 0 &&
            !mbar_wait(&empty_bar[g_first % S], (g_first / S) & 1, abort_v, 18))
          ok = false;
      }
    }
  } else if (warp == kMma) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, HU * 64, 1, 1);
      // descriptors are built once; a K step or a tile offset adds (bytes >> 4) to the start
      // address field (every address stays below 256 KB, so the field cannot carry)
      const uint64_t d0 = sdesc(smem_u32(smem), kTile, 1024);
      int g = 0, n = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++n) {
        const SegUnit su = seg_unit(u, nq, sg);
        const int ab = n & 1;
        const uint32_t acc = tmem + ab * Cfg::kAccCols;
        if (n >= 2 && !mbar_wait(&acc_empty[ab], ((n - 2) >> 1) & 1, abort_v, 19)) break;
        for (int i = 0; i < su.nb; ++i, ++g) {
          const int stage = g % S;
          if (!mbar_wait(&ready_bar[stage], (g / S) & 1, abort_v, 12)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ds = d0 + uint64_t(stage) * (Cfg::kStage >> 4);
          // low part of a first walk block: stage (g + S - 1) % S's x area
          const uint64_t dlo =
              d0 + uint64_t((g + S - 1) % S) * (Cfg::kStage >> 4) + ((2 * kTile) >> 4);
#pragma unroll
          for (int k = 0; k < kBlk / 16; ++k) {
            const uint64_t ad = ds + k * 128;                                   // B^T: M = n
            mma_ss(acc, ad, ad + ((2 * kTile) >> 4), idesc, (i > 0 || k > 0) ? 1u : 0u);  // X'
            if (i == 0) mma_ss(acc, ad, dlo + k * 128, idesc, 1u);            // X' low part
          }
          mma_commit(&empty_bar[stage]);
          if (i == su.nb - 1) mma_commit(&acc_full[ab]);
        }
      }
    }
  } else if (warp == kWts) {
    // ------------------------------ weights ------------------------------
    // w_t = exp(sum_{k > t, k in segment} a_k) dt_t, a_k = dt_k A log2(e) (log2 units); the
    // walk goes from the segment's last block to its first, so `run` (the blocks after the
    // current one) is a running total.  Blocks are numbered across units like the stages.
    // Without the dt box (HU = 2 only) lane l loads its rows itself, four blocks ahead.
    float v[kWtSlots][8];  // dt of block g in v[g % 4]: rows 4 lane + r, head h at [2r + h]
    int lu = blockIdx.x, li = 0;  // the (unit, walk block) of the next load
    auto load_next = [&](float (&w)[8]) {
      bool valid = lu < units;
      SegUnit su;
      if (valid) su = seg_unit(lu, nq, sg);
      const float* dtb = dt + (valid ? (int64_t(su.b) * seqlen * nheads + su.hq * HU) : 0);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t tok = valid ? int64_t(su.blk0 + su.nb - 1 - li) * kBlk + 4 * lane + r : 0;
        const bool in = valid && tok < seqlen;
        w[2 * r] = in ? dtb[tok * nheads] : 0.f;
        w[2 * r + 1] = in ? dtb[tok * nheads + 1] : 0.f;
      }
      if (valid && ++li == su.nb) {
        li = 0;
        lu += gridDim.x;
      }
    };
    if (!dt_tma) {
#pragma unroll
      for (int s = 0; s < kWtSlots; ++s) load_next(v[s]);
    }
    int g = 0;
    bool wok = true;
    for (int u = blockIdx.x; u < units && wok; u += gridDim.x) {
      const SegUnit su = seg_unit(u, nq, sg);
      const int h0 = su.hq * HU;
      float al[HU], run[HU];
#pragma unroll
      for (int h = 0; h < HU; ++h) {
        al[h] = A[h0 + h] * kLog2e;
        run[h] = 0.f;
      }
      for (int i = 0; i < su.nb && wok; ++i, ++g) {
        const int slot = g % kWtSlots;
        // (warp-uniform decisions: every lane reaches the same __syncwarp)
        if (g >= kWtSlots &&
            !__all_sync(0xffffffffu,
                        mbar_wait(&wt_empty[slot], ((g / kWtSlots) - 1) & 1, abort_v, 15))) {
          wok = false;
          break;
        }
        float d[4][HU];  // rows 4 lane + r, heads h
        if (dt_tma) {  // the stage's box: [128 tokens][4 heads from h0 & ~3]
          const int stage = g % S;
          if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], (g / S) & 1, abort_v, 21))) {
            wok = false;
            break;
          }
          const float* box =
              reinterpret_cast<const float*>(smem + Cfg::kDtOff + stage * Cfg::kDtBox);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            if (HU == 4) {
              const float4 dd = *reinterpret_cast<const float4*>(box + (4 * lane + r) * 4);
              d[r][0] = dd.x;
              d[r][HU > 1 ? 1 : 0] = dd.y;
              d[r][HU > 2 ? 2 : 0] = dd.z;
              d[r][HU > 3 ? 3 : 0] = dd.w;
            } else {
              const float2 dd =
                  *reinterpret_cast<const float2*>(box + (4 * lane + r) * 4 + (h0 & 3));
              d[r][0] = dd.x;
              d[r][HU > 1 ? 1 : 0] = dd.y;
            }
          }
        } else {
#pragma unroll
          for (int s = 0; s < kWtSlots; ++s)
            if (s == slot) {
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                d[r][0] = v[s][2 * r];
                d[r][HU > 1 ? 1 : 0] = v[s][2 * r + 1];
              }
            }
        }
#pragma unroll
        for (int h = 0; h < HU; ++h) {
          const float c0 = d[0][h] * al[h];
          const float c1 = fmaf(d[1][h], al[h], c0);
          const float c2 = fmaf(d[2][h], al[h], c1);
          const float c3 = fmaf(d[3][h], al[h], c2);
          const float incl = warp_inclusive_scan(c3);
          const float off = incl - c3;
          const float tot = __shfl_sync(0xffffffffu, incl, 31);
          const float rest = tot - off + run[h];  // minus the prefix through row 4 lane - 1
          *reinterpret_cast<float4*>(&wt_stage[slot][h][4 * lane]) =
              make_float4(ex2(rest - c0) * d[0][h], ex2(rest - c1) * d[1][h],
                          ex2(rest - c2) * d[2][h], ex2(rest - c3) * d[3][h]);
          run[h] += tot;
        }
        mbar_arrive_warp(&wt_full[slot]);
        if (!dt_tma) {
#pragma unroll
          for (int s = 0; s < kWtSlots; ++s)
            if (s == slot) load_next(v[s]);  // in flight while the next blocks are processed
        }
      }
      if (wok && lane < HU)
        seg_decay[(int64_t(su.b) * sg.nseg + su.seg) * nheads + h0 + lane] = run[lane];
    }
  } else if (warp < kProd) {
    // ------------------------------ compute warps ------------------------------
    const int row = tid & 127, j = tid >> 7;
    bool ok = true;
    int g = 0, n = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++n) {
      const SegUnit su = seg_unit(u, nq, sg);
      for (int i = 0; i < su.nb; ++i, ++g) {
        const int stage = g % S;
        const int slot = g % kWtSlots;
        ok = ok && mbar_wait(&wt_full[slot], (g / kWtSlots) & 1, abort_v, 16);
        const float wt = wt_stage[slot][j][row];
        mbar_arrive_warp(&wt_empty[slot]);
        ok = ok && mbar_wait(&full_bar[stage], (g / S) & 1, abort_v, 13);
        // a first walk block's low part overwrites stage (g + S - 1) % S's x area, whose
        // previous occupant is block g - 1: wait for its MMAs
        if (i == 0 && g >= 1)
          ok = ok && mbar_wait(&empty_bar[(g - 1) % S], ((g - 1) / S) & 1, abort_v, 20);
        if (ok) {
          uint8_t* xr = smem + stage * Cfg::kStage + (2 + j) * kTile;
          uint8_t* lr = smem + ((g + S - 1) % S) * Cfg::kStage + (2 + j) * kTile;
          if (i == 0) {  // bf16 high part in place, low part in the other stage
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4* ph = reinterpret_cast<uint4*>(xr + swz(row, c));
              const uint4 xv = *ph;
              uint4 hi, lo;
              split2(bf16lo(xv.x) * wt, bf16hi(xv.x) * wt, hi.x, lo.x);
              split2(bf16lo(xv.y) * wt, bf16hi(xv.y) * wt, hi.y, lo.y);
              split2(bf16lo(xv.z) * wt, bf16hi(xv.z) * wt, hi.z, lo.z);
              split2(bf16lo(xv.w) * wt, bf16hi(xv.w) * wt, hi.w, lo.w);
              *ph = hi;
              *reinterpret_cast<uint4*>(lr + swz(row, c)) = lo;
            }
          } else {  // bf16 X' in place
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4* ph = reinterpret_cast<uint4*>(xr + swz(row, c));
              const uint4 xv = *ph;
              const float2 ww = make_float2(wt, wt);
              *ph = make_uint4(scale_bf16x2(xv.x, ww), scale_bf16x2(xv.y, ww),
                               scale_bf16x2(xv.z, ww), scale_bf16x2(xv.w, ww));
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive_warp(&ready_bar[stage]);
      }
      // the unit's state: lane n = row, columns of head j
      const int ab = n & 1;
      ok = ok && mbar_wait(&acc_full[ab], (n >> 1) & 1, abort_v, 14);
      if (ok) {
        tc_fence_after();
        const uint32_t lane_addr =
            tmem + ab * Cfg::kAccCols + (uint32_t((warp & 3) * 32) << 16) + j * 64;
        float* out = seg_states +
                     (((int64_t(su.b) * sg.nseg + su.seg) * nheads + su.hq * HU + j) * kP) * kN +
                     row;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          uint32_t r[16];
          tmem_ld16(lane_addr + pc * 16, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) out[(pc * 16 + e) * kN] = __uint_as_float(r[e]);
        }
      }
      tc_fence_before();
      mbar_arrive_warp(&acc_empty[ab]);
      if (__any_sync(0xffffffffu, !ok || *abort_v)) break;
    }
  }
  // ------------------------------ teardown ------------------------------
  __syncthreads();
  if (*abort_v && warp == kMma && lane == 0) {  // let every issued MMA land before leaving
    mma_commit(&drain_bar);
    drain(&drain_bar, 0);
  }
  if (*abort_v && warp == kProd && lane == 0) {  // and every issued copy
    for (int i = 0; i < S; ++i)
      if (n_loads[i]) drain(&full_bar[i], (n_loads[i] - 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_free(tmem, 2 * Cfg::kAccCols);
}

// =============================================================================================
// seg_pass: the state passing between segments.  One thread per float4 of a (batch, head)
// state, all segments: H_in(0) = init, H_in(s + 1) = 2^decay(s) H_in(s) + S(s).  seg_states
// is overwritten in place with H_in; final_state receives the state after the last segment
// (it may alias init_state: each element is read before it is written, by one thread).  Only
// the first `useg` segments carry a summary S(s); with useg = nseg - 1 the entering state of
// the last segment is still written, and final_state must be NULL (the walk produces it).
// Segments are taken eight at a time so that eight loads are in flight per thread.
// =============================================================================================
constexpr int kPassThreads = 256;
__global__ void __launch_bounds__(kPassThreads, 4) seg_pass_kernel(
    float* __restrict__ seg_states, const float* __restrict__ seg_decay,
    const float* init_state, float* final_state, int batch, int nheads, int nseg, int useg) {
  constexpr int kVec = kP * kN / 4;  // float4 per (batch, head) state
  const int64_t e = int64_t(blockIdx.x) * kPassThreads + threadIdx.x;
  if (e >= int64_t(batch) * nheads * kVec) return;
  const int64_t bh = e / kVec;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int64_t off = (e % kVec) * 4;
  float4 run = init_state ? *reinterpret_cast<const float4*>(init_state + bh * kVec * 4 + off)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t stride = int64_t(nheads) * kP * kN;
  float* base = seg_states + (b * nseg * nheads + h) * int64_t(kP) * kN + off;
  const float* dbase = seg_decay + b * nseg * nheads + h;
  for (int s0 = 0; s0 < nseg; s0 += 8) {
    float4 v[8];
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (s0 + i < useg) {
        v[i] = *reinterpret_cast<const float4*>(base + (s0 + i) * stride);
        a[i] = ex2(dbase[int64_t(s0 + i) * nheads]);
      } else {
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        a[i] = 1.f;
      }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (s0 + i < nseg) {
        *reinterpret_cast<float4*>(base + (s0 + i) * stride) = run;
        run = make_float4(fmaf(a[i], run.x, v[i].x), fmaf(a[i], run.y, v[i].y),
                          fmaf(a[i], run.z, v[i].z), fmaf(a[i], run.w, v[i].w));
      }
  }
  if (final_state) *reinterpret_cast<float4*>(final_state + bh * kVec * 4 + off) = run;
}

// =============================================================================================
// scan_walk: the output pass.  The blocks of all (batch row, head pair) sequences, laid end to
// end (block k of sequence s at position s * nblk + k), are cut into `nct` equal ranges, one per
// CTA (taken by an atomic ticket in launch order).  A CTA walks its range block by block with
// the running state resident in TMEM; the range splits into items at segment boundaries (a
// segment is a stretch of a sequence whose entering state is known before the walk: the
// initial state for the first, a seg_state/seg_pass summary for the others).  An item that
// starts inside a segment continues the previous range's last item: that CTA walks its last item
// FIRST and publishes the state it ends with; this CTA walks such an item LAST and reads that
// state.  A CTA thus only ever waits on a lower ticket's first item, which waits on nothing.
// When every segment is a whole sequence there is no summary pass at all: x is read once and no
// state leaves the L2 except final_state.
//
// Per block k (G = C B^T once for both heads; masks; diagonal tiles (L o G o dt) X; off-
// diagonal C H; skip term D x; y store; then H <- exp(cs_end) H + B^T (w*x) in place), with
// block = 608 threads in four roles:
//   warps 0-15  compute (512 threads).  Thread (row = tid % 128, q = tid / 128): token row
//               `row` of a block (state row n = row in the state passes) and a quarter of the
//               columns: head j = q / 2 with p in [32 (q % 2), +32) for the state pass, X' and
//               the epilogue; G column groups q and q + 4 for the masks.  Four warps share
//               each TMEM lane quarter, so every phase is spread over all 16 warps (a phase's
//               latency, not only its instructions, bounds the block).  They also load each
//               item's entering state into TMEM and store its exit state.
//   warp 16     TMA producer (lane 0): B (double buffer), C, x (single buffers) per block; and,
//               with the whole warp, the cumsums: each block's dt of the two heads and its log2
//               cumsums in shared memory, up to two blocks ahead (lane l: rows 4l .. 4l+3).
//               x is not prefetched into L2 ahead of its load: TMA prefetches a block ahead
//               measured slower, as the C loads of the per-block chain then wait behind them.
//   warp 17     MMA issuer (lane 0).
//   warp 18     y writer (lane 0): TMA stores of each block's staged y, in two groups (one per
//               head) whose halves of the staging buffer are handed back separately.
// Warp w issues from scheduler w % 4; the compute warps of TMEM lane quarter 3 carry the most
// mask work, so the three role warps sit on the other three schedulers.
// Per block the compute warps write the masks (MMA: diagonal tiles), then the state pass
// (MMA: C H), then X' (MMA: state update) and the epilogue.  The masks come first so that the
// previous block's y stores, which read the staging buffer the state pass overwrites, drain
// while they are computed.  The last block of an item whose exit state is kept also sends the
// bf16 remainder of X' through the tensor core (written over C's tiles once C H is done), so
// that state carries about 16 bits of the block's input.  Roles hand blocks to each other
// through mbarriers only (blocks are numbered across items, so the rings run on from one item to
// the next); a thread is never more than one phase of a barrier ahead of the slowest, because
// every barrier it waits on next needs an arrival that the slowest makes after its own previous
// wait.
// Shared memory (1024-aligned, 12 x 16 KB):
//   sC   2 tiles  C, K-major (rows t), n halves
//   sB   4 tiles  B, rows s, n halves, two slots (blocks k % 2): K-major for G = C B^T,
//                 MN-major for B^T X'
//   sX   2 tiles  x of the two heads (rows t, 64 p), MN-major; scaled in place to X' = w x
//                 once the diagonal MMAs have read it
//   sHh  2 tiles  bf16 high part of the entering state of the two heads (rows n, 64 p)
//   sHl  2 tiles  bf16 low part (the state's rounding remainder), same layout
//   (sHh + sHl, free once C H has been computed, stage the block's y for the TMA stores)
// TMEM (512 columns): [0,128) running state H (head, p) | [128,256) diagonal accumulators |
//   [256,384) off-diagonal accumulators C H | [384,512) G = C B^T, overwritten in place by
//   the two heads' bf16 masked tiles (16-column group kk -> columns 8h .. 8h+7 for head h),
//   which the diagonal MMAs read as their A operand.
// =============================================================================================
constexpr uint32_t kOffC = 0, kOffB = 2 * kTile, kOffX = 6 * kTile, kOffHh = 8 * kTile,
                   kOffHl = 10 * kTile, kSmemTiles = 12 * kTile;

// y staging (in sHh/sHl) and its TMA stores.  Float32 y: 4 boxes {32 p, 128 t} (one per
// thread quarter q: head q/2, p-half q%2), 128B-swizzled.  Bf16 y: 2 boxes {64 p, 128 t} (one
// per head).
template <typename TY> struct ystage;
template <> struct ystage<float> {
  // thread (t, q) writes its 32 values (16 per call, half = 0/1) into box q, row t
  static __device__ __forceinline__ void put16(uint8_t* stage, int t, int q, int half,
                                               const float (&v)[16]) {
    uint8_t* box = stage + q * kTile;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(box + swz(t, half * 4 + i)) =
          make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  // part 0: the boxes over the staging's tiles 0 and 2 (sHh and sHl of head 0); part 1: tiles 1
  // and 3 (head 1)
  static __device__ __forceinline__ void store_part(const CUtensorMap* map, const uint8_t* stage,
                                                    int h0, int t0, int b, int part,
                                                    uint64_t policy) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int q = part + 2 * i;
      tma_store_3d_hint(map, stage + q * kTile, (h0 + q / 2) * kP + (q % 2) * 32, t0, b, policy);
    }
  }
};
template <> struct ystage<__nv_bfloat16> {
  static __device__ __forceinline__ void put16(uint8_t* stage, int t, int q, int half,
                                               const float (&v)[16]) {
    uint8_t* box = stage + (q / 2) * kTile;
    const int c0 = (q % 2) * 4 + half * 2;
    *reinterpret_cast<uint4*>(box + swz(t, c0)) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                   pack_bf16x2(v[6], v[7]));
    *reinterpret_cast<uint4*>(box + swz(t, c0 + 1)) =
        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                   pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
  }
  // part j: head j's box, over the staging's tile j
  static __device__ __forceinline__ void store_part(const CUtensorMap* map, const uint8_t* stage,
                                                    int h0, int t0, int b, int part,
                                                    uint64_t policy) {
    tma_store_3d_hint(map, stage + part * kTile, (h0 + part) * kP, t0, b, policy);
  }
};

// The plan of one call's walk (host-computed).
struct WalkPlan {
  int64_t total;  // batch * npair * nblk: every block of every (batch row, head pair) sequence
  int nblk;       // 128-token blocks per sequence
  int seg_blks;   // blocks per segment
  int nseg;       // segments per sequence (1: the entering state of a sequence is init_state)
  int npair;      // head pairs
  int nct;        // ranges (= CTAs)
  uint64_t wait_ns;  // limit of every bounded wait (2 s in production; 0: no waiting)
};
// Where an item's entering state comes from and where its exit state goes.
enum : int { kSrcInit = 0, kSrcSeg = 1, kSrcSlot = 2 };
enum : int { kDstNone = 0, kDstFinal = 1, kDstSlot = 2 };
struct WalkItem {
  int seq, k0, k1, src, dst;  // sequence b * npair + pair, blocks [k0, k1)
};
constexpr int kMaxItems = 16;
constexpr int kSlotFloats = 2 * kP * kN;  // one published state: two heads, [j][p][n]

// The items of range r in walk order (the publishing item first, the waiting one last), written
// to `out` (shared memory).  Returns their number, or -1 if there are more than kMaxItems (the
// host plans fewer).  Three passes over the range, one per class, so no local list is needed.
__device__ int walk_items(const WalkPlan& pl, int r, bool has_final, WalkItem* out) {
  const int64_t g0 = pl.total * r / pl.nct, g1 = pl.total * (r + 1) / pl.nct;
  int m = 0;
  for (int cls = 0; cls < 3; ++cls) {
    for (int64_t g = g0; g < g1;) {
      WalkItem w;
      w.seq = int(g / pl.nblk);
      w.k0 = int(g % pl.nblk);
      const int seg = w.k0 / pl.seg_blks;
      const int seg_end = min((seg + 1) * pl.seg_blks, pl.nblk);
      w.k1 = int(g1 - g < int64_t(seg_end - w.k0) ? w.k0 + (g1 - g) : int64_t(seg_end));
      w.src = (w.k0 % pl.seg_blks) ? kSrcSlot : (pl.nseg > 1 ? kSrcSeg : kSrcInit);
      w.dst = w.k1 < seg_end ? kDstSlot : ((w.k1 == pl.nblk && has_final) ? kDstFinal : kDstNone);
      const int c = w.dst == kDstSlot ? 0 : (w.src == kSrcSlot ? 2 : 1);
      if (c == cls) {
        if (m == kMaxItems) return -1;
        out[m++] = w;
      }
      g += w.k1 - w.k0;
    }
  }
  return m;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait (warp-collective) until *flag != 0: lane 0 polls, then every lane acquires.  The
// limit works as in mbar_wait (0: give up unless the flag is already set).
__device__ __forceinline__ bool flag_wait(const int* flag, volatile int* abort, unsigned site,
                                          uint64_t limit_ns) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t t0 = globaltimer();
    while (ld_acquire_gpu(flag) == 0) {
      if (*abort) {
        ok = 0;
        break;
      }
      if (limit_ns == 0 || globaltimer() - t0 > limit_ns) {
        latch_status(SSD_ERR_DEVICE_TIMEOUT, site);
        *abort = 1;
        ok = 0;
        break;
      }
      __nanosleep(256);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) (void)ld_acquire_gpu(flag);
  return ok != 0;
}

constexpr int kComputeThreads = 512;
constexpr int kWalkThreads = kComputeThreads + 96;

// mbarriers of the walk (all in shared memory)
struct OutBars {
  uint64_t c_full, b_full[2], x_full;        // TMA -> consumers
  uint64_t c_empty, b_empty[2], x_empty;     // MMA completion -> producer
  uint64_t g_done, d_done, o_done, st_done;  // MMA completion -> compute
  uint64_t m0_ready, m1_ready, h_ready, xp_ready;  // compute -> MMA issuer
  uint64_t y_staged;                         // compute -> y writer
  uint64_t stage_free[2];                    // y writer -> compute (halves of the staging)
  uint64_t cs_full[2], cs_empty[2];          // cumsum warp <-> compute (per cumsum buffer)
  uint64_t pub;                              // compute: exit state written (published item)
  uint64_t drain;
};

template <typename TY>
__global__ void __launch_bounds__(kWalkThreads, 1) scan_walk_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
    const float* __restrict__ dt, const float* __restrict__ A, const float* __restrict__ D,
    const float* init_state, const float* seg_hin, float* final_state, float* slots,
    int* flags, unsigned* ticket, int64_t seqlen, int nheads, int heads_per_group,
    WalkPlan pl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ OutBars bars;
  __shared__ uint32_t tmem_base_sh;
  // per block (two buffers, block k in buffer k % 2) and head: log2 cumsums cs, cl = cs -
  // log2(dt) (+inf where dt = 0), v_s = exp(cs_{s|15} - cs_s) dt_s
  __shared__ __align__(16) float cs_sh[2][2][kBlk];
  __shared__ __align__(16) float cl_sh[2][2][kBlk];
  __shared__ __align__(16) float v_sh[2][2][kBlk];
  __shared__ WalkItem items_sh[kMaxItems];
  __shared__ int nitems_sh, nblocks_sh, range_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  volatile int* abort_v = &abort_flag;
  uint32_t n_c = 0, n_x = 0, n_b[2] = {0, 0};  // the producer's loads issued per barrier

  if (tid == 0) {
    abort_flag = 0;
    const int r = int(atomicAdd(ticket, 1u));
    int n = r < pl.nct ? walk_items(pl, r, final_state != nullptr, items_sh) : 0;
    if (n < 0) {
      latch_status(SSD_ERR_UNSUPPORTED, 70);
      n = 0;
    }
    int nb = 0;
    for (int i = 0; i < n; ++i) nb += items_sh[i].k1 - items_sh[i].k0;
    range_sh = r;
    nitems_sh = n;
    nblocks_sh = nb;
    uint64_t* all = reinterpret_cast<uint64_t*>(&bars);
    for (int i = 0; i < int(sizeof(OutBars) / 8); ++i) mbar_init(all + i, 1);
    mbar_init(&bars.m0_ready, kComputeThreads);
    mbar_init(&bars.m1_ready, kComputeThreads);
    mbar_init(&bars.h_ready, kComputeThreads);
    mbar_init(&bars.xp_ready, kComputeThreads);
    mbar_init(&bars.y_staged, kComputeThreads);
    mbar_init(&bars.pub, kComputeThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.cs_full[i], 32);
      mbar_init(&bars.cs_empty[i], kComputeThreads);
    }
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tH = tmem, tD = tmem + 128, tO = tmem + 256, tG = tmem + 384;
  const uint32_t sbase = smem_u32(smem);
  const int nit = nitems_sh, nbt = nblocks_sh, range = range_sh;

  if (warp == 16) {
    // ------------------------------ TMA producer (lane 0) and cumsums (whole warp) -----------
    // Per block: B (double buffer), the block's cumsums, C, x.  Cumsums, per block and head:
    // cs_t = inclusive log2 cumsum of dt A (within the block), cl_t = cs_t - log2(dt_t) (+inf
    // where dt = 0), v_s = exp(cs_r(s) - cs_s) dt_s with r(s) = s | 15 (lane l: rows 4l .. 4l+3);
    // the next block's dt is loaded while the current one is processed.  The cumsums of block j
    // wait for block j - 2's compute to finish, which comes before block j - 1's C H, so the
    // C and x loads after them are not held back.
    const uint64_t keep = l2_evict_last(), stream = l2_evict_first();  // B/C reread, x once
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_c);
    }
    float v[8];  // dt of rows 4 lane + r, head h at v[2r + h]
    auto load_dt = [&](int it, int kb) {
      if (it >= nit) return;
      const WalkItem w = items_sh[it];
      const int b = w.seq / pl.npair, h0 = (w.seq % pl.npair) * 2;
      const float* dtb = dt + int64_t(b) * seqlen * nheads + h0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t tok = int64_t(kb) * kBlk + 4 * lane + r;
        const bool in = tok < seqlen;
        v[2 * r] = in ? dtb[tok * nheads] : 0.f;
        v[2 * r + 1] = in ? dtb[tok * nheads + 1] : 0.f;
      }
    };
    if (nit > 0) load_dt(0, items_sh[0].k0);
    const float inf = __int_as_float(0x7f800000);
    // bounded wait by every lane, the same result in all of them
    auto wait_all = [&](uint64_t* bar, uint32_t parity, unsigned site) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_v, site, pl.wait_ns));
    };
    int j = 0;
    bool ok = true;
    for (int it = 0; it < nit && ok; ++it) {
      const WalkItem w = items_sh[it];
      const int b = w.seq / pl.npair, h0 = (w.seq % pl.npair) * 2;
      const int g = h0 / heads_per_group;
      const float al[2] = {A[h0] * kLog2e, A[h0 + 1] * kLog2e};
      for (int k = w.k0; k < w.k1; ++k, ++j) {
        const int t0 = k * kBlk;
        // B of block j into slot j % 2 once block j - 2's G and state MMAs are done
        if (j >= 2 && !wait_all(&bars.b_empty[j & 1], ((j - 2) >> 1) & 1, 33)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* bdst = smem + kOffB + (j & 1) * 2 * kTile;
          ++n_b[j & 1];
          mbar_arrive_expect_tx(&bars.b_full[j & 1], 2 * kTile);
          tma_load_3d_hint(bdst, &tm_b, &bars.b_full[j & 1], g * kN, t0, b, keep);
          tma_load_3d_hint(bdst + kTile, &tm_b, &bars.b_full[j & 1], g * kN + 64, t0, b, keep);
        }
        // cumsums of block j into buffer j % 2 once block j - 2's compute is done with it
        const int bf = j & 1;
        if (j >= 2 && !wait_all(&bars.cs_empty[bf], ((j - 2) >> 1) & 1, 58)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float d0 = v[h], d1 = v[2 + h], d2 = v[4 + h], d3 = v[6 + h];
          float c0 = d0 * al[h];
          float c1 = fmaf(d1, al[h], c0);
          float c2 = fmaf(d2, al[h], c1);
          float c3 = fmaf(d3, al[h], c2);
          const float off = warp_inclusive_scan(c3) - c3;
          c0 += off;
          c1 += off;
          c2 += off;
          c3 += off;
          const float l0 = d0 > 0.f ? c0 - __log2f(d0) : inf;
          const float l1 = d1 > 0.f ? c1 - __log2f(d1) : inf;
          const float l2 = d2 > 0.f ? c2 - __log2f(d2) : inf;
          const float l3 = d3 > 0.f ? c3 - __log2f(d3) : inf;
          const float cr = __shfl_sync(0xffffffffu, c3, lane | 3);  // cs at row (4 lane) | 15
          *reinterpret_cast<float4*>(&cs_sh[bf][h][4 * lane]) = make_float4(c0, c1, c2, c3);
          *reinterpret_cast<float4*>(&cl_sh[bf][h][4 * lane]) = make_float4(l0, l1, l2, l3);
          *reinterpret_cast<float4*>(&v_sh[bf][h][4 * lane]) =
              make_float4(ex2(cr - l0), ex2(cr - l1), ex2(cr - l2), ex2(cr - l3));
        }
        mbar_arrive_warp(&bars.cs_full[bf]);
        if (k + 1 < w.k1) load_dt(it, k + 1);
        else if (it + 1 < nit) load_dt(it + 1, items_sh[it + 1].k0);
        // C once block j - 1's C H is done
        if (j >= 1 && !wait_all(&bars.c_empty, (j - 1) & 1, 31)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          ++n_c;
          mbar_arrive_expect_tx(&bars.c_full, 2 * kTile);
          tma_load_3d_hint(smem + kOffC, &tm_c, &bars.c_full, g * kN, t0, b, keep);
          tma_load_3d_hint(smem + kOffC + kTile, &tm_c, &bars.c_full, g * kN + 64, t0, b, keep);
        }
        // x once block j - 1's state MMA is done
        if (j >= 1 && !wait_all(&bars.x_empty, (j - 1) & 1, 32)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          ++n_x;
          mbar_arrive_expect_tx(&bars.x_full, 2 * kTile);
          tma_load_3d_hint(smem + kOffX, &tm_x, &bars.x_full, h0 * kP, t0, b, stream);
          tma_load_3d_hint(smem + kOffX + kTile, &tm_x, &bars.x_full, (h0 + 1) * kP, t0, b,
                           stream);
        }
      }
    }
  } else if (warp == 17) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t id_g = idesc_bf16(128, 128, 0, 0);
      const uint32_t id_off = idesc_bf16(128, 128, 0, 1);
      const uint32_t id_diag = idesc_bf16(128, 64, 0, 1);
      const uint32_t id_st = idesc_bf16(128, 128, 1, 1);
      // descriptors are built once; a K step or a tile offset adds (bytes >> 4) to the start
      // address field (every address stays below 256 KB, so the field cannot carry)
      const uint64_t dC = sdesc(sbase + kOffC, 16, 1024);       // K-major (rows t or s)
      const uint64_t dBk = sdesc(sbase + kOffB, 16, 1024);
      const uint64_t dBm = sdesc(sbase + kOffB, kTile, 1024);   // MN-major
      const uint64_t dX = sdesc(sbase + kOffX, kTile, 1024);
      const uint64_t dHh = sdesc(sbase + kOffHh, kTile, 1024);
      const uint64_t dHl = sdesc(sbase + kOffHl, kTile, 1024);
      auto kmaj = [](int kk) { return uint64_t(((kk >> 2) * kTile + (kk & 3) * 32) >> 4); };
      const uint64_t dXlo = sdesc(sbase + kOffC, kTile, 1024);  // X' low part over C's tiles
      int it = 0, kend = nit > 0 ? items_sh[0].k1 - items_sh[0].k0 : 0;
      for (int k = 0; k < nbt; ++k) {
        const uint32_t par = k & 1;
        const uint64_t bslot = (k & 1) ? uint64_t((2 * kTile) >> 4) : 0u;
        // the last block of an item whose exit state is kept also sends X's bf16 remainder
        while (it < nit && k >= kend) {
          ++it;
          if (it < nit) kend += items_sh[it].k1 - items_sh[it].k0;
        }
        const bool lo = it < nit && k == kend - 1 && items_sh[it].dst != kDstNone;
        if (k > 0 && !mbar_wait(&bars.d_done, par ^ 1, abort_v, 41, pl.wait_ns)) break;  // G region free
        if (!mbar_wait(&bars.c_full, par, abort_v, 42, pl.wait_ns)) break;
        if (!mbar_wait(&bars.b_full[k & 1], (k >> 1) & 1, abort_v, 43, pl.wait_ns)) break;
        tc_fence_after();
        // G = C B^T (M = t, N = s, K = n)
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk)
          mma_ss(tG, dC + kmaj(kk), dBk + bslot + kmaj(kk), id_g, kk > 0 ? 1u : 0u);
        mma_commit(&bars.g_done);
        // Diag_h = M_h X_h (M = t, N = p, K = s), A = head h's bf16 mask in TMEM (columns
        // 8h .. 8h+7 of each 16-column group); head 0 while head 1's mask is being written
        if (!mbar_wait(&bars.x_full, par, abort_v, 45, pl.wait_ns)) break;
        auto diag = [&](int h) {
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk)
            mma_ts(tD + h * 64, tG + kk * 16 + h * 8, dX + h * (kTile >> 4) + kk * 128, id_diag,
                   kk > 0 ? 1u : 0u);
        };
        if (!mbar_wait(&bars.m0_ready, par, abort_v, 46, pl.wait_ns)) break;
        tc_fence_after();
        diag(0);
        if (!mbar_wait(&bars.m1_ready, par, abort_v, 48, pl.wait_ns)) break;
        tc_fence_after();
        diag(1);
        mma_commit(&bars.d_done);
        // Off = C (Hhi + Hlo) (M = t, N = (head, p), K = n)
        if (!mbar_wait(&bars.h_ready, par, abort_v, 44, pl.wait_ns)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk) {
          mma_ss(tO, dC + kmaj(kk), dHh + kk * 128, id_off, kk > 0 ? 1u : 0u);
          mma_ss(tO, dC + kmaj(kk), dHl + kk * 128, id_off, 1u);
        }
        mma_commit(&bars.o_done);
        if (!lo) mma_commit(&bars.c_empty);
        // H += B^T X' (M = n, N = (head, p), K = t), plus B^T X'_lo from C's tiles
        if (!mbar_wait(&bars.xp_ready, par, abort_v, 47, pl.wait_ns)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          mma_ss(tH, dBm + bslot + kk * 128, dX + kk * 128, id_st, 1u);
          if (lo) mma_ss(tH, dBm + bslot + kk * 128, dXlo + kk * 128, id_st, 1u);
        }
        if (lo) mma_commit(&bars.c_empty);
        mma_commit(&bars.st_done);
        mma_commit(&bars.x_empty);
        mma_commit(&bars.b_empty[k & 1]);
      }
    }
  } else if (warp == 18) {
    // ------------------------------ y writer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tm_y);
      const uint64_t stream = l2_evict_first();  // y is not read again here
      const uint8_t* stage = smem + kOffHh;
      int j = 0;
      bool ok = true;
      for (int it = 0; it < nit && ok; ++it) {
        const WalkItem w = items_sh[it];
        const int b = w.seq / pl.npair, h0 = (w.seq % pl.npair) * 2;
        for (int k = w.k0; k < w.k1; ++k, ++j) {
          if (!mbar_wait(&bars.y_staged, j & 1, abort_v, 61, pl.wait_ns)) {
            ok = false;
            break;
          }
          // two store groups; each half of the staging buffer (head 0's sHh/sHl tiles, then head
          // 1's) is handed back once its group has read it
          ystage<TY>::store_part(&tm_y, stage, h0, k * kBlk, b, 0, stream);
          bulk_commit();
          ystage<TY>::store_part(&tm_y, stage, h0, k * kBlk, b, 1, stream);
          bulk_commit();
          bulk_wait_read_1();
          mbar_arrive(&bars.stage_free[0]);
          bulk_wait_read();
          mbar_arrive(&bars.stage_free[1]);
        }
      }
      bulk_wait_all();
    }
  } else {
    // ------------------------------ compute warps ------------------------------
    const int row = tid & 127, q = tid >> 7;
    const int j = q >> 1, p0 = (q & 1) * 32;        // head and p-range of the state/epilogue
    const int wq = warp & 3;                        // TMEM lane quarter of this warp
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    bool ok = true, stop = false;
    uint8_t* stage = smem + kOffHh;                 // y staging (sHh + sHl)
    const int t = row;
    const int wlast = wq * 32 + 31;                 // last row of this warp
    const bool live0 = q * 16 <= wlast, live1 = (q + 4) * 16 <= wlast;
    const uint32_t gaddr0 = tG + lane_off + q * 16, gaddr1 = gaddr0 + 64;
    int k = 0;                                      // blocks walked so far (all items)
    for (int it = 0; it < nit && !stop; ++it) {
      const WalkItem w = items_sh[it];
      const int b = w.seq / pl.npair, h0 = (w.seq % pl.npair) * 2;
      // ---- the item's entering state -> TMEM (lane n = row, columns (j, p0 .. p0+32)), once
      //      the previous item's last state MMA is done ----
      if (k > 0) ok = ok && mbar_wait(&bars.st_done, (k - 1) & 1, abort_v, 71, pl.wait_ns);
      const float* src = nullptr;
      ok = __all_sync(0xffffffffu, ok);
      if (w.src == kSrcSlot) {
        if (ok) ok = flag_wait(flags + (range - 1), abort_v, 74, pl.wait_ns);
        src = slots + int64_t(range - 1) * kSlotFloats + (j * kP + p0) * kN + row;
      } else if (w.src == kSrcSeg) {
        const int seg = w.k0 / pl.seg_blks;
        src = seg_hin + (((int64_t(b) * pl.nseg + seg) * nheads + h0 + j) * kP + p0) * kN + row;
      } else if (init_state) {
        src = init_state + ((int64_t(b) * nheads + h0 + j) * kP + p0) * kN + row;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = src ? __float_as_uint(src[(pc * 16 + e) * kN]) : 0u;
          tmem_st16(tH + lane_off + j * 64 + p0 + pc * 16, r);
        }
        tmem_wait_st();
      }
      const float Dh = D ? D[h0 + j] : 0.f;
      for (int kb = w.k0; kb < w.k1; ++kb, ++k) {
        const uint32_t par = k & 1;
        const int bf = k & 1;
        ok = ok && mbar_wait(&bars.cs_full[bf], (k >> 1) & 1, abort_v, 50, pl.wait_ns);
        // ---- masked tiles.  Thread (row t, q) owns the 16-column groups q and q + 4 of G
        //      (columns [16q, 16q+16) and [16q+64, 16q+80)), which spreads the rows' diagonal
        //      groups over all warps.  M_h[t, s] = G[t, s] exp(cs_t - cs_s) dt_s for s <= t, in
        //      bf16, written over TMEM columns 8h .. 8h+7 of the group.  Each warp takes one
        //      branch per group: the factorized product where all its rows are past the group,
        //      the exact exponent where some row meets it, zeros where none reaches it ----
        float gv[32];
        ok = ok && mbar_wait(&bars.g_done, par, abort_v, 52, pl.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && live0) {
          tc_fence_after();
          uint32_t r0[16], r1[16];
          tmem_ld16(gaddr0, r0);
          if (live1) tmem_ld16(gaddr1, r1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) { gv[e] = __uint_as_float(r0[e]); gv[16 + e] = __uint_as_float(r1[e]); }
        }
        // one 16-column group (gg = 0: group q, gg = 1: group q + 4) of head h's mask, packed
#define SSD_MASK_GROUP(H, GG, R)                                                               \
  {                                                                                            \
    const int s0 = (q + 4 * (GG)) * 16;                                                        \
    const bool live = (GG) ? live1 : live0;                                                    \
    if (wq * 32 >= s0 + 15) {                                                                  \
      const float u = ex2(cs_sh[bf][H][t] - cs_sh[bf][H][s0 + 15]);                            \
      const float2 uu = make_float2(u, u);                                                     \
      const float4* vp = reinterpret_cast<const float4*>(&v_sh[bf][H][s0]);                    \
      _Pragma("unroll") for (int e4 = 0; e4 < 4; ++e4) {                                      \
        const float4 vv = vp[e4];                                                              \
        const float* gq = &gv[(GG) * 16 + 4 * e4];                                             \
        const float2 a = mul2(make_float2(gq[0], gq[1]), mul2(uu, make_float2(vv.x, vv.y)));   \
        const float2 c = mul2(make_float2(gq[2], gq[3]), mul2(uu, make_float2(vv.z, vv.w)));   \
        R[2 * e4] = pack_bf16x2(a.x, a.y);                                                     \
        R[2 * e4 + 1] = pack_bf16x2(c.x, c.y);                                                 \
      }                                                                                        \
    } else if (live) {                                                                         \
      const float ct = cs_sh[bf][H][t];                                                        \
      const float2 cc = make_float2(ct, ct);                                                   \
      const float4* cp = reinterpret_cast<const float4*>(&cl_sh[bf][H][s0]);                   \
      _Pragma("unroll") for (int e4 = 0; e4 < 4; ++e4) {                                      \
        const float4 cl = cp[e4];                                                              \
        const int s = s0 + 4 * e4;                                                             \
        const float* gq = &gv[(GG) * 16 + 4 * e4];                                             \
        const float2 d01 = sub2(cc, make_float2(cl.x, cl.y));                                  \
        const float2 d23 = sub2(cc, make_float2(cl.z, cl.w));                                  \
        const float2 a = mul2(make_float2(gq[0], gq[1]), make_float2(ex2(d01.x), ex2(d01.y))); \
        const float2 c = mul2(make_float2(gq[2], gq[3]), make_float2(ex2(d23.x), ex2(d23.y))); \
        R[2 * e4] = pack_bf16x2(s + 0 <= t ? a.x : 0.f, s + 1 <= t ? a.y : 0.f);              \
        R[2 * e4 + 1] = pack_bf16x2(s + 2 <= t ? c.x : 0.f, s + 3 <= t ? c.y : 0.f);          \
      }                                                                                        \
    } else {                                                                                   \
      _Pragma("unroll") for (int e = 0; e < 8; ++e) R[e] = 0u;                                \
    }                                                                                          \
  }
        // head 0, then head 1 (its own TMEM columns, so no wait for the first diagonal MMA)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (ok) {
            uint32_t r0[8], r1[8];
            if (hh == 0) {
              SSD_MASK_GROUP(0, 0, r0)
              SSD_MASK_GROUP(0, 1, r1)
            } else {
              SSD_MASK_GROUP(1, 0, r0)
              SSD_MASK_GROUP(1, 1, r1)
            }
            tmem_st8(gaddr0 + hh * 8, r0);
            tmem_st8(gaddr1 + hh * 8, r1);
            tmem_wait_st();
          }
          tc_fence_before();
          mbar_arrive_warp(hh == 0 ? &bars.m0_ready : &bars.m1_ready);
        }
#undef SSD_MASK_GROUP
        // ---- state pass (lane n = row, columns (j, p0 .. p0+32)): bf16 high/low copy of H for
        //      C H (the decay H <- exp(cs_end) H follows in the X' phase).  Needs the previous
        //      block's state MMA and the previous block's y stores to have read the staging
        //      buffer (sHh/sHl) ----
        if (k > 0) ok = ok && mbar_wait(&bars.st_done, par ^ 1, abort_v, 51, pl.wait_ns);
        if (k > 0) ok = ok && mbar_wait(&bars.stage_free[j], par ^ 1, abort_v, 55, pl.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          uint8_t* hh = smem + kOffHh + j * kTile;
          uint8_t* hl = smem + kOffHl + j * kTile;
          uint32_t ra[16], rb[16];
          tmem_ld16(tH + lane_off + j * 64 + p0, ra);
          tmem_wait_ld();
#define SSD_HPASS(R, PC)                                                                      \
  {                                                                                           \
    uint32_t hi[8], lo[8];                                                                    \
    _Pragma("unroll") for (int e = 0; e < 8; ++e)                                            \
        split2(__uint_as_float(R[2 * e]), __uint_as_float(R[2 * e + 1]), hi[e], lo[e]);      \
    const int ch = (p0 >> 3) + (PC) * 2;                                                      \
    *reinterpret_cast<uint4*>(hh + swz(row, ch)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);    \
    *reinterpret_cast<uint4*>(hh + swz(row, ch + 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]); \
    *reinterpret_cast<uint4*>(hl + swz(row, ch)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);    \
    *reinterpret_cast<uint4*>(hl + swz(row, ch + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]); \
  }
          SSD_HPASS(ra, 0)
          tmem_ld16(tH + lane_off + j * 64 + p0 + 16, rb);
          tmem_wait_ld();
          SSD_HPASS(rb, 1)
#undef SSD_HPASS
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive_warp(&bars.h_ready);
        // ---- once the diagonal MMAs are done: X' = w x in place for the state MMA (row t,
        //      head j, p in [p0, p0+32)); then, once C H is done too, y_t = Diag + exp(cs_t) Off
        //      + D x_t staged in shared memory and written by TMA ----
        ok = ok && mbar_wait(&bars.d_done, par, abort_v, 54, pl.wait_ns);
        uint32_t xw[16];
        if (ok) {
          tc_fence_after();
          const float wj = ex2(cs_sh[bf][j][kBlk - 1] - cl_sh[bf][j][t]);
          uint8_t* xrow = smem + kOffX + j * kTile;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint4* pch = reinterpret_cast<uint4*>(xrow + swz(t, (p0 >> 3) + cc));
            const uint4 v = *pch;
            xw[cc * 4 + 0] = v.x; xw[cc * 4 + 1] = v.y; xw[cc * 4 + 2] = v.z; xw[cc * 4 + 3] = v.w;
            const float2 ww = make_float2(wj, wj);
            *pch = make_uint4(scale_bf16x2(v.x, ww), scale_bf16x2(v.y, ww), scale_bf16x2(v.z, ww),
                              scale_bf16x2(v.w, ww));
          }
          fence_proxy_async_smem();
          // H <- exp(cs_end) H in TMEM before the state MMA adds B^T X' (done here, off the
          // masks -> state pass -> C H -> next C chain, which only needs H's bf16 copy)
          const float al = ex2(cs_sh[bf][j][kBlk - 1]);
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {
            uint32_t r[16];
            tmem_ld16(tH + lane_off + j * 64 + p0 + pc * 16, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 sc = mul2(make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])),
                                     make_float2(al, al));
              r[2 * e] = __float_as_uint(sc.x);
              r[2 * e + 1] = __float_as_uint(sc.y);
            }
            tmem_st16(tH + lane_off + j * 64 + p0 + pc * 16, r);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        // the last block of an item whose exit state is kept also sends the bf16 remainder of
        // X' (over C's tiles, free once C H is done): its X' is handed over only then
        const bool lo = kb == w.k1 - 1 && w.dst != kDstNone;
        if (!lo) mbar_arrive_warp(&bars.xp_ready);
        ok = ok && mbar_wait(&bars.o_done, par, abort_v, 57, pl.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (lo) {
          if (ok) {
            tc_fence_after();
            const float wj = ex2(cs_sh[bf][j][kBlk - 1] - cl_sh[bf][j][t]);
            uint8_t* lrow = smem + kOffC + j * kTile;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t hi4[4], lo4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t xv = xw[cc * 4 + i];
                split2(bf16lo(xv) * wj, bf16hi(xv) * wj, hi4[i], lo4[i]);
              }
              *reinterpret_cast<uint4*>(lrow + swz(t, (p0 >> 3) + cc)) =
                  make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
            }
            fence_proxy_async_smem();
          }
          mbar_arrive_warp(&bars.xp_ready);
        }
        if (ok) {
          tc_fence_after();
          const float ej = ex2(cs_sh[bf][j][t]);
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {
            uint32_t rd[16], ro[16];
            tmem_ld16(tD + lane_off + j * 64 + p0 + pc * 16, rd);
            tmem_ld16(tO + lane_off + j * 64 + p0 + pc * 16, ro);
            tmem_wait_ld();
            float yv[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t xv = xw[pc * 8 + e];
              const float2 dd = fma2(make_float2(ej, ej),
                                     make_float2(__uint_as_float(ro[2 * e]), __uint_as_float(ro[2 * e + 1])),
                                     make_float2(__uint_as_float(rd[2 * e]), __uint_as_float(rd[2 * e + 1])));
              const float2 yy = fma2(make_float2(Dh, Dh), make_float2(bf16lo(xv), bf16hi(xv)), dd);
              yv[2 * e] = yy.x;
              yv[2 * e + 1] = yy.y;
            }
            ystage<TY>::put16(stage, t, q, pc, yv);
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive_warp(&bars.y_staged);
        mbar_arrive_warp(&bars.cs_empty[bf]);  // done with block k's cumsums and TMEM reads
        if (__any_sync(0xffffffffu, !ok || *abort_v)) {
          stop = true;
          break;
        }
      }
      if (stop) break;
      // ---- the item's exit state: final_state, or the slot the next range reads ----
      if (w.dst != kDstNone) {
        ok = ok && mbar_wait(&bars.st_done, (k - 1) & 1, abort_v, 72, pl.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          float* dst = w.dst == kDstFinal
                           ? final_state + ((int64_t(b) * nheads + h0 + j) * kP + p0) * kN + row
                           : slots + int64_t(range) * kSlotFloats + (j * kP + p0) * kN + row;
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {
            uint32_t r[16];
            tmem_ld16(tH + lane_off + j * 64 + p0 + pc * 16, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[(pc * 16 + e) * kN] = __uint_as_float(r[e]);
          }
        }
        tc_fence_before();
        if (w.dst == kDstSlot) {
          __threadfence();
          mbar_arrive_warp(&bars.pub);
          if (tid == 0 && mbar_wait(&bars.pub, 0, abort_v, 73, pl.wait_ns)) {
            __threadfence();
            st_release_gpu(flags + range, 1);
          }
        }
      }
      if (__any_sync(0xffffffffu, !ok || *abort_v)) break;
    }
  }
  // ------------------------------ teardown ------------------------------
  __syncthreads();
  if (*abort_v && warp == 17 && lane == 0) {  // let every issued MMA land before leaving
    mma_commit(&bars.drain);
    drain(&bars.drain, 0);
  }
  if (*abort_v && warp == 16 && lane == 0) {  // and every issued copy
    if (n_c) drain(&bars.c_full, (n_c - 1) & 1);
    if (n_x) drain(&bars.x_full, (n_x - 1) & 1);
    for (int i = 0; i < 2; ++i)
      if (n_b[i]) drain(&bars.b_full[i], (n_b[i] - 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_free(tmem, 512);
}

}  // namespace tc
}  // namespace ssd
