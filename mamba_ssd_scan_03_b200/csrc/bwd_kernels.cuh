// bwd_kernels.cuh -- gradients of the chunked scan on float32 CUDA cores.
//
// The parallel form exists so that the layer can be trained ("State Space Model"
// (book.paithon.it), "Un sistema che riassume il passato": one trains in the all-at-once form;
// "Architektury Mamba-2, State Space Models i liniowa atencja" (tech.tersel.eu), "Rewolucja
// Mamba-2 i teoria State Space Duality SSD": the SSD block algorithm speeds training up).  The
// pages give no gradient formulas; these follow from the recurrence by the chain rule.  With
// a_t = dt_t A_h, h_t = exp(a_t) h_{t-1} + dt_t x_t B_t^T ([P, N]) and y_t = h_t C_t + D x_t, the
// adjoint of h_t is G_t = dy_t C_t^T + exp(a_{t+1}) G_{t+1} (G after the last token = the
// gradient of the final state), and
//     dx_t = dt_t G_t B_t + D dy_t                dB_t += dt_t G_t^T x_t   (heads of a group)
//     dC_t += h_t^T dy_t                          dD   += <dy_t, x_t>
//     ddt_t = x_t^T G_t B_t + A <G_t, exp(a_t) h_{t-1}>     dA += dt_t <G_t, exp(a_t) h_{t-1}>
//     d init = exp(a_0) G_0.
//
// Blocked like the forward ("Mamba-2 (2024): SSM e attention sono la stessa cosa", "Il trucco a
// blocchi"): inside a chunk every term is a masked quadratic form over the chunk's tokens, and
// between chunks only two summaries travel -- the forward state entering each chunk (from the
// forward chunk-state and state-passing kernels) and the adjoint G carried into each chunk
// from the right, which the two kernels below pass backwards:
//
//   1. adj_state  S'_c[p, n] = sum_{t in c} exp(cs_t) dy_t[p] C_t[n]   (cs: inclusive cumsum)
//   2. adj_pass   R_last = dh_final; R_{c-1} = exp(cs_end(c)) R_c + S'_c, in place over S';
//                 d init = exp(cs_end(0)) R_0 + S'_0
//   3. chunk_bwd  per (batch, chunk, head): every per-token gradient of the chunk, and the
//                 head's contributions to dB, dC (to a scratch array) and to dA, dD (partials)
//   4. reduce     dB, dC summed over the heads of each group; dA, dD over batch and chunks
//
// Inside a chunk (tokens t, s, tau; L[tau, s] = exp(cs_tau - cs_s) for s <= tau; H the forward
// state entering the chunk, R the adjoint leaving it):
//   G_t B_t = sum_{tau >= t} L[tau, t] (C_tau . B_t) dy_tau + exp(cs_end - cs_t) R B_t
//   G_t^T x_t = sum_{tau >= t} L[tau, t] (x_t . dy_tau) C_tau + exp(cs_end - cs_t) R^T x_t
//   h_t^T dy_t = sum_{s <= t} L[t, s] dt_s (x_s . dy_t) B_s + exp(cs_t) H^T dy_t
// and <G_t, exp(a_t) h_{t-1}> = <G_t, h_t> - dt_t x_t^T G_t B_t with
//   <G_t, h_t> = sum_{s <= t <= tau} K[tau, s] + sum_{tau >= t} w_tau + sum_{s <= t} v_s
//                + exp(cs_end) <R, H>,
//   K[tau, s] = L[tau, s] dt_s (x_s . dy_tau)(C_tau . B_s),  w_tau = exp(cs_tau) dy_tau . (H C_tau),
//   v_s = exp(cs_end - cs_s) dt_s x_s . (R B_s);
// the first sum moves from t - 1 to t by adding column t of K and removing row t - 1.  Every
// exponent is of a non-positive number.
#pragma once
#include "ssd_common.cuh"

namespace ssd {
namespace bwd {

constexpr int kQ = 64;         // tokens per chunk of the backward (the result does not depend on it)
constexpr int kBwdThreads = 512;  // chunk_bwd: two halves of 256 threads

// ---- 1. adjoint summaries: grid (nchunks, batch * nheads), block 256 ------------------------
// S'_c[p, n] = sum_{t in c} exp(cs_t) dy_t[p] C_t[n], stored [b][c][h][p][n] (outer_sum).
template <typename T>
__global__ void __launch_bounds__(kOuterThreads) adj_state_kernel(
    const float* __restrict__ dy, const T* __restrict__ Cm, const float* __restrict__ cs,
    float* __restrict__ adj, int64_t seqlen, int nheads, int headdim, int dstate, int ngroups,
    int nchunks) {
  extern __shared__ float sm[];
  const int P4 = round4(headdim), N4 = round4(dstate), TS = outer_ts(headdim, dstate);
  float* us = sm;                    // [TS][P4]  exp(cs_t) dy_t
  float* vs = sm + TS * P4;          // [TS][N4]  C_t
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / (nheads / ngroups);
  const float* csb = cs + (bh * nchunks + c) * kQ;
  const int64_t t0 = int64_t(c) * kQ;
  float* out = adj + ((b * nchunks + c) * nheads + h) * int64_t(headdim) * dstate;
  const bool vy = vec4_ok(dy, headdim), vc = vec4_ok(Cm, dstate);
  auto stage = [&](int s0, int ts, float* u, float* v) {  // four columns per step
    const int gp = P4 / 4, gn = N4 / 4;
    for (int i = threadIdx.x; i < ts * gp; i += kOuterThreads) {
      const int s = i / gp, p = (i % gp) * 4;
      const int64_t tok = t0 + s0 + s;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (tok < seqlen) {
        const float w = expf(csb[s0 + s]);
        load4_row(dy, ((b * seqlen + tok) * nheads + h) * headdim + p, p, headdim, vy, e);
#pragma unroll
        for (int q = 0; q < 4; ++q) e[q] *= w;
      }
      *reinterpret_cast<float4*>(u + s * P4 + p) = make_float4(e[0], e[1], e[2], e[3]);
    }
    for (int i = threadIdx.x; i < ts * gn; i += kOuterThreads) {
      const int s = i / gn, n = (i % gn) * 4;
      const int64_t tok = t0 + s0 + s;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (tok < seqlen)
        load4_row(Cm, ((b * seqlen + tok) * ngroups + g) * dstate + n, n, dstate, vc, e);
      *reinterpret_cast<float4*>(v + s * N4 + n) = make_float4(e[0], e[1], e[2], e[3]);
    }
  };
  outer_sum(stage, kQ, headdim, dstate, out, us, vs);
}

// ---- 2. adjoint passing: one thread per state element, chunks last to first ------------------
// In: adj[c] = S'_c.  Out: adj[c] = R_c (the adjoint carried into chunk c from the right), and
// dinit = the gradient of the initial state.
__global__ void adj_pass_kernel(float* __restrict__ adj, const float* __restrict__ cs,
                                const float* dfinal, float* dinit, int64_t batch, int nheads,
                                int headdim, int dstate, int nchunks) {
  const int64_t per_bh = int64_t(headdim) * dstate;
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // over [b,h,p,n]
  if (e >= batch * nheads * per_bh) return;
  const int64_t bh = e / per_bh;
  const int64_t pn = e % per_bh;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  float run = dfinal ? dfinal[e] : 0.f;
  float* base = adj + (b * nchunks * nheads + h) * per_bh + pn;  // chunk c: + c * cstride
  const int64_t cstride = int64_t(nheads) * per_bh;
  const float* last = cs + bh * nchunks * kQ + kQ - 1;  // chunk c's last cumsum: + c * kQ
  // kBatch chunks' loads in flight at once, then the recurrence over them (last chunk first).
  // The loop counts chunks from the last one upwards: a count-down loop over the same chunks
  // took 4x the forward state pass's time under ncu, its loads not kept in flight together
  constexpr int kBatch = 8;
  for (int r0 = 0; r0 < nchunks; r0 += kBatch) {  // r: chunks counted from the last
    float sv[kBatch], lv[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int r = r0 + i;
      if (r < nchunks) {
        const int64_t c = nchunks - 1 - r;
        sv[i] = base[c * cstride];
        lv[i] = last[c * kQ];
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int r = r0 + i;
      if (r < nchunks) {
        const int64_t c = nchunks - 1 - r;
        base[c * cstride] = run;
        run = fmaf(expf(lv[i]), run, sv[i]);
      }
    }
  }
  if (dinit) dinit[e] = run;
}

// ---- 3. per-chunk gradients: grid (nchunks, batch * nheads), block 512 ------------------------
// Every product of the chunk is a small matrix product from shared memory, 4 x 4 outputs per
// thread and product (thread (a, b) = (i / 16, i % 16) of a half, i = tid % 256: rows
// 4a .. 4a+3, columns 4b .. 4b+3 of each 64-column pass) with float4 operand loads.  The two
// halves of the block take independent products: C.B / x.dy, the dx terms / H C, dB / dC.
// Shared memory (floats; rows of P4 or N4, the widths rounded up to multiples of 4):
//   x, dy [kQ][P4]; B, C [kQ][N4]; H, R [P4][N4] (as stored: [p][n]);
//   three [kQ][kQ] tables, first C.B, (x.dy)^T and L, then (in place) M[tau][t] =
//   L (C_tau . B_t), N2[tau][t] = L[tau][t] (x_t . dy_tau) and K2[t][s] = dt_s N2[t][s];
//   row and column partials of K; per-token scalars.
// x, B, H and R are read as four rows at a time by the lanes of a quarter-warp (the right-hand
// operand of the x.y^T-shaped products), rows 4 apart: their 16-byte groups are XOR-swizzled by
// bits of the row (swz), so those reads, and every other walk over them, hit distinct banks.
// Outputs: dx [b, t, h, p]; ddt [b, t, h]; the head's dB and dC rows into dbh, dch
// [b, t, h, n] (summed over the group by the reduce kernel); partial dA and dD per (b, c, h).
struct BwdSmem {
  static __host__ __device__ int px(int P) { return round4(P); }
  static __host__ __device__ int nx(int N) { return round4(N); }
  static __host__ __device__ size_t floats(int P, int N) {
    return size_t(kQ) * 2 * (px(P) + nx(N)) + 2 * size_t(round4(P)) * nx(N) +
           3 * size_t(kQ) * kQ + 2 * 16 * size_t(kQ) + 8 * kQ + 64;
  }
};
// The XOR swizzle of a row of `groups` 16-byte groups: the largest of 7, 3, 1, 0 that keeps the
// XOR inside the row.
__device__ __forceinline__ int swz_mask(int groups) {
  return groups % 8 == 0 ? 7 : (groups % 4 == 0 ? 3 : (groups % 2 == 0 ? 1 : 0));
}
// physical column of (row, col): the 16-byte group XOR (row / 4) & mask
__device__ __forceinline__ int swz(int row, int col, int mask) {
  return ((((col >> 2) ^ ((row >> 2) & mask))) << 2) | (col & 3);
}

// The products: am, bm are the operands' swizzle masks (0: plain rows).
// acc[i][j] += sum_{k0 <= k < k1} A[m0 + i][k] B[k][n0 + j]   (k0, k1, m0, n0 multiples of 4)
__device__ __forceinline__ void mm_nn(float (&acc)[4][4], const float* A, int sa, int am,
                                      const float* B, int sb, int bm, int m0, int n0, int k0,
                                      int k1) {
  for (int k = k0; k < k1; k += 4) {
    float4 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      a[i] = *reinterpret_cast<const float4*>(A + (m0 + i) * sa + swz(m0 + i, k, am));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 bv = *reinterpret_cast<const float4*>(B + (k + u) * sb + swz(k + u, n0, bm));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float av = u == 0 ? a[i].x : u == 1 ? a[i].y : u == 2 ? a[i].z : a[i].w;
        acc[i][0] = fmaf(av, bv.x, acc[i][0]);
        acc[i][1] = fmaf(av, bv.y, acc[i][1]);
        acc[i][2] = fmaf(av, bv.z, acc[i][2]);
        acc[i][3] = fmaf(av, bv.w, acc[i][3]);
      }
    }
  }
}
// acc[i][j] += sum_{k0 <= k < k1} A[k][m0 + i] B[k][n0 + j]
__device__ __forceinline__ void mm_tn(float (&acc)[4][4], const float* A, int sa, int am,
                                      const float* B, int sb, int bm, int m0, int n0, int k0,
                                      int k1) {
  for (int k = k0; k < k1; ++k) {
    const float4 av = *reinterpret_cast<const float4*>(A + k * sa + swz(k, m0, am));
    const float4 bv = *reinterpret_cast<const float4*>(B + k * sb + swz(k, n0, bm));
    const float aa[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i][0] = fmaf(aa[i], bv.x, acc[i][0]);
      acc[i][1] = fmaf(aa[i], bv.y, acc[i][1]);
      acc[i][2] = fmaf(aa[i], bv.z, acc[i][2]);
      acc[i][3] = fmaf(aa[i], bv.w, acc[i][3]);
    }
  }
}
// acc[i][j] += sum_{k0 <= k < k1} A[m0 + i][k] B[n0 + j][k]   (k0, k1 multiples of 4)
__device__ __forceinline__ void mm_nt(float (&acc)[4][4], const float* A, int sa, int am,
                                      const float* B, int sb, int bm, int m0, int n0, int k0,
                                      int k1) {
  for (int k = k0; k < k1; k += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = *reinterpret_cast<const float4*>(A + (m0 + i) * sa + swz(m0 + i, k, am));
      b[i] = *reinterpret_cast<const float4*>(B + (n0 + i) * sb + swz(n0 + i, k, bm));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = acc[i][j];
        v = fmaf(a[i].x, b[j].x, v);
        v = fmaf(a[i].y, b[j].y, v);
        v = fmaf(a[i].z, b[j].z, v);
        acc[i][j] = fmaf(a[i].w, b[j].w, v);
      }
  }
}
__device__ __forceinline__ void zero4x4(float (&acc)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads) chunk_bwd_kernel(
    const T* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
    const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ D,
    const float* __restrict__ dy, const float* __restrict__ cs,
    const float* __restrict__ hstates, const float* __restrict__ adj, float* __restrict__ dx,
    float* __restrict__ ddt, float* __restrict__ dbh, float* __restrict__ dch,
    float* __restrict__ dA_part, float* __restrict__ dD_part, int64_t seqlen, int nheads,
    int headdim, int dstate, int ngroups, int nchunks) {
  extern __shared__ float sm[];
  const int P = headdim, N = dstate, P4 = round4(P), N4 = round4(N);
  const int PX = BwdSmem::px(P), NX = BwdSmem::nx(N);
  float* xs = sm;                  // [kQ][PX]  x
  float* ys = xs + kQ * PX;        // [kQ][PX]  dy
  float* bs = ys + kQ * PX;        // [kQ][NX]  B
  float* cm = bs + kQ * NX;        // [kQ][NX]  C
  float* hs = cm + kQ * NX;        // [P4][NX]  H (forward state entering the chunk)
  float* rs = hs + P4 * NX;        // [P4][NX]  R (adjoint carried in from the right)
  float* T1 = rs + P4 * NX;        // [tau][s]  C_tau . B_s, then M
  float* T2 = T1 + kQ * kQ;        // [tau][s]  x_s . dy_tau, then K2 [t][s]
  float* T3 = T2 + kQ * kQ;        // [tau][s]  L, then N2
  float* rowP = T3 + kQ * kQ;      // [kQ][16]  partial row sums of K (by column tile)
  float* colP = rowP + 16 * kQ;    // [16][kQ]  partial column sums of K (by row tile)
  float* csv = colP + 16 * kQ;     // [kQ] cs
  float* dts = csv + kQ;           // [kQ] dt
  float* term1 = dts + kQ;         // [kQ] x_t . (G_t B_t)
  float* vv = term1 + kQ;          // [kQ] v_t
  float* ww = vv + kQ;             // [kQ] w_t
  float* rowK = ww + kQ;           // [kQ] sum_{s <= tau} K[tau, s]
  float* colK = rowK + kQ;         // [kQ] sum_{tau >= s} K[tau, s]
  float* dyx = colK + kQ;          // [kQ] dy_t . x_t
  float* red = dyx + kQ;           // [64] block reduction scratch

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = tid >> 8;                        // which half of the block
  const int ta = (tid & 255) >> 4, tb = tid & 15;  // this thread's row tile and column tile
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / (nheads / ngroups);
  const int64_t t0 = int64_t(c) * kQ;
  const int nvalid = int(seqlen - t0 < int64_t(kQ) ? seqlen - t0 : int64_t(kQ));
  const float Ah = A[h];
  const float Dh = D ? D[h] : 0.f;
  const float* csb = cs + (bh * nchunks + c) * kQ;
  const int mP = swz_mask(PX / 4), mN = swz_mask(NX / 4);  // swizzles of x and of B, H, R

  // ---- load the chunk (zeros in the padding and past the sequence's end) ----
  for (int i = tid; i < kQ * PX; i += kBwdThreads) {
    const int t = i / PX, p = i % PX;
    const bool in = t < nvalid && p < P;
    const int64_t off = ((b * seqlen + t0 + t) * nheads + h) * P + p;
    xs[t * PX + swz(t, p, mP)] = in ? io_traits<T>::load(x, off) : 0.f;
    ys[i] = in ? dy[off] : 0.f;
  }
  for (int i = tid; i < kQ * NX; i += kBwdThreads) {
    const int t = i / NX, n = i % NX;
    const bool in = t < nvalid && n < N;
    const int64_t off = ((b * seqlen + t0 + t) * ngroups + g) * N + n;
    bs[t * NX + swz(t, n, mN)] = in ? io_traits<T>::load(Bm, off) : 0.f;
    cm[i] = in ? io_traits<T>::load(Cm, off) : 0.f;
  }
  {
    const float* hsrc = hstates + ((b * nchunks + c) * nheads + h) * int64_t(P) * N;
    const float* rsrc = adj + ((b * nchunks + c) * nheads + h) * int64_t(P) * N;
    for (int i = tid; i < P4 * NX; i += kBwdThreads) {  // global [p][n] -> shared [p][n]
      const int p = i / NX, n = i % NX;
      const bool in = p < P && n < N;
      const int o = p * NX + swz(p, n, mN);
      hs[o] = in ? hsrc[int64_t(p) * N + n] : 0.f;
      rs[o] = in ? rsrc[int64_t(p) * N + n] : 0.f;
    }
  }
  for (int t = tid; t < kQ; t += kBwdThreads) {
    csv[t] = csb[t];
    dts[t] = t < nvalid ? dt[(b * seqlen + t0 + t) * nheads + h] : 0.f;
  }
  __syncthreads();
  const float cs_end = csv[kQ - 1];

  // ---- the chunk's quadratic tables: C.B, (x.dy)^T and L (4 x 4 per thread) ----
  {
    float acc[4][4];
    zero4x4(acc);
    if (half == 0) mm_nt(acc, cm, NX, 0, bs, NX, mN, 4 * ta, 4 * tb, 0, N4);  // C.B [tau][s]
    else mm_nt(acc, ys, PX, 0, xs, PX, mP, 4 * ta, 4 * tb, 0, P4);  // x_s . dy_tau [tau][s]
    float* dst = half == 0 ? T1 : T2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * ta + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = 4 * tb + j;
        dst[r * kQ + q] = acc[i][j];
        if (half == 0) T3[r * kQ + q] = q <= r ? expf(csv[r] - csv[q]) : 0.f;
      }
    }
  }
  __syncthreads();
  // ---- M, N2, K2 in place; the row and column sums of K = K2 (C.B), in a fixed order ----
  {
    float mv[4][4], n2[4][4], k2[4][4];
    if (half == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tau = 4 * ta + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = 4 * tb + j;
        const float lv = T3[tau * kQ + s], cbv = T1[tau * kQ + s];
        mv[i][j] = lv * cbv;
        n2[i][j] = lv * T2[tau * kQ + s];
        k2[i][j] = dts[s] * n2[i][j];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float rsum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) rsum = fmaf(k2[i][j], T1[(4 * ta + i) * kQ + 4 * tb + j], rsum);
      rowP[(4 * ta + i) * 16 + tb] = rsum;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float csum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) csum = fmaf(k2[i][j], T1[(4 * ta + i) * kQ + 4 * tb + j], csum);
      colP[ta * kQ + 4 * tb + j] = csum;
    }
    }
    __syncthreads();
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int o = (4 * ta + i) * kQ + 4 * tb + j;
          T1[o] = mv[i][j];
          T2[o] = k2[i][j];
          T3[o] = n2[i][j];
        }
    }
  }
  for (int i = tid; i < 2 * kQ; i += kBwdThreads) {
    const int r = i % kQ;
    float sum = 0.f;
    if (i < kQ) {
      for (int k = 0; k < 16; ++k) sum += rowP[r * 16 + k];
      rowK[r] = sum;
    } else {
      for (int k = 0; k < 16; ++k) sum += colP[k * kQ + r];
      colK[r] = sum;
    }
  }
  __syncthreads();

  // ---- per token t (rows 4ta..), p (columns).  Half 0: q = sum_tau M[tau][t] dy_tau +
  //      er_t R B_t, dx, and the per-token sums x.q, x.(R B), dy.x; half 1: dy.(H C) ----
  {
    float s1[4] = {0.f, 0.f, 0.f, 0.f}, sv[4] = {0.f, 0.f, 0.f, 0.f};
    float sw[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < P4; c0 += 64) {
      const int p0 = c0 + 4 * tb;
      if (p0 >= P4) continue;
      if (half == 0) {
        float q[4][4], rb[4][4];
        zero4x4(q);
        zero4x4(rb);
        mm_tn(q, T1, kQ, 0, ys, PX, 0, 4 * ta, p0, 4 * ta, kQ);
        mm_nt(rb, bs, NX, mN, rs, NX, mN, 4 * ta, p0, 0, N4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 4 * ta + i;
          const float er = expf(cs_end - csv[t]);
          float o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float qv = fmaf(er, rb[i][j], q[i][j]);
            const float xv = xs[t * PX + swz(t, p0 + j, mP)], yv = ys[t * PX + p0 + j];
            o[j] = fmaf(dts[t], qv, Dh * yv);
            s1[i] = fmaf(xv, qv, s1[i]);
            sv[i] = fmaf(xv, rb[i][j], sv[i]);
            sd[i] = fmaf(yv, xv, sd[i]);
          }
          if (t < nvalid) {
            float* dst = dx + ((b * seqlen + t0 + t) * nheads + h) * P + p0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (p0 + j < P) dst[j] = o[j];
          }
        }
      } else {
        float hc[4][4];
        zero4x4(hc);
        mm_nt(hc, cm, NX, 0, hs, NX, mN, 4 * ta, p0, 0, N4);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) sw[i] = fmaf(ys[(4 * ta + i) * PX + p0 + j], hc[i][j], sw[i]);
      }
    }
    // sum over the 16 column tiles (lanes tb = 0..15 of this half-warp), in a fixed order
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {
        s1[i] += __shfl_xor_sync(0xffffffffu, s1[i], off);
        sv[i] += __shfl_xor_sync(0xffffffffu, sv[i], off);
        sw[i] += __shfl_xor_sync(0xffffffffu, sw[i], off);
        sd[i] += __shfl_xor_sync(0xffffffffu, sd[i], off);
      }
      if (tb == 0) {
        const int t = 4 * ta + i;
        if (half == 0) {
          term1[t] = s1[i];
          vv[t] = expf(cs_end - csv[t]) * dts[t] * sv[i];
          dyx[t] = sd[i];
        } else {
          ww[t] = expf(csv[t]) * sw[i];
        }
      }
    }
  }

  // ---- per (t, n): this head's dB_t = dt_t (er_t R^T x_t + sum_tau N2[tau][t] C_tau) (half 0)
  //      and dC_t = exp(cs_t) H^T dy_t + sum_s K2[t][s] B_s (half 1) ----
  for (int c0 = 0; c0 < N4; c0 += 64) {
    const int n0 = c0 + 4 * tb;
    if (n0 >= N4) continue;
    if (half == 0) {
      float sb[4][4], xr[4][4];
      zero4x4(sb);
      zero4x4(xr);
      mm_tn(sb, T3, kQ, 0, cm, NX, 0, 4 * ta, n0, 4 * ta, kQ);
      mm_nn(xr, xs, PX, mP, rs, NX, mN, 4 * ta, n0, 0, P4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * ta + i;
        if (t >= nvalid) continue;
        const float er = expf(cs_end - csv[t]);
        float* dst = dbh + ((b * seqlen + t0 + t) * nheads + h) * N + n0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (n0 + j < N) dst[j] = dts[t] * fmaf(er, xr[i][j], sb[i][j]);
      }
    } else {
      float sc[4][4], yh[4][4];
      zero4x4(sc);
      zero4x4(yh);
      mm_nn(sc, T2, kQ, 0, bs, NX, mN, 4 * ta, n0, 0, 4 * ta + 4);
      mm_nn(yh, ys, PX, 0, hs, NX, mN, 4 * ta, n0, 0, P4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * ta + i;
        if (t >= nvalid) continue;
        const float et = expf(csv[t]);
        float* dst = dch + ((b * seqlen + t0 + t) * nheads + h) * N + n0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (n0 + j < N) dst[j] = fmaf(et, yh[i][j], sc[i][j]);
      }
    }
  }
  // exp(cs_end) <R, H> (R and H share one layout)
  float rh = 0.f;
  for (int i = tid; i < P4 * NX; i += kBwdThreads) rh = fmaf(rs[i], hs[i], rh);
  rh = warp_sum(rh);
  if (lane == 0) red[warp] = rh;
  __syncthreads();
  // ---- one warp: the per-token sums, ddt, and this chunk's dA and dD partials ----
  if (warp == 0) {
    float rht = 0.f;
    for (int w = 0; w < kBwdThreads / 32; ++w) rht += red[w];
    const float cst = expf(cs_end) * rht;
    // S_t = S_{t-1} + colK[t] - rowK[t-1]; W_t = sum_{tau >= t} w; V_t = sum_{s <= t} v.  Lane l
    // takes tokens 2l, 2l+1; the running sums are warp scans.
    float ga[2];
    float tot_w = 0.f;
    for (int tau = 0; tau < kQ; ++tau) tot_w += ww[tau];
    float loc_S[2], loc_V[2], loc_W[2];
    for (int r = 0; r < 2; ++r) {
      const int t = 2 * lane + r;
      loc_S[r] = colK[t] - (t > 0 ? rowK[t - 1] : 0.f);
      loc_V[r] = vv[t];
      loc_W[r] = ww[t];
    }
    const float sS = warp_inclusive_scan(loc_S[0] + loc_S[1]);
    const float sV = warp_inclusive_scan(loc_V[0] + loc_V[1]);
    const float sW = warp_inclusive_scan(loc_W[0] + loc_W[1]);
    const float pS = sS - loc_S[0] - loc_S[1], pV = sV - loc_V[0] - loc_V[1];
    const float pW = sW - loc_W[0] - loc_W[1];  // sum of w before token 2 lane
    float dA_acc = 0.f, dD_acc = 0.f;
    for (int r = 0; r < 2; ++r) {
      const int t = 2 * lane + r;
      const float S = pS + loc_S[0] + (r ? loc_S[1] : 0.f);
      const float V = pV + loc_V[0] + (r ? loc_V[1] : 0.f);
      const float Wsuf = tot_w - pW - (r ? loc_W[0] : 0.f);
      const float gh = S + V + Wsuf + cst;  // <G_t, h_t>
      ga[r] = gh - dts[t] * term1[t];       // <G_t, exp(a_t) h_{t-1}>
      if (t < nvalid) {
        ddt[(b * seqlen + t0 + t) * nheads + h] = fmaf(Ah, ga[r], term1[t]);
        dA_acc = fmaf(dts[t], ga[r], dA_acc);
        dD_acc += dyx[t];
      }
    }
    dA_acc = warp_sum(dA_acc);
    dD_acc = warp_sum(dD_acc);
    if (lane == 0) {
      dA_part[(b * nchunks + c) * nheads + h] = dA_acc;
      dD_part[(b * nchunks + c) * nheads + h] = dD_acc;
    }
  }
}

// ---- 4. reductions ------------------------------------------------------------------------
// dB[b, t, g, n] = sum over the heads of group g of dbh[b, t, h, n] (same for dC), in head
// order (deterministic).  One thread per output element.
template <typename TG>
__global__ void group_sum_kernel(const float* __restrict__ dbh, const float* __restrict__ dch,
                                 TG* __restrict__ dB, TG* __restrict__ dC, int64_t ntok,
                                 int nheads, int ngroups, int dstate) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // over [tok, g, n]
  if (e >= ntok * ngroups * dstate) return;
  const int n = int(e % dstate);
  const int64_t tg = e / dstate;
  const int g = int(tg % ngroups);
  const int64_t tok = tg / ngroups;
  const int hpg = nheads / ngroups;
  float sb = 0.f, sc = 0.f;
  for (int k = 0; k < hpg; ++k) {
    const int64_t off = (tok * nheads + g * hpg + k) * dstate + n;
    sb += dbh[off];
    sc += dch[off];
  }
  io_traits<TG>::store(dB, e, sb);
  io_traits<TG>::store(dC, e, sc);
}

// dA[h] = sum over (b, c) of dA_part; dD[h] likewise (fixed order).  One thread per head.
__global__ void head_sum_kernel(const float* __restrict__ dA_part,
                                const float* __restrict__ dD_part, float* __restrict__ dA,
                                float* __restrict__ dD, int64_t nbc, int nheads) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= nheads) return;
  float sa = 0.f, sd = 0.f;
  for (int64_t i = 0; i < nbc; ++i) {
    sa += dA_part[i * nheads + h];
    sd += dD_part[i * nheads + h];
  }
  dA[h] = sa;
  if (dD) dD[h] = sd;
}

}  // namespace bwd
}  // namespace ssd
