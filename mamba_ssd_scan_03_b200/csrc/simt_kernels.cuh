// simt_kernels.cuh -- the chunked scan on float32 CUDA cores (any supported shape, f32 or
// bf16 io).  Four kernels, in stream order:
//
//   1. cumsum      cs[b,h,c,t] = sum_{k=cQ..cQ+t} dt_k A_h            (within-chunk log-decay)
//   2. chunk_state S_c[n,p]   = sum_{s in c} exp(cs_end - cs_s) dt_s B_s[n] x_s[p]
//   3. state_pass  H_0 = init;  H_{c+1} = exp(cs_end(c)) H_c + S_c      (S_c replaced by H_c)
//   4. chunk_out   y_t = sum_{s<=t, s in c} exp(cs_t - cs_s) dt_s (C_t.B_s) x_s
//                        + exp(cs_t) C_t^T H_c + D x_t
//
// This is the blocked algorithm of "Mamba-2 (2024): SSM e attention sono la stessa cosa"
// (paithon.it), section "Il trucco a blocchi": the quadratic (attention-like) form inside
// each block, and only the summary state passed between blocks.  The block length is the
// caller's chunk.  Float32 throughout (the float32 workload's tolerance, 1e-4 of RMS(y),
// rules out TF32 tensor cores).
#pragma once
#include "ssd_common.cuh"

namespace ssd {
namespace simt {

// ---- 1. cumsum: grid (nchunks, batch*nheads), block = chunk threads ------------------------
__global__ void cumsum_kernel(const float* __restrict__ dt, const float* __restrict__ A,
                              float* __restrict__ cs, int64_t seqlen, int nheads, int chunk,
                              int nchunks) {
  __shared__ float warp_tot[8];
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int t = threadIdx.x;
  const int64_t tok = int64_t(c) * chunk + t;
  float a = tok < seqlen ? dt[(b * seqlen + tok) * nheads + h] * A[h] : 0.0f;
  float v = warp_inclusive_scan(a);
  const int warp = t >> 5, lane = t & 31;
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  float off = 0.0f;
  for (int w = 0; w < warp; ++w) off += warp_tot[w];
  cs[(bh * nchunks + c) * chunk + t] = v + off;
}

// ---- 2. chunk states: grid (nchunks, batch*nheads), block 256 --------------------------------
// S_c[p, n] stored [b][c][h][p][n]: the outer-product sum of (w_s x_s) and B_s over the chunk,
// 4 x 4 outputs per thread (outer_sum).
template <typename T>
__global__ void __launch_bounds__(kOuterThreads) chunk_state_kernel(
    const T* __restrict__ x, const float* __restrict__ dt, const T* __restrict__ Bm,
    const float* __restrict__ cs, float* __restrict__ states, int64_t seqlen, int nheads,
    int headdim, int dstate, int ngroups, int chunk, int nchunks) {
  extern __shared__ float sm[];
  const int P4 = round4(headdim), N4 = round4(dstate), TS = outer_ts(headdim, dstate);
  float* us = sm;                    // [TS][P4]  w_s x_s
  float* vs = sm + TS * P4;          // [TS][N4]  B_s
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / (nheads / ngroups);
  const float* csb = cs + (bh * nchunks + c) * chunk;
  const float cs_end = csb[chunk - 1];
  const int64_t t0 = int64_t(c) * chunk;
  float* out = states + ((b * nchunks + c) * nheads + h) * int64_t(headdim) * dstate;
  const bool vx = vec4_ok(x, headdim), vb = vec4_ok(Bm, dstate);
  auto stage = [&](int s0, int ts, float* u, float* v) {  // four columns per step
    const int gp = P4 / 4, gn = N4 / 4;
    for (int i = threadIdx.x; i < ts * gp; i += kOuterThreads) {
      const int s = i / gp, p = (i % gp) * 4;
      const int64_t tok = t0 + s0 + s;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (s0 + s < chunk && tok < seqlen) {
        const float w = expf(cs_end - csb[s0 + s]) * dt[(b * seqlen + tok) * nheads + h];
        load4_row(x, ((b * seqlen + tok) * nheads + h) * headdim + p, p, headdim, vx, e);
#pragma unroll
        for (int q = 0; q < 4; ++q) e[q] *= w;
      }
      *reinterpret_cast<float4*>(u + s * P4 + p) = make_float4(e[0], e[1], e[2], e[3]);
    }
    for (int i = threadIdx.x; i < ts * gn; i += kOuterThreads) {
      const int s = i / gn, n = (i % gn) * 4;
      const int64_t tok = t0 + s0 + s;
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      if (s0 + s < chunk && tok < seqlen)
        load4_row(Bm, ((b * seqlen + tok) * ngroups + g) * dstate + n, n, dstate, vb, e);
      *reinterpret_cast<float4*>(v + s * N4 + n) = make_float4(e[0], e[1], e[2], e[3]);
    }
  };
  outer_sum(stage, chunk, headdim, dstate, out, us, vs);
}

// ---- 3. state passing: one thread per state element, sequential over chunks -------------------
__global__ void state_pass_kernel(float* __restrict__ states, const float* __restrict__ cs,
                                  const float* init_state, float* final_state, int64_t batch,
                                  int nheads, int headdim, int dstate, int chunk,
                                  int nchunks) {
  const int64_t per_bh = int64_t(headdim) * dstate;
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // over [b,h,p,n]
  if (e >= batch * nheads * per_bh) return;
  const int64_t bh = e / per_bh;
  const int64_t pn = e % per_bh;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  float run = init_state ? init_state[e] : 0.0f;
  float* base = states + (b * nchunks * nheads + h) * per_bh + pn;  // chunk c: + c * cstride
  const int64_t cstride = int64_t(nheads) * per_bh;
  const float* last = cs + bh * nchunks * chunk + chunk - 1;  // chunk c's last cumsum: + c * chunk
  // kBatch chunks' loads in flight at once (they do not depend on the running state), then the
  // recurrence over them in order
  constexpr int kBatch = 8;
  for (int c0 = 0; c0 < nchunks; c0 += kBatch) {
    float sv[kBatch], lv[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t c = c0 + i;
      if (c < nchunks) {
        sv[i] = base[c * cstride];
        lv[i] = last[c * chunk];
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t c = c0 + i;
      if (c < nchunks) {
        base[c * cstride] = run;
        run = fmaf(expf(lv[i]), run, sv[i]);
      }
    }
  }
  if (final_state) final_state[e] = run;
}

// ---- 4. outputs: grid (nchunks, batch*nheads), block 256 -------------------------------------
template <typename T, typename TY>
__global__ void __launch_bounds__(256) chunk_out_kernel(
    const T* __restrict__ x, const float* __restrict__ dt, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ D, const float* __restrict__ cs,
    const float* __restrict__ states, TY* __restrict__ y, int64_t seqlen, int nheads,
    int headdim, int dstate, int ngroups, int chunk, int nchunks) {
  constexpr int TT = 32;  // token tile (rows t and columns s)
  constexpr int NC = 32;  // state slice
  constexpr int MAXO = 32;  // outputs per thread: TT * headdim / 256 (headdim <= 256)
  extern __shared__ float sm[];
  float* cst = sm;                    // [TT][NC]   C slice, rows t
  float* bst = cst + TT * NC;         // [TT][NC]   B slice, rows s
  float* mt = bst + TT * NC;          // [TT][TT]   masked C.B tile
  float* xt = mt + TT * TT;           // [TT][headdim]
  float* ht = xt + TT * headdim;      // [headdim][NC]  entering-state slice
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = int(bh % nheads);
  const int64_t b = bh / nheads;
  const int g = h / (nheads / ngroups);
  const float* csb = cs + (bh * nchunks + c) * chunk;
  const float* Hc = states + ((b * nchunks + c) * nheads + h) * int64_t(headdim) * dstate;
  const int64_t c0 = int64_t(c) * chunk;
  const float dh = D ? D[h] : 0.0f;
  const int nout = TT * headdim;
  for (int tt = 0; tt < chunk; tt += TT) {
    if (c0 + tt >= seqlen) break;
    float acc[MAXO];
#pragma unroll
    for (int i = 0; i < MAXO; ++i) acc[i] = 0.0f;
    // off-diagonal: exp(cs_t) * C_t^T H_c, accumulated over state slices
    for (int n0 = 0; n0 < dstate; n0 += NC) {
      __syncthreads();
      for (int i = threadIdx.x; i < TT * NC; i += 256) {
        const int r = i / NC, n = n0 + i % NC;
        const int64_t tok = c0 + tt + r;
        cst[i] = (tok < seqlen && n < dstate)
                     ? io_traits<T>::load(Cm, ((b * seqlen + tok) * ngroups + g) * dstate + n)
                     : 0.0f;
      }
      for (int i = threadIdx.x; i < headdim * NC; i += 256) {
        const int p = i / NC, n = n0 + i % NC;
        ht[i] = n < dstate ? Hc[int64_t(p) * dstate + n] : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < MAXO; ++i) {
        const int o = i * 256 + threadIdx.x;  // o = r * headdim + p
        if (o < nout) {
          const int r = o / headdim, p = o % headdim;
          float a = acc[i];
          for (int n = 0; n < NC; ++n) a = fmaf(cst[r * NC + n], ht[p * NC + n], a);
          acc[i] = a;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < MAXO; ++i) {
      const int o = i * 256 + threadIdx.x;
      if (o < nout) acc[i] *= expf(csb[tt + o / headdim]);
    }
    // diagonal: masked quadratic form over s-tiles up to and including this t-tile
    for (int ss = 0; ss <= tt; ss += TT) {
      float cb[4] = {0.f, 0.f, 0.f, 0.f};  // this thread's 4 entries of the TT x TT tile
      for (int n0 = 0; n0 < dstate; n0 += NC) {
        __syncthreads();
        for (int i = threadIdx.x; i < TT * NC; i += 256) {
          const int r = i / NC, n = n0 + i % NC;
          const int64_t tt_tok = c0 + tt + r, ss_tok = c0 + ss + r;
          cst[i] = (tt_tok < seqlen && n < dstate)
                       ? io_traits<T>::load(Cm, ((b * seqlen + tt_tok) * ngroups + g) * dstate + n)
                       : 0.0f;
          bst[i] = (ss_tok < seqlen && n < dstate)
                       ? io_traits<T>::load(Bm, ((b * seqlen + ss_tok) * ngroups + g) * dstate + n)
                       : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = k * 256 + threadIdx.x;  // e = r * TT + s
          const int r = e / TT, s = e % TT;
          float a = cb[k];
          for (int n = 0; n < NC; ++n) a = fmaf(cst[r * NC + n], bst[s * NC + n], a);
          cb[k] = a;
        }
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = k * 256 + threadIdx.x;
        const int r = e / TT, s = e % TT;
        const int ti = tt + r, si = ss + s;
        const int64_t stok = c0 + si;
        float m = 0.0f;
        if (si <= ti && stok < seqlen)
          m = cb[k] * expf(csb[ti] - csb[si]) * dt[(b * seqlen + stok) * nheads + h];
        mt[e] = m;
      }
      for (int i = threadIdx.x; i < TT * headdim; i += 256) {
        const int s = i / headdim, p = i % headdim;
        const int64_t tok = c0 + ss + s;
        xt[i] = tok < seqlen
                    ? io_traits<T>::load(x, ((b * seqlen + tok) * nheads + h) * headdim + p)
                    : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < MAXO; ++i) {
        const int o = i * 256 + threadIdx.x;
        if (o < nout) {
          const int r = o / headdim, p = o % headdim;
          float a = acc[i];
          for (int s = 0; s < TT; ++s) a = fmaf(mt[r * TT + s], xt[s * headdim + p], a);
          acc[i] = a;
        }
      }
    }
    // skip term and store
#pragma unroll
    for (int i = 0; i < MAXO; ++i) {
      const int o = i * 256 + threadIdx.x;
      if (o < nout) {
        const int r = o / headdim, p = o % headdim;
        const int64_t tok = c0 + tt + r;
        if (tok < seqlen) {
          const int64_t xi = ((b * seqlen + tok) * nheads + h) * headdim + p;
          io_traits<TY>::store(y, xi, acc[i] + dh * io_traits<T>::load(x, xi));
        }
      }
    }
  }
}

}  // namespace simt
}  // namespace ssd
