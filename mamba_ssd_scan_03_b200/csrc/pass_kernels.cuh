// pass_kernels.cuh -- helpers of the sequence-sliced scan: the total log-decay of a slice and
// the state passing between slices.
//
// A slice of the sequence is summarised by (total decay, state from a zero start): its
// steps compose like one step, h_out = exp(sum dt A) h_in + S ("State Space Model"
// (book.paithon.it), "Un sistema che riassume il passato": the steps fuse pairwise by
// associativity).  The state entering slice r is then an exclusive scan over the slices before
// it, which is what lets slices of one sequence run on different GPUs and exchange only these
// summaries ("Architektury Mamba-2, State Space Models i liniowa atencja" (tech.tersel.eu),
// "Wyzwania uczenia rozproszonego": only boundary states cross between devices).
#pragma once
#include "ssd_common.cuh"

namespace ssd {
namespace pass {

// total_decay[b, h] = A[h] * sum_t dt[b, t, h].  grid (batch, ceil(nheads / 32)), block 256:
// lane = head within a 32-head tile, warp w sums tokens w, w + 8, ...; the eight partial sums
// are added in a fixed order (deterministic).
__global__ void __launch_bounds__(256) decay_sum_kernel(const float* __restrict__ dt,
                                                        const float* __restrict__ A,
                                                        float* __restrict__ total_decay,
                                                        int64_t seqlen, int nheads) {
  __shared__ float part[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.x;
  const int h = blockIdx.y * 32 + lane;
  float s = 0.f;
  if (h < nheads) {
    const float* p = dt + b * seqlen * nheads + h;
    for (int64_t t = warp; t < seqlen; t += 8) s += p[t * nheads];
  }
  part[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && h < nheads) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += part[w][lane];
    total_decay[b * nheads + h] = A[h] * tot;
  }
}

// states [nslice][batch][nheads][P][N]: in, each slice's state from a zero start; out, the
// state entering each slice.  decay [nslice][batch][nheads] (natural log).  One thread per
// element of a [batch][nheads][P][N] state: H_in(0) = init (or 0), H_in(r + 1) =
// exp(decay(r)) H_in(r) + S(r); final = H_in(nslice).  Four slices' loads in flight.
__global__ void __launch_bounds__(256) slice_pass_kernel(float* __restrict__ states,
                                                         const float* __restrict__ decay,
                                                         const float* init_state,
                                                         float* final_state, int64_t nslice,
                                                         int64_t nbh, int64_t per_bh) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = nbh * per_bh;
  if (e >= n) return;
  const int64_t bh = e / per_bh;
  float run = init_state ? init_state[e] : 0.f;
  for (int64_t r0 = 0; r0 < nslice; r0 += 4) {
    float v[4], a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (r0 + i < nslice) {
        v[i] = states[(r0 + i) * n + e];
        a[i] = expf(decay[(r0 + i) * nbh + bh]);
      }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (r0 + i < nslice) {
        states[(r0 + i) * n + e] = run;
        run = fmaf(a[i], run, v[i]);
      }
  }
  if (final_state) final_state[e] = run;
}

}  // namespace pass
}  // namespace ssd
