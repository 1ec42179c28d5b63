// ssd_lib.cu -- the C ABI of libssd.so (declared in include/ssd.h): argument validation, path
// selection, workspace carving, TMA descriptor set-up and the stream-ordered launches.
// Single translation unit: the kernels live in the headers included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "bwd_kernels.cuh"
#include "glue_kernels.cuh"
#include "pass_kernels.cuh"
#include "selective_kernels.cuh"
#include "simt_kernels.cuh"
#include "ssd_common.cuh"
#include "step_kernels.cuh"
#include "tc_kernels.cuh"

namespace {

using ssd::tc::Seg;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool is_device_ptr(const void* p) {
  if (!p) return false;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
  int64_t batch, seqlen;
  int nheads, headdim, dstate, ngroups, chunk;
  ssd_dtype io;
};

ssd_status check_shape(const Shape& s) {
  if (s.batch <= 0 || s.seqlen <= 0 || s.nheads <= 0 || s.headdim <= 0 || s.dstate <= 0 ||
      s.ngroups <= 0)
    return SSD_ERR_INVALID_ARG;
  if (s.nheads % s.ngroups != 0) return SSD_ERR_INVALID_ARG;
  if (s.chunk != 64 && s.chunk != 128 && s.chunk != 256) return SSD_ERR_INVALID_ARG;
  if (s.io != SSD_F32 && s.io != SSD_BF16) return SSD_ERR_INVALID_ARG;
  return SSD_OK;
}

bool simt_supported(const Shape& s) {
  return s.headdim <= 256 && s.dstate <= 2048 && s.batch * s.nheads <= 65535 &&
         (s.seqlen + s.chunk - 1) / s.chunk <= (int64_t(1) << 30);
}

bool tc_shape_ok(const Shape& s) {
  const int hpg = s.nheads / s.ngroups;
  return s.io == SSD_BF16 && s.headdim == 64 && s.dstate == 128 && (hpg % 2) == 0 &&
         s.seqlen <= (int64_t(1) << 30) && s.batch <= (int64_t(1) << 20);
}

// Streaming multiprocessors of the current device (148 on a B200; also the answer when no
// device can be queried, so that workspace queries work on a host without a GPU).
int sm_count() {
  constexpr int kMaxDev = 256;
  static std::mutex mu;
  static int cache[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return 148;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

// Segments of the summary-only pass (ssd_chunk_state_fwd): enough (batch, segment, head pair)
// units to give every SM about eight.
Seg tc_segments(const Shape& s) {
  Seg sg;
  sg.nblk = int((s.seqlen + ssd::tc::kBlk - 1) / ssd::tc::kBlk);
  const int64_t pairs = s.batch * (s.nheads / 2);
  const int64_t target = 8 * int64_t(sm_count());
  int nseg = int(std::min<int64_t>(sg.nblk, std::max<int64_t>(1, (target + pairs - 1) / pairs)));
  sg.seg_blks = (sg.nblk + nseg - 1) / nseg;
  sg.nseg = (sg.nblk + sg.seg_blks - 1) / sg.seg_blks;
  sg.useg = sg.nseg;
  return sg;
}

// Tensor-core path scratch: segment states [b, seg, h, 64, 128] f32 | segment log2-decays
// [b, seg, h] f32.
struct SegScratch {
  float* states;
  float* decay;
};
size_t seg_scratch_bytes(const Shape& s, const Seg& sg) {
  return align256(size_t(s.batch) * sg.nseg * s.nheads * 64 * 128 * sizeof(float)) +
         align256(size_t(s.batch) * sg.nseg * s.nheads * sizeof(float));
}
SegScratch seg_scratch(const Shape& s, const Seg& sg, void* base) {
  char* p = static_cast<char*>(base);
  SegScratch r;
  r.states = reinterpret_cast<float*>(p);
  p += align256(size_t(s.batch) * sg.nseg * s.nheads * 64 * 128 * sizeof(float));
  r.decay = reinterpret_cast<float*>(p);
  return r;
}

// Options of the scan entry points (the defaults, all zero, are what ssd_chunk_scan_fwd uses).
struct ScanOpts {
  int max_ctas = 0;        // cap on the walk's CTAs (0: one per SM)
  int plan = 0;            // 0 automatic, 1 whole sequences, 2 segments with summaries
  int64_t wait_ns = 0;     // limit of every bounded wait in the walk (0: 2 s; -1: no waiting)
};

// The walk of ssd_chunk_scan_fwd on the tensor cores.  Whole sequences (no summary pass) when
// there are about as many (batch row, head pair) sequences as CTAs; otherwise each sequence is
// cut into segments whose entering states seg_state + seg_pass provide, so that the CTAs share
// the work evenly.
struct TcPlan {
  ssd::tc::WalkPlan w;
  Seg sg;  // sg.nseg > 1: seg_state over the first nseg - 1 segments and seg_pass run first
};
bool make_tc_plan(const Shape& s, const ScanOpts& o, TcPlan* out) {
  const int nsm = sm_count();
  const int cap = o.max_ctas > 0 ? std::min(nsm, o.max_ctas) : nsm;
  const int64_t nblk = (s.seqlen + ssd::tc::kBlk - 1) / ssd::tc::kBlk;
  const int64_t npair = s.nheads / 2, nseqs = s.batch * npair;
  if (nblk > (int64_t(1) << 30) || nseqs * nblk > (int64_t(1) << 40)) return false;
  // Whole sequences (one launch: a CTA walks max(nblk, total / cap) blocks) unless the segment
  // plan finishes sooner: its walk spreads total / cap blocks over every CTA, but its two
  // summary kernels cost about kSegOverheadBlocks blocks' time (measured on the 130M-layer,
  // 4K x 80-head and 1M-token shapes on B200).
  constexpr int64_t kSegOverheadBlocks = 9;
  const int64_t share = (nseqs * nblk + cap - 1) / cap;
  const bool whole =
      nblk == 1 || o.plan == 1 || (o.plan == 0 && nblk <= share + kSegOverheadBlocks);
  int64_t nseg = whole ? 1 : std::min<int64_t>(nblk, std::max<int64_t>(2, (cap + nseqs - 1) / nseqs));
  const int64_t seg_blks = (nblk + nseg - 1) / nseg;
  nseg = (nblk + seg_blks - 1) / seg_blks;
  const int64_t total = nseqs * nblk;
  // every range at least one segment long (a range inside one segment would wait on a chain of
  // ranges) and at most kMaxItems - 2 segments long (its items fit the kernel's list)
  int64_t nct = std::min<int64_t>(cap, nseqs * nseg);
  const int64_t per = seg_blks * (ssd::tc::kMaxItems - 2);
  nct = std::max<int64_t>(nct, (total + per - 1) / per);
  while (nct > 1 && total / nct < seg_blks) --nct;
  if ((total + nct - 1) / nct > per || nct > (int64_t(1) << 20)) return false;
  TcPlan p;
  p.w.total = total;
  p.w.nblk = int(nblk);
  p.w.seg_blks = int(seg_blks);
  p.w.nseg = int(nseg);
  p.w.npair = int(npair);
  p.w.nct = int(nct);
  p.w.wait_ns = o.wait_ns > 0 ? uint64_t(o.wait_ns) : (o.wait_ns < 0 ? 0ull : 2000000000ull);
  p.sg.nblk = int(nblk);
  p.sg.seg_blks = int(seg_blks);
  p.sg.nseg = int(nseg);
  p.sg.useg = int(nseg) - 1;
  *out = p;
  return true;
}

// Workspace of the walk: [ticket + one ready flag per range] | [one published state per range,
// two heads] | (segments) [entering state per (batch, segment, head)] [log2-decay of each].
struct WalkScratch {
  unsigned* ticket;
  int* flags;
  float* slots;
  float* states;
  float* decay;
  size_t header_bytes;
};
size_t walk_bytes(const Shape& s, const TcPlan& p) {
  size_t n = align256(size_t(p.w.nct + 1) * 4) +
             align256(size_t(p.w.nct) * ssd::tc::kSlotFloats * sizeof(float));
  if (p.sg.nseg > 1) n += seg_scratch_bytes(s, p.sg);
  return n;
}
WalkScratch walk_scratch(const Shape& s, const TcPlan& p, void* base) {
  char* c = static_cast<char*>(base);
  WalkScratch w{};
  w.header_bytes = align256(size_t(p.w.nct + 1) * 4);
  w.ticket = reinterpret_cast<unsigned*>(c);
  w.flags = reinterpret_cast<int*>(c) + 1;
  c += w.header_bytes;
  w.slots = reinterpret_cast<float*>(c);
  c += align256(size_t(p.w.nct) * ssd::tc::kSlotFloats * sizeof(float));
  if (p.sg.nseg > 1) {
    const SegScratch sc = seg_scratch(s, p.sg, c);
    w.states = sc.states;
    w.decay = sc.decay;
  }
  return w;
}

// ssd_chunk_scan_fwd and ssd_chunk_state_fwd share one workspace query: the larger need.
size_t tc_workspace(const Shape& s, const ScanOpts& o = ScanOpts()) {
  TcPlan p;
  const size_t walk = make_tc_plan(s, o, &p) ? walk_bytes(s, p) : 0;
  return std::max(walk, seg_scratch_bytes(s, tc_segments(s)));
}

size_t simt_workspace(const Shape& s) {
  const int64_t nchunks = (s.seqlen + s.chunk - 1) / s.chunk;
  const size_t cs = size_t(s.batch) * s.nheads * nchunks * s.chunk * sizeof(float);
  const size_t states =
      size_t(s.batch) * nchunks * s.nheads * size_t(s.headdim) * s.dstate * sizeof(float);
  return align256(cs) + align256(states);
}

// ---- TMA descriptor encoding through the driver entry point (no link-time libcuda) ---------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 3-D view [outer][mid][inner] with a {128 bytes of inner, 128, 1} box and 128-byte swizzle:
// bf16 tiles of 64 elements, float32 tiles of 32.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
              bool f32 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * es, inner * mid * es};
  cuuint32_t box[3] = {f32 ? 32u : 64u, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kTcSmem = ssd::tc::kSmemTiles + 1024;
template <int HU>
constexpr size_t kSegSmem = ssd::tc::SegCfg<HU>::kSmem;

// dt [B, L, H] float32 as TMA boxes {4 heads, 128 tokens}: needs H % 4 == 0 (16-byte rows) and
// a 16-byte aligned base; otherwise seg_state loads dt with plain loads.
bool make_dt_map(CUtensorMap* m, const float* dt, int64_t batch, int64_t seqlen, int nheads) {
  if (nheads % 4 != 0 || (reinterpret_cast<uintptr_t>(dt) & 15) != 0) return false;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {uint64_t(nheads), uint64_t(seqlen), uint64_t(batch)};
  cuuint64_t strides[2] = {uint64_t(nheads) * 4, uint64_t(nheads) * uint64_t(seqlen) * 4};
  cuuint32_t box[3] = {4, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(dt), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view {inner, mid, outer} of a row-major tensor with a {box_inner, box_mid, 1} box, no
// swizzle, zero fill outside the tensor (the selective scan's tiles).
bool make_box_map(CUtensorMap* m, const void* base, CUtensorMapDataType type, uint64_t es,
                  uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_inner,
                  uint32_t box_mid) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * es, inner * mid * es};
  cuuint32_t box[3] = {box_inner, box_mid, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, type, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared-memory limits of the kernels, set once per device (the attribute applies to
// the current device only).
ssd_status set_smem_attrs() {
  constexpr int kMaxDev = 256;
  static std::mutex mu;
  static signed char done[kMaxDev] = {};  // 0 not yet, 1 ok, -1 failed
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return SSD_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev] == 0) {
    bool ok = true;
    ok &= cudaFuncSetAttribute(ssd::tc::scan_walk_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmem)) ==
          cudaSuccess;
    ok &= cudaFuncSetAttribute(ssd::tc::scan_walk_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmem)) ==
          cudaSuccess;
    // the selective scan runs many small CTAs per SM: ask for the largest shared-memory
    // carve-out so that shared memory does not cap them
    for (auto f : {(const void*)ssd::sel::selective_scan_kernel<float, float>,
                   (const void*)ssd::sel::selective_scan_kernel<__nv_bfloat16, float>,
                   (const void*)ssd::sel::selective_scan_kernel<__nv_bfloat16, __nv_bfloat16>})
      ok &= cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 int(cudaSharedmemCarveoutMaxShared)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(ssd::tc::seg_state_kernel<2>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSegSmem<2>)) ==
          cudaSuccess;
    for (auto f : {(const void*)ssd::bwd::chunk_bwd_kernel<float>,
                   (const void*)ssd::bwd::chunk_bwd_kernel<__nv_bfloat16>})
      ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) ==
            cudaSuccess;
    for (auto f : {(const void*)ssd::simt::chunk_out_kernel<float, float>,
                   (const void*)ssd::simt::chunk_out_kernel<__nv_bfloat16, float>,
                   (const void*)ssd::simt::chunk_out_kernel<__nv_bfloat16, __nv_bfloat16>,
                   (const void*)ssd::simt::chunk_state_kernel<float>,
                   (const void*)ssd::simt::chunk_state_kernel<__nv_bfloat16>})
      ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ==
            cudaSuccess;
    if (!ok) cudaGetLastError();
    done[dev] = ok ? 1 : -1;
  }
  return done[dev] == 1 ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status launched() {
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

struct ScanArgs {
  ssd_dtype ydt;
  const void *x, *B, *C;
  const float *dt, *A, *D, *init;
  void* y;
  float* fin;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
};

ssd_status validate_scan(const Shape& s, const ScanArgs& a, size_t need) {
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  for (const void* p : {a.x, (const void*)a.dt, (const void*)a.A, a.B, a.C, (const void*)a.y})
    if (!is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  for (const void* p : {(const void*)a.D, (const void*)a.init, (const void*)a.fin})
    if (p && !is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  if (a.ydt != SSD_F32 && a.ydt != s.io) return SSD_ERR_INVALID_ARG;
  const size_t es = s.io == SSD_BF16 ? 2 : 4;
  const size_t ey = a.ydt == SSD_BF16 ? 2 : 4;
  const size_t nx = size_t(s.batch) * s.seqlen * s.nheads * s.headdim * es;
  const size_t ny = size_t(s.batch) * s.seqlen * s.nheads * s.headdim * ey;
  const size_t nbc = size_t(s.batch) * s.seqlen * s.ngroups * s.dstate * es;
  const size_t ndt = size_t(s.batch) * s.seqlen * s.nheads * 4;
  const size_t nst = size_t(s.batch) * s.nheads * s.headdim * s.dstate * 4;
  const size_t nh = size_t(s.nheads) * 4;
  if (overlaps(a.y, ny, a.x, nx) || overlaps(a.y, ny, a.B, nbc) || overlaps(a.y, ny, a.C, nbc) ||
      overlaps(a.y, ny, a.dt, ndt) || overlaps(a.y, ny, a.A, nh) || overlaps(a.y, ny, a.D, nh) ||
      overlaps(a.y, ny, a.init, nst) || overlaps(a.y, ny, a.fin, nst))
    return SSD_ERR_INVALID_ARG;
  if (a.fin && a.fin != a.init &&
      (overlaps(a.fin, nst, a.init, nst) || overlaps(a.fin, nst, a.x, nx) ||
       overlaps(a.fin, nst, a.B, nbc) || overlaps(a.fin, nst, a.C, nbc)))
    return SSD_ERR_INVALID_ARG;
  if (need > 0) {
    if (!a.ws || a.ws_bytes < need || (reinterpret_cast<uintptr_t>(a.ws) & 255u) ||
        !is_device_ptr(a.ws))
      return SSD_ERR_WORKSPACE;
    if (overlaps(a.ws, need, a.y, ny) || overlaps(a.ws, need, a.x, nx) ||
        overlaps(a.ws, need, a.init, nst) || overlaps(a.ws, need, a.fin, nst))
      return SSD_ERR_INVALID_ARG;
  }
  return SSD_OK;
}

template <typename T, typename TY>
ssd_status run_simt(const Shape& s, const ScanArgs& a, bool with_output = true) {
  const int64_t nchunks = (s.seqlen + s.chunk - 1) / s.chunk;
  float* cs = static_cast<float*>(a.ws);
  float* states = reinterpret_cast<float*>(
      static_cast<char*>(a.ws) +
      align256(size_t(s.batch) * s.nheads * nchunks * s.chunk * sizeof(float)));
  const dim3 grid(unsigned(nchunks), unsigned(s.batch * s.nheads));
  ssd::simt::cumsum_kernel<<<grid, s.chunk, 0, a.stream>>>(a.dt, a.A, cs, s.seqlen, s.nheads,
                                                           s.chunk, int(nchunks));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  const size_t sm_state = ssd::outer_smem_floats(s.headdim, s.dstate) * sizeof(float);
  ssd::simt::chunk_state_kernel<T><<<grid, ssd::kOuterThreads, sm_state, a.stream>>>(
      static_cast<const T*>(a.x), a.dt, static_cast<const T*>(a.B), cs, states, s.seqlen,
      s.nheads, s.headdim, s.dstate, s.ngroups, s.chunk, int(nchunks));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  const int64_t nel = s.batch * s.nheads * int64_t(s.headdim) * s.dstate;
  ssd::simt::state_pass_kernel<<<unsigned((nel + 255) / 256), 256, 0, a.stream>>>(
      states, cs, a.init, a.fin, s.batch, s.nheads, s.headdim, s.dstate, s.chunk, int(nchunks));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  if (!with_output) return SSD_OK;
  const size_t sm_out = (3072 + 64 * size_t(s.headdim)) * sizeof(float);
  ssd::simt::chunk_out_kernel<T, TY><<<grid, 256, sm_out, a.stream>>>(
      static_cast<const T*>(a.x), a.dt, static_cast<const T*>(a.B), static_cast<const T*>(a.C),
      a.D, cs, states, static_cast<TY*>(a.y), s.seqlen, s.nheads, s.headdim, s.dstate,
      s.ngroups, s.chunk, int(nchunks));
  return launched();
}

// seg_state over the first sg.useg segments of every sequence (persistent, one CTA per SM).
ssd_status launch_seg_state(const Shape& s, const ScanArgs& a, const Seg& sg, const CUtensorMap& mx,
                            const CUtensorMap& mb, float* states, float* decay) {
  const int hpg = s.nheads / s.ngroups;
  const int64_t units = s.batch * int64_t(sg.useg) * (s.nheads / 2);
  if (units <= 0) return SSD_OK;
  CUtensorMap mdt;
  std::memset(&mdt, 0, sizeof mdt);
  const int dt_tma = make_dt_map(&mdt, a.dt, s.batch, s.seqlen, s.nheads) ? 1 : 0;
  // two heads per unit: four (one B tile for four heads) measured slower at the 2.7B shape
  // (two 96 KB stages instead of three of 64 KB, and half as many units to balance over SMs)
  ssd::tc::seg_state_kernel<2><<<unsigned(std::min<int64_t>(units, sm_count())),
                                 ssd::tc::SegCfg<2>::kThreads, kSegSmem<2>, a.stream>>>(
      mx, mb, mdt, dt_tma, a.dt, a.A, states, decay, s.seqlen, s.nheads, hpg, sg, int(units));
  return launched();
}

ssd_status launch_seg_pass(const Shape& s, const ScanArgs& a, const Seg& sg, float* states,
                           const float* decay, float* fin) {
  const int64_t nvec = s.batch * s.nheads * int64_t(64) * 128 / 4;
  ssd::tc::seg_pass_kernel<<<unsigned((nvec + ssd::tc::kPassThreads - 1) / ssd::tc::kPassThreads),
                             ssd::tc::kPassThreads, 0, a.stream>>>(
      states, decay, a.init, fin, int(s.batch), s.nheads, sg.nseg, sg.useg);
  return launched();
}

// The states only (seg_state over every segment, seg_pass with the final state), for
// ssd_chunk_state_fwd.
ssd_status run_tc_state(const Shape& s, const ScanArgs& a, void* scratch) {
  const Seg sg = tc_segments(s);
  const SegScratch w = seg_scratch(s, sg, scratch);
  CUtensorMap mx, mb;
  const uint64_t HP = uint64_t(s.nheads) * 64, GN = uint64_t(s.ngroups) * 128;
  if (!make_map(&mx, a.x, HP, s.seqlen, s.batch) || !make_map(&mb, a.B, GN, s.seqlen, s.batch))
    return SSD_ERR_CUDA;
  ssd_status st = launch_seg_state(s, a, sg, mx, mb, w.states, w.decay);
  if (st != SSD_OK) return st;
  return launch_seg_pass(s, a, sg, w.states, w.decay, a.fin);
}

// The scan: (segments only) seg_state + seg_pass, then the walk.
ssd_status run_tc_walk(const Shape& s, const ScanArgs& a, const TcPlan& p, void* scratch) {
  const WalkScratch w = walk_scratch(s, p, scratch);
  CUtensorMap mx, mb, mc, my;
  const uint64_t HP = uint64_t(s.nheads) * 64, GN = uint64_t(s.ngroups) * 128;
  if (!make_map(&mx, a.x, HP, s.seqlen, s.batch) || !make_map(&mb, a.B, GN, s.seqlen, s.batch) ||
      !make_map(&mc, a.C, GN, s.seqlen, s.batch) ||
      !make_map(&my, a.y, HP, s.seqlen, s.batch, a.ydt == SSD_F32))
    return SSD_ERR_CUDA;
  // the ticket and the ready flags start at zero every call
  if (cudaMemsetAsync(w.ticket, 0, w.header_bytes, a.stream) != cudaSuccess) {
    cudaGetLastError();
    return SSD_ERR_CUDA;
  }
  if (p.sg.nseg > 1) {
    ssd_status st = launch_seg_state(s, a, p.sg, mx, mb, w.states, w.decay);
    if (st != SSD_OK) return st;
    st = launch_seg_pass(s, a, p.sg, w.states, w.decay, nullptr);
    if (st != SSD_OK) return st;
  }
  const int hpg = s.nheads / s.ngroups;
  if (a.ydt == SSD_F32)
    ssd::tc::scan_walk_kernel<float><<<unsigned(p.w.nct), ssd::tc::kWalkThreads, kTcSmem,
                                       a.stream>>>(
        mx, mb, mc, my, a.dt, a.A, a.D, a.init, w.states, a.fin, w.slots, w.flags, w.ticket,
        s.seqlen, s.nheads, hpg, p.w);
  else
    ssd::tc::scan_walk_kernel<__nv_bfloat16><<<unsigned(p.w.nct), ssd::tc::kWalkThreads, kTcSmem,
                                               a.stream>>>(
        mx, mb, mc, my, a.dt, a.A, a.D, a.init, w.states, a.fin, w.slots, w.flags, w.ticket,
        s.seqlen, s.nheads, hpg, p.w);
  return launched();
}

ssd_status run_simt_any(const Shape& s, const ScanArgs& a) {
  if (s.io == SSD_F32) return run_simt<float, float>(s, a);
  if (a.ydt == SSD_F32) return run_simt<__nv_bfloat16, float>(s, a);
  return run_simt<__nv_bfloat16, __nv_bfloat16>(s, a);
}

bool tc_pointers_ok(const ScanArgs& a) {
  return aligned16(a.x) && aligned16(a.B) && aligned16(a.C) && aligned16(a.y);
}

ssd_status validate_state(const Shape& s, const ScanArgs& a, float* total_decay, size_t need) {
  for (const void* p : {a.x, (const void*)a.dt, (const void*)a.A, a.B, (const void*)a.fin,
                        (const void*)total_decay})
    if (!is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  if (a.init && !is_device_ptr(a.init)) return SSD_ERR_INVALID_ARG;
  const size_t es = s.io == SSD_BF16 ? 2 : 4;
  const size_t nx = size_t(s.batch) * s.seqlen * s.nheads * s.headdim * es;
  const size_t nbc = size_t(s.batch) * s.seqlen * s.ngroups * s.dstate * es;
  const size_t ndt = size_t(s.batch) * s.seqlen * s.nheads * 4;
  const size_t nst = size_t(s.batch) * s.nheads * s.headdim * s.dstate * 4;
  const size_t nd = size_t(s.batch) * s.nheads * 4;
  if ((a.fin != a.init && overlaps(a.fin, nst, a.init, nst)) || overlaps(a.fin, nst, a.x, nx) ||
      overlaps(a.fin, nst, a.B, nbc) || overlaps(a.fin, nst, a.dt, ndt) ||
      overlaps(total_decay, nd, a.fin, nst) || overlaps(total_decay, nd, a.dt, ndt) ||
      overlaps(total_decay, nd, a.x, nx) || overlaps(total_decay, nd, a.B, nbc) ||
      overlaps(total_decay, nd, a.init, nst))
    return SSD_ERR_INVALID_ARG;
  if (need > 0) {
    if (!a.ws || a.ws_bytes < need || (reinterpret_cast<uintptr_t>(a.ws) & 255u) ||
        !is_device_ptr(a.ws))
      return SSD_ERR_WORKSPACE;
    if (overlaps(a.ws, need, a.x, nx) || overlaps(a.ws, need, a.init, nst) ||
        overlaps(a.ws, need, a.fin, nst) || overlaps(a.ws, need, total_decay, nd))
      return SSD_ERR_INVALID_ARG;
  }
  return SSD_OK;
}

// ---- backward ---------------------------------------------------------------------------
// Workspace: cs [B, H, nc, kQ] | forward entering states [B, nc, H, P, N] | adjoints (same) |
// per-head dB, dC rows [B, L, H, N] each | dA, dD partials [B, nc, H] each.
size_t bwd_workspace(const Shape& s) {
  const int64_t nc = (s.seqlen + ssd::bwd::kQ - 1) / ssd::bwd::kQ;
  const size_t st = size_t(s.batch) * nc * s.nheads * size_t(s.headdim) * s.dstate * 4;
  const size_t rows = size_t(s.batch) * s.seqlen * s.nheads * size_t(s.dstate) * 4;
  const size_t part = size_t(s.batch) * nc * s.nheads * 4;
  return align256(size_t(s.batch) * s.nheads * nc * ssd::bwd::kQ * 4) + 2 * align256(st) +
         2 * align256(rows) + 2 * align256(part);
}

bool bwd_supported(const Shape& s) {
  const size_t smem = ssd::bwd::BwdSmem::floats(s.headdim, s.dstate) * sizeof(float);
  return smem <= 227 * 1024 && s.batch * s.nheads <= 65535 &&
         (s.seqlen + ssd::bwd::kQ - 1) / ssd::bwd::kQ <= (int64_t(1) << 30);
}

template <typename T>
ssd_status run_bwd(const Shape& s, const ScanArgs& a, const float* dy, const float* dfinal,
                   float* dx, float* ddt, float* dA, float* dB, float* dC, float* dD,
                   float* dinit) {
  namespace bw = ssd::bwd;
  const int64_t nc = (s.seqlen + bw::kQ - 1) / bw::kQ;
  const size_t st = size_t(s.batch) * nc * s.nheads * size_t(s.headdim) * s.dstate * 4;
  const size_t rows = size_t(s.batch) * s.seqlen * s.nheads * size_t(s.dstate) * 4;
  const size_t part = size_t(s.batch) * nc * s.nheads * 4;
  char* w = static_cast<char*>(a.ws);
  float* cs = reinterpret_cast<float*>(w);
  w += align256(size_t(s.batch) * s.nheads * nc * bw::kQ * 4);
  float* hst = reinterpret_cast<float*>(w);
  w += align256(st);
  float* adj = reinterpret_cast<float*>(w);
  w += align256(st);
  float* dbh = reinterpret_cast<float*>(w);
  w += align256(rows);
  float* dch = reinterpret_cast<float*>(w);
  w += align256(rows);
  float* dA_part = reinterpret_cast<float*>(w);
  w += align256(part);
  float* dD_part = reinterpret_cast<float*>(w);
  const dim3 grid(unsigned(nc), unsigned(s.batch * s.nheads));
  const int P = s.headdim, N = s.dstate;
  // forward: within-chunk cumsums, chunk states, and the state entering every chunk
  ssd::simt::cumsum_kernel<<<grid, bw::kQ, 0, a.stream>>>(a.dt, a.A, cs, s.seqlen, s.nheads,
                                                          bw::kQ, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  const size_t sm_outer = ssd::outer_smem_floats(P, N) * sizeof(float);
  ssd::simt::chunk_state_kernel<T><<<grid, ssd::kOuterThreads, sm_outer, a.stream>>>(
      static_cast<const T*>(a.x), a.dt, static_cast<const T*>(a.B), cs, hst, s.seqlen, s.nheads,
      P, N, s.ngroups, bw::kQ, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  const int64_t nel = s.batch * s.nheads * int64_t(P) * N;
  ssd::simt::state_pass_kernel<<<unsigned((nel + 255) / 256), 256, 0, a.stream>>>(
      hst, cs, a.init, nullptr, s.batch, s.nheads, P, N, bw::kQ, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  // backward: adjoint summaries, the adjoint entering every chunk from the right, then chunks
  bw::adj_state_kernel<T><<<grid, ssd::kOuterThreads, sm_outer, a.stream>>>(
      dy, static_cast<const T*>(a.C), cs, adj, s.seqlen, s.nheads, P, N, s.ngroups, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  bw::adj_pass_kernel<<<unsigned((nel + 255) / 256), 256, 0, a.stream>>>(
      adj, cs, dfinal, dinit, s.batch, s.nheads, P, N, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  bw::chunk_bwd_kernel<T><<<grid, bw::kBwdThreads, bw::BwdSmem::floats(P, N) * sizeof(float),
                            a.stream>>>(
      static_cast<const T*>(a.x), a.dt, a.A, static_cast<const T*>(a.B),
      static_cast<const T*>(a.C), a.D, dy, cs, hst, adj, dx, ddt, dbh, dch, dA_part, dD_part,
      s.seqlen, s.nheads, P, N, s.ngroups, int(nc));
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  const int64_t ngn = s.batch * s.seqlen * s.ngroups * int64_t(N);
  bw::group_sum_kernel<float><<<unsigned((ngn + 255) / 256), 256, 0, a.stream>>>(
      dbh, dch, dB, dC, s.batch * s.seqlen, s.nheads, s.ngroups, N);
  if (launched() != SSD_OK) return SSD_ERR_CUDA;
  bw::head_sum_kernel<<<unsigned((s.nheads + 127) / 128), 128, 0, a.stream>>>(
      dA_part, dD_part, dA, dD, s.batch * nc, s.nheads);
  return launched();
}

}  // namespace

extern "C" {

size_t ssd_chunk_scan_workspace_size(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                     int dstate, int ngroups, int chunk, ssd_dtype io) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  if (check_shape(s) != SSD_OK) return 0;
  if (tc_shape_ok(s)) return tc_workspace(s);
  return simt_supported(s) ? simt_workspace(s) : 0;
}

ssd_path ssd_chunk_scan_path(int64_t batch, int64_t seqlen, int nheads, int headdim, int dstate,
                             int ngroups, int chunk, ssd_dtype io) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  return (check_shape(s) == SSD_OK && tc_shape_ok(s)) ? SSD_PATH_TCGEN05 : SSD_PATH_SIMT;
}

size_t ssd_chunk_scan_simt_workspace_size(int64_t batch, int64_t seqlen, int nheads,
                                          int headdim, int dstate, int ngroups, int chunk,
                                          ssd_dtype io) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  if (check_shape(s) != SSD_OK || !simt_supported(s)) return 0;
  return simt_workspace(s);
}

ssd_status ssd_chunk_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                              const void* C, const float* D, const float* init_state, void* y,
                              float* final_state, int64_t batch, int64_t seqlen, int nheads,
                              int headdim, int dstate, int ngroups, int chunk, ssd_dtype io,
                              ssd_dtype y_dtype, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  const ScanArgs a{y_dtype, x, B, C, dt, A, D, init_state, y, final_state, workspace,
                   workspace_bytes, stream};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  const bool tc = tc_shape_ok(s);
  if (!tc && !simt_supported(s)) return SSD_ERR_UNSUPPORTED;
  TcPlan plan;
  if (tc && !make_tc_plan(s, ScanOpts(), &plan)) return SSD_ERR_UNSUPPORTED;
  st = validate_scan(s, a, tc ? tc_workspace(s) : simt_workspace(s));
  if (st != SSD_OK) return st;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  if (tc) {
    if (!tc_pointers_ok(a)) return SSD_ERR_UNSUPPORTED;
    return run_tc_walk(s, a, plan, a.ws);
  }
  return run_simt_any(s, a);
}

size_t ssd_chunk_scan_workspace_size_ex(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                        int dstate, int ngroups, int chunk, ssd_dtype io,
                                        const ssd_scan_options* opt) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  if (check_shape(s) != SSD_OK || !tc_shape_ok(s)) return 0;
  ScanOpts o;
  if (opt) {
    o.max_ctas = opt->max_ctas;
    o.plan = opt->plan;
    o.wait_ns = opt->wait_limit_ns;
  }
  return tc_workspace(s, o);
}

ssd_status ssd_chunk_scan_plan_info(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                    int dstate, int ngroups, int chunk, ssd_dtype io,
                                    const ssd_scan_options* opt, ssd_plan_info* info) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  if (!info || check_shape(s) != SSD_OK) return SSD_ERR_INVALID_ARG;
  if (!tc_shape_ok(s)) return SSD_ERR_UNSUPPORTED;
  ScanOpts o;
  if (opt) {
    o.max_ctas = opt->max_ctas;
    o.plan = opt->plan;
    o.wait_ns = opt->wait_limit_ns;
  }
  TcPlan p;
  if (!make_tc_plan(s, o, &p)) return SSD_ERR_UNSUPPORTED;
  info->launches = p.sg.nseg > 1 ? 3 : 1;
  info->ctas = p.w.nct;
  info->segments = p.w.nseg;
  return SSD_OK;
}

ssd_status ssd_chunk_scan_fwd_ex(const void* x, const float* dt, const float* A, const void* B,
                                 const void* C, const float* D, const float* init_state,
                                 void* y, float* final_state, int64_t batch, int64_t seqlen,
                                 int nheads, int headdim, int dstate, int ngroups, int chunk,
                                 ssd_dtype io, ssd_dtype y_dtype, void* workspace,
                                 size_t workspace_bytes, const ssd_scan_options* opt,
                                 cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  const ScanArgs a{y_dtype, x, B, C, dt, A, D, init_state, y, final_state, workspace,
                   workspace_bytes, stream};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  ScanOpts o;
  if (opt) {
    if (opt->max_ctas < 0 || opt->plan < 0 || opt->plan > 2 || opt->wait_limit_ns < -1)
      return SSD_ERR_INVALID_ARG;
    o.max_ctas = opt->max_ctas;
    o.plan = opt->plan;
    o.wait_ns = opt->wait_limit_ns;
  }
  if (!tc_shape_ok(s)) return SSD_ERR_UNSUPPORTED;
  TcPlan plan;
  if (!make_tc_plan(s, o, &plan)) return SSD_ERR_UNSUPPORTED;
  st = validate_scan(s, a, tc_workspace(s, o));
  if (st != SSD_OK) return st;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  if (!tc_pointers_ok(a)) return SSD_ERR_UNSUPPORTED;
  return run_tc_walk(s, a, plan, a.ws);
}

ssd_status ssd_chunk_scan_fwd_simt(const void* x, const float* dt, const float* A,
                                   const void* B, const void* C, const float* D,
                                   const float* init_state, void* y, float* final_state,
                                   int64_t batch, int64_t seqlen, int nheads, int headdim,
                                   int dstate, int ngroups, int chunk, ssd_dtype io,
                                   ssd_dtype y_dtype, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  const ScanArgs a{y_dtype, x, B, C, dt, A, D, init_state, y, final_state, workspace,
                   workspace_bytes, stream};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  if (!simt_supported(s)) return SSD_ERR_UNSUPPORTED;
  st = validate_scan(s, a, simt_workspace(s));
  if (st != SSD_OK) return st;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  return run_simt_any(s, a);
}

ssd_status ssd_step(float* state, const void* x, const float* dt, const float* A,
                    const void* B, const void* C, const float* D, void* y, int64_t batch,
                    int nheads, int headdim, int dstate, int ngroups, ssd_dtype io,
                    ssd_dtype y_dtype, cudaStream_t stream) {
  if (batch <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
      nheads % ngroups != 0 || (io != SSD_F32 && io != SSD_BF16) ||
      (y_dtype != SSD_F32 && y_dtype != io))
    return SSD_ERR_INVALID_ARG;
  if (batch * nheads > (int64_t(1) << 31) - 1) return SSD_ERR_UNSUPPORTED;
  for (const void* p : {(const void*)state, x, (const void*)dt, (const void*)A, B, C,
                        (const void*)y})
    if (!is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  if (D && !is_device_ptr(D)) return SSD_ERR_INVALID_ARG;
  const size_t es = io == SSD_BF16 ? 2 : 4;
  const size_t nst = size_t(batch) * nheads * headdim * dstate * 4;
  const size_t nx = size_t(batch) * nheads * headdim * es;
  const size_t ny = size_t(batch) * nheads * headdim * (y_dtype == SSD_BF16 ? 2 : 4);
  const size_t nbc = size_t(batch) * ngroups * dstate * es;
  const size_t ndt = size_t(batch) * nheads * 4, nh = size_t(nheads) * 4;
  if (overlaps(y, ny, state, nst) || overlaps(y, ny, x, nx) || overlaps(y, ny, B, nbc) ||
      overlaps(y, ny, C, nbc) || overlaps(y, ny, dt, ndt) || overlaps(y, ny, A, nh) ||
      overlaps(y, ny, D, nh) || overlaps(state, nst, x, nx) || overlaps(state, nst, B, nbc) ||
      overlaps(state, nst, C, nbc) || overlaps(state, nst, dt, ndt) ||
      overlaps(state, nst, A, nh) || overlaps(state, nst, D, nh))
    return SSD_ERR_INVALID_ARG;
  const int hpg = nheads / ngroups;
  const unsigned grid = unsigned(batch * nheads);
  const bool fast = dstate == 128 && headdim % 8 == 0 && aligned16(state) &&
                    (headdim / 8 == 1 || headdim / 8 == 2 || headdim / 8 == 4 ||
                     headdim / 8 == 8 || headdim / 8 == 16);
#define SSD_STEP_FAST(T, TY, RPW)                                                          \
  ssd::step_n128_kernel<T, TY, RPW><<<grid, 256, 0, stream>>>(                             \
      state, static_cast<const T*>(x), dt, A, static_cast<const T*>(B),                    \
      static_cast<const T*>(C), D, static_cast<TY*>(y), nheads, hpg, ngroups)
#define SSD_STEP_DISPATCH(T, TY)                      \
  switch (headdim / 8) {                              \
    case 1: SSD_STEP_FAST(T, TY, 1); break;           \
    case 2: SSD_STEP_FAST(T, TY, 2); break;           \
    case 4: SSD_STEP_FAST(T, TY, 4); break;           \
    case 8: SSD_STEP_FAST(T, TY, 8); break;           \
    default: SSD_STEP_FAST(T, TY, 16); break;         \
  }
#define SSD_STEP_GENERIC(T, TY)                                                            \
  ssd::step_generic_kernel<T, TY><<<grid, 256, 0, stream>>>(                               \
      state, static_cast<const T*>(x), dt, A, static_cast<const T*>(B),                    \
      static_cast<const T*>(C), D, static_cast<TY*>(y), nheads, headdim, dstate, hpg, ngroups)
  if (fast) {
    if (io == SSD_F32) { SSD_STEP_DISPATCH(float, float) }
    else if (y_dtype == SSD_F32) { SSD_STEP_DISPATCH(__nv_bfloat16, float) }
    else { SSD_STEP_DISPATCH(__nv_bfloat16, __nv_bfloat16) }
  } else {
    if (io == SSD_F32) { SSD_STEP_GENERIC(float, float); }
    else if (y_dtype == SSD_F32) { SSD_STEP_GENERIC(__nv_bfloat16, float); }
    else { SSD_STEP_GENERIC(__nv_bfloat16, __nv_bfloat16); }
  }
#undef SSD_STEP_GENERIC
#undef SSD_STEP_DISPATCH
#undef SSD_STEP_FAST
  return launched();
}

size_t ssd_chunk_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int nheads,
                                         int headdim, int dstate, int ngroups, ssd_dtype io) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, 64, io};
  if (check_shape(s) != SSD_OK || !bwd_supported(s)) return 0;
  return bwd_workspace(s);
}

ssd_status ssd_chunk_scan_bwd(const void* x, const float* dt, const float* A, const void* B,
                              const void* C, const float* D, const float* init_state,
                              const float* dy, const float* dfinal, float* dx, float* ddt,
                              float* dA, float* dB, float* dC, float* dD, float* dinit,
                              int64_t batch, int64_t seqlen, int nheads, int headdim, int dstate,
                              int ngroups, ssd_dtype io, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, 64, io};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  if (!bwd_supported(s)) return SSD_ERR_UNSUPPORTED;
  for (const void* p : {x, (const void*)dt, (const void*)A, B, C, (const void*)dy, (const void*)dx,
                        (const void*)ddt, (const void*)dA, (const void*)dB, (const void*)dC})
    if (!is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  for (const void* p : {(const void*)D, (const void*)init_state, (const void*)dfinal,
                        (const void*)dD, (const void*)dinit})
    if (p && !is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  const size_t es = io == SSD_BF16 ? 2 : 4;
  const size_t ntok = size_t(batch) * seqlen;
  const size_t nx = ntok * nheads * headdim * es, nxf = ntok * nheads * headdim * 4;
  const size_t ndt = ntok * nheads * 4, nbc = ntok * ngroups * dstate * es;
  const size_t nbcf = ntok * ngroups * dstate * 4, nh = size_t(nheads) * 4;
  const size_t nst = size_t(batch) * nheads * headdim * dstate * 4;
  const std::pair<const void*, size_t> ins[] = {{x, nx}, {dt, ndt}, {A, nh}, {B, nbc}, {C, nbc},
                                                {D, nh}, {init_state, nst}, {dy, nxf},
                                                {dfinal, nst}};
  const std::pair<const void*, size_t> outs[] = {{dx, nxf}, {ddt, ndt}, {dA, nh}, {dB, nbcf},
                                                 {dC, nbcf}, {dD, nh}, {dinit, nst}};
  for (const auto& o : outs) {
    for (const auto& i : ins)
      if (overlaps(o.first, o.second, i.first, i.second)) return SSD_ERR_INVALID_ARG;
    for (const auto& o2 : outs)
      if (&o2 != &o && overlaps(o.first, o.second, o2.first, o2.second))
        return SSD_ERR_INVALID_ARG;
  }
  const size_t need = bwd_workspace(s);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      !is_device_ptr(workspace))
    return SSD_ERR_WORKSPACE;
  for (const auto& o : outs)
    if (overlaps(workspace, need, o.first, o.second)) return SSD_ERR_INVALID_ARG;
  for (const auto& i : ins)
    if (overlaps(workspace, need, i.first, i.second)) return SSD_ERR_INVALID_ARG;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  const ScanArgs a{SSD_F32, x, B, C, dt, A, D, init_state, nullptr, nullptr, workspace,
                   workspace_bytes, stream};
  if (io == SSD_BF16)
    return run_bwd<__nv_bfloat16>(s, a, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit);
  return run_bwd<float>(s, a, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit);
}

const char* ssd_status_string(ssd_status s) {
  switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape or alignment not supported";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA launch or runtime failure";
    case SSD_ERR_DEVICE_TIMEOUT: return "SSD_ERR_DEVICE_TIMEOUT: a kernel's bounded wait expired";
  }
  return "unknown ssd_status";
}

ssd_status ssd_chunk_state_fwd(const void* x, const float* dt, const float* A, const void* B,
                               const float* init_state, float* final_state, float* total_decay,
                               int64_t batch, int64_t seqlen, int nheads, int headdim,
                               int dstate, int ngroups, int chunk, ssd_dtype io,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  const ScanArgs a{SSD_F32, x, B, nullptr, dt, A, nullptr, init_state, nullptr, final_state,
                   workspace, workspace_bytes, stream};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  const bool tc = tc_shape_ok(s);
  if (!tc && !simt_supported(s)) return SSD_ERR_UNSUPPORTED;
  st = validate_state(s, a, total_decay, tc ? tc_workspace(s) : simt_workspace(s));
  if (st != SSD_OK) return st;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  if (tc) {
    if (!aligned16(x) || !aligned16(B)) return SSD_ERR_UNSUPPORTED;
    st = run_tc_state(s, a, a.ws);
  } else {
    st = s.io == SSD_F32 ? run_simt<float, float>(s, a, false)
                         : run_simt<__nv_bfloat16, float>(s, a, false);
  }
  if (st != SSD_OK) return st;
  const dim3 grid(unsigned(batch), unsigned((nheads + 31) / 32));
  ssd::pass::decay_sum_kernel<<<grid, 256, 0, stream>>>(dt, A, total_decay, seqlen, nheads);
  return launched();
}

ssd_status ssd_state_pass(float* states, const float* decay, const float* init_state,
                          float* final_state, int64_t nslices, int64_t batch, int nheads,
                          int headdim, int dstate, cudaStream_t stream) {
  if (nslices < 1 || batch < 1 || nheads < 1 || headdim < 1 || dstate < 1)
    return SSD_ERR_INVALID_ARG;
  if (!is_device_ptr(states) || !is_device_ptr(decay)) return SSD_ERR_INVALID_ARG;
  if ((init_state && !is_device_ptr(init_state)) || (final_state && !is_device_ptr(final_state)))
    return SSD_ERR_INVALID_ARG;
  const int64_t nbh = batch * nheads, per_bh = int64_t(headdim) * dstate;
  const size_t nst = size_t(nbh * per_bh) * 4;
  if (overlaps(final_state, nst, states, nst * size_t(nslices)) ||
      overlaps(decay, size_t(nslices * nbh) * 4, states, nst * size_t(nslices)) ||
      (final_state != init_state && overlaps(final_state, nst, init_state, nst)))
    return SSD_ERR_INVALID_ARG;
  const int64_t n = nbh * per_bh;
  ssd::pass::slice_pass_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(
      states, decay, init_state, final_state, nslices, nbh, per_bh);
  return launched();
}

ssd_status ssd_conv_silu(const void* u, const float* w, const float* bias, void* out,
                         int64_t batch, int64_t seqlen, int cdim, int kwidth, ssd_dtype io,
                         cudaStream_t stream) {
  if (batch < 1 || seqlen < 1 || cdim < 1 || kwidth < 1 || kwidth > 8 ||
      (io != SSD_F32 && io != SSD_BF16))
    return SSD_ERR_INVALID_ARG;
  if (!is_device_ptr(u) || !is_device_ptr(w) || !is_device_ptr(out) ||
      (bias && !is_device_ptr(bias)))
    return SSD_ERR_INVALID_ARG;
  const size_t es = io == SSD_BF16 ? 2 : 4;
  const int64_t ntok = batch * seqlen;
  const size_t nb = size_t(ntok) * cdim * es;
  if (overlaps(out, nb, u, nb) || overlaps(out, nb, w, size_t(cdim) * kwidth * 4) ||
      overlaps(out, nb, bias, size_t(cdim) * 4))
    return SSD_ERR_INVALID_ARG;
  const int vw = io == SSD_BF16 ? 8 : 4;
  if (cdim % vw != 0 || !aligned16(u) || !aligned16(out) || !aligned16(w))
    return SSD_ERR_UNSUPPORTED;
  const int64_t runs = (seqlen + ssd::glue::kConvTok - 1) / ssd::glue::kConvTok;
  if (runs > 65535 || batch > 65535) return SSD_ERR_UNSUPPORTED;
  // one warp per block: the finest split of the grid over the SMs (blocks of 96 and 128 threads
  // measured 4% and 7% slower at the 2.7B shape)
  const dim3 grid(unsigned((cdim / vw + 31) / 32), unsigned(runs), unsigned(batch));
#define SSD_CONV(T, KW)                                                                    \
  ssd::glue::conv_silu_kernel<T, KW><<<grid, 32, 0, stream>>>(                            \
      static_cast<const T*>(u), w, bias, static_cast<T*>(out), seqlen, cdim)
#define SSD_CONV_K(T)                                                                      \
  switch (kwidth) {                                                                        \
    case 1: SSD_CONV(T, 1); break;                                                         \
    case 2: SSD_CONV(T, 2); break;                                                         \
    case 3: SSD_CONV(T, 3); break;                                                         \
    case 4: SSD_CONV(T, 4); break;                                                         \
    case 5: SSD_CONV(T, 5); break;                                                         \
    case 6: SSD_CONV(T, 6); break;                                                         \
    case 7: SSD_CONV(T, 7); break;                                                         \
    default: SSD_CONV(T, 8); break;                                                        \
  }
  if (io == SSD_BF16) { SSD_CONV_K(__nv_bfloat16) }
  else { SSD_CONV_K(float) }
#undef SSD_CONV_K
#undef SSD_CONV
  return launched();
}

ssd_status ssd_dt_softplus(const float* raw, const float* bias, float* dt, int64_t batch,
                           int64_t seqlen, int nheads, cudaStream_t stream) {
  if (batch < 1 || seqlen < 1 || nheads < 1) return SSD_ERR_INVALID_ARG;
  if (!is_device_ptr(raw) || !is_device_ptr(dt) || (bias && !is_device_ptr(bias)))
    return SSD_ERR_INVALID_ARG;
  const int64_t n = batch * seqlen * nheads;
  if (dt != raw && overlaps(dt, size_t(n) * 4, raw, size_t(n) * 4)) return SSD_ERR_INVALID_ARG;
  if (overlaps(dt, size_t(n) * 4, bias, size_t(nheads) * 4)) return SSD_ERR_INVALID_ARG;
  const int64_t nthr = (n + 7) / 8;
  if ((nthr + 255) / 256 > INT32_MAX) return SSD_ERR_UNSUPPORTED;
  ssd::glue::dt_softplus_kernel<<<unsigned((nthr + 255) / 256), 256, 0, stream>>>(
      raw, bias, dt, n, nheads, aligned16(raw) && aligned16(dt));
  return launched();
}

ssd_status ssd_gate_silu(const float* y, const void* z, void* out, int64_t n, ssd_dtype z_dtype,
                         ssd_dtype out_dtype, cudaStream_t stream) {
  if (n < 1 || (z_dtype != SSD_F32 && z_dtype != SSD_BF16) ||
      (out_dtype != SSD_F32 && out_dtype != z_dtype))
    return SSD_ERR_INVALID_ARG;
  if (!is_device_ptr(y) || !is_device_ptr(z) || !is_device_ptr(out)) return SSD_ERR_INVALID_ARG;
  const size_t nz = size_t(n) * (z_dtype == SSD_BF16 ? 2 : 4);
  const size_t no = size_t(n) * (out_dtype == SSD_BF16 ? 2 : 4);
  // in place over y only with a float32 out: a narrower out would let one thread overwrite y
  // elements that a lower-index thread has not read yet
  if (out == static_cast<const void*>(y) && out_dtype != SSD_F32) return SSD_ERR_INVALID_ARG;
  if ((out != static_cast<const void*>(y) && overlaps(out, no, y, size_t(n) * 4)) ||
      overlaps(out, no, z, nz))
    return SSD_ERR_INVALID_ARG;
  const int vw = z_dtype == SSD_BF16 ? 8 : 4;
  if (n % vw != 0 || !aligned16(y) || !aligned16(z) || !aligned16(out) ||
      (n / vw + 255) / 256 > INT32_MAX)
    return SSD_ERR_UNSUPPORTED;
  const unsigned grid = unsigned((n / vw + 255) / 256);
  if (z_dtype == SSD_F32)
    ssd::glue::gate_silu_kernel<float, float><<<grid, 256, 0, stream>>>(
        y, static_cast<const float*>(z), static_cast<float*>(out), n);
  else if (out_dtype == SSD_F32)
    ssd::glue::gate_silu_kernel<__nv_bfloat16, float><<<grid, 256, 0, stream>>>(
        y, static_cast<const __nv_bfloat16*>(z), static_cast<float*>(out), n);
  else
    ssd::glue::gate_silu_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, stream>>>(
        y, static_cast<const __nv_bfloat16*>(z), static_cast<__nv_bfloat16*>(out), n);
  return launched();
}

ssd_status ssd_selective_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const float* init_state,
                                  void* y, float* final_state, int64_t batch, int64_t seqlen,
                                  int dim, int dstate, int ngroups, ssd_dtype io,
                                  ssd_dtype y_dtype, cudaStream_t stream) {
  if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1 || ngroups < 1 || dim % ngroups != 0 ||
      (io != SSD_F32 && io != SSD_BF16) || (y_dtype != SSD_F32 && y_dtype != io))
    return SSD_ERR_INVALID_ARG;
  for (const void* p : {x, (const void*)dt, (const void*)A, B, C, (const void*)y})
    if (!is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  for (const void* p : {(const void*)D, (const void*)init_state, (const void*)final_state})
    if (p && !is_device_ptr(p)) return SSD_ERR_INVALID_ARG;
  const size_t es = io == SSD_BF16 ? 2 : 4;
  const size_t ntok = size_t(batch) * size_t(seqlen);
  const size_t nx = ntok * dim * es, ndt = ntok * dim * 4;
  const size_t ny = ntok * dim * (y_dtype == SSD_BF16 ? 2 : 4);
  const size_t nbc = ntok * ngroups * dstate * es;
  const size_t nst = size_t(batch) * dim * dstate * 4;
  for (const auto& in : {std::make_pair(x, nx), std::make_pair((const void*)dt, ndt),
                         std::make_pair(B, nbc), std::make_pair(C, nbc),
                         std::make_pair((const void*)init_state, nst)}) {
    if (overlaps(y, ny, in.first, in.second)) return SSD_ERR_INVALID_ARG;
    if (final_state && in.first != init_state && overlaps(final_state, nst, in.first, in.second))
      return SSD_ERR_INVALID_ARG;
  }
  if (overlaps(y, ny, final_state, nst)) return SSD_ERR_INVALID_ARG;
  if (final_state && init_state && final_state != init_state &&
      overlaps(final_state, nst, init_state, nst))
    return SSD_ERR_INVALID_ARG;
  namespace sel = ssd::sel;
  if (dstate != sel::kN || dim % sel::kCpw != 0 || (dim / ngroups) % sel::kCpw != 0)
    return SSD_ERR_UNSUPPORTED;
  const int cw = sel::kCpw;  // channels per CTA (one warp)
  for (const void* p : {x, (const void*)dt, (const void*)A, B, C, (const void*)y,
                        (const void*)init_state, (const void*)final_state})
    if (p && !aligned16(p)) return SSD_ERR_UNSUPPORTED;
  const int64_t ctas = batch * (dim / cw);
  if (ctas > INT32_MAX || seqlen > INT32_MAX - sel::kTok || batch > INT32_MAX)
    return SSD_ERR_UNSUPPORTED;
  const bool bf = io == SSD_BF16, ybf = y_dtype == SSD_BF16;
  const CUtensorMapDataType tio = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t L = uint64_t(seqlen), Bn = uint64_t(batch), GN = uint64_t(ngroups) * sel::kN;
  CUtensorMap mx, mdt, mb, mc, my;
  if (!make_box_map(&mx, x, tio, es, dim, L, Bn, uint32_t(cw), sel::kTok) ||
      !make_box_map(&mdt, dt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dim, L, Bn, uint32_t(cw),
                    sel::kTok) ||
      !make_box_map(&mb, B, tio, es, GN, L, Bn, sel::kN, sel::kTok) ||
      !make_box_map(&mc, C, tio, es, GN, L, Bn, sel::kN, sel::kTok) ||
      !make_box_map(&my, y,
                    ybf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    ybf ? 2 : 4, dim, L, Bn, uint32_t(cw), sel::kTok))
    return SSD_ERR_CUDA;
  if (set_smem_attrs() != SSD_OK) return SSD_ERR_CUDA;
  const unsigned grid = unsigned(ctas);
#define SSD_SEL(T, TY)                                                                  \
  sel::selective_scan_kernel<T, TY><<<grid, 32, sel::Smem<T, TY>::kBytes, stream>>>(       \
      mx, mdt, mb, mc, my, A, D, init_state, final_state, seqlen, dim, ngroups)
  if (!bf) SSD_SEL(float, float);
  else if (!ybf) SSD_SEL(__nv_bfloat16, float);
  else SSD_SEL(__nv_bfloat16, __nv_bfloat16);
#undef SSD_SEL
  return launched();
}

ssd_status ssd_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SSD_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, ssd::g_status, sizeof v) != cudaSuccess) return SSD_ERR_CUDA;
  if (v == 0) return SSD_OK;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(ssd::g_status, &zero, sizeof zero) != cudaSuccess) return SSD_ERR_CUDA;
  return static_cast<ssd_status>(v & 0xffu);
}

const char* ssd_version(void) { return "ssd-b200 0.1 sm_100a"; }

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// ssd_chunk_scan_fwd_noalloc: the tensor-core scan with its scratch (the walk's ticket, ready
// flags and published boundary states, and the segments' entering states where the walk needs
// them) in a fixed device array instead of a caller workspace, for callers that cannot allocate
// device memory.  The array lives in every GPU that loads this library until exit.
// ---------------------------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};  // device address of the array, per device

// Once per device, with that device current: the array's device address (host code may not use
// the symbol itself, which on the host is only a stand-in) and the kernels' shared-memory limits.
ssd_status noalloc_setup(void** scratch) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SSD_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SSD_ERR_CUDA;
    }
    const bool ok =
        cudaFuncSetAttribute(ssd::tc::seg_state_kernel<2>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSegSmem<2>)) ==
            cudaSuccess &&
        cudaFuncSetAttribute(ssd::tc::scan_walk_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmem)) ==
            cudaSuccess &&
        cudaFuncSetAttribute(ssd::tc::scan_walk_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmem)) ==
            cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return SSD_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *scratch = g_noalloc_addr[dev];
  return SSD_OK;
}

// The usual plan, or one with fewer CTAs (fewer published states, and fewer segments where
// there are any) when its scratch would not fit in `cap` bytes.  False when none fits.
bool plan_within(const Shape& s, size_t cap, TcPlan* out) {
  for (int ctas = sm_count(); ctas >= 1; ctas /= 2) {
    ScanOpts o;
    o.max_ctas = ctas;
    TcPlan p;
    if (make_tc_plan(s, o, &p) && walk_bytes(s, p) <= cap) {
      *out = p;
      return true;
    }
  }
  return false;
}

}  // namespace

extern "C" ssd_status ssd_chunk_scan_fwd_noalloc(
    const void* x, const float* dt, const float* A, const void* B, const void* C,
    const float* D, const float* init_state, void* y, float* final_state, int64_t batch,
    int64_t seqlen, int nheads, int headdim, int dstate, int ngroups, int chunk, ssd_dtype io,
    ssd_dtype y_dtype, cudaStream_t stream) {
  const Shape s{batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io};
  const ScanArgs a{y_dtype, x, B, C, dt, A, D, init_state, y, final_state, nullptr, 0, stream};
  ssd_status st = check_shape(s);
  if (st != SSD_OK) return st;
  if (!tc_shape_ok(s)) return SSD_ERR_UNSUPPORTED;
  TcPlan plan;
  if (!plan_within(s, SSD_NOALLOC_SCRATCH_BYTES, &plan)) return SSD_ERR_UNSUPPORTED;
  st = validate_scan(s, a, 0);
  if (st != SSD_OK) return st;
  if (!tc_pointers_ok(a)) return SSD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  st = noalloc_setup(&scratch);
  if (st != SSD_OK) return st;
  return run_tc_walk(s, a, plan, scratch);
}
