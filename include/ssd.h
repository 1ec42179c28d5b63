/*
 * ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 SSD layer library (libssd.so).
 *
 * The layer (per batch row b and head h, scalar decay A_h, input-dependent dt, B, C):
 *
 *   h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * B_t x_t^T        (state h: dstate x headdim)
 *   y_t = C_t^T h_t + D_h * x_t
 *
 * equivalently y_t = sum_{s<=t} C_t^T (prod_{k=s+1..t} exp(dt_k A_h)) B_s dt_s x_s + D_h x_t,
 * the lower-triangular semiseparable matrix of "Mamba-2 (2024): SSM e attention sono la
 * stessa cosa" (paithon.it), section "Due modi di guardare la stessa matrice".  The
 * recurrence is the one of "State Space Model" (book.paithon.it), sections "Un sistema
 * che riassume il passato" (decay exp(Delta A), input term Delta B) and "Due strade, una
 * meta" (h_t = A_t h_{t-1} + b_t with a scalar transition); the D x skip term is from
 * "Puntata 205 -- State Space Models e Mamba" (aiperbabbani.it), "Cos'e un SSM".
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are CUDA device pointers owned by the caller (device or managed
 *    memory; anything else is rejected with SSD_ERR_INVALID_ARG before any launch).  The
 *    library never allocates device memory; scratch comes from the caller's workspace.
 *  - Layouts are dense row-major (contiguous):
 *        x            [batch, seqlen, nheads, headdim]   io dtype
 *        y            [batch, seqlen, nheads, headdim]   y dtype
 *        dt           [batch, seqlen, nheads]            float32 (used as given, > 0)
 *        A, D         [nheads]                           float32 (A < 0; D may be NULL = 0)
 *        B, C         [batch, seqlen, ngroups, dstate]   io dtype
 *        states       [batch, nheads, headdim, dstate]   float32; element [b,h,p,n] is h[n,p]
 *    Head h reads group g = h / (nheads / ngroups).
 *  - io dtype (x, B, C): SSD_F32 or SSD_BF16.  y dtype: SSD_F32 or equal to the io dtype.
 *    Arithmetic is float32 with float32 accumulation (tensor-core operands are bf16, split
 *    into a high and a low bf16 part where a single bf16 would cost accuracy); y is written in
 *    its dtype, rounded to nearest even.  A bf16 y carries up to half a bf16 ulp of rounding
 *    (2^-9 relative), so a float32 y is the default of the Python binding.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).  Argument errors are
 *    reported synchronously and nothing is launched.  A launch failure returns
 *    SSD_ERR_CUDA.  Errors found by the kernels themselves (a bounded wait that expired)
 *    are latched in a device status word and reported by ssd_get_device_status().
 *  - Not thread-safe per stream: two calls that share a workspace must be ordered.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1,    /* NULL required pointer, non-device pointer, bad size, aliasing */
  SSD_ERR_UNSUPPORTED = 2,    /* valid but outside what the kernels are built for */
  SSD_ERR_WORKSPACE = 3,      /* workspace NULL or smaller than the query returned */
  SSD_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  SSD_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait expired (see ssd_get_device_status) */
} ssd_status;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/* Which kernels ssd_chunk_scan_fwd uses for a shape. */
typedef enum { SSD_PATH_SIMT = 0, SSD_PATH_TCGEN05 = 1 } ssd_path;

/*
 * Bytes of device workspace ssd_chunk_scan_fwd needs for this shape (0 is possible).
 * Returns 0 as well for invalid arguments; ssd_chunk_scan_fwd then reports the error.
 */
size_t ssd_chunk_scan_workspace_size(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                     int dstate, int ngroups, int chunk, ssd_dtype io);

/* The path ssd_chunk_scan_fwd takes for this shape.  On the tensor-core path x, B, C and y
 * must be 16-byte aligned (TMA tiles); a misaligned pointer there returns
 * SSD_ERR_UNSUPPORTED (ssd_chunk_scan_fwd_simt accepts any element-aligned pointers). */
ssd_path ssd_chunk_scan_path(int64_t batch, int64_t seqlen, int nheads, int headdim,
                             int dstate, int ngroups, int chunk, ssd_dtype io);

/*
 * Chunked forward scan (prefill / training forward): y over the whole sequence and the
 * state after its last token.  The sequence is cut into contiguous blocks; inside a block
 * the output is the masked quadratic (attention-like) form, and only a state summary is
 * passed from block to block ("Il trucco a blocchi" of the Mamba-2 page above; block
 * sizes 64 or 128 per "Rewolucja Mamba-2 i teoria State Space Duality SSD" of the
 * tech.tersel.eu article).  The result does not depend on the block size.
 *
 *   x, dt, A, B, C, D : inputs as above (D may be NULL).
 *   init_state        : [batch, nheads, headdim, dstate] float32, the state before token 0
 *                       (token 0 decays it once); NULL means zeros.
 *   y                 : output [batch, seqlen, nheads, headdim] in y_dtype (SSD_F32 or the io
 *                       dtype); must not overlap any input.
 *   final_state       : output state after token seqlen-1, float32; NULL = not written.
 *                       May equal init_state (in-place streaming prefill).
 *   chunk             : 64, 128 or 256.  The SIMT path uses it as its block length; the
 *                       tensor-core path evaluates 128-token blocks (the tcgen05 M=128
 *                       tile) for every admissible chunk.
 *   seqlen            : >= 1; need not be a multiple of chunk.
 *   Path: io = BF16, headdim = 64, dstate = 128 and an even number of heads per group ->
 *         tcgen05 tensor cores (TMA, TMEM); everything else (including every F32 call) ->
 *         float32 SIMT kernels (headdim <= 256, dstate <= 2048, batch*nheads <= 65535;
 *         larger shapes return SSD_ERR_UNSUPPORTED).
 *   workspace         : device scratch of at least ssd_chunk_scan_workspace_size() bytes,
 *                       256-byte aligned; contents on entry are ignored.
 */
ssd_status ssd_chunk_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                              const void* C, const float* D, const float* init_state, void* y,
                              float* final_state, int64_t batch, int64_t seqlen, int nheads,
                              int headdim, int dstate, int ngroups, int chunk, ssd_dtype io,
                              ssd_dtype y_dtype, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * ssd_chunk_scan_fwd on the tensor-core path with its plan and its kernels' bounded waits under
 * the caller's control -- for tests and tuning; the pages have no counterpart.  opt == NULL (or
 * all fields 0) is exactly ssd_chunk_scan_fwd.
 *   max_ctas       cap on the walk's CTAs (0: one per SM).  Fewer CTAs than (batch row, head
 *                  pair) sequences make ranges that start inside a sequence, so the published
 *                  boundary states are exercised on small shapes.
 *   plan           0 automatic; 1 whole sequences (no summary pass); 2 segments whose entering
 *                  states come from a summary pass (seg_state + seg_pass) before the walk.
 *   wait_limit_ns  limit of every bounded wait in the walk (0: 2 s; -1: no waiting, i.e. a
 *                  wait whose event has not already happened gives up at once).  A wait that
 *                  gives up makes the kernel latch SSD_ERR_DEVICE_TIMEOUT in the device status
 *                  word, let its copies and MMAs land, free its tensor memory and return; y and
 *                  final_state are then undefined, and the next call works normally.
 * Only tensor-core shapes (else SSD_ERR_UNSUPPORTED); max_ctas < 0, plan outside 0..2 or
 * wait_limit_ns < -1 return
 * SSD_ERR_INVALID_ARG.  The workspace must hold ssd_chunk_scan_workspace_size_ex() bytes for
 * the same options.
 */
typedef struct {
  int max_ctas;
  int plan;
  int64_t wait_limit_ns;
} ssd_scan_options;
size_t ssd_chunk_scan_workspace_size_ex(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                        int dstate, int ngroups, int chunk, ssd_dtype io,
                                        const ssd_scan_options* opt);
ssd_status ssd_chunk_scan_fwd_ex(const void* x, const float* dt, const float* A, const void* B,
                                 const void* C, const float* D, const float* init_state,
                                 void* y, float* final_state, int64_t batch, int64_t seqlen,
                                 int nheads, int headdim, int dstate, int ngroups, int chunk,
                                 ssd_dtype io, ssd_dtype y_dtype, void* workspace,
                                 size_t workspace_bytes, const ssd_scan_options* opt,
                                 cudaStream_t stream);

/*
 * How ssd_chunk_scan_fwd (or _ex with `opt`) runs this shape on the tensor cores: the kernels it
 * launches per call, the CTAs of its walk, and the segments each sequence is cut into (1: no
 * summary pass).  Returns SSD_ERR_UNSUPPORTED for shapes that do not take the tensor-core path
 * and SSD_ERR_INVALID_ARG for invalid ones or a NULL `info`.  Host only; launches nothing.
 */
typedef struct {
  int launches;  /* kernels per call (the call also clears a few bytes of workspace with a memset) */
  int ctas;      /* CTAs of the walk */
  int segments;  /* segments per sequence */
} ssd_plan_info;
ssd_status ssd_chunk_scan_plan_info(int64_t batch, int64_t seqlen, int nheads, int headdim,
                                    int dstate, int ngroups, int chunk, ssd_dtype io,
                                    const ssd_scan_options* opt, ssd_plan_info* info);

/* The same operation forced onto the float32 SIMT kernels (any supported shape), with its
 * own workspace query.  Used as a second GPU reference and for float32 io. */
size_t ssd_chunk_scan_simt_workspace_size(int64_t batch, int64_t seqlen, int nheads,
                                          int headdim, int dstate, int ngroups, int chunk,
                                          ssd_dtype io);
ssd_status ssd_chunk_scan_fwd_simt(const void* x, const float* dt, const float* A,
                                   const void* B, const void* C, const float* D,
                                   const float* init_state, void* y, float* final_state,
                                   int64_t batch, int64_t seqlen, int nheads, int headdim,
                                   int dstate, int ngroups, int chunk, ssd_dtype io,
                                   ssd_dtype y_dtype, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * One recurrent step (generation / decode), updating `state` in place:
 *   alpha = exp(dt[b,h] * A[h]);  state[b,h,p,n] = alpha*state[b,h,p,n] + dt[b,h]*x[b,h,p]*B[b,g,n]
 *   y[b,h,p] = sum_n C[b,g,n] * state[b,h,p,n] (updated) + D[h] * x[b,h,p]
 * "State Space Models (SSM)" (ultralytics.com glossary), section "Come funzionano gli SSM":
 * the recurrent form used during generation, constant memory per token.
 *   state [batch, nheads, headdim, dstate] float32 (read and written once per call);
 *   x [batch, nheads, headdim] io dtype; y the same shape in y_dtype (SSD_F32 or io);
 *   dt [batch, nheads] float32;
 *   B, C [batch, ngroups, dstate] io dtype; A, D [nheads] float32 (D may be NULL).
 *   y must not overlap state or any input.  No workspace, no allocation.
 */
ssd_status ssd_step(float* state, const void* x, const float* dt, const float* A,
                    const void* B, const void* C, const float* D, void* y, int64_t batch,
                    int nheads, int headdim, int dstate, int ngroups, ssd_dtype io,
                    ssd_dtype y_dtype, cudaStream_t stream);

/*
 * ssd_chunk_scan_fwd without a workspace argument, for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or forbidden (inside an allocator-free
 * serving loop, a plugin that owns no memory pool, a context whose allocator is locked), or
 * that must not grow the process's device footprint per call.  The pages have no counterpart;
 * this is a deployment convenience around the same tensor-core kernels.
 *
 * Scratch comes from one fixed array of SSD_NOALLOC_SCRATCH_BYTES (32 MiB) that the library
 * holds in every GPU that loads it, until the process exits.  The call allocates nothing.
 *   - Shapes: the tensor-core shapes only (io = SSD_BF16, headdim 64, dstate 128, an even
 *     number of heads per group).  The array holds the walk's bookkeeping and one published
 *     boundary state (64 KiB) per CTA, plus, where sequences are cut into segments, one float32
 *     headdim x dstate state per batch row, segment and head; the call uses fewer CTAs when that
 *     does not fit, and returns SSD_ERR_UNSUPPORTED before launching anything when even a
 *     single CTA's plan does not.  Other shapes also return SSD_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address (and configures the
 *     kernels) for that device; make that first call before any stream capture.
 *   - Every call on a device shares the one array.  Calls whose kernels overlap on the GPU
 *     (different streams without ordering, or several host threads) race on it and give wrong
 *     results: order them.  Each call clears the part that must start at zero (the ticket and
 *     the ready flags) and writes every other scratch value before it reads it.
 * Arguments, layouts and the result are exactly those of ssd_chunk_scan_fwd.
 */
#define SSD_NOALLOC_SCRATCH_BYTES (32u << 20)
ssd_status ssd_chunk_scan_fwd_noalloc(const void* x, const float* dt, const float* A,
                                      const void* B, const void* C, const float* D,
                                      const float* init_state, void* y, float* final_state,
                                      int64_t batch, int64_t seqlen, int nheads, int headdim,
                                      int dstate, int ngroups, int chunk, ssd_dtype io,
                                      ssd_dtype y_dtype, cudaStream_t stream);

/*
 * Gradients of ssd_chunk_scan_fwd (training backward), for L = sum(dy * y) + sum(dfinal *
 * final_state): the chain rule applied to the recurrence, in the same blocked form as the
 * forward ("Mamba-2 (2024): SSM e attention sono la stessa cosa", "Il trucco a blocchi": masked
 * quadratic forms inside each chunk; between chunks only the forward state entering each chunk
 * and the adjoint carried into it from the right).  The pages give no gradient formulas; the
 * all-at-once (parallel) form is the one used for training ("State Space Model"
 * (book.paithon.it), "Un sistema che riassume il passato").
 *   Inputs: x, dt, A, B, C, D, init_state exactly as given to the forward (D and init_state may
 *           be NULL); dy [batch, seqlen, nheads, headdim] float32; dfinal [batch, nheads,
 *           headdim, dstate] float32 or NULL (zero).
 *   Outputs (float32, device, caller-owned, none overlapping an input or another output):
 *           dx [batch, seqlen, nheads, headdim]; ddt [batch, seqlen, nheads]; dA [nheads];
 *           dB, dC [batch, seqlen, ngroups, dstate] (summed over the heads of each group);
 *           dD [nheads] or NULL (not written); dinit [batch, nheads, headdim, dstate] or NULL.
 *   io: SSD_F32 or SSD_BF16 (x, B, C).  Float32 CUDA-core arithmetic throughout, chunks of 64
 *   tokens; the result does not depend on the chunk.  Deterministic (fixed summation orders).
 *   Supported: headdim * dstate small enough for one chunk's tiles in shared memory (headdim 64
 *   with dstate 128, or smaller), batch * nheads <= 65535; else SSD_ERR_UNSUPPORTED.
 *   workspace: ssd_chunk_scan_bwd_workspace_size() bytes, 256-byte aligned.
 * Asynchronous on `stream`; argument errors are returned before any launch.
 */
size_t ssd_chunk_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int nheads,
                                         int headdim, int dstate, int ngroups, ssd_dtype io);
ssd_status ssd_chunk_scan_bwd(const void* x, const float* dt, const float* A, const void* B,
                              const void* C, const float* D, const float* init_state,
                              const float* dy, const float* dfinal, float* dx, float* ddt,
                              float* dA, float* dB, float* dC, float* dD, float* dinit,
                              int64_t batch, int64_t seqlen, int nheads, int headdim, int dstate,
                              int ngroups, ssd_dtype io, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* ssd_status_string(ssd_status s);

/*
 * Summary of a slice of the sequence: the state after its last token and its total log-decay,
 * without y.  Sequence-sliced (multi-GPU) long context: each rank summarises its own slice from
 * a zero state, the summaries are exchanged, ssd_state_pass gives every slice its entering state,
 * and each rank runs ssd_chunk_scan_fwd on its slice from that state.  A slice's steps compose
 * like a single step, h_out = exp(total_decay) h_in + S ("State Space Model", "Un sistema che
 * riassume il passato": steps fuse pairwise by associativity); only these boundary summaries
 * cross between devices ("Architektury Mamba-2, State Space Models i liniowa atencja" of the
 * tech.tersel.eu article, "Wyzwania uczenia rozproszonego").
 *
 *   x, dt, A, B       : as for ssd_chunk_scan_fwd (the slice's tokens).
 *   init_state        : state before the slice's first token, NULL = zeros.
 *   final_state       : output [batch, nheads, headdim, dstate] float32 (required); may equal
 *                       init_state.
 *   total_decay       : output [batch, nheads] float32, sum over the slice of dt[b,t,h]*A[h]
 *                       (natural log; the slice decays a state by exp(total_decay)).
 *   workspace         : ssd_chunk_scan_workspace_size() bytes for the same shape and chunk.
 * Same shapes, paths, errors and asynchrony as ssd_chunk_scan_fwd.
 */
ssd_status ssd_chunk_state_fwd(const void* x, const float* dt, const float* A, const void* B,
                               const float* init_state, float* final_state, float* total_decay,
                               int64_t batch, int64_t seqlen, int nheads, int headdim,
                               int dstate, int ngroups, int chunk, ssd_dtype io,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The state passing between slices: an exclusive scan over slice summaries.
 *   states            : [nslices, batch, nheads, headdim, dstate] float32, in place.  In: each
 *                       slice's state from a zero start (ssd_chunk_state_fwd with init NULL).
 *                       Out: the state entering each slice, H_in(0) = init_state,
 *                       H_in(r+1) = exp(decay[r]) * H_in(r) + S(r).
 *   decay             : [nslices, batch, nheads] float32, each slice's total_decay.
 *   init_state        : [batch, nheads, headdim, dstate] float32 before slice 0, NULL = zeros.
 *   final_state       : output, the state after the last slice (NULL = not written); may equal
 *                       init_state, must not overlap `states`.
 * Any headdim and dstate.  Asynchronous on `stream`; argument errors are returned before any
 * launch.
 */
ssd_status ssd_state_pass(float* states, const float* decay, const float* init_state,
                          float* final_state, int64_t nslices, int64_t batch, int nheads,
                          int headdim, int dstate, cudaStream_t stream);

/*
 * Steps either side of the layer inside a Mamba block ("State Space Models (SSM)"
 * (ultralytics.com glossary), section "Da S4 a Mamba": every Mamba block wraps the selective
 * SSM with a short convolution and a SiLU gate).  silu(v) = v / (1 + exp(-v)).  Float32 arithmetic,
 * outputs rounded to nearest even in their dtype; asynchronous on `stream`; argument errors are
 * returned before any launch.
 *
 * ssd_conv_silu: the short causal depthwise convolution with SiLU, applied to the layer's
 *   inputs (x, and B, C where they come from the same projection):
 *     out[b,t,c] = silu(bias[c] + sum_{k<kwidth} w[c,k] * u[b, t-kwidth+1+k, c]),
 *   u taken as 0 before t = 0 (no history).
 *   u, out : [batch, seqlen, cdim] in `io` (SSD_BF16 or SSD_F32), must not overlap; w
 *   [cdim, kwidth] float32, kwidth 1..8; bias [cdim] float32 or NULL.  cdim a multiple of 8
 *   (bf16) or 4 (f32), u, out and w 16-byte aligned, batch <= 65535 and seqlen <= 64 * 65535,
 *   else SSD_ERR_UNSUPPORTED.  SiLU here uses the hardware exponential and an approximate
 *   divide (a few float32 ulps).
 */
ssd_status ssd_conv_silu(const void* u, const float* w, const float* bias, void* out,
                         int64_t batch, int64_t seqlen, int cdim, int kwidth, ssd_dtype io,
                         cudaStream_t stream);

/* ssd_dt_softplus: the positive step size dt[b,t,h] = softplus(raw[b,t,h] + bias[h]),
 *   softplus(v) = log(1 + exp(v)).  raw, dt [batch, seqlen, nheads] float32 (dt may equal raw);
 *   bias [nheads] float32 or NULL. */
ssd_status ssd_dt_softplus(const float* raw, const float* bias, float* dt, int64_t batch,
                           int64_t seqlen, int nheads, cudaStream_t stream);

/* ssd_gate_silu: the output gate out[i] = y[i] * silu(z[i]) over n elements (y as the layer
 *   writes it, [batch, seqlen, nheads, headdim]).  y float32; z in z_dtype (SSD_BF16 or SSD_F32);
 *   out in out_dtype (SSD_F32 or z_dtype).  out may equal y only when out_dtype is SSD_F32 (a
 *   narrower out in place would overwrite y elements before they are read: SSD_ERR_INVALID_ARG);
 *   otherwise it must not overlap y or z.  n a multiple of 8 (bf16 z) or 4 (f32 z) and all
 *   pointers 16-byte aligned, else SSD_ERR_UNSUPPORTED. */
ssd_status ssd_gate_silu(const float* y, const void* z, void* out, int64_t n, ssd_dtype z_dtype,
                         ssd_dtype out_dtype, cudaStream_t stream);

/*
 * ssd_selective_scan_fwd: the selective scan with a per-state (diagonal) transition -- the
 * first Mamba generation's layer, which the SSD layer replaces ("Architektury Mamba-2, State
 * Space Models i liniowa atencja" (tech.tersel.eu), section "Od S4 do Mamba-1: Wprowadzenie
 * mechanizmu selektywnego": input-dependent B, C and dt, scanned on CUDA cores with the state on
 * chip).  Per batch row b and channel d, with g = d / (dim / ngroups):
 *     h_t[n] = exp(dt_t[d] A[d,n]) h_{t-1}[n] + dt_t[d] B_t[g,n] x_t[d]
 *     y_t[d] = sum_n C_t[g,n] h_t[n] + D[d] x_t[d]          (h_{-1} = init_state or 0)
 *   x            : [batch, seqlen, dim] in `io` (SSD_BF16 or SSD_F32)
 *   dt           : [batch, seqlen, dim] float32, used as given
 *   A            : [dim, dstate] float32 (one decay rate per channel and state)
 *   B, C         : [batch, seqlen, ngroups, dstate] in `io`
 *   D            : [dim] float32, or NULL for no skip term
 *   init_state   : [batch, dim, dstate] float32, or NULL for zeros
 *   y            : output [batch, seqlen, dim] in y_dtype (SSD_F32 or `io`)
 *   final_state  : output [batch, dim, dstate] float32, or NULL; may equal init_state
 * All pointers are device memory owned by the caller; y and final_state must not overlap the
 * inputs.  Float32 arithmetic, hardware exp2 for the decays; asynchronous on `stream`.
 * Supported: dstate == 16, dim and dim / ngroups multiples of 8, every pointer 16-byte aligned
 * (else SSD_ERR_UNSUPPORTED).  Argument errors are returned before any launch; the kernel's
 * waits on its TMA tiles are bounded, and an expired wait is reported by
 * ssd_get_device_status (the final state is then not written).
 */
ssd_status ssd_selective_scan_fwd(const void* x, const float* dt, const float* A, const void* B,
                                  const void* C, const float* D, const float* init_state,
                                  void* y, float* final_state, int64_t batch, int64_t seqlen,
                                  int dim, int dstate, int ngroups, ssd_dtype io,
                                  ssd_dtype y_dtype, cudaStream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word that kernels latch
 * when a bounded wait expires (for the current device).  Returns SSD_OK,
 * SSD_ERR_DEVICE_TIMEOUT, or SSD_ERR_CUDA if the synchronisation itself failed.
 */
ssd_status ssd_get_device_status(cudaStream_t stream);

/* Library version string, e.g. "ssd-b200 0.1 sm_100a". */
const char* ssd_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SSD_H_ */
