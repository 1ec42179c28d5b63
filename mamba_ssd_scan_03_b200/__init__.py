"""B200 (sm_100a) Mamba-2 SSD layer: thin Python binding over the C ABI in include/ssd.h.

Every step of the computation runs in the CUDA kernels of ``libssd.so``; this module only
checks tensors, allocates outputs and workspace with PyTorch (device memory and streams are
PyTorch's job here), and passes raw pointers plus the current CUDA stream.  There is no CPU
path: if the library is missing or no CUDA device is present, the calls raise.

    y, final_state = chunk_scan_fwd(x, dt, A, B, C, D, chunk, init_state=None)
    y = step(state, x, dt, A, B, C, D)          # updates `state` in place
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
SSD_PATH_SIMT, SSD_PATH_TCGEN05 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED",
          3: "SSD_ERR_WORKSPACE", 4: "SSD_ERR_CUDA", 5: "SSD_ERR_DEVICE_TIMEOUT"}

# The symbols include/ssd.h declares (tests check that the library exports each one).
EXPORTS = ("ssd_chunk_scan_workspace_size", "ssd_chunk_scan_path", "ssd_chunk_scan_fwd",
           "ssd_chunk_scan_simt_workspace_size", "ssd_chunk_scan_fwd_simt", "ssd_step",
           "ssd_chunk_scan_fwd_noalloc", "ssd_chunk_scan_workspace_size_ex",
           "ssd_chunk_scan_fwd_ex", "ssd_chunk_scan_plan_info",
           "ssd_chunk_scan_bwd_workspace_size", "ssd_chunk_scan_bwd", "ssd_chunk_state_fwd",
           "ssd_state_pass",
           "ssd_conv_silu", "ssd_dt_softplus", "ssd_gate_silu", "ssd_selective_scan_fwd",
           "ssd_status_string",
           "ssd_get_device_status", "ssd_version")

# Size of the fixed device array ssd_chunk_scan_fwd_noalloc uses instead of a workspace.
NOALLOC_SCRATCH_BYTES = 32 << 20


class SSDError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_status_string(code)})")


_lib = None

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SHAPE = [_i64, _i64, _i32, _i32, _i32, _i32, _i32, _i32]  # batch .. chunk, io
_SCAN = [_vp] * 9 + [_i64, _i64, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]


class PlanInfo(ctypes.Structure):
    """ssd_plan_info: kernels per call, CTAs of the walk, segments per sequence."""
    _fields_ = [("launches", ctypes.c_int), ("ctas", ctypes.c_int), ("segments", ctypes.c_int)]


class ScanOptions(ctypes.Structure):
    """ssd_scan_options: the walk's plan and wait limit (tests and tuning; zeros = defaults)."""
    _fields_ = [("max_ctas", ctypes.c_int), ("plan", ctypes.c_int),
                ("wait_limit_ns", ctypes.c_int64)]


def load():
    """Load libssd.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m mamba_ssd_scan_03_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.ssd_chunk_scan_workspace_size.restype = _sz
    lib.ssd_chunk_scan_workspace_size.argtypes = _SHAPE
    lib.ssd_chunk_scan_simt_workspace_size.restype = _sz
    lib.ssd_chunk_scan_simt_workspace_size.argtypes = _SHAPE
    lib.ssd_chunk_scan_path.restype = _i32
    lib.ssd_chunk_scan_path.argtypes = _SHAPE
    for fn in (lib.ssd_chunk_scan_fwd, lib.ssd_chunk_scan_fwd_simt):
        fn.restype = _i32
        fn.argtypes = _SCAN
    lib.ssd_chunk_scan_workspace_size_ex.restype = _sz
    lib.ssd_chunk_scan_workspace_size_ex.argtypes = _SHAPE + [ctypes.POINTER(ScanOptions)]
    lib.ssd_chunk_scan_plan_info.restype = _i32
    lib.ssd_chunk_scan_plan_info.argtypes = _SHAPE + [ctypes.POINTER(ScanOptions),
                                                      ctypes.POINTER(PlanInfo)]
    lib.ssd_chunk_scan_fwd_ex.restype = _i32
    lib.ssd_chunk_scan_fwd_ex.argtypes = _SCAN[:-1] + [ctypes.POINTER(ScanOptions), _vp]
    lib.ssd_chunk_scan_fwd_noalloc.restype = _i32
    lib.ssd_chunk_scan_fwd_noalloc.argtypes = [_vp] * 9 + [_i64, _i64] + [_i32] * 7 + [_vp]
    lib.ssd_chunk_scan_bwd_workspace_size.restype = _sz
    lib.ssd_chunk_scan_bwd_workspace_size.argtypes = [_i64, _i64] + [_i32] * 5
    lib.ssd_chunk_scan_bwd.restype = _i32
    lib.ssd_chunk_scan_bwd.argtypes = [_vp] * 16 + [_i64, _i64] + [_i32] * 5 + [_vp, _sz, _vp]
    lib.ssd_chunk_state_fwd.restype = _i32
    lib.ssd_chunk_state_fwd.argtypes = [_vp] * 7 + [_i64, _i64] + [_i32] * 6 + [_vp, _sz, _vp]
    lib.ssd_state_pass.restype = _i32
    lib.ssd_state_pass.argtypes = [_vp] * 4 + [_i64, _i64, _i32, _i32, _i32, _vp]
    lib.ssd_conv_silu.restype = _i32
    lib.ssd_conv_silu.argtypes = [_vp] * 4 + [_i64, _i64, _i32, _i32, _i32, _vp]
    lib.ssd_dt_softplus.restype = _i32
    lib.ssd_dt_softplus.argtypes = [_vp] * 3 + [_i64, _i64, _i32, _vp]
    lib.ssd_gate_silu.restype = _i32
    lib.ssd_gate_silu.argtypes = [_vp] * 3 + [_i64, _i32, _i32, _vp]
    lib.ssd_selective_scan_fwd.restype = _i32
    lib.ssd_selective_scan_fwd.argtypes = [_vp] * 9 + [_i64, _i64, _i32, _i32, _i32, _i32,
                                                       _i32, _vp]
    lib.ssd_step.restype = _i32
    lib.ssd_step.argtypes = [_vp] * 8 + [_i64, _i32, _i32, _i32, _i32, _i32, _i32, _vp]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [_i32]
    lib.ssd_get_device_status.restype = _i32
    lib.ssd_get_device_status.argtypes = [_vp]
    lib.ssd_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _status_string(code):
    try:
        return load().ssd_status_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(code, what):
    if code != 0:
        raise SSDError(code, what)


def _io(t):
    return _code(t.dtype)


def _code(dtype):
    if dtype == torch.bfloat16:
        return SSD_BF16
    if dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"tensor dtype must be bfloat16 or float32, got {dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _scan_shape(x, B, chunk):
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return Bt, L, H, P, N, G, int(chunk), _io(x)


def workspace_size(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io=SSD_BF16,
                   simt=False):
    fn = load().ssd_chunk_scan_simt_workspace_size if simt else \
        load().ssd_chunk_scan_workspace_size
    return fn(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io)


def plan_info(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io=SSD_BF16, max_ctas=0,
              plan=0):
    """The tensor-core plan of a shape: dict(launches, ctas, segments)."""
    info = PlanInfo()
    opts = ScanOptions(int(max_ctas), int(plan), 0)
    rc = load().ssd_chunk_scan_plan_info(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                                         io, ctypes.byref(opts), ctypes.byref(info))
    _check(rc, "ssd_chunk_scan_plan_info")
    return dict(launches=info.launches, ctas=info.ctas, segments=info.segments)


def path(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io=SSD_BF16):
    return load().ssd_chunk_scan_path(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, io)


def _scan(entry, simt, x, dt, A, B, C, D, chunk, init_state, want_final, workspace, out,
          final_out, y_dtype, opts=None):
    lib = load()
    _need(x, "x")
    dev = x.device
    Bt, L, H, P, N, G, Q, io = _scan_shape(x, B, chunk)
    _need(B, "B", x.dtype, (Bt, L, G, N), dev)
    _need(C, "C", x.dtype, (Bt, L, G, N), dev)
    _need(dt, "dt", torch.float32, (Bt, L, H), dev)
    _need(A, "A", torch.float32, (H,), dev)
    if D is not None:
        _need(D, "D", torch.float32, (H,), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, H, P, N), dev)
    y_dtype = out.dtype if out is not None else y_dtype
    y = out if out is not None else torch.empty(x.shape, dtype=y_dtype, device=dev)
    _need(y, "out", y_dtype, x.shape, dev)
    fin = None
    if want_final:
        fin = final_out if final_out is not None else torch.empty(
            (Bt, H, P, N), dtype=torch.float32, device=dev)
        _need(fin, "final_state", torch.float32, (Bt, H, P, N), dev)
    if opts is None:
        need = workspace_size(Bt, L, H, P, N, G, Q, io, simt=simt)
    else:
        need = lib.ssd_chunk_scan_workspace_size_ex(Bt, L, H, P, N, G, Q, io, ctypes.byref(opts))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    extra = () if opts is None else (ctypes.byref(opts),)
    with torch.cuda.device(dev):
        rc = entry(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                   _ptr(y), _ptr(fin), Bt, L, H, P, N, G, Q, io, _code(y_dtype), _ptr(workspace),
                   workspace.numel(), *extra, _stream(dev))
    _check(rc, getattr(entry, "__name__", "ssd_chunk_scan_fwd"))
    return y, fin


def chunk_scan_fwd(x, dt, A, B, C, D, chunk, init_state=None, want_final=True,
                   workspace=None, out=None, final_out=None, y_dtype=torch.float32):
    """Chunked forward scan.  x [B,L,H,P], dt [B,L,H] f32, A [H] f32, B/C [B,L,G,N],
    D [H] f32 or None, init_state [B,H,P,N] f32 or None.  y is float32 by default (or the io
    dtype).  Returns (y, final_state)."""
    return _scan(load().ssd_chunk_scan_fwd, False, x, dt, A, B, C, D, chunk, init_state,
                 want_final, workspace, out, final_out, y_dtype)


def chunk_scan_fwd_ex(x, dt, A, B, C, D, chunk, init_state=None, want_final=True,
                      workspace=None, out=None, final_out=None, y_dtype=torch.float32,
                      max_ctas=0, plan=0, wait_limit_ns=0):
    """ssd_chunk_scan_fwd_ex: the tensor-core scan with its plan (max_ctas, plan 0 auto / 1
    whole sequences / 2 segments) and the kernels' wait limit set by the caller (tests)."""
    opts = ScanOptions(int(max_ctas), int(plan), int(wait_limit_ns))
    return _scan(load().ssd_chunk_scan_fwd_ex, False, x, dt, A, B, C, D, chunk, init_state,
                 want_final, workspace, out, final_out, y_dtype, opts)


def chunk_scan_fwd_simt(x, dt, A, B, C, D, chunk, init_state=None, want_final=True,
                        workspace=None, out=None, final_out=None, y_dtype=torch.float32):
    """The same operation on the float32 SIMT kernels (second GPU reference)."""
    return _scan(load().ssd_chunk_scan_fwd_simt, True, x, dt, A, B, C, D, chunk, init_state,
                 want_final, workspace, out, final_out, y_dtype)


def chunk_scan_fwd_noalloc(x, dt, A, B, C, D, chunk, init_state=None, want_final=True,
                           out=None, final_out=None, y_dtype=torch.float32):
    """The chunked scan for callers that cannot allocate device memory: the library's scratch
    lives in a fixed 32 MiB device array (NOALLOC_SCRATCH_BYTES) instead of a workspace.
    Tensor-core shapes only.  Calls that overlap on the GPU share that array and race, so
    order them; the first call on a device sets the array up and should precede any stream
    capture.  (This wrapper still allocates y and the final state with PyTorch unless `out`
    and `final_out` are given.)"""
    lib = load()
    _need(x, "x")
    dev = x.device
    Bt, L, H, P, N, G, Q, io = _scan_shape(x, B, chunk)
    _need(B, "B", x.dtype, (Bt, L, G, N), dev)
    _need(C, "C", x.dtype, (Bt, L, G, N), dev)
    _need(dt, "dt", torch.float32, (Bt, L, H), dev)
    _need(A, "A", torch.float32, (H,), dev)
    if D is not None:
        _need(D, "D", torch.float32, (H,), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, H, P, N), dev)
    y_dtype = out.dtype if out is not None else y_dtype
    y = out if out is not None else torch.empty(x.shape, dtype=y_dtype, device=dev)
    _need(y, "out", y_dtype, x.shape, dev)
    fin = None
    if want_final:
        fin = final_out if final_out is not None else torch.empty(
            (Bt, H, P, N), dtype=torch.float32, device=dev)
        _need(fin, "final_state", torch.float32, (Bt, H, P, N), dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_chunk_scan_fwd_noalloc(
            _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(y),
            _ptr(fin), Bt, L, H, P, N, G, Q, io, _code(y_dtype), _stream(dev))
    _check(rc, "ssd_chunk_scan_fwd_noalloc")
    return y, fin


def chunk_scan_bwd(x, dt, A, B, C, D, dy, init_state=None, dfinal=None, workspace=None):
    """Gradients of L = sum(dy * y) + sum(dfinal * final_state) through the chunked scan.
    Inputs as for chunk_scan_fwd; dy [B,L,H,P] f32; dfinal [B,H,P,N] f32 or None.  Returns a
    dict of float32 tensors: x, dt, A, B, C, D, init (the gradient of each input)."""
    lib = load()
    _need(x, "x")
    dev = x.device
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = _io(x)
    _need(B, "B", x.dtype, (Bt, L, G, N), dev)
    _need(C, "C", x.dtype, (Bt, L, G, N), dev)
    _need(dt, "dt", torch.float32, (Bt, L, H), dev)
    _need(A, "A", torch.float32, (H,), dev)
    _need(dy, "dy", torch.float32, (Bt, L, H, P), dev)
    if D is not None:
        _need(D, "D", torch.float32, (H,), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, H, P, N), dev)
    if dfinal is not None:
        _need(dfinal, "dfinal", torch.float32, (Bt, H, P, N), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"x": torch.empty((Bt, L, H, P), **f32), "dt": torch.empty((Bt, L, H), **f32),
         "A": torch.empty((H,), **f32), "B": torch.empty((Bt, L, G, N), **f32),
         "C": torch.empty((Bt, L, G, N), **f32), "D": torch.empty((H,), **f32),
         "init": torch.empty((Bt, H, P, N), **f32)}
    need = lib.ssd_chunk_scan_bwd_workspace_size(Bt, L, H, P, N, G, io)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_chunk_scan_bwd(
            _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(dy),
            _ptr(dfinal), _ptr(g["x"]), _ptr(g["dt"]), _ptr(g["A"]), _ptr(g["B"]), _ptr(g["C"]),
            _ptr(g["D"]), _ptr(g["init"]), Bt, L, H, P, N, G, io, _ptr(workspace),
            workspace.numel(), _stream(dev))
    _check(rc, "ssd_chunk_scan_bwd")
    return g


def chunk_state_fwd(x, dt, A, B, chunk, init_state=None, workspace=None, final_out=None):
    """Summary of a slice of the sequence: (final_state [B,H,P,N] f32, total_decay [B,H] f32 =
    sum_t dt*A) from init_state (None = zeros), without y."""
    lib = load()
    _need(x, "x")
    dev = x.device
    Bt, L, H, P, N, G, Q, io = _scan_shape(x, B, chunk)
    _need(B, "B", x.dtype, (Bt, L, G, N), dev)
    _need(dt, "dt", torch.float32, (Bt, L, H), dev)
    _need(A, "A", torch.float32, (H,), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, H, P, N), dev)
    fin = final_out if final_out is not None else torch.empty(
        (Bt, H, P, N), dtype=torch.float32, device=dev)
    _need(fin, "final_state", torch.float32, (Bt, H, P, N), dev)
    dec = torch.empty((Bt, H), dtype=torch.float32, device=dev)
    need = workspace_size(Bt, L, H, P, N, G, Q, io)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_chunk_state_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(init_state),
                                     _ptr(fin), _ptr(dec), Bt, L, H, P, N, G, Q, io,
                                     _ptr(workspace), workspace.numel(), _stream(dev))
    _check(rc, "ssd_chunk_state_fwd")
    return fin, dec


def state_pass(states, decay, init_state=None, final_out=None):
    """Exclusive scan over slice summaries.  states [R,B,H,P,N] f32 (each slice's state from a
    zero start) becomes, in place, the state entering each slice; decay [R,B,H] f32.  Returns
    the state after the last slice."""
    lib = load()
    _need(states, "states", torch.float32)
    dev = states.device
    R, Bt, H, P, N = states.shape
    _need(decay, "decay", torch.float32, (R, Bt, H), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, H, P, N), dev)
    fin = final_out if final_out is not None else torch.empty(
        (Bt, H, P, N), dtype=torch.float32, device=dev)
    _need(fin, "final_state", torch.float32, (Bt, H, P, N), dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_state_pass(_ptr(states), _ptr(decay), _ptr(init_state), _ptr(fin), R, Bt,
                                H, P, N, _stream(dev))
    _check(rc, "ssd_state_pass")
    return fin


def conv_silu(u, w, bias=None, out=None):
    """Short causal depthwise convolution + SiLU: u [B,L,C] (bf16 or f32), w [C,K] f32,
    bias [C] f32 or None -> out [B,L,C] in u's dtype."""
    lib = load()
    _need(u, "u")
    dev = u.device
    Bt, L, Cd = u.shape
    K = w.shape[1]
    _need(w, "w", torch.float32, (Cd, K), dev)
    if bias is not None:
        _need(bias, "bias", torch.float32, (Cd,), dev)
    out = torch.empty_like(u) if out is None else out
    _need(out, "out", u.dtype, u.shape, dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_conv_silu(_ptr(u), _ptr(w), _ptr(bias), _ptr(out), Bt, L, Cd, K, _io(u),
                               _stream(dev))
    _check(rc, "ssd_conv_silu")
    return out


def dt_softplus(raw, bias=None, out=None):
    """dt = softplus(raw + bias): raw [B,L,H] f32, bias [H] f32 or None -> dt [B,L,H] f32."""
    lib = load()
    _need(raw, "raw", torch.float32)
    dev = raw.device
    Bt, L, H = raw.shape
    if bias is not None:
        _need(bias, "bias", torch.float32, (H,), dev)
    out = torch.empty_like(raw) if out is None else out
    _need(out, "out", torch.float32, raw.shape, dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_dt_softplus(_ptr(raw), _ptr(bias), _ptr(out), Bt, L, H, _stream(dev))
    _check(rc, "ssd_dt_softplus")
    return out


def gate_silu(y, z, out=None, out_dtype=torch.float32):
    """Output gate y * silu(z): y f32, z (bf16 or f32) of the same shape -> out (f32 or z's
    dtype)."""
    lib = load()
    _need(y, "y", torch.float32)
    dev = y.device
    _need(z, "z", None, y.shape, dev)
    out_dtype = out.dtype if out is not None else out_dtype
    out = torch.empty(y.shape, dtype=out_dtype, device=dev) if out is None else out
    _need(out, "out", out_dtype, y.shape, dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_gate_silu(_ptr(y), _ptr(z), _ptr(out), y.numel(), _io(z), _code(out_dtype),
                               _stream(dev))
    _check(rc, "ssd_gate_silu")
    return out


def selective_scan_fwd(x, dt, A, B, C, D=None, init_state=None, want_final=True, out=None,
                       y_dtype=torch.float32, final_out=None):
    """Selective scan with a per-state transition: x [Bt,L,dim] (bf16 or f32), dt [Bt,L,dim]
    f32, A [dim,N] f32, B, C [Bt,L,G,N] in x's dtype, D [dim] f32 or None, init_state
    [Bt,dim,N] f32 or None -> (y [Bt,L,dim] in y_dtype, final state [Bt,dim,N] f32 or None)."""
    lib = load()
    _need(x, "x")
    dev = x.device
    Bt, L, dim = x.shape
    _need(dt, "dt", torch.float32, (Bt, L, dim), dev)
    _need(A, "A", torch.float32, None, dev)
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError(f"A must be [dim, dstate] with dim {dim}, got {tuple(A.shape)}")
    N = A.shape[1]
    _need(B, "B", x.dtype, None, dev)
    if B.dim() != 4 or tuple(B.shape[:2]) != (Bt, L) or B.shape[3] != N:
        raise ValueError(f"B must be [{Bt},{L},G,{N}], got {tuple(B.shape)}")
    G = B.shape[2]
    _need(C, "C", x.dtype, B.shape, dev)
    if D is not None:
        _need(D, "D", torch.float32, (dim,), dev)
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (Bt, dim, N), dev)
    y_dtype = out.dtype if out is not None else y_dtype
    y = torch.empty((Bt, L, dim), dtype=y_dtype, device=dev) if out is None else out
    _need(y, "out", y_dtype, (Bt, L, dim), dev)
    fin = None
    if want_final:
        fin = torch.empty((Bt, dim, N), dtype=torch.float32, device=dev) \
            if final_out is None else final_out
        _need(fin, "final_out", torch.float32, (Bt, dim, N), dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_selective_scan_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                        _ptr(init_state), _ptr(y), _ptr(fin), Bt, L, dim, N, G,
                                        _io(x), _code(y_dtype), _stream(dev))
    _check(rc, "ssd_selective_scan_fwd")
    return y, fin


def step(state, x, dt, A, B, C, D, out=None, y_dtype=torch.float32):
    """One decode step; updates ``state`` [B,H,P,N] f32 in place and returns y [B,H,P]
    (float32 by default, or the io dtype)."""
    lib = load()
    _need(state, "state", torch.float32)
    dev = state.device
    Bt, H, P, N = state.shape
    io = _io(x)
    _need(x, "x", x.dtype, (Bt, H, P), dev)
    G = B.shape[1]
    _need(B, "B", x.dtype, (Bt, G, N), dev)
    _need(C, "C", x.dtype, (Bt, G, N), dev)
    _need(dt, "dt", torch.float32, (Bt, H), dev)
    _need(A, "A", torch.float32, (H,), dev)
    if D is not None:
        _need(D, "D", torch.float32, (H,), dev)
    y_dtype = out.dtype if out is not None else y_dtype
    y = out if out is not None else torch.empty(x.shape, dtype=y_dtype, device=dev)
    _need(y, "out", y_dtype, x.shape, dev)
    with torch.cuda.device(dev):
        rc = lib.ssd_step(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                          _ptr(y), Bt, H, P, N, G, io, _code(y_dtype), _stream(dev))
    _check(rc, "ssd_step")
    return y


def device_status(device=None):
    """Synchronise the current stream and read/clear the kernels' device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return load().ssd_get_device_status(_stream(dev))


def version():
    return load().ssd_version().decode()
