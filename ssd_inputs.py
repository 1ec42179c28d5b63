"""Seeded synthetic inputs for the SSD layer, shared by the tests, the oracle checks and bench.py.

This module holds none of the layer's arithmetic: it only draws random tensors with the
distributions of the five workloads and stores them in their storage dtypes.  Both the CUDA
path and the float64 oracle read exactly the stored bits, so the bits (not the RNG) are the
parity surface.

Recipe (per workload, seed = 1000 + workload index unless given):
  SeedSequence(seed).spawn(8) -> child streams, in order: x, dt, A, B, C, D, init, decode
  x ~ N(0, 1)                        [batch, seqlen, nheads, headdim]
  dt = softplus(z), z ~ N(-2, 0.5)   [batch, seqlen, nheads]      (softplus(z) = ln(1 + e^z))
  A_h = -exp(u), u ~ U(ln 1, ln 16)  [nheads]                     (so A in [-16, -1])
  B, C ~ N(0, 1) / sqrt(dstate)      [batch, seqlen, ngroups, dstate]
  D ~ N(0, 1)                        [nheads]
  init ~ N(0, 0.1) (std 0.1) or zeros, [batch, nheads, headdim, dstate]
Draws are float64; storage: x, B, C in the io dtype (bf16 as uint16 bit patterns, rounded
to nearest even through float32), dt, A, D, init in float32.  Large tensors are drawn in
slabs of SLAB_TOKENS tokens from one generator, so a tensor's values do not depend on how
many slabs it takes.  Decode inputs for step k come from the decode child's k-th spawn.
"""
import math

import numpy as np

SLAB_TOKENS = 1 << 16

# The five workloads (name, shapes, dtypes, initial state).
CONFIGS = [
    dict(name="tiny_f32", batch=1, seqlen=256, nheads=4, headdim=16, dstate=16, ngroups=1,
         chunk=64, io="f32", init="zeros"),
    dict(name="mamba2_130m_layer", batch=8, seqlen=2048, nheads=24, headdim=64, dstate=128,
         ngroups=1, chunk=256, io="bf16", init="zeros"),
    dict(name="mamba2_2p7b_layer", batch=4, seqlen=8192, nheads=80, headdim=64, dstate=128,
         ngroups=1, chunk=256, io="bf16", init="normal0.1"),
    dict(name="million_token_context", batch=1, seqlen=1 << 20, nheads=24, headdim=64,
         dstate=128, ngroups=1, chunk=256, io="bf16", init="zeros"),
    dict(name="recurrent_decode", batch=256, seqlen=1, nheads=80, headdim=64, dstate=128,
         ngroups=1, chunk=None, io="bf16", init="normal0.1", decode_steps=1000),
]


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _store(a64, io):
    a32 = a64.astype(np.float32)
    return f32_to_bf16_bits(a32) if io == "bf16" else a32


def _softplus(z):
    return np.log1p(np.exp(-np.abs(z))) + np.maximum(z, 0.0)


def _normal_slabs(gen, shape, io, scale=1.0, mean=0.0):
    """Draw N(mean, scale) of ``shape`` (token axis = 1) slab by slab, store in io dtype."""
    out_dtype = np.uint16 if io == "bf16" else np.float32
    out = np.empty(shape, dtype=out_dtype)
    bsz, L = shape[0], shape[1]
    for b in range(bsz):
        for t0 in range(0, L, SLAB_TOKENS):
            t1 = min(L, t0 + SLAB_TOKENS)
            z = gen.standard_normal((t1 - t0,) + tuple(shape[2:]))
            out[b, t0:t1] = _store(mean + scale * z, io)
    return out


def resolve(cfg, **overrides):
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    cfg = dict(cfg)
    cfg.update({k: v for k, v in overrides.items() if v is not None})
    return cfg


def make_scan_inputs(cfg, seed=None, **overrides):
    """Inputs of one chunked-scan workload.  ``cfg`` is an index into CONFIGS or a dict;
    keyword overrides (seqlen=..., nheads=..., A_range=(lo, hi), init=...) change a copy.

    Returns a dict: x, dt, A, B, C, D, init (None for zeros) plus the resolved cfg.
    """
    idx = cfg if isinstance(cfg, int) else None
    a_range = overrides.pop("A_range", None)
    cfg = resolve(cfg, **overrides)
    if seed is None:
        seed = 1000 + (idx if idx is not None else 0)
    kids = np.random.SeedSequence(seed).spawn(8)
    g = [np.random.Generator(np.random.PCG64(k)) for k in kids]
    Bt, L, H, P = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"]
    G, N, io = cfg["ngroups"], cfg["dstate"], cfg["io"]
    x = _normal_slabs(g[0], (Bt, L, H, P), io)
    dt = np.empty((Bt, L, H), dtype=np.float32)
    for b in range(Bt):
        for t0 in range(0, L, SLAB_TOKENS):
            t1 = min(L, t0 + SLAB_TOKENS)
            dt[b, t0:t1] = _softplus(-2.0 + 0.5 * g[1].standard_normal((t1 - t0, H)))
    lo, hi = a_range if a_range is not None else (1.0, 16.0)
    A = (-np.exp(g[2].uniform(math.log(lo), math.log(hi), size=H))).astype(np.float32)
    B = _normal_slabs(g[3], (Bt, L, G, N), io, scale=1.0 / math.sqrt(N))
    C = _normal_slabs(g[4], (Bt, L, G, N), io, scale=1.0 / math.sqrt(N))
    D = g[5].standard_normal(H).astype(np.float32)
    init = None
    if cfg["init"] == "normal0.1":
        init = (0.1 * g[6].standard_normal((Bt, H, P, N))).astype(np.float32)
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, init=init, cfg=cfg)


def make_decode_inputs(cfg=4, seed=None, **overrides):
    """Fixed parts of the decode workload: A, D and the initial fp32 state, plus cfg."""
    idx = cfg if isinstance(cfg, int) else None
    cfg = resolve(cfg, **overrides)
    if seed is None:
        seed = 1000 + (idx if idx is not None else 4)
    kids = np.random.SeedSequence(seed).spawn(8)
    g = [np.random.Generator(np.random.PCG64(k)) for k in kids]
    Bt, H, P, N = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    A = (-np.exp(g[2].uniform(0.0, math.log(16.0), size=H))).astype(np.float32)
    D = g[5].standard_normal(H).astype(np.float32)
    state = np.empty((Bt, H, P, N), dtype=np.float32)
    for b in range(Bt):
        state[b] = 0.1 * g[6].standard_normal((H, P, N))
    return dict(A=A, D=D, state=state, cfg=cfg, step_seeds=kids[7])


def decode_step_inputs(dec, k):
    """Per-step decode inputs (x, dt, B, C) of step k (0-based) from the decode child stream."""
    cfg = dec["cfg"]
    Bt, H, P, N, G, io = (cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                          cfg["ngroups"], cfg["io"])
    ss = np.random.SeedSequence(entropy=dec["step_seeds"].entropy,
                                spawn_key=tuple(dec["step_seeds"].spawn_key) + (k,))
    gen = np.random.Generator(np.random.PCG64(ss))
    x = _store(gen.standard_normal((Bt, H, P)), io)
    dt = _softplus(-2.0 + 0.5 * gen.standard_normal((Bt, H))).astype(np.float32)
    B = _store(gen.standard_normal((Bt, G, N)) / math.sqrt(N), io)
    C = _store(gen.standard_normal((Bt, G, N)) / math.sqrt(N), io)
    return dict(x=x, dt=dt, B=B, C=C)


def make_glue_inputs(batch, seqlen, cdim, kwidth, nheads, headdim, io="bf16", seed=2000):
    """Inputs of the block steps around the layer.

      u ~ N(0, 1)                 [batch, seqlen, cdim]   (io dtype) convolution input
      w ~ N(0, 1) / sqrt(kwidth)  [cdim, kwidth]          float32
      conv_bias ~ N(0, 0.1)       [cdim]                  float32
      raw ~ N(0, 1)               [batch, seqlen, nheads] float32 (dt projection output)
      dt_bias ~ U(-6, -2)         [nheads]                float32
      y ~ N(0, 1)                 [batch, seqlen, nheads, headdim] float32
      z ~ N(0, 1)                 [batch, seqlen, nheads, headdim] (io dtype) gate branch
    """
    kids = np.random.SeedSequence(seed).spawn(7)
    g = [np.random.Generator(np.random.PCG64(k)) for k in kids]
    u = _normal_slabs(g[0], (batch, seqlen, cdim), io)
    w = (g[1].standard_normal((cdim, kwidth)) / math.sqrt(kwidth)).astype(np.float32)
    conv_bias = (0.1 * g[2].standard_normal(cdim)).astype(np.float32)
    raw = _normal_slabs(g[3], (batch, seqlen, nheads), "f32")
    dt_bias = g[4].uniform(-6.0, -2.0, size=nheads).astype(np.float32)
    y = _normal_slabs(g[5], (batch, seqlen, nheads, headdim), "f32")
    z = _normal_slabs(g[6], (batch, seqlen, nheads, headdim), io)
    return dict(u=u, w=w, conv_bias=conv_bias, raw=raw, dt_bias=dt_bias, y=y, z=z, io=io)


# Selective scan with a per-state transition (the first Mamba generation): the same x and y
# as the 2.7B-shape SSD workload (5120 = 80 x 64 channels), 16 states per channel.
SELECTIVE_CONFIGS = [
    dict(name="selective_small", batch=2, seqlen=300, dim=64, dstate=16, ngroups=1, io="bf16",
         init="normal0.1"),
    dict(name="selective_5120x16", batch=4, seqlen=8192, dim=5120, dstate=16, ngroups=1,
         io="bf16", init="zeros"),
]


def make_selective_inputs(cfg, seed=None, **overrides):
    """Inputs of one selective-scan workload (``cfg``: index into SELECTIVE_CONFIGS or a dict).

      x ~ N(0, 1)                          [batch, seqlen, dim]            io dtype
      dt = softplus(z), z ~ N(-2, 0.5)     [batch, seqlen, dim]            float32
      A[d, n] = -exp(u), u ~ U(ln 1, ln 16), independent per (d, n)   [dim, dstate] float32
      B, C ~ N(0, 1) / sqrt(dstate)        [batch, seqlen, ngroups, dstate] io dtype
      D ~ N(0, 1)                          [dim]                           float32
      init ~ N(0, 0.1) or zeros            [batch, dim, dstate]            float32
    seed = 3000 + index unless given; SeedSequence(seed).spawn(7) children in that order.
    """
    idx = cfg if isinstance(cfg, int) else None
    if isinstance(cfg, int):
        cfg = SELECTIVE_CONFIGS[cfg]
    cfg = dict(cfg)
    cfg.update({k: v for k, v in overrides.items() if v is not None})
    if seed is None:
        seed = 3000 + (idx if idx is not None else 0)
    g = [np.random.Generator(np.random.PCG64(k)) for k in np.random.SeedSequence(seed).spawn(7)]
    Bt, L, dim, N, G, io = (cfg["batch"], cfg["seqlen"], cfg["dim"], cfg["dstate"],
                            cfg["ngroups"], cfg["io"])
    x = _normal_slabs(g[0], (Bt, L, dim), io)
    dt = np.empty((Bt, L, dim), dtype=np.float32)
    for b in range(Bt):
        for t0 in range(0, L, SLAB_TOKENS):
            t1 = min(L, t0 + SLAB_TOKENS)
            dt[b, t0:t1] = _softplus(-2.0 + 0.5 * g[1].standard_normal((t1 - t0, dim)))
    A = (-np.exp(g[2].uniform(0.0, math.log(16.0), size=(dim, N)))).astype(np.float32)
    B = _normal_slabs(g[3], (Bt, L, G, N), io, scale=1.0 / math.sqrt(N))
    C = _normal_slabs(g[4], (Bt, L, G, N), io, scale=1.0 / math.sqrt(N))
    D = g[5].standard_normal(dim).astype(np.float32)
    init = None
    if cfg["init"] == "normal0.1":
        init = (0.1 * g[6].standard_normal((Bt, dim, N))).astype(np.float32)
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, init=init, cfg=cfg)
