"""Seeded synthetic inputs for the SSD forward scan.

This module holds no arithmetic of the method: it only draws random numbers
and rounds them to the storage dtype.  It is the one module shared by the CUDA
path's tests/benchmark and the oracle's tests.

Distributions (the Mamba-2 layer workloads):
    x ~ N(0, 1)                         [B, T, H, P]
    dt = exp(U(ln 1e-3, ln 1e-1))       [B, T, H]   (log-uniform, already positive)
    A_h = -exp(U(0, ln 16))             [H]
    B, C ~ N(0, 1) / sqrt(N)            [B, T, G, N]
    D ~ N(0, 1)                         [H]
    h0 ~ N(0, 0.1^2)                    [B, H, P, N] (only when requested)
drawn in that order from ``numpy.random.default_rng(seed)`` in fp64, then
x/B/C rounded to the storage dtype (round-to-nearest-even for bf16) and
dt/A/D/h0 rounded to fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round an fp32/fp64 array to the nearest bf16 value (ties to even).

    Returns float32 values that are exactly representable in bf16."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    # NaN/Inf pass through unchanged (never produced by these distributions)
    bad = ~np.isfinite(f)
    if bad.any():
        out = out.copy()
        out[bad] = f[bad]
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-representable float32 values (the bf16 storage)."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return (f.view(np.uint32) >> 16).astype(np.uint16)


@dataclass
class SSDInputs:
    x: np.ndarray
    dt: np.ndarray
    A: np.ndarray
    B: np.ndarray
    C: np.ndarray
    D: np.ndarray
    h0: np.ndarray | None
    dtype: str  # "f32" or "bf16": storage dtype of x, B, C (and y)
    chunk_len: int
    meta: dict = field(default_factory=dict)

    @property
    def dims(self):
        bsz, T, H, P = self.x.shape
        return dict(batch=bsz, seqlen=T, nheads=H, headdim=P,
                    dstate=self.B.shape[3], ngroups=self.B.shape[2])


def make_inputs(batch, seqlen, nheads, headdim, dstate, ngroups, chunk_len, dtype="bf16",
                seed=0, init_state=False, h0_std=0.1) -> SSDInputs:
    """Draw one seeded problem.  All arrays are numpy float32 (x/B/C hold
    bf16-representable values when dtype == 'bf16')."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, seqlen, nheads, headdim))
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=(batch, seqlen, nheads)))
    A = -np.exp(rng.uniform(0.0, np.log(16.0), size=(nheads,)))
    B = rng.standard_normal((batch, seqlen, ngroups, dstate)) / np.sqrt(dstate)
    C = rng.standard_normal((batch, seqlen, ngroups, dstate)) / np.sqrt(dstate)
    D = rng.standard_normal((nheads,))
    h0 = rng.normal(0.0, h0_std, size=(batch, nheads, headdim, dstate)) if init_state else None
    if dtype == "bf16":
        cast = round_to_bf16
    elif dtype == "f32":
        def cast(a):
            return np.ascontiguousarray(a, dtype=np.float32)
    else:
        raise ValueError(dtype)
    f32 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return SSDInputs(x=cast(x), dt=f32(dt), A=f32(A), B=cast(B), C=cast(C), D=f32(D),
                     h0=f32(h0), dtype=dtype, chunk_len=int(chunk_len),
                     meta=dict(seed=seed))


# The workloads: a tiny fp32 case, Mamba-2-130M- and 2.7B-shaped layers, a long
# grouped layer with an initial state, and a state-size x chunk-length sweep.
WORKLOADS = {
    "tiny_f32": dict(batch=1, seqlen=256, nheads=2, headdim=16, dstate=16, ngroups=1,
                     chunk_len=64, dtype="f32", init_state=False, seed=1000),
    "mamba2_130m": dict(batch=8, seqlen=2048, nheads=24, headdim=64, dstate=128, ngroups=1,
                        chunk_len=256, dtype="bf16", init_state=False, seed=1001),
    "mamba2_2p7b": dict(batch=4, seqlen=4096, nheads=80, headdim=64, dstate=128, ngroups=1,
                        chunk_len=256, dtype="bf16", init_state=False, seed=1002,
                        final_state=True),
    "long_g8": dict(batch=1, seqlen=65536, nheads=32, headdim=64, dstate=128, ngroups=8,
                    chunk_len=256, dtype="bf16", init_state=True, seed=1003, final_state=True),
}
for _i, (_n, _q) in enumerate([(n, q) for n in (16, 64, 128, 256) for q in (64, 128, 256)]):
    WORKLOADS[f"sweep_N{_n}_Q{_q}"] = dict(batch=2, seqlen=8192, nheads=32, headdim=64,
                                           dstate=_n, ngroups=1, chunk_len=_q, dtype="bf16",
                                           init_state=False, seed=1400 + _i)


def make_workload(name: str, **overrides) -> SSDInputs:
    """Inputs for a named workload; ``overrides`` may shrink sizes (e.g. seqlen)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    cfg.pop("final_state", None)
    inp = make_inputs(**cfg)
    inp.meta["workload"] = name
    return inp
