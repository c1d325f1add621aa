"""fp64 CPU oracle for the Mamba-2 SSD forward scan -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
and the library never calls it.

Python side: argument marshalling to the C implementation in ``ssd_oracle.c``
(every function widens its inputs to fp64; bf16-valued inputs widen exactly).

Method (per batch b, head h, group g = h // (H // G)):
    h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D_h x_t
-- the scalar-identity SSM recurrence (akillness.github.io "State Space Duality
and Mamba-2", "Mathematical Foundations" and "The Scalar-Identity Structural
Constraint"; aifetchly blog "Mamba-2 Architecture: State Space Duality
Explained", section 1 "The Core Duality", the sum form of y_t), with the step
size dt on the decay and on the input.

Shapes: x, y [B,T,H,P]; dt [B,T,H]; A, D [H]; B, C [B,T,G,N];
init/final state [B,H,P,N].
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

__all__ = ["ssd_recurrent", "ssd_quadratic", "ssd_chunked", "ssd_step", "default_threads",
           "dt_transform", "gated_rmsnorm", "ssd_block", "ssd_recurrent_grad"]


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups")]


_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_ssd_recurrent.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 9 + [
            ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, ctypes.c_int]
        lib.oracle_ssd_recurrent.restype = ctypes.c_int
        lib.oracle_ssd_quadratic.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 9
        lib.oracle_ssd_quadratic.restype = ctypes.c_int
        lib.oracle_ssd_chunked.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int64] + [dp] * 14
        lib.oracle_ssd_chunked.restype = ctypes.c_int
        lib.oracle_default_threads.argtypes = []
        lib.oracle_default_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    """Number of host cores in this process's affinity mask."""
    return int(_load().oracle_default_threads())


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(x, B):
    bsz, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return _Dims(bsz, T, H, P, N, G)


def _prep(x, dt, A, B, C, D, h0):
    x, dt, A, B, C = (_f64(v) for v in (x, dt, A, B, C))
    D, h0 = _f64(D), _f64(h0)
    bsz, T, H, P = x.shape
    if dt.shape != (bsz, T, H) or A.shape != (H,):
        raise ValueError("dt must be [B,T,H] and A [H]")
    if B.shape != C.shape or B.shape[:2] != (bsz, T):
        raise ValueError("B and C must be [B,T,G,N]")
    if D is not None and D.shape != (H,):
        raise ValueError("D must be [H]")
    if h0 is not None and h0.shape != (bsz, H, P, B.shape[3]):
        raise ValueError("init state must be [B,H,P,N]")
    return x, dt, A, B, C, D, h0


def ssd_recurrent(x, dt, A, B, C, D=None, h0=None, units=None, nthreads=0):
    """Token-by-token recurrence in fp64 (the oracle).

    ``units``: optional iterable of (b, h) pairs; only those heads are evaluated
    and the other entries of the returned arrays are NaN.
    Returns (y [B,T,H,P], final_state [B,H,P,N]) as float64 arrays.
    """
    x, dt, A, B, C, D, h0 = _prep(x, dt, A, B, C, D, h0)
    d = _dims(x, B)
    y = np.full(x.shape, np.nan)
    fin = np.full((d.batch, d.nheads, d.headdim, d.dstate), np.nan)
    if units is None:
        uarr, nu = None, 0
    else:
        ul = np.ascontiguousarray([b * d.nheads + h for (b, h) in units], dtype=np.int64)
        uarr, nu = ul.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(ul)
    rc = _load().oracle_ssd_recurrent(ctypes.byref(d), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                      _ptr(C), _ptr(D), _ptr(h0), _ptr(y), _ptr(fin),
                                      uarr, nu, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_ssd_recurrent failed ({rc})")
    return y, fin


def ssd_quadratic(x, dt, A, B, C, D=None, h0=None):
    """Dual form with the explicit T x T semiseparable matrix (small T only)."""
    x, dt, A, B, C, D, h0 = _prep(x, dt, A, B, C, D, h0)
    d = _dims(x, B)
    y = np.zeros(x.shape)
    fin = np.zeros((d.batch, d.nheads, d.headdim, d.dstate))
    rc = _load().oracle_ssd_quadratic(ctypes.byref(d), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                      _ptr(C), _ptr(D), _ptr(h0), _ptr(y), _ptr(fin))
    if rc != 0:
        raise ValueError(f"oracle_ssd_quadratic failed ({rc})")
    return y, fin


def ssd_chunked(x, dt, A, B, C, chunk_len, D=None, h0=None, intermediates=False):
    """Chunked algorithm in fp64.

    Returns (y, final_state) or, with ``intermediates=True``,
    (y, final_state, dict(l, w, alpha, S, s_in)) where
    l, w [B,H,nc,Q]; alpha [B,H,nc]; S [B,nc,H,P,N]; s_in [B,nc,H,P,N]
    (the state entering each chunk).
    """
    x, dt, A, B, C, D, h0 = _prep(x, dt, A, B, C, D, h0)
    d = _dims(x, B)
    Q = int(chunk_len)
    if Q <= 0 or d.seqlen % Q:
        raise ValueError("chunk_len must divide T")
    nc = d.seqlen // Q
    y = np.zeros(x.shape)
    fin = np.zeros((d.batch, d.nheads, d.headdim, d.dstate))
    if intermediates:
        l = np.zeros((d.batch, d.nheads, nc, Q))
        w = np.zeros_like(l)
        alpha = np.zeros((d.batch, d.nheads, nc))
        S = np.zeros((d.batch, nc, d.nheads, d.headdim, d.dstate))
        s_in = np.zeros((d.batch, nc + 1, d.nheads, d.headdim, d.dstate))
    else:
        l = w = alpha = S = s_in = None
    rc = _load().oracle_ssd_chunked(ctypes.byref(d), Q, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                    _ptr(C), _ptr(D), _ptr(h0), _ptr(y), _ptr(fin),
                                    _ptr(l), _ptr(w), _ptr(alpha), _ptr(S), _ptr(s_in))
    if rc != 0:
        raise ValueError(f"oracle_ssd_chunked failed ({rc})")
    if intermediates:
        return y, fin, dict(l=l, w=w, alpha=alpha, S=S, s_in=s_in[:, :nc])
    return y, fin


def ssd_step(state, x, dt, A, B, C, D=None):
    """One token of the recurrence for every (batch, head) in fp64 (numpy): the
    decode step.  Per batch b, head h, group g = h // (H // G):
        state' = exp(dt A_h) state + dt x B^T,   y = state' C + D_h x
    (akillness.github.io "State Space Duality and Mamba-2", "Mathematical
    Foundations": the recurrent form, one token).

    state [B,H,P,N]; x [B,H,P]; dt [B,H]; A, D [H]; B, C [B,G,N].
    Returns (y [B,H,P], new_state [B,H,P,N]) as float64 arrays; ``state`` is
    not modified.
    """
    h = _f64(state)
    x, dt, A, B, C, D = (_f64(v) for v in (x, dt, A, B, C, D))
    bsz, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if h.shape != (bsz, H, P, N) or dt.shape != (bsz, H) or A.shape != (H,) or C.shape != B.shape:
        raise ValueError("state [B,H,P,N], x [B,H,P], dt [B,H], A [H], B and C [B,G,N]")
    if H % G:
        raise ValueError("nheads must be a multiple of ngroups")
    group = np.arange(H) // (H // G)        # head -> group
    Bh = B[:, group, :]                     # [B,H,N]
    Ch = C[:, group, :]
    decay = np.exp(dt * A[None, :])         # [B,H]
    new = decay[:, :, None, None] * h + (dt[:, :, None] * x)[:, :, :, None] * Bh[:, :, None, :]
    y = np.einsum("bhpn,bhn->bhp", new, Ch)
    if D is not None:
        y = y + D[None, :, None] * x
    return y, new


# ---------------------------------------------------------------------------
# the scan's neighbours in the Mamba-2 block (aifetchly blog "Mamba-2
# Architecture: State Space Duality Explained", "Step 2: Full Mamba-2 Block with
# Gated Projections": softplus on dt before the SSD call; the SSD output gated by
# silu of the z branch; RMSNorm over d_inner = H * P; akillness.github.io "State
# Space Duality and Mamba-2", the block diagram: "Element-wise Gating", RMSNorm)
# ---------------------------------------------------------------------------
def dt_transform(dt, dt_bias=None, softplus=False):
    """The step size the scan uses: dt + dt_bias[h], then softplus if asked,
    softplus(v) = log(1 + exp(v)), in fp64.  dt [B,T,H]; dt_bias [H] or None."""
    v = _f64(dt).copy()
    if dt_bias is not None:
        v = v + _f64(dt_bias)[None, None, :]
    if softplus:
        # log(1 + e^v) = max(v, 0) + log(1 + e^-|v|): the same number, without overflow
        v = np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))
    return v


def gated_rmsnorm(y, z=None, weight=None, eps=1e-5):
    """The block's output side, in fp64: g = y * silu(z) (silu(z) = z / (1 +
    e^-z); no gate when z is None), then RMSNorm over each token's H * P values,
    out = g / sqrt(mean(g^2) + eps) * weight (weight [H*P]; no norm when weight is
    None).  y, z [B,T,H,P].  Returns (out [B,T,H,P], rstd [B,T] or None)."""
    g = _f64(y)
    if z is not None:
        zz = _f64(z)
        g = g * (zz / (1.0 + np.exp(-zz)))
    if weight is None:
        return g, None
    bsz, T, H, P = g.shape
    flat = g.reshape(bsz, T, H * P)
    rstd = 1.0 / np.sqrt(np.mean(flat * flat, axis=-1) + float(eps))
    out = flat * rstd[..., None] * _f64(weight)[None, None, :]
    return out.reshape(bsz, T, H, P), rstd


def ssd_block(x, dt, A, B, C, D=None, h0=None, dt_bias=None, dt_softplus=False, z=None,
              norm_weight=None, norm_eps=1e-5, units=None, nthreads=0):
    """The scan with its neighbours, in the block's order: dt_transform, the
    recurrence (ssd_recurrent), gated_rmsnorm.  Returns (out, final_state,
    rstd)."""
    dte = dt_transform(dt, dt_bias, dt_softplus)
    y, fin = ssd_recurrent(x, dte, A, B, C, D=D, h0=h0, units=units, nthreads=nthreads)
    out, rstd = gated_rmsnorm(y, z, norm_weight, norm_eps)
    return out, fin, rstd


def ssd_recurrent_grad(x, dt, A, B, C, dy, D=None, h0=None, dfinal=None):
    """Reverse mode of the recurrence, in fp64: the gradients of
    L = sum(y * dy) + sum(final * dfinal) with respect to every input.

    Forward (per b, h, g = h // (H // G)), as ssd_recurrent:
        a_t = exp(dt_t A_h),  h_t = a_t h_{t-1} + dt_t x_t B_t^T,  y_t = h_t C_t + D_h x_t
    Reverse, token by token from the last (G_t = dL/dh_t, with the future's
    share G' = dL/dh_t through h_{t+1}, starting from dfinal):
        G_t    = dy_t C_t^T + G'
        dx_t   = dt_t G_t B_t + D_h dy_t
        dB_t  += dt_t G_t^T x_t           (summed over the group's heads)
        dC_t  += h_t^T dy_t               (summed over the group's heads)
        ddt_t  = x_t . (G_t B_t) + A_h a_t (G_t : h_{t-1})
        dA_h  += dt_t a_t (G_t : h_{t-1})
        G'     = a_t G_t                  (dL/dh_{t-1}; dh0 at the end)
        dD_h  += dy_t . x_t
    Every forward state is kept (small problems only).  Returns a dict with dx,
    ddt, dA, dB, dC, dD, dh0 (float64)."""
    x, dt, A, B, C, D, h0 = _prep(x, dt, A, B, C, D, h0)
    dy = _f64(dy)
    bsz, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dy.shape != x.shape:
        raise ValueError("dy must be shaped like x")
    rep = H // G
    Bh = np.repeat(B, rep, axis=2)  # [B,T,H,N]: each head's B and C
    Ch = np.repeat(C, rep, axis=2)
    h = np.zeros((bsz, H, P, N)) if h0 is None else h0.copy()
    hs = [h]
    for t in range(T):
        a = np.exp(dt[:, t, :] * A[None, :])
        h = a[:, :, None, None] * h + (dt[:, t, :, None, None] * x[:, t, :, :, None]) * Bh[:, t, :, None, :]
        hs.append(h)  # hs[t + 1] = h_t
    Gn = np.zeros((bsz, H, P, N)) if dfinal is None else _f64(dfinal).copy()
    dx = np.zeros_like(x)
    ddt = np.zeros_like(dt)
    dA = np.zeros(H)
    dBh = np.zeros_like(Bh)
    dCh = np.zeros_like(Ch)
    Dv = np.zeros(H) if D is None else D
    for t in range(T - 1, -1, -1):
        Gt = dy[:, t, :, :, None] * Ch[:, t, :, None, :] + Gn
        a = np.exp(dt[:, t, :] * A[None, :])
        hprev = hs[t]
        GB = np.einsum("bhpn,bhn->bhp", Gt, Bh[:, t])
        dx[:, t] = dt[:, t, :, None] * GB + Dv[None, :, None] * dy[:, t]
        dBh[:, t] = dt[:, t, :, None] * np.einsum("bhpn,bhp->bhn", Gt, x[:, t])
        dCh[:, t] = np.einsum("bhpn,bhp->bhn", hs[t + 1], dy[:, t])
        gh = np.einsum("bhpn,bhpn->bh", Gt, hprev)
        ddt[:, t] = np.einsum("bhp,bhp->bh", x[:, t], GB) + A[None, :] * a * gh
        dA += np.sum(dt[:, t] * a * gh, axis=0)
        Gn = a[:, :, None, None] * Gt
    dB = dBh.reshape(bsz, T, G, rep, N).sum(axis=3)
    dC = dCh.reshape(bsz, T, G, rep, N).sum(axis=3)
    dD = np.einsum("bthp,bthp->h", dy, x)
    return dict(dx=dx, ddt=ddt, dA=dA, dB=dB, dC=dC, dD=dD, dh0=Gn)
