"""ctypes binding of ``libssd.so`` (the C ABI in ``include/ssd.h``).

Argument marshalling only: shapes, dtypes and devices of torch tensors are
checked, their device pointers and the current CUDA stream are passed to the C
call, and a non-zero status is raised as :class:`SSDError`.  Every step of the
computation runs in the library's CUDA kernels; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_NULL_ARG", 2: "SSD_ERR_INVALID_DIM", 3: "SSD_ERR_UNSUPPORTED",
          4: "SSD_ERR_MISALIGNED", 5: "SSD_ERR_CUDA", 6: "SSD_ERR_DEVICE_TIMEOUT",
          7: "SSD_ERR_WORKSPACE"}

EXPORTS = ("ssd_forward", "ssd_forward_ws", "ssd_forward_stage", "ssd_workspace_bytes",
           "ssd_workspace_layout", "ssd_device_status", "ssd_status_string", "ssd_version",
           "ssd_forward_static", "ssd_step", "ssd_forward_block", "ssd_block_workspace_bytes",
           "ssd_forward_varlen", "ssd_varlen_workspace_bytes", "ssd_backward", "ssd_workspace_trim")
STAGES = ("ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing", "ssd_chunk_scan")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("l_offset", ctypes.c_size_t),
                ("w_offset", ctypes.c_size_t), ("dtq_offset", ctypes.c_size_t),
                ("beta_offset", ctypes.c_size_t),
                ("alpha_offset", ctypes.c_size_t),
                ("states_offset", ctypes.c_size_t), ("s_in_offset", ctypes.c_size_t),
                ("s_in_dtype", ctypes.c_int32), ("tensor_core", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("states_dtype", ctypes.c_int32),
                ("fused_state", ctypes.c_int32), ("single_pass", ctypes.c_int32),
                ("scan_engine", ctypes.c_int32), ("chunk_len", ctypes.c_int32)]


# ssd_scan_engine_t: which kernel computes y
SCAN_ENGINES = {0: "simt", 1: "tile", 2: "block_factored", 3: "chunk_wide", 4: "single_pass"}


class BlockOpts(ctypes.Structure):
    """ssd_block_opts_t: the scan's neighbours in the Mamba-2 block."""
    _fields_ = [("dt_bias", ctypes.c_void_p), ("dt_softplus", ctypes.c_int32),
                ("norm_apply", ctypes.c_int32), ("z", ctypes.c_void_p),
                ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float),
                ("reserved0", ctypes.c_int32), ("rstd_out", ctypes.c_void_p)]


class SSDError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libssd.so (raises if it has not been built; there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m structured_state_space_mamba_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp = ctypes.c_void_p, ctypes.c_void_p
    dims_p = ctypes.POINTER(Dims)
    lib.ssd_forward.argtypes = [dims_p, vp, fp, fp, vp, vp, fp, ctypes.c_int, fp, vp, fp, vp]
    lib.ssd_forward.restype = ctypes.c_int
    lib.ssd_forward_ws.argtypes = [dims_p, vp, fp, fp, vp, vp, fp, ctypes.c_int, fp, vp, fp,
                                   vp, ctypes.c_size_t, vp]
    lib.ssd_forward_ws.restype = ctypes.c_int
    lib.ssd_forward_static.argtypes = lib.ssd_forward.argtypes
    lib.ssd_forward_static.restype = ctypes.c_int
    lib.ssd_step.argtypes = [dims_p, vp, fp, fp, vp, vp, fp, fp, vp, vp]
    lib.ssd_step.restype = ctypes.c_int
    lib.ssd_forward_stage.argtypes = [ctypes.c_int] + lib.ssd_forward_ws.argtypes
    lib.ssd_forward_stage.restype = ctypes.c_int
    lib.ssd_forward_block.argtypes = [dims_p, vp, fp, fp, vp, vp, fp, ctypes.c_int, fp, vp, fp,
                                      ctypes.POINTER(BlockOpts), vp, ctypes.c_size_t, vp]
    lib.ssd_forward_block.restype = ctypes.c_int
    lib.ssd_block_workspace_bytes.argtypes = [dims_p, ctypes.c_int, ctypes.POINTER(BlockOpts)]
    lib.ssd_block_workspace_bytes.restype = ctypes.c_size_t
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.ssd_forward_varlen.argtypes = [dims_p, i64p, ctypes.c_int64, vp, fp, fp, vp, vp, fp, ctypes.c_int, fp,
                                       vp, fp, vp, ctypes.c_size_t, vp]
    lib.ssd_forward_varlen.restype = ctypes.c_int
    lib.ssd_varlen_workspace_bytes.argtypes = [dims_p, i64p, ctypes.c_int64, ctypes.c_int]
    lib.ssd_varlen_workspace_bytes.restype = ctypes.c_size_t
    lib.ssd_backward.argtypes = [dims_p, vp, fp, fp, vp, vp, fp, ctypes.c_int, fp, vp, fp, vp, fp, fp, vp, vp, fp,
                                 fp, vp]
    lib.ssd_backward.restype = ctypes.c_int
    lib.ssd_workspace_bytes.argtypes = [dims_p, ctypes.c_int]
    lib.ssd_workspace_bytes.restype = ctypes.c_size_t
    lib.ssd_workspace_layout.argtypes = [dims_p, ctypes.c_int, ctypes.POINTER(WorkspaceLayout)]
    lib.ssd_workspace_layout.restype = ctypes.c_int
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_device_status.argtypes = [ctypes.c_void_p]
    lib.ssd_device_status.restype = ctypes.c_int
    lib.ssd_version.argtypes = []
    lib.ssd_version.restype = ctypes.c_char_p
    lib.ssd_workspace_trim.argtypes = []
    lib.ssd_workspace_trim.restype = ctypes.c_int
    _lib = lib
    return lib


def make_dims(batch, seqlen, nheads, headdim, dstate, ngroups, dtype) -> Dims:
    code = {"f32": SSD_F32, "bf16": SSD_BF16, torch.float32: SSD_F32,
            torch.bfloat16: SSD_BF16}[dtype]
    return Dims(batch, seqlen, nheads, headdim, dstate, ngroups, code, 0)


def _check(status: int):
    if status != 0:
        raise SSDError(status, load().ssd_status_string(status).decode())


def workspace_bytes(dims: Dims, chunk_len: int) -> int:
    return int(load().ssd_workspace_bytes(ctypes.byref(dims), int(chunk_len)))


def workspace_layout(dims: Dims, chunk_len: int) -> WorkspaceLayout:
    out = WorkspaceLayout()
    _check(load().ssd_workspace_layout(ctypes.byref(dims), int(chunk_len), ctypes.byref(out)))
    return out


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _validate(x, dt, A, B, C, D, init_state):
    if not x.is_cuda:
        raise ValueError("ssd.forward runs on CUDA tensors only")
    dev = x.device
    for name, t in (("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D),
                    ("init_state", init_state)):
        if t is None:
            continue
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, x on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if x.dtype not in (torch.float32, torch.bfloat16) or B.dtype != x.dtype or C.dtype != x.dtype:
        raise ValueError("x, B and C must share a dtype: float32 or bfloat16")
    for name, t in (("dt", dt), ("A", A), ("D", D), ("init_state", init_state)):
        if t is not None and t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32")
    bsz, T, H, P = x.shape
    if B.dim() != 4 or B.shape[:2] != (bsz, T) or C.shape != B.shape:
        raise ValueError("B and C must be [batch, seqlen, ngroups, dstate]")
    G, N = B.shape[2], B.shape[3]
    if dt.shape != (bsz, T, H) or A.shape != (H,):
        raise ValueError("dt must be [batch, seqlen, nheads] and A [nheads]")
    if D is not None and D.shape != (H,):
        raise ValueError("D must be [nheads]")
    if init_state is not None and init_state.shape != (bsz, H, P, N):
        raise ValueError("init_state must be [batch, nheads, headdim, dstate]")
    return make_dims(bsz, T, H, P, N, G, x.dtype)


def forward(x, dt, A, B, C, D=None, chunk_len=256, init_state=None, return_final_state=False,
            out=None, final_out=None, workspace=None, stream=None, stage=None):
    """y (and optionally the final state) of the SSD forward scan.

    x [B,T,H,P], B/C [B,T,G,N] (float32 or bfloat16); dt [B,T,H], A [H], D [H],
    init_state [B,H,P,N] float32.  Returns ``y`` or ``(y, final_state)``.
    ``workspace``: optional uint8 CUDA tensor of at least ``workspace_bytes``
    bytes (otherwise the library allocates it stream-ordered).
    """
    dims = _validate(x, dt, A, B, C, D, init_state)
    y = out if out is not None else torch.empty_like(x)
    fin = final_out
    if fin is None and return_final_state:
        fin = torch.empty((dims.batch, dims.nheads, dims.headdim, dims.dstate),
                          dtype=torch.float32, device=x.device)
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    lib = load()
    args = [ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
            int(chunk_len), _ptr(init_state), _ptr(y), _ptr(fin)]
    with torch.cuda.device(x.device):
        if stage is not None:
            if workspace is None:
                raise ValueError("a single stage needs workspace=")
            st = lib.ssd_forward_stage(int(stage), *args, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       ctypes.c_void_p(stream))
        elif workspace is None:
            st = lib.ssd_forward(*args, ctypes.c_void_p(stream))
        else:
            st = lib.ssd_forward_ws(*args, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    ctypes.c_void_p(stream))
    _check(st)
    if return_final_state or final_out is not None:
        return y, fin
    return y


def forward_block(x, dt, A, B, C, D=None, chunk_len=256, init_state=None, dt_bias=None,
                  dt_softplus=False, z=None, norm_weight=None, norm_eps=1e-5, norm_apply=True,
                  return_rstd=False, return_final_state=False, out=None, final_out=None,
                  workspace=None, stream=None):
    """The scan with its block neighbours through ``ssd_forward_block``:
    softplus(dt + dt_bias) as the step size, then y * silu(z) and RMSNorm over
    each token's H * P values with ``norm_weight`` [H*P] float32.  With
    ``norm_apply=False`` the output is the gated, weighted y and the per-token
    factor rstd [B, T] is returned for the caller to apply.
    Returns ``out`` plus, as asked, the final state and rstd (in that order)."""
    dims = _validate(x, dt, A, B, C, D, init_state)
    dev = x.device
    for name, t in (("dt_bias", dt_bias), ("norm_weight", norm_weight)):
        if t is not None and (t.device != dev or t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 tensor on {dev}")
    if z is not None and (z.device != dev or z.dtype != x.dtype or z.shape != x.shape or not z.is_contiguous()):
        raise ValueError("z must be a contiguous tensor like x")
    y = out if out is not None else torch.empty_like(x)
    fin = final_out
    if fin is None and return_final_state:
        fin = torch.empty((dims.batch, dims.nheads, dims.headdim, dims.dstate),
                          dtype=torch.float32, device=dev)
    rstd = None
    if norm_weight is not None and (return_rstd or not norm_apply):
        rstd = torch.empty((dims.batch, dims.seqlen), dtype=torch.float32, device=dev)
    opts = BlockOpts(dt_bias=None if dt_bias is None else dt_bias.data_ptr(),
                     dt_softplus=1 if dt_softplus else 0, norm_apply=1 if norm_apply else 0,
                     z=None if z is None else z.data_ptr(),
                     norm_weight=None if norm_weight is None else norm_weight.data_ptr(),
                     norm_eps=float(norm_eps), reserved0=0,
                     rstd_out=None if rstd is None else rstd.data_ptr())
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = load().ssd_forward_block(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                      _ptr(D), int(chunk_len), _ptr(init_state), _ptr(y), _ptr(fin),
                                      ctypes.byref(opts), _ptr(workspace), wsz, ctypes.c_void_p(stream))
    _check(st)
    res = [y]
    if return_final_state or final_out is not None:
        res.append(fin)
    if rstd is not None:
        res.append(rstd)
    return res[0] if len(res) == 1 else tuple(res)


def _cu_array(cu_seqlens):
    import numpy as np
    cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens,
                                         dtype=np.int64))
    if cu.ndim != 1 or cu.size < 2:
        raise ValueError("cu_seqlens must be a 1-D array of nseq + 1 offsets")
    return cu


def varlen_workspace_bytes(dims: Dims, cu_seqlens, chunk_len: int) -> int:
    cu = _cu_array(cu_seqlens)
    return int(load().ssd_varlen_workspace_bytes(ctypes.byref(dims), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                                 cu.size - 1, int(chunk_len)))


def forward_varlen(x, dt, A, B, C, cu_seqlens, D=None, chunk_len=256, init_states=None,
                   return_final_states=False, out=None, final_out=None, workspace=None, stream=None):
    """Several sequences packed along the token axis through ``ssd_forward_varlen``.

    x [1, T, H, P], dt [1, T, H], B/C [1, T, G, N]; ``cu_seqlens`` (host: a list,
    a numpy array or a CPU tensor) holds nseq + 1 offsets; ``init_states`` and
    the final states are [nseq, H, P, N] float32.  Returns y (and the final
    states)."""
    cu = _cu_array(cu_seqlens)
    nseq = cu.size - 1
    dims = _validate(x, dt, A, B, C, D, None)
    dev = x.device
    st_shape = (nseq, dims.nheads, dims.headdim, dims.dstate)
    if init_states is not None and (init_states.device != dev or init_states.dtype != torch.float32
                                    or tuple(init_states.shape) != st_shape or not init_states.is_contiguous()):
        raise ValueError(f"init_states must be a contiguous float32 tensor {st_shape} on {dev}")
    y = out if out is not None else torch.empty_like(x)
    fin = final_out
    if fin is None and return_final_states:
        fin = torch.empty(st_shape, dtype=torch.float32, device=dev)
    cu_p = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    if workspace is None:
        need = int(load().ssd_varlen_workspace_bytes(ctypes.byref(dims), cu_p, nseq, int(chunk_len)))
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        wsz = workspace.numel() * workspace.element_size()
        st = load().ssd_forward_varlen(ctypes.byref(dims), cu_p, nseq, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                       _ptr(C), _ptr(D), int(chunk_len), _ptr(init_states), _ptr(y), _ptr(fin),
                                       _ptr(workspace), wsz, ctypes.c_void_p(stream))
    _check(st)
    return (y, fin) if (return_final_states or final_out is not None) else y


def backward(x, dt, A, B, C, dy, D=None, chunk_len=256, init_state=None, dfinal_state=None, stream=None):
    """Gradients through ``ssd_backward``: returns a dict with dx, ddt, dA, dB,
    dC, dD (None without D) and dinit_state (None without an initial state)."""
    dims = _validate(x, dt, A, B, C, D, init_state)
    dev = x.device
    if dy.shape != x.shape or dy.dtype != x.dtype or dy.device != dev or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous tensor like x")
    if dfinal_state is not None and (dfinal_state.dtype != torch.float32 or not dfinal_state.is_contiguous()
                                     or tuple(dfinal_state.shape) != (dims.batch, dims.nheads, dims.headdim,
                                                                      dims.dstate)):
        raise ValueError("dfinal_state must be a contiguous float32 [batch, nheads, headdim, dstate] tensor")
    out = dict(dx=torch.empty_like(x), ddt=torch.empty_like(dt), dA=torch.empty_like(A),
               dB=torch.empty_like(B), dC=torch.empty_like(C),
               dD=None if D is None else torch.empty_like(D),
               dinit_state=None if init_state is None else torch.empty_like(init_state))
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = load().ssd_backward(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                 int(chunk_len), _ptr(init_state), _ptr(dy), _ptr(dfinal_state), _ptr(out["dx"]),
                                 _ptr(out["ddt"]), _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
                                 _ptr(out["dD"]), _ptr(out["dinit_state"]), ctypes.c_void_p(stream))
    _check(st)
    return out


def block_workspace_bytes(dims: Dims, chunk_len: int, dt_transform: bool) -> int:
    opts = BlockOpts(dt_softplus=1 if dt_transform else 0)
    return int(load().ssd_block_workspace_bytes(ctypes.byref(dims), int(chunk_len), ctypes.byref(opts)))


def forward_ws(*args, **kwargs):
    """``forward`` with a required ``workspace`` keyword."""
    if kwargs.get("workspace") is None:
        raise ValueError("forward_ws needs workspace=")
    return forward(*args, **kwargs)


def forward_static(x, dt, A, B, C, D=None, chunk_len=256, init_state=None,
                   return_final_state=False, out=None, final_out=None, stream=None):
    """``forward`` through ``ssd_forward_static``: the intermediates live in the
    library's fixed per-device scratch array, and nothing is allocated.  A
    workload whose workspace exceeds ``STATIC_SCRATCH_BYTES`` raises (status
    SSD_ERR_WORKSPACE); calls that overlap in time on one device race on the
    shared scratch."""
    dims = _validate(x, dt, A, B, C, D, init_state)
    y = out if out is not None else torch.empty_like(x)
    fin = final_out
    if fin is None and return_final_state:
        fin = torch.empty((dims.batch, dims.nheads, dims.headdim, dims.dstate),
                          dtype=torch.float32, device=x.device)
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    with torch.cuda.device(x.device):
        st = load().ssd_forward_static(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                       _ptr(C), _ptr(D), int(chunk_len), _ptr(init_state),
                                       _ptr(y), _ptr(fin), ctypes.c_void_p(stream))
    _check(st)
    if return_final_state or final_out is not None:
        return y, fin
    return y


STATIC_SCRATCH_BYTES = 64 << 20  # SSD_STATIC_SCRATCH_BYTES in include/ssd.h


def step(state, x, dt, A, B, C, D=None, out=None, stream=None):
    """One decode step through ``ssd_step``: ``state`` [B,H,P,N] float32 is
    updated in place to exp(dt A) state + dt x B^T and y = state C + D x is
    returned.  x [B,H,P], B/C [B,G,N] (float32 or bfloat16, one dtype);
    dt [B,H], A [H], D [H] float32."""
    if not x.is_cuda:
        raise ValueError("ssd.step runs on CUDA tensors only")
    dev = x.device
    for name, t in (("state", state), ("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D)):
        if t is None:
            continue
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, x on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if x.dtype not in (torch.float32, torch.bfloat16) or B.dtype != x.dtype or C.dtype != x.dtype:
        raise ValueError("x, B and C must share a dtype: float32 or bfloat16")
    for name, t in (("state", state), ("dt", dt), ("A", A), ("D", D)):
        if t is not None and t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32")
    bsz, H, P = x.shape
    if B.dim() != 3 or B.shape[0] != bsz or C.shape != B.shape:
        raise ValueError("B and C must be [batch, ngroups, dstate]")
    G, N = B.shape[1], B.shape[2]
    if dt.shape != (bsz, H) or A.shape != (H,) or state.shape != (bsz, H, P, N):
        raise ValueError("dt must be [batch, nheads], A [nheads], state [batch, nheads, headdim, dstate]")
    if D is not None and D.shape != (H,):
        raise ValueError("D must be [nheads]")
    dims = make_dims(bsz, 1, H, P, N, G, x.dtype)
    y = out if out is not None else torch.empty_like(x)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = load().ssd_step(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                             _ptr(state), _ptr(y), ctypes.c_void_p(stream))
    _check(st)
    return y


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error
    status: 0 (SSD_OK) or 6 (SSD_ERR_DEVICE_TIMEOUT)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(load().ssd_device_status(
            ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))


def workspace_trim(device=None) -> int:
    """Synchronise the device and return the library pool's unused workspace
    memory to the system; 0 (SSD_OK) or an ssd_status_t error code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(load().ssd_workspace_trim())


def version() -> str:
    return load().ssd_version().decode()
