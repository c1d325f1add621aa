"""The C ABI boundary on the CPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything.

Every call here that passes pointers returns an error from the host-side
checks (nothing is launched), so the fake addresses are never dereferenced.
"""
import ctypes
import os
import re

import numpy as np

import pytest

from structured_state_space_mamba_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    from structured_state_space_mamba_b200 import build
    build.build()
    return binding.load()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", src)


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("ssd_forward", "ssd_forward_ws", "ssd_workspace_bytes", "ssd_workspace_layout",
              "ssd_status_string", "ssd_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(binding.EXPORTS) <= set(declared_functions())


def test_struct_sizes_match_header(lib):
    assert ctypes.sizeof(binding.Dims) == 6 * 8 + 2 * 4
    assert ctypes.sizeof(binding.WorkspaceLayout) == 8 * 8 + 8 * 4  # 8 int32 fields


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        s = lib.ssd_status_string(code).decode()
        assert s.startswith(name)
    assert lib.ssd_status_string(99).decode().startswith("SSD_ERR_UNKNOWN")
    assert "sm_100a" in lib.ssd_version().decode()


def dims(**kw):
    base = dict(batch=2, seqlen=512, nheads=8, headdim=64, dstate=128, ngroups=2, dtype="bf16")
    base.update(kw)
    return binding.make_dims(**base)


def test_workspace_layout(lib):
    d = dims()
    lay = binding.workspace_layout(d, 128)
    # the four-kernel tensor-core path runs 256-token chunks; the arrays
    # describe the chunks the kernels run
    q = lay.chunk_len
    assert q == 256
    nc = 512 // q
    assert lay.l_offset == 0
    assert lay.w_offset >= 2 * 8 * nc * q * 4
    assert lay.states_offset % 256 == 0 and lay.s_in_offset % 256 == 0
    state_elems = 2 * nc * 8 * 64 * 128
    ssz = 2 if lay.states_dtype == binding.SSD_BF16 else 4
    assert lay.s_in_offset >= lay.states_offset + state_elems * ssz
    sz = 2 if lay.s_in_dtype == binding.SSD_BF16 else 4
    assert lay.total_bytes >= lay.s_in_offset + state_elems * sz
    # N = 128: chunk-wide scan + block-factored pass over steep tiles
    assert lay.launches == 5 and lay.fused_state == 0
    assert binding.workspace_bytes(d, 128) == lay.total_bytes
    # fp32 storage never uses the tensor-core kernels
    lay32 = binding.workspace_layout(dims(dtype="f32"), 128)
    assert lay32.tensor_core == 0 and lay32.s_in_dtype == binding.SSD_F32


def test_fused_state_layout_for_many_head_pairs(lib):
    """0.6 x 148 <= (batch x head pairs) <= 148 SMs at a dstate the single-pass
    kernel does not take: chunk_state and state_passing run as one kernel, so no
    states region is reserved and one launch fewer is made."""
    d = binding.make_dims(batch=8, seqlen=2048, nheads=24, headdim=64, dstate=32, ngroups=1,
                          dtype="bf16")
    lay = binding.workspace_layout(d, 256)
    assert lay.fused_state == 1 and lay.single_pass == 0 and lay.tensor_core == 1
    assert lay.states_offset == lay.s_in_offset
    # N = 32 keeps the one-launch scan
    n32 = binding.workspace_layout(binding.make_dims(batch=2, seqlen=1024, nheads=8, headdim=64,
                                                     dstate=32, ngroups=1, dtype="bf16"), 256)
    assert n32.launches == 4 and n32.single_pass == 0


def test_single_pass_layout_selection(lib):
    """bf16, P = 64, N = 64 or 128, chunk_len 128 / 256 and enough (batch, head
    pair) chains (>= 40% of the 148 SMs) run the single-pass kernel: three
    launches, no chunk-state region; few chains keep the four-kernel sequence."""
    for b, h, q, n in ((4, 80, 256, 128), (8, 24, 256, 128), (8, 32, 128, 128), (4, 32, 256, 128),
                       (4, 80, 256, 64), (8, 24, 128, 64)):
        lay = binding.workspace_layout(binding.make_dims(batch=b, seqlen=4096, nheads=h, headdim=64,
                                                         dstate=n, ngroups=1, dtype="bf16"), q)
        assert lay.single_pass == 1 and lay.launches == 3, (b, h, q, n)
        assert lay.fused_state == 0 and lay.states_offset == lay.s_in_offset
        assert binding.SCAN_ENGINES[lay.scan_engine] == "single_pass"
    # 16 chains of 256 chunks: the presolved single pass (the range states, then
    # the single pass from them: five launches, no chunk-state region)
    few = binding.workspace_layout(binding.make_dims(batch=1, seqlen=65536, nheads=32, headdim=64,
                                                     dstate=128, ngroups=8, dtype="bf16"), 256)
    assert few.single_pass == 1 and few.launches == 5
    assert binding.SCAN_ENGINES[few.scan_engine] == "single_pass"
    assert few.s_in_offset == few.states_offset
    # 32 chains of 32 chunks at dstate 128: short ranges keep the four-kernel sequence
    short = binding.workspace_layout(binding.make_dims(batch=2, seqlen=8192, nheads=32, headdim=64,
                                                       dstate=128, ngroups=1, dtype="bf16"), 256)
    assert short.single_pass == 0 and short.launches == 5
    assert binding.SCAN_ENGINES[short.scan_engine] == "chunk_wide"
    assert short.s_in_offset > short.states_offset
    # the same at dstate 64: presolved (the alternative is the block-factored scan)
    n64 = binding.workspace_layout(binding.make_dims(batch=2, seqlen=8192, nheads=32, headdim=64,
                                                     dstate=64, ngroups=1, dtype="bf16"), 256)
    assert n64.single_pass == 1 and n64.launches == 5
    # an odd number of heads per group, dstate 32 or 256: not taken
    for kw, q in ((dict(nheads=81, ngroups=1), 256), (dict(nheads=80, ngroups=1, dstate=32), 256),
                  (dict(nheads=80, ngroups=1, dstate=256), 256)):
        args = dict(batch=4, seqlen=4096, headdim=64, dstate=128, dtype="bf16")
        args.update(kw)
        assert binding.workspace_layout(binding.make_dims(**args), q).single_pass == 0, (kw, q)
    # chunk_len 64 runs with 128-token chunks (two per tensor-core tile)
    lay = binding.workspace_layout(binding.make_dims(batch=4, seqlen=4096, nheads=80, headdim=64,
                                                     dstate=128, ngroups=1, dtype="bf16"), 64)
    assert lay.single_pass == 1 and lay.chunk_len == 128


def test_chunk_len_64_on_the_tensor_cores(lib):
    """bf16 chunk_len 32 / 64 / 128 on the four-kernel tensor-core path runs
    256-token chunks (dstate 256: 128-token chunks) when that does not lengthen
    the ragged tail; where the single pass applies, chunk_len 64 runs 128-token
    chunks; fp32 keeps the caller's chunk_len."""
    for q in (32, 64, 128):
        for n in (16, 32, 64, 128, 256):
            lay = binding.workspace_layout(binding.make_dims(2, 1024, 8, 64, n, 1, "bf16"), q)
            assert lay.tensor_core == 1 and lay.chunk_len == (128 if n == 256 else 256), (q, n)
            assert binding.SCAN_ENGINES[lay.scan_engine] != "simt", (q, n)
    # T mod 256 = 192 > T mod 64 = 0: the tail would grow, chunk_len 64 stays
    odd = binding.workspace_layout(binding.make_dims(2, 960, 8, 64, 128, 1, "bf16"), 64)
    assert odd.chunk_len == 64
    # T mod 256 = 64 = T mod 128: 256-token chunks, the same 64-token tail
    tail = binding.workspace_layout(binding.make_dims(2, 1088, 8, 64, 128, 1, "bf16"), 128)
    assert tail.chunk_len == 256
    # enough chains for the single pass: it keeps 128-token chunks
    single = binding.workspace_layout(binding.make_dims(4, 4096, 80, 64, 128, 1, "bf16"), 64)
    assert single.single_pass == 1 and single.chunk_len == 128
    f32 = binding.workspace_layout(binding.make_dims(2, 1024, 8, 64, 128, 1, "f32"), 64)
    assert f32.chunk_len == 64 and f32.tensor_core == 0


@pytest.mark.parametrize("kw,chunk,code", [
    (dict(seqlen=500), 128, 0),          # T % chunk_len != 0: the tail kernel takes the rest
    (dict(seqlen=500, dtype="f32", dstate=24), 128, 3),  # ... with a dstate it cannot split
    (dict(nheads=6, ngroups=4), 128, 2),  # H % G != 0
    (dict(batch=0), 128, 2),
    (dict(dstate=-1), 128, 2),
    ({}, 96, 3),                          # chunk_len not supported
    (dict(headdim=512), 128, 3),
    (dict(dstate=300), 128, 3),
    (dict(headdim=60), 128, 3),           # bf16 needs P % 8 == 0
    (dict(dtype="f32", headdim=60), 128, 0),  # fp32 accepts any P <= 256
])
def test_dims_validation(lib, kw, chunk, code):
    d = dims(**kw)
    lay = binding.WorkspaceLayout()
    assert lib.ssd_workspace_layout(ctypes.byref(d), chunk, ctypes.byref(lay)) == code
    assert (lib.ssd_workspace_bytes(ctypes.byref(d), chunk) > 0) == (code == 0)


FAKE = 0x10000  # never dereferenced: each call below fails its host checks


def call_forward(lib, d, chunk=128, **ptrs):
    p = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, h0=None, y=FAKE, fin=None)
    p.update(ptrs)
    v = {k: (None if val is None else ctypes.c_void_p(val)) for k, val in p.items()}
    return lib.ssd_forward(ctypes.byref(d), v["x"], v["dt"], v["A"], v["B"], v["C"], v["D"],
                           chunk, v["h0"], v["y"], v["fin"], None)


@pytest.mark.parametrize("name", ["x", "dt", "A", "B", "C", "y"])
def test_null_required_pointer(lib, name):
    assert call_forward(lib, dims(), **{name: None}) == 1


@pytest.mark.parametrize("name", ["x", "dt", "A", "B", "C", "D", "h0", "y", "fin"])
def test_misaligned_pointer(lib, name):
    assert call_forward(lib, dims(), **{name: FAKE + 4}) == 4


def test_bad_dims_before_pointers(lib):
    assert call_forward(lib, dims(nheads=6, ngroups=4)) == 2
    assert lib.ssd_forward(None, None, None, None, None, None, None, 128, None, None, None,
                           None) == 1


def test_workspace_too_small(lib):
    d = dims()
    need = binding.workspace_bytes(d, 128)
    f = ctypes.c_void_p(FAKE)
    args = [ctypes.byref(d), f, f, f, f, f, None, 128, None, f, None]
    assert lib.ssd_forward_ws(*args, None, need, None) == 7
    assert lib.ssd_forward_ws(*args, ctypes.c_void_p(1 << 20), need - 1, None) == 7
    assert lib.ssd_forward_ws(*args, ctypes.c_void_p((1 << 20) + 16), need, None) == 7


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 2, 16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.forward(x, torch.zeros(1, 64, 2), torch.zeros(2), torch.zeros(1, 64, 1, 16),
                        torch.zeros(1, 64, 1, 16), chunk_len=64)


def test_step_argument_checks(lib):
    """ssd_step validates before any CUDA call (the pointers are never touched)."""
    f = ctypes.c_void_p(FAKE)

    def call(d, **kw):
        v = dict(x=f, dt=f, A=f, B=f, C=f, D=None, state=f, y=f)
        v.update(kw)
        return lib.ssd_step(ctypes.byref(d) if d is not None else None, v["x"], v["dt"], v["A"],
                            v["B"], v["C"], v["D"], v["state"], v["y"], None)

    assert call(None) == 1
    for name in ("x", "dt", "A", "B", "C", "state", "y"):
        assert call(binding.make_dims(2, 1, 4, 64, 128, 2, "bf16"), **{name: None}) == 1, name
    assert call(binding.make_dims(2, 2, 4, 64, 128, 2, "bf16")) == 2       # seqlen must be 1
    assert call(binding.make_dims(2, 1, 4, 64, 128, 3, "bf16")) == 2       # H % G
    assert call(binding.make_dims(2, 1, 4, 300, 128, 2, "f32")) == 3       # headdim > 256
    bad = binding.make_dims(2, 1, 4, 64, 128, 2, "bf16")
    bad.dtype = 7
    assert call(bad) == 3


def test_binding_step_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        binding.step(torch.zeros(1, 2, 16, 16), torch.zeros(1, 2, 16), torch.zeros(1, 2),
                     torch.zeros(2), torch.zeros(1, 1, 16), torch.zeros(1, 1, 16))


def test_block_argument_checks(lib):
    """ssd_forward_block rejects a deferred norm without rstd_out, a norm eps
    <= 0, a misaligned neighbour pointer and a nonzero reserved field before
    anything is launched or allocated."""
    d = dims()
    f = ctypes.c_void_p(FAKE)

    def call(**kw):
        o = binding.BlockOpts(**kw)
        return lib.ssd_forward_block(ctypes.byref(d), f, f, f, f, f, None, 128, None, f, None,
                                     ctypes.byref(o), None, 0, None)

    assert call(norm_weight=FAKE, norm_eps=1e-5, norm_apply=0) == 1       # no rstd_out
    assert call(norm_weight=FAKE, norm_eps=0.0, norm_apply=1) == 2         # eps <= 0
    assert call(z=FAKE + 4) == 4
    assert call(dt_bias=FAKE + 8) == 4
    assert call(reserved0=1) == 2
    # the dt transform adds one fp32 [B, T, H] array to the workspace
    base = binding.workspace_bytes(d, 128)
    assert binding.block_workspace_bytes(d, 128, False) == base
    assert binding.block_workspace_bytes(d, 128, True) >= base + 2 * 512 * 8 * 4


def test_ragged_length_layout(lib):
    """A length that is not a multiple of chunk_len: the full chunks keep their
    kernels, one launch more runs the tail, and the workspace holds the state
    between them; shorter than one chunk, only the tail kernel runs."""
    full = binding.workspace_layout(dims(seqlen=512), 128)
    ragged = binding.workspace_layout(dims(seqlen=600), 128)
    assert ragged.launches == full.launches + 1
    assert ragged.total_bytes >= full.total_bytes + 2 * 8 * 64 * 128 * 4
    short = binding.workspace_layout(dims(seqlen=100), 128)
    assert short.launches == 1


def test_varlen_argument_checks(lib):
    """ssd_forward_varlen validates the packing before anything runs: batch 1,
    cu_seqlens from 0 to seqlen and non-decreasing; the workspace is the
    largest one of its sequences' plans."""
    d = binding.make_dims(1, 1000, 8, 64, 128, 2, "bf16")
    i64 = ctypes.POINTER(ctypes.c_int64)

    def ws(cu, q=256):
        a = np.asarray(cu, dtype=np.int64)
        return lib.ssd_varlen_workspace_bytes(ctypes.byref(d), a.ctypes.data_as(i64), a.size - 1, q)

    good = ws([0, 300, 300, 1000])
    assert good > 0
    one = binding.make_dims(1, 700, 8, 64, 128, 2, "bf16")
    assert good == binding.workspace_bytes(one, 256)  # the longest sequence's plan
    assert ws([0, 300, 999]) == 0                       # does not end at seqlen
    assert ws([1, 300, 1000]) == 0                      # does not start at 0
    assert ws([0, 600, 300, 1000]) == 0                 # decreasing
    d2 = binding.make_dims(2, 1000, 8, 64, 128, 2, "bf16")
    a = np.asarray([0, 1000], dtype=np.int64)
    assert lib.ssd_varlen_workspace_bytes(ctypes.byref(d2), a.ctypes.data_as(i64), 1, 256) == 0  # batch != 1
    # the entry point returns the same errors before touching any pointer
    bad = np.asarray([0, 600, 300, 1000], dtype=np.int64)
    st = lib.ssd_forward_varlen(ctypes.byref(d), bad.ctypes.data_as(i64), 3, None, None, None, None, None, None,
                                256, None, None, None, None, 0, None)
    assert st == 2  # SSD_ERR_INVALID_DIM
    cu = np.asarray([0, 300, 1000], dtype=np.int64)
    st = lib.ssd_forward_varlen(ctypes.byref(d), cu.ctypes.data_as(i64), 2, None, None, None, None, None, None,
                                256, None, None, None, None, 0, None)
    assert st == 1  # SSD_ERR_NULL_ARG


def test_backward_argument_checks(lib):
    """ssd_backward validates before anything runs: missing required tensors
    give SSD_ERR_NULL_ARG, more heads than its per-row kernels hold give
    SSD_ERR_UNSUPPORTED (no pointer is touched on either path)."""
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: the checks return first

    def call(d, ptr):
        return lib.ssd_backward(ctypes.byref(d), ptr, ptr, ptr, ptr, ptr, None, 128, None, ptr, None, ptr, ptr,
                                ptr, ptr, ptr, None, None, None)

    d = binding.make_dims(1, 256, 4, 64, 64, 1, "bf16")
    assert call(d, None) == 1  # SSD_ERR_NULL_ARG
    many = binding.make_dims(1, 256, 12289, 64, 64, 1, "bf16")
    assert call(many, fake) == 3  # SSD_ERR_UNSUPPORTED
