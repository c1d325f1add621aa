"""ssd_forward_static: the forward scan on the library's fixed per-device
scratch array, with no allocation.  Its results must equal ssd_forward's bit
for bit (same plan, same kernels), call after call.  The file name keeps it
last in collection, so it also runs after every other test in one process."""
import ctypes

import numpy as np
import pytest
import torch

from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import make_inputs

SSD_ERR_WORKSPACE = 7


def test_static_scratch_size_limit_is_enforced_before_cuda():
    """A workload whose workspace exceeds the 64 MiB scratch is refused on the
    host, before any CUDA call (so this runs without a GPU)."""
    lib = binding.load()
    big = binding.make_dims(batch=4, seqlen=4096, nheads=80, headdim=64, dstate=128,
                            ngroups=1, dtype="bf16")
    assert binding.workspace_bytes(big, 256) > binding.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    st = lib.ssd_forward_static(ctypes.byref(big), fake, fake, fake, fake, fake, None, 256,
                                None, fake, None, None)
    assert st == SSD_ERR_WORKSPACE
    assert binding.STATUS[st] == "SSD_ERR_WORKSPACE"
    small = binding.make_dims(batch=8, seqlen=2048, nheads=24, headdim=64, dstate=128,
                              ngroups=1, dtype="bf16")
    assert binding.workspace_bytes(small, 256) <= binding.STATIC_SCRATCH_BYTES


def _dev(inp):
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    t = lambda a, ty=torch.float32: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0").to(ty)  # noqa: E731
    return dict(x=t(inp.x, dt), dt=t(inp.dt), A=t(inp.A), B=t(inp.B, dt), C=t(inp.C, dt),
                D=t(inp.D), init_state=t(inp.h0))


@pytest.mark.gpu
def test_static_entry_matches_forward_on_consecutive_calls():
    cases = [
        make_inputs(2, 1024, 8, 64, 128, 2, 256, dtype="bf16", seed=31, init_state=True),
        make_inputs(1, 512, 4, 64, 64, 1, 128, dtype="bf16", seed=32, init_state=False),
        make_inputs(1, 256, 2, 16, 16, 1, 64, dtype="f32", seed=33, init_state=True),
    ]
    for inp in cases:
        a = _dev(inp)
        kw = dict(D=a["D"], chunk_len=inp.chunk_len, init_state=a["init_state"],
                  return_final_state=True)
        y_ref, f_ref = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], **kw)
        # two static calls in a row: the second finds the scratch holding the
        # first call's intermediates and must not depend on them
        for _ in range(2):
            y, f = binding.forward_static(a["x"], a["dt"], a["A"], a["B"], a["C"], **kw)
            torch.cuda.synchronize()
            assert binding.device_status() == 0
            assert torch.equal(y, y_ref)
            assert torch.equal(f, f_ref)
