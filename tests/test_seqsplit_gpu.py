"""GPU parity of the sequence split (structured_state_space_mamba_b200.seqsplit)
with the library's scan as every slice's local pass.

The slices of one sequence are processed in one process, in rank order: each
slice's summary (alpha, S) comes from the library on the GPU, the exchange is
the list of summaries (the collective itself is covered by the gloo tests on
the CPU), every slice's entering state follows from the summaries before it,
and the slice is scanned again from that state.  The stitched y and every
slice's final state must match the oracle's recurrence over the whole sequence
(akillness.github.io "State Space Duality and Mamba-2", "Mathematical
Foundations") at the scan's tolerances.
"""
import numpy as np
import pytest
import torch

from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import make_inputs
from structured_state_space_mamba_b200.seqsplit import entering_state, slice_summary

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
DEV = torch.device("cuda:0")


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def library_scan(x, dt, A, B, C, D, chunk_len, h0):
    return binding.forward(x, dt, A, B, C, D=D, chunk_len=chunk_len, init_state=h0, return_final_state=True)


CASES = [
    # slices of whole chunks, a ragged slice, and a slice shorter than a chunk
    dict(cuts=[0, 1024, 2311, 4096], bsz=2, nheads=8, headdim=64, dstate=128, ngroups=1, chunk_len=256, dtype="bf16"),
    dict(cuts=[0, 700, 777, 1536], bsz=1, nheads=16, headdim=64, dstate=64, ngroups=2, chunk_len=128, dtype="bf16"),
    dict(cuts=[0, 300, 512], bsz=2, nheads=4, headdim=32, dstate=16, ngroups=1, chunk_len=64, dtype="f32"),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("with_h0", [False, True])
def test_sequence_split_on_the_gpu(oracle, case, with_h0):
    cuts = case["cuts"]
    T = cuts[-1]
    H, P, N = case["nheads"], case["headdim"], case["dstate"]
    inp = make_inputs(case["bsz"], T, H, P, N, case["ngroups"], case["chunk_len"], dtype=case["dtype"],
                      seed=71, init_state=with_h0, h0_std=0.5)
    tt = torch.bfloat16 if case["dtype"] == "bf16" else torch.float32
    t = lambda a, ty=torch.float32: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV).to(ty)  # noqa: E731
    A, D = t(inp.A), t(inp.D)
    h0 = t(inp.h0)
    slices = []
    for r in range(len(cuts) - 1):
        a, b = cuts[r], cuts[r + 1]
        slices.append((t(inp.x[:, a:b], tt), t(inp.dt[:, a:b]), t(inp.B[:, a:b], tt), t(inp.C[:, a:b], tt)))
    # 1. every slice's summary; 2. the exchange (in rank order)
    alphas, states = [], []
    for x, dt, Bm, Cm in slices:
        alpha, S = slice_summary(library_scan, x, dt, A, Bm, Cm, case["chunk_len"])
        alphas.append(alpha)
        states.append(S)
    # 3. and 4. every slice from its entering state
    ys, fins = [], []
    for r, (x, dt, Bm, Cm) in enumerate(slices):
        s_in = entering_state(alphas, states, r, h0)
        y, fin = library_scan(x, dt, A, Bm, Cm, D, case["chunk_len"], s_in)
        ys.append(y)
        fins.append(fin)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    y = torch.cat(ys, dim=1).double().cpu().numpy()
    assert np.isfinite(y).all()
    tol = TOL[case["dtype"]]
    y_ref, _ = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert rel(y, y_ref) <= tol, rel(y, y_ref)
    for r in range(len(cuts) - 1):
        e = cuts[r + 1]
        _, f_r = oracle.ssd_recurrent(inp.x[:, :e], inp.dt[:, :e], inp.A, inp.B[:, :e], inp.C[:, :e], h0=inp.h0)
        got = fins[r].double().cpu().numpy()
        assert rel(got, f_r) <= tol, (r, rel(got, f_r))
