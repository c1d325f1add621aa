"""GPU parity of ssd_forward_varlen: sequences packed along one row, each the
recurrence on its own tokens from its own initial state (akillness.github.io
"State Space Duality and Mamba-2", "Mathematical Foundations").  The oracle is
ssd_recurrent run on every sequence separately; y and every final state are
compared in full at the scan's tolerances.
"""
import numpy as np
import pytest
import torch

from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
DEV = torch.device("cuda:0")


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


CASES = [
    # lengths: a chunk multiple, ragged, shorter than a chunk, empty, long
    dict(lens=[512, 300, 0, 77, 1024], nheads=8, headdim=64, dstate=128, ngroups=2, chunk_len=256, dtype="bf16"),
    # many chains: the long sequences take the single-pass kernel
    dict(lens=[1024, 256, 513], nheads=128, headdim=64, dstate=128, ngroups=1, chunk_len=256, dtype="bf16"),
    dict(lens=[640, 128, 5], nheads=6, headdim=64, dstate=64, ngroups=3, chunk_len=128, dtype="bf16"),
    dict(lens=[200, 0, 56], nheads=4, headdim=16, dstate=16, ngroups=1, chunk_len=64, dtype="f32"),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("h0", [False, True])
def test_varlen_against_per_sequence_oracle(oracle, case, h0):
    lens = case["lens"]
    total = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    inp = make_inputs(1, total, case["nheads"], case["headdim"], case["dstate"], case["ngroups"],
                      case["chunk_len"], dtype=case["dtype"], seed=51)
    rng = np.random.default_rng(52)
    H, P, N = case["nheads"], case["headdim"], case["dstate"]
    hs = rng.normal(0.0, 0.5, size=(len(lens), H, P, N)) if h0 else None
    tt = torch.bfloat16 if case["dtype"] == "bf16" else torch.float32
    t = lambda a, ty=torch.float32: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV).to(ty)  # noqa: E731
    y, fin = binding.forward_varlen(t(inp.x, tt), t(inp.dt), t(inp.A), t(inp.B, tt), t(inp.C, tt), cu,
                                    D=t(inp.D), chunk_len=case["chunk_len"], init_states=t(hs),
                                    return_final_states=True)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    y = y.double().cpu().numpy()
    fin = fin.double().cpu().numpy()
    assert np.isfinite(y).all()
    tol = TOL[case["dtype"]]
    for i, n in enumerate(lens):
        a, b = cu[i], cu[i + 1]
        h0i = None if hs is None else hs[i:i + 1]
        if n == 0:
            want = np.zeros((H, P, N)) if hs is None else hs[i]
            np.testing.assert_array_equal(fin[i], want.astype(np.float32).astype(np.float64))
            continue
        yr, fr = oracle.ssd_recurrent(inp.x[:, a:b], inp.dt[:, a:b], inp.A, inp.B[:, a:b], inp.C[:, a:b],
                                      D=inp.D, h0=h0i)
        assert rel(y[:, a:b], yr) <= tol, (i, rel(y[:, a:b], yr))
        assert rel(fin[i:i + 1], fr) <= tol, (i, rel(fin[i:i + 1], fr))


def test_varlen_one_sequence_equals_forward():
    inp = make_inputs(1, 768, 8, 64, 128, 2, 256, dtype="bf16", seed=53, init_state=True)
    tt = torch.bfloat16
    t = lambda a, ty=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(DEV).to(ty)  # noqa: E731
    args = (t(inp.x, tt), t(inp.dt), t(inp.A), t(inp.B, tt), t(inp.C, tt))
    y0, f0 = binding.forward(*args, D=t(inp.D), chunk_len=256, init_state=t(inp.h0), return_final_state=True)
    y1, f1 = binding.forward_varlen(*args, [0, 768], D=t(inp.D), chunk_len=256, init_states=t(inp.h0),
                                    return_final_states=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(f0, f1)
