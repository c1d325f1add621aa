"""GPU parity of the decode step (ssd_step) against the fp64 oracle step.

Tolerances as for the scan: max |y_gpu - y_oracle| / max |y_oracle| <= 2e-2 for
bf16 storage of x, B, C, y and 1e-4 for fp32; the fp32 state is compared with
1e-5 (one fp32 update from the same starting state).
"""
import numpy as np
import pytest
import torch

from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

TOL_Y = {"f32": 1e-4, "bf16": 2e-2}
TOL_STATE = 1e-5


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def draw(batch, H, P, N, G, dtype, seed, state_std=1.0):
    """One token of synthetic decode inputs (the forward scan's distributions)
    plus a state drawn N(0, state_std^2)."""
    inp = make_inputs(batch, 1, H, P, N, G, 1, dtype=dtype, seed=seed, init_state=True,
                      h0_std=state_std)
    return dict(x=inp.x[:, 0], dt=inp.dt[:, 0], A=inp.A, B=inp.B[:, 0], C=inp.C[:, 0], D=inp.D,
                state=inp.h0)


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0").to(dtype)


def run_step(v, dtype, state_t=None, with_d=True):
    sd = torch.bfloat16 if dtype == "bf16" else torch.float32
    state = dev(v["state"]) if state_t is None else state_t
    y = binding.step(state, dev(v["x"], sd), dev(v["dt"]), dev(v["A"]), dev(v["B"], sd),
                     dev(v["C"], sd), D=dev(v["D"]) if with_d else None)
    torch.cuda.synchronize()
    return y.double().cpu().numpy(), state.double().cpu().numpy()


@pytest.mark.parametrize("shape", [
    dict(batch=2, H=8, P=64, N=128, G=2, dtype="bf16"),   # vectorised, one warp per row
    dict(batch=3, H=4, P=64, N=16, G=1, dtype="bf16"),    # 4 lanes per row
    dict(batch=1, H=6, P=64, N=256, G=3, dtype="bf16"),   # two vectors per lane
    dict(batch=2, H=5, P=40, N=64, G=5, dtype="bf16"),    # ragged row passes
    dict(batch=2, H=4, P=32, N=32, G=2, dtype="f32"),
    dict(batch=2, H=3, P=5, N=20, G=1, dtype="f32"),      # scalar kernel (N not 2^k)
    dict(batch=1, H=2, P=256, N=8, G=1, dtype="f32"),     # scalar kernel, widest P
])
def test_step_matches_oracle(oracle, shape):
    v = draw(shape["batch"], shape["H"], shape["P"], shape["N"], shape["G"], shape["dtype"], seed=31)
    y, s = run_step(v, shape["dtype"])
    yr, sr = oracle.ssd_step(v["state"], v["x"], v["dt"], v["A"], v["B"], v["C"], D=v["D"])
    assert np.isfinite(y).all()
    assert rel(y, yr) <= TOL_Y[shape["dtype"]], rel(y, yr)
    assert rel(s, sr) <= TOL_STATE, rel(s, sr)


def test_step_without_skip(oracle):
    v = draw(2, 4, 64, 128, 1, "bf16", seed=32)
    y, s = run_step(v, "bf16", with_d=False)
    yr, sr = oracle.ssd_step(v["state"], v["x"], v["dt"], v["A"], v["B"], v["C"])
    assert rel(y, yr) <= TOL_Y["bf16"]
    assert rel(s, sr) <= TOL_STATE


def test_step_misaligned_state_takes_scalar_kernel(oracle):
    """A state that starts 4 bytes past a 16-byte boundary: same results."""
    v = draw(2, 4, 64, 128, 2, "bf16", seed=33)
    flat = torch.zeros(v["state"].size + 1, dtype=torch.float32, device="cuda:0")
    state = flat[1:].view(v["state"].shape)
    assert state.data_ptr() % 16 != 0
    state.copy_(dev(v["state"]))
    y, s = run_step(v, "bf16", state_t=state)
    yr, sr = oracle.ssd_step(v["state"], v["x"], v["dt"], v["A"], v["B"], v["C"], D=v["D"])
    assert rel(y, yr) <= TOL_Y["bf16"]
    assert rel(s, sr) <= TOL_STATE


def test_scan_then_steps_continue_the_sequence(oracle):
    """The forward scan over T tokens, then K decode steps on its final state,
    give the oracle recurrence over all T + K tokens."""
    T, K = 512, 6
    inp = make_inputs(2, T + K, 8, 64, 128, 2, 256, dtype="bf16", seed=34, init_state=True)
    sd = torch.bfloat16
    sl = lambda a, s: np.ascontiguousarray(a[:, s])  # noqa: E731
    y_scan, fin = binding.forward(dev(sl(inp.x, slice(0, T)), sd), dev(sl(inp.dt, slice(0, T))),
                                  dev(inp.A), dev(sl(inp.B, slice(0, T)), sd),
                                  dev(sl(inp.C, slice(0, T)), sd), D=dev(inp.D), chunk_len=256,
                                  init_state=dev(inp.h0), return_final_state=True)
    ys = []
    for t in range(T, T + K):
        ys.append(binding.step(fin, dev(inp.x[:, t], sd), dev(inp.dt[:, t]), dev(inp.A),
                               dev(inp.B[:, t], sd), dev(inp.C[:, t], sd), D=dev(inp.D)))
    torch.cuda.synchronize()
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    y_steps = torch.stack(ys, dim=1).double().cpu().numpy()
    assert rel(y_scan.double().cpu().numpy(), yr[:, :T]) <= TOL_Y["bf16"]
    assert rel(y_steps, yr[:, T:]) <= TOL_Y["bf16"], rel(y_steps, yr[:, T:])
    assert rel(fin.double().cpu().numpy(), fr) <= TOL_Y["bf16"]


def test_step_full_size_decode_shape(oracle):
    """The benchmarked decode shape (batch 64, 2.7B heads), checked on sampled
    (batch, head) pairs."""
    v = draw(64, 80, 64, 128, 1, "bf16", seed=35)
    y, s = run_step(v, "bf16")
    pick = [(0, 0), (13, 41), (63, 79), (31, 7)]
    for b, h in pick:
        sub = dict(state=v["state"][b:b + 1, h:h + 1], x=v["x"][b:b + 1, h:h + 1], dt=v["dt"][b:b + 1, h:h + 1],
                   A=v["A"][h:h + 1], B=v["B"][b:b + 1], C=v["C"][b:b + 1], D=v["D"][h:h + 1])
        yr, sr = oracle.ssd_step(sub["state"], sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"], D=sub["D"])
        assert rel(y[b:b + 1, h:h + 1], yr) <= TOL_Y["bf16"]
        assert rel(s[b:b + 1, h:h + 1], sr) <= TOL_STATE
