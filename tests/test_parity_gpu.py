"""GPU parity: libssd.so against the fp64 oracle, element by element.

Tolerance (max |y_gpu - y_oracle| / max |y_oracle|, and the same for the final
state): 1e-4 for fp32 storage, 2e-2 for bf16 storage.  Every case, the
full-size workloads included, is compared in full.
"""
import numpy as np
import pytest
import torch

from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import WORKLOADS, make_inputs, make_workload

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(inp):
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    dev = torch.device("cuda:0")
    t = lambda a, ty=torch.float32: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(ty)  # noqa: E731
    return dict(x=t(inp.x, dt), dt=t(inp.dt), A=t(inp.A), B=t(inp.B, dt), C=t(inp.C, dt),
                D=t(inp.D), init_state=t(inp.h0))


def run_gpu(inp, final=True, **kw):
    a = to_dev(inp)
    out = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"],
                          chunk_len=inp.chunk_len, init_state=a["init_state"],
                          return_final_state=final, **kw)
    torch.cuda.synchronize()
    assert binding.device_status() == 0  # no bounded device wait expired
    if final:
        y, f = out
        return y.double().cpu().numpy(), f.double().cpu().numpy()
    return out.double().cpu().numpy(), None


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def check_full(inp, oracle, final=True):
    y, f = run_gpu(inp, final=final)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    tol = TOL[inp.dtype]
    assert np.isfinite(y).all()
    assert rel(y, yr) <= tol, rel(y, yr)
    if final:
        assert rel(f, fr) <= tol, rel(f, fr)
    return rel(y, yr), (rel(f, fr) if final else None)


def check_sampled(inp, oracle, units, final=True):
    y, f = run_gpu(inp, final=final)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0,
                                  units=units)
    tol = TOL[inp.dtype]
    assert np.isfinite(y).all()
    ys = np.stack([y[b, :, h] for b, h in units])
    yrs = np.stack([yr[b, :, h] for b, h in units])
    assert rel(ys, yrs) <= tol, rel(ys, yrs)
    if final:
        fs = np.stack([f[b, h] for b, h in units])
        frs = np.stack([fr[b, h] for b, h in units])
        assert rel(fs, frs) <= tol, rel(fs, frs)


# ---------------------------------------------------------------------------
# small shapes, compared in full
# ---------------------------------------------------------------------------
def test_tiny_f32_workload(oracle):
    check_full(make_workload("tiny_f32"), oracle)


@pytest.mark.parametrize("shape", [
    dict(batch=1, seqlen=64, nheads=1, headdim=16, dstate=16, ngroups=1, chunk_len=64),
    dict(batch=2, seqlen=96, nheads=3, headdim=5, dstate=7, ngroups=1, chunk_len=32),
    dict(batch=1, seqlen=256, nheads=4, headdim=64, dstate=128, ngroups=2, chunk_len=128),
    dict(batch=1, seqlen=512, nheads=2, headdim=256, dstate=256, ngroups=2, chunk_len=256),
    # eight heads per group share one block's scores; P and N not multiples of 16
    dict(batch=2, seqlen=256, nheads=16, headdim=48, dstate=40, ngroups=2, chunk_len=128),
])
@pytest.mark.parametrize("h0", [False, True])
def test_f32_shapes(oracle, shape, h0):
    inp = make_inputs(**shape, dtype="f32", seed=7, init_state=h0)
    check_full(inp, oracle)


@pytest.mark.parametrize("shape", [
    dict(batch=1, seqlen=256, nheads=2, headdim=64, dstate=128, ngroups=1, chunk_len=256),
    dict(batch=2, seqlen=512, nheads=4, headdim=64, dstate=128, ngroups=1, chunk_len=128),
    dict(batch=1, seqlen=512, nheads=8, headdim=64, dstate=64, ngroups=2, chunk_len=64),
    dict(batch=1, seqlen=768, nheads=4, headdim=64, dstate=16, ngroups=4, chunk_len=256),
    dict(batch=1, seqlen=512, nheads=2, headdim=64, dstate=256, ngroups=1, chunk_len=256),
    dict(batch=1, seqlen=256, nheads=2, headdim=32, dstate=32, ngroups=1, chunk_len=64),
    dict(batch=3, seqlen=1024, nheads=6, headdim=64, dstate=128, ngroups=3, chunk_len=256),
    dict(batch=1, seqlen=512, nheads=2, headdim=64, dstate=32, ngroups=1, chunk_len=256),
    dict(batch=1, seqlen=1024, nheads=24, headdim=64, dstate=32, ngroups=2, chunk_len=256),
    dict(batch=1, seqlen=1024, nheads=12, headdim=64, dstate=64, ngroups=2, chunk_len=256),
    dict(batch=2, seqlen=1024, nheads=10, headdim=64, dstate=16, ngroups=5, chunk_len=128),
])
@pytest.mark.parametrize("h0", [False, True])
def test_bf16_shapes(oracle, shape, h0):
    inp = make_inputs(**shape, dtype="bf16", seed=11, init_state=h0)
    check_full(inp, oracle)


def test_tensor_core_path_selected():
    """bf16 with P = 64 runs the tcgen05 kernels for every chunk_len (64 as
    128-token chunks) and dstate, and the scan engine is a tensor-core one."""
    for n in (16, 32, 64, 128, 256):
        for q in (64, 128, 256):
            lay = binding.workspace_layout(binding.make_dims(2, 1024, 8, 64, n, 1, "bf16"), q)
            assert lay.tensor_core == 1 and lay.s_in_dtype == binding.SSD_BF16, (n, q)
            assert binding.SCAN_ENGINES[lay.scan_engine] != "simt", (n, q)
            # dstate 32 takes the block-factored scan, 64 the presolved single
            # pass, 256 the chunk-wide scan on 128-token chunks; the others run
            # 256-token chunks
            want = {32: "block_factored", 64: "single_pass", 256: "chunk_wide"}.get(n)
            if want:
                assert binding.SCAN_ENGINES[lay.scan_engine] == want, (n, q)
            assert lay.chunk_len == (128 if n == 256 else 256), (n, q)
    lay = binding.workspace_layout(binding.make_dims(2, 1024, 8, 32, 64, 1, "bf16"), 128)
    assert lay.tensor_core == 0


def test_no_skip_term(oracle):
    inp = make_inputs(1, 256, 2, 64, 128, 1, 128, dtype="bf16", seed=3)
    inp.D = None
    check_full(inp, oracle)


@pytest.mark.parametrize("dstate", [16, 32, 64, 128, 256])
def test_decay_range_across_the_chunk(oracle, dstate):
    """Per-token decays of about e^-0.4 (head 0): each 128-token tile spans ~e^-51
    but the 256-token chunk ~e^-102, so the chunk-wide scan moves its reference
    to the middle of the chunk; head 1 stays below the threshold, head 2 exceeds
    it inside a tile (block-factored path), head 3 barely decays."""
    inp = make_inputs(2, 1024, 4, 64, dstate, 1, 256, dtype="bf16", seed=19, init_state=True, h0_std=1.0)
    rng = np.random.default_rng(19)
    inp.dt = rng.uniform(0.3, 0.5, size=inp.dt.shape).astype(np.float32)
    inp.A = np.array([-1.0, -0.5, -2.0, -0.01], dtype=np.float32)
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    for h in range(4):
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))
    # the carried state reaches the first tokens of every chunk
    yc = y[:, 256::256, 0][:, :, None]
    yrc = yr[:, 256::256, 0][:, :, None]
    assert rel(yc, yrc) <= TOL["bf16"]


@pytest.mark.parametrize("shape", [
    dict(batch=2, seqlen=677, nheads=6, headdim=64, dstate=256, ngroups=3, chunk_len=256),
    dict(batch=1, seqlen=1024, nheads=8, headdim=64, dstate=256, ngroups=1, chunk_len=128),
    dict(batch=2, seqlen=384, nheads=4, headdim=64, dstate=256, ngroups=2, chunk_len=64),
])
@pytest.mark.parametrize("h0", [False, True])
def test_dstate_256_chunk_wide(oracle, shape, h0):
    """dstate 256 on the chunk-wide tensor-core scan at 128-token chunks, for
    every caller chunk_len, a ragged length (tail kernel) and groups."""
    inp = make_inputs(**shape, dtype="bf16", seed=23, init_state=h0)
    d = binding.make_dims(**{k: shape[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate",
                                                     "ngroups")}, dtype="bf16")
    lay = binding.workspace_layout(d, shape["chunk_len"])
    assert binding.SCAN_ENGINES[lay.scan_engine] == "chunk_wide" and lay.chunk_len == 128
    check_full(inp, oracle)


def test_dstate_256_steep_list(oracle):
    """Every tile of every head but head 1 decays past the chunk-wide scan's
    range (at least e^-150 per 128 tokens), so it lists 7 * 2 * 16 = 224 tiles
    for the per-tile scan, which walks the list with one CTA per SM: more items
    than CTAs, so most CTAs take two."""
    inp = make_inputs(2, 2048, 8, 64, 256, 2, 256, dtype="bf16", seed=29, init_state=True, h0_std=1.0)
    rng = np.random.default_rng(29)
    inp.dt = rng.uniform(0.3, 0.5, size=inp.dt.shape).astype(np.float32)
    inp.A = np.array([-4.0, -0.05, -8.0, -16.0, -3.0, -5.0, -6.0, -7.0], dtype=np.float32)
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    for h in range(8):
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))


@pytest.mark.parametrize("shape", [
    # 4 chains of 8 chunks over 32 CTAs: every range inside one chain
    dict(batch=1, seqlen=2048, nheads=8, headdim=64, dstate=64, ngroups=2, chunk_len=256),
    # 9 chains, 128-token chunks and a ragged tail (the tail kernel continues from the final state)
    dict(batch=3, seqlen=1000, nheads=6, headdim=64, dstate=64, ngroups=3, chunk_len=128),
    # 32 chains over 148 CTAs: ranges of about 3.5 chunks, most spanning two chains
    dict(batch=2, seqlen=4096, nheads=32, headdim=64, dstate=64, ngroups=1, chunk_len=256),
])
@pytest.mark.parametrize("h0", [False, True])
def test_presolved_single_pass(oracle, shape, h0):
    """The presolved single pass: each CTA's range starts from the state that the
    range-state passes computed (the partial states of the ranges before it,
    chained along the chain), not from a hand-off."""
    d = binding.make_dims(**{k: shape[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate",
                                                     "ngroups")}, dtype="bf16")
    lay = binding.workspace_layout(d, shape["chunk_len"])
    assert lay.single_pass == 1 and lay.launches == 5 + (1 if shape["seqlen"] % lay.chunk_len else 0)
    inp = make_inputs(**shape, dtype="bf16", seed=31, init_state=h0)
    check_full(inp, oracle)


def test_presolved_single_pass_steep_tiles(oracle):
    """Steep heads on the presolved path: the chunks of flagged tiles get their
    s_in written and the block-factored scan finishes those tiles; the range
    states stay exact (their factors never exceed 1)."""
    inp = make_inputs(2, 2048, 8, 64, 64, 2, 256, dtype="bf16", seed=37, init_state=True, h0_std=1.0)
    rng = np.random.default_rng(37)
    inp.dt = rng.uniform(0.3, 0.5, size=inp.dt.shape).astype(np.float32)
    inp.A = np.array([-4.0, -0.05, -16.0, -0.5, -1.0, -0.01, -2.0, -8.0], dtype=np.float32)
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    for h in range(8):
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))


@pytest.mark.parametrize("chunk_len", [128, 256])
def test_zero_dt_tokens(oracle, chunk_len):
    """dt = 0 on a run of tokens (the state holds, only D x reaches y there) and on
    every token of one head (y = C h0 + D x); the other tokens keep their dt."""
    inp = make_inputs(2, 1024, 4, 64, 128, 1, chunk_len, dtype="bf16", seed=17, init_state=True)
    inp.dt[0, 100:260, 1] = 0.0
    inp.dt[1, 300:301, 0] = 0.0
    inp.dt[:, :, 3] = 0.0
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    for h in range(4):
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))


def test_final_state_may_alias_init_state(oracle):
    inp = make_inputs(1, 512, 4, 64, 128, 2, 256, dtype="bf16", seed=5, init_state=True)
    a = to_dev(inp)
    h = a["init_state"].clone()
    y, f = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=256,
                           init_state=h, final_out=h)
    torch.cuda.synchronize()
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert rel(y.double().cpu().numpy(), yr) <= 2e-2
    assert rel(h.double().cpu().numpy(), fr) <= 2e-2


def test_strong_decay_stays_finite(oracle):
    """dt*|A| up to ~16 per token: the decays underflow to zero, never overflow."""
    inp = make_inputs(1, 512, 4, 64, 128, 1, 256, dtype="bf16", seed=9, init_state=True)
    inp.dt = (inp.dt * 10.0).astype(np.float32)
    check_full(inp, oracle)


def test_steep_decay_inside_32_token_blocks(oracle):
    """A_h = -16 and dt in [0.2, 1]: the decay across any 32 tokens exceeds e^-80,
    so the chunk scan's diagonal blocks take the per-element exact path; one head
    keeps a gentle decay so both paths meet in the same launch."""
    inp = make_inputs(1, 1024, 4, 64, 128, 1, 256, dtype="bf16", seed=13, init_state=True)
    rng = np.random.default_rng(13)
    inp.dt = rng.uniform(0.2, 1.0, size=inp.dt.shape).astype(np.float32)
    inp.A = np.array([-16.0, -16.0, -12.0, -0.01], dtype=np.float32)
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert np.isfinite(y).all() and np.isfinite(f).all()
    for h in range(4):  # per head: the gentle head's scale must not hide the others
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))


def test_chunk_len_invariance_on_gpu(oracle):
    ys = []
    for q in (64, 128, 256):
        inp = make_inputs(1, 1024, 4, 64, 128, 1, q, dtype="bf16", seed=21)
        y, f = run_gpu(inp)
        ys.append(y)
    yr, _ = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D)
    for y in ys:
        assert rel(y, yr) <= 2e-2


def test_repeated_calls_deterministic():
    inp = make_inputs(2, 1024, 8, 64, 128, 1, 256, dtype="bf16", seed=2)
    y1, f1 = run_gpu(inp)
    y2, f2 = run_gpu(inp)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(f1, f2)


def test_workspace_entry_point_and_intermediates(oracle):
    """ssd_forward_ws gives the same output, and the workspace afterwards
    holds each stage's intermediates, checked against the fp64 chunked form so
    a failure names its kernel."""
    inp = make_inputs(1, 512, 4, 64, 128, 2, 128, dtype="bf16", seed=4, init_state=True)
    a = to_dev(inp)
    d = binding.make_dims(1, 512, 4, 64, 128, 2, "bf16")
    lay = binding.workspace_layout(d, 128)
    ws = torch.zeros(lay.total_bytes, dtype=torch.uint8, device="cuda:0")
    y, f = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=128,
                           init_state=a["init_state"], return_final_state=True, workspace=ws)
    y0, f0 = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=128,
                             init_state=a["init_state"], return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(y, y0) and torch.equal(f, f0)
    # the intermediates describe the chunks the kernels ran (lay.chunk_len)
    q = lay.chunk_len
    _, _, it = oracle.ssd_chunked(inp.x, inp.dt, inp.A, inp.B, inp.C, q, D=inp.D, h0=inp.h0,
                                  intermediates=True)
    nc = 512 // q

    def view(off, count, dtype):
        return ws[off: off + count * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    l = view(lay.l_offset, 4 * nc * q, torch.float32).double().cpu().numpy().reshape(1, 4, nc, q)
    w = view(lay.w_offset, 4 * nc * q, torch.float32).double().cpu().numpy().reshape(1, 4, nc, q)
    al = view(lay.alpha_offset, 4 * nc, torch.float32).double().cpu().numpy().reshape(1, 4, nc)
    stdt = torch.bfloat16 if lay.states_dtype == binding.SSD_BF16 else torch.float32
    S = view(lay.states_offset, nc * 4 * 64 * 128, stdt).double().cpu().numpy()
    sdt = torch.bfloat16 if lay.s_in_dtype == binding.SSD_BF16 else torch.float32
    s_in = view(lay.s_in_offset, nc * 4 * 64 * 128, sdt).double().cpu().numpy()
    assert rel(l, it["l"]) < 1e-5          # ssd_chunk_cumsum
    assert rel(al, it["alpha"]) < 1e-5
    assert rel(w, it["w"]) < 1e-5
    assert rel(S.reshape(it["S"].shape), it["S"]) < 2e-2          # ssd_chunk_state
    assert rel(s_in.reshape(it["s_in"].shape), it["s_in"]) < 2e-2  # ssd_state_passing


# ---------------------------------------------------------------------------
# fused chunk_state + state_passing (enough (batch, head pair) units)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [
    dict(batch=3, seqlen=512, nheads=64, headdim=64, dstate=32, ngroups=1, chunk_len=128),
    dict(batch=2, seqlen=256, nheads=96, headdim=64, dstate=32, ngroups=2, chunk_len=128),
    dict(batch=2, seqlen=512, nheads=90, headdim=64, dstate=16, ngroups=1, chunk_len=256),
    dict(batch=1, seqlen=256, nheads=93, headdim=64, dstate=32, ngroups=3, chunk_len=128),
])
@pytest.mark.parametrize("h0", [False, True])
def test_fused_state_path(oracle, shape, h0):
    inp = make_inputs(**shape, dtype="bf16", seed=17, init_state=h0)
    d = binding.make_dims(**{k: shape[k] for k in ("batch", "seqlen", "nheads", "headdim",
                                                     "dstate", "ngroups")}, dtype="bf16")
    assert binding.workspace_layout(d, shape["chunk_len"]).fused_state == 1
    check_full(inp, oracle)


def test_fused_state_intermediates(oracle):
    """s_in written by the fused kernel, against the fp64 chunked form."""
    shape = dict(batch=3, seqlen=512, nheads=64, headdim=64, dstate=32, ngroups=1)
    inp = make_inputs(**shape, chunk_len=128, dtype="bf16", seed=18, init_state=True)
    a = to_dev(inp)
    lay = binding.workspace_layout(binding.make_dims(**shape, dtype="bf16"), 128)
    assert lay.fused_state == 1
    ws = torch.zeros(lay.total_bytes, dtype=torch.uint8, device="cuda:0")
    binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=128,
                    init_state=a["init_state"], return_final_state=True, workspace=ws)
    torch.cuda.synchronize()
    _, _, it = oracle.ssd_chunked(inp.x, inp.dt, inp.A, inp.B, inp.C, lay.chunk_len, D=inp.D, h0=inp.h0,
                                  intermediates=True)
    n = it["s_in"].size
    s_in = ws[lay.s_in_offset: lay.s_in_offset + 2 * n].view(torch.bfloat16)
    s_in = s_in.double().cpu().numpy().reshape(it["s_in"].shape)
    assert rel(s_in, it["s_in"]) < 2e-2


# ---------------------------------------------------------------------------
# the single-pass kernel (chunk state + state passing + scan in one launch)
# ---------------------------------------------------------------------------
def single_pass(shape):
    d = binding.make_dims(**{k: shape[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate",
                                                     "ngroups")}, dtype="bf16")
    return binding.workspace_layout(d, shape["chunk_len"]).single_pass == 1


SINGLE_SHAPES = [
    # fewer (batch, pair) chains than SMs: one CTA walks each chain
    dict(batch=1, seqlen=512, nheads=128, headdim=64, dstate=128, ngroups=1, chunk_len=256),
    dict(batch=2, seqlen=1024, nheads=64, headdim=64, dstate=128, ngroups=4, chunk_len=128),
    # more chains than SMs: tickets round-robin, states handed between CTAs
    dict(batch=4, seqlen=1024, nheads=80, headdim=64, dstate=128, ngroups=1, chunk_len=256),
    dict(batch=3, seqlen=768, nheads=112, headdim=64, dstate=128, ngroups=2, chunk_len=128),
    # dstate 64: one 64-column slab per operand, a four-stage x ring
    dict(batch=2, seqlen=1024, nheads=96, headdim=64, dstate=64, ngroups=1, chunk_len=256),
    dict(batch=4, seqlen=512, nheads=80, headdim=64, dstate=64, ngroups=2, chunk_len=128),
]


@pytest.mark.parametrize("shape", SINGLE_SHAPES)
@pytest.mark.parametrize("h0", [False, True])
def test_single_pass_shapes(oracle, shape, h0):
    assert single_pass(shape)
    inp = make_inputs(**shape, dtype="bf16", seed=31, init_state=h0)
    check_full(inp, oracle)


def test_single_pass_no_skip_no_final(oracle):
    shape = SINGLE_SHAPES[2]
    inp = make_inputs(**shape, dtype="bf16", seed=32, init_state=True)
    inp.D = None
    check_full(inp, oracle, final=False)


@pytest.mark.parametrize("shape", [SINGLE_SHAPES[0], SINGLE_SHAPES[3], SINGLE_SHAPES[5]])
def test_single_pass_steep_and_zero_dt(oracle, shape):
    """Per head: a decay steep enough that tiles go to the block-factored scan,
    a decay range across the chunk (reference moved to the middle), zero dt on
    a run of tokens, and a gentle decay, all in one launch."""
    assert single_pass(shape)
    inp = make_inputs(**shape, dtype="bf16", seed=33, init_state=True, h0_std=1.0)
    rng = np.random.default_rng(33)
    H = shape["nheads"]
    A = inp.A.copy()
    dt = inp.dt.copy()
    A[0::4] = -16.0                                      # steep: tiles listed
    dt[:, :, 0::4] = rng.uniform(0.2, 1.0, size=dt[:, :, 0::4].shape)
    A[1::4] = -1.0                                       # ~e^-0.4 per token
    dt[:, :, 1::4] = rng.uniform(0.3, 0.5, size=dt[:, :, 1::4].shape)
    dt[:, 100:260, 2::4] = 0.0                           # zero dt: skip term only
    A[3::4] = -0.01
    inp.A, inp.dt = A.astype(np.float32), dt.astype(np.float32)
    y, f = run_gpu(inp)
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert np.isfinite(y).all() and np.isfinite(f).all()
    for h in range(min(H, 8)):
        assert rel(y[:, :, h], yr[:, :, h]) <= TOL["bf16"], (h, rel(y[:, :, h], yr[:, :, h]))
        assert rel(f[:, h], fr[:, h]) <= TOL["bf16"], (h, rel(f[:, h], fr[:, h]))
    assert rel(y, yr) <= TOL["bf16"] and rel(f, fr) <= TOL["bf16"]


def test_single_pass_final_aliases_init(oracle):
    shape = SINGLE_SHAPES[2]
    inp = make_inputs(**shape, dtype="bf16", seed=34, init_state=True)
    a = to_dev(inp)
    h = a["init_state"].clone()
    y, _ = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=shape["chunk_len"],
                           init_state=h, final_out=h)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert rel(y.double().cpu().numpy(), yr) <= 2e-2
    assert rel(h.double().cpu().numpy(), fr) <= 2e-2


def test_single_pass_repeated_calls_deterministic():
    inp = make_inputs(**SINGLE_SHAPES[3], dtype="bf16", seed=35, init_state=True)
    y1, f1 = run_gpu(inp)
    y2, f2 = run_gpu(inp)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(f1, f2)


# ---------------------------------------------------------------------------
# lengths that are not a multiple of chunk_len: full chunks, then the tail
# kernel from the state they leave (or from h0 when there is no full chunk)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [
    dict(batch=2, seqlen=1000, nheads=8, headdim=64, dstate=128, ngroups=2, chunk_len=256, dtype="bf16"),
    dict(batch=1, seqlen=600, nheads=128, headdim=64, dstate=128, ngroups=1, chunk_len=256, dtype="bf16"),
    dict(batch=2, seqlen=100, nheads=4, headdim=64, dstate=64, ngroups=1, chunk_len=128, dtype="bf16"),
    dict(batch=1, seqlen=700, nheads=2, headdim=64, dstate=256, ngroups=1, chunk_len=256, dtype="bf16"),
    dict(batch=1, seqlen=300, nheads=2, headdim=16, dstate=16, ngroups=1, chunk_len=64, dtype="f32"),
    dict(batch=2, seqlen=200, nheads=3, headdim=32, dstate=8, ngroups=3, chunk_len=32, dtype="f32"),
])
@pytest.mark.parametrize("h0", [False, True])
def test_ragged_lengths(oracle, shape, h0):
    inp = make_inputs(**shape, seed=51, init_state=h0)
    check_full(inp, oracle)


def test_ragged_length_with_final_aliasing_init(oracle):
    inp = make_inputs(2, 1000, 8, 64, 128, 2, 256, dtype="bf16", seed=52, init_state=True)
    a = to_dev(inp)
    h = a["init_state"].clone()
    y, _ = binding.forward(a["x"], a["dt"], a["A"], a["B"], a["C"], D=a["D"], chunk_len=256,
                           init_state=h, final_out=h)
    torch.cuda.synchronize()
    yr, fr = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert rel(y.double().cpu().numpy(), yr) <= 2e-2
    assert rel(h.double().cpu().numpy(), fr) <= 2e-2


# ---------------------------------------------------------------------------
# full-size workloads, in the bench's launch configuration, every (batch, head)
# unit compared (the persistent grids split runs of heads across CTAs, so a
# fault at a CTA's range boundary shows only in a full comparison)
# ---------------------------------------------------------------------------
def test_mamba2_130m_layer(oracle):
    check_full(make_workload("mamba2_130m"), oracle, final=False)


def test_mamba2_2p7b_layer(oracle):
    check_full(make_workload("mamba2_2p7b"), oracle)


def test_long_context_grouped_layer(oracle):
    check_full(make_workload("long_g8"), oracle)


@pytest.mark.parametrize("name", [n for n in WORKLOADS if n.startswith("sweep_")])
def test_state_chunk_sweep(oracle, name):
    check_full(make_workload(name), oracle)
