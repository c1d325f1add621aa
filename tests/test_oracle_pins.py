"""Pins for the fp64 oracle, checked against things other than itself.

Every check is CPU-only.  The pins are exact identities of the method (fp64,
relative error <= 1e-12), hand-worked values from the printed 3x3
semiseparable matrix, and closed forms computed here with plain numpy:

* recurrence == explicit T x T dual matrix (akillness.github.io "State Space
  Duality and Mamba-2", "Mathematical Foundations": y = M x,
  M[j,i] = C_j (prod_{k=i+1..j} A_k) B_i, diagonal included as in the 3x3 matrix);
* recurrence == chunked algorithm for every chunk length dividing T (aifetchly
  blog "Mamba-2 Architecture", "The Chunked SSD Algorithm"; d-central glossary
  "State Space Duality": the blockwise form is the same operation);
* A = 0: causal linear attention, prefix sums of dt_s x_s B_s^T (aifetchly blog,
  "The Core Duality": linear attention with a mask of ones; x->V, B->K, C->Q);
* dt = 0: y = h0 C + D x and the state is unchanged;
* T = 1 hand formula;
* split sequence with the state carried across the split (the constant-size
  recurrent state of the recurrent mode);
* linearity in x, superposition in (x, h0), group sharing, head permutation;
* the decode step: T single steps == the recurrence over T tokens, and one step
  == the same hand formula written element by element.
"""
import json
import os

import numpy as np
import pytest

from structured_state_space_mamba_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale)


def small(seed=0, batch=2, T=24, H=4, P=3, N=5, G=2, h0=True, dtype="f32"):
    inp = make_inputs(batch, T, H, P, N, G, chunk_len=T, dtype=dtype, seed=seed,
                      init_state=h0, h0_std=0.5)
    return inp


def args(inp, with_h0=True):
    return (inp.x, inp.dt, inp.A, inp.B, inp.C), dict(D=inp.D, h0=inp.h0 if with_h0 else None)


# --------------------------------------------------------------------------
# golden: the printed 3x3 semiseparable matrix, worked by hand
# --------------------------------------------------------------------------
def test_golden_semiseparable_3x3(oracle):
    with open(os.path.join(GOLDEN, "semiseparable_3x3.json")) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        x = np.array(case["x"]).reshape(1, 3, 1, 1)
        dt = np.array(case["dt"]).reshape(1, 3, 1)
        A = np.array([-np.log(2.0)])
        B = np.array(case["B"]).reshape(1, 3, 1, 1)
        C = np.array(case["C"]).reshape(1, 3, 1, 1)
        D = np.array([case["D"]])
        for fn in (oracle.ssd_recurrent, oracle.ssd_quadratic):
            y, fin = fn(x, dt, A, B, C, D=D)
            np.testing.assert_allclose(y.reshape(3), case["y"], rtol=0, atol=1e-12,
                                       err_msg=f"{fn.__name__} {case['name']}")
            np.testing.assert_allclose(fin.reshape(()), case["final"], rtol=0, atol=1e-12)
        for Q in (1, 3):
            y, fin = oracle.ssd_chunked(x, dt, A, B, C, Q, D=D)
            np.testing.assert_allclose(y.reshape(3), case["y"], rtol=0, atol=1e-12)
            np.testing.assert_allclose(fin.reshape(()), case["final"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# dual forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_recurrent_equals_quadratic(oracle, seed):
    inp = small(seed=seed)
    a, kw = args(inp)
    y_r, f_r = oracle.ssd_recurrent(*a, **kw)
    y_q, f_q = oracle.ssd_quadratic(*a, **kw)
    assert rel_err(y_r, y_q) < 1e-12
    assert rel_err(f_r, f_q) < 1e-12


def test_recurrent_equals_quadratic_strong_decay(oracle):
    """Large dt*|A| (decays far below 1) exercises the decay products."""
    inp = small(seed=7, T=40)
    dt = inp.dt * 30.0
    y_r, f_r = oracle.ssd_recurrent(inp.x, dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    y_q, f_q = oracle.ssd_quadratic(inp.x, dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    assert rel_err(y_r, y_q) < 1e-12
    assert rel_err(f_r, f_q) < 1e-12


@pytest.mark.parametrize("Q", [1, 2, 3, 4, 6, 8, 12, 24])
def test_chunk_length_invariance(oracle, Q):
    inp = small(seed=3, T=24)
    a, kw = args(inp)
    y_r, f_r = oracle.ssd_recurrent(*a, **kw)
    y_c, f_c = oracle.ssd_chunked(*a, Q, **kw)
    assert rel_err(y_c, y_r) < 1e-12
    assert rel_err(f_c, f_r) < 1e-12


def test_chunked_intermediates_consistent(oracle):
    """Stage outputs obey their own definitions: alpha = exp(l_last), w at the
    last token = dt, the first incoming state is h0 and the last S/alpha step
    lands on the final state."""
    inp = small(seed=4, T=24)
    a, kw = args(inp)
    y, fin, it = oracle.ssd_chunked(*a, 8, intermediates=True, **kw)
    dt = inp.dt.astype(np.float64)
    l = it["l"]
    # l is the chunk-local inclusive cumsum of dt*A
    dtc = dt.transpose(0, 2, 1).reshape(2, 4, 3, 8)
    np.testing.assert_allclose(l, np.cumsum(dtc * inp.A.astype(np.float64)[None, :, None, None],
                                            axis=-1), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(it["alpha"], np.exp(l[..., -1]), rtol=1e-14)
    np.testing.assert_allclose(it["w"][..., -1], dtc[..., -1], rtol=1e-14)
    np.testing.assert_allclose(it["s_in"][:, 0], inp.h0.astype(np.float64), rtol=1e-14)
    last = it["alpha"][:, :, -1][..., None, None] * it["s_in"][:, -1] + it["S"][:, -1]
    np.testing.assert_allclose(fin, last, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# every intermediate of the chunked form, pinned to the recurrence
# --------------------------------------------------------------------------
# Each stage output of the chunked algorithm (aifetchly blog "Mamba-2
# Architecture", "The Chunked SSD Algorithm", steps 1-2) is a state of the
# recurrence over some token range, so the token-by-token oracle -- itself
# pinned above to the explicit T x T dual matrix and the hand-worked 3x3 case
# -- fixes all of them without restating their formulas:
#   S_c      = final state of the recurrence over chunk c alone, from zero;
#   s_in[c]  = final state of the recurrence over tokens [0, cQ), from h0;
#   alpha_c  = final state over chunk c with x = 0, from an all-ones state;
#   w_s      = final state over chunk c with x zero except at token s, from
#              zero, divided by x_s[p] B_s[n] (the state is w_s x_s B_s^T).

_PIN_Q = 8


def _slice_t(inp, t0, t1):
    return (inp.x[:, t0:t1], inp.dt[:, t0:t1], inp.A, inp.B[:, t0:t1], inp.C[:, t0:t1])


def _intermediate_pins(oracle, inp, Q, it):
    """Check (w, S, alpha, s_in) of the chunked form against recurrence runs;
    returns the largest relative error of each."""
    bsz, T, H, P = inp.x.shape
    N = inp.B.shape[3]
    nc = T // Q
    h0 = inp.h0.astype(np.float64)
    errs = {"S": 0.0, "s_in": 0.0, "alpha": 0.0, "w": 0.0}
    for c in range(nc):
        t0, t1 = c * Q, (c + 1) * Q
        _, S_ref = oracle.ssd_recurrent(*_slice_t(inp, t0, t1))
        errs["S"] = max(errs["S"], rel_err(it["S"][:, c], S_ref))
        if c == 0:
            s_ref = h0
        else:
            _, s_ref = oracle.ssd_recurrent(*_slice_t(inp, 0, t0), h0=h0)
        errs["s_in"] = max(errs["s_in"], rel_err(it["s_in"][:, c], s_ref))
        a = _slice_t(inp, t0, t1)
        _, ones_fin = oracle.ssd_recurrent(np.zeros_like(a[0]), *a[1:],
                                           h0=np.ones((bsz, H, P, N)))
        errs["alpha"] = max(errs["alpha"],
                            rel_err(it["alpha"][:, :, c][..., None, None] * np.ones((P, N)),
                                    ones_fin))
        x64 = a[0].astype(np.float64)
        B64 = a[3].astype(np.float64)
        r = H // inp.B.shape[2]
        for s in range(Q):
            xs = np.zeros_like(x64)
            xs[:, s] = x64[:, s]
            _, fin_s = oracle.ssd_recurrent(xs, *a[1:])
            # fin_s[b,h,p,n] = w_s x_s[b,h,p] B_s[b,g(h),n]: read w at (p, n) = (0, 0)
            denom = x64[:, s, :, 0] * np.repeat(B64[:, s, :, 0], r, axis=1)  # [b,h]
            w_ref = fin_s[:, :, 0, 0] / denom
            errs["w"] = max(errs["w"], rel_err(it["w"][:, :, c, s], w_ref))
    return errs


def test_chunked_intermediates_pinned_to_recurrence(oracle):
    """Every chunk's S, s_in, alpha and every token's w equal the recurrence
    states that define them (fp64, 1e-12)."""
    inp = small(seed=4, T=24)
    a, kw = args(inp)
    _, _, it = oracle.ssd_chunked(*a, _PIN_Q, intermediates=True, **kw)
    errs = _intermediate_pins(oracle, inp, _PIN_Q, it)
    for k, e in errs.items():
        assert e < 1e-12, (k, e)


def test_intermediate_pins_reject_planted_mistakes(oracle):
    """The pins above fail for plausible mistakes in the stage outputs: a flipped
    sign in w's exponent, S and s_in taken one chunk off, and alpha without
    the exponential's last term."""
    inp = small(seed=4, T=24)
    a, kw = args(inp)
    _, _, it = oracle.ssd_chunked(*a, _PIN_Q, intermediates=True, **kw)
    l = it["l"]
    dtc = inp.dt.astype(np.float64).transpose(0, 2, 1).reshape(l.shape)
    planted = {
        "w": dict(it, w=np.exp(l - l[..., -1:]) * dtc),              # exp(l_s - l_last) dt_s
        "S": dict(it, S=np.roll(it["S"], 1, axis=1)),               # chunk offset off by one
        "s_in": dict(it, s_in=np.roll(it["s_in"], -1, axis=1)),     # next chunk's state
        "alpha": dict(it, alpha=np.exp(l[..., -2])),                # decay of Q-1 tokens
    }
    for key, bent in planted.items():
        errs = _intermediate_pins(oracle, inp, _PIN_Q, bent)
        assert errs[key] > 1e-3, (key, errs)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def test_A_zero_is_causal_linear_attention(oracle):
    inp = small(seed=5, T=20)
    A0 = np.zeros_like(inp.A)
    y, fin = oracle.ssd_recurrent(inp.x, inp.dt, A0, inp.B, inp.C, D=inp.D, h0=inp.h0)
    x = inp.x.astype(np.float64)
    dt = inp.dt.astype(np.float64)
    r = inp.x.shape[2] // inp.B.shape[2]
    Bh = np.repeat(inp.B.astype(np.float64), r, axis=2)  # [b,t,h,n]
    Ch = np.repeat(inp.C.astype(np.float64), r, axis=2)
    # S_t = h0 + sum_{s<=t} dt_s x_s B_s^T  (prefix sum), y_t = S_t C_t + D x_t
    outer = dt[..., None, None] * x[..., :, None] * Bh[..., None, :]  # [b,t,h,p,n]
    S = np.cumsum(outer, axis=1) + inp.h0.astype(np.float64)[:, None]
    y_ref = np.einsum("bthpn,bthn->bthp", S, Ch) + inp.D.astype(np.float64)[None, None, :, None] * x
    assert rel_err(y, y_ref) < 1e-12
    assert rel_err(fin, S[:, -1]) < 1e-12


def test_dt_zero_keeps_state(oracle):
    inp = small(seed=6)
    dt0 = np.zeros_like(inp.dt)
    y, fin = oracle.ssd_recurrent(inp.x, dt0, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    r = inp.x.shape[2] // inp.B.shape[2]
    Ch = np.repeat(inp.C.astype(np.float64), r, axis=2)
    y_ref = (np.einsum("bhpn,bthn->bthp", inp.h0.astype(np.float64), Ch)
             + inp.D.astype(np.float64)[None, None, :, None] * inp.x)
    assert rel_err(y, y_ref) < 1e-12
    np.testing.assert_array_equal(fin, inp.h0.astype(np.float64))
    # and with a zero initial state the output is the skip term alone
    y2, fin2 = oracle.ssd_recurrent(inp.x, dt0, inp.A, inp.B, inp.C, D=inp.D)
    np.testing.assert_allclose(y2, inp.D.astype(np.float64)[None, None, :, None] * inp.x,
                               rtol=0, atol=1e-15)
    assert np.all(fin2 == 0)


def test_single_step_hand_formula(oracle):
    inp = small(seed=8, T=1, batch=1, H=2, G=1)
    y, fin = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    x = inp.x[0, 0].astype(np.float64)    # [H,P]
    dt = inp.dt[0, 0].astype(np.float64)  # [H]
    Bv = inp.B[0, 0, 0].astype(np.float64)
    Cv = inp.C[0, 0, 0].astype(np.float64)
    for h in range(2):
        h1 = np.exp(dt[h] * inp.A[h]) * inp.h0[0, h].astype(np.float64) + dt[h] * np.outer(x[h], Bv)
        np.testing.assert_allclose(fin[0, h], h1, rtol=1e-14, atol=1e-16)
        np.testing.assert_allclose(y[0, 0, h], h1 @ Cv + inp.D[h] * x[h], rtol=1e-13, atol=1e-15)


def test_split_sequence_carries_state(oracle):
    inp = small(seed=9, T=30)
    a, kw = args(inp)
    y, fin = oracle.ssd_recurrent(*a, **kw)
    T1 = 11
    sl = lambda v, s: None if v is None else v[:, s]  # noqa: E731
    first = [sl(v, slice(0, T1)) for v in (inp.x, inp.dt)] + [inp.A] + \
            [sl(v, slice(0, T1)) for v in (inp.B, inp.C)]
    second = [sl(v, slice(T1, None)) for v in (inp.x, inp.dt)] + [inp.A] + \
             [sl(v, slice(T1, None)) for v in (inp.B, inp.C)]
    y1, f1 = oracle.ssd_recurrent(*first, D=inp.D, h0=inp.h0)
    y2, f2 = oracle.ssd_recurrent(*second, D=inp.D, h0=f1)
    assert rel_err(np.concatenate([y1, y2], axis=1), y) < 1e-12
    assert rel_err(f2, fin) < 1e-12


def test_linearity_and_superposition(oracle):
    inp = small(seed=10)
    x2 = make_inputs(2, 24, 4, 3, 5, 2, 24, dtype="f32", seed=11).x
    base = (inp.dt, inp.A, inp.B, inp.C)
    ya, fa = oracle.ssd_recurrent(inp.x, *base, D=inp.D)
    yb, fb = oracle.ssd_recurrent(x2, *base, D=inp.D)
    xab = 2.0 * inp.x.astype(np.float64) - 3.0 * x2.astype(np.float64)
    yab, fab = oracle.ssd_recurrent(xab, *base, D=inp.D)
    assert rel_err(yab, 2 * ya - 3 * yb) < 1e-12
    assert rel_err(fab, 2 * fa - 3 * fb) < 1e-12
    # superposition of input and initial state
    yh, fh = oracle.ssd_recurrent(np.zeros_like(inp.x), *base, D=inp.D, h0=inp.h0)
    yfull, ffull = oracle.ssd_recurrent(inp.x, *base, D=inp.D, h0=inp.h0)
    assert rel_err(yfull, ya + yh) < 1e-12
    assert rel_err(ffull, fa + fh) < 1e-12


def test_groups_equal_repeated_single_group(oracle):
    """G = H with B/C repeated per head equals G = 1 (and G = 2 shares B/C
    between consecutive heads: heads 0,1 -> group 0; 2,3 -> group 1)."""
    inp = small(seed=12, G=1, H=4)
    a, kw = args(inp)
    y1, f1 = oracle.ssd_recurrent(*a, **kw)
    Brep = np.repeat(inp.B, 4, axis=2)
    Crep = np.repeat(inp.C, 4, axis=2)
    y4, f4 = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, Brep, Crep, **kw)
    assert rel_err(y4, y1) < 1e-14
    assert rel_err(f4, f1) < 1e-14
    inp2 = small(seed=13, G=2, H=4)
    a2, kw2 = args(inp2)
    y2, f2 = oracle.ssd_recurrent(*a2, **kw2)
    Bx = inp2.B[:, :, [0, 0, 1, 1]]
    Cx = inp2.C[:, :, [0, 0, 1, 1]]
    y2b, f2b = oracle.ssd_recurrent(inp2.x, inp2.dt, inp2.A, Bx, Cx, **kw2)
    assert rel_err(y2b, y2) < 1e-14
    assert rel_err(f2b, f2) < 1e-14


def test_head_permutation(oracle):
    inp = small(seed=14, G=1, H=4)
    a, kw = args(inp)
    y, f = oracle.ssd_recurrent(*a, **kw)
    perm = np.array([2, 0, 3, 1])
    yp, fp = oracle.ssd_recurrent(inp.x[:, :, perm], inp.dt[:, :, perm], inp.A[perm], inp.B,
                                  inp.C, D=inp.D[perm], h0=inp.h0[:, perm])
    assert rel_err(yp, y[:, :, perm]) < 1e-14
    assert rel_err(fp, f[:, perm]) < 1e-14


# --------------------------------------------------------------------------
# plumbing of the oracle itself
# --------------------------------------------------------------------------
def test_units_subset_and_threads(oracle):
    inp = small(seed=15, batch=3, H=4, G=2)
    a, kw = args(inp)
    y, f = oracle.ssd_recurrent(*a, nthreads=1, **kw)
    y4, f4 = oracle.ssd_recurrent(*a, nthreads=4, **kw)
    np.testing.assert_array_equal(y, y4)
    np.testing.assert_array_equal(f, f4)
    units = [(2, 3), (0, 1)]
    ys, fs = oracle.ssd_recurrent(*a, units=units, **kw)
    for b, h in units:
        np.testing.assert_array_equal(ys[b, :, h], y[b, :, h])
        np.testing.assert_array_equal(fs[b, h], f[b, h])
    assert np.isnan(ys[1, :, 0]).all()


def _scalar_variant(variant, x, dt, Bv, Cv, A, D):
    """A scalar recurrence with one planted mistake (or none)."""
    h, out = 0.0, []
    for t in range(len(x)):
        a = np.exp(dt[t] * A)
        if variant == "read_before_update":
            out.append(h * Cv[t] + D * x[t])
            h = a * h + dt[t] * x[t] * Bv[t]
            continue
        if variant == "no_dt_input":
            h = a * h + x[t] * Bv[t]
        elif variant == "decay_after_input":
            h = a * (h + dt[t] * x[t] * Bv[t])
        elif variant == "sign_flip_decay":
            h = np.exp(-dt[t] * A) * h + dt[t] * x[t] * Bv[t]
        else:
            h = a * h + dt[t] * x[t] * Bv[t]
        out.append(h * Cv[t] + D * x[t])
    return np.array(out), h


def test_golden_rejects_planted_mistakes(oracle):
    """The hand-worked 3x3 values catch a dropped dt on the input, a decay
    applied after the input, a sign flip in the exponent and an output read
    before the state update; the unmutated scalar recurrence and the oracle
    both match them."""
    with open(os.path.join(GOLDEN, "semiseparable_3x3.json")) as f:
        gold = json.load(f)
    A = -np.log(2.0)
    for case in gold["cases"]:
        arr = [np.array(case[k], dtype=np.float64) for k in ("x", "dt", "B", "C")]
        y, fin = _scalar_variant("correct", *arr, A, case["D"])
        np.testing.assert_allclose(y, case["y"], atol=1e-12)
        for v in ("no_dt_input", "decay_after_input", "sign_flip_decay", "read_before_update"):
            yv, _ = _scalar_variant(v, *arr, A, case["D"])
            if case["name"] == "unit_step" and v == "no_dt_input":
                continue  # dt = 1 makes that mistake invisible; the other cases catch it
            assert np.max(np.abs(yv - np.array(case["y"]))) > 1e-3, (case["name"], v)


# --------------------------------------------------------------------------
# the decode step (one token of the recurrence)
# --------------------------------------------------------------------------
def test_steps_equal_recurrence(oracle):
    """Applying ssd_step token by token reproduces the recurrence oracle."""
    inp = small(seed=21, T=17, H=6, G=3)
    y_ref, fin_ref = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    state = inp.h0.astype(np.float64)
    ys = []
    for t in range(inp.x.shape[1]):
        y_t, state = oracle.ssd_step(state, inp.x[:, t], inp.dt[:, t], inp.A, inp.B[:, t], inp.C[:, t],
                                     D=inp.D)
        ys.append(y_t)
    assert rel_err(np.stack(ys, axis=1), y_ref) < 1e-12
    assert rel_err(state, fin_ref) < 1e-12


def test_step_hand_formula_elementwise(oracle):
    """One step written out element by element with scalar loops (no numpy
    broadcasting): group map, decay, input outer product, readout and skip."""
    rng = np.random.default_rng(22)
    bsz, H, P, N, G = 2, 4, 3, 5, 2
    state = rng.standard_normal((bsz, H, P, N))
    x = rng.standard_normal((bsz, H, P))
    dt = rng.uniform(0.01, 0.5, size=(bsz, H))
    A = -rng.uniform(0.1, 4.0, size=H)
    B = rng.standard_normal((bsz, G, N))
    C = rng.standard_normal((bsz, G, N))
    D = rng.standard_normal(H)
    y, new = oracle.ssd_step(state, x, dt, A, B, C, D=D)
    import math
    for b in range(bsz):
        for h in range(H):
            g = h // (H // G)
            a = math.exp(dt[b, h] * A[h])
            for p in range(P):
                acc = 0.0
                for n in range(N):
                    s_new = a * state[b, h, p, n] + dt[b, h] * x[b, h, p] * B[b, g, n]
                    assert abs(new[b, h, p, n] - s_new) <= 1e-13 * max(1.0, abs(s_new))
                    acc += s_new * C[b, g, n]
                want = acc + D[h] * x[b, h, p]
                assert abs(y[b, h, p] - want) <= 1e-12 * max(1.0, abs(want))


def test_step_dt_zero_and_no_skip(oracle):
    """dt = 0 leaves the state and reads it out; D = None drops the skip term."""
    rng = np.random.default_rng(23)
    state = rng.standard_normal((1, 2, 3, 4))
    x = rng.standard_normal((1, 2, 3))
    B = rng.standard_normal((1, 1, 4))
    C = rng.standard_normal((1, 1, 4))
    D = np.array([0.5, -2.0])
    y, new = oracle.ssd_step(state, x, np.zeros((1, 2)), np.array([-1.0, -3.0]), B, C, D=D)
    assert np.array_equal(new, state)
    np.testing.assert_allclose(y, np.einsum("bhpn,n->bhp", state, C[0, 0]) + D[None, :, None] * x,
                               rtol=1e-14, atol=1e-14)
    y0, _ = oracle.ssd_step(state, x, np.zeros((1, 2)), np.array([-1.0, -3.0]), B, C)
    np.testing.assert_allclose(y0, np.einsum("bhpn,n->bhp", state, C[0, 0]), rtol=1e-14, atol=1e-14)


def _step_variant(kind, state, x, dt, A, B, C, D):
    """A numpy step with one plausible mistake planted (or none: 'correct')."""
    H, G = x.shape[1], B.shape[1]
    group = np.arange(H) // (H // G)
    if kind == "group_modulo":          # head h -> group h % G instead of h // (H/G)
        group = np.arange(H) % G
    Bh, Ch = B[:, group, :], C[:, group, :]
    decay = np.exp(dt * A[None, :])
    if kind == "decay_without_dt":
        decay = np.exp(np.broadcast_to(A[None, :], dt.shape))
    inp = dt[:, :, None] * x
    if kind == "no_dt_input":
        inp = x
    new = decay[:, :, None, None] * state + inp[:, :, :, None] * Bh[:, :, None, :]
    read = state if kind == "read_before_update" else new
    y = np.einsum("bhpn,bhn->bhp", read, Ch) + D[None, :, None] * x
    return y, new


def test_step_pins_reject_planted_mistakes(oracle):
    """The steps-equal-recurrence pin fails for each planted mistake and holds
    for the unmutated step (and for the oracle's own)."""
    inp = small(seed=24, T=9, H=4, G=2)
    y_ref, fin_ref = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    args64 = [np.asarray(a, np.float64) for a in (inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.h0)]
    x, dt, A, B, C, D, h0 = args64

    def run(kind):
        state, ys = h0, []
        for t in range(x.shape[1]):
            y_t, state = _step_variant(kind, state, x[:, t], dt[:, t], A, B[:, t], C[:, t], D)
            ys.append(y_t)
        return np.stack(ys, axis=1), state

    y, fin = run("correct")
    assert rel_err(y, y_ref) < 1e-12 and rel_err(fin, fin_ref) < 1e-12
    for kind in ("group_modulo", "decay_without_dt", "no_dt_input", "read_before_update"):
        yv, fv = run(kind)
        assert rel_err(yv, y_ref) > 1e-3, kind
