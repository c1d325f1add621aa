"""Pins for the oracle's reverse mode (CPU only).

`oracle.ssd_recurrent_grad` is the reverse mode of the recurrence written token by
token.  It is pinned to the forward oracle itself through central finite
differences: for L = sum(y * Wy) + sum(final * Wf) with random weights, every
partial derivative of L with respect to every input element (x, dt, A, B, C, D,
h0) is compared with (L(v + e) - L(v - e)) / 2e on small problems in fp64,
including groups (G = 2, H = 4) and a missing D / h0 / dfinal.  A
planted-mistake test shows the pin rejects a decay term dropped from ddt, the
future's gradient not decayed, and dB without dt.
"""
import numpy as np
import pytest

from structured_state_space_mamba_b200.inputs import make_inputs

EPS = 1e-6


def loss(oracle, v, Wy, Wf):
    y, fin = oracle.ssd_recurrent(v["x"], v["dt"], v["A"], v["B"], v["C"], D=v["D"], h0=v["h0"])
    out = float(np.sum(y * Wy))
    if Wf is not None:
        out += float(np.sum(fin * Wf))
    return out


def numeric_grad(oracle, v, name, Wy, Wf):
    base = v[name]
    g = np.zeros_like(base)
    it = np.nditer(base, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        keep = base[i]
        base[i] = keep + EPS
        lp = loss(oracle, v, Wy, Wf)
        base[i] = keep - EPS
        lm = loss(oracle, v, Wy, Wf)
        base[i] = keep
        g[i] = (lp - lm) / (2 * EPS)
    return g


def problem(G, h0, D, seed):
    inp = make_inputs(1, 7, 4, 3, 5, G, 7, dtype="f32", seed=seed, init_state=h0)
    rng = np.random.default_rng(seed + 100)
    v = dict(x=np.array(inp.x, dtype=np.float64), dt=np.array(inp.dt, dtype=np.float64) * 5.0,
             A=np.array(inp.A, dtype=np.float64), B=np.array(inp.B, dtype=np.float64),
             C=np.array(inp.C, dtype=np.float64), D=None if not D else np.array(inp.D, dtype=np.float64),
             h0=None if inp.h0 is None else np.array(inp.h0, dtype=np.float64))
    Wy = rng.standard_normal(v["x"].shape)
    return v, Wy, rng


def analytic(oracle, v, Wy, Wf, grad_fn=None):
    fn = grad_fn or oracle.ssd_recurrent_grad
    return fn(v["x"], v["dt"], v["A"], v["B"], v["C"], Wy, D=v["D"], h0=v["h0"], dfinal=Wf)


@pytest.mark.parametrize("G,h0,D,final", [(1, True, True, True), (2, True, True, False),
                                          (1, False, False, True), (4, False, True, False)])
def test_grad_matches_finite_differences(oracle, G, h0, D, final):
    v, Wy, rng = problem(G, h0, D, seed=7 + G)
    Wf = rng.standard_normal((1, 4, 3, 5)) if final else None
    g = analytic(oracle, v, Wy, Wf)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC"}
    if D:
        names["D"] = "dD"
    if h0:
        names["h0"] = "dh0"
    for name, gname in names.items():
        num = numeric_grad(oracle, v, name, Wy, Wf)
        scale = max(np.max(np.abs(num)), 1e-12)
        assert np.max(np.abs(g[gname] - num)) / scale < 1e-6, (name, np.max(np.abs(g[gname] - num)) / scale)
    if not h0:
        # the gradient of the (zero) initial state is still the state's cotangent
        assert g["dh0"].shape == (1, 4, 3, 5)


def _bad_grad(kind):
    """A copy of the reverse mode with one planted mistake."""
    def fn(x, dt, A, B, C, dy, D=None, h0=None, dfinal=None):
        bsz, T, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        rep = H // G
        Bh, Ch = np.repeat(B, rep, axis=2), np.repeat(C, rep, axis=2)
        h = np.zeros((bsz, H, P, N)) if h0 is None else h0.copy()
        hs = [h]
        for t in range(T):
            a = np.exp(dt[:, t] * A)
            h = a[:, :, None, None] * h + (dt[:, t, :, None, None] * x[:, t, :, :, None]) * Bh[:, t, :, None, :]
            hs.append(h)
        Gn = np.zeros((bsz, H, P, N)) if dfinal is None else dfinal.copy()
        dx, ddt, dA = np.zeros_like(x), np.zeros_like(dt), np.zeros(H)
        dBh, dCh = np.zeros_like(Bh), np.zeros_like(Ch)
        Dv = np.zeros(H) if D is None else D
        for t in range(T - 1, -1, -1):
            Gt = dy[:, t, :, :, None] * Ch[:, t, :, None, :] + Gn
            a = np.exp(dt[:, t] * A)
            GB = np.einsum("bhpn,bhn->bhp", Gt, Bh[:, t])
            dx[:, t] = dt[:, t, :, None] * GB + Dv[None, :, None] * dy[:, t]
            scale_b = 1.0 if kind == "dB_without_dt" else dt[:, t, :, None]
            dBh[:, t] = scale_b * np.einsum("bhpn,bhp->bhn", Gt, x[:, t])
            dCh[:, t] = np.einsum("bhpn,bhp->bhn", hs[t + 1], dy[:, t])
            gh = np.einsum("bhpn,bhpn->bh", Gt, hs[t])
            decay = 0.0 if kind == "no_decay_term" else A[None, :] * a * gh
            ddt[:, t] = np.einsum("bhp,bhp->bh", x[:, t], GB) + decay
            dA += np.sum(dt[:, t] * a * gh, axis=0)
            Gn = Gt if kind == "future_not_decayed" else a[:, :, None, None] * Gt
        return dict(dx=dx, ddt=ddt, dA=dA, dB=dBh.reshape(bsz, T, G, rep, N).sum(3),
                    dC=dCh.reshape(bsz, T, G, rep, N).sum(3), dD=np.einsum("bthp,bthp->h", dy, x), dh0=Gn)
    return fn


@pytest.mark.parametrize("kind,name,gname", [("no_decay_term", "dt", "ddt"),
                                             ("future_not_decayed", "x", "dx"),
                                             ("dB_without_dt", "B", "dB")])
def test_grad_pins_reject_planted_mistakes(oracle, kind, name, gname):
    v, Wy, rng = problem(1, True, True, seed=11)
    Wf = rng.standard_normal((1, 4, 3, 5))
    # the planted copy agrees with the oracle's own reverse mode where it is right...
    good = analytic(oracle, v, Wy, Wf)
    bad = analytic(oracle, v, Wy, Wf, grad_fn=_bad_grad(kind))
    num = numeric_grad(oracle, v, name, Wy, Wf)
    scale = np.max(np.abs(num))
    assert np.max(np.abs(good[gname] - num)) / scale < 1e-6
    # ...and the finite-difference pin catches the mistake
    assert np.max(np.abs(bad[gname] - num)) / scale > 1e-3
