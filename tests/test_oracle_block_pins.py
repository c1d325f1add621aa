"""Pins for the oracle's block neighbours of the scan (CPU only).

The Mamba-2 block applies softplus to dt before the SSD call, gates the SSD
output with silu of the z branch and normalises each token's H * P outputs with
RMSNorm (aifetchly blog "Mamba-2 Architecture: State Space Duality Explained",
"Step 2: Full Mamba-2 Block with Gated Projections"; akillness.github.io "State
Space Duality and Mamba-2", the block diagram).  Each oracle function is pinned
to identities that its definition fixes, not to a restatement of its formula:

* softplus: e^softplus(v) - 1 = e^v (the definition inverted), softplus(0) =
  ln 2, softplus(v) - softplus(-v) = v (also for |v| = 60, where a naive
  log(1 + e^v) overflows);
* silu gate: g(y, 0) = 0 and g(y, z) - g(y, -z) = y z (silu(z) - silu(-z) = z);
* RMSNorm over H * P: with weight 1 and eps 0, every token's output has mean
  square 1, is unchanged when the token's inputs are scaled, and keeps the
  ratios between ALL its H * P values (one factor per token, not per head);
  rstd * sqrt(mean(g^2) + eps) = 1;
* the composition with everything off is the recurrence itself.
A planted-mistake test shows these pins reject a sigmoid gate, a per-head norm
and a softplus without its bias.
"""
import math

import numpy as np
import pytest

from structured_state_space_mamba_b200.inputs import make_inputs


def test_softplus_identities(oracle):
    v = np.linspace(-8.0, 8.0, 33).reshape(1, 33, 1)
    sp = oracle.dt_transform(v, softplus=True)
    np.testing.assert_allclose(np.expm1(sp), np.exp(v), rtol=1e-13)
    assert abs(oracle.dt_transform(np.zeros((1, 1, 1)), softplus=True)[0, 0, 0] - math.log(2.0)) < 1e-15
    big = np.array([-60.0, -30.0, 0.5, 30.0, 60.0]).reshape(1, 5, 1)
    d = oracle.dt_transform(big, softplus=True) - oracle.dt_transform(-big, softplus=True)
    np.testing.assert_allclose(d, big, rtol=1e-14, atol=1e-14)
    assert np.all(oracle.dt_transform(big, softplus=True) > 0)


def test_dt_bias_adds_per_head(oracle):
    rng = np.random.default_rng(1)
    dt = rng.uniform(-2, 2, size=(2, 5, 3))
    bias = np.array([0.5, -1.0, 2.0])
    got = oracle.dt_transform(dt, bias)
    for h in range(3):
        np.testing.assert_array_equal(got[:, :, h], dt[:, :, h] + bias[h])
    # the bias enters before the softplus
    sp = oracle.dt_transform(dt, bias, softplus=True)
    np.testing.assert_allclose(np.expm1(sp), np.exp(got), rtol=1e-13)


def test_silu_gate_identities(oracle):
    rng = np.random.default_rng(2)
    y = rng.standard_normal((1, 4, 3, 5))
    z = rng.standard_normal((1, 4, 3, 5)) * 3
    g0, r0 = oracle.gated_rmsnorm(y, np.zeros_like(z))
    assert r0 is None and np.all(g0 == 0)
    gp, _ = oracle.gated_rmsnorm(y, z)
    gm, _ = oracle.gated_rmsnorm(y, -z)
    np.testing.assert_allclose(gp - gm, y * z, rtol=1e-13, atol=1e-14)
    # no gate: y passes through
    g, _ = oracle.gated_rmsnorm(y)
    np.testing.assert_array_equal(g, y)


def test_rmsnorm_is_one_factor_per_token(oracle):
    rng = np.random.default_rng(3)
    B, T, H, P = 2, 6, 4, 8
    y = rng.standard_normal((B, T, H, P))
    y[:, :, 0] *= 10.0  # heads on different scales inside one token
    w1 = np.ones(H * P)
    out, rstd = oracle.gated_rmsnorm(y, None, w1, eps=0.0)
    flat = out.reshape(B, T, H * P)
    np.testing.assert_allclose(np.mean(flat * flat, axis=-1), 1.0, rtol=1e-13)
    # ratios between all H*P values of a token are kept (one factor per token)
    np.testing.assert_allclose(flat / y.reshape(B, T, H * P),
                               np.broadcast_to(rstd[..., None], flat.shape), rtol=1e-13)
    # scaling a token's inputs leaves its output unchanged
    out2, _ = oracle.gated_rmsnorm(3.5 * y, None, w1, eps=0.0)
    np.testing.assert_allclose(out2, out, rtol=1e-13)
    # eps enters as mean(g^2) + eps
    _, r = oracle.gated_rmsnorm(y, None, w1, eps=0.25)
    np.testing.assert_allclose(r * np.sqrt(np.mean(y.reshape(B, T, -1) ** 2, axis=-1) + 0.25), 1.0,
                               rtol=1e-13)
    # the weight multiplies element by element
    w = rng.standard_normal(H * P)
    outw, _ = oracle.gated_rmsnorm(y, None, w, eps=0.0)
    np.testing.assert_allclose(outw.reshape(B, T, -1), flat * w, rtol=1e-13, atol=1e-15)


def test_block_with_everything_off_is_the_recurrence(oracle):
    inp = make_inputs(1, 32, 4, 8, 6, 2, 32, dtype="f32", seed=4, init_state=True)
    out, fin, rstd = oracle.ssd_block(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    y, f = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    np.testing.assert_array_equal(out, y)
    np.testing.assert_array_equal(fin, f)
    assert rstd is None


def _sigmoid_gate(y, z):
    return y / (1.0 + np.exp(-z))


def _per_head_norm(g, w, eps):
    ms = np.mean(g * g, axis=-1, keepdims=True)
    return g / np.sqrt(ms + eps) * w.reshape(g.shape[2], g.shape[3])


def test_block_pins_reject_planted_mistakes(oracle):
    rng = np.random.default_rng(5)
    y = rng.standard_normal((1, 4, 3, 5))
    y[:, :, 0] *= 10.0
    z = rng.standard_normal((1, 4, 3, 5)) * 3
    # a sigmoid gate breaks g(y, z) - g(y, -z) = y z
    d = _sigmoid_gate(y, z) - _sigmoid_gate(y, -z)
    assert np.max(np.abs(d - y * z)) > 1e-2
    # a per-head norm breaks "one factor per token"
    out = _per_head_norm(y, np.ones(15), 0.0).reshape(1, 4, 15)
    ratio = out / y.reshape(1, 4, 15)
    assert np.max(np.abs(ratio - ratio[..., :1])) > 1e-2
    # a softplus that drops the bias breaks e^sp - 1 = e^(dt + bias)
    dt = rng.uniform(-2, 2, size=(1, 5, 3))
    bias = np.array([0.5, -1.0, 2.0])
    wrong = oracle.dt_transform(dt, None, softplus=True)
    assert np.max(np.abs(np.expm1(wrong) - np.exp(dt + bias))) > 1e-2
