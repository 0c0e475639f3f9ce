"""Pins of the causal depthwise conv + SiLU oracle (TransformerLens docs, ssm_mixer: the
scan's x is SiLU of the conv1d output; a decode step carries the conv's input state).
CPU only."""
import numpy as np
import pytest


def _silu(v):
    return v / (1.0 + np.exp(-v))


def _rand(seed, b=2, c=3, L=11, K=4, state=True):
    g = np.random.default_rng(seed)
    return (g.standard_normal((b, c, L)), g.standard_normal((c, K)), g.standard_normal(c),
            g.standard_normal((b, c, K - 1)) if state else None)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("with_state", [False, True])
def test_matches_numpy_correlate(orc, K, with_state):
    """x = silu(b + correlate(state ++ u, w, 'valid')): numpy's routine, row by row."""
    u, w, cb, st = _rand(10 + K, K=K, state=with_state and K > 1)
    out = orc.conv_silu(u, w, cb, st)
    for bi in range(u.shape[0]):
        for c in range(u.shape[1]):
            pre = st[bi, c] if st is not None else np.zeros(K - 1)
            full = np.concatenate([pre, u[bi, c]])
            ref = _silu(cb[c] + np.correlate(full, w[c], mode="valid"))
            np.testing.assert_allclose(out["x"][bi, c], ref, rtol=1e-13, atol=1e-14)
            np.testing.assert_array_equal(out["state"][bi, c], full[len(full) - (K - 1):] if K > 1 else [])


def test_identity_and_delay_taps(orc):
    u, _, cb, _ = _rand(20, state=False)
    ident = np.zeros((3, 4)); ident[:, 3] = 1.0
    np.testing.assert_allclose(orc.conv_silu(u, ident, cb)["x"], _silu(u + cb[None, :, None]), rtol=1e-14)
    delay = np.zeros((3, 4)); delay[:, 0] = 1.0
    x = orc.conv_silu(u, delay, cb)["x"]
    np.testing.assert_allclose(x[:, :, 3:], _silu(u[:, :, :-3] + cb[None, :, None]), rtol=1e-14)
    np.testing.assert_allclose(x[:, :, :3], _silu(np.zeros_like(u[:, :, :3]) + cb[None, :, None]), rtol=1e-14)


def test_causal(orc):
    u, w, cb, st = _rand(21)
    a = orc.conv_silu(u, w, cb, st)["x"]
    u2 = u.copy(); u2[:, :, 7] += 5.0
    b = orc.conv_silu(u2, w, cb, st)["x"]
    np.testing.assert_array_equal(a[:, :, :7], b[:, :, :7])
    assert np.all(np.abs(a[:, :, 7] - b[:, :, 7]) > 0)


@pytest.mark.parametrize("split", [1, 2, 5])
def test_chaining_through_the_state(orc, split):
    """conv over u equals conv over u[:split] then u[split:] from the returned state,
    including a first part shorter than the state."""
    u, w, cb, st = _rand(22, L=9)
    full = orc.conv_silu(u, w, cb, st)
    a = orc.conv_silu(u[:, :, :split], w, cb, st)
    b = orc.conv_silu(u[:, :, split:], w, cb, a["state"])
    np.testing.assert_array_equal(np.concatenate([a["x"], b["x"]], 2), full["x"])
    np.testing.assert_array_equal(b["state"], full["state"])
