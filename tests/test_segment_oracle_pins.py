"""Pins of the oracle's segment composite and its joining (CPU only).

A sequence cut into segments is joined by the composite each segment applies to the
state that enters it ("s6_reset" draft, Associative Boundary Resetting: the
resettable operator on (decay, increment) pairs, folded over the segment).  These
tests pin ``oracle.segment`` and ``oracle.join_segments`` against what the
mathematics fixes, independently of how the composite is computed:

  * the token-loop scan of the whole sequence (itself pinned in test_oracle_pins);
  * the closed form of the decay product without resets, exp(A * sum_t dt_t);
  * a reset inside the segment: decay exactly 0, state = the scan of the tail that
    starts at the last reset;
  * A = 0 (no decay): decay exactly 1 and the state is a plain sum;
  * a one-token segment: (exp(dt A), dt B x).
"""
import numpy as np
import pytest

from oracle import oracle


def _softplus(r):
    return np.logaddexp(0.0, r)


def _problem(seed, bt=2, ch=3, n=4, L=96, resets=False):
    r = np.random.default_rng(seed)
    p = {
        "x": r.standard_normal((bt, ch, L)),
        "dt": r.standard_normal((bt, ch, L)) - 1.0,
        "A": -(np.arange(1, n + 1)[None, :] * (0.5 + r.random((ch, n)))),
        "B": r.standard_normal((bt, n, L)),
        "C": r.standard_normal((bt, n, L)),
        "D": r.standard_normal(ch),
        "z": r.standard_normal((bt, ch, L)),
        "dt_bias": r.standard_normal(ch) * 0.5,
    }
    if resets:
        m = np.zeros((bt, L), dtype=np.uint8)
        m[0, [0, 17, 40, 41]] = 1
        m[1, [63]] = 1
        p["reset"] = m
    return p


def _cut(p, a, b):
    q = dict(p)
    for k in ("x", "dt", "B", "C", "z"):
        q[k] = p[k][..., a:b]
    if "reset" in p:
        q["reset"] = p["reset"][:, a:b]
    return q


def _segment(q, dt_softplus=True):
    return oracle.segment(q["x"], q["dt"], q["A"], q["B"], q.get("dt_bias"), q.get("reset"),
                          dt_softplus=dt_softplus)


@pytest.mark.parametrize("resets", [False, True])
@pytest.mark.parametrize("cuts", [[0, 96], [0, 40, 96], [0, 1, 17, 18, 63, 96], [0, 30, 60, 90, 96]])
def test_joined_segments_equal_the_whole_scan(resets, cuts):
    p = _problem(3, resets=resets)
    h0 = np.random.default_rng(9).standard_normal((2, 3, 4))
    whole = oracle.scan(**p, h0=h0)
    parts = [_cut(p, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    comps = [_segment(q) for q in parts]
    carries, final = oracle.join_segments([c["decay"] for c in comps], [c["state"] for c in comps], h0)
    scale = 1.0 + np.abs(whole["h_last"]).max()
    assert np.abs(final - whole["h_last"]).max() <= 1e-12 * scale
    # each segment rescanned from the state that enters it gives the whole scan's outputs
    for (a, b), q, carry in zip(zip(cuts[:-1], cuts[1:]), parts, carries):
        seg = oracle.scan(**q, h0=carry)
        ref = whole["y"][..., a:b]
        assert np.abs(seg["y"] - ref).max() <= 1e-12 * (1.0 + np.abs(ref).max())


@pytest.mark.parametrize("dt_softplus", [True, False])
def test_decay_without_resets_is_exp_of_summed_steps(dt_softplus):
    p = _problem(5)
    if not dt_softplus:
        p["dt"] = np.abs(p["dt"]) * 0.1  # keep the steps positive
    comp = _segment(p, dt_softplus)
    r = p["dt"] + p["dt_bias"][None, :, None]
    steps = _softplus(r) if dt_softplus else r
    ref = np.exp(p["A"][None, :, :] * steps.sum(-1)[:, :, None])
    assert np.allclose(comp["decay"], ref, rtol=1e-12, atol=0)


def test_reset_inside_segment_discards_the_entering_state():
    p = _problem(7, resets=True)
    comp = _segment(p)
    # both batch rows hold a reset: the decay is exactly zero
    assert np.all(comp["decay"] == 0.0)
    # the end state is the scan, from zero, of the tail that starts at the last reset
    for b, last in ((0, 41), (1, 63)):
        tail = _cut({k: (v[b:b + 1] if k in ("x", "dt", "B", "C", "z", "reset") else v)
                     for k, v in p.items()}, last, 96)
        ref = oracle.scan(**tail)["h_last"][0]
        assert np.abs(comp["state"][b] - ref).max() <= 1e-12 * (1.0 + np.abs(ref).max())


def test_zero_A_gives_unit_decay_and_a_plain_sum():
    p = _problem(11)
    p["A"] = np.zeros_like(p["A"])
    comp = _segment(p)
    assert np.all(comp["decay"] == 1.0)
    steps = _softplus(p["dt"] + p["dt_bias"][None, :, None])
    ref = np.einsum("bct,bnt->bcn", steps * p["x"], p["B"])
    assert np.abs(comp["state"] - ref).max() <= 1e-12 * (1.0 + np.abs(ref).max())


def test_one_token_segment():
    p = _cut(_problem(13), 5, 6)
    comp = _segment(p)
    d = _softplus(p["dt"][..., 0] + p["dt_bias"][None, :])
    assert np.allclose(comp["decay"], np.exp(d[:, :, None] * p["A"][None]), rtol=1e-14, atol=0)
    ref = d[:, :, None] * p["x"][..., 0][:, :, None] * p["B"][..., 0][:, None, :]
    assert np.allclose(comp["state"], ref, rtol=1e-14, atol=1e-300)


def test_join_order_matters():
    """Joining the same composites in the wrong order gives another state: the join is
    not a sum, so a swapped index would be caught."""
    p = _problem(17)
    parts = [_cut(p, 0, 50), _cut(p, 50, 96)]
    comps = [_segment(q) for q in parts]
    _, right = oracle.join_segments([c["decay"] for c in comps], [c["state"] for c in comps])
    _, wrong = oracle.join_segments([c["decay"] for c in comps[::-1]], [c["state"] for c in comps[::-1]])
    assert np.abs(right - wrong).max() > 1e-3
