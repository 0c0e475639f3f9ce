"""Pins of the gated state scan oracle ("Mamba 2 Gated State Scan" exercise page:
S_t = gamma_t S_{t-1} + k_t v_t^T, y_t = q_t^T S_t, each batch state starting at zero,
the output reading the updated state).  CPU only."""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _cases(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases("gated_state_scan_page_examples.json"), ids=lambda c: c["name"])
def test_page_examples(orc, case):
    """The page's printed examples, exactly."""
    out = orc.gated_scan(np.array(case["q"], float), np.array(case["k"], float), np.array(case["v"], float),
                         np.array(case["gamma"], float))
    np.testing.assert_array_equal(out["outputs"], np.array(case["outputs"], float))
    np.testing.assert_array_equal(out["final_state"], np.array(case["final_state"], float))


@pytest.mark.parametrize("case", _cases("gated_state_scan_cases.json"), ids=lambda c: c["name"])
def test_hand_worked_cases(orc, case):
    """Cases worked by hand from the two equations (gamma = 0 where the case resets)."""
    gamma = np.where(np.array(case["reset"]) == 1, 0.0, np.array(case["gamma"], float))
    out = orc.gated_scan(np.array(case["q"], float)[None], np.array(case["k"], float)[None],
                         np.array(case["v"], float)[None], gamma[None])
    np.testing.assert_allclose(out["outputs"][0], np.array(case["outputs"], float), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["final_state"][0], np.array(case["final_state"], float), rtol=1e-12, atol=1e-12)


def _rand(seed, B=2, S=7, dk=3, dv=2):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, S, dk)), g.standard_normal((B, S, dk)), g.standard_normal((B, S, dv)),
            g.uniform(0.0, 1.0, (B, S)), g.standard_normal((B, dk, dv)))


def test_unrolled_sum_brute_force(orc):
    """S_t = prod_{r<=t} gamma_r h0 + sum_{j<=t} (prod_{j<r<=t} gamma_r) k_j v_j^T."""
    q, k, v, gam, h0 = _rand(1)
    out = orc.gated_scan(q, k, v, gam, h0)
    B, S, dk = q.shape
    for b in range(B):
        for t in range(S):
            St = np.prod(gam[b, :t + 1]) * h0[b]
            for j in range(t + 1):
                St = St + np.prod(gam[b, j + 1:t + 1]) * np.outer(k[b, j], v[b, j])
            np.testing.assert_allclose(out["outputs"][b, t], q[b, t] @ St, rtol=1e-12, atol=1e-12)
            if t == S - 1:
                np.testing.assert_allclose(out["final_state"][b], St, rtol=1e-12, atol=1e-12)


def test_unit_gate_is_a_prefix_sum(orc):
    q, k, v, _, _ = _rand(2, S=9)
    gam = np.ones(q.shape[:2])
    out = orc.gated_scan(q, k, v, gam)
    S_t = np.cumsum(np.einsum("bti,btj->btij", k, v), axis=1)
    np.testing.assert_allclose(out["outputs"], np.einsum("bti,btij->btj", q, S_t), rtol=1e-12, atol=1e-12)


def test_zero_gate_reads_only_the_current_token(orc):
    q, k, v, _, h0 = _rand(3)
    out = orc.gated_scan(q, k, v, np.zeros(q.shape[:2]), h0)
    np.testing.assert_allclose(out["outputs"], np.einsum("bti,bti->bt", q, k)[..., None] * v, rtol=1e-12)


def test_chaining_through_final_state(orc):
    q, k, v, gam, _ = _rand(4, S=12)
    full = orc.gated_scan(q, k, v, gam)
    a = orc.gated_scan(q[:, :5], k[:, :5], v[:, :5], gam[:, :5])
    b = orc.gated_scan(q[:, 5:], k[:, 5:], v[:, 5:], gam[:, 5:], a["final_state"])
    np.testing.assert_allclose(np.concatenate([a["outputs"], b["outputs"]], 1), full["outputs"], rtol=1e-12)
    np.testing.assert_allclose(b["final_state"], full["final_state"], rtol=1e-12)


def test_agrees_with_the_s6_oracle_reduction(orc):
    """The S6 token loop with B = k, C = q, one channel per value column, A = -1 and a
    shared step g_t = -ln gamma_t (so exp(A g) = gamma) and x = v / g computes the same
    recurrence: an independent second path through different code."""
    q, k, v, gam, _ = _rand(5, B=1, S=10, dk=4, dv=3)
    gam = np.clip(gam, 0.05, 0.95)
    g = -np.log(gam[0])
    dv, S = v.shape[2], v.shape[1]
    out6 = orc.scan(x=(v[0].T / g[None, :])[None], dt=np.broadcast_to(g[None, None, :], (1, dv, S)).copy(),
                    A=np.full((dv, q.shape[2]), -1.0), B=k[0].T[None], C=q[0].T[None], dt_softplus=False)
    out = orc.gated_scan(q, k, v, gam)
    np.testing.assert_allclose(out6["y"][0].T, out["outputs"][0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out6["h_last"][0].T, out["final_state"][0], rtol=1e-10, atol=1e-12)
