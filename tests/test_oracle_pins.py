"""Pins for the float64 oracle against what the pages and the mathematics fix.

Each test ties the oracle to something other than itself: the unrolled closed
forms of the TransformerLens "ssm_mixer" page, the associative formulation of the
"s6_reset" blog draft (an independent ordering), segment isolation under resets,
hand-worked cases of the gated state scan, closed-form special cases and
invariants.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

from selective_state_space_18_b200.inputs import make_scan_inputs, make_update_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return None if t is None else t.double().numpy()


def _softplus(r):
    return np.logaddexp(0.0, r)


def _small(seed, b=2, c=3, n=4, L=12, **kw):
    return make_scan_inputs(b, c, n, L, "f32", seed=seed, **kw)


def _rel(a, b):
    return float(np.max(np.abs(a - b) / (1.0 + np.abs(b))))


# --------------------------------------------------------------------------------------
# 1. Closed forms of the TransformerLens "ssm_mixer" page
# --------------------------------------------------------------------------------------

def _effective_attention(dt, A, B, C):
    """M[b,c,i,j] = sum_n C[i,n] * prod_{k=j+1..i} exp(A[c,n] dt[c,k]) * B[j,n] (j <= i),
    built by brute force from the compute_effective_attention formula."""
    bt, ch, L = dt.shape
    n = A.shape[1]
    M = np.zeros((bt, ch, L, L))
    for b in range(bt):
        for c in range(ch):
            for i in range(L):
                for j in range(i + 1):
                    total = 0.0
                    for s in range(n):
                        prod = 1.0
                        for k in range(j + 1, i + 1):
                            prod *= math.exp(A[c, s] * dt[b, c, k])
                        total += C[b, s, i] * prod * B[b, s, j]
                    M[b, c, i, j] = total
    return M


@pytest.mark.parametrize("seed", [1, 2])
def test_effective_attention_reconstructs_y(orc, seed):
    """y[c,i] = sum_j M[c,i,j] dt[c,j] x[c,j] + D[c] x[c,i] (compute_effective_attention,
    include_dt_scaling), against the token loop with no gate."""
    inp = _small(seed, z=False)
    dt = _softplus(_np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None])
    x, A, B, C, D = (_np(inp[k]) for k in ("x", "A", "B", "C", "D"))
    M = _effective_attention(dt, A, B, C)
    y_ref = np.einsum("bcij,bcj->bci", M, dt * x) + D[None, :, None] * x
    out = orc.scan(**inp)
    assert _rel(out["y"], y_ref) < 1e-12


def test_unrolled_state_matches_every_token(orc):
    """S_t[c,s] = sum_{j<=t} prod_{k=j+1..t} exp(A[c,s] dt_k) * dt_j x_j B_j[s]
    (compute_ssm_state), checked at every token and at the final state; the page's
    own check y_t = sum_s C_t[s] S_t[c,s] + D x_t holds too."""
    inp = _small(3, z=False)
    dt = _softplus(_np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None])
    x, A, B, C, D = (_np(inp[k]) for k in ("x", "A", "B", "C", "D"))
    bt, ch, L = x.shape
    n = A.shape[1]
    S = np.zeros((bt, ch, L, n))
    for b in range(bt):
        for c in range(ch):
            for s in range(n):
                for t in range(L):
                    acc = 0.0
                    for j in range(t + 1):
                        decay = math.exp(A[c, s] * dt[b, c, j + 1:t + 1].sum())
                        acc += decay * dt[b, c, j] * x[b, c, j] * B[b, s, j]
                    S[b, c, t, s] = acc
    out = orc.scan(**inp, return_states=True)
    assert _rel(out["h_all"], S) < 1e-12
    assert _rel(out["h_last"], S[:, :, -1, :]) < 1e-12
    y_from_S = np.einsum("bst,bcts->bct", C, S) + D[None, :, None] * x
    assert _rel(out["y"], y_from_S) < 1e-12


# --------------------------------------------------------------------------------------
# 2. Two orderings ("s6_reset": sequential lax.scan vs associative_scan)
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("resets", [False, True])
@pytest.mark.parametrize("with_h0", [False, True])
@pytest.mark.parametrize("softplus", [True, False])
def test_tree_scan_equals_token_loop(orc, resets, with_h0, softplus):
    inp = make_scan_inputs(2, 5, 8, 37, "f32", seed=11, h0=with_h0,
                           reset_mean_doc=6 if resets else 0)
    if not softplus:  # keep the step positive without the softplus
        inp["dt"] = inp["dt"].abs() * 0.3
        inp["dt_bias"] = inp["dt_bias"].abs() * 0.1
    seq = orc.scan(**inp, dt_softplus=softplus)
    tree = orc.tree_scan(**inp, dt_softplus=softplus)
    assert _rel(tree["y"], seq["y"]) < 1e-12
    assert _rel(tree["h_last"], seq["h_last"]) < 1e-12


# --------------------------------------------------------------------------------------
# 3. Enforced boundary resets ("s6_reset", Enforced Boundary Resetting)
# --------------------------------------------------------------------------------------

def test_reset_equals_each_document_alone(orc):
    """In a packed row, each document's outputs equal the scan of that document
    alone from zeros -- bit for bit in the token loop."""
    inp = make_scan_inputs(2, 4, 4, 200, "f32", seed=21, reset_mean_doc=23, h0=True)
    packed = orc.scan(**inp)
    mask = inp["reset"].numpy()
    for b in range(2):
        starts = list(np.flatnonzero(mask[b])) + [mask.shape[1]]
        assert starts[0] == 0 and len(starts) > 3
        for s0, s1 in zip(starts[:-1], starts[1:]):
            alone = {k: (None if v is None else v) for k, v in inp.items()}
            alone["x"] = inp["x"][b:b + 1, :, s0:s1]
            alone["dt"] = inp["dt"][b:b + 1, :, s0:s1]
            alone["z"] = inp["z"][b:b + 1, :, s0:s1]
            alone["B"] = inp["B"][b:b + 1, :, s0:s1]
            alone["C"] = inp["C"][b:b + 1, :, s0:s1]
            alone["reset"] = None
            alone["h0"] = None
            ref = orc.scan(**alone)
            np.testing.assert_array_equal(packed["y"][b, :, s0:s1], ref["y"][0])
            if s1 == mask.shape[1]:
                np.testing.assert_array_equal(packed["h_last"][b], ref["h_last"][0])


def test_reset_at_first_token_discards_h0(orc):
    inp = make_scan_inputs(1, 3, 4, 9, "f32", seed=22, h0=True)
    inp["reset"] = np.zeros((1, 9), np.uint8)
    inp["reset"][0, 0] = 1
    with_h0 = orc.scan(**inp)
    inp["h0"] = None
    without = orc.scan(**inp)
    np.testing.assert_array_equal(with_h0["y"], without["y"])


def _naive_reset_op(ei, ej):
    """The naive reset operator the blog draft shows to break associativity."""
    ai, bi, ri = ei
    aj, bj, rj = ej
    if ri:
        return (aj, bj, rj)
    if rj:
        return (0.0, 0.0, rj)
    return (ai * aj, aj * bi + bj, False)


def _flag_op(ei, ej):
    """Affine maps h -> (r ? u : a h + u), composed left then right."""
    ai, ui, ri = ei
    aj, uj, rj = ej
    if rj:
        return (aj, uj, True)
    if ri:
        return (1.0, aj * ui + uj, True)
    return (ai * aj, aj * ui + uj, False)


def _apply(e, h):
    a, u, r = e
    return u if r else a * h + u


def test_naive_reset_operator_is_not_associative():
    """The [X, r, Y] counterexample: left and right association disagree."""
    X = (0.5, 2.0, False)
    r = (0.7, 3.0, True)
    Y = (0.25, 5.0, False)
    left = _naive_reset_op(_naive_reset_op(X, r), Y)
    right = _naive_reset_op(X, _naive_reset_op(r, Y))
    assert left != right


def test_flag_operator_is_associative_and_matches_zeroed_decay():
    """The resettable operator is associative for all 8 flag patterns, and applying
    a composite equals the token loop with the decay set to 0 at reset tokens."""
    rng = np.random.default_rng(5)
    for flags in range(8):
        for _ in range(50):
            es = [(rng.uniform(0, 1), rng.normal(), bool(flags >> i & 1)) for i in range(3)]
            l = _flag_op(_flag_op(es[0], es[1]), es[2])
            r = _flag_op(es[0], _flag_op(es[1], es[2]))
            h = rng.normal()
            assert abs(_apply(l, h) - _apply(r, h)) < 1e-12
            hs = h
            for a, u, rr in es:
                hs = (0.0 if rr else a) * hs + u
            assert abs(_apply(l, h) - hs) < 1e-12


# --------------------------------------------------------------------------------------
# 4-5. Decode step and chaining (nnterp: the state after the call's last token is
#      what the next decode step starts from)
# --------------------------------------------------------------------------------------

def test_decode_equals_last_scan_step(orc):
    inp = make_scan_inputs(2, 6, 8, 17, "f32", seed=31, h0=True)
    full = orc.scan(**inp)
    head = dict(inp)
    for k in ("x", "dt", "z", "B", "C"):
        head[k] = inp[k][:, :, :-1]
    first = orc.scan(**head)
    step = orc.update(first["h_last"], inp["x"][:, :, -1], inp["dt"][:, :, -1], inp["A"],
                      inp["B"][:, :, -1], inp["C"][:, :, -1], inp["D"], inp["z"][:, :, -1],
                      inp["dt_bias"])
    np.testing.assert_allclose(step["y"], full["y"][:, :, -1], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(step["state"], full["h_last"], rtol=1e-15, atol=1e-15)


def test_chaining_through_h0(orc):
    inp = make_scan_inputs(2, 5, 4, 40, "f32", seed=41)
    full = orc.scan(**inp)
    a, b = dict(inp), dict(inp)
    for k in ("x", "dt", "z", "B", "C"):
        a[k] = inp[k][:, :, :25]
        b[k] = inp[k][:, :, 25:]
    ra = orc.scan(**a)
    b["h0"] = ra["h_last"]
    rb = orc.scan(**b)
    np.testing.assert_array_equal(np.concatenate([ra["y"], rb["y"]], axis=2), full["y"])
    np.testing.assert_array_equal(rb["h_last"], full["h_last"])


# --------------------------------------------------------------------------------------
# 6. Closed-form special cases
# --------------------------------------------------------------------------------------

def _one(dt_raw, *, bias=None, x=3.0, B=2.0, C=0.5, D=1.0, z=None, A=-1.0, softplus=True):
    arr = lambda v: np.array(v, dtype=np.float64)
    return dict(x=arr([[[x]]]), dt=arr([[[dt_raw]]]), A=arr([[A]]), B=arr([[[B]]]),
                C=arr([[[C]]]), D=arr([D]), z=None if z is None else arr([[[z]]]),
                dt_bias=None if bias is None else arr([bias])), softplus


def test_single_token_closed_form(orc):
    """L = 1, N = 1 from zeros: y = C * dt * B * x + D * x.  With dt_raw + bias = 0
    the step is softplus(0) = ln 2, so y = 0.5 * ln2 * 2 * 3 + 3 = 3 ln 2 + 3."""
    kw, sp = _one(0.5, bias=-0.5)
    out = orc.scan(**kw, dt_softplus=sp)
    assert out["y"][0, 0, 0] == pytest.approx(3 * math.log(2) + 3, rel=1e-15)
    assert out["h_last"][0, 0, 0] == pytest.approx(math.log(2) * 6, rel=1e-15)


def test_single_token_gate(orc):
    """With z = ln 3, sigmoid(z) = 3/4, so the gate multiplies the pre-gate output
    (3 ln 2 + 3) by (3/4) ln 3; z = 0 gives exactly 0."""
    kw, sp = _one(0.5, bias=-0.5, z=math.log(3.0))
    out = orc.scan(**kw, dt_softplus=sp)
    assert out["y"][0, 0, 0] == pytest.approx((3 * math.log(2) + 3) * 0.75 * math.log(3), rel=1e-14)
    kw, sp = _one(0.5, bias=-0.5, z=0.0)
    assert orc.scan(**kw, dt_softplus=sp)["y"][0, 0, 0] == 0.0


def test_softplus_values(orc):
    """With A = 0, B = C = x = 1, D = 0 the output is the step itself.  softplus(0) =
    ln 2, and softplus(r) - softplus(-r) = r for every r (also far in the tails)."""
    def step(r):
        kw, sp = _one(r, x=1.0, B=1.0, C=1.0, D=0.0, A=0.0)
        return orc.scan(**kw, dt_softplus=sp)["y"][0, 0, 0]
    assert step(0.0) == pytest.approx(math.log(2), rel=1e-15)
    for r in (0.3, 2.0, 17.0, 40.0, 300.0):
        assert step(r) - step(-r) == pytest.approx(r, rel=1e-15, abs=1e-300)
    assert step(-40.0) == pytest.approx(math.exp(-40.0), rel=1e-12)
    kw, sp = _one(0.25, x=1.0, B=1.0, C=1.0, D=0.0, A=0.0, softplus=False)
    assert orc.scan(**kw, dt_softplus=False)["y"][0, 0, 0] == 0.25


def test_silu_identity(orc):
    """silu(v) - silu(-v) = v: with C = 0, D = x = 1 the output is silu(z)."""
    for v in (0.5, 1.7, 6.0, 30.0):
        ys = []
        for zz in (v, -v):
            kw, sp = _one(0.1, x=1.0, C=0.0, D=1.0, z=zz)
            ys.append(orc.scan(**kw, dt_softplus=sp)["y"][0, 0, 0])
        assert ys[0] - ys[1] == pytest.approx(v, rel=1e-14)


def test_zero_decay_rate_is_prefix_sum(orc):
    """A = 0: h_t = sum_{j<=t} dt_j B_j x_j (no decay), so y is a cumulative sum."""
    inp = _small(51, z=False, D=False)
    inp["A"] = inp["A"] * 0.0
    dt = _softplus(_np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None])
    x, B, C = _np(inp["x"]), _np(inp["B"]), _np(inp["C"])
    h = np.cumsum(dt[:, :, :, None] * x[:, :, :, None] * np.transpose(B, (0, 2, 1))[:, None], axis=2)
    y_ref = np.einsum("bcts,bst->bct", h, C)
    out = orc.scan(**inp)
    assert _rel(out["y"], y_ref) < 1e-12


def test_fast_decay_forgets(orc):
    """Very negative dt*A: the decay underflows to 0, so h_t = dt_t B_t x_t."""
    inp = _small(52, z=False)
    inp["A"] = inp["A"] * 1e4
    inp["dt"] = inp["dt"].abs() + 1.0
    dt = _softplus(_np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None])
    x, B, C, D = (_np(inp[k]) for k in ("x", "B", "C", "D"))
    y_ref = np.einsum("bst,bct->bct", B * C, dt * x) + D[None, :, None] * x
    assert _rel(orc.scan(**inp)["y"], y_ref) < 1e-13


def test_dt_bias_enters_before_softplus(orc):
    inp = _small(53)
    shifted = dict(inp)
    shifted["dt"] = _np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None]
    shifted["dt_bias"] = None
    np.testing.assert_array_equal(orc.scan(**inp)["y"], orc.scan(**shifted)["y"])


# --------------------------------------------------------------------------------------
# 7. Mamba-2 gated state scan as a special case (hand-worked golden cases)
# --------------------------------------------------------------------------------------

def _golden_cases():
    with open(os.path.join(GOLDEN, "gated_state_scan_cases.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_gated_state_scan_reduction(orc, case):
    """S6 with D = 0, no gate, no softplus, B = k, C = q, one channel per value
    column and a step g_t shared by all channels is S_t = gamma_t S_{t-1} + k_t v_t^T
    with gamma_t = exp(A g_t) and v_t = g_t x_t:
      gamma in (0,1): A = -1, g = -ln gamma;  gamma = 1: A = 0, g = 1;
      gamma = 0: the reset flag (g = 1)."""
    q = np.array(case["q"], float)
    k = np.array(case["k"], float)
    v = np.array(case["v"], float)
    gamma = np.array(case["gamma"], float)
    reset = np.array(case["reset"], np.uint8)
    S, dk = q.shape
    dv = v.shape[1]
    unit = bool(np.all(gamma == 1.0))
    g = np.where((gamma > 0) & (gamma < 1), -np.log(np.where(gamma > 0, gamma, 1.0)), 1.0)
    A = np.full((dv, dk), 0.0 if unit else -1.0)
    dt = np.broadcast_to(g[None, None, :], (1, dv, S)).copy()
    x = (v.T / g[None, :])[None]
    out = orc.scan(x=x, dt=dt, A=A, B=k.T[None], C=q.T[None], reset=reset[None],
                   dt_softplus=False)
    np.testing.assert_allclose(out["y"][0].T, np.array(case["outputs"], float), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["h_last"][0].T, np.array(case["final_state"], float),
                               rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------------------
# 8. Invariants
# --------------------------------------------------------------------------------------

def test_linear_in_x(orc):
    a = _small(61, z=False)
    b = _small(62, z=False)
    mix = dict(a)
    mix["x"] = 2.0 * _np(a["x"]) - 3.0 * _np(b["x"])
    ya = orc.scan(**a)["y"]
    b_same_dt = dict(a)
    b_same_dt["x"] = b["x"]
    yb = orc.scan(**b_same_dt)["y"]
    assert _rel(orc.scan(**mix)["y"], 2.0 * ya - 3.0 * yb) < 1e-12


def test_channel_permutation_equivariance(orc):
    inp = _small(63, c=6, h0=True)
    perm = np.array([3, 0, 5, 1, 4, 2])
    p = dict(inp)
    for k in ("x", "dt", "z"):
        p[k] = _np(inp[k])[:, perm]
    for k in ("A", "D", "dt_bias"):
        p[k] = _np(inp[k])[perm]
    p["h0"] = _np(inp["h0"])[:, perm]
    ref = orc.scan(**inp)
    out = orc.scan(**p)
    np.testing.assert_array_equal(out["y"], ref["y"][:, perm])
    np.testing.assert_array_equal(out["h_last"], ref["h_last"][:, perm])


def test_batch_items_independent(orc):
    inp = make_scan_inputs(3, 4, 4, 20, "f32", seed=64, reset_mean_doc=7, h0=True)
    full = orc.scan(**inp)
    for b in range(3):
        one = {k: (None if v is None else v[b:b + 1]) if k not in ("A", "D", "dt_bias") else v
               for k, v in inp.items()}
        out = orc.scan(**one)
        np.testing.assert_array_equal(out["y"][0], full["y"][b])
        np.testing.assert_array_equal(out["h_last"][0], full["h_last"][b])


def test_decode_update_batch_independent_and_copy(orc):
    inp = make_update_inputs(3, 5, 8, "f32", seed=65)
    before = inp["state"].clone()
    full = orc.update(**inp)
    assert np.array_equal(inp["state"].numpy(), before.numpy())
    for b in range(3):
        one = {k: (None if v is None else v[b:b + 1]) if k not in ("A", "D", "dt_bias") else v
               for k, v in inp.items()}
        out = orc.update(**one)
        np.testing.assert_array_equal(out["y"][0], full["y"][b])
        np.testing.assert_array_equal(out["state"][0], full["state"][b])


# --------------------------------------------------------------------------------------
# 7. Per-token step sizes ("betas" of the nnterp selective_scan page) and log decays
# --------------------------------------------------------------------------------------

def test_betas_closed_forms(orc):
    """The step size per token and channel: softplus(0) = ln 2 (dt_raw = -bias),
    softplus(r) - softplus(-r) = r, the raw sum when the softplus is off, and the bias
    added per channel before the softplus."""
    arr = lambda v: np.array(v, dtype=np.float64)
    r = arr([0.0, 0.3, -0.3, 2.0, -2.0, 40.0, -40.0])
    L = r.size
    kw = dict(x=np.ones((1, 2, L)), dt=np.stack([r, r])[None] - arr([0.5, -1.25])[None, :, None],
              A=-np.ones((2, 1)), B=np.ones((1, 1, L)), C=np.ones((1, 1, L)), dt_bias=arr([0.5, -1.25]))
    b = orc.scan(**kw, return_betas=True)["betas"]
    for c in range(2):
        assert b[0, c, 0] == pytest.approx(math.log(2), rel=1e-15)
        for i in (1, 3, 5):
            assert b[0, c, i] - b[0, c, i + 1] == pytest.approx(r[i], rel=1e-15)
    raw = orc.scan(**kw, dt_softplus=False, return_betas=True)["betas"]
    np.testing.assert_allclose(raw[0], np.stack([r, r]), rtol=0, atol=1e-15)


def test_betas_are_the_recurrence_steps(orc):
    """With B = 0 the state only decays: h_t = h0 exp(A sum_{s<=t} beta_s), so the
    states after every token follow from the betas and A alone (the log decays beta_t A
    summed); and with A = 0, C = x = 1, D = 0, the output increments by exactly
    beta_t B_t at each token."""
    inp = _small(71, b=2, c=3, n=4, L=20, h0=True)
    inp["B"] = inp["B"] * 0
    out = orc.scan(**inp, return_states=True, return_betas=True)
    betas = out["betas"]
    A = _np(inp["A"])
    want = _np(inp["h0"])[:, :, None, :] * np.exp(A[None, :, None, :] * np.cumsum(betas, axis=2)[..., None])
    assert _rel(out["h_all"], want) < 1e-13
    inp = _small(72, b=1, c=2, n=1, L=16, z=False, D=False)
    inp["A"] = inp["A"] * 0
    inp["C"] = inp["C"] * 0 + 1
    inp["x"] = inp["x"] * 0 + 1
    out = orc.scan(**inp, return_betas=True)
    inc = np.diff(np.concatenate([np.zeros((1, 2, 1)), out["y"]], axis=2), axis=2)
    assert _rel(inc, out["betas"] * _np(inp["B"])[:, 0:1, :]) < 1e-13
    # and they are the softplus of the biased raw steps, token by token, in place
    want = _softplus(_np(inp["dt"]) + _np(inp["dt_bias"])[None, :, None])
    assert _rel(out["betas"], want) < 1e-15
