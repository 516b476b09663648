"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Nothing here re-types the oracle's own loop: every expected value comes from
a printed result on the pages, a closed form, a library routine, exact
rational arithmetic of a different formula (the product form of the "KDA
cheat sheet"), or the chunkwise form of the same cheat sheet.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

import oracle
from tests.chunkwise_fp64 import chunkwise_scan
from workloads import random_scan_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _alpha_bounded(rng, shape, g_min=-5.0):
    """Retention factors inside the bounded range, drawn directly (not via the gate)."""
    return np.exp(rng.uniform(g_min, 0.0, size=shape))


def _rand_case(seed, B=2, T=9, H=3, K=4, V=5, init=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, V))
    alpha = _alpha_bounded(rng, (B, T, H, K))
    beta = rng.uniform(0.0, 1.0, size=(B, T, H))
    s0 = rng.standard_normal((B, H, K, V)) * 0.3 if init else None
    return q, k, v, alpha, beta, s0


def _product_form(q, k, v, alpha, beta, S0):
    """Independent evaluation of the cheat sheet's product form, one head:
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t."""
    K = q.shape[1]
    S = S0.copy()
    outs = []
    for t in range(q.shape[0]):
        erase = np.eye(K) - beta[t] * np.outer(k[t], k[t])
        S = erase @ np.diag(alpha[t]) @ S + beta[t] * np.outer(k[t], v[t])
        outs.append(S.T @ q[t])
    return np.array(outs).reshape(q.shape[0], -1), S


# ----------------------------------------------------------------------------------------
# Scan pins
# ----------------------------------------------------------------------------------------

def test_toy_write_overwrite_retain_exact():
    """The printed toy outputs [2, 7, 5, 1.25] (PaperLeet, Toy experiment)."""
    g = _load("toy_write_overwrite_retain.json")
    T = len(g["beta"])
    q = np.array(g["q"], float).reshape(1, T, 1, g["K"])
    k = np.array(g["k"], float).reshape(1, T, 1, g["K"])
    v = np.array(g["v"], float).reshape(1, T, 1, g["V"])
    a = np.array(g["alpha"], float).reshape(1, T, 1, g["K"])
    b = np.array(g["beta"], float).reshape(1, T, 1)
    o, sf = oracle.scan(q, k, v, a, b)
    assert o[0, :, 0, 0].tolist() == g["expected_o"]          # exact, not approximate
    assert sf[0, 0, :, 0].tolist() == [1.25, 7.0]


@pytest.mark.parametrize("seed", range(6))
def test_matches_independent_product_form(seed):
    """Eq. 1 of the PaperLeet page equals the cheat sheet's product form, K != V, with an initial state."""
    q, k, v, alpha, beta, s0 = _rand_case(seed, K=3 + seed % 3, V=2 + seed)
    o, sf = oracle.scan(q, k, v, alpha, beta, s0)
    for b_ in range(q.shape[0]):
        for h in range(q.shape[2]):
            po, ps = _product_form(q[b_, :, h], k[b_, :, h], v[b_, :, h], alpha[b_, :, h],
                                   beta[b_, :, h], s0[b_, h])
            np.testing.assert_allclose(o[b_, :, h], po, rtol=0, atol=1e-12)
            np.testing.assert_allclose(sf[b_, h], ps, rtol=0, atol=1e-12)


def test_product_form_exact_rationals():
    """Exact rational evaluation of the product form agrees with the fp64 oracle to 1e-14."""
    rng = np.random.default_rng(11)
    T, K, V = 6, 3, 2
    Fr = lambda x: Fraction(int(x), 16)  # noqa: E731  (rationals with denominator 16)
    q = [[Fr(rng.integers(-16, 17)) for _ in range(K)] for _ in range(T)]
    k = [[Fr(rng.integers(-8, 9)) for _ in range(K)] for _ in range(T)]
    v = [[Fr(rng.integers(-32, 33)) for _ in range(V)] for _ in range(T)]
    a = [[Fr(rng.integers(1, 17)) for _ in range(K)] for _ in range(T)]
    be = [Fr(rng.integers(0, 17)) for _ in range(T)]
    S = [[Fraction(0)] * V for _ in range(K)]
    exact_o = []
    for t in range(T):
        DS = [[a[t][i] * S[i][j] for j in range(V)] for i in range(K)]
        E = [[(1 if i == r else 0) - be[t] * k[t][i] * k[t][r] for r in range(K)] for i in range(K)]
        S = [[sum(E[i][r] * DS[r][j] for r in range(K)) + be[t] * k[t][i] * v[t][j]
              for j in range(V)] for i in range(K)]
        exact_o.append([sum(S[i][j] * q[t][i] for i in range(K)) for j in range(V)])
    f = lambda m: np.array([[float(x) for x in row] for row in m])  # noqa: E731
    o, sf = oracle.scan(f(q).reshape(1, T, 1, K), f(k).reshape(1, T, 1, K), f(v).reshape(1, T, 1, V),
                        f(a).reshape(1, T, 1, K), np.array([float(x) for x in be]).reshape(1, T, 1))
    np.testing.assert_allclose(o[0, :, 0], f(exact_o), rtol=0, atol=1e-14 * max(1.0, np.abs(f(exact_o)).max()))
    np.testing.assert_allclose(sf[0, 0], f(S), rtol=0, atol=1e-14 * max(1.0, np.abs(f(S)).max()))


def test_identity_alpha_one_beta_zero():
    """alpha = 1, beta = 0 leaves the state unchanged and every read is S0^T q_t."""
    q, k, v, _, _, s0 = _rand_case(1)
    alpha = np.ones_like(q)
    beta = np.zeros(q.shape[:3])
    o, sf = oracle.scan(q, k, v, alpha, beta, s0)
    np.testing.assert_array_equal(sf, s0)
    np.testing.assert_allclose(o, np.einsum("bhkv,bthk->bthv", s0, q), rtol=0, atol=1e-13)


def test_zero_writes_closed_form():
    """beta = 0: S_t = Diag(prod_{r<=t} alpha_r) S0 and o_t = S_t^T q_t (pure fade)."""
    q, k, v, alpha, _, s0 = _rand_case(2)
    beta = np.zeros(q.shape[:3])
    o, sf = oracle.scan(q, k, v, alpha, beta, s0)
    cum = np.cumprod(alpha, axis=1)                          # [B,T,H,K]
    expect_o = np.einsum("bthk,bhkv,bthk->bthv", cum, s0, q)
    np.testing.assert_allclose(o, expect_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sf, cum[:, -1][..., None] * s0, rtol=1e-12, atol=1e-13)


def test_scalar_closed_form_k_v_one():
    """K = V = 1: s <- alpha s (1 - beta k^2) + beta k v and o = s q."""
    rng = np.random.default_rng(5)
    T = 12
    q, k, v = rng.standard_normal((3, T))
    a = rng.uniform(0.1, 1.0, T)
    b = rng.uniform(0.0, 1.0, T)
    s, outs = 0.7, []
    for t in range(T):
        s = a[t] * s * (1 - b[t] * k[t] ** 2) + b[t] * k[t] * v[t]
        outs.append(s * q[t])
    o, sf = oracle.scan(q.reshape(1, T, 1, 1), k.reshape(1, T, 1, 1), v.reshape(1, T, 1, 1),
                        a.reshape(1, T, 1, 1), b.reshape(1, T, 1), np.full((1, 1, 1, 1), 0.7))
    np.testing.assert_allclose(o.ravel(), outs, rtol=1e-13, atol=1e-14)
    assert abs(sf.ravel()[0] - s) < 1e-13


def test_deltanet_orthonormal_overwrite():
    """DeltaNet limit (alpha = 1, beta = 1, cheat sheet Lineage): with orthonormal keys,
    each write replaces the value stored at its key; reads return the last write."""
    rng = np.random.default_rng(7)
    K, V, T = 4, 3, 10
    basis, _ = np.linalg.qr(rng.standard_normal((K, K)))     # orthonormal columns
    slots = rng.integers(0, K, T)
    k = basis[:, slots].T
    v = rng.standard_normal((T, V))
    qsel = rng.integers(0, K, T)
    q = basis[:, qsel].T
    o, sf = oracle.scan(q.reshape(1, T, 1, K), k.reshape(1, T, 1, K), v.reshape(1, T, 1, V),
                        np.ones((1, T, 1, K)), np.ones((1, T, 1)))
    stored = {}
    for t in range(T):
        stored[slots[t]] = v[t]
        expect = stored.get(qsel[t], np.zeros(V))
        np.testing.assert_allclose(o[0, t, 0], expect, atol=1e-12)


def test_gated_linear_attention_orthogonal_keys():
    """Keys used once and mutually orthogonal never erase anything, so with a scalar
    per-token decay a_t (Gated DeltaNet's shared rate) the state is a decayed sum of
    writes: o_t = sum_{i<=t} (prod_{i<r<=t} a_r) beta_i <q_t, k_i> v_i."""
    rng = np.random.default_rng(9)
    K, V, T = 8, 3, 8
    basis, _ = np.linalg.qr(rng.standard_normal((K, K)))
    k = basis.T[:T]
    q = rng.standard_normal((T, K))
    v = rng.standard_normal((T, V))
    a = rng.uniform(0.2, 1.0, T)
    b = rng.uniform(0.1, 1.0, T)
    alpha = np.repeat(a[:, None], K, axis=1)
    o, _ = oracle.scan(q.reshape(1, T, 1, K), k.reshape(1, T, 1, K), v.reshape(1, T, 1, V),
                       alpha.reshape(1, T, 1, K), b.reshape(1, T, 1))
    for t in range(T):
        exp_o = sum(np.prod(a[i + 1:t + 1]) * b[i] * (q[t] @ k[i]) * v[i] for i in range(t + 1))
        np.testing.assert_allclose(o[0, t, 0], exp_o, atol=1e-12)


@pytest.mark.parametrize("with_init", [True, False])
def test_empty_sequence_returns_input_state(with_init):
    """T = 0: output has zero length; final state equals the initial state, or zeros."""
    B, H, K, V = 2, 3, 4, 5
    s0 = np.random.default_rng(0).standard_normal((B, H, K, V)) if with_init else None
    z = np.zeros((B, 0, H, K))
    o, sf = oracle.scan(z, z, np.zeros((B, 0, H, V)), z, np.zeros((B, 0, H)), s0)
    assert o.shape == (B, 0, H, V)
    np.testing.assert_array_equal(sf, s0 if with_init else np.zeros((B, H, K, V)))


@pytest.mark.parametrize("split", [1, 5, 8])
def test_split_and_resume(split):
    """Segmented continuation: scanning [0,split) then [split,T) from final_state equals one scan."""
    q, k, v, alpha, beta, s0 = _rand_case(3, T=9)
    o, sf = oracle.scan(q, k, v, alpha, beta, s0)
    o1, s1 = oracle.scan(q[:, :split], k[:, :split], v[:, :split], alpha[:, :split], beta[:, :split], s0)
    o2, s2 = oracle.scan(q[:, split:], k[:, split:], v[:, split:], alpha[:, split:], beta[:, split:], s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, sf, rtol=0, atol=1e-12)


def test_causal_prefix():
    """Changing tokens after t leaves every output up to t unchanged."""
    q, k, v, alpha, beta, s0 = _rand_case(4, T=10)
    o, _ = oracle.scan(q, k, v, alpha, beta, s0)
    rng = np.random.default_rng(40)
    t0 = 6
    q2, k2, v2, a2, b2 = (x.copy() for x in (q, k, v, alpha, beta))
    q2[:, t0:] = rng.standard_normal(q2[:, t0:].shape)
    k2[:, t0:] = rng.standard_normal(k2[:, t0:].shape)
    v2[:, t0:] = rng.standard_normal(v2[:, t0:].shape)
    a2[:, t0:] = rng.uniform(0.01, 1.0, a2[:, t0:].shape)
    b2[:, t0:] = rng.uniform(0, 1, b2[:, t0:].shape)
    o2, _ = oracle.scan(q2, k2, v2, a2, b2, s0)
    np.testing.assert_array_equal(o2[:, :t0], o[:, :t0])
    assert np.abs(o2[:, t0:] - o[:, t0:]).max() > 1e-3


def test_stability_bound_unit_keys():
    """With ||k|| = 1, beta in [0,1], alpha in (0,1]: the erase-and-fade map is a contraction,
    so ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t|| (follows from the product form)."""
    rng = np.random.default_rng(12)
    K, V, T = 6, 5, 40
    k = rng.standard_normal((T, K))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    q, v = rng.standard_normal((T, K)), rng.standard_normal((T, V))
    a, b = _alpha_bounded(rng, (T, K)), rng.uniform(0, 1, T)
    s0 = rng.standard_normal((K, V))
    prev = np.linalg.norm(s0)
    for t in range(T):
        _, sf = oracle.scan(q[: t + 1].reshape(1, -1, 1, K), k[: t + 1].reshape(1, -1, 1, K),
                            v[: t + 1].reshape(1, -1, 1, V), a[: t + 1].reshape(1, -1, 1, K),
                            b[: t + 1].reshape(1, -1, 1), s0.reshape(1, 1, K, V))
        cur = np.linalg.norm(sf)
        assert cur <= prev + b[t] * np.linalg.norm(v[t]) + 1e-12
        prev = cur


def test_varlen_equals_separate_sequences():
    """Packed sequences (cu_seqlens) equal independent scans, zero-length segments included."""
    rng = np.random.default_rng(13)
    lens = [3, 0, 5, 1, 0, 4]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, K, V = int(cu[-1]), 2, 3, 4
    q, k, v = rng.standard_normal((1, T, H, K)), rng.standard_normal((1, T, H, K)), rng.standard_normal((1, T, H, V))
    a, b = _alpha_bounded(rng, (1, T, H, K)), rng.uniform(0, 1, (1, T, H))
    s0 = rng.standard_normal((len(lens), H, K, V))
    o, sf = oracle.scan(q, k, v, a, b, s0, cu_seqlens=cu)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        on, sn = oracle.scan(q[:, s:e], k[:, s:e], v[:, s:e], a[:, s:e], b[:, s:e], s0[n:n + 1])
        np.testing.assert_array_equal(o[:, s:e], on)
        np.testing.assert_array_equal(sf[n:n + 1], sn)


@pytest.mark.parametrize("C", [1, 2, 16, 64, 150])
def test_chunkwise_form_equals_oracle(C):
    """The cheat sheet's chunkwise form (eqs. 3-4 with the re-derived UT transform) equals the
    recurrence for several chunk sizes, a ragged last chunk and K != V."""
    d = random_scan_case(B=1, T=150, H=2, K=8, V=6, seed=21, init_std=0.2)
    alpha = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"])
    args = (d["q"], d["k"], d["v"], alpha, d["beta"])
    o, sf = oracle.scan(*args, d["initial_state"])
    oc, sc = chunkwise_scan(*args, d["initial_state"].double().numpy(), C)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-10)
    np.testing.assert_allclose(sc, sf, rtol=0, atol=1e-10)


def test_inputs_not_mutated():
    q, k, v, alpha, beta, s0 = _rand_case(6)
    before = [x.copy() for x in (q, k, v, alpha, beta, s0)]
    oracle.scan(q, k, v, alpha, beta, s0)
    for x, y in zip(before, (q, k, v, alpha, beta, s0)):
        np.testing.assert_array_equal(x, y)


# ----------------------------------------------------------------------------------------
# Gate pins
# ----------------------------------------------------------------------------------------

def test_gate_figure3a_points():
    """Closed-form points of the bounded gate at A = 0, g_min = -5 (Figure 3(a) redraw)."""
    g = _load("gate_figure3a_points.json")
    z = np.array([p["z"] for p in g["points"]]).reshape(1, -1, 1, 1)
    alpha, lg = oracle.bounded_decay(z, np.array([g["A"]]), g["g_min"], return_log=True)
    for i, p in enumerate(g["points"]):
        assert lg.ravel()[i] == pytest.approx(p["g"], rel=1e-14, abs=0)
        assert alpha.ravel()[i] == pytest.approx(math.exp(p["g"]), rel=1e-14)


def test_gate_against_library_sigmoid_and_range():
    """g = g_min * expit(e^A z) (scipy's logistic), g in (g_min, 0), alpha in (e^g_min, 1)
    strictly for |e^A z| <= 8 and in the closed interval everywhere; decreasing in z."""
    rng = np.random.default_rng(3)
    H, K = 4, 64
    A = rng.normal(0, 0.5, H)
    z = np.concatenate([np.linspace(-40, 40, 7 * K).reshape(1, 7, 1, K).repeat(H, 2),
                        rng.normal(0, 2, (1, 9, H, K))], axis=1)
    for g_min in (-5.0, -1.0, -12.0):
        alpha, lg = oracle.bounded_decay(z, A, g_min, return_log=True)
        x = np.exp(A)[None, None, :, None] * z
        np.testing.assert_allclose(lg, g_min * scipy.special.expit(x), rtol=1e-14, atol=0)
        np.testing.assert_allclose(alpha, np.exp(g_min * scipy.special.expit(x)), rtol=1e-14)
        moderate = np.abs(x) <= 8
        assert np.all((lg[moderate] > g_min) & (lg[moderate] < 0))
        assert np.all((alpha[moderate] > math.exp(g_min)) & (alpha[moderate] < 1))
        assert np.all((alpha >= math.exp(g_min)) & (alpha <= 1))
        assert np.all(np.diff(lg[0, :7, 0].ravel()) <= 0)   # non-increasing along the sorted grid


def test_gate_log_scale_rescales_logits():
    """A shifts the curve's scale: gate(z; A) = gate(e^A z; 0)."""
    rng = np.random.default_rng(4)
    z = rng.normal(0, 2, (2, 3, 2, 8))
    A = np.array([0.7, -0.4])
    a1 = oracle.bounded_decay(z, A, -5.0)
    a0 = oracle.bounded_decay(z * np.exp(A)[None, None, :, None], np.zeros(2), -5.0)
    np.testing.assert_allclose(a1, a0, rtol=1e-14)


def test_gate_contrast_with_unbounded_softplus_gate():
    """Figure 3(a) contrast: Kimi Linear's -softplus(z) log-decay is unbounded below, the
    bounded gate never passes g_min (same logits, A = 0)."""
    z = np.linspace(-10, 10, 201).reshape(1, -1, 1, 1)
    lg = oracle.bounded_decay(z, np.zeros(1), -5.0, return_log=True)[1].ravel()
    unbounded = -np.logaddexp(0.0, z.ravel())                # -softplus, numpy's log-add-exp
    assert unbounded.min() < -10.0 and lg.min() > -5.0
    assert np.all(lg >= -5.0) and np.all(lg <= 0.0)


def test_gate_bias_shifts_the_logits_before_the_scale():
    """The bias enters as z + b inside the sigmoid's argument, before the e^A scale ("KDA cheat sheet",
    How the inputs are produced: z = W_up W_down x + b). With z = -b[h, c] on every entry the argument is
    exactly 0 and g = g_min / 2; a bias added after the scale (e^A z + b), to g, or read transposed
    ([c, h] for [h, c]) leaves a non-zero argument on some entry."""
    H, K = 2, 3
    b = np.array([[0.5, -1.25, 2.0], [3.0, -0.75, 1.5]])
    z = np.broadcast_to(-b, (1, 4, H, K)).copy()
    A = np.array([0.7, -0.3])
    for g_min in (-5.0, -8.0):
        alpha, lg = oracle.bounded_decay(z, A, g_min, return_log=True, dt_bias=b)
        assert np.all(lg == g_min / 2) and np.allclose(alpha, math.exp(g_min / 2), rtol=1e-15)
    # z = 0 and b = ln 3 / e^A: the argument is ln 3, sigmoid(ln 3) = 3/4, g = 0.75 g_min
    b2 = np.log(3.0) * np.exp(-A)[:, None] * np.ones((H, K))
    lg2 = oracle.bounded_decay(np.zeros((1, 2, H, K)), A, -5.0, return_log=True, dt_bias=b2)[1]
    np.testing.assert_allclose(lg2, -3.75, rtol=1e-14)
    # the unbounded gate takes the same bias: z = -b gives softplus(0) = ln 2, g = -e^A ln 2
    lgs = oracle.softplus_decay(z, A, return_log=True, dt_bias=b)[1]
    np.testing.assert_allclose(lgs, -np.exp(A)[None, None, :, None] * np.log(2.0) * np.ones_like(z), rtol=1e-15)


# ---------------------------------------------------------------------------------------------
# Input preparation ("KDA cheat sheet", How the inputs are produced): L2Norm of q, k; beta = Sigmoid
# ---------------------------------------------------------------------------------------------

def test_l2norm_pythagorean_rows_and_axis():
    # Rows (3, 4) and (5, 12) have norms 5 and 13; the epsilon under the root is 1e-6.
    x = np.array([[[3.0, 4.0], [5.0, 12.0]]])
    y = oracle.l2norm(x)
    np.testing.assert_allclose(y[0, 0], np.array([3.0, 4.0]) / np.sqrt(25.0 + 1e-6), rtol=1e-15)
    np.testing.assert_allclose(y[0, 1], np.array([5.0, 12.0]) / np.sqrt(169.0 + 1e-6), rtol=1e-15)
    # Normalising over the wrong axis would mix the two rows; each row keeps its direction.
    assert abs(y[0, 0, 0] / y[0, 0, 1] - 0.75) < 1e-15 and abs(y[0, 1, 0] / y[0, 1, 1] - 5 / 12) < 1e-15


def test_l2norm_unit_scale_invariance_and_zero_row():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(5, 3, 16))
    y = oracle.l2norm(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-6)   # unit rows (up to the epsilon)
    np.testing.assert_allclose(oracle.l2norm(1e3 * x), y, atol=1e-9)           # scale invariant
    assert np.all(oracle.l2norm(np.zeros((2, 8))) == 0.0)                      # no NaN for a zero row


def test_sigmoid_exact_points_symmetry_and_range():
    assert oracle.sigmoid(0.0) == 0.5
    np.testing.assert_allclose(oracle.sigmoid(np.log(3.0)), 0.75, rtol=1e-15)
    np.testing.assert_allclose(oracle.sigmoid(-np.log(3.0)), 0.25, rtol=1e-15)
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(oracle.sigmoid(x) + oracle.sigmoid(-x), 1.0, atol=1e-15)
    with np.errstate(over="raise", invalid="raise", divide="raise"):  # underflow to 0 is the right answer
        assert oracle.sigmoid(-800.0) == 0.0 and oracle.sigmoid(800.0) == 1.0


# ---------------------------------------------------------------------------------------------
# Kimi Linear's unbounded gate, g = -e^A softplus(z) (Figure 3(a) contrast; cheat sheet g_min table)
# ---------------------------------------------------------------------------------------------

def _sp(z, A=0.0):
    z = np.asarray(z, dtype=np.float64).reshape(1, -1, 1, 1)
    return oracle.softplus_decay(z, np.array([A]), return_log=True)[1].ravel()


def test_softplus_gate_exact_point_and_reflection():
    assert abs(_sp([0.0])[0] + np.log(2.0)) < 1e-16                     # softplus(0) = ln 2
    z = np.linspace(-40, 40, 161)
    np.testing.assert_allclose(_sp(z) - _sp(-z), -z, atol=1e-12)         # softplus(z) - softplus(-z) = z


def test_softplus_gate_slope_is_minus_sigmoid_and_scale():
    z = np.linspace(-12, 12, 97)
    h = 1e-5
    slope = (_sp(z + h) - _sp(z - h)) / (2 * h)
    np.testing.assert_allclose(slope, -oracle.sigmoid(z), atol=1e-9)    # d softplus / dz = sigmoid
    np.testing.assert_allclose(_sp(z, A=0.7), np.exp(0.7) * _sp(z), rtol=1e-14)


def test_softplus_gate_is_unbounded_below_and_stable():
    g = _sp([10.0, 50.0, 800.0, -50.0])
    assert g[0] < -10.0 and abs(g[1] + 50.0) < 1e-12 and g[2] == -800.0   # no overflow, no lower bound
    assert -1e-21 < g[3] < 0.0                                             # -softplus(-50) = -e^-50 (1 - ...)
    alpha = np.exp(g)
    assert np.all(alpha <= 1.0) and np.all(alpha >= 0.0)


# ---------------------------------------------------------------------------------------------
# Gradients (the contract is differentiable): the fp64 torch restatement and its autograd
# ---------------------------------------------------------------------------------------------

def test_torch_scan_equals_c_oracle():
    import torch
    rng = np.random.default_rng(8)
    B, T, H, K, V = 2, 9, 2, 5, 3
    q, k, v = rng.normal(size=(B, T, H, K)), rng.normal(size=(B, T, H, K)), rng.normal(size=(B, T, H, V))
    a, b, s0 = rng.uniform(0.1, 1, (B, T, H, K)), rng.uniform(0, 1, (B, T, H)), rng.normal(size=(B, H, K, V))
    o, sf = oracle.scan_torch(*(torch.tensor(x) for x in (q, k, v, a, b, s0)))
    ro, rs = oracle.scan(q, k, v, a, b, s0)
    np.testing.assert_allclose(o.numpy(), ro, atol=1e-12)
    np.testing.assert_allclose(sf.numpy(), rs, atol=1e-12)


def test_scan_gradients_match_finite_differences():
    import torch
    rng = np.random.default_rng(9)
    B, T, H, K, V = 1, 4, 1, 3, 2
    args = [torch.tensor(x, requires_grad=True) for x in (
        rng.normal(size=(B, T, H, K)), rng.normal(size=(B, T, H, K)), rng.normal(size=(B, T, H, V)),
        rng.uniform(0.2, 1, (B, T, H, K)), rng.uniform(0.1, 0.9, (B, T, H)), rng.normal(size=(B, H, K, V)))]
    do, dsf = rng.normal(size=(B, T, H, V)), rng.normal(size=(B, H, K, V))

    def loss(*a):
        o, sf = oracle.scan_torch(*a)
        return (o * torch.tensor(do)).sum() + (sf * torch.tensor(dsf)).sum()
    assert torch.autograd.gradcheck(loss, args, eps=1e-6, atol=1e-8)
    g = oracle.scan_backward(*(x.detach().numpy() for x in args), do, dsf)
    auto = torch.autograd.grad(loss(*args), args)
    for name, ga in zip(("q", "k", "v", "alpha", "beta", "initial_state"), auto):
        np.testing.assert_allclose(g[name], ga.numpy(), atol=1e-12)


def test_gate_gradients_match_finite_differences():
    import torch
    rng = np.random.default_rng(10)
    z, A = rng.normal(size=(1, 3, 2, 4)), rng.normal(size=2) * 0.5
    dg = rng.normal(size=(1, 3, 2, 4))
    dz, dA = oracle.bounded_decay_backward(z, A, -5.0, dg)
    f = lambda zz, aa: (-5.0 * torch.sigmoid(torch.exp(aa)[None, None, :, None] * zz) * torch.tensor(dg)).sum()  # noqa: E731
    assert torch.autograd.gradcheck(f, (torch.tensor(z, requires_grad=True), torch.tensor(A, requires_grad=True)))
    h = 1e-6
    zp, zm = z.copy(), z.copy()
    zp[0, 1, 1, 2] += h
    zm[0, 1, 1, 2] -= h
    num = (f(torch.tensor(zp), torch.tensor(A)) - f(torch.tensor(zm), torch.tensor(A))).item() / (2 * h)
    assert abs(num - dz[0, 1, 1, 2]) < 1e-7


# The unbounded gate on the chunked path ("Kimi K3: Bounded Decay and Delta Memory", Figure 3(a) contrast;
# "KDA cheat sheet", the BF16 reciprocal-rescale argument): with g = -e^A softplus(z) the reciprocal of a
# 16-token block's decay leaves the fp32 range, so the diagonal blocks are formed pairwise, while every
# factor that crosses a block boundary stays <= 1. Checked in fp32 arithmetic against the pairwise
# definition in fp64.

def _a_qk_exact(q, k, G):
    d = G[:, None, :] - G[None, :, :]
    ratio = np.where(np.tril(np.ones((len(q), len(q)), bool))[:, :, None], np.exp(np.minimum(d, 0.0)), 0.0)
    return np.einsum("tc,ic,tic->ti", q, k, ratio)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_block_factorisation_needs_pairwise_diagonal_blocks_for_the_unbounded_gate():
    from tests.chunkwise_fp64 import block_factored_a
    rng = np.random.default_rng(7)
    n, K = 64, 32
    q, k = _unit(rng.standard_normal((n, K))), _unit(rng.standard_normal((n, K)))
    z = rng.standard_normal((n, K)) * 4.0
    g = -np.exp(4.0) * (np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z))))   # softplus gate, e^A = e^4
    G = np.cumsum(g, axis=0)
    assert (G[15] - 0.0).min() < -1000.0                                      # a block's decay is e^-1000 or less
    exact = _a_qk_exact(q, k, G)
    A_split, _ = block_factored_a(q, k, G, pairwise_diag=False)
    assert not np.all(np.isfinite(A_split))                                   # the split diagonal overflows
    A_pair, worst = block_factored_a(q, k, G, pairwise_diag=True)
    assert worst <= 1.0                                                       # every cross-block factor <= 1
    assert np.all(np.isfinite(A_pair))
    np.testing.assert_allclose(A_pair, exact, rtol=0, atol=1e-5)


def test_block_factorisation_is_safe_for_the_bounded_gate():
    from tests.chunkwise_fp64 import block_factored_a
    rng = np.random.default_rng(8)
    n, K = 64, 32
    q, k = _unit(rng.standard_normal((n, K))), _unit(rng.standard_normal((n, K)))
    g = np.full((n, K), -5.0)                                                 # the bound itself, every token
    G = np.cumsum(g, axis=0)
    exact = _a_qk_exact(q, k, G)
    A_split, worst = block_factored_a(q, k, G, pairwise_diag=False)
    assert worst <= 1.0 and np.all(np.isfinite(A_split))                      # e^80 at most on the diagonal
    np.testing.assert_allclose(A_split, exact, rtol=0, atol=1e-5)


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunkwise_backward_derivation_matches_the_oracle_gradients(C):
    # The adjoint of the chunkwise form (tests/chunkwise_fp64.py: dU, dS0, dT through the UT transform's
    # inverse, the bilinear forms A_qk and A_kk, the Gamma factors, dlog(alpha) as a reverse cumulative sum),
    # walked chunk by chunk from the end, equals the token-level autograd gradients of eq. 1 for every chunk
    # length, a ragged last chunk included.
    from tests.chunkwise_fp64 import chunkwise_backward
    rng = np.random.default_rng(3)
    B, T, H, K, V = 1, 37, 2, 6, 5
    q, k = rng.standard_normal((B, T, H, K)), rng.standard_normal((B, T, H, K)) * 0.5
    v = rng.standard_normal((B, T, H, V))
    alpha = np.exp(-rng.uniform(0.01, 2.0, (B, T, H, K)))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    s0 = rng.standard_normal((B, H, K, V)) * 0.3
    do = rng.standard_normal((B, T, H, V))
    dsf = rng.standard_normal((B, H, K, V)) * 0.3
    ref = oracle.scan_backward(q, k, v, alpha, beta, s0, do, dsf)
    got = chunkwise_backward(q, k, v, alpha, beta, s0, do, dsf, C)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name], rtol=0, atol=1e-12 * float(np.abs(ref[name]).max()))


@pytest.mark.parametrize("C", [4, 16, 64])
def test_chunkwise_backward_three_pass_split_matches_the_oracle(C):
    # The same gradients computed as a chunked backward's kernels would: state-independent operands per
    # chunk, one reverse recurrence over dS that emits dU, then every other gradient per chunk in parallel.
    from tests.chunkwise_fp64 import chunkwise_backward_split
    rng = np.random.default_rng(5)
    T, K, V = 45, 7, 4
    q, k = rng.standard_normal((T, K)), rng.standard_normal((T, K)) * 0.5
    v = rng.standard_normal((T, V))
    alpha = np.exp(-rng.uniform(0.01, 2.0, (T, K)))
    beta = rng.uniform(0.1, 0.9, T)
    s0 = rng.standard_normal((K, V)) * 0.3
    do = rng.standard_normal((T, V))
    dsf = rng.standard_normal((K, V)) * 0.3
    ref = oracle.scan_backward(q[None, :, None], k[None, :, None], v[None, :, None], alpha[None, :, None],
                               beta[None, :, None], s0[None, None], do[None, :, None], dsf[None, None])
    got = chunkwise_backward_split(q, k, v, alpha, beta, s0, do, dsf, C)
    for g, name in zip(got, ("q", "k", "v", "alpha", "beta", "initial_state")):
        r = ref[name][0, :, 0] if name != "initial_state" else ref[name][0, 0]
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-12 * float(np.abs(r).max()))
