"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something fixed by the pages or by the
mathematics, not against itself: a hand-worked example, closed forms from the
pages' identities, special cases that reduce to a textbook matmul, and
agreement with routes that follow different passages.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_inputs(rng, B, T, H, dk, dv, gates, s0=False, k_unit=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if k_unit:
        k = unit(k)
    v = rng.standard_normal((B, T, H, dv))
    shape = lambda kind: (B, T, H) if kind == "scalar" else (B, T, H, dk)
    alpha = None if gates["alpha"] == "none" else np.exp(-np.log1p(np.exp(rng.standard_normal(shape(gates["alpha"])))))
    b = None if gates["b"] == "none" else rng.random(shape(gates["b"]))
    w = None if gates["w"] in ("none", "tied") else rng.random(shape(gates["w"]))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3 if s0 else None
    return q, k, v, alpha, b, w, S0


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()])
    return vals


GEN = {"alpha": "channel", "b": "channel", "w": "channel"}


# --- hand-worked example -----------------------------------------------------

def test_golden_worked_example():
    """tests/golden/worked_example_dk2_dv3.txt: two tokens worked by hand."""
    g = read_golden("worked_example_dk2_dv3.txt")
    T, dk, dv = 2, 2, 3
    sh = lambda x, d: x.reshape(1, T, 1, d)
    q, k, v = sh(g["q"], dk), sh(g["k"], dk), sh(g["v"], dv)
    a, b, w = sh(g["alpha"], dk), sh(g["b"], dk), sh(g["w"], dk)
    S0 = g["S0"].reshape(1, 1, dk, dv)
    o, ST = oracle.recurrence(q, k, v, a, b, w, S0, GEN)
    np.testing.assert_array_equal(o.reshape(-1), g["o"])
    np.testing.assert_array_equal(ST.reshape(-1), g["S2"])
    # the same two tokens through the decode entry, state carried between calls
    S = S0
    for t, Sref in ((0, g["S1"]), (1, g["S2"])):
        sl = lambda x: x[:, t]
        ot, S = oracle.decode_step(sl(q), sl(k), sl(v), sl(a), sl(b), sl(w), S, GEN)
        np.testing.assert_array_equal(S.reshape(-1), Sref)
        np.testing.assert_array_equal(ot.reshape(-1), g["o"][t * dv:(t + 1) * dv])
    o2, ST2 = oracle.recurrence_py(q, k, v, a, b, w, S0, GEN)
    np.testing.assert_array_equal(o2.reshape(-1), g["o"])


# --- identities printed on the pages ---------------------------------------

def test_self_read_after_one_write():
    """Query with the key just written from S=0 returns ||k||^2 v ("Recurrent
    Memory: Write, Erase, Decay, Read", section 01); with a write gate w the
    stored key is w.k, so the read is (k.(w.k)) v."""
    dk, dv = 7, 5
    k = RNG.standard_normal((1, 1, 1, dk)) * 1.7          # not unit: the factor shows
    v = RNG.standard_normal((1, 1, 1, dv))
    o, _ = oracle.recurrence(k, k, v, gates={"alpha": "none", "b": "none", "w": "none"})
    np.testing.assert_allclose(o[0, 0, 0], np.sum(k ** 2) * v[0, 0, 0], rtol=1e-13)
    w = RNG.random((1, 1, 1, dk))
    b = RNG.random((1, 1, 1, dk))
    a = RNG.random((1, 1, 1, dk)) + 0.1
    o, _ = oracle.recurrence(k, k, v, a, b, w, None, GEN)
    np.testing.assert_allclose(o[0, 0, 0], np.sum(k * w * k) * v[0, 0, 0], rtol=1e-13)


def test_overwrite_returns_latest_value():
    """Writing the same unit key twice with b=w=1, alpha=1 returns the second
    value ("Recurrent Memory", section 02/03; "The Eraser Trilogy", "Eraser
    two"); memories orthogonal to k are untouched (section 03, projection at
    beta=1). Pure accumulation (b=0) returns the sum instead (section 02)."""
    dk, dv = 8, 4
    Q, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    k1, k2 = Q[0], Q[1]
    v1, v2, v3 = RNG.standard_normal((3, dv))
    k = np.stack([k2, k1, k1])[None, :, None]
    v = np.stack([v3, v1, v2])[None, :, None]
    q = np.stack([k2, k1, k1])[None, :, None]
    ones = np.ones((1, 3, 1, dk))
    o, _ = oracle.recurrence(q, k, v, None, ones, ones, None,
                             {"alpha": "none", "b": "channel", "w": "channel"})
    np.testing.assert_allclose(o[0, 2, 0], v2, atol=1e-13)
    o_k2, _ = oracle.recurrence(np.stack([k2, k2, k2])[None, :, None], k, v, None, ones, ones,
                                None, {"alpha": "none", "b": "channel", "w": "channel"})
    np.testing.assert_allclose(o_k2[0, 2, 0], v3, atol=1e-13)
    o_acc, _ = oracle.recurrence(q, k, v, gates={"alpha": "none", "b": "none", "w": "none"})
    np.testing.assert_allclose(o_acc[0, 2, 0], v1 + v2, atol=1e-13)


def test_orthonormal_capacity_and_crosstalk():
    """A d_k x d_v board stores d_k orthonormal keys exactly; the (d_k+1)-th key
    necessarily overlaps a stored one ("Recurrent Memory", section 02)."""
    dk, dv = 6, 3
    Q, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    vals = RNG.standard_normal((dk, dv))
    for gates in ({"alpha": "none", "b": "none", "w": "none"},
                  {"alpha": "none", "b": "scalar", "w": "tied"}):
        k = Q[None, :, None]
        v = vals[None, :, None]
        bb = np.ones((1, dk, 1)) if gates["b"] == "scalar" else None
        _, S = oracle.recurrence(k, k, v, None, bb, None, None, gates)
        np.testing.assert_allclose(Q @ S[0, 0], vals, atol=1e-12)
        extra = unit(RNG.standard_normal(dk))
        k7 = np.concatenate([Q, extra[None]])[None, :, None]
        v7 = np.concatenate([vals, RNG.standard_normal((1, dv))])[None, :, None]
        bb7 = np.ones((1, dk + 1, 1)) if gates["b"] == "scalar" else None
        _, S7 = oracle.recurrence(k7, k7, v7, None, bb7, None, None, gates)
        assert np.max(np.abs(Q @ S7[0, 0] - vals)) > 1e-3


def test_beta_blend():
    """Tied gates b = w = beta, alpha = 1, unit k: reading with k gives
    (1-beta) k S_{t-1} + beta v ("Recurrent Memory", section 03 steps 2-3;
    "The Eraser Trilogy": beta as the learning rate of one gradient step)."""
    dk, dv = 9, 5
    k = unit(RNG.standard_normal((1, 1, 1, dk)))
    v = RNG.standard_normal((1, 1, 1, dv))
    S0 = RNG.standard_normal((1, 1, dk, dv))
    for beta in (0.0, 0.3, 1.0):
        bt = np.full((1, 1, 1), beta)
        o, _ = oracle.recurrence(k, k, v, None, bt, None, S0, {"alpha": "none", "b": "scalar", "w": "tied"})
        np.testing.assert_allclose(o[0, 0, 0], (1 - beta) * (k[0, 0, 0] @ S0[0, 0]) + beta * v[0, 0, 0],
                                   atol=1e-13)


def test_erase_eigenstructure():
    """I - beta k^T k with unit k scales the k component by 1-beta and leaves
    the orthogonal complement unchanged ("Recurrent Memory", section 03)."""
    dk, dv = 5, 4
    Q, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    k, u = Q[0], Q[1]
    v0, v1 = RNG.standard_normal((2, dv))
    S0 = (np.outer(k, v0) + np.outer(u, v1))[None, None]
    beta = 0.35
    zero_w = np.zeros((1, 1, 1))                       # no write this step
    kk = k[None, None, None]
    _, S = oracle.recurrence(kk, kk, np.zeros((1, 1, 1, dv)), None, np.full((1, 1, 1), beta), zero_w,
                             S0, {"alpha": "none", "b": "scalar", "w": "scalar"})
    np.testing.assert_allclose(k @ S[0, 0], (1 - beta) * v0, atol=1e-13)
    np.testing.assert_allclose(u @ S[0, 0], v1, atol=1e-13)


def test_decay_survival_factor():
    """A write survives t later steps scaled by the product of the decays
    applied after it, per channel for channel-wise alpha ("Recurrent Memory",
    section 04: product of alphas = exp of the sum of log alphas)."""
    dk, dv, T = 6, 3, 9
    k0 = unit(RNG.standard_normal(dk))
    v0 = RNG.standard_normal(dv)
    k = RNG.standard_normal((1, T, 1, dk))
    k[0, 0, 0] = k0
    v = np.zeros((1, T, 1, dv))
    v[0, 0, 0] = v0                                     # later tokens write nothing
    alpha = RNG.random((1, T, 1, dk)) * 0.9 + 0.05
    q = RNG.standard_normal((1, T, 1, dk))
    o, _ = oracle.recurrence(q, k, v, alpha, None, None, None, {"alpha": "channel", "b": "none", "w": "none"})
    for t in range(T):
        surv = np.exp(np.sum(np.log(alpha[0, 1:t + 1, 0]), axis=0))   # steps after the write
        np.testing.assert_allclose(o[0, t, 0], np.sum(q[0, t, 0] * surv * k0) * v0, rtol=1e-12, atol=1e-14)


# --- reductions of the general gates ----------------------------------------

def test_gdn2_reduces_to_kda_gdn_deltanet_linear_attention():
    """General gates collapse to the named forms ("Recurrent Memory", section
    05; "The Eraser Trilogy", "Eraser three"; "Erase-then-Delta Attention"
    abstract): b = w = beta gives KDA (channel alpha) and Gated DeltaNet
    (scalar alpha); alpha = 1 gives DeltaNet; b = 0, alpha = w = 1 gives
    linear attention, o = causal(Q K^T) V (the masked-matrix reading of "The
    Rosetta Stone", computed here as a dense matmul)."""
    B, T, H, dk, dv = 2, 17, 2, 6, 5
    rng = np.random.default_rng(7)
    q, k, v, _, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv, GEN, s0=True)
    beta = rng.random((B, T, H))
    alpha_ch = rng.random((B, T, H, dk)) * 0.8 + 0.2
    alpha_sc = rng.random((B, T, H)) * 0.8 + 0.2
    bfull = np.repeat(beta[..., None], dk, axis=-1)
    # KDA: channel alpha, scalar beta
    o, ST = oracle.recurrence(q, k, v, alpha_ch, bfull, bfull, S0, GEN)
    o3, ST3 = oracle.delta_three_line(q, k, v, alpha_ch, beta, S0, alpha_kind="channel")
    np.testing.assert_allclose(o, o3, atol=1e-12)
    np.testing.assert_allclose(ST, ST3, atol=1e-12)
    # Gated DeltaNet: scalar alpha; also equals the page's decay-after-erase order
    o, ST = oracle.recurrence(q, k, v, alpha_sc, beta, None, S0, {"alpha": "scalar", "b": "scalar", "w": "tied"})
    o3, _ = oracle.delta_three_line(q, k, v, alpha_sc, beta, S0, alpha_kind="scalar")
    np.testing.assert_allclose(o, o3, atol=1e-12)
    o5 = oracle.unified_decay_after_erase(q, k, v, np.repeat(alpha_sc[..., None], dk, -1), beta, S0)
    np.testing.assert_allclose(o, o5, atol=1e-12)
    # DeltaNet: alpha = 1
    o, _ = oracle.recurrence(q, k, v, None, beta, None, S0, {"alpha": "none", "b": "scalar", "w": "tied"})
    o3, _ = oracle.delta_three_line(q, k, v, None, beta, S0)
    np.testing.assert_allclose(o, o3, atol=1e-12)
    # linear attention
    o, _ = oracle.recurrence(q, k, v, gates={"alpha": "none", "b": "none", "w": "none"})
    for bi in range(B):
        for h in range(H):
            ref = np.tril(q[bi, :, h] @ k[bi, :, h].T) @ v[bi, :, h]
            np.testing.assert_allclose(o[bi, :, h], ref, atol=1e-12)


def test_decay_order_reading():
    """The section-05 equation of "Recurrent Memory" applies the decay after
    the erase; the recurrence built here applies it before (decay absorbed
    into the erase factor, "Erase-then-Delta Attention" abstract). The two
    agree for scalar alpha and differ for channel-wise alpha."""
    B, T, H, dk, dv = 1, 6, 1, 5, 4
    rng = np.random.default_rng(3)
    q, k, v, _, _, _, _ = rand_inputs(rng, B, T, H, dk, dv, GEN)
    beta = rng.random((B, T, H)) * 0.5 + 0.5
    a_ch = rng.random((B, T, H, dk)) * 0.9 + 0.1
    o_ns, _ = oracle.recurrence(q, k, v, a_ch, beta, None, None, {"alpha": "channel", "b": "scalar", "w": "tied"})
    o_p1 = oracle.unified_decay_after_erase(q, k, v, a_ch, beta)
    assert np.max(np.abs(o_ns - o_p1)) > 1e-3


def test_erase_reads_with_b_removes_along_k():
    """Asymmetric erase I - k^T (b.k): the erase reads the state with b.k and
    removes along k ("Erase-then-Delta Attention" abstract). With memory only
    under e_0, k = (e_0+e_1)/sqrt2 and b = e_1, the read b.k sees nothing, so
    nothing is erased; the other side assignment would erase."""
    dk, dv = 3, 2
    v0 = np.array([1.0, -2.0])
    S0 = np.zeros((1, 1, dk, dv))
    S0[0, 0, 0] = v0
    k = np.zeros((1, 1, 1, dk))
    k[..., 0] = k[..., 1] = 1 / np.sqrt(2)
    b = np.zeros((1, 1, 1, dk))
    b[..., 1] = 1.0
    w = np.zeros((1, 1, 1, dk))
    _, S = oracle.recurrence(k, k, np.zeros((1, 1, 1, dv)), None, b, w, S0,
                             {"alpha": "none", "b": "channel", "w": "channel"})
    np.testing.assert_allclose(S, S0, atol=1e-15)
    b[..., 0], b[..., 1] = 1.0, 0.0                    # now b.k sees e_0's memory
    _, S = oracle.recurrence(k, k, np.zeros((1, 1, 1, dv)), None, b, w, S0,
                             {"alpha": "none", "b": "channel", "w": "channel"})
    r = v0 / np.sqrt(2)
    np.testing.assert_allclose(S[0, 0, 0], v0 - r / np.sqrt(2), atol=1e-15)
    np.testing.assert_allclose(S[0, 0, 1], -r / np.sqrt(2), atol=1e-15)


# --- independent routes -----------------------------------------------------

@pytest.mark.parametrize("gates,s0", [
    (GEN, True),
    ({"alpha": "scalar", "b": "scalar", "w": "tied"}, False),
    ({"alpha": "channel", "b": "scalar", "w": "tied"}, True),
    ({"alpha": "none", "b": "channel", "w": "none"}, True),
])
def test_unrolled_contributions(gates, s0):
    """State as a sum of contributions with explicit transition matrices ("How
    Linear Attention Remembers", Analytical Framework)."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 1, 10, 2, 4, 3
    q, k, v, a, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv, gates, s0=s0, k_unit=False)
    o, ST = oracle.recurrence(q, k, v, a, b, w, S0, gates)
    ou, STu = oracle.unrolled_contributions(q, k, v, a, b, w, S0, gates)
    np.testing.assert_allclose(o, ou, atol=1e-12)
    np.testing.assert_allclose(ST, STu, atol=1e-12)


@pytest.mark.parametrize("akind", ["channel", "scalar", "none"])
def test_masked_matrix_form(akind):
    """Erase-free recurrence equals its structured-masked-matrix form ("The
    Eraser Trilogy", "The Rosetta Stone")."""
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 2, 23, 1, 5, 7
    gates = {"alpha": akind, "b": "none", "w": "channel"}
    q, k, v, a, _, w, _ = rand_inputs(rng, B, T, H, dk, dv, gates)
    o, _ = oracle.recurrence(q, k, v, a, None, w, None, gates)
    om = oracle.masked_matrix(q, k, v, a, w, gates)
    np.testing.assert_allclose(o, om, atol=1e-12)


def test_python_and_c_token_loops_agree():
    rng = np.random.default_rng(9)
    for gates in (GEN, {"alpha": "scalar", "b": "scalar", "w": "tied"}):
        q, k, v, a, b, w, S0 = rand_inputs(rng, 2, 33, 3, 8, 6, gates, s0=True)
        o, ST = oracle.recurrence(q, k, v, a, b, w, S0, gates, nthreads=2)
        o2, ST2 = oracle.recurrence_py(q, k, v, a, b, w, S0, gates)
        np.testing.assert_allclose(o, o2, atol=1e-12)
        np.testing.assert_allclose(ST, ST2, atol=1e-12)


def test_split_sequence_resumes_from_state():
    """Running T tokens equals running T1 then T-T1 with S0 := S_T of the first
    part (the state is the whole memory; "How Linear Attention Remembers",
    Analytical Framework)."""
    rng = np.random.default_rng(13)
    q, k, v, a, b, w, S0 = rand_inputs(rng, 1, 50, 2, 8, 4, GEN, s0=True)
    o, ST = oracle.recurrence(q, k, v, a, b, w, S0, GEN)
    T1 = 21
    sl = lambda x, s: None if x is None else x[:, s]
    o1, S1 = oracle.recurrence(sl(q, slice(0, T1)), sl(k, slice(0, T1)), sl(v, slice(0, T1)),
                               sl(a, slice(0, T1)), sl(b, slice(0, T1)), sl(w, slice(0, T1)), S0, GEN)
    o2, S2 = oracle.recurrence(sl(q, slice(T1, None)), sl(k, slice(T1, None)), sl(v, slice(T1, None)),
                               sl(a, slice(T1, None)), sl(b, slice(T1, None)), sl(w, slice(T1, None)), S1, GEN)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, atol=1e-12)
    np.testing.assert_allclose(S2, ST, atol=1e-12)


def test_empty_sequence_returns_initial_state():
    q = np.zeros((2, 0, 3, 4))
    v = np.zeros((2, 0, 3, 5))
    S0 = RNG.standard_normal((2, 3, 4, 5))
    o, ST = oracle.recurrence(q, q, v, None, None, None, S0, {"alpha": "none", "b": "none", "w": "none"})
    assert o.shape == (2, 0, 3, 5)
    np.testing.assert_array_equal(ST, S0)
