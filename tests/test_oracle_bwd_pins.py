"""Pins for the oracle's backward pass (no GPU).

The pages name a gate-aware backward pass ("Erase-then-Delta Attention"
(Gated DeltaNet-2), abstract) without a formula, so the gradient is fixed by
the mathematics alone: it must equal the derivative of the forward oracle
(central finite differences of `oracle.recurrence`, itself pinned in
test_oracle_pins.py), and it must reduce to closed forms where the forward is
a plain masked matrix product ("The Eraser Trilogy", "The Rosetta Stone").
"""
import zlib

import numpy as np
import pytest

import oracle
from test_oracle_pins import rand_inputs

GRAD_OF = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "b": "db", "w": "dw", "S0": "dS0"}


def loss(args, gates, dO, dS_T, lib=None):
    o, ST = oracle.recurrence(args["q"], args["k"], args["v"], args["alpha"], args["b"],
                              args["w"], args["S0"], gates, lib=lib)
    return float((o * dO).sum() + (0.0 if dS_T is None else (ST * dS_T).sum()))


def finite_difference(args, gates, dO, dS_T, name, eps=1e-6, lib=None):
    x = args[name]
    fd = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        a = dict(args)
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        a[name] = xp
        lp = loss(a, gates, dO, dS_T, lib)
        a[name] = xm
        lm = loss(a, gates, dO, dS_T, lib)
        fd[idx] = (lp - lm) / (2 * eps)
    return fd


def fd_mismatch(gates, s0, dst, seed, lib=None, T=5, dk=3, dv=4):
    """Largest |analytic - finite difference| / (1 + max|fd|) over every input."""
    rng = np.random.default_rng(seed)
    q, k, v, a, b, w, S0 = rand_inputs(rng, 1, T, 2, dk, dv, gates, s0=s0, k_unit=False)
    args = dict(q=q, k=k, v=v, alpha=a, b=b, w=w, S0=S0 if s0 else np.zeros((1, 2, dk, dv)))
    dO = rng.standard_normal(v.shape)
    dS_T = rng.standard_normal((1, 2, dk, dv)) if dst else None
    g = oracle.recurrence_bwd(q, k, v, a, b, w, args["S0"], gates, dO, dS_T, lib=lib)
    worst = 0.0
    for name, x in args.items():
        if x is None:
            assert g[GRAD_OF[name]] is None
            continue
        fd = finite_difference(args, gates, dO, dS_T, name, lib=lib)
        worst = max(worst, float(np.abs(fd - g[GRAD_OF[name]]).max() / (1 + np.abs(fd).max())))
    return worst


@pytest.mark.parametrize("gates", [
    {"alpha": "channel", "b": "channel", "w": "channel"},    # Gated DeltaNet-2
    {"alpha": "channel", "b": "scalar", "w": "tied"},        # KDA
    {"alpha": "scalar", "b": "scalar", "w": "tied"},         # Gated DeltaNet
    {"alpha": "none", "b": "scalar", "w": "tied"},           # DeltaNet
    {"alpha": "channel", "b": "none", "w": "none"},          # GLA (erase-free)
    {"alpha": "scalar", "b": "channel", "w": "scalar"},
    {"alpha": "none", "b": "none", "w": "none"},             # linear attention
])
@pytest.mark.parametrize("s0,dst", [(True, True), (False, False)])
def test_gradient_equals_finite_difference(gates, s0, dst):
    assert fd_mismatch(gates, s0, dst, seed=zlib.crc32(f"{gates}{s0}".encode()) % 1000) < 1e-7


def test_linear_attention_closed_form():
    """alpha = 1, b = 0, w = 1, S0 = 0: o = tril(Q K^T) V, so
    dQ = tril(dO V^T) K, dK = tril(dO V^T)^T Q, dV = tril(Q K^T)^T dO."""
    rng = np.random.default_rng(3)
    T, dk, dv = 37, 6, 5
    q, k, v = (rng.standard_normal((1, T, 1, d)) for d in (dk, dk, dv))
    dO = rng.standard_normal((1, T, 1, dv))
    none = {"alpha": "none", "b": "none", "w": "none"}
    g = oracle.recurrence_bwd(q, k, v, gates=none, dO=dO)
    Q, K, V, D = q[0, :, 0], k[0, :, 0], v[0, :, 0], dO[0, :, 0]
    np.testing.assert_allclose(g["dq"][0, :, 0], np.tril(D @ V.T) @ K, atol=1e-11)
    np.testing.assert_allclose(g["dk"][0, :, 0], np.tril(D @ V.T).T @ Q, atol=1e-11)
    np.testing.assert_allclose(g["dv"][0, :, 0], np.tril(Q @ K.T).T @ D, atol=1e-11)
    np.testing.assert_allclose(g["dS0"][0, 0], Q.T @ D, atol=1e-11)


def test_erase_free_initial_state_gradient_closed_form():
    """b = 0: S_t = Diag(gamma_t) S0 + (terms without S0), gamma_t the running
    product of alpha, so dS0 = sum_t (q_t . gamma_t)^T dO_t + Diag(gamma_T) dS_T
    ("Recurrent Memory", section 04: survival factor of a stored entry)."""
    rng = np.random.default_rng(4)
    T, dk, dv = 23, 5, 4
    gates = {"alpha": "channel", "b": "none", "w": "channel"}
    q, k, v, a, b, w, S0 = rand_inputs(rng, 1, T, 1, dk, dv, gates, s0=True)
    dO = rng.standard_normal(v.shape)
    dS_T = rng.standard_normal(S0.shape)
    g = oracle.recurrence_bwd(q, k, v, a, None, w, S0, gates, dO, dS_T)
    gamma = np.cumprod(a[0, :, 0], axis=0)
    want = (q[0, :, 0] * gamma).T @ dO[0, :, 0] + gamma[-1][:, None] * dS_T[0, 0]
    np.testing.assert_allclose(g["dS0"][0, 0], want, atol=1e-11)


def test_zero_length_gradient_is_dS_T():
    rng = np.random.default_rng(5)
    dS_T = rng.standard_normal((2, 3, 4, 5))
    z = lambda *s: np.zeros(s)
    g = oracle.recurrence_bwd(z(2, 0, 3, 4), z(2, 0, 3, 4), z(2, 0, 3, 5), gates={},
                              S0=z(2, 3, 4, 5), dO=z(2, 0, 3, 5), dS_T=dS_T)
    np.testing.assert_array_equal(g["dS0"], dS_T)


@pytest.mark.parametrize("gates", [
    {"alpha": "channel", "b": "channel", "w": "channel"},
    {"alpha": "scalar", "b": "scalar", "w": "tied"},
    {"alpha": "channel", "b": "none", "w": "none"},
    {"alpha": "none", "b": "scalar", "w": "tied"},
])
@pytest.mark.parametrize("T", [1, 8, 21])
def test_chunkwise_route_agrees(gates, T):
    """The chunkwise route (masked products per chunk from the scans' r and
    dr, decay gradient through the running product's logarithm) equals the
    reverse token loop, including ragged final chunks."""
    rng = np.random.default_rng(100 + T)
    q, k, v, a, b, w, S0 = rand_inputs(rng, 2, T, 2, 5, 4, gates, s0=True, k_unit=False)
    dO = rng.standard_normal(v.shape)
    dS_T = rng.standard_normal(S0.shape)
    ref = oracle.recurrence_bwd(q, k, v, a, b, w, S0, gates, dO, dS_T)
    got = oracle.chunkwise_bwd(q, k, v, a, b, w, S0, gates, dO, dS_T, chunk=8)
    for n, x in ref.items():
        if x is None:
            assert got[n] is None, n
        else:
            np.testing.assert_allclose(got[n], x, atol=1e-10 * max(1.0, np.abs(x).max()), err_msg=n)


def _chunk_state_gradient(q, k, alpha, beta, dO, dS_T, chunk):
    """The Gated DeltaNet state-gradient recurrence G_t = q_t^T dO_t +
    alpha_{t+1} (I - beta_{t+1} k_{t+1}^T k_{t+1}) G_{t+1}, taken a chunk at a
    time in reverse (the algebra of the tensor-core gradient pass): with g the
    decay product from the chunk's start, A the masked key products, Aq the
    masked q k^T block and Y_j = k_j G_j,
      (I + A)^T Y = Diag(g_{n-1}/g) K G_in + Aq^T dO,
      G_out = g_{n-1} G_in + (Diag(g) Q)^T dO - (Diag(beta g) K)^T Y.
    One head: q, k [T, d_k]; alpha, beta [T]; dO [T, d_v]. Returns dv = beta Y
    per token and dS0 = the final G_out."""
    T = q.shape[0]
    G = dS_T.copy()
    dv = np.zeros((T, dO.shape[1]))
    for t0 in reversed(range(0, T, chunk)):
        K, Q, D = k[t0:t0 + chunk], q[t0:t0 + chunk], dO[t0:t0 + chunk]
        b = beta[t0:t0 + chunk]
        g = np.cumprod(alpha[t0:t0 + chunk])
        ratio = g[:, None] / g[None, :]
        A = np.tril(b[:, None] * (K @ K.T) * ratio, -1)
        Aq = np.tril((Q @ K.T) * ratio)
        Y = np.linalg.solve((np.eye(len(g)) + A).T, (g[-1] / g)[:, None] * (K @ G) + Aq.T @ D)
        dv[t0:t0 + chunk] = b[:, None] * Y
        G = g[-1] * G + (g[:, None] * Q).T @ D - (b[:, None] * g[:, None] * K).T @ Y
    return dv, G


@pytest.mark.parametrize("T", [1, 8, 21])
def test_chunk_state_gradient_algebra_agrees(T):
    """The chunk form of the state-gradient recurrence (what the tensor-core
    gradient pass computes) gives the reverse token loop's dv and dS0 exactly,
    ragged final chunks included."""
    gates = {"alpha": "scalar", "b": "scalar", "w": "tied"}
    rng = np.random.default_rng(300 + T)
    q, k, v, a, b, w, S0 = rand_inputs(rng, 1, T, 1, 5, 4, gates, s0=True, k_unit=False)
    dO = rng.standard_normal(v.shape)
    dS_T = rng.standard_normal(S0.shape)
    ref = oracle.recurrence_bwd(q, k, v, a, b, w, S0, gates, dO, dS_T)
    dv, dS0 = _chunk_state_gradient(q[0, :, 0], k[0, :, 0], a[0, :, 0], b[0, :, 0], dO[0, :, 0],
                                    dS_T[0, 0], chunk=8)
    np.testing.assert_allclose(dv, ref["dv"][0, :, 0], atol=1e-10 * np.abs(ref["dv"]).max())
    np.testing.assert_allclose(dS0, ref["dS0"][0, 0], atol=1e-10 * np.abs(ref["dS0"]).max())
