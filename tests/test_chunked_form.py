"""The chunked equations, checked against the oracle in fp64 (CPU).

The CUDA prefill engines implement the chunked form of the recurrence (Kimi
Linear summary, es.news.hada.io/topic?id=31936, section "Algoritmo paralelo
por chunks": fixed-length chunks that start from the previous chunk's last
state, the WY representation of the rank-1 updates, the UT transform with the
lower-triangular inverse taken row by row by forward substitution, a matrix
state update per chunk, and outputs that add the inter-chunk recurrent part to
the intra-chunk parallel part). This file writes those equations out in plain
NumPy, in exact (un-anchored) form, and checks that they reach the oracle's
result: the forward against ``oracle.forward``, and the chunked backward --
the same chunks in reverse, with the state gradient as the sequential chain --
against ``oracle.grad.backward``. It shares no code with the CUDA sources.

Per chunk (g = in-chunk prefix sum of log alpha, gamma = e^{g_C}):
    A_ij = beta_i k_i.(k_j e^{g_i - g_j}) (j < i),  P_ij = q_i.(k_j e^{g_i - g_j}) (j <= i)
    T = (I + A)^{-1} Diag(beta),  W = T (K e^{g}),  U' = T V
    U = U' - W S,  O = (Q e^{g}) S + P U,  S <- Diag(gamma) S + (K e^{g_C - g})^T U
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import grad


def unit_lower_inverse(A):
    """(I + A)^{-1} for strictly lower-triangular A, row by row by forward substitution."""
    n = A.shape[0]
    X = np.zeros((n, n))
    for i in range(n):
        X[i, i] = 1.0
        X[i, :i] = -A[i, :i] @ X[:i, :i]
    return X


def chunk_terms(qc, kc, vc, lc, bc):
    n = qc.shape[0]
    g = np.cumsum(lc, axis=0)
    D = np.exp(g[:, None, :] - g[None, :, :])                     # e^{g_i - g_j}, [i, j, channel]
    lower, lower_eq = np.tril(np.ones((n, n)), -1), np.tril(np.ones((n, n)))
    At = np.einsum("ic,jc,ijc->ij", kc, kc, D) * lower
    P = np.einsum("ic,jc,ijc->ij", qc, kc, D) * lower_eq
    X = unit_lower_inverse(At * bc[:, None])
    Tm = X * bc[None, :]
    Ks, Qs, Kb = kc * np.exp(g), qc * np.exp(g), kc * np.exp(g[-1] - g)
    return dict(g=g, At=At, P=P, X=X, T=Tm, Ks=Ks, Qs=Qs, Kb=Kb, W=Tm @ Ks, Up=Tm @ vc,
                gamma=np.exp(g[-1]), lower=lower, lower_eq=lower_eq)


def chunked_forward(q, k, v, la, be, S0, C):
    S = S0.copy()
    out = np.zeros((q.shape[0], v.shape[1]))
    states = []
    for t0 in range(0, q.shape[0], C):
        sl = slice(t0, min(t0 + C, q.shape[0]))
        c = chunk_terms(q[sl], k[sl], v[sl], la[sl], be[sl])
        states.append(S.copy())
        U = c["Up"] - c["W"] @ S
        out[sl] = c["Qs"] @ S + c["P"] @ U
        S = c["gamma"][:, None] * S + c["Kb"].T @ U
    return out, S, states


def chunked_backward(q, k, v, la, be, S0, dO, dST, C):
    _, _, states = chunked_forward(q, k, v, la, be, S0, C)
    res = {n: np.zeros_like(a) for n, a in (("dq", q), ("dk", k), ("dv", v), ("dlog_alpha", la),
                                             ("dbeta", be))}
    dS = dST.copy()                                     # gradient of the state leaving the chunk
    starts = list(range(0, q.shape[0], C))
    for ci in reversed(range(len(starts))):
        sl = slice(starts[ci], min(starts[ci] + C, q.shape[0]))
        S, c = states[ci], chunk_terms(q[sl], k[sl], v[sl], la[sl], be[sl])
        vc, do = v[sl], dO[sl]
        U = c["Up"] - c["W"] @ S
        # the sequential part: the state gradient through one chunk
        dU = c["P"].T @ do + c["Kb"] @ dS
        dS_in = c["Qs"].T @ do + c["gamma"][:, None] * dS - c["W"].T @ dU
        # everything else is local to the chunk once dU, dS and S are known
        dQs, dP, dKb = do @ S.T, (do @ U.T) * c["lower_eq"], U @ dS.T
        dW = -dU @ S.T
        dT = dW @ c["Ks"].T + dU @ vc.T
        dKs = c["T"].T @ dW
        res["dv"][sl] = c["T"].T @ dU
        dX = dT * be[sl][None, :]
        dA = -(c["X"].T @ dX @ c["X"].T) * c["lower"]
        res["dbeta"][sl] = np.sum(dT * c["X"], axis=0) + np.sum(dA * c["At"], axis=1)
        dAt = dA * be[sl][:, None]
        g = c["g"]
        Kt, Kh, Qt = k[sl] * np.exp(g), k[sl] * np.exp(-g), q[sl] * np.exp(g)
        dKt, dQt = dAt @ Kh, dP @ Kh
        dKh = dAt.T @ Kt + dP.T @ Qt
        res["dk"][sl] = dKt * np.exp(g) + dKh * np.exp(-g) + dKs * np.exp(g) + dKb * np.exp(g[-1] - g)
        res["dq"][sl] = dQt * np.exp(g) + dQs * np.exp(g)
        dg = (dKt * Kt - dKh * Kh + dQt * Qt + dKs * c["Ks"] + dQs * c["Qs"] - dKb * c["Kb"])
        dg[-1] += np.sum(dS * S, axis=1) * c["gamma"] + np.sum(dKb * c["Kb"], axis=0)
        res["dlog_alpha"][sl] = np.cumsum(dg[::-1], axis=0)[::-1]
        dS = dS_in
    res["dS0"] = dS
    return res


def head_problem(T, d, dv, seed):
    rng = np.random.default_rng(seed)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)      # inputs the C oracle reads exactly
    q = f32(rng.standard_normal((T, d)))
    k = rng.standard_normal((T, d))
    k = f32(k / np.linalg.norm(k, axis=1, keepdims=True))
    v = f32(rng.standard_normal((T, dv)))
    la = f32(-np.log1p(np.exp(rng.standard_normal((T, d)))))
    be = f32(1.0 / (1.0 + np.exp(-rng.standard_normal(T))))
    S0 = 0.3 * rng.standard_normal((d, dv))
    return q, k, v, la, be, S0, rng.standard_normal((T, dv)), rng.standard_normal((d, dv))


CASES = [(64, 8, 6, 16, 0), (50, 8, 6, 16, 1), (130, 16, 8, 64, 2), (97, 12, 4, 32, 3), (5, 4, 4, 64, 4)]


@pytest.mark.parametrize("T,d,dv,C,seed", CASES)
def test_chunked_forward_equals_the_recurrence(T, d, dv, C, seed):
    q, k, v, la, be, S0, _, _ = head_problem(T, d, dv, seed)
    out, ST, _ = chunked_forward(q, k, v, la, be, S0, C)
    t = lambda a: torch.from_numpy(a[None, :, None].astype(np.float32))
    ref_o, ref_s = oracle.forward(t(q), t(k), t(v), t(la), torch.from_numpy(be[None, :, None].astype(np.float32)),
                                  torch.from_numpy(S0[None, None]))
    np.testing.assert_allclose(out, ref_o[0, :, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(ST, ref_s[0, 0], rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("T,d,dv,C,seed", CASES)
def test_chunked_backward_equals_the_reverse_recurrence(T, d, dv, C, seed):
    q, k, v, la, be, S0, dO, dST = head_problem(T, d, dv, seed)
    mine = chunked_backward(q, k, v, la, be, S0, dO, dST, C)
    e = lambda a: a[None, :, None]
    ref = grad.backward(e(q), e(k), e(v), e(la), e(be), e(dO), S0=S0[None, None], dS_T=dST[None, None])
    for n in ["dq", "dk", "dv", "dlog_alpha", "dbeta"]:
        np.testing.assert_allclose(mine[n], ref[n][0, :, 0], rtol=1e-9, atol=1e-10, err_msg=n)
    np.testing.assert_allclose(mine["dS0"], ref["dS0"][0, 0], rtol=1e-9, atol=1e-10)


def test_forward_substitution_inverts():
    rng = np.random.default_rng(0)
    A = np.tril(rng.standard_normal((20, 20)), -1)
    np.testing.assert_allclose(unit_lower_inverse(A) @ (np.eye(20) + A), np.eye(20), atol=1e-10)


def test_blocked_inverse_of_the_16_token_chunk():
    """The 16-token kernels solve (I + A)^{-1}, A = Diag(beta) At, in 8 x 8 blocks: the
    diagonal blocks by forward substitution, X10 = -X11 (A10 X00), X01 = 0. The same
    steps in NumPy, on the At of real chunks (strong and weak gates), equal the dense
    inverse."""
    rng = np.random.default_rng(3)
    for gate_scale in (0.05, 1.0, 4.0):
        kc = rng.standard_normal((16, 8))
        kc /= np.linalg.norm(kc, axis=1, keepdims=True)
        lc = -gate_scale * np.log1p(np.exp(rng.standard_normal((16, 8))))
        bc = 1.0 / (1.0 + np.exp(-rng.standard_normal(16)))
        At = chunk_terms(kc, kc, kc, lc, bc)["At"]
        X00 = unit_lower_inverse(bc[:8, None] * At[:8, :8])
        X11 = unit_lower_inverse(bc[8:, None] * At[8:, 8:])
        Y = (bc[8:, None] * At[8:, :8]) @ X00
        X = np.zeros((16, 16))
        X[:8, :8], X[8:, 8:], X[8:, :8] = X00, X11, -X11 @ Y
        np.testing.assert_allclose(X, np.linalg.inv(np.eye(16) + bc[:, None] * At), rtol=1e-12, atol=1e-13)


def chunked_chain(q, k, v, la, be, S_init, C):
    """The chunked chain from S_init; returns outputs and final state (columns of
    S_init evolve independently, so S_init may be any d x n matrix)."""
    out, S, _ = chunked_forward(q, k, v, la, be, S_init, C)
    return out, S


@pytest.mark.parametrize("T,split,C,seed", [(256, 128, 64, 0), (200, 64, 32, 1), (131, 64, 64, 2)])
def test_sequence_split_with_output_correction(T, split, C, seed):
    """Two segments of one head computed independently, then joined.

    The second segment runs its chain twice, side by side: from a zero state
    with values V (outputs O0, final state S0_end), and from the identity with
    zero values (its "outputs" are Y = Qs M - P W M, with M the transition
    product up to each chunk, and its final state is M_end). With the first
    segment's final state S_mid:
        O = O0 + Y S_mid,     S_T = S0_end + M_end S_mid.
    Both halves of the augmented state [0 | I] (values [V | 0]) are value
    columns of one chain, so each is the engine's chain as it stands."""
    d, dv = 8, 6
    q, k, v, la, be, S0, _, _ = head_problem(T, d, dv, seed)
    first = slice(0, split)
    second = slice(split, T)
    o1, S_mid = chunked_chain(q[first], k[first], v[first], la[first], be[first], S0, C)
    aug = np.concatenate([np.zeros((d, dv)), np.eye(d)], axis=1)          # [0 | I]
    v_aug = np.concatenate([v[second], np.zeros((T - split, d))], axis=1)   # [V | 0]
    o_aug, S_aug = chunked_chain(q[second], k[second], v_aug, la[second], be[second], aug, C)
    O0, Y = o_aug[:, :dv], o_aug[:, dv:]
    o2 = O0 + Y @ S_mid
    ST = S_aug[:, :dv] + S_aug[:, dv:] @ S_mid
    out = np.concatenate([o1, o2])
    t = lambda a: torch.from_numpy(a[None, :, None].astype(np.float32))
    ref_o, ref_s = oracle.forward(t(q), t(k), t(v), t(la), torch.from_numpy(be[None, :, None].astype(np.float32)),
                                  torch.from_numpy(S0[None, None]))
    np.testing.assert_allclose(out, ref_o[0, :, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(ST, ref_s[0, 0], rtol=1e-9, atol=1e-10)


# --- the anchored factorisations of the intra-chunk products -----------------------------
# The tensor-core engine never forms e^{g_i - g_j} per term; it splits the factor so that
# every piece stays in floating-point range (the summary's secondary chunking, section
# "Menor cantidad de operaciones que DPLR general"). These checks write both of its
# factorisations out in NumPy and compare them with the direct products above.

def direct_products(qc, kc, lc):
    g = np.cumsum(lc, axis=0)
    D = np.exp(np.minimum(g[:, None, :] - g[None, :, :], 0.0))   # j > i is masked below
    n = qc.shape[0]
    return (np.einsum("ic,jc,ijc->ij", kc, kc, D) * np.tril(np.ones((n, n)), -1),
            np.einsum("ic,jc,ijc->ij", qc, kc, D) * np.tril(np.ones((n, n))))


def one_anchor_products(qc, kc, lc):
    """Factors anchored at the chunk midpoint: rows e^{g - g_C/2}, columns e^{g_C/2 - g}."""
    g = np.cumsum(lc, axis=0)
    ga = 0.5 * g[-1]
    E, F = np.exp(g - ga), np.exp(ga - g)
    n = qc.shape[0]
    return (((kc * E) @ (kc * F).T) * np.tril(np.ones((n, n)), -1),
            ((qc * E) @ (kc * F).T) * np.tril(np.ones((n, n))))


def subchunk_products(qc, kc, lc, S=16, range_log=-87.0, clamp_log=-10.0):
    """16-token sub-chunks: a block (I, J < I) as e^{g_i - G_I} e^{G_I - G_{J+1}} e^{G_{J+1} - g_j}
    (G_I = g at the end of sub-chunk I-1; every factor <= 1); a diagonal block anchored at
    the sub-chunk's 8th token m, e^{g_i - g_m} e^{g_m - g_j}, with the factors of a channel
    whose sub-chunk decays below e^{range_log} taken from log alpha clamped at clamp_log."""
    n, d = qc.shape
    g = np.cumsum(lc, axis=0)
    nb = n // S
    G = np.zeros((nb + 1, d))
    for I in range(nb):
        G[I + 1] = g[S * I + S - 1]
    A, P = np.zeros((n, n)), np.zeros((n, n))
    for I in range(nb):
        ri = slice(S * I, S * I + S)
        for J in range(I):
            rj = slice(S * J, S * J + S)
            row = np.exp(g[ri] - G[I])               # e^{g_i - G_I}
            mid = np.exp(G[I] - G[J + 1])            # e^{G_I - G_{J+1}}, per channel
            col = np.exp(G[J + 1] - g[rj])           # e^{G_{J+1} - g_j}
            A[ri, rj] = (kc[ri] * row * mid) @ (kc[rj] * col).T
            P[ri, rj] = (qc[ri] * row * mid) @ (kc[rj] * col).T
        gl = g[ri] - G[I]                            # prefix inside the sub-chunk
        tot = gl[-1]
        far = tot < range_log
        glc = np.cumsum(np.maximum(lc[ri], clamp_log), axis=0)
        gl_use = np.where(far[None, :], glc, gl)
        m = gl_use[7]
        rowf, colf = np.exp(gl_use - m), np.exp(m - gl_use)
        A[ri, ri] = np.tril((kc[ri] * rowf) @ (kc[ri] * colf).T, -1)
        P[ri, ri] = np.tril((qc[ri] * rowf) @ (kc[ri] * colf).T)
    return A, P


def _chunk_inputs(seed, gate):
    rng = np.random.default_rng(seed)
    n, d = 64, 24
    q, k = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    la = -np.log1p(np.exp(rng.standard_normal((n, d))))
    if gate == "steep":           # -5 per token: sub-chunks at e^-80, inside the anchors' range
        la[:, 0::6], la[:, 1::6] = -5.0, 0.0
    elif gate == "strong":        # -12 per token on some channels: sub-chunks at e^-192
        la[:, 0::6], la[:, 1::6], la[:, 2::6] = -4.0, 0.0, -12.0
    elif gate == "edge":          # every sub-chunk at e^-39.8: the one-anchor path's limit
        la[:] = -2.49
    elif gate == "far":           # sub-chunks below e^-87 on some channels: the clamped fallback
        la[:, 0::3] = -30.0
    return q, k, la


@pytest.mark.parametrize("gate,seed", [("softplus", 0), ("steep", 1), ("edge", 2)])
def test_subchunk_factorisation_is_exact(gate, seed):
    q, k, la = _chunk_inputs(seed, gate)
    A0, P0 = direct_products(q, k, la)
    A1, P1 = subchunk_products(q, k, la)
    np.testing.assert_allclose(A1, A0, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(P1, P0, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("gate,seed", [("softplus", 3), ("edge", 4)])
def test_one_anchor_factorisation_is_exact_in_range(gate, seed):
    q, k, la = _chunk_inputs(seed, gate)
    assert (np.cumsum(la, 0)[15::16] - np.vstack([np.zeros((1, la.shape[1])), np.cumsum(la, 0)[15::16][:-1]])).min() >= -40
    A0, P0 = direct_products(q, k, la)
    A1, P1 = one_anchor_products(q, k, la)
    np.testing.assert_allclose(A1, A0, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(P1, P0, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("gate,seed", [("far", 5), ("strong", 6)])
def test_clamped_fallback_changes_only_tiny_products(gate, seed):
    """With log alpha = -30 or -12 on some channels (sub-chunks far below e^-87), the clamped
    factors change only products that are below e^-10 before and after: the difference is
    at most e^-10 times the sum of |k_i k_j| over the channels that take the fallback."""
    q, k, la = _chunk_inputs(seed, gate)
    A0, P0 = direct_products(q, k, la)
    A1, P1 = subchunk_products(q, k, la)
    g = np.cumsum(la, axis=0)
    far = np.zeros(la.shape[1], dtype=bool)
    for I in range(4):
        far |= (g[16 * I + 15] - (g[16 * I - 1] if I else 0.0)) < -87.0
    assert far.any()
    bound_a = 2 * np.exp(-10.0) * (np.abs(k[:, far]) @ np.abs(k[:, far]).T)
    bound_p = 2 * np.exp(-10.0) * (np.abs(q[:, far]) @ np.abs(k[:, far]).T)
    assert np.all(np.abs(A1 - A0) <= bound_a + 1e-15)
    assert np.all(np.abs(P1 - P0) <= bound_p + 1e-15)
    # and the one-anchor form is out of range there: its factors overflow
    with np.errstate(over="ignore", invalid="ignore"):
        A2, _ = one_anchor_products(q, k, la)
    assert not np.all(np.isfinite(A2)) or np.abs(A2 - A0).max() > 1e-6
