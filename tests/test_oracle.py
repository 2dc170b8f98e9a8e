"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test compares the oracle (the token-by-token KDA recurrence in C) with an
independent statement of a special case, a closed form, a brute-force
evaluation or an invariant. Sources (Kimi Linear summary,
es.news.hada.io/topic?id=31936):

* "De la atencion lineal a Gated DeltaNet": linear attention as an additive
  fast-weight state; DeltaNet's delta rule (rank-1 generalised Householder
  update); GDN's scalar forget gate.
* "Control fino de memoria en Kimi Delta Attention": the per-channel
  diagonal gate (GLA-like granularity) inside the delta rule.
* "Algoritmo paralelo por chunks": each chunk starts from the last state of
  the previous one (split-run equivalence).
* "Configuracion del modelo Kimi Linear": L2-normalised keys (the Householder
  spectrum check).
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(B, T, H, dk, dv, seed, gate_scale=1.0, unit_k=True):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, T, H, dk))
    k = g.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = g.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-g.standard_normal((B, T, H))))
    log_alpha = -gate_scale * np.log1p(np.exp(g.standard_normal((B, T, H, dk))))
    S0 = g.standard_normal((B, H, dk, dv))
    f = lambda a: a.astype(np.float32)
    return f(q), f(k), f(v), f(log_alpha), f(beta), S0


def _d(a):
    return np.asarray(a, dtype=np.float64)


# --- S1: plain linear attention -------------------------------------------------

def test_linear_attention_special_case():
    """alpha = 1, no erase, write weight 1, S0 = 0: o = (Q K^T masked causal) V."""
    B, T, H, dk, dv = 2, 19, 3, 5, 7
    q, k, v, _, _, _ = _rand(B, T, H, dk, dv, 1, unit_k=False)
    zeros_gate = np.zeros((B, T, H, dk), np.float32)
    out, st = oracle.forward(q, k, v, zeros_gate, np.zeros((B, T, H), np.float32),
                             beta_write=np.ones((B, T, H), np.float32))
    for b in range(B):
        for h in range(H):
            Q, K, V = _d(q[b, :, h]), _d(k[b, :, h]), _d(v[b, :, h])
            expect = np.tril(Q @ K.T) @ V
            np.testing.assert_allclose(out[b, :, h], expect, rtol=0, atol=1e-12)
            np.testing.assert_allclose(st[b, h], K.T @ V, rtol=0, atol=1e-12)


# --- S2: gated linear attention (channel-wise gate, no erase) --------------------

def test_gated_linear_attention_closed_form():
    """No erase, write weight 1: o_t = sum_{j<=t} (q_t*exp(g_t-g_j)).k_j v_j + (q_t*exp(g_t))^T S0."""
    B, T, H, dk, dv = 1, 13, 2, 6, 4
    q, k, v, la, _, S0 = _rand(B, T, H, dk, dv, 2, gate_scale=0.3)
    out, st = oracle.forward(q, k, v, la, np.zeros((B, T, H), np.float32), S0=S0,
                             beta_write=np.ones((B, T, H), np.float32))
    for h in range(H):
        g = np.cumsum(_d(la[0, :, h]), axis=0)            # g_t = sum_{s<=t} log a_s
        Q, K, V = _d(q[0, :, h]), _d(k[0, :, h]), _d(v[0, :, h])
        for t in range(T):
            coeff = np.array([np.sum(Q[t] * np.exp(g[t] - g[j]) * K[j]) for j in range(t + 1)])
            expect = coeff @ V[: t + 1] + (Q[t] * np.exp(g[t])) @ S0[0, h]
            np.testing.assert_allclose(out[0, t, h], expect, rtol=1e-12, atol=1e-12)
        ST = np.exp(g[-1])[:, None] * S0[0, h] + sum(
            np.outer(np.exp(g[-1] - g[j]) * K[j], V[j]) for j in range(T))
        np.testing.assert_allclose(st[0, h], ST, rtol=1e-12, atol=1e-12)


# --- S3: scalar-gated GDN -------------------------------------------------------------

def test_gdn_scalar_gate_special_case():
    """Gate equal across channels: S_t = a_t (I - b k k^T) S_{t-1} + b k v^T (dense matrices)."""
    B, T, H, dk, dv = 1, 17, 2, 6, 5
    q, k, v, _, beta, S0 = _rand(B, T, H, dk, dv, 3)
    rng = np.random.default_rng(33)
    scalar = (-np.log1p(np.exp(rng.standard_normal((B, T, H))))).astype(np.float32)
    la = np.repeat(scalar[..., None], dk, axis=-1)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk, vv, qq = _d(k[0, t, h]), _d(v[0, t, h]), _d(q[0, t, h])
            b, a = float(beta[0, t, h]), float(np.exp(_d(scalar[0, t, h])))
            S = a * (np.eye(dk) - b * np.outer(kk, kk)) @ S + b * np.outer(kk, vv)
            np.testing.assert_allclose(out[0, t, h], S.T @ qq, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(st[0, h], S, rtol=1e-11, atol=1e-12)


# --- S4: DeltaNet with basis keys -------------------------------------------------

def test_deltanet_basis_keys_overwrite_rows():
    """alpha = 1, k_t = e_i: the update sets row i to (1-b) S_i + b v_t and leaves the rest."""
    B, T, H, dk, dv = 1, 23, 1, 4, 3
    rng = np.random.default_rng(4)
    idx = rng.integers(0, dk, size=T)
    k = np.zeros((B, T, H, dk), np.float32)
    k[0, np.arange(T), 0, idx] = 1.0
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    beta = rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv))
    out, st = oracle.forward(q, k, v, np.zeros((B, T, H, dk), np.float32), beta, S0=S0)
    S = S0[0, 0].copy()
    for t in range(T):
        b = float(beta[0, t, 0])
        S[idx[t]] = (1.0 - b) * S[idx[t]] + b * _d(v[0, t, 0])
        np.testing.assert_allclose(out[0, t, 0], S.T @ _d(q[0, t, 0]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(st[0, 0], S, rtol=0, atol=1e-13)


# --- S5: beta = 0 (literal) ------------------------------------------------------------

def test_beta_zero_is_pure_decay():
    """beta = 0: S_T = Diag(prod a) S0 and o_t = S0^T (q_t * prod_{s<=t} a_s)."""
    B, T, H, dk, dv = 2, 11, 2, 5, 6
    q, k, v, la, _, S0 = _rand(B, T, H, dk, dv, 5)
    out, st = oracle.forward(q, k, v, la, np.zeros((B, T, H), np.float32), S0=S0)
    for b in range(B):
        for h in range(H):
            gam = np.cumprod(np.exp(_d(la[b, :, h])), axis=0)    # prod_{s<=t} a_s
            for t in range(T):
                np.testing.assert_allclose(out[b, t, h], S0[b, h].T @ (_d(q[b, t, h]) * gam[t]),
                                           rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(st[b, h], gam[-1][:, None] * S0[b, h], rtol=1e-12, atol=1e-14)


# --- B1: brute-force products of dense transition matrices -------------------------

@pytest.mark.parametrize("T,dk,dv", [(1, 3, 2), (7, 4, 6), (16, 8, 5)])
def test_bruteforce_transition_products(T, dk, dv):
    """S_t = M_t..M_1 S0 + sum_j M_t..M_{j+1} b_j k_j v_j^T with M_t = (I - b k k^T) Diag(a)."""
    B, H = 1, 2
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 100 + T)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    for h in range(H):
        M = []
        for t in range(T):
            kk = _d(k[0, t, h])
            M.append((np.eye(dk) - float(beta[0, t, h]) * np.outer(kk, kk))
                     @ np.diag(np.exp(_d(la[0, t, h]))))
        for t in range(T):
            prod_all = np.eye(dk)
            for s in range(t + 1):
                prod_all = M[s] @ prod_all                      # M_t ... M_1
            S = prod_all @ S0[0, h]
            for j in range(t + 1):
                P = np.eye(dk)
                for s in range(j + 1, t + 1):
                    P = M[s] @ P                                # M_t ... M_{j+1}
                S = S + P @ (float(beta[0, j, h]) * np.outer(_d(k[0, j, h]), _d(v[0, j, h])))
            np.testing.assert_allclose(out[0, t, h], S.T @ _d(q[0, t, h]), rtol=1e-11, atol=1e-12)
            if t == T - 1:
                np.testing.assert_allclose(st[0, h], S, rtol=1e-11, atol=1e-12)


# --- hand-worked golden fixture ------------------------------------------------

def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *nums = line.split()
                vals[key] = np.array([float(x) for x in nums])
    return vals


def test_handworked_example():
    g = _read_golden("kda_handworked_d2.txt")
    T, d = 2, 2
    stack = lambda name, n: np.stack([g[f"{name}_{t + 1}"] for t in range(T)]).reshape(1, T, 1, n)
    q = stack("q", d).astype(np.float32)
    k = stack("k", d).astype(np.float32)
    v = stack("v", d).astype(np.float32)
    la = stack("log_alpha", d).astype(np.float32)
    beta = stack("beta", 1).reshape(1, T, 1).astype(np.float32)
    S0 = g["S0"].reshape(1, 1, d, d)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    np.testing.assert_allclose(out[0, 0, 0], g["expect_o_1"], rtol=0, atol=1e-6)
    np.testing.assert_allclose(out[0, 1, 0], g["expect_o_2"], rtol=0, atol=1e-6)
    np.testing.assert_allclose(st[0, 0].reshape(-1), g["expect_S_T"], rtol=0, atol=1e-6)


# --- invariants ---------------------------------------------------------------------

def test_householder_spectrum_and_norm_bound():
    """With |k| = 1, I - b k k^T has eigenvalues {1 (d-1 times), 1-b}; hence, with
    a <= 1, |S_t|_F <= |S_{t-1}|_F + b |k| |v_t| along the oracle's trajectory."""
    B, T, H, dk, dv = 1, 12, 1, 6, 4
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 7)
    for t in range(T):
        kk = _d(k[0, t, 0])
        kk = kk / np.linalg.norm(kk)
        ev = np.sort(np.linalg.eigvalsh(np.eye(dk) - float(beta[0, t, 0]) * np.outer(kk, kk)))
        np.testing.assert_allclose(ev, np.sort([1.0] * (dk - 1) + [1.0 - float(beta[0, t, 0])]),
                                   atol=1e-12)
    prev = S0[0, 0]
    for t in range(T):
        _, st = oracle.forward(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], la[:, t:t + 1],
                               beta[:, t:t + 1], S0=prev[None, None])
        cur = st[0, 0]
        bound = np.linalg.norm(prev) + float(beta[0, t, 0]) * np.linalg.norm(_d(k[0, t, 0])) \
            * np.linalg.norm(_d(v[0, t, 0]))
        assert np.linalg.norm(cur) <= bound + 1e-12
        prev = cur


def test_value_column_permutation():
    B, T, H, dk, dv = 2, 9, 2, 4, 6
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 8)
    perm = np.random.default_rng(0).permutation(dv)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    out_p, st_p = oracle.forward(q, k, v[..., perm], la, beta, S0=S0[..., perm])
    np.testing.assert_array_equal(out_p, out[..., perm])
    np.testing.assert_array_equal(st_p, st[..., perm])


def test_head_and_batch_permutation():
    B, T, H, dk, dv = 3, 6, 4, 3, 3
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 9)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    hp, bp = np.array([2, 0, 3, 1]), np.array([1, 2, 0])
    p = lambda a: a[bp][:, :, hp]
    out2, st2 = oracle.forward(p(q), p(k), p(v), p(la), p(beta), S0=S0[bp][:, hp])
    np.testing.assert_array_equal(out2, p(out))
    np.testing.assert_array_equal(st2, st[bp][:, hp])


@pytest.mark.parametrize("T1", [1, 5, 16])
def test_split_run_equivalence(T1):
    """Running T1 tokens, then the rest from S_T, equals one run (each chunk starts
    from the previous chunk's last state)."""
    B, T, H, dk, dv = 1, 21, 2, 5, 3
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 10)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    s = slice(0, T1)
    r = slice(T1, T)
    o1, s1 = oracle.forward(q[:, s], k[:, s], v[:, s], la[:, s], beta[:, s], S0=S0)
    o2, s2 = oracle.forward(q[:, r], k[:, r], v[:, r], la[:, r], beta[:, r], S0=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(s2, st, rtol=0, atol=1e-13)


def test_bf16_inputs_widen_exactly():
    B, T, H, dk, dv = 1, 8, 2, 4, 4
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 11)
    qb, kb, vb = (torch.from_numpy(x).to(torch.bfloat16) for x in (q, k, v))
    out_b, st_b = oracle.forward(qb, kb, vb, la, beta, S0=S0)
    out_f, st_f = oracle.forward(qb.float(), kb.float(), vb.float(), la, beta, S0=S0)
    np.testing.assert_array_equal(out_b, out_f)
    np.testing.assert_array_equal(st_b, st_f)


def test_head_subset_and_empty():
    B, T, H, dk, dv = 2, 7, 3, 4, 5
    q, k, v, la, beta, S0 = _rand(B, T, H, dk, dv, 12)
    out, st = oracle.forward(q, k, v, la, beta, S0=S0)
    out_s, st_s = oracle.forward(q, k, v, la, beta, S0=S0, heads=[4, 1])
    for bh in (4, 1):
        b, h = divmod(bh, H)
        np.testing.assert_array_equal(out_s[b, :, h], out[b, :, h])
        np.testing.assert_array_equal(st_s[b, h], st[b, h])
    assert np.isnan(out_s[0, :, 0]).all()
    # T = 0: the state passes through unchanged
    e = slice(0, 0)
    o0, s0 = oracle.forward(q[:, e], k[:, e], v[:, e], la[:, e], beta[:, e], S0=S0)
    assert o0.shape == (B, 0, H, dv)
    np.testing.assert_array_equal(s0, S0)


def test_decode_step_matches_one_token_forward():
    N, H, dk, dv = 5, 2, 4, 3
    q, k, v, la, beta, _ = _rand(N, 1, H, dk, dv, 13)
    rng = np.random.default_rng(14)
    state = rng.standard_normal((7, H, dk, dv)).astype(np.float32)
    slot = np.array([6, 0, 3, 2, 5])
    t = lambda a: torch.from_numpy(a[:, 0])
    out, new = oracle.decode_step(t(q), t(k), t(v), t(la), t(beta), torch.from_numpy(state), slot=slot)
    o_ref, s_ref = oracle.forward(q, k, v, la, beta, S0=state[slot].astype(np.float64))
    np.testing.assert_array_equal(out, o_ref[:, 0])
    np.testing.assert_array_equal(new, s_ref)
