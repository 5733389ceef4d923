"""Pins for the fp64 KDA oracle against facts fixed by the Chimera paper and by
mathematics, independent of the oracle's own code.

The scan being pinned is Eq. 14 of the paper (section 3.3, pchao.org translation; the
agifrontier summary gives the parenthesised LaTeX form):
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
read out as o_t = S_t^T q_t with S_t the state after token t (same section).
Each test is chosen so that a plausible slip in the oracle (dropped decay, erase
applied before the decay, wrong sign, transposed state, readout before the update,
missing S0) fails at least one of them.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _rand_unit(rng, shape):
    z = rng.standard_normal(shape)
    return z / np.linalg.norm(z, axis=-1, keepdims=True)


# --------------------------------------------------------------------------------------
# 1. Exact rational brute force: the closed-form solution of the linear recurrence,
#    S_t = A_t...A_1 S0 + sum_s A_t...A_{s+1} beta_s k_s v_s^T,
#    A_r = (I - beta_r k_r k_r^T) Diag(alpha_r), evaluated in exact rationals.
# --------------------------------------------------------------------------------------

def _mat_mul(A, B):
    return [[sum(A[i][p] * B[p][j] for p in range(len(B))) for j in range(len(B[0]))]
            for i in range(len(A))]


def _mat_add(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def _ident(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def _brute_force_states(alpha, beta, k, v, S0):
    T, dk = len(alpha), len(alpha[0])
    dv = len(v[0])
    A = []
    for r in range(T):
        erase = [[(Fraction(int(i == j)) - beta[r] * k[r][i] * k[r][j]) for j in range(dk)]
                 for i in range(dk)]
        diag = [[alpha[r][i] if i == j else Fraction(0) for j in range(dk)] for i in range(dk)]
        A.append(_mat_mul(erase, diag))
    states = []
    for t in range(T):
        # product A_t ... A_1 applied to S0
        P = _ident(dk)
        for r in range(t + 1):
            P = _mat_mul(A[r], P)
        S = _mat_mul(P, S0)
        for s in range(t + 1):
            Ps = _ident(dk)
            for r in range(s + 1, t + 1):
                Ps = _mat_mul(A[r], Ps)
            outer = [[beta[s] * k[s][i] * v[s][j] for j in range(dv)] for i in range(dk)]
            S = _mat_add(S, _mat_mul(Ps, outer))
        states.append(S)
    return states


@pytest.mark.parametrize("seed,T,dk,dv", [(0, 1, 1, 1), (1, 3, 2, 3), (2, 5, 3, 2), (3, 8, 4, 4)])
def test_exact_rational_brute_force(seed, T, dk, dv):
    rnd = random.Random(seed)

    def rq(lo, hi, den=8):
        return Fraction(rnd.randint(lo * den, hi * den), den)

    alpha = [[Fraction(rnd.randint(1, 15), 16) for _ in range(dk)] for _ in range(T)]
    beta = [Fraction(rnd.randint(0, 8), 8) for _ in range(T)]
    k = [[rq(-1, 1) for _ in range(dk)] for _ in range(T)]
    q = [[rq(-1, 1) for _ in range(dk)] for _ in range(T)]
    v = [[rq(-2, 2) for _ in range(dv)] for _ in range(T)]
    S0 = [[rq(-1, 1) for _ in range(dv)] for _ in range(dk)]
    states = _brute_force_states(alpha, beta, k, v, S0)

    f = lambda M: np.array([[float(x) for x in row] for row in M], dtype=np.float64)
    qa = f(q).reshape(1, T, 1, dk)
    ka = f(k).reshape(1, T, 1, dk)
    va = f(v).reshape(1, T, 1, dv)
    ga = np.log(f(alpha)).reshape(1, T, 1, dk)
    ba = np.array([float(b) for b in beta]).reshape(1, T, 1)
    o, ST = O.kda_forward(qa, ka, va, ga, ba, f(S0).reshape(1, 1, dk, dv))
    for t in range(T):
        St = f(states[t])
        ot = np.array([float(sum(states[t][i][j] * q[t][i] for i in range(dk))) for j in range(dv)])
        scale = max(1.0, np.abs(ot).max())
        assert np.abs(o[0, t, 0] - ot).max() <= 1e-13 * scale
    St = f(states[-1])
    assert np.abs(ST[0, 0] - St).max() <= 1e-13 * max(1.0, np.abs(St).max())


# --------------------------------------------------------------------------------------
# 2. Delta-rule invariant (decay first, then erase, then write): with beta = 1 and a
#    unit key, k_t^T S_t = v_t^T for any alpha and any S0.  Feeding q = k makes the
#    readout equal k_t^T S_t, so o_t must equal v_t.  Applying the decay after the
#    write, or reading out before the update, breaks it.
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv,T", [(4, 3, 20), (32, 32, 64), (128, 128, 40)])
def test_delta_rule_invariant(dk, dv, T):
    rng = np.random.default_rng(dk * 1000 + T)
    k = _rand_unit(rng, (1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.uniform(0.0, 0.5, (1, T, 1, dk))
    beta = np.ones((1, T, 1))
    S0 = rng.standard_normal((1, 1, dk, dv))
    o, _ = O.kda_forward(k, k, v, g, beta, S0)
    assert np.abs(o - v).max() <= 1e-12 * max(1.0, np.abs(v).max()) * dk


# --------------------------------------------------------------------------------------
# 3. Pure decay: beta = 0 leaves only the channel-wise forget gate, so
#    S_t = Diag(prod_{r<=t} alpha_r) S0 and o_t = S_t^T q_t in closed form.
# --------------------------------------------------------------------------------------

def test_pure_decay_closed_form():
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 2, 33, 3, 8, 5
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    g = -rng.uniform(0, 0.3, (B, T, H, dk))
    beta = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    o, ST = O.kda_forward(q, k, v, g, beta, S0)
    cum = np.exp(np.cumsum(g, axis=1))              # [B,T,H,dk] = prod alpha
    S_t = cum[..., None] * S0[:, None]               # [B,T,H,dk,dv]
    o_ref = np.einsum("bthij,bthi->bthj", S_t, q)
    assert np.abs(o - o_ref).max() <= 1e-12
    assert np.abs(ST - S_t[:, -1]).max() <= 1e-12


# --------------------------------------------------------------------------------------
# 4. Orthonormal keys reduce KDA to gated linear attention: with k_t = e_{sigma(t)}
#    (distinct), beta = 1, S0 = 0, each written row keeps v_s decayed by the later
#    gates of its channel:
#    o_t = sum_{s<=t} q_t[sigma(s)] * prod_{u=s+1..t} alpha_u[sigma(s)] * v_s.
# --------------------------------------------------------------------------------------

def test_orthonormal_keys_gated_linear_attention():
    rng = np.random.default_rng(11)
    dk, dv, T = 16, 6, 16
    sigma = rng.permutation(dk)[:T]
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, sigma] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.uniform(0, 0.4, (1, T, 1, dk))
    beta = np.ones((1, T, 1))
    o, _ = O.kda_forward(q, k, v, g, beta)
    alpha = np.exp(g[0, :, 0])
    o_ref = np.zeros((T, dv))
    for t in range(T):
        for s in range(t + 1):
            c = sigma[s]
            decay = np.prod(alpha[s + 1:t + 1, c])
            o_ref[t] += q[0, t, 0, c] * decay * v[0, s, 0]
    assert np.abs(o[0, :, 0] - o_ref).max() <= 1e-12


# --------------------------------------------------------------------------------------
# 5. Basis keys with repeats and general beta: every state row is an exponential
#    moving average.  Row r after token T equals the explicit sum
#    sum_s [sigma(s)=r] beta_s v_s prod_{u>s} c_u(r),  c_u(r) = alpha_u[r] (1 - beta_u [sigma(u)=r]),
#    plus S0's row carried by prod_u c_u(r).
# --------------------------------------------------------------------------------------

def test_basis_keys_row_ema():
    rng = np.random.default_rng(5)
    dk, dv, T = 4, 3, 30
    sigma = rng.integers(0, dk, T)
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, sigma] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.uniform(0, 0.2, (1, T, 1, dk))
    beta = rng.uniform(0, 1, (1, T, 1))
    S0 = rng.standard_normal((1, 1, dk, dv))
    _, ST = O.kda_forward(q, k, v, g, beta, S0)
    alpha = np.exp(g[0, :, 0])
    b = beta[0, :, 0]
    ref = np.zeros((dk, dv))
    for r in range(dk):
        c = alpha[:, r] * (1.0 - b * (sigma == r))
        ref[r] = np.prod(c) * S0[0, 0, r]
        for s in range(T):
            if sigma[s] == r:
                ref[r] += b[s] * v[0, s, 0] * np.prod(c[s + 1:])
    assert np.abs(ST[0, 0] - ref).max() <= 1e-12


# --------------------------------------------------------------------------------------
# 6. Structural properties: resuming from S_T equals one pass (the reset/carry rule of
#    section 3.3), the result is linear in (v, S0) jointly, (b,h) pairs are independent,
#    and bf16 inputs are read exactly (same values given as fp32 give the same result).
# --------------------------------------------------------------------------------------

def test_split_resume_equals_one_pass():
    rng = np.random.default_rng(3)
    B, T, H, d = 1, 50, 2, 8
    q, k = _rand_unit(rng, (B, T, H, d)), _rand_unit(rng, (B, T, H, d))
    v = rng.standard_normal((B, T, H, d))
    g = -rng.uniform(0, 0.1, (B, T, H, d))
    beta = rng.uniform(0, 1, (B, T, H))
    o, ST = O.kda_forward(q, k, v, g, beta)
    t0 = 17
    o1, S1 = O.kda_forward(q[:, :t0], k[:, :t0], v[:, :t0], g[:, :t0], beta[:, :t0])
    o2, S2 = O.kda_forward(q[:, t0:], k[:, t0:], v[:, t0:], g[:, t0:], beta[:, t0:], S1)
    assert np.abs(np.concatenate([o1, o2], 1) - o).max() <= 1e-12
    assert np.abs(S2 - ST).max() <= 1e-12


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(4)
    B, T, H, d = 1, 24, 1, 6
    q, k = _rand_unit(rng, (B, T, H, d)), _rand_unit(rng, (B, T, H, d))
    g = -rng.uniform(0, 0.2, (B, T, H, d))
    beta = rng.uniform(0, 1, (B, T, H))
    v1, v2 = rng.standard_normal((2, B, T, H, d))
    S1, S2 = rng.standard_normal((2, B, H, d, d))
    oa, Sa = O.kda_forward(q, k, v1, g, beta, S1)
    ob, Sb = O.kda_forward(q, k, v2, g, beta, S2)
    oc, Sc = O.kda_forward(q, k, 2.0 * v1 - v2, g, beta, 2.0 * S1 - S2)
    assert np.abs(oc - (2 * oa - ob)).max() <= 1e-12
    assert np.abs(Sc - (2 * Sa - Sb)).max() <= 1e-12


def test_pairs_subset_matches_full_run():
    rng = np.random.default_rng(9)
    B, T, H, d = 2, 20, 3, 4
    q, k = _rand_unit(rng, (B, T, H, d)), _rand_unit(rng, (B, T, H, d))
    v = rng.standard_normal((B, T, H, d))
    g = -rng.uniform(0, 0.2, (B, T, H, d))
    beta = rng.uniform(0, 1, (B, T, H))
    o, ST = O.kda_forward(q, k, v, g, beta)
    o2, ST2 = O.kda_forward(q, k, v, g, beta, pairs=[(1, 2), (0, 1)])
    assert np.array_equal(o2[1, :, 2], o[1, :, 2]) and np.array_equal(o2[0, :, 1], o[0, :, 1])
    assert np.array_equal(ST2[1, 2], ST[1, 2])
    oh, Sh = O.kda_forward_head(q, k, v, g, beta, 1, 2)
    assert np.array_equal(oh, o[1, :, 2]) and np.array_equal(Sh, ST[1, 2])


def test_bf16_inputs_read_exactly():
    gen = torch.Generator().manual_seed(0)
    B, T, H, d = 1, 12, 2, 8
    mk = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    q, k, v = mk(B, T, H, d), mk(B, T, H, d), mk(B, T, H, d)
    g = (-torch.rand(B, T, H, d, generator=gen) * 0.1).to(torch.bfloat16)
    beta = torch.rand(B, T, H, generator=gen).to(torch.bfloat16)
    o1, S1 = O.kda_forward(q, k, v, g, beta)
    o2, S2 = O.kda_forward(q.float(), k.float(), v.float(), g.float(), beta.float())
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_rejects_bad_arguments():
    z = np.zeros((1, 4, 1, 2))
    with pytest.raises(ValueError):
        O.kda_forward(z, z, z, z, np.zeros((1, 4, 2)))
    with pytest.raises(TypeError):
        O.kda_forward(z.astype(np.float32), z, z, z, np.zeros((1, 4, 1)))


# ---- output side of Eq. 15: Sigmoid(gate) * RMSNorm(o) -----------------------------------
def _small_gated(seed=0, B=1, T=9, H=2, D=8):
    gen = torch.Generator().manual_seed(seed)
    f = dict(generator=gen, dtype=torch.float64)
    unit = lambda z: z / torch.linalg.vector_norm(z, dim=-1, keepdim=True)
    q, k = unit(torch.randn(B, T, H, D, **f)), unit(torch.randn(B, T, H, D, **f))
    v = torch.randn(B, T, H, D, **f)
    g = -0.1 * torch.rand(B, T, H, D, **f)
    beta = torch.rand(B, T, H, **f)
    gate = torch.randn(B, T, H, D, **f)
    gamma = 0.5 + torch.rand(H, D, **f)
    return q, k, v, g, beta, gate, gamma


def test_gated_rmsnorm_is_invariant_to_scaling_the_values():
    """RMSNorm removes the scale: o is linear in v (S0 = 0), so scaling v by c > 0
    leaves the gated output unchanged (eps = 0)."""
    q, k, v, g, beta, gate, gamma = _small_gated(1)
    y1, _ = O.kda_forward_gated(q, k, v, g, beta, gate, gamma, eps=0.0)
    y2, _ = O.kda_forward_gated(q, k, 37.5 * v, g, beta, gate, gamma, eps=0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-14)


def test_gated_rmsnorm_unit_rms_and_gate_limits():
    """With gamma = 1 and a gate far above zero the sigmoid is 1 and every (token, head)
    row has unit RMS; a zero gate halves it; a gate far below zero closes it."""
    q, k, v, g, beta, gate, _ = _small_gated(2)
    o, _ = O.kda_forward(q, k, v, g, beta)
    y_open = O.gated_rmsnorm(o, np.full(o.shape, 60.0), None, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y_open ** 2, axis=-1)), 1.0, rtol=1e-12)
    y_half = O.gated_rmsnorm(o, np.zeros(o.shape), None, eps=0.0)
    np.testing.assert_allclose(y_half, 0.5 * y_open, rtol=1e-12, atol=1e-15)
    y_shut = O.gated_rmsnorm(o, np.full(o.shape, -60.0), None, eps=0.0)
    assert np.abs(y_shut).max() < 1e-25


def test_gated_rmsnorm_gain_and_eps():
    """gamma multiplies channel-wise per head; eps enters as mean(o^2) + eps (an all-zero
    row stays zero, a row of constant c gets c / sqrt(c^2 + eps))."""
    q, k, v, g, beta, gate, gamma = _small_gated(3)
    o, _ = O.kda_forward(q, k, v, g, beta)
    y1 = O.gated_rmsnorm(o, gate, None, eps=1e-3)
    y2 = O.gated_rmsnorm(o, gate, gamma, eps=1e-3)
    np.testing.assert_allclose(y2, y1 * gamma.numpy()[None, None], rtol=1e-12, atol=1e-15)
    row = np.full((1, 1, 1, 4), 0.2)
    y = O.gated_rmsnorm(row, np.full(row.shape, 60.0), None, eps=0.01)
    np.testing.assert_allclose(y, 0.2 / np.sqrt(0.04 + 0.01), rtol=1e-12)
    assert np.all(O.gated_rmsnorm(np.zeros((1, 2, 1, 4)), np.zeros((1, 2, 1, 4)), None, eps=0.0) == 0.0)


# ---- packed samples --------------------------------------------------------------------
def test_varlen_samples_are_independent_scans():
    """Each packed sample is the scan of that sample alone from its own S0 (the reset at a
    sample start): a single sample equals kda_forward, and changing one sample's values
    leaves every other sample's output and final state bit-for-bit unchanged."""
    gen = torch.Generator().manual_seed(11)
    T, H, D = 23, 2, 4
    f = dict(generator=gen, dtype=torch.float64)
    q, k, g = torch.randn(T, H, D, **f), torch.randn(T, H, D, **f), -0.2 * torch.rand(T, H, D, **f)
    v, beta = torch.randn(T, H, D, **f), torch.rand(T, H, **f)
    S0 = torch.randn(4, H, D, D, **f)
    cu = [0, 6, 6, 15, 23]
    o, S = O.kda_forward_varlen(q, k, v, g, beta, cu, S0)
    o1, S1 = O.kda_forward(q[6:15][None], k[6:15][None], v[6:15][None], g[6:15][None], beta[6:15][None],
                           S0[2:3].numpy())
    np.testing.assert_array_equal(o[6:15], o1[0])
    np.testing.assert_array_equal(S[2], S1[0])
    np.testing.assert_array_equal(S[1], S0[1].numpy())          # empty sample: S_T = S0
    v2 = v.clone()
    v2[6:15] *= -3.0
    o2, Sb = O.kda_forward_varlen(q, k, v2, g, beta, cu, S0)
    for (a, b, i) in [(0, 6, 0), (15, 23, 3)]:
        np.testing.assert_array_equal(o2[a:b], o[a:b])
        np.testing.assert_array_equal(Sb[i], S[i])
    assert not np.array_equal(o2[6:15], o[6:15])
