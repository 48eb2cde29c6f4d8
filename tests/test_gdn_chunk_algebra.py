"""The closed form the Gated DeltaNet kernels evaluate per 32-token chunk,
restated in numpy (fp32) and checked against the oracle's token-by-token
recurrence.

The CUDA path solves each chunk in closed form:
- gamma is the running sum of the log decays inside the chunk;
- A_ij = beta_i e^(gamma_i - gamma_j) k_i.k_j for j < i;
- (I + A)^-1 comes from forward substitution;
- Tt = diag(e^(gamma_31 - gamma)) (I + A)^-1;
- M = W_qk (I + A)^-1, with W_qk_ij = e^(gamma_i - gamma_j) q_i.k_j for j <= i.

Each state row s then takes Pk = s.k_i and Pq = s.q_i and forms
r = beta (v - e^gamma Pk). The outputs are e^gamma Pq + M r, and the row
leaving the chunk is e^gamma_31 s + sum_i (Tt r)_i k_i. A ragged tail is
padded with zero tokens (k = q = v = 0, g = 0, beta = 0).

This file checks that algebra, including the padding convention and the
worst-conditioned solve (repeated keys at full strength). It runs on the
CPU. The restatement shares no code with the CUDA path, and the oracle
serves only as the reference it is compared with.
"""

import numpy as np
import pytest

from oracle import gated_deltanet_oracle as gdn

F = np.float32
CH = 32


def _chunk_matrices(k, q, g, beta):
    gam = np.cumsum(g.astype(F)).astype(F)
    eg = np.exp(gam).astype(F)
    dec = np.exp(gam[-1] - gam).astype(F)
    E = np.exp(np.minimum(gam[:, None] - gam[None, :], 0)).astype(F)
    A = np.tril(beta[:, None] * E * (k @ k.T), -1).astype(F)
    T = np.zeros((CH, CH), F)
    for j in range(CH):  # forward substitution, one column at a time
        col = np.zeros(CH, F)
        for i in range(CH):
            acc = F(0)
            for m in range(i):
                acc = F(acc + A[i, m] * col[m])
            col[i] = 0 if i < j else (1 if i == j else -acc)
        T[:, j] = col
    Wqk = np.tril(E * (q @ k.T)).astype(F)
    return eg, (dec[:, None] * T).astype(F), (Wqk @ T).astype(F)


def _chunked(q, k, v, g, beta, S0):
    T_, H, dk = k.shape
    tp = (T_ + CH - 1) // CH * CH
    pad = lambda a: np.concatenate([np.asarray(a, F), np.zeros((tp - T_,) + a.shape[1:], F)])
    q, k, v, g, beta = (pad(x) for x in (q, k, v, g, beta))
    S = np.array(S0, F)
    o = np.zeros((tp, H, v.shape[2]), F)
    for h in range(H):
        for c in range(tp // CH):
            sl = slice(CH * c, CH * (c + 1))
            eg, Tt, M = _chunk_matrices(k[sl, h], q[sl, h], g[sl, h], beta[sl, h])
            Pk, Pq = S[h] @ k[sl, h].T, S[h] @ q[sl, h].T
            r = beta[sl, h][None, :] * (v[sl, h].T - eg[None, :] * Pk)
            o[sl, h] = (eg[None, :] * Pq + r @ M.T).T
            S[h] = eg[-1] * S[h] + (r @ Tt.T) @ k[sl, h]
    return o[:T_], S


def _inputs(rng, T, H, dk, dv, repeated=False, strong_decay=False):
    k = gdn.l2_normalize(rng.standard_normal((T, H, dk)))
    if repeated:
        k[:] = k[:1]
    q = gdn.l2_normalize(rng.standard_normal((T, H, dk))) / np.sqrt(dk)
    v = rng.standard_normal((T, H, dv))
    g = -rng.uniform(0, 0.3, (T, H))
    if strong_decay:
        g[:, 0] = -80.0  # alpha ~ 1.8e-35: products of decays underflow fp32
    beta = np.ones((T, H)) if repeated else rng.uniform(0, 1, (T, H))
    S0 = 0.3 * rng.standard_normal((H, dv, dk))
    return q, k, v, g, beta, S0


@pytest.mark.parametrize("T,repeated,strong", [(1, False, False), (31, False, False),
                                               (32, False, False), (77, False, False),
                                               (70, True, False), (64, False, True)])
def test_chunked_closed_form_equals_the_recurrence(T, repeated, strong):
    rng = np.random.default_rng(T + 7 * repeated + 13 * strong)
    q, k, v, g, beta, S0 = _inputs(rng, T, 2, 32, 8, repeated, strong)
    o_ref, S_ref = gdn.gated_delta_rule(q, k, v, g, beta, S0)
    o, S = _chunked(q, k, v, g, beta, S0)
    scale = max(1.0, np.abs(o_ref).max())
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=2e-6 * scale)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=2e-6 * max(1.0, np.abs(S_ref).max()))


def test_zero_tokens_are_neutral():
    # the padding convention: a zero token (k = q = v = 0, g = 0, beta = 0)
    # leaves the state exactly as it was and outputs zero
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = _inputs(rng, 40, 1, 16, 4)
    z = lambda a: np.concatenate([a, np.zeros((5,) + a.shape[1:])])
    o_ref, S_ref = gdn.gated_delta_rule(q, k, v, g, beta, S0)
    o2, S2 = gdn.gated_delta_rule(z(q), z(k), z(v), z(g), z(beta), S0)
    np.testing.assert_array_equal(S2, S_ref)
    np.testing.assert_array_equal(o2[:40], o_ref)
    np.testing.assert_array_equal(o2[40:], 0.0)
