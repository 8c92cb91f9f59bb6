"""P6: the chunked (WY / UT-transform) form of the gated delta rule, in fp64 numpy, equals the
sequential oracle.  This pins the algorithm the CUDA prefill kernels implement, separately from
their precision (CPU only).

Per value head and chunk of L tokens (G = inclusive cumulative sum of g inside the chunk):
  A_ij = beta_i exp(G_i - G_j) k_i.k_j  (j < i),   T = (I + A)^-1
  W = T diag(beta e^G) K,   U~ = T diag(beta) V
  U = U~ - W S^T                                  (S = state entering the chunk, [d_v, d_k])
  O = diag(e^G) Q S^T + P U,  P_ij = e^(G_i - G_j) q_i.k_j  (j <= i)
  S <- e^(G_L) S + U^T diag(e^(G_L - G)) K
Derivation: unroll S_i = e^(G_i) S + sum_{j<=i} e^(G_i - G_j) u_j k_j^T inside the chunk and
substitute it into u_i = beta_i (v_i - alpha_i S_(i-1) k_i).

The kernels also rely on two facts checked here:
  * padding a partial chunk with k = q = v = 0, beta = 0, g = 0 leaves every result unchanged;
  * the 128-token inverse can be assembled from the two 64-token diagonal inverses:
    T = T_h - T_h N T_h, T_h = blockdiag((I + A_00)^-1, (I + A_11)^-1), N = lower-left block of A;
  * each 64-token inverse from its two 32-token diagonal inverses, both at once:
    T_h = D - D L1 D, D = blockdiag of the four 32-token inverses, L1 = the blocks (1,0) and
    (3,2) of A (exact: (L1 D)^2 = 0 inside each 64-token block);
  * the 32-token inverses by row substitution T[l] = e_l - sum_{j<l} A[l][j] T[j];
  * d_v column blocks of the state evolve independently (the chain's split across CTAs);
  * the look-ahead form of the chain step, X_(c+1) = e^(G_L) W_(c+1) S_c^T + E_(c+1) U^_c.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_layer_02_b200 import inputs


def _masked_decay(G, strict):
    diff = G[:, None] - G[None, :]
    L = len(G)
    mask = np.tril(np.ones((L, L), bool), -1 if strict else 0)
    return np.where(mask, np.exp(np.where(mask, diff, 0.0)), 0.0)


def chunked_head(q, k, v, beta, g, S, C, pad_to=None):
    """One value head over one sequence.  q, k [T, dk] (normalised), v [T, dv], S [dv, dk]."""
    T = q.shape[0]
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        Q, K, V, b, gg = q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1], g[c0:c1]
        if pad_to is not None and c1 - c0 < pad_to:
            p = pad_to - (c1 - c0)
            Q, K, V = (np.pad(a, ((0, p), (0, 0))) for a in (Q, K, V))
            b, gg = np.pad(b, (0, p)), np.pad(gg, (0, p))
        G = np.cumsum(gg)
        A = b[:, None] * _masked_decay(G, True) * (K @ K.T)
        Tm = np.linalg.inv(np.eye(len(G)) + A)
        W = Tm @ ((b * np.exp(G))[:, None] * K)
        Ut = Tm @ (b[:, None] * V)
        U = Ut - W @ S.T
        P = _masked_decay(G, False) * (Q @ K.T)
        O = np.exp(G)[:, None] * (Q @ S.T) + P @ U
        S = np.exp(G[-1]) * S + (U * np.exp(G[-1] - G)[:, None]).T @ K
        out[c0:c1] = O[: c1 - c0]
    return out, S


def _normalised_inputs(seed, lengths, hk, hv, d, g_low):
    r = np.random.default_rng(seed)
    T = sum(lengths)
    q, k = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d))
    v = r.standard_normal((T, hv, d))
    beta = r.uniform(0, 1, (T, hv)).astype(np.float32)
    g = r.uniform(g_low, 0, (T, hv)).astype(np.float32)
    S0 = (r.standard_normal((len(lengths), hv, d, d)) * 0.3).astype(np.float32)
    return q, k, v, beta, g, S0


@pytest.mark.parametrize("C,pad", [(4, None), (16, None), (32, None), (16, 16), (64, 64)])
@pytest.mark.parametrize("g_low", [-0.05, -1.5])
def test_p6_chunked_equals_sequential(C, pad, g_low):
    lengths = [1, 37, 64, 50]
    hk, hv, d = 1, 2, 16
    q, k, v, beta, g, S0 = _normalised_inputs(6, lengths, hk, hv, d, g_low)
    T = sum(lengths)
    x = np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], 1)
    dims = oracle.Dims(hk, hv, d, 4, 1.0, 0.0, 1e-6)
    ref_o, ref_S, _ = oracle.prefill(dims, torch.from_numpy(x), torch.from_numpy(beta),
                                     torch.from_numpy(g), inputs.cu_seqlens_of(lengths),
                                     S0=torch.from_numpy(S0), nthreads=2)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    for n in range(len(lengths)):
        s = slice(cu[n], cu[n + 1])
        for h in range(hv):
            o, S = chunked_head(qn[s, h // (hv // hk)], kn[s, h // (hv // hk)], v[s, h],
                                beta[s, h].astype(np.float64), g[s, h].astype(np.float64),
                                S0[n, h].astype(np.float64), C, pad)
            np.testing.assert_allclose(o, ref_o[s, h], rtol=1e-9, atol=1e-10)
            np.testing.assert_allclose(S, ref_S[n, h], rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("g_low", [-0.05, -1.0])
def test_block_inverse_assembly(g_low):
    r = np.random.default_rng(61)
    C, d = 128, 128
    K = r.standard_normal((C, d)) + 0.5           # correlated keys (a mean component)
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    b = r.uniform(0, 1, C)
    G = np.cumsum(r.uniform(g_low, 0, C))
    A = b[:, None] * _masked_decay(G, True) * (K @ K.T)
    h = C // 2
    Th = np.zeros((C, C))
    Th[:h, :h] = np.linalg.inv(np.eye(h) + A[:h, :h])
    Th[h:, h:] = np.linalg.inv(np.eye(h) + A[h:, h:])
    N = np.zeros((C, C))
    N[h:, :h] = A[h:, :h]
    T = Th - Th @ N @ Th
    np.testing.assert_allclose(T, np.linalg.inv(np.eye(C) + A), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("g_low", [-0.05, -1.0])
def test_two_level_block_inverse_assembly(g_low):
    # the order the prep kernel uses: 32-token blocks by row substitution, joined in pairs by
    # D - D L1 D, then the two 64-token halves by T_h - T_h N T_h
    r = np.random.default_rng(62)
    C, d = 128, 128
    K = r.standard_normal((C, d)) + 0.5
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    b = r.uniform(0, 1, C)
    G = np.cumsum(r.uniform(g_low, 0, C))
    A = b[:, None] * _masked_decay(G, True) * (K @ K.T)
    D = np.zeros((C, C))
    for q in range(4):
        blk = A[32 * q:32 * q + 32, 32 * q:32 * q + 32]
        T = np.zeros((32, 32))
        for l in range(32):  # row substitution, as the warps do it
            T[l] = np.eye(32)[l] - blk[l, :l] @ T[:l]
        D[32 * q:32 * q + 32, 32 * q:32 * q + 32] = T
    L1 = np.zeros((C, C))
    L1[32:64, 0:32] = A[32:64, 0:32]
    L1[96:128, 64:96] = A[96:128, 64:96]
    Th = D - D @ L1 @ D
    N = np.zeros((C, C))
    N[64:, :64] = A[64:, :64]
    T = Th - Th @ N @ Th
    np.testing.assert_allclose(Th[:64, :64], np.linalg.inv(np.eye(64) + A[:64, :64]),
                               rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(T, np.linalg.inv(np.eye(C) + A), rtol=1e-10, atol=1e-12)


def _chunk_terms(Q, K, V, b, gg):
    G = np.cumsum(gg)
    A = b[:, None] * _masked_decay(G, True) * (K @ K.T)
    Tm = np.linalg.inv(np.eye(len(G)) + A)
    return G, Tm @ ((b * np.exp(G))[:, None] * K), Tm @ (b[:, None] * V)


@pytest.mark.parametrize("g_low", [-0.05, -1.5])
def test_look_ahead_product_of_the_chain(g_low):
    """X of chunk c+1 from the state entering chunk c: with U^_c = diag(e^(G_L - G)) U_c and
    E_(c+1) = W_(c+1) K_c^T (available before the chain reaches chunk c),
    X_(c+1) = W_(c+1) S_(c+1)^T = e^(G_L) W_(c+1) S_c^T + E_(c+1) U^_c, so one product follows
    U_c instead of two (the form measured as the look-ahead chain)."""
    C, d = 32, 16
    q, k, v, beta, g, S0 = _normalised_inputs(61, [2 * C], 1, 1, d, g_low)
    k = k[:, 0] / np.linalg.norm(k[:, 0], axis=1, keepdims=True)
    v, b, gg = v[:, 0], beta[:, 0].astype(np.float64), g[:, 0].astype(np.float64)
    S = S0[0, 0].astype(np.float64)
    G0, W0, Ut0 = _chunk_terms(None, k[:C], v[:C], b[:C], gg[:C])
    G1, W1, Ut1 = _chunk_terms(None, k[C:], v[C:], b[C:], gg[C:])
    U0 = Ut0 - W0 @ S.T
    Uhat = np.exp(G0[-1] - G0)[:, None] * U0
    S1 = np.exp(G0[-1]) * S + Uhat.T @ k[:C]
    X1 = W1 @ S1.T
    E1 = W1 @ k[:C].T
    np.testing.assert_allclose(np.exp(G0[-1]) * (W1 @ S.T) + E1 @ Uhat, X1, rtol=1e-11,
                               atol=1e-11)


def test_value_column_blocks_evolve_independently():
    """Each d_v block of the state (rows of S, columns of V and U) follows the recurrence on its
    own: the chain may split d_v across CTAs with no exchange."""
    lengths, d = [70], 16
    q, k, v, beta, g, S0 = _normalised_inputs(62, lengths, 1, 1, d, -0.5)
    qn = q[:, 0] / np.linalg.norm(q[:, 0], axis=1, keepdims=True)
    kn = k[:, 0] / np.linalg.norm(k[:, 0], axis=1, keepdims=True)
    b, gg, S = beta[:, 0].astype(np.float64), g[:, 0].astype(np.float64), S0[0, 0].astype(np.float64)
    full_o, full_S = chunked_head(qn, kn, v[:, 0], b, gg, S, 16)
    for c0 in range(0, d, 4):
        o, Sb = chunked_head(qn, kn, v[:, 0, c0:c0 + 4], b, gg, S[c0:c0 + 4], 16)
        np.testing.assert_allclose(o, full_o[:, c0:c0 + 4], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Sb, full_S[c0:c0 + 4], rtol=1e-12, atol=1e-12)
