"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test fixes one part of the definition with a closed form, an invariant, brute force on a
tiny input or a library routine, so that a dropped term, a wrong sign, index or transposed
operand anywhere in the oracle fails at least one of them:

  P1  beta = 0: the state only decays, S_T = exp(sum g) S_0, o_t = S_t q_t.
  P2  alpha = beta = 1 with orthonormal keys: querying with a written key returns its value.
  P3  beta = 1, unit keys: the delta rule writes exactly, S_t k_t = v_t after every token.
  P4  T = 1 closed form of one update (matrix form), including S_0 = 0.
  P5  brute force: the explicit product of dense (I - beta k k^T) factors on tiny inputs.
  P7  split invariance (state hand-off) and decode steps = prefill of the same tokens.
  P8  packed variable-length batch = separate runs; key head shared by consecutive value heads.
  P9  conv + SiLU = torch.nn.functional.conv1d (library routine) then SiLU.
  P10 gated RMSNorm = torch.nn.functional.rms_norm (library routine) * w * silu(z); z = 0 -> 0.
  P11 contraction bound |S_t|_F <= alpha_t |S_{t-1}|_F + beta_t |v_t|.
  P12 token-mixer gates: sigmoid / softplus special values and torch's softplus; with
      identity projections the token mixer reduces to the layer.
  P13 error scales (the tolerance the GPU tests use): M >= |S| and c >= |o| element-wise
      (triangle inequality); T = 1 closed form of M; beta = 0 gives M = exp(sum g) |S_0|;
      the normalised-output scale is invariant, and M scales linearly, when v and S_0 are
      scaled together; decode steps carry M exactly as the prefill does; the scales leave
      out, SN and convN untouched.
The chunked (WY/UT) form the CUDA path uses is checked against the oracle in
test_chunk_algebra.py (P6).
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from gated_deltanet_layer_02_b200 import inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
HERE = os.path.dirname(os.path.abspath(__file__))


def _rng(seed):
    return np.random.default_rng(seed)


def _dims(hk=1, hv=1, d=8, K=4, l2_eps=0.0, norm_eps=1e-6):
    return oracle.Dims(hk, hv, d, K, 1.0, l2_eps, norm_eps)


def _unit(a):
    return a / np.linalg.norm(a, axis=-1, keepdims=True)


def _pack_x(q, k, v):
    """Conv input row [q (Hk*d) | k (Hk*d) | v (Hv*d)] from per-head arrays [T, H, d]."""
    T = q.shape[0]
    return np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], axis=1)


def _f32(a):
    return np.asarray(a, np.float32)


def _run(dims, x, beta, g, S0=None, lengths=None, **kw):
    T = x.shape[0]
    lengths = lengths or [T]
    cu = inputs.cu_seqlens_of(lengths)
    return oracle.prefill(dims, torch.from_numpy(np.ascontiguousarray(x)),
                          torch.from_numpy(_f32(beta)), torch.from_numpy(_f32(g)), cu,
                          S0=None if S0 is None else torch.from_numpy(_f32(S0)), nthreads=2, **kw)


# ---------------------------------------------------------------------------------------- P1
def test_p1_beta_zero_pure_decay():
    r = _rng(1)
    T, d, hk, hv = 7, 8, 1, 2
    q, k, v = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hv, d))
    g = _f32(r.uniform(-0.7, 0.0, (T, hv)))
    S0 = _f32(r.standard_normal((1, hv, d, d)))
    out, SN, _ = _run(_dims(hk, hv, d), _pack_x(q, k, v), np.zeros((T, hv)), g, S0=S0)
    qn = _unit(q)
    for h in range(hv):
        G = np.cumsum(g[:, h].astype(np.float64))
        np.testing.assert_allclose(SN[0, h], np.exp(G[-1]) * S0[0, h], rtol=1e-12, atol=1e-12)
        for t in range(T):
            np.testing.assert_allclose(out[t, h], np.exp(G[t]) * S0[0, h].astype(np.float64) @ qn[t, 0],
                                       rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------- P2
def test_p2_orthonormal_keys_retrieve_values():
    r = _rng(2)
    d, T = 16, 12
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    keys = Qm[:T]                          # T orthonormal rows
    scale = r.uniform(0.5, 3.0, (T, 1))    # L2-normalisation must remove any scale
    v = r.standard_normal((T, 1, d))
    # query at token t with the key written at token perm[t] <= t, and perm != identity
    perm = np.array([max(0, t - 1 - (t % 3)) for t in range(T)])
    q = keys[perm] * 2.0
    out, SN, _ = _run(_dims(1, 1, d), _pack_x(q[:, None], (keys * scale)[:, None], v),
                      np.ones((T, 1)), np.zeros((T, 1)))
    for t in range(T):
        np.testing.assert_allclose(out[t, 0], v[perm[t], 0], rtol=0, atol=1e-12)
    # final state is the sum of outer products v_i k_i^T
    np.testing.assert_allclose(SN[0, 0], sum(np.outer(v[i, 0], keys[i]) for i in range(T)), atol=1e-12)


# ---------------------------------------------------------------------------------------- P3
def test_p3_delta_rule_writes_exactly():
    r = _rng(3)
    T, d = 20, 8
    k = r.standard_normal((T, 1, d))
    v = r.standard_normal((T, 1, d)) * 3
    g = r.uniform(-1.0, 0.0, (T, 1))
    S0 = r.standard_normal((1, 1, d, d))
    # q = k at every token, so o_t = S_t k_t must equal v_t
    out, _, _ = _run(_dims(1, 1, d), _pack_x(k, k, v), np.ones((T, 1)), g, S0=S0)
    np.testing.assert_allclose(out[:, 0], v[:, 0], rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------------------- P4
@pytest.mark.parametrize("zero_state", [False, True])
def test_p4_single_token_closed_form(zero_state):
    r = _rng(4)
    d = 8
    q, k, v = r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d))
    beta, g = _f32([[0.37]]), _f32([[-0.21]])
    S0 = np.zeros((1, 1, d, d), np.float32) if zero_state else _f32(r.standard_normal((1, 1, d, d)))
    out, SN, _ = _run(_dims(1, 1, d), _pack_x(q, k, v), beta, g, S0=S0)
    a, b = np.exp(np.float64(g[0, 0])), np.float64(beta[0, 0])
    kn, qn, vv, S = _unit(k[0, 0]), _unit(q[0, 0]), v[0, 0], S0[0, 0].astype(np.float64)
    S1 = a * S - a * b * np.outer(S @ kn, kn) + b * np.outer(vv, kn)
    np.testing.assert_allclose(SN[0, 0], S1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(out[0, 0], S1 @ qn, rtol=1e-12, atol=1e-13)
    if zero_state:
        np.testing.assert_allclose(out[0, 0], b * (kn @ qn) * vv, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------------------- P5
def _brute_force(qn, kn, v, beta, g, S0):
    """Dense product form: S_T = S_0 prod_t A_t + sum_i beta_i v_i k_i^T prod_{j>i} A_j,
    A_t = alpha_t (I - beta_t k_t k_t^T); outputs from the same form at every prefix."""
    T, d = kn.shape
    I = np.eye(d)
    A = [np.exp(g[t]) * (I - beta[t] * np.outer(kn[t], kn[t])) for t in range(T)]
    outs, states = [], []
    for t in range(T):
        S = S0.copy()
        for j in range(t + 1):
            S = S @ A[j]
        for i in range(t + 1):
            term = beta[i] * np.outer(v[i], kn[i])
            for j in range(i + 1, t + 1):
                term = term @ A[j]
            S = S + term
        states.append(S)
        outs.append(S @ qn[t])
    return np.array(outs), states


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_p5_brute_force_product(seed):
    r = _rng(seed)
    T, d, hk, hv = 6, 4, 2, 4
    q, k, v = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hv, d))
    beta = _f32(r.uniform(0, 1, (T, hv)))
    g = _f32(r.uniform(-0.8, 0, (T, hv)))
    S0 = _f32(r.standard_normal((1, hv, d, d)))  # not symmetric: a transposed state fails
    dims = _dims(hk, hv, d, l2_eps=1e-6)
    out, SN, _ = _run(dims, _pack_x(q, k, v), beta, g, S0=S0)
    for h in range(hv):
        hkh = h // (hv // hk)
        qn = q[:, hkh] / np.sqrt((q[:, hkh] ** 2).sum(-1, keepdims=True) + 1e-6)
        kn = k[:, hkh] / np.sqrt((k[:, hkh] ** 2).sum(-1, keepdims=True) + 1e-6)
        o_bf, states = _brute_force(qn, kn, v[:, h], beta[:, h].astype(np.float64),
                                    g[:, h].astype(np.float64), S0[0, h].astype(np.float64))
        np.testing.assert_allclose(out[:, h], o_bf, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(SN[0, h], states[-1], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------------------- P7
def test_p7_split_invariance_and_decode_equivalence():
    w = inputs.custom(num_k_heads=1, num_v_heads=2, head_dim=16, dtype=torch.float32,
                      lengths=(11,), s0_std=0.3)
    d = inputs.prefill_inputs(w, 77, with_conv0=True)
    dims = oracle.Dims(1, 2, 16, 4, 1.0, 1e-6, 1e-6)
    full = oracle.prefill(dims, d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                          z=d["z"], norm_w=d["norm_w"], S0=d["S0"], conv0=d["conv0"])
    for T1 in (1, 2, 5, 10):
        a = oracle.prefill(dims, d["x"][:T1], d["beta"][:T1], d["g"][:T1],
                           inputs.cu_seqlens_of([T1]), conv_w=d["conv_w"], z=d["z"][:T1],
                           norm_w=d["norm_w"], S0=d["S0"], conv0=d["conv0"])
        b = oracle.prefill(dims, d["x"][T1:], d["beta"][T1:], d["g"][T1:],
                           inputs.cu_seqlens_of([11 - T1]), conv_w=d["conv_w"], z=d["z"][T1:],
                           norm_w=d["norm_w"], S0=torch.from_numpy(a[1]).float(),
                           conv0=torch.from_numpy(a[2]).float())
        # the hand-off rounds the state to fp32 once, hence the tolerance
        np.testing.assert_allclose(np.concatenate([a[0], b[0]]), full[0], rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(b[1], full[1], rtol=1e-6, atol=1e-7)
        np.testing.assert_array_equal(b[2], full[2])
    # 11 decode steps reproduce the prefill exactly (the decode oracle keeps fp64 state)
    S = d["S0"].double().numpy().copy()
    cs = d["conv0"].double().numpy().copy()
    outs = []
    for t in range(11):
        outs.append(oracle.decode_step(dims, d["x"][t:t + 1], d["beta"][t:t + 1], d["g"][t:t + 1],
                                       cs, S, conv_w=d["conv_w"], z=d["z"][t:t + 1],
                                       norm_w=d["norm_w"]))
    np.testing.assert_allclose(np.concatenate(outs), full[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, full[1], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cs, full[2])


def test_p7_decode_slots_and_conv_shift():
    dims = oracle.Dims(1, 2, 8, 4, 1.0, 1e-6, 1e-6)
    r = _rng(71)
    B, slots, Cc = 3, 5, dims.channels
    x = torch.from_numpy(r.standard_normal((B, Cc)))
    cw = torch.from_numpy(r.standard_normal((Cc, 4)) * 0.5)
    beta = torch.from_numpy(_f32(r.uniform(0, 1, (B, 2))))
    g = torch.from_numpy(_f32(r.uniform(-1, 0, (B, 2))))
    cs = r.standard_normal((slots, 3, Cc))
    S = r.standard_normal((slots, 2, 8, 8))
    slot = np.array([4, 0, 2], np.int32)
    cs0, S0 = cs.copy(), S.copy()
    out = oracle.decode_step(dims, x, beta, g, cs, S, conv_w=cw, slot_idx=torch.from_numpy(slot))
    for b, s in enumerate(slot):
        np.testing.assert_array_equal(cs[s, :2], cs0[s, 1:])
        np.testing.assert_array_equal(cs[s, 2], x[b].numpy())
        # the same token as a one-token prefill with that slot's history
        ref = oracle.prefill(dims, x[b:b + 1], beta[b:b + 1], g[b:b + 1], inputs.cu_seqlens_of([1]),
                             conv_w=cw, S0=None, conv0=torch.from_numpy(cs0[s:s + 1]))
        # S0 in prefill is fp32; compare the state-independent case via a zero-state copy
        S_zero = np.zeros((1, 2, 8, 8))
        cs_copy = cs0[s:s + 1].copy()
        o2 = oracle.decode_step(dims, x[b:b + 1], beta[b:b + 1], g[b:b + 1], cs_copy, S_zero, conv_w=cw)
        np.testing.assert_allclose(o2, ref[0], rtol=1e-12, atol=1e-13)
    for s in (1, 3):  # untouched slots
        np.testing.assert_array_equal(cs[s], cs0[s])
        np.testing.assert_array_equal(S[s], S0[s])
    assert out.shape == (B, 2, 8)


# ---------------------------------------------------------------------------------------- P8
def test_p8_varlen_equals_separate_runs():
    w = inputs.custom(num_k_heads=2, num_v_heads=4, head_dim=16, dtype=torch.bfloat16,
                      lengths=(1, 5, 2, 9), s0_std=0.2)
    d = inputs.prefill_inputs(w, 88, with_conv0=True)
    dims = oracle.Dims(2, 4, 16, 4, 1.0, 1e-6, 1e-6)
    packed = oracle.prefill(dims, d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                            z=d["z"], norm_w=d["norm_w"], S0=d["S0"], conv0=d["conv0"])
    cu = d["cu_seqlens"].tolist()
    for n in range(4):
        s = slice(cu[n], cu[n + 1])
        one = oracle.prefill(dims, d["x"][s], d["beta"][s], d["g"][s],
                             inputs.cu_seqlens_of([cu[n + 1] - cu[n]]), conv_w=d["conv_w"],
                             z=d["z"][s], norm_w=d["norm_w"], S0=d["S0"][n:n + 1],
                             conv0=d["conv0"][n:n + 1])
        np.testing.assert_array_equal(packed[0][s], one[0])
        np.testing.assert_array_equal(packed[1][n], one[1][0])
        np.testing.assert_array_equal(packed[2][n], one[2][0])


def test_p8_gqa_key_head_of_each_value_head():
    r = _rng(8)
    T, d, hk, hv = 9, 8, 2, 4
    q, k = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d))
    v1 = r.standard_normal((T, 1, d))
    v = np.repeat(v1, hv, axis=1)                 # identical values for all value heads
    beta = np.repeat(_f32(r.uniform(0, 1, (T, 1))), hv, 1)
    g = np.repeat(_f32(r.uniform(-1, 0, (T, 1))), hv, 1)
    out, _, _ = _run(_dims(hk, hv, d, l2_eps=1e-6), _pack_x(q, k, v), beta, g)
    # value heads 2h and 2h+1 read key head h: equal outputs within a pair, different across
    np.testing.assert_array_equal(out[:, 0], out[:, 1])
    np.testing.assert_array_equal(out[:, 2], out[:, 3])
    assert np.abs(out[:, 0] - out[:, 2]).max() > 1e-3
    # and the pair (0, 1) really uses key head 0: rerun with key head 1 replaced
    q2, k2 = q.copy(), k.copy()
    q2[:, 1], k2[:, 1] = r.standard_normal((T, d)), r.standard_normal((T, d))
    out2, _, _ = _run(_dims(hk, hv, d, l2_eps=1e-6), _pack_x(q2, k2, v), beta, g)
    np.testing.assert_array_equal(out2[:, :2], out[:, :2])
    assert np.abs(out2[:, 2:] - out[:, 2:]).max() > 1e-3


# ---------------------------------------------------------------------------------------- P9
@pytest.mark.parametrize("with_state", [False, True])
def test_p9_conv_matches_torch_conv1d(with_state):
    r = _rng(9)
    C, K = 24, 4
    lengths = [1, 2, 7, 13]
    T = sum(lengths)
    x = r.standard_normal((T, C))
    w = r.standard_normal((C, K)) * 0.5
    st = r.standard_normal((len(lengths), K - 1, C)) if with_state else None
    y, st_out = oracle.conv1d_silu(torch.from_numpy(x), torch.from_numpy(w), inputs.cu_seqlens_of(lengths),
                                   None if st is None else torch.from_numpy(st))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    for n, L in enumerate(lengths):
        hist = st[n] if with_state else np.zeros((K - 1, C))
        ext = np.concatenate([hist, x[cu[n]:cu[n + 1]]])             # [K-1+L, C]
        ref = F.conv1d(torch.from_numpy(ext.T[None]), torch.from_numpy(w[:, None, :]), groups=C)
        ref = F.silu(ref)[0].T.numpy()                                # [L, C]
        np.testing.assert_allclose(y[cu[n]:cu[n + 1]], ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(st_out[n], ext[-(K - 1):])


def test_p9_layer_conv_matches_standalone_conv():
    """The full-layer oracle's conv (per head group) equals the standalone conv oracle."""
    dims = oracle.Dims(1, 2, 8, 4, 1.0, 1e-6, 1e-6)
    r = _rng(91)
    T, Cc = 6, dims.channels
    x = r.standard_normal((T, Cc))
    w = r.standard_normal((Cc, 4)) * 0.5
    y, _ = oracle.conv1d_silu(torch.from_numpy(x), torch.from_numpy(w), inputs.cu_seqlens_of([T]))
    # beta = 0, S0 = I-like probe: o_t = exp(G_t) S0 q_t reveals the normalised conv q
    S0 = np.zeros((1, 2, 8, 8), np.float32)
    S0[0, :] = np.eye(8, dtype=np.float32)
    out, _, _ = oracle.prefill(dims, torch.from_numpy(x), torch.zeros(T, 2), torch.zeros(T, 2),
                               inputs.cu_seqlens_of([T]), conv_w=torch.from_numpy(w),
                               S0=torch.from_numpy(S0))
    qn = y[:, :8] / np.sqrt((y[:, :8] ** 2).sum(-1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(out[:, 0], qn, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------------------- P10
def test_p10_gated_rmsnorm_matches_torch():
    r = _rng(10)
    M, d, eps = 17, 128, 1e-6
    o, z, w = r.standard_normal((M, d)), r.standard_normal((M, d)), r.standard_normal(d)
    y = oracle.gated_rmsnorm(torch.from_numpy(o), torch.from_numpy(z), torch.from_numpy(w), eps)
    ref = F.rms_norm(torch.from_numpy(o), (d,), eps=eps) * torch.from_numpy(w) * F.silu(torch.from_numpy(z))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-13)
    # z = 0 gives 0; mean square of y / (w silu z) is m / (m + eps)
    y0 = oracle.gated_rmsnorm(torch.from_numpy(o), torch.zeros(M, d, dtype=torch.float64), None, eps)
    assert np.all(y0 == 0)
    y1 = oracle.gated_rmsnorm(torch.from_numpy(o * 1e-3), torch.from_numpy(z), None, eps)
    m = ((o * 1e-3) ** 2).mean(-1)
    ratio = y1 / (z / (1 + np.exp(-z)))
    np.testing.assert_allclose((ratio ** 2).mean(-1), m / (m + eps), rtol=1e-10)


def test_p10_layer_norm_matches_standalone_norm():
    w = inputs.custom(num_k_heads=1, num_v_heads=2, head_dim=16, dtype=torch.float32, lengths=(5,))
    d = inputs.prefill_inputs(w, 101)
    dims = oracle.Dims(1, 2, 16, 4, 1.0, 1e-6, 1e-6)
    plain = oracle.prefill(dims, d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"])
    normed = oracle.prefill(dims, d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                            z=d["z"], norm_w=d["norm_w"])
    ref = oracle.gated_rmsnorm(torch.from_numpy(plain[0].reshape(-1, 16)),
                               d["z"].double().reshape(-1, 16), d["norm_w"].double(), 1e-6)
    np.testing.assert_allclose(normed[0].reshape(-1, 16), ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------------------- P11
def test_p11_contraction_bound():
    r = _rng(11)
    T, d = 10, 8
    q, k, v = r.standard_normal((T, 1, d)), r.standard_normal((T, 1, d)), r.standard_normal((T, 1, d))
    beta = _f32(r.uniform(0, 1, (T, 1)))
    g = _f32(r.uniform(-0.5, 0, (T, 1)))
    S0 = _f32(r.standard_normal((1, 1, d, d)))
    x = _pack_x(q, k, v)
    prev = np.linalg.norm(S0[0, 0].astype(np.float64))
    for t in range(1, T + 1):
        _, SN, _ = _run(_dims(1, 1, d, l2_eps=1e-6), x[:t], beta[:t], g[:t], S0=S0)
        cur = np.linalg.norm(SN[0, 0])
        bound = np.exp(np.float64(g[t - 1, 0])) * prev + np.float64(beta[t - 1, 0]) * np.linalg.norm(v[t - 1, 0])
        assert cur <= bound * (1 + 1e-12)
        prev = cur


# ------------------------------------------------------------------------------ golden shapes
def test_layer_constants_match_model_card():
    with open(os.path.join(HERE, "golden", "layer_constants.json")) as f:
        c = json.load(f)
    w = inputs.CONFIGS[1]
    assert w.num_k_heads == c["linear_num_key_heads"]
    assert w.num_v_heads == c["linear_num_value_heads"]
    assert w.head_dim == c["linear_key_head_dim"] == c["linear_value_head_dim"]
    assert w.conv_kernel == c["linear_conv_kernel_dim"]
    assert w.dtype == torch.bfloat16 and c["torch_dtype"] == "bfloat16"
    assert oracle.Dims().norm_eps == c["rms_norm_eps"]
    assert inputs.CONFIGS[4].tokens == c["max_position_embeddings"]
    assert inputs.CONFIGS[2].tokens == 40677


# ---------------------------------------------------------------------------------------- P12
def test_p12_block_gates_special_values():
    Hv = 3
    ba = np.zeros((2, 2 * Hv))
    ba[1, :Hv] = [40.0, -40.0, np.log(3.0)]            # b
    ba[1, Hv:] = [60.0, -3.0, 1.5]                     # a
    beta, g = oracle.block_gates(ba, np.zeros(Hv), np.zeros(Hv))
    np.testing.assert_allclose(beta[0], 0.5, rtol=0, atol=0)        # sigmoid(0)
    np.testing.assert_allclose(g[0], -np.log(2.0), rtol=1e-15)      # -softplus(0)
    np.testing.assert_allclose(beta[1], [1.0, 0.0, 0.75], atol=1e-15)
    np.testing.assert_allclose(g[1, 0], -60.0, rtol=1e-15)          # softplus(u) -> u
    # A_log scales, dt_bias shifts: against torch's softplus (library routine)
    rng = _rng(12)
    ba = rng.normal(0, 2, (50, 2 * Hv))
    a_log, dt = rng.normal(0, 1, Hv), rng.normal(0, 1, Hv)
    beta, g = oracle.block_gates(ba, a_log, dt)
    sp = F.softplus(torch.from_numpy(ba[:, Hv:] + dt)).numpy()
    np.testing.assert_allclose(g, -np.exp(a_log) * sp, rtol=1e-12)
    np.testing.assert_allclose(beta + oracle.block_gates(-ba, a_log, dt)[0], 1.0, rtol=1e-14)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))


def test_p12_block_with_identity_projections_is_the_layer():
    d, hk, hv = 8, 1, 2
    dims = _dims(hk, hv, d)
    Cc, T = (2 * hk + hv) * d, 11
    rng = _rng(1212)
    x = rng.normal(0, 1, (T, Cc))
    z = rng.normal(0, 1, (T, hv * d))
    ba = rng.normal(0, 1, (T, 2 * hv))
    H = Cc + hv * d + 2 * hv
    h = np.concatenate([x, z, ba], axis=1)              # the hidden row holds x | z | b a
    eye = np.eye(H)
    w_qkv, w_z, w_ba = eye[:, :Cc], eye[:, Cc:Cc + hv * d], eye[:, Cc + hv * d:]
    a_log, dt = rng.normal(0, 0.5, hv), rng.normal(0, 1, hv)
    w_out = rng.normal(0, 1, (hv * d, 5))
    conv_w = rng.normal(0, 0.5, (Cc, 4))
    norm_w = rng.normal(1, 0.1, d)
    cu = inputs.cu_seqlens_of([4, 7])
    y, SN, convN = oracle.block_prefill(dims, h, w_qkv, w_z, w_ba, a_log, dt, w_out, cu,
                                        conv_w=conv_w, norm_w=norm_w, nthreads=2)
    beta = 1.0 / (1.0 + np.exp(-ba[:, :hv]))
    g = -np.exp(a_log) * F.softplus(torch.from_numpy(ba[:, hv:] + dt)).numpy()
    o, SN2, convN2 = oracle.prefill(dims, torch.from_numpy(x), torch.from_numpy(_f32(beta)),
                                    torch.from_numpy(_f32(g)), cu,
                                    conv_w=torch.from_numpy(conv_w), z=torch.from_numpy(z),
                                    norm_w=torch.from_numpy(norm_w), nthreads=2)
    np.testing.assert_allclose(y, o.reshape(T, -1) @ w_out, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(SN, SN2)
    np.testing.assert_array_equal(convN, convN2)


# --------------------------------------------------------------------------------------- P13
def _scaled_run(dims, x, beta, g, S0=None, **kw):
    return _run(dims, x, beta, g, S0=S0, with_scales=True, **kw)


def test_p13_scales_bound_values_and_leave_results_unchanged():
    r = _rng(131)
    T, d, hk, hv = 9, 8, 1, 2
    q, k, v = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hv, d))
    beta, g = r.uniform(0, 1, (T, hv)), r.uniform(-0.5, 0, (T, hv))
    S0 = _f32(r.standard_normal((1, hv, d, d)))
    x = _pack_x(q, k, v)
    out, SN, convN, osc, M = _scaled_run(_dims(hk, hv, d), x, beta, g, S0=S0)
    out2, SN2, convN2 = _run(_dims(hk, hv, d), x, beta, g, S0=S0)
    assert np.array_equal(out, out2) and np.array_equal(SN, SN2) and np.array_equal(convN, convN2)
    assert np.all(M >= np.abs(SN) * (1 - 1e-12))
    assert np.all(osc >= np.abs(out) * (1 - 1e-12))


def test_p13_single_token_closed_form():
    r = _rng(132)
    d = 8
    q, k, v = r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d))
    beta, g = np.array([[0.6]]), np.array([[-0.3]])
    S0 = _f32(r.standard_normal((1, 1, d, d)))
    out, SN, _, osc, M = _scaled_run(_dims(1, 1, d), _pack_x(q, k, v), beta, g, S0=S0)
    a, b = np.exp(np.float64(_f32(g)[0, 0])), np.float64(_f32(beta)[0, 0])
    kn, qn = np.abs(_unit(k[0, 0])), np.abs(_unit(q[0, 0]))
    S0a = np.abs(S0[0, 0].astype(np.float64))
    M1 = a * S0a + b * np.outer(np.abs(v[0, 0]) + a * S0a @ kn, kn)
    np.testing.assert_allclose(M[0, 0], M1, rtol=1e-12)
    np.testing.assert_allclose(osc[0, 0], M1 @ qn, rtol=1e-12)


def test_p13_no_write_decays_the_magnitude():
    r = _rng(133)
    T, d = 6, 8
    q, k, v = r.standard_normal((T, 1, d)), r.standard_normal((T, 1, d)), r.standard_normal((T, 1, d))
    g = r.uniform(-0.5, 0, (T, 1))
    S0 = _f32(r.standard_normal((1, 1, d, d)))
    _, _, _, _, M = _scaled_run(_dims(1, 1, d), _pack_x(q, k, v), np.zeros((T, 1)), g, S0=S0)
    G = np.sum(_f32(g).astype(np.float64))
    np.testing.assert_allclose(M[0, 0], np.exp(G) * np.abs(S0[0, 0]), rtol=1e-12)


def test_p13_scales_follow_the_magnitude_of_v_and_S0():
    # conv off: scaling the v channels and S0 by 4 scales S, M and the pre-norm scales by 4 and
    # leaves the normalised output and its scale unchanged (up to the norm's eps)
    r = _rng(134)
    T, d, hv = 11, 8, 2
    q, k, v = r.standard_normal((T, 1, d)), r.standard_normal((T, 1, d)), r.standard_normal((T, hv, d))
    beta, g = r.uniform(0, 1, (T, hv)), r.uniform(-0.5, 0, (T, hv))
    S0 = _f32(r.standard_normal((1, hv, d, d)))
    z = torch.from_numpy(r.standard_normal((T, hv, d)))
    dims = _dims(1, hv, d, norm_eps=0.0)
    one = _scaled_run(dims, _pack_x(q, k, v), beta, g, S0=S0, z=z)
    four = _scaled_run(dims, _pack_x(q, k, 4 * v), beta, g, S0=4 * S0, z=z)
    np.testing.assert_allclose(four[4], 4 * one[4], rtol=1e-12)
    np.testing.assert_allclose(four[0], one[0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(four[3], one[3], rtol=1e-10)
    plain_one = _scaled_run(dims, _pack_x(q, k, v), beta, g, S0=S0)
    plain_four = _scaled_run(dims, _pack_x(q, k, 4 * v), beta, g, S0=4 * S0)
    np.testing.assert_allclose(plain_four[3], 4 * plain_one[3], rtol=1e-12)


def test_p13_decode_carries_the_magnitude_like_prefill():
    r = _rng(135)
    T, d, hk, hv = 4, 8, 1, 2
    dims = _dims(hk, hv, d)
    q, k, v = r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hv, d))
    beta, g = r.uniform(0, 1, (T, hv)), r.uniform(-0.5, 0, (T, hv))
    S0 = _f32(r.standard_normal((1, hv, d, d)))
    x = _pack_x(q, k, v)
    cw = torch.from_numpy(r.standard_normal((x.shape[1], 4)))
    pre = oracle.prefill(dims, torch.from_numpy(x), torch.from_numpy(_f32(beta)),
                         torch.from_numpy(_f32(g)), inputs.cu_seqlens_of([T]), conv_w=cw,
                         S0=torch.from_numpy(S0), nthreads=1, with_scales=True)
    S = S0.astype(np.float64).copy()
    M = np.abs(S)
    cs = np.zeros((1, 3, x.shape[1]))
    for t in range(T):
        _, sc = oracle.decode_step(dims, torch.from_numpy(x[t:t + 1]),
                                   torch.from_numpy(_f32(beta[t:t + 1])),
                                   torch.from_numpy(_f32(g[t:t + 1])), cs, S, conv_w=cw, M=M)
        np.testing.assert_allclose(sc[0], pre[3][t], rtol=1e-12)
    np.testing.assert_allclose(M, pre[4], rtol=1e-12)


def test_p13_conv_magnitudes_single_token():
    # conv on, zero history, S0 = 0, T = 1: the conv output of channel c is silu(w[c,3] x[c]) with
    # magnitude 1.1 |w[c,3] x[c]|; q and k magnitudes are divided by the norm of their conv
    # output; M_1 = beta vm km^T and the output scale is M_1 qm
    r = _rng(136)
    d = 8
    q, k, v = r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d))
    x = _pack_x(q, k, v)
    w = r.standard_normal((x.shape[1], 4))
    beta, g = np.array([[0.7]]), np.array([[-0.2]])
    dims = _dims(1, 1, d)
    out, SN, _, osc, M = oracle.prefill(
        dims, torch.from_numpy(x), torch.from_numpy(_f32(beta)), torch.from_numpy(_f32(g)),
        inputs.cu_seqlens_of([1]), conv_w=torch.from_numpy(w), nthreads=1, with_scales=True)
    acc = w[:, 3] * x[0]
    silu = acc / (1 + np.exp(-acc))
    mag = 1.1 * np.abs(acc)
    qm = mag[:d] / np.linalg.norm(silu[:d])
    km = mag[d:2 * d] / np.linalg.norm(silu[d:2 * d])
    vm = mag[2 * d:]
    b = np.float64(_f32(beta)[0, 0])
    M1 = b * np.outer(vm, km)
    np.testing.assert_allclose(M[0, 0], M1, rtol=1e-12)
    np.testing.assert_allclose(osc[0, 0], M1 @ qm, rtol=1e-12)
    assert np.all(M[0, 0] >= np.abs(SN[0, 0]) * (1 - 1e-12))
