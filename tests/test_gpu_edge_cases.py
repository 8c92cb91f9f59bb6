"""GPU parity on the degenerate and extreme cases of the gated delta rule, at the Qwen3-Next head
layout (16 key heads, 32 value heads, d = 128), through the bf16 chunked prefill, the fp32
prefill and the decode step, each against the fp64 oracle (whose behaviour in these cases is
pinned on the CPU by tests/test_oracle_pins.py):

  beta0    beta = 0: no write, the state only decays (S_t = exp(sum g) S_0)
  alpha1   g = 0 (alpha = 1): no decay; exp(G_i - G_j) = 1 across every 128-token chunk
  ortho    alpha = beta = 1, keys = Hadamard rows (exactly orthogonal in bf16), conv and norm off:
           the query k_{t-5} returns v_{t-5}, also checked against that closed form
  decay20  g ~ U(-25, -15) per token: exp(G_i - G_j) underflows to 0 inside a chunk
  large    x and S_0 scaled by 64 (exact in bf16): v and the state 64x the workload's size

The recurrence these follow is the delta rule of the hyper.ai Qwen3-Next paragraph: beta sets
how strongly each token's value overwrites what the state returns for its key (kv_mem), alpha
decays the whole state.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import (assert_close, dev, dims_of, ensure_built, gpu_prefill, np64,
                      oracle_dims_of, oracle_prefill)

pytestmark = pytest.mark.gpu

HK, HV, D = 16, 32, 128
CASES = ["beta0", "alpha1", "ortho", "decay20", "large"]
SCALE = {"large": 64.0}
LAG = 5


def _hadamard(n):
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _edge_prefill_inputs(case, dtype, lengths, seed):
    ortho = case == "ortho"
    w = inputs.custom(HK, HV, D, dtype, lengths=lengths, conv=not ortho, norm=not ortho,
                      s0_std=0.0 if ortho else 0.1)
    inp = inputs.prefill_inputs(w, seed, with_conv0=not ortho)
    T = w.tokens
    if case == "beta0":
        inp["beta"].zero_()
    elif case == "alpha1":
        inp["g"].zero_()
    elif case == "decay20":
        rng = np.random.default_rng(seed)
        inp["g"] = torch.from_numpy(rng.uniform(-25.0, -15.0, (T, HV)).astype(np.float32))
    elif case == "large":
        inp["x"] = (inp["x"].float() * 64).to(dtype)
        inp["S0"] = inp["S0"] * 64
    elif case == "ortho":
        inp["beta"].fill_(1.0)
        inp["g"].zero_()
        H = _hadamard(D)
        x = inp["x"].float().numpy()
        starts = np.cumsum([0] + list(lengths))
        for n, L in enumerate(lengths):
            for j in range(L):
                t = int(starts[n]) + j
                for hk in range(HK):
                    key = H[(j + 7 * hk) % D]
                    x[t, (HK + hk) * D:(HK + hk + 1) * D] = key
                    # query: the key written LAG tokens earlier in the same sequence (or its own)
                    jq = j - LAG if j >= LAG else j
                    x[t, hk * D:(hk + 1) * D] = H[(jq + 7 * hk) % D]
        inp["x"] = torch.from_numpy(x).to(dtype)
    return w, inp


def _ortho_closed_form(inp, lengths):
    """o_t = v_{t-LAG} (v_t for the first LAG tokens of a sequence): with alpha = beta = 1 and
    keys orthogonal inside every window of 128 tokens, the state returns the value last written
    under the queried key."""
    x = inp["x"].double().numpy()
    v = x[:, 2 * HK * D:].reshape(-1, HV, D)
    ref = np.empty_like(v)
    starts = np.cumsum([0] + list(lengths))
    for n, L in enumerate(lengths):
        for j in range(L):
            t = int(starts[n]) + j
            ref[t] = v[t - LAG] if j >= LAG else v[t]
    return ref


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("case", CASES)
def test_prefill_edge_case(case, dtype):
    lengths = (300, 130) if dtype == torch.bfloat16 else (200,)
    w, inp = _edge_prefill_inputs(case, dtype, lengths, 5000 + CASES.index(case))
    out, SN, convN = gpu_prefill(w, inp)
    ref = oracle_prefill(w, inp)
    ref_o = ref[0]
    s = SCALE.get(case, 1.0)
    tag = f"{case} {'bf16' if dtype == torch.bfloat16 else 'f32'} prefill"
    assert_close(out, ref_o, dtype, f"{tag}: out", scale=ref.out_scale, f32_scale=s)
    assert_close(SN, ref[1], dtype, f"{tag}: final state", scale=ref.SN_scale, f32_scale=s)
    if w.conv:
        np.testing.assert_array_equal(np64(convN), ref[2])
    if case == "beta0":
        # no write: the state only decays, S_T = exp(sum_t g_t) S_0 per (sequence, value head)
        cu = inp["cu_seqlens"].numpy()
        g = inp["g"].double().numpy()
        S0 = inp["S0"].double().numpy()
        for n in range(len(lengths)):
            decay = np.exp(g[cu[n]:cu[n + 1]].sum(axis=0))
            assert_close(SN[n], decay[:, None, None] * S0[n], dtype, f"{tag}: closed-form state",
                         scale=ref.SN_scale[n])
    if case == "ortho":
        assert_close(out, _ortho_closed_form(inp, lengths), dtype, f"{tag}: retrieval",
                     scale=ref.out_scale)


def _decode_workload(dtype):
    return inputs.Workload("edge_decode", "decode", HK, HV, D, dtype, batch=64, steps=4,
                           s0_std=0.1)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("case", ["beta0", "alpha1", "decay20", "large"])
def test_decode_edge_case(case, dtype):
    ensure_built()
    w = _decode_workload(dtype)
    seed = 5100 + CASES.index(case)
    st = inputs.decode_state(w, seed)
    s = SCALE.get(case, 1.0)
    S = st["S"] * s
    S_d, cs_d = dev(S), dev(st["conv_state"])
    S_ref = S.double().numpy().copy()
    M_ref = np.abs(S_ref)
    cs_ref = st["conv_state"].double().numpy().copy()
    cw, nw = dev(st["conv_w"]), dev(st["norm_w"])
    dims, od = dims_of(w), oracle_dims_of(w)
    for step in range(w.steps):
        si = inputs.decode_step_inputs(w, seed, step)
        if case == "beta0":
            si["beta"].zero_()
        elif case == "alpha1":
            si["g"].zero_()
        elif case == "decay20":
            rng = np.random.default_rng(seed + step)
            si["g"] = torch.from_numpy(rng.uniform(-25.0, -15.0, (w.batch, HV)).astype(np.float32))
        elif case == "large":
            si["x"] = (si["x"].float() * 64).to(dtype)
        out = gdn.decode_step(dev(si["x"]), dev(si["beta"]), dev(si["g"]), cs_d, S_d, cw,
                              z=dev(si["z"]), norm_w=nw, dims=dims)
        torch.cuda.synchronize()
        ref, sc = oracle.decode_step(od, si["x"], si["beta"], si["g"], cs_ref, S_ref,
                                     conv_w=st["conv_w"], z=si["z"], norm_w=st["norm_w"], M=M_ref)
        assert_close(out, ref, dtype, f"{case} decode out step {step}", scale=sc, f32_scale=s)
    assert_close(S_d, S_ref, dtype, f"{case} decode state after {w.steps} steps", scale=M_ref,
                 f32_scale=s)
    np.testing.assert_array_equal(np64(cs_d), cs_ref)
