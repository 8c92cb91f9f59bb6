"""Multi-token decode (verification of speculative draft tokens): k tokens per sequence in one
call equal k one-token steps, on the GPU (bit for bit) and against the fp64 oracle; the state
snapshot after each token equals the oracle state after that token."""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, dims_of, ensure_built, np64, oracle_dims_of

pytestmark = pytest.mark.gpu


def _workload(dtype, B, Hk=16, Hv=32):
    return inputs.Workload("decode_multi", "decode", Hk, Hv, 128, dtype, batch=B, steps=8,
                           s0_std=0.1)


def _token_inputs(w, seed, k):
    steps = [inputs.decode_step_inputs(w, seed, t) for t in range(k)]
    stack = lambda key: torch.stack([s[key] for s in steps], dim=1).contiguous()  # noqa: E731
    return {key: stack(key) for key in ("x", "beta", "g", "z")}, steps


@pytest.mark.parametrize("dtype,k", [(torch.bfloat16, 4), (torch.bfloat16, 1), (torch.bfloat16, 8),
                                     (torch.float32, 3)])
def test_multi_equals_single_steps_and_oracle(dtype, k):
    ensure_built()
    w = _workload(dtype, B=12)
    seed = 4100 + k
    st = inputs.decode_state(w, seed)
    toks, steps = _token_inputs(w, seed, k)
    cw, nw = dev(st["conv_w"]), dev(st["norm_w"])
    dims = dims_of(w)
    # reversed slots: sequence b lives in slot B - 1 - b
    B = w.batch
    slot = torch.arange(B - 1, -1, -1, dtype=torch.int32)
    S_pool, cs_pool = st["S"].clone(), st["conv_state"].clone()
    S_m, cs_m = dev(S_pool), dev(cs_pool)
    S_s, cs_s = dev(S_pool), dev(cs_pool)
    snaps = torch.empty((B, k, w.num_v_heads, 128, 128), dtype=torch.float32, device="cuda")
    out_m = gdn.decode_multi(dev(toks["x"]), dev(toks["beta"]), dev(toks["g"]), cs_m, S_m, cw,
                             z=dev(toks["z"]), norm_w=nw, slot_idx=dev(slot), snapshots=snaps,
                             dims=dims)
    outs = []
    for t in range(k):
        s = steps[t]
        outs.append(gdn.decode_step(dev(s["x"]), dev(s["beta"]), dev(s["g"]), cs_s, S_s, cw,
                                    z=dev(s["z"]), norm_w=nw, slot_idx=dev(slot), dims=dims))
    torch.cuda.synchronize()
    # one call of k tokens = k calls of one token, to the bit
    assert torch.equal(out_m, torch.stack(outs, dim=1))
    assert torch.equal(S_m, S_s) and torch.equal(cs_m, cs_s)
    # and the oracle, token by token, with the snapshots
    od = oracle_dims_of(w)
    S_ref = S_pool.double().numpy()[slot.long().numpy()].copy()
    cs_ref = cs_pool.double().numpy()[slot.long().numpy()].copy()
    M_ref = np.abs(S_ref)
    for t in range(k):
        s = steps[t]
        ref, sc = oracle.decode_step(od, s["x"], s["beta"], s["g"], cs_ref, S_ref,
                                     conv_w=st["conv_w"], z=s["z"], norm_w=st["norm_w"], M=M_ref)
        assert_close(out_m[:, t], ref, dtype, f"k={k} token {t}: out", scale=sc)
        assert_close(snaps[:, t], S_ref, dtype, f"k={k} token {t}: state snapshot", scale=M_ref)
    assert_close(S_m[slot.long()], S_ref, dtype, f"k={k}: final state", scale=M_ref)
    np.testing.assert_array_equal(np64(cs_m[slot.long()]), cs_ref)
