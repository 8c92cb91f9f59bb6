"""GPU parity on the five workload configurations at full size (the launch configuration the
benchmark times), against the fp64 oracle on the same seeded inputs.

  tiny fp32 T=128 (Hk=2, Hv=4, conv/norm off)   max-abs <= 1e-4 on outputs and final state
  T=4096 prefill, Qwen3-Next layer shape         element-wise (tests/gpu_util.py)
  8-sequence packed varlen prefill, S0 ~ N(0,.1) element-wise, final states returned
  decode, 256 sequences x 64 steps               outputs every step, states after step 64
  T=262144 prefill, slow decay                   last 4096 outputs and the final state
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


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_prefill_config(idx):
    w = inputs.CONFIGS[idx]
    inp = inputs.prefill_inputs(w, inputs.config_seed(idx))
    out, SN, convN = gpu_prefill(w, inp)
    ref = oracle_prefill(w, inp)
    e_o = assert_close(out, ref[0], w.dtype, f"{w.name}: out", scale=ref.out_scale)
    e_s = assert_close(SN, ref[1], w.dtype, f"{w.name}: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(np64(convN), ref[2])
    print(f"{w.name}: out err {e_o:.3g}, state err {e_s:.3g}")


@pytest.mark.slow
def test_long_context_config():
    w = inputs.CONFIGS[4]
    inp = inputs.prefill_inputs(w, inputs.config_seed(4))
    out, SN, _ = gpu_prefill(w, inp, want_state=True)
    T = w.tokens
    tail = out[T - 4096:].cpu()
    del out
    torch.cuda.empty_cache()
    ref = oracle_prefill(w, inp, out_t0=T - 4096)
    e_o = assert_close(tail, ref[0], w.dtype, "T=262144: last 4096 outputs", scale=ref.out_scale)
    e_s = assert_close(SN, ref[1], w.dtype, "T=262144: final state", scale=ref.SN_scale)
    print(f"{w.name}: out err {e_o:.3g}, state err {e_s:.3g}")


def test_decode_config():
    ensure_built()
    w = inputs.CONFIGS[3]
    seed = inputs.config_seed(3)
    st = inputs.decode_state(w, seed)
    S_d, cs_d = dev(st["S"]), dev(st["conv_state"])
    S_ref = st["S"].double().numpy().copy()
    M_ref = np.abs(S_ref)
    cs_ref = st["conv_state"].double().numpy().copy()
    cw, nw = dev(st["conv_w"]), dev(st["norm_w"])
    dims, od = dims_of(w), oracle_dims_of(w)
    worst = 0.0
    for step in range(w.steps):
        s = inputs.decode_step_inputs(w, seed, step)
        out = gdn.decode_step(dev(s["x"]), dev(s["beta"]), dev(s["g"]), cs_d, S_d, cw,
                              z=dev(s["z"]), norm_w=nw, dims=dims)
        torch.cuda.synchronize()
        ref, sc = oracle.decode_step(od, s["x"], s["beta"], s["g"], cs_ref, S_ref,
                                     conv_w=st["conv_w"], z=s["z"], norm_w=st["norm_w"], M=M_ref)
        worst = max(worst, assert_close(out, ref, w.dtype, f"decode out step {step}", scale=sc))
    e_s = assert_close(S_d, S_ref, w.dtype, "decode state after 64 steps", scale=M_ref)
    np.testing.assert_array_equal(np64(cs_d), cs_ref)
    print(f"decode: worst out err {worst:.3g}, state err {e_s:.3g}")


def test_decode_config_bf16_state():
    # the decode workload with the recurrent state stored in bf16: the oracle state is rounded to
    # bf16 after every step, as the kernel stores it (fp32 arithmetic in between)
    ensure_built()
    w = inputs.CONFIGS[3]
    seed = inputs.config_seed(3)
    st = inputs.decode_state(w, seed)
    S_d = dev(st["S"]).to(torch.bfloat16)
    cs_d = dev(st["conv_state"])
    S_ref = S_d.double().cpu().numpy().copy()
    M_ref = np.abs(S_ref)
    cs_ref = st["conv_state"].double().numpy().copy()
    cw, nw = dev(st["conv_w"]), dev(st["norm_w"])
    dims, od = dims_of(w), oracle_dims_of(w)
    worst = 0.0
    for step in range(16):
        s = inputs.decode_step_inputs(w, seed, step)
        out = gdn.decode_step(dev(s["x"]), dev(s["beta"]), dev(s["g"]), cs_d, S_d, cw,
                              z=dev(s["z"]), norm_w=nw, dims=dims)
        torch.cuda.synchronize()
        ref, sc = oracle.decode_step(od, s["x"], s["beta"], s["g"], cs_ref, S_ref,
                                     conv_w=st["conv_w"], z=s["z"], norm_w=st["norm_w"], M=M_ref)
        S_ref[...] = torch.from_numpy(S_ref).to(torch.bfloat16).double().numpy()
        worst = max(worst, assert_close(out, ref, w.dtype, f"bf16-state decode out step {step}",
                                        scale=sc))
    assert S_d.dtype == torch.bfloat16
    e_s = assert_close(S_d, S_ref, torch.bfloat16, "bf16 decode state after 16 steps",
                       scale=M_ref)
    np.testing.assert_array_equal(np64(cs_d), cs_ref)
    print(f"bf16-state decode: worst out err {worst:.3g}, state err {e_s:.3g}")
