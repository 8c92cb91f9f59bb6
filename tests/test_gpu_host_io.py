"""GPU checks of gdn_chunk_prefill_host (per-token tensors in host memory, copies overlapped
with the layer segment by segment): bit for bit the device call when every segment holds one
sequence, the oracle's result on a ragged batch with initial states, and pageable buffers."""
import numpy as np
import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, dims_of, ensure_built, gpu_prefill, oracle_prefill

pytestmark = pytest.mark.gpu


def _host_run(w, inp, seg, pin=True):
    ensure_built()
    h = (lambda t: None if t is None else (t.pin_memory() if pin else t.clone()))
    z = inp["z"]
    out, SN, convN = gdn.chunk_prefill_host(
        h(inp["x"]), h(inp["beta"]), h(inp["g"]), inp["cu_seqlens"], conv_w=dev(inp["conv_w"]),
        z=h(z.reshape(z.shape[0], -1)) if z is not None else None, norm_w=dev(inp["norm_w"]),
        S0=dev(inp["S0"]), conv0=dev(inp["conv0"]), segment_tokens=seg, dims=dims_of(w))
    torch.cuda.synchronize()
    return out, SN, convN


@pytest.mark.parametrize("seg", [128, 256, 0])
def test_host_single_sequence_equals_device_call(seg):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(1000,), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1400 + seg, with_conv0=True)
    out_h, SN_h, conv_h = _host_run(w, inp, seg)
    out_d, SN_d, conv_d = gpu_prefill(w, inp)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(SN_h, SN_d)
    assert torch.equal(conv_h, conv_d)


@pytest.mark.parametrize("seg", [128, 384])
def test_host_ragged_batch_against_oracle(seg):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(1, 0, 130, 2, 257, 0, 64, 300),
                      s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1500 + seg, with_conv0=True)
    out, SN, convN = _host_run(w, inp, seg)
    ref = oracle_prefill(w, inp)
    assert_close(out, ref[0], w.dtype, f"host seg={seg}: out", scale=ref.out_scale)
    assert_close(SN, ref[1], w.dtype, f"host seg={seg}: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(convN.float().cpu().double().numpy(), ref[2])


def test_host_pageable_buffers_and_model_heads():
    w = inputs.custom(16, 32, 128, torch.bfloat16, lengths=(700, 129))
    inp = inputs.prefill_inputs(w, 1600)
    out, SN, convN = _host_run(w, inp, 256, pin=False)
    ref = oracle_prefill(w, inp)
    assert_close(out, ref[0], w.dtype, "pageable: out", scale=ref.out_scale)
    assert_close(SN, ref[1], w.dtype, "pageable: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(convN.float().cpu().double().numpy(), ref[2])
