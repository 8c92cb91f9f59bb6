"""GPU parity of gdn_block_prefill (input projections, gates, layer, output projection)
against the fp64 oracle's token mixer: small heads over ragged sequences with states, the
model's own head counts and hidden size, and a call without tokens that carries the states."""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, dims_of, ensure_built, oracle_dims_of

pytestmark = pytest.mark.gpu


def _run(w, hidden, seed, with_conv0=False):
    ensure_built()
    inp = inputs.block_inputs(w, seed, hidden, with_conv0=with_conv0)
    y, SN, convN = gdn.block_prefill(
        dev(inp["h"]), dev(inp["w_qkv"]), dev(inp["w_z"]), dev(inp["w_ba"]), dev(inp["a_log"]),
        dev(inp["dt_bias"]), dev(inp["w_out"]), dev(inp["cu_seqlens"]), conv_w=dev(inp["conv_w"]),
        norm_w=dev(inp["norm_w"]), S0=dev(inp["S0"]), conv0=dev(inp["conv0"]), dims=dims_of(w))
    torch.cuda.synchronize()
    ref = oracle.block_prefill(oracle_dims_of(w), inp["h"], inp["w_qkv"], inp["w_z"],
                               inp["w_ba"], inp["a_log"], inp["dt_bias"], inp["w_out"],
                               inp["cu_seqlens"], conv_w=inp["conv_w"], norm_w=inp["norm_w"],
                               S0=inp["S0"], conv0=inp["conv0"], with_scales=True)
    return (y, SN, convN), ref


def _check(got, ref, what):
    # x leaves the projection rounded to bf16, so the conv history (no element scale of its own:
    # it is x itself) is compared against the tensor's RMS plus one rounding
    y_ref, S_ref, c_ref, y_scale, S_scale = ref
    assert_close(got[0], y_ref, torch.bfloat16, f"{what}: y", scale=y_scale)
    assert_close(got[1], S_ref, torch.bfloat16, f"{what}: final state", scale=S_scale)
    assert_close(got[2], c_ref, torch.bfloat16, f"{what}: conv history")


@pytest.mark.parametrize("lengths", [(300, 129), (1, 0, 130, 64)])
def test_block_small_heads(lengths):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=lengths, s0_std=0.1)
    got, ref = _run(w, 256, 4100 + len(lengths), with_conv0=True)
    _check(got, ref, f"lengths={lengths}")


def test_block_model_heads_and_hidden():
    w = inputs.custom(16, 32, 128, torch.bfloat16, lengths=(384, 200))
    got, ref = _run(w, 2048, 4200)
    _check(got, ref, "16/32 heads, hidden 2048")


def test_block_without_tokens_carries_states():
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(0, 0), s0_std=0.1)
    (y, SN, convN), ref = _run(w, 256, 4300, with_conv0=True)
    inp = inputs.block_inputs(w, 4300, 256, with_conv0=True)
    assert y.numel() == 0
    np.testing.assert_array_equal(SN.cpu().numpy(), inp["S0"].numpy())
    assert torch.equal(convN.cpu(), inp["conv0"])
