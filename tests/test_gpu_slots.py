"""GPU checks of gdn_chunk_prefill_slots: a prefill whose initial and final states sit in pools
shared with decode.  It must equal gdn_chunk_prefill on the gathered states bit for bit, leave
the other pool rows untouched, and match the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, dims_of, ensure_built, oracle_prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_slots_equal_gathered_dense_call(dtype):
    ensure_built()
    lengths, slots, n_slots = (130, 0, 5, 257), [4, 1, 0, 2], 6
    w = inputs.custom(2, 4, 128, dtype, lengths=lengths)
    inp = inputs.prefill_inputs(w, 1300 + (dtype == torch.float32))
    Hv, d, Cc = w.num_v_heads, w.head_dim, w.channels
    gen = torch.Generator().manual_seed(1301)
    S_pool = (0.1 * torch.randn(n_slots, Hv, d, d, generator=gen)).cuda()
    conv_pool = torch.randn(n_slots, 3, Cc, generator=gen).to(dtype).cuda()
    slot = torch.tensor(slots, dtype=torch.int32).cuda()
    S_before, conv_before = S_pool.clone(), conv_pool.clone()
    out_s = gdn.chunk_prefill_slots(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]), S_pool,
        slot_idx=slot, conv_pool=conv_pool, conv_w=dev(inp["conv_w"]), z=dev(inp["z"]),
        norm_w=dev(inp["norm_w"]), dims=dims_of(w))
    S0, conv0 = S_before[slot.long()].contiguous(), conv_before[slot.long()].contiguous()
    out_d, SN_d, convN_d = gdn.chunk_prefill(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]),
        conv_w=dev(inp["conv_w"]), z=dev(inp["z"]), norm_w=dev(inp["norm_w"]), S0=S0,
        conv0=conv0, dims=dims_of(w))
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_d)
    assert torch.equal(S_pool[slot.long()], SN_d)
    assert torch.equal(conv_pool[slot.long()], convN_d)
    others = [i for i in range(n_slots) if i not in slots]
    assert torch.equal(S_pool[others], S_before[others])
    assert torch.equal(conv_pool[others], conv_before[others])
    # and against the oracle on the gathered states
    inp = dict(inp, S0=S0.cpu(), conv0=conv0.cpu())
    ref_o, ref_S, ref_c = oracle_prefill(w, inp)
    assert_close(out_s, ref_o, dtype, "slots: out")
    assert_close(S_pool[slot.long()], ref_S, dtype, "slots: final state")
    np.testing.assert_array_equal(conv_pool[slot.long()].float().cpu().double().numpy(), ref_c)
