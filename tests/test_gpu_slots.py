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
    ref = oracle_prefill(w, inp)
    assert_close(out_s, ref[0], dtype, "slots: out", scale=ref.out_scale)
    assert_close(S_pool[slot.long()], ref[1], dtype, "slots: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(conv_pool[slot.long()].float().cpu().double().numpy(), ref[2])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_slot_out_of_range_is_skipped_and_reported(dtype):
    # slots 9 and -1 lie outside a pool of 6 rows: those sequences start from zero states, write
    # no state, and the call reports GDN_ERR_INVALID_ARG; the others are unaffected
    ensure_built()
    lengths, slots, n_slots = (130, 7, 5, 257), [4, 9, 0, -1], 6
    w = inputs.custom(2, 4, 128, dtype, lengths=lengths)
    inp = inputs.prefill_inputs(w, 1310 + (dtype == torch.float32))
    Hv, d, Cc = w.num_v_heads, w.head_dim, w.channels
    gen = torch.Generator().manual_seed(1311)
    S_pool = (0.1 * torch.randn(n_slots, Hv, d, d, generator=gen)).cuda()
    conv_pool = torch.randn(n_slots, 3, Cc, generator=gen).to(dtype).cuda()
    slot = torch.tensor(slots, dtype=torch.int32).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S_before, conv_before = S_pool.clone(), conv_pool.clone()
    out_s = gdn.chunk_prefill_slots(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]), S_pool,
        slot_idx=slot, conv_pool=conv_pool, conv_w=dev(inp["conv_w"]), z=dev(inp["z"]),
        norm_w=dev(inp["norm_w"]), dev_status=status, dims=dims_of(w))
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_INVALID_ARG
    valid = [n for n, s in enumerate(slots) if 0 <= s < n_slots]
    S0 = torch.zeros(len(slots), Hv, d, d, device="cuda")
    conv0 = torch.zeros(len(slots), 3, Cc, dtype=dtype, device="cuda")
    for n in valid:
        S0[n], conv0[n] = S_before[slots[n]], conv_before[slots[n]]
    out_d, SN_d, convN_d = gdn.chunk_prefill(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]),
        conv_w=dev(inp["conv_w"]), z=dev(inp["z"]), norm_w=dev(inp["norm_w"]), S0=S0,
        conv0=conv0, dims=dims_of(w))
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_d)
    for n in valid:
        assert torch.equal(S_pool[slots[n]], SN_d[n])
        assert torch.equal(conv_pool[slots[n]], convN_d[n])
    others = [i for i in range(n_slots) if i not in slots]
    assert torch.equal(S_pool[others], S_before[others])
    assert torch.equal(conv_pool[others], conv_before[others])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_slot_out_of_range_is_skipped_and_reported(dtype):
    ensure_built()
    dims = gdn.Dims(2, 4)
    B, n_slots, Cc = 4, 5, dims.channels
    gen = torch.Generator().manual_seed(1320)
    S = (0.1 * torch.randn(n_slots, 4, 128, 128, generator=gen)).cuda()
    cs = torch.randn(n_slots, 3, Cc, generator=gen).to(dtype).cuda()
    x = torch.randn(B, Cc, generator=gen).to(dtype).cuda()
    beta = torch.sigmoid(torch.randn(B, 4, generator=gen)).cuda()
    g = -torch.rand(B, 4, generator=gen).cuda()
    w = (0.5 * torch.randn(Cc, 4, generator=gen)).to(dtype).cuda()
    good = torch.tensor([3, 0, 1, 4], dtype=torch.int32).cuda()
    bad = torch.tensor([3, 5, 1, -2], dtype=torch.int32).cuda()
    S_ref, cs_ref = S.clone(), cs.clone()
    o_ref = gdn.decode_step(x, beta, g, cs_ref, S_ref, w, slot_idx=good, dims=dims)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((B, 4, 128), 7.0, dtype=dtype, device="cuda")
    S_before, cs_before = S.clone(), cs.clone()
    gdn.decode_step(x, beta, g, cs, S, w, slot_idx=bad, out=out, dev_status=status, dims=dims)
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_INVALID_ARG
    for b in (0, 2):   # valid sequences: as with a good slot map
        assert torch.equal(out[b], o_ref[b])
        s = int(good[b])
        assert torch.equal(S[s], S_ref[s]) and torch.equal(cs[s], cs_ref[s])
    for b in (1, 3):   # skipped: output rows untouched
        assert torch.all(out[b] == 7.0)
    for s in (0, 2, 4):  # rows no valid sequence maps to: untouched
        assert torch.equal(S[s], S_before[s]) and torch.equal(cs[s], cs_before[s])
