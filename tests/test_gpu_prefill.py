"""GPU parity of gdn_chunk_prefill against the fp64 oracle on small and edge-case inputs:
ragged tails around the 128-token chunk, sequences shorter than the conv window, empty
sequences, initial states, conv/norm switched off, every chain split, determinism."""
import numpy as np
import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, dims_of, gpu_prefill, np64, oracle_prefill

pytestmark = pytest.mark.gpu


def _check(w, inp, what):
    out, SN, convN = gpu_prefill(w, inp)
    ref = oracle_prefill(w, inp)
    e1 = assert_close(out, ref[0], w.dtype, f"{what}: out", scale=ref.out_scale)
    e2 = assert_close(SN, ref[1], w.dtype, f"{what}: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(np64(convN), ref[2])
    return e1, e2


@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65, 127, 128, 129, 300])
def test_bf16_single_sequence_lengths(T):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(T,))
    _check(w, inputs.prefill_inputs(w, 500 + T), f"T={T}")


@pytest.mark.parametrize("T", [1, 3, 129, 300])
def test_f32_single_sequence_lengths(T):
    w = inputs.custom(2, 4, 128, torch.float32, lengths=(T,))
    _check(w, inputs.prefill_inputs(w, 600 + T), f"f32 T={T}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_varlen_with_states_and_empty_sequences(dtype):
    w = inputs.custom(2, 4, 128, dtype, lengths=(1, 0, 130, 2, 257, 0, 64), s0_std=0.1)
    _check(w, inputs.prefill_inputs(w, 700, with_conv0=True), "varlen")


@pytest.mark.parametrize("conv,norm", [(False, True), (True, False), (False, False)])
def test_bf16_conv_and_norm_switches(conv, norm):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(200,), conv=conv, norm=norm)
    _check(w, inputs.prefill_inputs(w, 800 + 2 * conv + norm), f"conv={conv} norm={norm}")


@pytest.mark.parametrize("nseq", [1, 20, 40])
def test_bf16_every_chain_split(nseq):
    # N*Hv units decide the d_v split of the chain kernel: 4 -> 4 blocks, 80 -> 2, 160 -> 1
    lengths = tuple(int(v) for v in np.random.default_rng(900 + nseq).integers(1, 300, nseq))
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=lengths, s0_std=0.1)
    _check(w, inputs.prefill_inputs(w, 900 + nseq), f"nseq={nseq}")


def test_bf16_long_memory_gates():
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(1000,), g_dist="uniform", g_low=-0.05,
                      s0_std=0.1)
    _check(w, inputs.prefill_inputs(w, 950), "slow decay")


def test_bf16_state_in_place_and_deterministic():
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(77, 300), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 960, with_conv0=True)
    a = gpu_prefill(w, inp)
    b = gpu_prefill(w, inp)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    # S0 == SN and conv0 == convN (in-place state update)
    S = inp["S0"].cuda()
    c = inp["conv0"].cuda()
    out, _, _ = gdn.chunk_prefill(inp["x"].cuda(), inp["beta"].cuda(), inp["g"].cuda(),
                                  inp["cu_seqlens"].cuda(), conv_w=inp["conv_w"].cuda(),
                                  z=inp["z"].cuda(), norm_w=inp["norm_w"].cuda(), S0=S, SN=S,
                                  conv0=c, convN=c, dims=gdn.Dims(2, 4))
    torch.cuda.synchronize()
    assert torch.equal(out, a[0])
    assert torch.equal(S, a[1])
    assert torch.equal(c, a[2])


def test_split_prefill_matches_whole():
    """prefill(0..T) == prefill(0..T1) then prefill(T1..T) with the carried states."""
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(390,), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 970, with_conv0=True)
    full = gpu_prefill(w, inp)
    T1 = 200
    first = {k: v for k, v in inp.items()}
    second = {k: v for k, v in inp.items()}
    for k in ("x", "beta", "g", "z"):
        first[k], second[k] = inp[k][:T1], inp[k][T1:]
    first["cu_seqlens"] = inputs.cu_seqlens_of([T1])
    second["cu_seqlens"] = inputs.cu_seqlens_of([390 - T1])
    a = gpu_prefill(w, first)
    second["S0"], second["conv0"] = a[1].cpu(), a[2].cpu()
    b = gpu_prefill(w, second)
    ref = oracle_prefill(w, inp)
    assert_close(torch.cat([a[0], b[0]]), ref[0], w.dtype, "split out", scale=ref.out_scale)
    assert_close(b[1], ref[1], w.dtype, "split state", scale=ref.SN_scale)
    assert torch.equal(b[2], full[2])


@pytest.mark.parametrize("seg", [1, 2, 3, 5])
@pytest.mark.parametrize("split", [1, 2, 4])
def test_bf16_pipelined_segments(seg, split):
    # Segments of `seg` chunks: sequences cross segment boundaries (the state is carried in
    # fp32 between launches), short and empty sequences fall inside one segment, and the
    # chain's d_v split is forced so that every split meets every boundary case.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(700, 0, 5, 129, 0, 1100, 64, 260),
                      s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1200 + 10 * seg + split, with_conv0=True)
    with gdn.debug_options(segment_chunks=seg, chain_split=split):
        _check(w, inp, f"seg={seg} split={split}")


def test_bf16_pipelined_matches_single_launch_bitwise():
    # The pipeline reorders launches only: with the same split, the segmented and the single
    # launch runs perform the same arithmetic and must agree to the bit.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(900, 33, 1500), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1300, with_conv0=True)
    with gdn.debug_options(segment_chunks=1 << 19, chain_split=2):
        one = gpu_prefill(w, inp)
    with gdn.debug_options(segment_chunks=2, chain_split=2):
        seg = gpu_prefill(w, inp)
    for a, b, name in zip(one, seg, ("out", "final state", "conv state")):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("segmented", [False, True])
@pytest.mark.parametrize("split", [0, 2, 1])
def test_chain_wait_runs_out_and_the_context_stays_usable(segmented, split):
    # A load the chain waits for is left out on purpose (debug fault injection): the chain's
    # bounded wait must run out within its limit (5 ms here), write GDN_ERR_TIMEOUT, let its
    # other copies land (TMA loads, and with d_v blocks of 64 or 128 the TMA stores of S and U),
    # free its TMEM and end; afterwards the same stream runs a normal prefill that matches the
    # one before the fault bit for bit.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(700, 300), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1350, with_conv0=True)
    seg = 2 if segmented else 0
    with gdn.debug_options(segment_chunks=seg, chain_split=split):
        good = gpu_prefill(w, inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    import time
    t0 = time.perf_counter()
    with gdn.debug_options(wait_limit_us=5000, segment_chunks=seg, chain_split=split,
                           fault=gdn.GDN_FAULT_SKIP_CHAIN_LOAD, fault_chunk=2):
        gpu_prefill(w, inp, dev_status=status)
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == gdn.GDN_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed     # gave up after its 5 ms limit, not the 2 s default
    with gdn.debug_options(segment_chunks=seg, chain_split=split):
        again = gpu_prefill(w, inp)
    for a, b, name in zip(good, again, ("out", "final state", "conv state")):
        assert torch.equal(a, b), name


def test_bf16_states_updated_in_place():
    # SN = S0 and convN = conv0: the call reads the initial states and overwrites them, as a
    # serving loop does; the conv history then comes from its own kernel after the layer.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 0, 2, 129), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1500, with_conv0=True)
    ref = oracle_prefill(w, inp)
    S = dev(inp["S0"]).clone()
    conv = dev(inp["conv0"]).clone()
    out, SN, convN = gdn.chunk_prefill(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]),
        conv_w=dev(inp["conv_w"]), z=dev(inp["z"]), norm_w=dev(inp["norm_w"]), S0=S, SN=S,
        conv0=conv, convN=conv, dims=dims_of(w))
    torch.cuda.synchronize()
    assert SN.data_ptr() == S.data_ptr() and convN.data_ptr() == conv.data_ptr()
    assert_close(out, ref[0], w.dtype, "in place: out", scale=ref.out_scale)
    assert_close(S, ref[1], w.dtype, "in place: final state", scale=ref.SN_scale)
    np.testing.assert_array_equal(np64(conv), ref[2])


@pytest.mark.parametrize("seg,split", [(0, 0), (1, 4), (2, 1)])
def test_bf16_chunk_boundary_states(seg, split):
    # gdn_chunk_prefill_states: entry c is the state after chunk c of the sequence-by-sequence
    # chunk numbering; the oracle gives it as the final state of the prefix ending there
    with gdn.debug_options(segment_chunks=seg, chain_split=split):
        _chunk_boundary_states(seg)


def _chunk_boundary_states(seg):
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 0, 129, 256, 5), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1600 + seg, with_conv0=True)
    lengths = [int(v) for v in w.lengths]
    C = sum((L + 127) // 128 for L in lengths)
    cs = torch.full((C, w.num_v_heads, 128, 128), float("nan"), dtype=torch.float32,
                    device="cuda")
    out, SN, convN = gpu_prefill(w, inp, chunk_states=cs)
    starts = np.cumsum([0] + lengths)
    c = 0
    for n, L in enumerate(lengths):
        for j in range((L + 127) // 128):
            P = min(128 * (j + 1), L)
            t0 = int(starts[n])
            sub = dict(inp)
            for k in ("x", "beta", "g", "z"):
                if inp[k] is not None:
                    sub[k] = inp[k][t0:t0 + P].contiguous()
            sub["cu_seqlens"] = torch.tensor([0, P], dtype=torch.int32)
            sub["S0"] = inp["S0"][n:n + 1].contiguous()
            sub["conv0"] = inp["conv0"][n:n + 1].contiguous()
            ref = oracle_prefill(w, sub)
            assert_close(cs[c], ref[1][0], w.dtype, f"state after chunk {c} (sequence {n})",
                         scale=ref.SN_scale[0])
            c += 1
    assert c == C
    last = np.cumsum([(L + 127) // 128 for L in lengths]) - 1
    for n, L in enumerate(lengths):
        if L:
            assert torch.equal(cs[int(last[n])], SN[n]), f"last chunk of sequence {n}"


@pytest.mark.parametrize("seg,split", [(0, 0), (1, 4), (2, 2), (3, 1)])
def test_bf16_page64_states(seg, split):
    # gdn_chunk_prefill_pages with 64-token pages: entry p is the state after page p of the
    # sequence-by-sequence page numbering (the middle of a 128-token chunk for even pages of
    # chunks longer than 64); the oracle gives each as the final state of the prefix ending there
    with gdn.debug_options(segment_chunks=seg, chain_split=split):
        w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 0, 129, 64, 65, 5, 200),
                          s0_std=0.1)
        inp = inputs.prefill_inputs(w, 1700 + 10 * seg + split, with_conv0=True)
        lengths = [int(v) for v in w.lengths]
        P = sum((L + 63) // 64 for L in lengths)
        ps = torch.full((P, w.num_v_heads, 128, 128), float("nan"), dtype=torch.float32,
                        device="cuda")
        out, SN, convN = gpu_prefill(w, inp, page_states=ps, page_size=64)
    ref_full = oracle_prefill(w, inp)
    assert_close(out, ref_full[0], w.dtype, "pages: out", scale=ref_full.out_scale)
    starts = np.cumsum([0] + lengths)
    p = 0
    for n, L in enumerate(lengths):
        for j in range((L + 63) // 64):
            E = min(64 * (j + 1), L)
            t0 = int(starts[n])
            sub = dict(inp)
            for k in ("x", "beta", "g", "z"):
                if inp[k] is not None:
                    sub[k] = inp[k][t0:t0 + E].contiguous()
            sub["cu_seqlens"] = torch.tensor([0, E], dtype=torch.int32)
            sub["S0"] = inp["S0"][n:n + 1].contiguous()
            sub["conv0"] = inp["conv0"][n:n + 1].contiguous()
            ref = oracle_prefill(w, sub)
            assert_close(ps[p], ref[1][0], w.dtype, f"state after page {j} of sequence {n}",
                         scale=ref.SN_scale[0])
            p += 1
        if L:
            assert torch.equal(ps[p - 1], SN[n]), f"last page of sequence {n}"
    assert p == P


def test_bf16_page128_states_equal_chunk_states():
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 129, 5), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1750, with_conv0=True)
    C = sum((int(L) + 127) // 128 for L in w.lengths)
    cs = torch.empty((C, w.num_v_heads, 128, 128), dtype=torch.float32, device="cuda")
    ps = torch.empty_like(cs)
    a = gpu_prefill(w, inp, chunk_states=cs)
    b = gpu_prefill(w, inp, page_states=ps, page_size=128)
    assert torch.equal(cs, ps)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bf16_output_at_a_16_byte_offset():
    # The output kernel writes whole 32-byte sectors when the output allows it and 16-byte
    # pieces otherwise (the ABI asks for 16-byte alignment only): both give the same bits.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 130), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1400)
    T, Hv, d = w.tokens, w.num_v_heads, w.head_dim
    base = torch.empty(T * Hv * d + 8, dtype=torch.bfloat16, device="cuda")
    aligned = base[:T * Hv * d].view(T, Hv, d)
    shifted = base[8:].view(T, Hv, d)    # 16 bytes past a 256-byte aligned allocation
    assert shifted.data_ptr() % 32 == 16
    a = gpu_prefill(w, inp, out=aligned)[0].clone()
    b = gpu_prefill(w, inp, out=shifted)[0]
    assert torch.equal(a, b)
