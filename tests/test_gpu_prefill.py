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
    ref_o, ref_S, ref_c = oracle_prefill(w, inp)
    e1 = assert_close(out, ref_o, w.dtype, f"{what}: out")
    e2 = assert_close(SN, ref_S, w.dtype, f"{what}: final state")
    np.testing.assert_array_equal(np64(convN), ref_c)
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
    ref_o, ref_S, _ = oracle_prefill(w, inp)
    assert_close(torch.cat([a[0], b[0]]), ref_o, w.dtype, "split out")
    assert_close(b[1], ref_S, w.dtype, "split state")
    assert torch.equal(b[2], full[2])


@pytest.fixture
def pipeline_env(monkeypatch):
    """Sets the library's pipeline knobs (segment length in chunks, chain d_v split)."""
    def set_(seg, split):
        monkeypatch.setenv("GDN_SEGMENT_CHUNKS", str(seg))
        monkeypatch.setenv("GDN_CHAIN_SPLIT", str(split))
    return set_


@pytest.mark.parametrize("seg", [1, 2, 3, 5])
@pytest.mark.parametrize("split", [1, 2, 4])
def test_bf16_pipelined_segments(pipeline_env, seg, split):
    # Segments of `seg` chunks: sequences cross segment boundaries (the state is carried in
    # fp32 between launches), short and empty sequences fall inside one segment, and the
    # chain's d_v split is forced so that every split meets every boundary case.
    pipeline_env(seg, split)
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(700, 0, 5, 129, 0, 1100, 64, 260),
                      s0_std=0.1)
    _check(w, inputs.prefill_inputs(w, 1200 + 10 * seg + split, with_conv0=True),
           f"seg={seg} split={split}")


def test_bf16_pipelined_matches_single_launch_bitwise(pipeline_env):
    # The pipeline reorders launches only: with the same split, the segmented and the single
    # launch runs perform the same arithmetic and must agree to the bit.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(900, 33, 1500), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1300, with_conv0=True)
    pipeline_env(1 << 19, 2)
    one = gpu_prefill(w, inp)
    pipeline_env(2, 2)
    seg = gpu_prefill(w, inp)
    for a, b, name in zip(one, seg, ("out", "final state", "conv state")):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("lengths", [(300,), (1, 0, 700, 129), (2000,)])
def test_bf16_fused_prep_and_chain(monkeypatch, lengths):
    # The opt-in persistent prep + chain kernel (chains waiting on flags the prep workers set).
    monkeypatch.setenv("GDN_FUSED", "1")
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=lengths, s0_std=0.1)
    _check(w, inputs.prefill_inputs(w, 1400 + len(lengths), with_conv0=True), f"fused {lengths}")


def test_bf16_fused_matches_separate_launches_bitwise(monkeypatch):
    # The persistent prep + chain kernel runs the same arithmetic as the separate launches with
    # 32-column chain blocks; only the schedule differs.
    w = inputs.custom(16, 32, 128, torch.bfloat16, lengths=(1500,), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1450, with_conv0=True)
    monkeypatch.setenv("GDN_FUSED", "0")
    monkeypatch.setenv("GDN_CHAIN_SPLIT", "4")
    sep = gpu_prefill(w, inp)
    monkeypatch.setenv("GDN_FUSED", "1")
    fused = gpu_prefill(w, inp)
    for x, y, name in zip(sep, fused, ("out", "final state", "conv state")):
        assert torch.equal(x, y), name


def test_bf16_states_updated_in_place():
    # SN = S0 and convN = conv0: the call reads the initial states and overwrites them, as a
    # serving loop does; the conv history then comes from its own kernel after the layer.
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 0, 2, 129), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 1500, with_conv0=True)
    ref_o, ref_S, ref_c = oracle_prefill(w, inp)
    S = dev(inp["S0"]).clone()
    conv = dev(inp["conv0"]).clone()
    out, SN, convN = gdn.chunk_prefill(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]),
        conv_w=dev(inp["conv_w"]), z=dev(inp["z"]), norm_w=dev(inp["norm_w"]), S0=S, SN=S,
        conv0=conv, convN=conv, dims=dims_of(w))
    torch.cuda.synchronize()
    assert SN.data_ptr() == S.data_ptr() and convN.data_ptr() == conv.data_ptr()
    assert_close(out, ref_o, w.dtype, "in place: out")
    assert_close(S, ref_S, w.dtype, "in place: final state")
    np.testing.assert_array_equal(np64(conv), ref_c)


@pytest.mark.parametrize("seg,split", [(0, 0), (1, 4), (2, 1)])
def test_bf16_chunk_boundary_states(pipeline_env, seg, split):
    # gdn_chunk_prefill_states: entry c is the state after chunk c of the sequence-by-sequence
    # chunk numbering; the oracle gives it as the final state of the prefix ending there
    if seg:
        pipeline_env(seg, split)
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
            _, ref_S, _ = oracle_prefill(w, sub)
            assert_close(cs[c], ref_S[0], w.dtype, f"state after chunk {c} (sequence {n})")
            c += 1
    assert c == C
    last = np.cumsum([(L + 127) // 128 for L in lengths]) - 1
    for n, L in enumerate(lengths):
        if L:
            assert torch.equal(cs[int(last[n])], SN[n]), f"last chunk of sequence {n}"
