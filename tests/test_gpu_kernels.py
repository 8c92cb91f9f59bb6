"""GPU parity of the standalone kernels against the fp64 oracle: conv1d + SiLU, gated RMSNorm,
decode step; plus the bounded device wait (no fault, no hang)."""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import assert_close, dev, ensure_built, np64

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]


def _randn(shape, dtype, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dtype)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("lengths", [[1], [5, 0, 2, 17, 1], [40, 3, 64]])
def test_conv1d_update(dtype, with_state, lengths):
    ensure_built()
    dims = gdn.Dims(2, 4)
    Cc = dims.channels
    T, N = sum(lengths), len(lengths)
    x = _randn((T, Cc), dtype, 1)
    w = _randn((Cc, 4), dtype, 2, 0.5)
    st = _randn((N, 3, Cc), dtype, 3) if with_state else None
    cu = inputs.cu_seqlens_of(lengths)
    st_out = torch.empty((N, 3, Cc), dtype=dtype, device="cuda")
    y = gdn.conv1d_update(dev(x), dev(w), dev(cu), dev(st), st_out, dims=dims)
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.conv1d_silu(x, w, cu, st)
    assert_close(y, y_ref, dtype, "conv y")
    np.testing.assert_array_equal(np64(st_out), st_ref)


@pytest.mark.parametrize("dtype", DTYPES)
def test_conv1d_state_in_place(dtype):
    ensure_built()
    dims = gdn.Dims(2, 4)
    Cc, lengths = dims.channels, [2, 9, 1]
    x = _randn((12, Cc), dtype, 4)
    w = _randn((Cc, 4), dtype, 5, 0.5)
    st = _randn((3, 3, Cc), dtype, 6)
    cu = inputs.cu_seqlens_of(lengths)
    y_ref, st_ref = oracle.conv1d_silu(x, w, cu, st)
    st_d = dev(st)
    y = gdn.conv1d_update(dev(x), dev(w), dev(cu), st_d, st_d, dims=dims)
    torch.cuda.synchronize()
    assert_close(y, y_ref, dtype, "conv y")
    np.testing.assert_array_equal(np64(st_d), st_ref)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("dim", [128, 64, 256, 1024, 8])
@pytest.mark.parametrize("with_w", [False, True])
def test_gated_rmsnorm(dtype, dim, with_w):
    ensure_built()
    M = 37
    o, z = _randn((M, dim), dtype, 7), _randn((M, dim), dtype, 8)
    w = _randn((dim,), dtype, 9) if with_w else None
    y = gdn.gated_rmsnorm(dev(o), dev(z), dev(w), 1e-6)
    torch.cuda.synchronize()
    assert_close(y, oracle.gated_rmsnorm(o, z, w, 1e-6), dtype, "gated rmsnorm")
    # in place
    od = dev(o)
    gdn.gated_rmsnorm(od, dev(z), dev(w), 1e-6, y=od)
    torch.cuda.synchronize()
    assert_close(od, oracle.gated_rmsnorm(o, z, w, 1e-6), dtype, "gated rmsnorm in place")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("with_z", [False, True])
def test_decode_steps_with_slots(dtype, with_z):
    ensure_built()
    dims = gdn.Dims(2, 4)
    od = oracle.Dims(2, 4)
    B, slots, Cc, steps = 5, 9, dims.channels, 4
    slot_idx = torch.tensor([7, 0, 3, 8, 2], dtype=torch.int32)
    S = _randn((slots, 4, 128, 128), torch.float32, 10, 0.1)
    cs = _randn((slots, 3, Cc), dtype, 11)
    w = _randn((Cc, 4), dtype, 12, 0.5)
    nw = _randn((128,), dtype, 13) if with_z else None
    S_d, cs_d = dev(S), dev(cs)
    S_ref, cs_ref = S.double().numpy().copy(), cs.double().numpy().copy()
    M_ref = np.abs(S_ref)
    for step in range(steps):
        x = _randn((B, Cc), dtype, 100 + step)
        z = _randn((B, 4, 128), dtype, 200 + step) if with_z else None
        beta = torch.sigmoid(_randn((B, 4), torch.float32, 300 + step))
        g = -torch.rand((B, 4), generator=torch.Generator().manual_seed(400 + step))
        out = gdn.decode_step(dev(x), dev(beta), dev(g), cs_d, S_d, dev(w), z=dev(z),
                              norm_w=dev(nw), slot_idx=dev(slot_idx), dims=dims)
        torch.cuda.synchronize()
        ref, sc = oracle.decode_step(od, x, beta, g, cs_ref, S_ref, conv_w=w, z=z, norm_w=nw,
                                     slot_idx=slot_idx, M=M_ref)
        assert_close(out, ref, dtype, f"decode out step {step}", scale=sc)
    np.testing.assert_array_equal(np64(cs_d), cs_ref)
    err = np.max(np.abs(np64(S_d) - S_ref))
    assert err <= 1e-4, err
    # untouched slots keep their state exactly
    for s in (1, 4, 5, 6):
        assert torch.equal(S_d[s].cpu(), S[s])


def test_bounded_wait_reports_timeout_and_stream_stays_usable():
    ensure_built()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.debug_wait_probe(status, 2000)  # 2 ms limit, nothing ever completes the wait
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_TIMEOUT
    # the context is intact: a normal kernel runs afterwards
    o = torch.ones(4, 128, dtype=torch.float32, device="cuda")
    y = gdn.gated_rmsnorm(o, torch.zeros_like(o))
    torch.cuda.synchronize()
    assert torch.all(y == 0)


def test_trace_records_kernel_times():
    ensure_built()
    o = torch.ones(64, 128, dtype=torch.bfloat16, device="cuda")
    tr = gdn.Trace()
    with tr:
        gdn.gated_rmsnorm(o, o)
        gdn.gated_rmsnorm(o, o)
    recs = tr.records()
    tr.close()
    assert [r[0] for r in recs] == ["gated_rmsnorm", "gated_rmsnorm"]
    assert all(r[1] > 0 for r in recs)
