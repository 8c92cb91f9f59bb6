"""CPU checks of the segment plan of gdn_chunk_prefill_host (the host-buffer prefill): the
segments tile the packed batch in order, cut a sequence only at a multiple of 128 tokens from
its start, hold at most segment_tokens tokens, and end early only when the next 128 tokens of
the next sequence do not fit; and the entry point's argument checks (no device needed)."""
import ctypes

import numpy as np
import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import build as gdn_build
from gated_deltanet_layer_02_b200 import inputs


@pytest.fixture(scope="module", autouse=True)
def _lib():
    gdn_build.build()


def _check_plan(lengths, seg):
    cu = inputs.cu_seqlens_of(lengths)
    T = int(cu[-1])
    plan = gdn.host_plan(cu, seg).numpy()
    eff = seg or max(512, (T // 8 + 127) // 128 * 128)
    cu = cu.numpy()
    pos = 0
    for k, (n0, nseq, t0, nt) in enumerate(plan):
        assert t0 == pos and 0 < nt <= eff
        t1 = t0 + nt
        # first and last sequence of the segment hold its first and last token
        assert cu[n0] <= t0 and (t0 < cu[n0 + 1] or lengths[n0] == 0)
        last = n0 + nseq - 1
        assert cu[last] <= t1 <= cu[last + 1] and (cu[last] < t1 or lengths[last] == 0)
        # cuts inside a sequence are chunk-aligned from its start
        for t in (t0, t1):
            n = np.searchsorted(cu, t, side="right") - 1
            if n < len(lengths) and cu[n] < t < cu[n + 1]:
                assert (t - cu[n]) % 128 == 0
        if k + 1 < len(plan) and nt < eff:   # ended early: the next piece did not fit
            room = eff - nt
            n = plan[k + 1][0]
            left = cu[n + 1] - t1
            assert left > room and room < 128
        pos = t1
    assert pos == T
    return plan


@pytest.mark.parametrize("seg", [0, 128, 256, 512, 1024])
def test_plan_tiles_random_batches(seg):
    rng = np.random.default_rng(77 + seg)
    for _ in range(30):
        n = int(rng.integers(1, 12))
        lengths = [int(v) for v in rng.integers(0, 1500, n)]
        lengths[int(rng.integers(0, n))] = 0
        _check_plan(lengths, seg)


def test_plan_examples():
    p = _check_plan([4096], 512)
    assert p.tolist() == [[0, 1, 512 * k, 512] for k in range(8)]
    p = _check_plan([300, 129], 256)   # 256 of the first; its 44 + the 129 next; the rest
    assert p.tolist() == [[0, 1, 0, 256], [0, 2, 256, 173]]
    p = _check_plan([0, 0, 5, 0], 128)
    assert p.tolist() == [[0, 4, 0, 5]]   # empty sequences ride along
    assert gdn.host_plan(inputs.cu_seqlens_of([0, 0]), 128).shape[0] == 0


def test_plan_rejects_bad_arguments():
    L = gdn.lib()
    cu = torch.tensor([0, 5, 3], dtype=torch.int32)   # decreasing
    p = ctypes.c_void_p(cu.data_ptr())
    assert L.gdn_chunk_prefill_host_plan(p, 2, 3, 128, None, 0) == gdn.GDN_ERR_INVALID_ARG
    ok = torch.tensor([0, 5, 9], dtype=torch.int32)
    q = ctypes.c_void_p(ok.data_ptr())
    assert L.gdn_chunk_prefill_host_plan(q, 2, 10, 128, None, 0) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_prefill_host_plan(q, 2, 9, 100, None, 0) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_prefill_host_plan(None, 2, 9, 128, None, 0) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_prefill_host_plan(q, 2, 9, 128, None, 0) == 1
    seg = (ctypes.c_int32 * 4)()
    assert L.gdn_chunk_prefill_host_plan(q, 2, 9, 128, seg, 0) == gdn.GDN_ERR_WORKSPACE


def test_host_entry_point_argument_checks():
    L = gdn.lib()
    d = ctypes.byref(gdn.Dims())
    cu = torch.tensor([0, 300], dtype=torch.int32)
    cp = ctypes.c_void_p(cu.data_ptr())
    A = ctypes.c_void_p(1 << 20)
    size = L.gdn_chunk_prefill_host_workspace_size
    need = size(d, cp, 1, 300, 128)
    # device copies of x, beta, g, z, out + carry buffers + the largest segment's scratch
    assert need >= 300 * (8192 * 2 + 2 * 32 * 4 + 2 * 4096 * 2) + 32 * 128 * 128 * 4
    assert size(None, cp, 1, 300, 128) == 0
    assert size(d, cp, 1, 299, 128) == 0          # cu[N] != T

    def call(dims=d, x=A, cu_p=cp, T=300, seg=128, ws=A, ws_bytes=need, S0=None):
        return L.gdn_chunk_prefill_host(dims, x, None, A, A, None, None, cu_p, 1, T, S0, None,
                                        None, None, A, seg, ws, ws_bytes, None, None)
    assert call(dims=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(dims=ctypes.byref(gdn.Dims(16, 16))) == gdn.GDN_ERR_UNSUPPORTED
    assert call(dims=ctypes.byref(gdn.Dims(1, 2))) == gdn.GDN_ERR_UNSUPPORTED   # Hv % 4
    assert call(x=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(cu_p=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(T=301) == gdn.GDN_ERR_INVALID_ARG
    assert call(seg=200) == gdn.GDN_ERR_INVALID_ARG
    assert call(S0=ctypes.c_void_p((1 << 20) + 4)) == gdn.GDN_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == gdn.GDN_ERR_INVALID_ARG
    assert call(ws=None) == gdn.GDN_ERR_WORKSPACE
    assert call(ws_bytes=need - 1) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_chunk_prefill_host(d, None, None, None, None, None, None, None, 0, 0, None, None,
                                    None, None, None, 0, None, 0, None, None) == gdn.GDN_OK
