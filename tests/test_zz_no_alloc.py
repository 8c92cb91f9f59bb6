"""The allocation-free prefill entry point (collected last on purpose).

gdn_chunk_prefill_static_ws serves callers that cannot allocate device memory (plugins whose
host owns every allocation, C callers without a caching allocator, loops that must avoid the
implicit synchronisation of cudaMalloc).  It uses the library's own static device scratch
instead of a caller workspace.  Here it is called through the C ABI twice in a row, on inputs
of different sizes, and each result is checked against the regular entry point
(gdn_chunk_prefill with a caller-provided workspace) on the same inputs.  Both run the same
kernels with the same arithmetic, only the scratch differs, so the results must agree bit for
bit.  The second call runs on scratch that still holds the first call's data, which must not
matter.
"""
import ctypes

import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import dev, dims_of, ensure_built, gpu_prefill

pytestmark = pytest.mark.gpu


def _static_call(w, inp):
    """gdn_chunk_prefill_static_ws through the C ABI (ctypes, raw pointers)."""
    L = gdn.lib()
    d = {k: dev(v) for k, v in inp.items()}
    T, N = w.tokens, len(w.lengths)
    out = torch.empty((T, w.num_v_heads, w.head_dim), dtype=w.dtype, device="cuda")
    SN = torch.empty((N, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32,
                     device="cuda")
    convN = torch.empty((N, w.conv_kernel - 1, w.channels), dtype=w.dtype, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    dims = dims_of(w)
    rc = L.gdn_chunk_prefill_static_ws(
        ctypes.byref(dims), gdn.GDN_BF16 if w.dtype == torch.bfloat16 else gdn.GDN_F32,
        p(d["x"]), p(d["conv_w"]), p(d["beta"]), p(d["g"]), p(d["z"]), p(d["norm_w"]),
        p(d["cu_seqlens"]), N, T, p(d["S0"]), p(SN), p(d["conv0"]), p(convN), p(out), p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == gdn.GDN_OK, gdn.status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, SN, convN


def test_static_scratch_matches_workspace_entry_point_twice():
    ensure_built()
    cases = [
        inputs.custom(16, 32, 128, torch.bfloat16, lengths=(1000, 300), s0_std=0.1),
        inputs.custom(2, 4, 128, torch.bfloat16, lengths=(5, 129, 64), s0_std=0.1),
    ]
    for i, w in enumerate(cases):
        inp = inputs.prefill_inputs(w, 3100 + i, with_conv0=True)
        need = gdn.prefill_workspace_size(len(w.lengths), w.tokens, w.dtype, dims_of(w))
        assert need <= gdn.STATIC_WORKSPACE_BYTES
        got = _static_call(w, inp)
        ref = gpu_prefill(w, inp)
        for a, b, name in zip(got, ref, ("out", "final state", "conv state")):
            assert torch.equal(a, b), f"call {i + 1}: {name} differs from the workspace call"
