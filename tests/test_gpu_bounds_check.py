"""GPU checks of the bounds-check build (libgdn_checked.so, kernels compiled with
-DGDN_BOUNDS_CHECK): on valid inputs it reports nothing and returns what the normal build
returns, bit for bit; on a cu_seqlens array that goes backwards it skips the bad sequence,
reports GDN_ERR_BOUNDS in the status word, and no access leaves the caller's tensors."""
import ctypes

import pytest
import torch

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import build as gdn_build
from gated_deltanet_layer_02_b200 import inputs
from gpu_util import dev, dims_of, ensure_built, gpu_prefill

pytestmark = pytest.mark.gpu


def _checked_prefill(Lc, w, inp, cu):
    d = {k: dev(v) for k, v in inp.items()}
    T, N = w.tokens, cu.numel() - 1
    dims = dims_of(w)
    out = torch.zeros((T, w.num_v_heads, w.head_dim), dtype=w.dtype, device="cuda")
    SN = torch.zeros((N, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32,
                     device="cuda")
    convN = torch.zeros((N, w.conv_kernel - 1, w.channels), dtype=w.dtype, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = Lc.gdn_chunk_prefill_workspace_size(ctypes.byref(dims), gdn.GDN_BF16, N, T)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = Lc.gdn_chunk_prefill(
        ctypes.byref(dims), gdn.GDN_BF16, p(d["x"]), p(d["conv_w"]), p(d["beta"]), p(d["g"]),
        p(d["z"]), p(d["norm_w"]), p(cu.cuda()), N, T, p(d["S0"]), p(SN), p(d["conv0"]),
        p(convN), p(out), p(ws), need, p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == gdn.GDN_OK
    torch.cuda.synchronize()
    return (out, SN, convN), int(status.item())


def test_checked_build_matches_normal_build_and_reports_bad_cu_seqlens():
    ensure_built()
    gdn_build.build(bounds_check=True)
    Lc = gdn.lib_checked()
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 129), s0_std=0.1)
    inp = inputs.prefill_inputs(w, 3300, with_conv0=True)
    got, st = _checked_prefill(Lc, w, inp, inp["cu_seqlens"])
    ref = gpu_prefill(w, inp)
    assert st == 0
    for a, b, name in zip(got, ref, ("out", "final state", "conv state")):
        assert torch.equal(a, b), name
    # cu_seqlens going backwards in the middle: [0, 300, 200, 429] over 429 tokens
    w3 = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300, 29, 100), s0_std=0.1)
    inp3 = inputs.prefill_inputs(w3, 3301, with_conv0=True)
    bad = torch.tensor([0, 300, 200, 429], dtype=torch.int32)
    _, st = _checked_prefill(Lc, w3, inp3, bad)
    assert st == gdn.GDN_ERR_BOUNDS
