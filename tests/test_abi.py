"""C-ABI checks that need no GPU: the library loads, exports every symbol include/gdn.h
declares, and rejects bad arguments with the documented status before launching anything."""
import ctypes
import os
import re

import pytest

import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gdn_build.build()
    return gdn.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "gdn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(gdn.EXPORTS)


def test_abi_version_and_status_strings(L):
    assert L.gdn_abi_version() == 2
    for code, text in [(0, "ok"), (-1, "invalid argument"), (-2, "unsupported shape or dtype"),
                       (-3, "CUDA error"), (-4, "device wait timed out"),
                       (-5, "workspace too small"), (7, "unknown status")]:
        assert gdn.status_string(code) == text


def test_conv_channels(L):
    assert gdn.conv_channels(gdn.Dims()) == 8192
    assert gdn.conv_channels(gdn.Dims(2, 4)) == 1024
    assert L.gdn_conv_channels(None) == -1


P = ctypes.c_void_p
A = P(1 << 20)          # an aligned fake address: never dereferenced on these paths
MIS = P((1 << 20) + 8)  # misaligned


def _prefill(L, dims, dtype=gdn.GDN_BF16, x=A, ws=A, ws_bytes=1 << 40, N=1, T=16, cu=A, out=A,
             beta=A, g=A):
    return L.gdn_chunk_prefill(dims, dtype, x, None, beta, g, None, None, cu, N, T, None, None,
                               None, None, out, ws, ws_bytes, None, None)


def test_prefill_argument_errors(L):
    d = gdn.Dims()
    assert _prefill(L, None) == gdn.GDN_ERR_INVALID_ARG
    assert _prefill(L, ctypes.byref(gdn.Dims(head_dim=64))) == gdn.GDN_ERR_UNSUPPORTED
    assert _prefill(L, ctypes.byref(gdn.Dims(conv_kernel=3))) == gdn.GDN_ERR_UNSUPPORTED
    assert _prefill(L, ctypes.byref(gdn.Dims(16, 24))) == gdn.GDN_ERR_INVALID_ARG   # 24 % 16
    assert _prefill(L, ctypes.byref(gdn.Dims(8, 32))) == gdn.GDN_ERR_UNSUPPORTED    # bf16 ratio 4
    assert _prefill(L, ctypes.byref(d), dtype=5) == gdn.GDN_ERR_UNSUPPORTED
    assert _prefill(L, ctypes.byref(d), x=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _prefill(L, ctypes.byref(d), x=None) == gdn.GDN_ERR_INVALID_ARG
    assert _prefill(L, ctypes.byref(d), cu=None) == gdn.GDN_ERR_INVALID_ARG
    assert _prefill(L, ctypes.byref(d), N=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _prefill(L, ctypes.byref(d), N=0) == gdn.GDN_ERR_INVALID_ARG           # tokens, no seqs
    assert _prefill(L, ctypes.byref(d), ws=None) == gdn.GDN_ERR_WORKSPACE
    assert _prefill(L, ctypes.byref(d), ws_bytes=1024) == gdn.GDN_ERR_WORKSPACE
    assert _prefill(L, ctypes.byref(d), ws=P((1 << 20) + 16)) == gdn.GDN_ERR_INVALID_ARG
    bad = gdn.Dims()
    bad.l2_eps = -1.0
    assert _prefill(L, ctypes.byref(bad)) == gdn.GDN_ERR_INVALID_ARG


def test_workspace_size(L):
    d = ctypes.byref(gdn.Dims())
    f = L.gdn_chunk_prefill_workspace_size
    assert f(None, 1, 1, 10) == 0
    assert f(d, 0, -1, 10) == 0
    assert f(d, gdn.GDN_F32, 1, 4096) == 256
    small, big = f(d, 1, 1, 4096), f(d, 1, 1, 8192)
    assert 0 < small < big
    assert f(d, 1, 8, 4096) > small      # more sequences -> more partial chunks


def test_other_entry_points_reject_bad_arguments(L):
    d = ctypes.byref(gdn.Dims())
    assert L.gdn_conv1d_update(None, 1, A, A, A, A, 1, 4, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_conv1d_update(d, 1, A, A, A, None, 1, 4, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_conv1d_update(d, 1, A, A, A, A, 1, 4, MIS, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_conv1d_update(d, 1, A, A, A, A, 1, -4, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_gated_rmsnorm(1, A, A, None, 1e-6, 4, 12, A, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_gated_rmsnorm(1, A, A, None, 1e-6, 4, 2048, A, None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_gated_rmsnorm(1, A, None, None, 1e-6, 4, 128, A, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_gated_rmsnorm(1, A, A, None, -1.0, 4, 128, A, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_gated_rmsnorm(3, A, A, None, 1e-6, 4, 128, A, None) == gdn.GDN_ERR_UNSUPPORTED
    # (dims, dtype, x, conv_w, beta, g, z, norm_w, conv_state, S, slot_idx, num_slots, batch,
    #  out, dev_status, stream)
    assert L.gdn_decode_step(d, 1, A, A, A, A, None, None, A, A, None, 0, -1, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_step(d, 1, A, None, A, A, None, None, A, A, None, 4, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_step(d, 1, A, A, A, A, None, None, A, MIS, None, 4, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_step(ctypes.byref(gdn.Dims(1, 16)), 1, A, A, A, A, None, None, A, A, None,
                             4, 4, A, None, None) == gdn.GDN_ERR_UNSUPPORTED
    # pools smaller than the batch without a slot map, and a negative pool size
    assert L.gdn_decode_step(d, 1, A, A, A, A, None, None, A, A, None, 3, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_step(d, 1, A, A, A, A, None, None, A, A, A, -1, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    bs = L.gdn_decode_step_bf16_state
    assert bs(d, 1, A, A, A, A, None, None, A, A, None, 0, -1, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert bs(d, 1, A, A, A, A, None, None, A, None, None, 4, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert bs(d, 1, A, A, A, A, None, None, A, MIS, None, 4, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert bs(d, 3, A, A, A, A, None, None, A, A, None, 4, 4, A, None, None) == gdn.GDN_ERR_UNSUPPORTED
    assert bs(d, 1, A, A, A, A, None, None, A, A, None, 2, 4, A, None, None) == gdn.GDN_ERR_INVALID_ARG
    mt = L.gdn_decode_multi
    # (..., slot_idx, num_slots, batch, tokens, out, snapshots, dev_status, stream)
    assert mt(d, 1, A, A, A, A, None, None, A, A, None, 4, 4, -1, A, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert mt(d, 1, A, A, A, A, None, None, A, A, None, 4, 4, 9, A, None, None, None) == gdn.GDN_ERR_UNSUPPORTED
    assert mt(d, 1, A, None, A, A, None, None, A, A, None, 4, 4, 4, A, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert mt(d, 1, A, A, A, A, None, None, A, A, None, 4, 4, 4, A, MIS, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert mt(d, 1, A, A, A, A, None, None, A, A, None, 1, 4, 4, A, None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_debug_wait_probe(None, 10, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_debug_wait_probe(A, 10_000_000, None) == gdn.GDN_ERR_INVALID_ARG


def _block(L, dims, hidden=256, N=1, T=16, h=A, ws=A, ws_bytes=1 << 40, y=A, a_log=A):
    return L.gdn_block_prefill(dims, hidden, h, A, A, A, a_log, A, None, None, A, A, N, T, None,
                               None, None, None, y, ws, ws_bytes, None, None)


def test_block_prefill_argument_errors(L):
    d = ctypes.byref(gdn.Dims())
    size = L.gdn_block_prefill_workspace_size
    assert size(None, 256, 1, 16) == 0
    assert size(d, 0, 1, 16) == 0
    assert size(d, 256, -1, 16) == 0
    layer = L.gdn_chunk_prefill_workspace_size(d, 1, 1, 4096)
    # layer scratch + bf16 x, z, o and fp32 beta, g per token (the gates leave the GEMM directly)
    assert size(d, 2048, 1, 4096) >= layer + 4096 * (8192 * 2 + 2 * 4096 * 2 + 2 * 32 * 4)
    assert _block(L, None) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, hidden=0) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, hidden=260) == gdn.GDN_ERR_INVALID_ARG      # rows of 16-byte multiples
    assert _block(L, d, N=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, N=0) == gdn.GDN_ERR_INVALID_ARG              # tokens, no sequences
    assert _block(L, d, h=None) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, y=None) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, a_log=None) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, h=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, ws=P((1 << 20) + 16)) == gdn.GDN_ERR_INVALID_ARG
    assert _block(L, d, ws=None) == gdn.GDN_ERR_WORKSPACE
    assert _block(L, d, ws_bytes=1024) == gdn.GDN_ERR_WORKSPACE
    assert _block(L, ctypes.byref(gdn.Dims(head_dim=64))) == gdn.GDN_ERR_INVALID_ARG
    # no sequences and no tokens: valid, nothing to launch
    assert L.gdn_block_prefill(d, 256, None, None, None, None, None, None, None, None, None, None,
                               0, 0, None, None, None, None, None, A, 1 << 30, None,
                               None) == gdn.GDN_OK


def test_prefill_slots_argument_errors(L):
    d = ctypes.byref(gdn.Dims())
    f = L.gdn_chunk_prefill_slots

    def call(dims=d, dtype=1, x=A, N=1, T=16, slot=A, slots=8, pool=A, conv=A, ws=A,
             ws_bytes=1 << 40):
        return f(dims, dtype, x, None, A, A, None, None, A, N, T, slot, slots, pool, conv, A, ws,
                 ws_bytes, None, None)
    assert call(pool=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(pool=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert call(conv=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert call(dims=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(dtype=5) == gdn.GDN_ERR_UNSUPPORTED
    assert call(ws=None) == gdn.GDN_ERR_WORKSPACE
    assert call(x=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(slots=-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(slots=0) == gdn.GDN_ERR_INVALID_ARG                  # a slot map into no rows
    assert call(slot=None, N=4, T=16, slots=3) == gdn.GDN_ERR_INVALID_ARG  # identity needs N rows
    assert call(N=0, T=0, pool=None, slot=None, conv=None, slots=0) == gdn.GDN_OK


def test_zero_size_calls_launch_nothing(L):
    d = ctypes.byref(gdn.Dims())
    # no sequences, no tokens: valid and a no-op
    assert L.gdn_chunk_prefill(d, 1, None, None, None, None, None, None, None, 0, 0, None, None,
                               None, None, None, A, 1 << 30, None, None) == gdn.GDN_OK
    assert L.gdn_decode_step(d, 1, None, None, None, None, None, None, None, None, None, 0, 0,
                             None, None, None) == gdn.GDN_OK
    assert L.gdn_decode_step_bf16_state(d, 1, None, None, None, None, None, None, None, None,
                                        None, 0, 0, None, None, None) == gdn.GDN_OK
    assert L.gdn_decode_multi(d, 1, None, None, None, None, None, None, None, None, None, 0, 0, 4,
                              None, None, None, None) == gdn.GDN_OK
    assert L.gdn_decode_multi(d, 1, None, None, None, None, None, None, None, None, None, 4, 4, 0,
                              None, None, None, None) == gdn.GDN_OK
    assert L.gdn_gated_rmsnorm(1, None, None, None, 1e-6, 0, 128, None, None) == gdn.GDN_OK


def test_trace_object_lifecycle(L):
    h = P()
    assert L.gdn_trace_create(ctypes.byref(h)) == gdn.GDN_OK
    assert L.gdn_trace_count(h) == 0
    assert L.gdn_trace_attach(h) == gdn.GDN_OK
    assert L.gdn_trace_attach(None) == gdn.GDN_OK
    assert L.gdn_trace_get(h, 0, None, None) == gdn.GDN_ERR_INVALID_ARG
    f = ctypes.c_float()
    assert L.gdn_trace_span(h, 0, ctypes.byref(f), ctypes.byref(f)) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_trace_reset(h) == gdn.GDN_OK
    assert L.gdn_trace_destroy(h) == gdn.GDN_OK
    assert L.gdn_trace_create(None) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 8192, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        gdn.conv1d_update(x, torch.zeros(8192, 4, dtype=torch.bfloat16),
                          torch.tensor([0, 4], dtype=torch.int32))


def test_static_workspace_entry_point_rejects_oversized_calls(L):
    """Sizes whose scratch exceeds the library's static array are refused before any launch."""
    d = ctypes.byref(gdn.Dims())
    f = L.gdn_chunk_prefill_workspace_size
    assert f(d, 1, 1, 1791) <= gdn.STATIC_WORKSPACE_BYTES < f(d, 1, 1, 1792)
    args = (d, 1, A, None, A, A, None, None, A)
    tail = (None, None, None, None, A, None, None)
    assert L.gdn_chunk_prefill_static_ws(*args, 1, 1792, *tail) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_chunk_prefill_static_ws(*args, 64, 64, *tail) == gdn.GDN_ERR_WORKSPACE
    # invalid shapes keep the regular entry point's status codes
    assert L.gdn_chunk_prefill_static_ws(None, 1, A, None, A, A, None, None, A, 1, 16,
                                         *tail) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_prefill_static_ws(ctypes.byref(gdn.Dims(head_dim=64)), 1, A, None, A, A,
                                         None, None, A, 1, 16, *tail) == gdn.GDN_ERR_UNSUPPORTED


def test_plain_c_consumer(L, tmp_path):
    """include/gdn.h compiles as C99 (-pedantic) and a C program links libgdn.so and calls it."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "consumer.c"
    src.write_text(
        '#include <stdio.h>\n#include "gdn.h"\n'
        "int main(void) {\n"
        "  gdn_dims d = {16, 32, 128, 4, 1.0f, 1e-6f, 1e-6f};\n"
        "  int32_t cu[3] = {0, 300, 429};\n"
        "  int32_t seg[8];\n"
        "  int n = gdn_chunk_prefill_host_plan(cu, 2, 429, 256, seg, 2);\n"
        '  printf("%d %d %lld %s %d %d %d %d\\n", gdn_abi_version(), n,\n'
        "         (long long)gdn_conv_channels(&d), gdn_status_string(GDN_ERR_WORKSPACE),\n"
        "         seg[4], seg[5], seg[6], seg[7]);\n"
        "  return 0;\n}\n")
    exe = tmp_path / "consumer"
    lib_dir = os.path.dirname(gdn.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", lib_dir, "-l:libgdn.so", f"-Wl,-rpath,{lib_dir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == ["2", "2", "8192", "workspace", "too", "small", "0", "2", "256", "173"]


def test_binding_refuses_undersized_buffers(L):
    """The binding checks every buffer against the sizes the call touches before it hands bare
    pointers to the library (CPU tensors: the size check comes before the device check)."""
    import torch
    d = gdn.Dims(2, 4)
    T, N, Cc, Hv = 10, 1, d.channels, d.num_v_heads
    cu = torch.tensor([0, T], dtype=torch.int32)
    ok = dict(x=torch.zeros(T, Cc, dtype=torch.bfloat16), beta=torch.zeros(T, Hv),
              g=torch.zeros(T, Hv))
    with pytest.raises(ValueError, match="CUDA"):          # sizes fine: stops at the device check
        gdn.chunk_prefill(ok["x"], ok["beta"], ok["g"], cu, dims=d)
    with pytest.raises(ValueError, match="beta holds"):
        gdn.chunk_prefill(ok["x"], ok["beta"][:5], ok["g"], cu, dims=d)
    with pytest.raises(ValueError, match="x holds"):
        gdn.chunk_prefill(ok["x"][:, :512], ok["beta"], ok["g"], cu, dims=d)
    with pytest.raises(ValueError, match="S0 holds"):
        gdn.chunk_prefill(ok["x"], ok["beta"], ok["g"], cu, S0=torch.zeros(1, Hv, 128, 64),
                          dims=d)
    with pytest.raises(ValueError, match="conv_w holds"):
        gdn.chunk_prefill(ok["x"], ok["beta"], ok["g"], cu, dims=d,
                          conv_w=torch.zeros(Cc, 3, dtype=torch.bfloat16))
    B = 3
    xs = torch.zeros(B, Cc, dtype=torch.bfloat16)
    cw = torch.zeros(Cc, 4, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pools hold 2 rows"):  # identity slots need B rows
        gdn.decode_step(xs, torch.zeros(B, Hv), torch.zeros(B, Hv),
                        torch.zeros(B, 3, Cc, dtype=torch.bfloat16),
                        torch.zeros(B - 1, Hv, 128, 128), cw, dims=d)
    with pytest.raises(ValueError, match="slot_idx holds"):
        gdn.decode_step(xs, torch.zeros(B, Hv), torch.zeros(B, Hv),
                        torch.zeros(1, 3, Cc, dtype=torch.bfloat16),
                        torch.zeros(1, Hv, 128, 128), cw, slot_idx=torch.zeros(2, dtype=torch.int32),
                        dims=d)
    with pytest.raises(ValueError, match="snapshots holds"):
        gdn.decode_multi(torch.zeros(B, 2, Cc, dtype=torch.bfloat16), torch.zeros(B, 2, Hv),
                         torch.zeros(B, 2, Hv), torch.zeros(B, 3, Cc, dtype=torch.bfloat16),
                         torch.zeros(B, Hv, 128, 128), cw,
                         snapshots=torch.zeros(B, 1, Hv, 128, 128), dims=d)
    with pytest.raises(ValueError, match="z holds"):
        gdn.gated_rmsnorm(torch.zeros(4, 128, dtype=torch.bfloat16),
                          torch.zeros(3, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="w_out holds"):
        H = 256
        gdn.block_prefill(torch.zeros(T, H, dtype=torch.bfloat16),
                          torch.zeros(H, Cc, dtype=torch.bfloat16),
                          torch.zeros(H, Hv * 128, dtype=torch.bfloat16),
                          torch.zeros(H, 2 * Hv, dtype=torch.bfloat16), torch.zeros(Hv),
                          torch.zeros(Hv), torch.zeros(Hv * 128, H - 1, dtype=torch.bfloat16),
                          cu, dims=d)


def test_bounds_check_build_compiles_and_exports_every_symbol():
    """The bounds-check variant (-DGDN_BOUNDS_CHECK) builds for sm_100a and exports the same
    entry points; its status strings know GDN_ERR_BOUNDS."""
    from gated_deltanet_layer_02_b200 import build as gdn_build
    path = gdn_build.build(bounds_check=True)
    assert os.path.basename(path) == "libgdn_checked.so"
    Lc = gdn.lib_checked()
    for name in gdn.EXPORTS:
        assert hasattr(Lc, name), name
    assert Lc.gdn_status_string(gdn.GDN_ERR_BOUNDS).decode().startswith("index check failed")
    assert Lc.gdn_abi_version() == L_abi_version()


def L_abi_version():
    return gdn.lib().gdn_abi_version()


def test_debug_options_are_checked(L):
    bad = [dict(chain_split=3), dict(segment_chunks=-1), dict(fault=7),
           dict(fault=1, fault_chunk=-1), dict(wait_limit_us=10_000_001)]
    for kw in bad:
        opts = gdn.DebugOptions(**{**dict(wait_limit_us=0, segment_chunks=0, chain_split=0,
                                          fault=0, fault_chunk=0), **kw})
        assert L.gdn_debug_set(ctypes.byref(opts)) == gdn.GDN_ERR_INVALID_ARG, kw
    ok = gdn.DebugOptions(5000, 2, 4, gdn.GDN_FAULT_SKIP_CHAIN_LOAD, 3)
    assert L.gdn_debug_set(ctypes.byref(ok)) == gdn.GDN_OK
    assert L.gdn_debug_set(None) == gdn.GDN_OK
    # the workspace size follows the segment length (one fp32 state per segment boundary)
    d = ctypes.byref(gdn.Dims())
    plain = L.gdn_chunk_prefill_workspace_size(d, 1, 1, 4096)
    with gdn.debug_options(segment_chunks=8):
        seg = L.gdn_chunk_prefill_workspace_size(d, 1, 1, 4096)
    assert seg > plain
    assert L.gdn_chunk_prefill_workspace_size(d, 1, 1, 4096) == plain


def test_default_pipeline_segments(L):
    # Calls are cut into segments from 512 chunks on (64 chunks each, 128 from 1024 chunks),
    # one fp32 carry state [Hv, d, d] per segment boundary in the workspace: the workspace size
    # shows the number of segments the library chose.
    d = ctypes.byref(gdn.Dims())
    carry = 32 * 128 * 128 * 4

    def carries(T):
        size = L.gdn_chunk_prefill_workspace_size(d, 1, 1, T)
        with gdn.debug_options(segment_chunks=1 << 19):   # one launch of each kernel
            single = L.gdn_chunk_prefill_workspace_size(d, 1, 1, T)
        assert (size - single) % carry == 0
        return (size - single) // carry

    assert carries(510 * 128) == 0       # 511 chunks: one launch
    assert carries(511 * 128) == 7       # 512 chunks: 8 segments of 64
    assert carries(1023 * 128) == 7      # 1024 chunks: 8 segments of 128
    assert carries(262144) == 16         # 2049 chunks: 17 segments of 121
