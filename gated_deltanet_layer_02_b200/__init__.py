"""B200-native Gated DeltaNet layer: thin Python binding over libgdn.so (see include/gdn.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of libgdn.so.
PyTorch provides device memory and the current stream.  There is no CPU fallback: if the
library is missing or a tensor is not on a CUDA device, the call raises.

    import gated_deltanet_layer_02_b200 as gdn
    out, SN, convN = gdn.chunk_prefill(x, beta, g, cu_seqlens, conv_w=w, z=z, norm_w=nw)
    out = gdn.decode_step(x_t, beta_t, g_t, conv_state, S, conv_w=w, z=z_t, norm_w=nw)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, \
    GDN_ERR_WORKSPACE, GDN_ERR_BOUNDS = 0, -1, -2, -3, -4, -5, -6
GDN_F32, GDN_BF16 = 0, 1

#: every symbol include/gdn.h declares
EXPORTS = (
    "gdn_abi_version", "gdn_conv_channels", "gdn_status_string", "gdn_conv1d_update",
    "gdn_gated_rmsnorm", "gdn_chunk_prefill_workspace_size", "gdn_chunk_prefill",
    "gdn_decode_step", "gdn_trace_create", "gdn_trace_destroy", "gdn_trace_attach",
    "gdn_trace_reset", "gdn_trace_count", "gdn_trace_get", "gdn_debug_wait_probe",
    "gdn_chunk_prefill_static_ws", "gdn_trace_span", "gdn_decode_step_bf16_state",
    "gdn_chunk_prefill_states", "gdn_decode_multi", "gdn_block_prefill_workspace_size",
    "gdn_block_prefill", "gdn_chunk_prefill_slots", "gdn_chunk_prefill_host_plan",
    "gdn_chunk_prefill_host_workspace_size", "gdn_chunk_prefill_host", "gdn_debug_set",
    "gdn_chunk_prefill_pages",
)

#: size of the library-owned scratch used by chunk_prefill_static_ws (GDN_STATIC_WORKSPACE_BYTES)
STATIC_WORKSPACE_BYTES = 64 << 20


GDN_FAULT_NONE, GDN_FAULT_SKIP_CHAIN_LOAD = 0, 1


class DebugOptions(ctypes.Structure):
    """gdn_debug_options (see gdn.h): test and debug controls of the calling host thread."""
    _fields_ = [("wait_limit_us", ctypes.c_uint32), ("segment_chunks", ctypes.c_int32),
                ("chain_split", ctypes.c_int32), ("fault", ctypes.c_int32),
                ("fault_chunk", ctypes.c_int32), ("timestamps", ctypes.c_void_p)]


class GdnError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")
        self.code = code


class Dims(ctypes.Structure):
    """gdn_dims: layer shape.  Defaults are the Qwen3-Next values."""
    _fields_ = [("num_k_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("conv_kernel", ctypes.c_int32),
                ("q_scale", ctypes.c_float), ("l2_eps", ctypes.c_float),
                ("norm_eps", ctypes.c_float)]

    def __init__(self, num_k_heads=16, num_v_heads=32, head_dim=128, conv_kernel=4, q_scale=1.0,
                 l2_eps=1e-6, norm_eps=1e-6):
        super().__init__(num_k_heads, num_v_heads, head_dim, conv_kernel, q_scale, l2_eps, norm_eps)

    @property
    def channels(self) -> int:
        return (2 * self.num_k_heads + self.num_v_heads) * self.head_dim


_lib = None
_lock = threading.Lock()
LIB_CHECKED_PATH = os.path.join(_HERE, "libgdn_checked.so")


def _configure(L):
    """Sets the ctypes signatures of every entry point on a loaded libgdn (or its checked
    variant) and checks that each declared symbol resolves."""
    vp, i32, dp = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(Dims)
    L.gdn_abi_version.restype = ctypes.c_int
    L.gdn_conv_channels.argtypes = [dp]
    L.gdn_conv_channels.restype = ctypes.c_int64
    L.gdn_status_string.argtypes = [ctypes.c_int]
    L.gdn_status_string.restype = ctypes.c_char_p
    L.gdn_conv1d_update.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, i32, i32, vp, vp, vp]
    L.gdn_gated_rmsnorm.argtypes = [ctypes.c_int, vp, vp, vp, ctypes.c_float, i32, i32, vp, vp]
    L.gdn_chunk_prefill_workspace_size.argtypes = [dp, ctypes.c_int, i32, i32]
    L.gdn_chunk_prefill_workspace_size.restype = ctypes.c_size_t
    L.gdn_chunk_prefill.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, i32, i32,
                                    vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
    L.gdn_chunk_prefill_states.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                           i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                           ctypes.c_size_t, vp, vp]
    L.gdn_chunk_prefill_pages.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, i32,
                                          i32, vp, vp, vp, vp, vp, i32, vp, vp,
                                          ctypes.c_size_t, vp, vp]
    L.gdn_decode_step.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                  i32, vp, vp, vp]
    L.gdn_decode_step_bf16_state.argtypes = L.gdn_decode_step.argtypes
    L.gdn_decode_multi.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   i32, i32, i32, vp, vp, vp, vp]
    L.gdn_chunk_prefill_slots.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                          i32, i32, vp, i32, vp, vp, vp, vp,
                                          ctypes.c_size_t, vp, vp]
    L.gdn_chunk_prefill_host_plan.argtypes = [vp, i32, i32, i32, vp, i32]
    L.gdn_chunk_prefill_host_plan.restype = ctypes.c_int32
    L.gdn_chunk_prefill_host_workspace_size.argtypes = [dp, vp, i32, i32, i32]
    L.gdn_chunk_prefill_host_workspace_size.restype = ctypes.c_size_t
    L.gdn_chunk_prefill_host.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp,
                                         vp, vp, vp, i32, vp, ctypes.c_size_t, vp, vp]
    L.gdn_block_prefill_workspace_size.argtypes = [dp, i32, i32, i32]
    L.gdn_block_prefill_workspace_size.restype = ctypes.c_size_t
    L.gdn_block_prefill.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                    i32, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
    L.gdn_trace_create.argtypes = [ctypes.POINTER(vp)]
    L.gdn_trace_destroy.argtypes = [vp]
    L.gdn_trace_attach.argtypes = [vp]
    L.gdn_trace_reset.argtypes = [vp]
    L.gdn_trace_count.argtypes = [vp]
    L.gdn_trace_get.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_char_p),
                                ctypes.POINTER(ctypes.c_float)]
    L.gdn_trace_span.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_float),
                                 ctypes.POINTER(ctypes.c_float)]
    L.gdn_debug_wait_probe.argtypes = [vp, ctypes.c_uint32, vp]
    L.gdn_debug_set.argtypes = [ctypes.POINTER(DebugOptions)]
    L.gdn_chunk_prefill_static_ws.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                              i32, i32, vp, vp, vp, vp, vp, vp, vp]
    for name in EXPORTS:  # every declared symbol must resolve
        getattr(L, name)
    return L


def lib_checked():
    """The bounds-check build (libgdn_checked.so, built with
    `python -m gated_deltanet_layer_02_b200.build --bounds-check`), loaded beside libgdn.so for
    tests: the same entry points, kernels compiled with -DGDN_BOUNDS_CHECK."""
    if not os.path.exists(LIB_CHECKED_PATH):
        raise RuntimeError(f"{LIB_CHECKED_PATH} is missing: build it with "
                           "`python -m gated_deltanet_layer_02_b200.build --bounds-check`")
    return _configure(ctypes.CDLL(LIB_CHECKED_PATH))


def lib():
    """The loaded libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m gated_deltanet_layer_02_b200.build`")
            _lib = _configure(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def _check(fn, code):
    if code != GDN_OK:
        raise GdnError(fn, code)


def _ptr(t, name, dtype=None, allow_none=True):
    if t is None:
        if not allow_none:
            raise ValueError(f"{name} is required")
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device (no CPU fallback)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _need(t, name, n):
    """The C ABI takes bare pointers: refuse a tensor too small for what the call touches."""
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {n}")


def _need_layer(dims, T, N, x=None, beta=None, g=None, z=None, out=None, conv_w=None,
                norm_w=None, S0=None, SN=None, conv0=None, convN=None):
    Cc, Hv, d, K = dims.channels, dims.num_v_heads, dims.head_dim, dims.conv_kernel
    for t, name, n in ((x, "x", T * Cc), (beta, "beta", T * Hv), (g, "g", T * Hv),
                       (z, "z", T * Hv * d), (out, "out", T * Hv * d), (conv_w, "conv_w", Cc * K),
                       (norm_w, "norm_w", d), (S0, "S0", N * Hv * d * d),
                       (SN, "SN", N * Hv * d * d), (conv0, "conv0", N * (K - 1) * Cc),
                       (convN, "convN", N * (K - 1) * Cc)):
        _need(t, name, n)


def _pool_rows(S, conv_state, dims):
    """Rows of a state pool pair: whole [Hv, d, d] states in S that have a conv history row."""
    per_S = dims.num_v_heads * dims.head_dim ** 2
    rows = S.numel() // per_S if S is not None else 0
    if conv_state is not None:
        rows = min(rows, conv_state.numel() // ((dims.conv_kernel - 1) * dims.channels))
    return rows


def _act_dtype(t):
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"activations must be bfloat16 or float32, got {t.dtype}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def conv_channels(dims: Dims) -> int:
    return int(lib().gdn_conv_channels(ctypes.byref(dims)))


def conv1d_update(x, conv_w, cu_seqlens, conv_state_in=None, conv_state_out=None, y=None,
                  dims: Dims | None = None):
    """silu(causal depthwise conv) of packed sequences; returns y [T, Cc]."""
    dims = dims or Dims()
    dt = _act_dtype(x)
    y = torch.empty_like(x) if y is None else y
    N = cu_seqlens.numel() - 1
    Cc, K, T = dims.channels, dims.conv_kernel, x.shape[0]
    for t, name, n in ((x, "x", T * Cc), (y, "y", T * Cc), (conv_w, "conv_w", Cc * K),
                       (conv_state_in, "conv_state_in", N * (K - 1) * Cc),
                       (conv_state_out, "conv_state_out", N * (K - 1) * Cc)):
        _need(t, name, n)
    _check("gdn_conv1d_update", lib().gdn_conv1d_update(
        ctypes.byref(dims), dt, _ptr(x, "x", x.dtype), _ptr(y, "y", x.dtype),
        _ptr(conv_w, "conv_w", x.dtype), _ptr(cu_seqlens, "cu_seqlens", torch.int32), N,
        x.shape[0], _ptr(conv_state_in, "conv_state_in", x.dtype),
        _ptr(conv_state_out, "conv_state_out", x.dtype), _stream()))
    return y


def gated_rmsnorm(o, z, w=None, eps: float = 1e-6, y=None):
    """y = o / sqrt(mean(o^2) + eps) * w * silu(z) over the last dim."""
    dt = _act_dtype(o)
    y = torch.empty_like(o) if y is None else y
    dim = o.shape[-1]
    rows = o.numel() // dim if dim else 0
    _need(z, "z", rows * dim)
    _need(y, "y", rows * dim)
    _need(w, "w", dim)
    _check("gdn_gated_rmsnorm", lib().gdn_gated_rmsnorm(
        dt, _ptr(o, "o", o.dtype), _ptr(z, "z", o.dtype), _ptr(w, "w", o.dtype), float(eps),
        rows, dim, _ptr(y, "y", o.dtype), _stream()))
    return y


def prefill_workspace_size(num_seqs: int, num_tokens: int, dtype=torch.bfloat16,
                           dims: Dims | None = None) -> int:
    dims = dims or Dims()
    return int(lib().gdn_chunk_prefill_workspace_size(
        ctypes.byref(dims), GDN_BF16 if dtype == torch.bfloat16 else GDN_F32, num_seqs,
        num_tokens))


def chunk_prefill(x, beta, g, cu_seqlens, conv_w=None, z=None, norm_w=None, S0=None, SN=None,
                  conv0=None, convN=None, out=None, workspace=None, dev_status=None,
                  want_state=True, dims: Dims | None = None, chunk_states=None,
                  page_states=None, page_size: int = 128):
    """The whole layer over packed sequences.  Returns (out, SN, convN).

    x [T, Cc], beta/g [T, Hv] fp32, z [T, Hv, d] or None, cu_seqlens [N+1] int32 (device),
    S0 [N, Hv, d, d] fp32 or None, conv0 [N, K-1, Cc] or None.  chunk_states [C, Hv, d, d] fp32
    (C = sum of ceil(L_n / 128)) receives the state after every 128-token chunk
    (gdn_chunk_prefill_states); page_states [P, Hv, d, d] (P = sum of ceil(L_n / page_size))
    the state after every page of 64 or 128 tokens (gdn_chunk_prefill_pages).
    """
    dims = dims or Dims()
    dt = _act_dtype(x)
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    Hv, d, K = dims.num_v_heads, dims.head_dim, dims.conv_kernel
    dev = x.device
    if out is None:
        out = torch.empty((T, Hv, d), dtype=x.dtype, device=dev)
    if want_state and SN is None:
        SN = torch.empty((N, Hv, d, d), dtype=torch.float32, device=dev)
    if want_state and convN is None:
        convN = torch.empty((N, K - 1, dims.channels), dtype=x.dtype, device=dev)
    _need_layer(dims, T, N, x, beta, g, z, out, conv_w, norm_w, S0, SN, conv0, convN)
    need = prefill_workspace_size(N, T, x.dtype, dims)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    head = (ctypes.byref(dims), dt, _ptr(x, "x", x.dtype), _ptr(conv_w, "conv_w", x.dtype),
            _ptr(beta, "beta", torch.float32), _ptr(g, "g", torch.float32), _ptr(z, "z", x.dtype),
            _ptr(norm_w, "norm_w", x.dtype), _ptr(cu_seqlens, "cu_seqlens", torch.int32), N, T,
            _ptr(S0, "S0", torch.float32), _ptr(SN, "SN", torch.float32),
            _ptr(conv0, "conv0", x.dtype), _ptr(convN, "convN", x.dtype),
            _ptr(out, "out", x.dtype))
    tail = (_ptr(workspace, "workspace", torch.uint8), workspace.numel(),
            _ptr(dev_status, "dev_status", torch.int32), _stream())
    if page_states is not None:
        _check("gdn_chunk_prefill_pages", lib().gdn_chunk_prefill_pages(
            *head, int(page_size), _ptr(page_states, "page_states", torch.float32), *tail))
    elif chunk_states is None:
        _check("gdn_chunk_prefill", lib().gdn_chunk_prefill(*head, *tail))
    else:
        _check("gdn_chunk_prefill_states", lib().gdn_chunk_prefill_states(
            *head, _ptr(chunk_states, "chunk_states", torch.float32), *tail))
    return out, SN, convN


def chunk_prefill_slots(x, beta, g, cu_seqlens, S_pool, slot_idx=None, conv_pool=None,
                        conv_w=None, z=None, norm_w=None, out=None, workspace=None,
                        dev_status=None, dims: Dims | None = None):
    """chunk_prefill with the states in pools shared with decode_step: sequence n starts from
    and overwrites S_pool[slot_idx[n]] ([slots, Hv, d, d] fp32) and conv_pool[slot_idx[n]]
    ([slots, K-1, Cc]).  Slots must be distinct; a slot outside [0, slots) is skipped on the
    device and reported in dev_status (GDN_ERR_INVALID_ARG).  Returns out [T, Hv, d]."""
    dims = dims or Dims()
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, dims.num_v_heads, dims.head_dim), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(prefill_workspace_size(N, T, x.dtype, dims), 256),
                                dtype=torch.uint8, device=x.device)
    _need_layer(dims, T, N, x, beta, g, z, out, conv_w, norm_w)
    num_slots = _pool_rows(S_pool, conv_pool, dims)
    if slot_idx is None and num_slots < N:   # identity slots: rows 0 .. N-1 of the pools
        raise ValueError(f"the pools hold {num_slots} rows; the call needs {N}")
    _need(slot_idx, "slot_idx", N)
    _check("gdn_chunk_prefill_slots", lib().gdn_chunk_prefill_slots(
        ctypes.byref(dims), _act_dtype(x), _ptr(x, "x", x.dtype), _ptr(conv_w, "conv_w", x.dtype),
        _ptr(beta, "beta", torch.float32), _ptr(g, "g", torch.float32), _ptr(z, "z", x.dtype),
        _ptr(norm_w, "norm_w", x.dtype), _ptr(cu_seqlens, "cu_seqlens", torch.int32), N, T,
        _ptr(slot_idx, "slot_idx", torch.int32), num_slots, _ptr(S_pool, "S_pool", torch.float32),
        _ptr(conv_pool, "conv_pool", x.dtype), _ptr(out, "out", x.dtype),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return out


def _hptr(t, name, dtype, allow_none=True):
    """Pointer of a host (CPU) tensor."""
    if t is None:
        if not allow_none:
            raise ValueError(f"{name} is required")
        return None
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a CPU tensor (host memory)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def host_plan(cu_seqlens, segment_tokens: int = 0):
    """The segments gdn_chunk_prefill_host cuts a batch into: [k, 4] int32 rows
    (first sequence, sequences, first token, tokens).  cu_seqlens: CPU int32."""
    cu = cu_seqlens.to(torch.int32).contiguous()
    N, T = cu.numel() - 1, int(cu[-1]) if cu.numel() else 0
    L = lib()
    n = L.gdn_chunk_prefill_host_plan(_hptr(cu, "cu_seqlens", torch.int32), N, T,
                                      segment_tokens, None, 0)
    _check("gdn_chunk_prefill_host_plan", min(n, 0))
    segs = torch.zeros((max(n, 1), 4), dtype=torch.int32)
    n2 = L.gdn_chunk_prefill_host_plan(_hptr(cu, "cu_seqlens", torch.int32), N, T,
                                       segment_tokens, _hptr(segs, "segments", torch.int32), n)
    _check("gdn_chunk_prefill_host_plan", min(n2, 0))
    return segs[:n]


def chunk_prefill_host(x, beta, g, cu_seqlens, conv_w=None, z=None, norm_w=None, S0=None, SN=None,
                       conv0=None, convN=None, out=None, workspace=None, segment_tokens: int = 0,
                       dev_status=None, dims: Dims | None = None):
    """chunk_prefill (bf16) with x, beta, g, z, cu_seqlens and out in HOST memory (pin them for
    the copies to overlap the kernels); weights, states and the workspace on the device.
    Returns (out, SN, convN); out is valid once the current stream has reached the call."""
    dims = dims or Dims()
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    Hv, d, K = dims.num_v_heads, dims.head_dim, dims.conv_kernel
    dev = torch.device("cuda", torch.cuda.current_device())
    bf = torch.bfloat16
    if out is None:
        out = torch.empty((T, Hv, d), dtype=bf, pin_memory=True)
    if SN is None:
        SN = torch.empty((N, Hv, d, d), dtype=torch.float32, device=dev)
    if convN is None:
        convN = torch.empty((N, K - 1, dims.channels), dtype=bf, device=dev)
    _need_layer(dims, T, N, x, beta, g, z, out, conv_w, norm_w, S0, SN, conv0, convN)
    cu_p = _hptr(cu_seqlens, "cu_seqlens", torch.int32, allow_none=False)
    need = lib().gdn_chunk_prefill_host_workspace_size(ctypes.byref(dims), cu_p, N, T,
                                                       segment_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check("gdn_chunk_prefill_host", lib().gdn_chunk_prefill_host(
        ctypes.byref(dims), _hptr(x, "x", bf), _ptr(conv_w, "conv_w", bf),
        _hptr(beta, "beta", torch.float32), _hptr(g, "g", torch.float32), _hptr(z, "z", bf),
        _ptr(norm_w, "norm_w", bf), cu_p, N, T, _ptr(S0, "S0", torch.float32),
        _ptr(SN, "SN", torch.float32), _ptr(conv0, "conv0", bf), _ptr(convN, "convN", bf),
        _hptr(out, "out", bf), segment_tokens, _ptr(workspace, "workspace", torch.uint8),
        workspace.numel(), _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return out, SN, convN


def chunk_prefill_static_ws(x, beta, g, cu_seqlens, conv_w=None, z=None, norm_w=None, S0=None,
                            SN=None, conv0=None, convN=None, out=None, dev_status=None,
                            want_state=True, dims: Dims | None = None):
    """chunk_prefill without a caller workspace: the library's own 64 MiB device scratch is used.

    For callers that cannot allocate device memory.  Calls on one device share that scratch, so
    they must not overlap on the GPU.  Sizes needing more scratch raise GdnError
    (GDN_ERR_WORKSPACE).  Returns (out, SN, convN) like chunk_prefill.
    """
    dims = dims or Dims()
    dt = _act_dtype(x)
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    Hv, d, K = dims.num_v_heads, dims.head_dim, dims.conv_kernel
    dev = x.device
    if out is None:
        out = torch.empty((T, Hv, d), dtype=x.dtype, device=dev)
    if want_state and SN is None:
        SN = torch.empty((N, Hv, d, d), dtype=torch.float32, device=dev)
    if want_state and convN is None:
        convN = torch.empty((N, K - 1, dims.channels), dtype=x.dtype, device=dev)
    _need_layer(dims, T, N, x, beta, g, z, out, conv_w, norm_w, S0, SN, conv0, convN)
    _check("gdn_chunk_prefill_static_ws", lib().gdn_chunk_prefill_static_ws(
        ctypes.byref(dims), dt, _ptr(x, "x", x.dtype), _ptr(conv_w, "conv_w", x.dtype),
        _ptr(beta, "beta", torch.float32), _ptr(g, "g", torch.float32), _ptr(z, "z", x.dtype),
        _ptr(norm_w, "norm_w", x.dtype), _ptr(cu_seqlens, "cu_seqlens", torch.int32), N, T,
        _ptr(S0, "S0", torch.float32), _ptr(SN, "SN", torch.float32),
        _ptr(conv0, "conv0", x.dtype), _ptr(convN, "convN", x.dtype), _ptr(out, "out", x.dtype),
        _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return out, SN, convN


def decode_step(x, beta, g, conv_state, S, conv_w, z=None, norm_w=None, slot_idx=None,
                out=None, dev_status=None, dims: Dims | None = None):
    """One token per sequence; conv_state and S are updated in place.  Returns out [B, Hv, d].
    S may be fp32 (gdn_decode_step) or bf16 (gdn_decode_step_bf16_state).  A slot outside the
    pools is skipped on the device and reported in dev_status (GDN_ERR_INVALID_ARG)."""
    dims = dims or Dims()
    dt = _act_dtype(x)
    B = x.shape[0]
    if out is None:
        out = torch.empty((B, dims.num_v_heads, dims.head_dim), dtype=x.dtype, device=x.device)
    bf16_state = S is not None and S.dtype == torch.bfloat16
    _need_layer(dims, B, 0, x, beta, g, z, out, conv_w, norm_w)
    num_slots = _pool_rows(S, conv_state, dims)
    if slot_idx is None and num_slots < B:   # identity slots: rows 0 .. B-1 of the pools
        raise ValueError(f"the state pools hold {num_slots} rows; the call needs {B}")
    _need(slot_idx, "slot_idx", B)
    name = "gdn_decode_step_bf16_state" if bf16_state else "gdn_decode_step"
    _check(name, getattr(lib(), name)(
        ctypes.byref(dims), dt, _ptr(x, "x", x.dtype), _ptr(conv_w, "conv_w", x.dtype, False),
        _ptr(beta, "beta", torch.float32), _ptr(g, "g", torch.float32), _ptr(z, "z", x.dtype),
        _ptr(norm_w, "norm_w", x.dtype), _ptr(conv_state, "conv_state", x.dtype),
        _ptr(S, "S", torch.bfloat16 if bf16_state else torch.float32),
        _ptr(slot_idx, "slot_idx", torch.int32), num_slots, B, _ptr(out, "out", x.dtype),
        _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return out


def decode_multi(x, beta, g, conv_state, S, conv_w, z=None, norm_w=None, slot_idx=None,
                 out=None, snapshots=None, dev_status=None, dims: Dims | None = None):
    """k tokens per sequence (x [B, k, Cc]); conv_state and S (fp32) are updated in place.
    Returns out [B, k, Hv, d]; snapshots [B, k, Hv, d, d] fp32 receives the state after each
    token when given."""
    dims = dims or Dims()
    dt = _act_dtype(x)
    B, k = x.shape[0], x.shape[1]
    if out is None:
        out = torch.empty((B, k, dims.num_v_heads, dims.head_dim), dtype=x.dtype, device=x.device)
    _need_layer(dims, B * k, 0, x, beta, g, z, out, conv_w, norm_w)
    num_slots = _pool_rows(S, conv_state, dims)
    if slot_idx is None and num_slots < B:   # identity slots: rows 0 .. B-1 of the pools
        raise ValueError(f"the state pools hold {num_slots} rows; the call needs {B}")
    _need(slot_idx, "slot_idx", B)
    _need(snapshots, "snapshots", B * k * dims.num_v_heads * dims.head_dim ** 2)
    _check("gdn_decode_multi", lib().gdn_decode_multi(
        ctypes.byref(dims), dt, _ptr(x, "x", x.dtype), _ptr(conv_w, "conv_w", x.dtype, False),
        _ptr(beta, "beta", torch.float32), _ptr(g, "g", torch.float32), _ptr(z, "z", x.dtype),
        _ptr(norm_w, "norm_w", x.dtype), _ptr(conv_state, "conv_state", x.dtype),
        _ptr(S, "S", torch.float32), _ptr(slot_idx, "slot_idx", torch.int32), num_slots, B, k,
        _ptr(out, "out", x.dtype), _ptr(snapshots, "snapshots", torch.float32),
        _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return out


def block_prefill(h, w_qkv, w_z, w_ba, a_log, dt_bias, w_out, cu_seqlens, conv_w=None,
                  norm_w=None, S0=None, SN=None, conv0=None, convN=None, y=None, workspace=None,
                  dev_status=None, dims: Dims | None = None):
    """Projections + gates + layer + output projection (bf16).  h [T, H] -> y [T, H].
    Returns (y, SN, convN)."""
    dims = dims or Dims()
    T, H = h.shape
    N = cu_seqlens.numel() - 1
    Hv, d, K = dims.num_v_heads, dims.head_dim, dims.conv_kernel
    dev = h.device
    if y is None:
        y = torch.empty((T, H), dtype=h.dtype, device=dev)
    if SN is None:
        SN = torch.empty((N, Hv, d, d), dtype=torch.float32, device=dev)
    if convN is None:
        convN = torch.empty((N, K - 1, dims.channels), dtype=h.dtype, device=dev)
    Cc, HD = dims.channels, Hv * d
    for t, name, n in ((h, "h", T * H), (y, "y", T * H), (w_qkv, "w_qkv", H * Cc),
                       (w_z, "w_z", H * HD), (w_ba, "w_ba", H * 2 * Hv), (a_log, "a_log", Hv),
                       (dt_bias, "dt_bias", Hv), (w_out, "w_out", HD * H)):
        _need(t, name, n)
    _need_layer(dims, T, N, conv_w=conv_w, norm_w=norm_w, S0=S0, SN=SN, conv0=conv0,
                convN=convN)
    need = lib().gdn_block_prefill_workspace_size(ctypes.byref(dims), H, N, T)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    bf = torch.bfloat16
    _check("gdn_block_prefill", lib().gdn_block_prefill(
        ctypes.byref(dims), H, _ptr(h, "h", bf), _ptr(w_qkv, "w_qkv", bf), _ptr(w_z, "w_z", bf),
        _ptr(w_ba, "w_ba", bf), _ptr(a_log, "a_log", torch.float32),
        _ptr(dt_bias, "dt_bias", torch.float32), _ptr(conv_w, "conv_w", bf),
        _ptr(norm_w, "norm_w", bf), _ptr(w_out, "w_out", bf),
        _ptr(cu_seqlens, "cu_seqlens", torch.int32), N, T, _ptr(S0, "S0", torch.float32),
        _ptr(SN, "SN", torch.float32), _ptr(conv0, "conv0", bf), _ptr(convN, "convN", bf),
        _ptr(y, "y", bf), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _ptr(dev_status, "dev_status", torch.int32), _stream()))
    return y, SN, convN


class debug_options:
    """Context manager around gdn_debug_set: the library calls of this host thread inside the
    block use the given settings; leaving the block restores the defaults.

        with gdn.debug_options(segment_chunks=2, chain_split=4):
            gdn.chunk_prefill(...)
    """

    def __init__(self, wait_limit_us=0, segment_chunks=0, chain_split=0, fault=GDN_FAULT_NONE,
                 fault_chunk=0, timestamps=None):
        ts = None if timestamps is None else _ptr(timestamps, "timestamps", torch.int64)
        self.opts = DebugOptions(wait_limit_us, segment_chunks, chain_split, fault, fault_chunk,
                                 ts)

    def __enter__(self):
        _check("gdn_debug_set", lib().gdn_debug_set(ctypes.byref(self.opts)))
        return self

    def __exit__(self, *exc):
        lib().gdn_debug_set(None)


def debug_wait_probe(dev_status, limit_us: int):
    """Launch a kernel whose wait nothing satisfies; it gives up after limit_us."""
    _check("gdn_debug_wait_probe", lib().gdn_debug_wait_probe(
        _ptr(dev_status, "dev_status", torch.int32, False), int(limit_us), _stream()))


class Trace:
    """Per-launch device times of the library's kernels (CUDA events on the launch stream)."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check("gdn_trace_create", lib().gdn_trace_create(ctypes.byref(h)))
        self._h = h

    def __enter__(self):
        lib().gdn_trace_attach(self._h)
        return self

    def __exit__(self, *exc):
        lib().gdn_trace_attach(None)

    def reset(self):
        lib().gdn_trace_reset(self._h)

    def records(self):
        """[(kernel name, ms)] in launch order (synchronises on each end event)."""
        out = []
        for i in range(lib().gdn_trace_count(self._h)):
            name, ms = ctypes.c_char_p(), ctypes.c_float()
            _check("gdn_trace_get", lib().gdn_trace_get(self._h, i, ctypes.byref(name),
                                                        ctypes.byref(ms)))
            out.append((name.value.decode(), ms.value))
        return out

    def timeline(self):
        """[(kernel name, start ms, end ms)] relative to the start of the first launch."""
        out = []
        for i in range(lib().gdn_trace_count(self._h)):
            name, a, b = ctypes.c_char_p(), ctypes.c_float(), ctypes.c_float()
            _check("gdn_trace_get", lib().gdn_trace_get(self._h, i, ctypes.byref(name), None))
            _check("gdn_trace_span", lib().gdn_trace_span(self._h, i, ctypes.byref(a),
                                                          ctypes.byref(b)))
            out.append((name.value.decode(), a.value, b.value))
        return out

    def close(self):
        if self._h:
            lib().gdn_trace_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


__all__ = ["Dims", "GdnError", "lib", "conv1d_update", "gated_rmsnorm", "chunk_prefill",
           "decode_multi", "block_prefill", "chunk_prefill_slots",
           "chunk_prefill_host", "host_plan",
           "chunk_prefill_static_ws", "STATIC_WORKSPACE_BYTES",
           "decode_step", "prefill_workspace_size", "conv_channels", "status_string", "Trace",
           "debug_wait_probe", "debug_options", "DebugOptions", "EXPORTS", "LIB_PATH"]
