"""fp64 CPU oracle for the Gated DeltaNet layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import this package.  The CUDA product path never imports it, and
the two share no code; the only thing both sides use is the seeded input generator module
(``gated_deltanet_layer_02_b200.inputs``), which holds none of the layer's arithmetic.

This module is argument marshalling around ``gdn_oracle.c`` (plain C, fp64, sequential per
(sequence, value head) unit).  The header of that file lists what is computed, the sources and
every reading taken where the pages are silent.

``block_prefill`` composes the layer with plain matrix products and ``block_gates``.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` (closed forms,
invariants, brute force, library routines); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, F64 = 0, 1, 2


class _Dims(ctypes.Structure):
    _fields_ = [
        ("num_k_heads", ctypes.c_int32),
        ("num_v_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("conv_kernel", ctypes.c_int32),
        ("q_scale", ctypes.c_double),
        ("l2_eps", ctypes.c_double),
        ("norm_eps", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into oracle/_build/liboracle.so (gcc, -O2, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp, _SRC,
             "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, ip = ctypes.c_void_p, ctypes.c_int
            lib.orc_conv1d_silu.argtypes = [ip, vp, vp, vp, ip, ip, ip, ip, vp, vp, vp]
            lib.orc_gated_rmsnorm.argtypes = [ip, vp, vp, vp, ctypes.c_double, ip, ip, vp]
            lib.orc_prefill.argtypes = [ctypes.POINTER(_Dims), ip, vp, vp, vp, vp, vp, vp, vp, ip,
                                        ip, vp, vp, ctypes.c_longlong, vp, vp, vp, vp, vp, ip]
            lib.orc_decode_step.argtypes = [ctypes.POINTER(_Dims), ip, vp, vp, vp, vp, vp, vp, vp,
                                            vp, vp, ip, vp, vp, vp, ip]
            for f in (lib.orc_conv1d_silu, lib.orc_gated_rmsnorm, lib.orc_prefill,
                      lib.orc_decode_step):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


class Dims:
    """Layer shape: key/value heads, head dim, conv width, q scale and the two epsilons."""

    def __init__(self, num_k_heads=16, num_v_heads=32, head_dim=128, conv_kernel=4, q_scale=1.0,
                 l2_eps=1e-6, norm_eps=1e-6):
        self.num_k_heads, self.num_v_heads = num_k_heads, num_v_heads
        self.head_dim, self.conv_kernel = head_dim, conv_kernel
        self.q_scale, self.l2_eps, self.norm_eps = q_scale, l2_eps, norm_eps

    @property
    def channels(self) -> int:
        return (2 * self.num_k_heads + self.num_v_heads) * self.head_dim

    def _c(self) -> _Dims:
        return _Dims(self.num_k_heads, self.num_v_heads, self.head_dim, self.conv_kernel,
                     self.q_scale, self.l2_eps, self.norm_eps)


def _act(t, keep):
    """(dtype code, pointer) of an activation-like CPU tensor; `keep` holds references."""
    if t is None:
        return None, None
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        code = BF16
    elif t.dtype == torch.float32:
        code = F32
    elif t.dtype == torch.float64:
        code = F64
    else:
        raise TypeError(f"unsupported dtype {t.dtype}")
    keep.append(t)
    return code, ctypes.c_void_p(t.data_ptr())


def _f32(t, keep):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    t = t.detach().cpu().to(torch.float32).contiguous()
    keep.append(t)
    return ctypes.c_void_p(t.data_ptr())


def _i32(t, keep):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    t = t.detach().cpu().to(torch.int32).contiguous()
    keep.append(t)
    return ctypes.c_void_p(t.data_ptr())


def _same_dtype(codes):
    codes = [c for c in codes if c is not None]
    if len(set(codes)) > 1:
        raise TypeError("activation tensors must share one dtype")
    return codes[0] if codes else F32


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def conv1d_silu(x, w, cu_seqlens, conv_in=None):
    """Causal depthwise conv (width K) + SiLU over packed sequences.

    x [T, C], w [C, K], cu_seqlens [N+1], conv_in [N, K-1, C] or None.
    Returns (y [T, C] fp64, conv_out [N, K-1, C] fp64) as numpy arrays.
    """
    keep = []
    cx, px = _act(x, keep)
    cw, pw = _act(w, keep)
    cc, pc = _act(conv_in, keep)
    code = _same_dtype([cx, cw, cc])
    T, C = x.shape
    K = w.shape[1]
    N = len(cu_seqlens) - 1
    y = np.zeros((T, C), np.float64)
    conv_out = np.zeros((N, max(K - 1, 0), C), np.float64)
    rc = _load().orc_conv1d_silu(code, px, pw, _i32(cu_seqlens, keep), N, T, C, K, pc,
                                 y.ctypes.data_as(ctypes.c_void_p),
                                 conv_out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"orc_conv1d_silu failed: {rc}")
    return y, conv_out


def gated_rmsnorm(o, z, w, eps):
    """y = o / sqrt(mean(o^2) + eps) * w * silu(z) per row; o, z [M, d], w [d] or None."""
    keep = []
    co, po = _act(o, keep)
    cz, pz = _act(z, keep)
    cw, pw = _act(w, keep)
    code = _same_dtype([co, cz, cw])
    M, d = o.shape
    y = np.zeros((M, d), np.float64)
    rc = _load().orc_gated_rmsnorm(code, po, pz, pw, float(eps), M, d,
                                   y.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"orc_gated_rmsnorm failed: {rc}")
    return y


def prefill(dims: Dims, x, beta, g, cu_seqlens, conv_w=None, z=None, norm_w=None, S0=None,
            conv0=None, out_t0: int = 0, want_state: bool = True, nthreads: int | None = None,
            with_scales: bool = False):
    """Full layer over packed sequences (see gdn_oracle.c for the definition).

    Returns (out [T - out_t0, Hv, d], SN [N, Hv, d, d] or None, convN [N, K-1, Cc] or None),
    all fp64 numpy arrays.  With ``with_scales`` two more arrays follow: the element scales of
    out and the state magnitudes M (the error scales of the gdn_oracle.c header).
    """
    keep = []
    cx, px = _act(x, keep)
    cw, pw = _act(conv_w, keep)
    cz, pz = _act(z, keep)
    cn, pn = _act(norm_w, keep)
    cc, pc = _act(conv0, keep)
    code = _same_dtype([cx, cw, cz, cn, cc])
    T = x.shape[0]
    N = len(cu_seqlens) - 1
    Hv, d, K = dims.num_v_heads, dims.head_dim, dims.conv_kernel
    out = np.zeros((T - out_t0, Hv, d), np.float64)
    SN = np.zeros((N, Hv, d, d), np.float64) if want_state else None
    convN = np.zeros((N, K - 1, dims.channels), np.float64) if want_state else None
    out_scale = np.zeros_like(out) if with_scales else None
    SN_scale = np.zeros((N, Hv, d, d), np.float64) if with_scales else None
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p) if a is not None else None  # noqa: E731
    c_dims = dims._c()
    rc = _load().orc_prefill(
        ctypes.byref(c_dims), code, px, pw, _f32(beta, keep), _f32(g, keep), pz, pn,
        _i32(cu_seqlens, keep), N, T, _f32(S0, keep), pc, int(out_t0), ptr(out), ptr(SN),
        ptr(convN), ptr(out_scale), ptr(SN_scale), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"orc_prefill failed: {rc}")
    if with_scales:
        return out, SN, convN, out_scale, SN_scale
    return out, SN, convN


def block_gates(ba, a_log, dt_bias):
    """Per-token, per-value-head gates of the token mixer from the [T, 2 Hv] projection rows
    [b | a]: beta = sigmoid(b) and g = log(alpha) = -exp(A_log) * softplus(a + dt_bias).
    The pages (hyper.ai's Qwen3-Next paragraph) say only that beta sets the update strength
    and alpha the decay; this parameterisation is the reading taken for it.  fp64 numpy."""
    ba = np.asarray(ba, np.float64)
    Hv = ba.shape[1] // 2
    b, a = ba[:, :Hv], ba[:, Hv:] + np.asarray(dt_bias, np.float64)[None, :]
    beta = 1.0 / (1.0 + np.exp(-b))
    softplus = np.logaddexp(0.0, a)
    g = -np.exp(np.asarray(a_log, np.float64))[None, :] * softplus
    return beta, g


def block_prefill(dims: Dims, h, w_qkv, w_z, w_ba, a_log, dt_bias, w_out, cu_seqlens,
                  conv_w=None, norm_w=None, S0=None, conv0=None, nthreads: int | None = None,
                  with_scales: bool = False):
    """The token mixer of a decoder layer in fp64: x = h W_qkv, z = h W_z, [b | a] = h W_ba,
    the gates of block_gates, the layer (prefill) and y = o W_out.  Weights are [in, out].
    Returns (y [T, H], SN, convN) as fp64 numpy; the gates enter the layer rounded to fp32
    (its beta and g are fp32 inputs).  With ``with_scales`` the element scales of y (the
    layer's output scales carried through |W_out|) and the state magnitudes follow."""
    f64 = lambda t: np.asarray(t.detach().cpu().double().numpy() if isinstance(t, torch.Tensor)
                               else t, np.float64)
    hh = f64(h)
    T = hh.shape[0]
    x = hh @ f64(w_qkv)
    z = hh @ f64(w_z)
    beta, g = block_gates(hh @ f64(w_ba), f64(a_log), f64(dt_bias))
    to64 = lambda t: None if t is None else torch.from_numpy(f64(t))
    res = prefill(dims, torch.from_numpy(x), beta.astype(np.float32),
                  g.astype(np.float32), cu_seqlens, conv_w=to64(conv_w),
                  z=torch.from_numpy(z), norm_w=to64(norm_w), S0=S0, conv0=to64(conv0),
                  nthreads=nthreads, with_scales=with_scales)
    o, SN, convN = res[:3]
    HD = dims.num_v_heads * dims.head_dim
    y = o.reshape(T, HD) @ f64(w_out)
    if with_scales:
        y_scale = res[3].reshape(T, HD) @ np.abs(f64(w_out))
        return y, SN, convN, y_scale, res[4]
    return y, SN, convN


def decode_step(dims: Dims, x, beta, g, conv_state, S, conv_w=None, z=None, norm_w=None,
                slot_idx=None, nthreads: int | None = None, M=None):
    """One decode token per sequence; conv_state [slots, K-1, Cc] and S [slots, Hv, d, d] are
    fp64 numpy arrays updated in place.  Returns out [B, Hv, d] fp64.

    With ``M`` (fp64 like S; start it as |S|) the state magnitude of the gdn_oracle.c header is
    carried in place as well, and the call returns (out, element scales of out)."""
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert S.dtype == np.float64 and S.flags.c_contiguous
    if M is not None:
        assert M.dtype == np.float64 and M.flags.c_contiguous and M.shape == S.shape
    keep = []
    cx, px = _act(x, keep)
    cw, pw = _act(conv_w, keep)
    cz, pz = _act(z, keep)
    cn, pn = _act(norm_w, keep)
    code = _same_dtype([cx, cw, cz, cn])
    B = x.shape[0]
    out = np.zeros((B, dims.num_v_heads, dims.head_dim), np.float64)
    out_scale = np.zeros_like(out) if M is not None else None
    c_dims = dims._c()
    rc = _load().orc_decode_step(
        ctypes.byref(c_dims), code, px, pw, _f32(beta, keep), _f32(g, keep), pz, pn,
        conv_state.ctypes.data_as(ctypes.c_void_p), S.ctypes.data_as(ctypes.c_void_p),
        _i32(slot_idx, keep), B, out.ctypes.data_as(ctypes.c_void_p),
        M.ctypes.data_as(ctypes.c_void_p) if M is not None else None,
        out_scale.ctypes.data_as(ctypes.c_void_p) if out_scale is not None else None,
        int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"orc_decode_step failed: {rc}")
    return out if M is None else (out, out_scale)
