"""Helpers shared by the GPU parity tests: run the CUDA path through the binding and the
fp64 oracle on the same seeded CPU tensors, and compare."""
import json
import os

import numpy as np
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import build as gdn_build

#: Tolerances, all element-wise.
#:  * fp32 activations: max |gpu - oracle| <= 1e-4 on outputs and states.
#:  * bf16 activations: every element within 2e-2 of its error scale, plus one bf16 rounding
#:    of the value for bf16 tensors:   |gpu - oracle| <= 2e-2 * scale + 2^-8 * |oracle|
#:    (2^-8 only for bf16 results; fp32 recurrent states get 2e-2 * scale alone).  The scale of
#:    an element is the oracle's own measure of the terms that form it (gdn_oracle.c header:
#:    the magnitude M of the state recurrence, M |q| for an output, carried through the gated
#:    RMSNorm), so a small element made of large cancelling terms gets the tolerance of those
#:    terms.  Checks without such a scale (conv, standalone RMSNorm, conv history) use the
#:    tensor's RMS.  On top, the relative RMS error of the tensor must stay <= 2e-2.
#:    Near and below the smallest normal number of fp32 and bf16 (2^-126, the same 8-bit
#:    exponent in both) the path keeps no relative precision: an fp32 state that has decayed
#:    past it underflows, and a subnormal bf16 operand (e^G for G < -87 times a row of q) carries
#:    an absolute error of up to 2^-134, which a 128-term product and the RMSNorm (up to 1/sqrt
#:    of its eps, 10^3) multiply by far less than 2^34.  So 2^-100 (about 8e-31, some 10^29 below
#:    any tensor's RMS here) is added to every bound: results smaller than that count as zero.
#:    Why not 2e-2 * rms(oracle) + 2^-8 |oracle|: one bf16 rounding of the normalised q and k
#:    (the tensor-core operands) already moves the exact output by more than that on some
#:    elements (tests/test_tolerance_reading.py), so that bound measures the conditioning of
#:    the problem rather than the implementation.
#: Each check's figures go to the test output and, with GDN_PARITY_LOG=<file>, to a JSON-lines
#: log.
TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2
BF16_ULP_REL = 2.0 ** -8
TINY = 2.0 ** -100

_built = False


def ensure_built():
    global _built
    if not _built:
        gdn_build.build()
        _built = True


def dev(t):
    return None if t is None else t.cuda()


def dims_of(w, **kw):
    return gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel, **kw)


def oracle_dims_of(w, **kw):
    return oracle.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel, **kw)


def gpu_prefill(w, inp, dev_status=None, **kw):
    ensure_built()
    out, SN, convN = gdn.chunk_prefill(
        dev(inp["x"]), dev(inp["beta"]), dev(inp["g"]), dev(inp["cu_seqlens"]),
        conv_w=dev(inp["conv_w"]), z=dev(inp["z"]), norm_w=dev(inp["norm_w"]), S0=dev(inp["S0"]),
        conv0=dev(inp["conv0"]), dims=dims_of(w), dev_status=dev_status, **kw)
    torch.cuda.synchronize()
    return out, SN, convN


class Ref(tuple):
    """(out, SN, convN) of the oracle, unpacking like a 3-tuple, with the error scales of the
    out and SN elements as attributes (out_scale, SN_scale)."""

    def __new__(cls, out, SN, convN, out_scale=None, SN_scale=None):
        r = super().__new__(cls, (out, SN, convN))
        r.out_scale, r.SN_scale = out_scale, SN_scale
        return r


def oracle_prefill(w, inp, out_t0=0):
    r = oracle.prefill(oracle_dims_of(w), inp["x"], inp["beta"], inp["g"], inp["cu_seqlens"],
                       conv_w=inp["conv_w"], z=inp["z"], norm_w=inp["norm_w"], S0=inp["S0"],
                       conv0=inp["conv0"], out_t0=out_t0, with_scales=True)
    return Ref(*r)


def np64(t):
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else t


def rel_rms(got, ref):
    got, ref = np64(got), np64(ref)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.sqrt(np.mean((got - ref) ** 2)) / max(rms, 1e-30))


def max_abs_over_rms(got, ref):
    got, ref = np64(got), np64(ref)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-30))


def max_abs(got, ref):
    return float(np.max(np.abs(np64(got) - np64(ref)))) if np64(ref).size else 0.0


def _log(rec):
    path = os.environ.get("GDN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
    print("parity " + json.dumps(rec))


def assert_close(got, ref, dtype, what, scale=None, f32_scale=1.0):
    """Parity bar of the path (element-wise); returns the figure it was judged on.

    dtype is the activation dtype of the run; ``scale`` the oracle's error scale of every
    element (None: the tensor's RMS).  ``f32_scale`` multiplies the fp32 absolute bound for
    inputs deliberately drawn at that multiple of the workload's magnitude."""
    g, r = np64(got), np64(ref)
    assert g.shape == r.shape, f"{what}: shape {g.shape} != {r.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = np.abs(g - r)
    rms = float(np.sqrt(np.mean(r ** 2))) if r.size else 0.0
    rec = {"what": what, "n": int(r.size), "rms": rms,
           "max_abs": float(err.max()) if r.size else 0.0,
           "rel_rms": rel_rms(got, ref) if r.size else 0.0,
           "max_abs_over_rms": float(err.max() / max(rms, 1e-30)) if r.size else 0.0}
    if dtype == torch.float32:
        rec["kind"], rec["bound"] = "f32 max-abs", TOL_F32_ABS * f32_scale
        _log(rec)
        assert rec["max_abs"] <= TOL_F32_ABS * f32_scale, f"{what}: {rec}"
        return rec["max_abs"]
    is_bf16_tensor = isinstance(got, torch.Tensor) and got.dtype == torch.bfloat16
    s = rms if scale is None else np64(scale)
    if scale is not None:
        assert np.shape(s) == r.shape, f"{what}: scale shape {np.shape(s)} != {r.shape}"
    bound = TOL_BF16_REL * s + (BF16_ULP_REL * np.abs(r) if is_bf16_tensor else 0.0) + TINY
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if r.size else 0.0
    rec["kind"] = ("bf16 " if is_bf16_tensor else "fp32 ") + ("element scale" if scale is not None
                                                               else "tensor rms")
    rec["worst_over_bound"] = ratio
    _log(rec)
    assert rec["rel_rms"] <= TOL_BF16_REL, f"{what}: {rec}"
    assert ratio <= 1.0, f"{what}: {rec}"
    return ratio
