"""Helpers shared by the GPU parity tests: run the CUDA path through the binding and the
fp64 oracle on the same seeded CPU tensors, and compare."""
import numpy as np
import torch

import oracle
import gated_deltanet_layer_02_b200 as gdn
from gated_deltanet_layer_02_b200 import build as gdn_build

#: Tolerances.  fp32 activations: max-abs error <= 1e-4.  bf16 activations: relative RMS
#: error ||gpu - oracle||_2 / ||oracle||_2 <= 2e-2 per tensor (outputs and final states
#: separately).  The max-abs / rms reading is not used for bf16: rounding the exact result to
#: bf16 already exceeds it on heavy-tailed normalised outputs (tests/test_tolerance_reading.py).
#: A guard against localised errors that an RMS can hide: at most 0.2% of the elements may be
#: off by more than 0.1 * rms(oracle).
TOL_F32_ABS = 1e-4
TOL_BF16_REL_RMS = 2e-2
GUARD_FRAC, GUARD_LEVEL = 2e-3, 0.1

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


def oracle_prefill(w, inp, out_t0=0):
    return oracle.prefill(oracle_dims_of(w), inp["x"], inp["beta"], inp["g"], inp["cu_seqlens"],
                          conv_w=inp["conv_w"], z=inp["z"], norm_w=inp["norm_w"], S0=inp["S0"],
                          conv0=inp["conv0"], out_t0=out_t0)


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


def outlier_fraction(got, ref, level=GUARD_LEVEL):
    got, ref = np64(got), np64(ref)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.mean(np.abs(got - ref) > level * rms))


def max_abs(got, ref):
    return float(np.max(np.abs(np64(got) - np64(ref)))) if np64(ref).size else 0.0


def assert_close(got, ref, dtype, what):
    """Parity bar of the path; returns the error figure it was judged on."""
    assert np.all(np.isfinite(np64(got))), f"{what}: non-finite values"
    if dtype == torch.float32:
        err = max_abs(got, ref)
        assert err <= TOL_F32_ABS, f"{what}: max-abs {err:.3g} > {TOL_F32_ABS}"
        return err
    err = rel_rms(got, ref)
    frac = outlier_fraction(got, ref)
    info = f"rel-rms {err:.3g}, max-abs/rms {max_abs_over_rms(got, ref):.3g}, outliers {frac:.2g}"
    assert err <= TOL_BF16_REL_RMS, f"{what}: {info}"
    assert frac <= GUARD_FRAC, f"{what}: {info}"
    return err
