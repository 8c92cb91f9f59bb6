"""What the bf16 parity bar can and cannot ask (CPU only).

The workload statement asks for agreement "within 2e-2 relative-to-RMS" for bf16 activations.
Read as max|gpu - oracle| / rms(oracle), the bar would reject even the exact result rounded once
to bf16, because the z-gated RMSNorm output is heavy-tailed (elements reach 10-15x its RMS and
bf16 keeps 8 significant bits).  Read as ||gpu - oracle||_2 / ||oracle||_2 it is met by that
rounding with a wide margin.

An element-wise bar 2e-2 * rms(oracle) + 2^-8 |oracle| (one rounding of the value on top of the
RMS term) still fails for any implementation that feeds bf16 operands to the tensor cores: one
bf16 rounding of the L2-normalised q and k alone moves the exact output by more than that where
an output is a small sum of large terms.  The GPU tests therefore scale each element's
tolerance by the oracle's error scale of that element (gdn_oracle.c header), which the same
perturbation respects with a wide margin.
"""
import numpy as np
import torch

import oracle
from gated_deltanet_layer_02_b200 import inputs


def test_bf16_rounding_of_exact_output_breaks_max_abs_reading_only():
    w = inputs.custom(2, 4, 128, torch.bfloat16, lengths=(300,))
    inp = inputs.prefill_inputs(w, 800)
    ref, _, _ = oracle.prefill(oracle.Dims(2, 4), inp["x"], inp["beta"], inp["g"],
                               inp["cu_seqlens"], conv_w=inp["conv_w"], z=inp["z"],
                               norm_w=inp["norm_w"], want_state=False)
    rounded = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    rms = np.sqrt(np.mean(ref ** 2))
    max_abs_reading = np.max(np.abs(rounded - ref)) / rms
    rel_rms_reading = np.sqrt(np.mean((rounded - ref) ** 2)) / rms
    assert max_abs_reading > 2e-2          # the exact answer in bf16 "fails"
    assert rel_rms_reading < 2e-3          # and sits 10x inside the relative RMS bar
    assert np.max(np.abs(ref)) > 10 * rms  # because the normalised output is heavy-tailed


def test_bench_work_model_matches_the_closed_forms():
    # the per-kernel split of the algorithmic work adds up to F(C) and 33,024 B/token
    import bench
    w = inputs.CONFIGS[1]
    Hv, Hk, d = w.num_v_heads, w.num_k_heads, w.head_dim
    for C in (64, 128):
        f = bench.flops_per_token_by_kernel(w, C)
        total = sum(f.values())
        F = 2 * (Hv * (3 * d * d + 1.5 * C * d + C * C / 6) + Hk * C * d)
        assert abs(total - F) < 1e-6 * F
    assert abs(sum(bench.flops_per_token_by_kernel(w, 128).values()) - 5.4176e6) < 1e3
    b = bench.bytes_per_token_by_kernel(w)
    assert sum(b.values()) == 33024


def test_one_rounding_of_q_and_k_breaks_the_rms_element_bound_but_not_the_scaled_one():
    # conv off, so that x's q/k channels are the vectors the layer normalises; rounding the
    # normalised q and k to bf16 (what a bf16 tensor-core path feeds its products) is the
    # perturbation under test, applied to the exact oracle
    w = inputs.custom(2, 4, 128, torch.float32, lengths=(300,), conv=False)
    inp = inputs.prefill_inputs(w, 801)
    dims = oracle.Dims(2, 4)
    x = inp["x"].double().numpy()
    Hk, d = 2, 128
    qk = x[:, :2 * Hk * d].reshape(300, 2 * Hk, d)
    qk = qk / np.linalg.norm(qk, axis=-1, keepdims=True)
    xr = x.copy()
    xr[:, :2 * Hk * d] = torch.from_numpy(qk).to(torch.bfloat16).double().numpy().reshape(300, -1)
    args = dict(z=inp["z"].double(), norm_w=inp["norm_w"].double())
    ref, _, _, scale, _ = oracle.prefill(dims, torch.from_numpy(x), inp["beta"], inp["g"],
                                         inp["cu_seqlens"], with_scales=True, **args)
    pert, _, _ = oracle.prefill(dims, torch.from_numpy(xr), inp["beta"], inp["g"],
                                inp["cu_seqlens"], **args)
    err = np.abs(pert - ref)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(err / (2e-2 * rms + 2 ** -8 * np.abs(ref))) > 1.0   # the RMS element bound fails
    assert np.sqrt(np.mean(err ** 2)) / rms < 2e-2                     # the RMS bar holds
    assert np.max(err / (2e-2 * scale + 2 ** -8 * np.abs(ref))) < 0.5  # the scaled bound holds
