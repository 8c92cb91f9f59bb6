"""Why the bf16 parity bar is the relative RMS error (CPU only).

The workload statement asks for agreement "within 2e-2 relative-to-RMS" for bf16 activations.
Read as max|gpu - oracle| / rms(oracle), the bar would reject even the exact result rounded once
to bf16, because the z-gated RMSNorm output is heavy-tailed (elements reach 10-15x its RMS and
bf16 keeps 8 significant bits).  Read as ||gpu - oracle||_2 / ||oracle||_2 it is met by that
rounding with a wide margin.  The tests use the second reading.
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
        total = sum(v for k, v in f.items() if k != "gdn_prep_chain")
        F = 2 * (Hv * (3 * d * d + 1.5 * C * d + C * C / 6) + Hk * C * d)
        assert abs(total - F) < 1e-6 * F
    assert abs(sum(v for k, v in bench.flops_per_token_by_kernel(w, 128).items()
                   if k != "gdn_prep_chain") - 5.4176e6) < 1e3
    b = bench.bytes_per_token_by_kernel(w)
    assert sum(v for k, v in b.items() if k != "gdn_prep_chain") == 33024
