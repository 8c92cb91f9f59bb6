"""Seeded synthetic inputs for the Gated DeltaNet layer.

This module is shared by the tests, the benchmark and the oracle side.  It holds only the
workload definitions and random-number draws -- none of the layer's arithmetic.

Shapes follow the "Qwen3-Coder-Next" model card (llm-atlas), raw config.json fields:
16 key heads, 32 value heads, head dim 128, conv width 4, rms_norm_eps 1e-6, bf16 weights.
No dataset is involved: every tensor is drawn from the distributions listed in ``CONFIGS``.

Seeding: configuration k uses ``numpy.random.SeedSequence(1000 + k)`` spawned into one child
stream per tensor in the fixed order (x, z, beta, g, conv_w, S0, conv0); large tensors are
drawn in blocks of ``ROW_BLOCK`` tokens so that a shorter sample is a prefix of a longer one.
The variable-length configuration draws its sequence lengths first, from
``numpy.random.default_rng(1002).integers(512, 8193, 8)``.  Values are drawn in fp32/fp64,
then rounded once to the activation dtype (bf16: round to nearest even); the rounded tensor is
what both the CUDA path and the oracle receive.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

ROW_BLOCK = 64

#: tensor order of the child streams
_STREAMS = ("x", "z", "beta", "g", "conv_w", "S0", "conv0")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                  # "prefill" or "decode"
    num_k_heads: int
    num_v_heads: int
    head_dim: int
    dtype: torch.dtype         # activation dtype (state is always fp32)
    lengths: tuple = ()        # prefill: sequence lengths
    conv: bool = True          # conv1d + SiLU on
    norm: bool = True          # z-gated RMSNorm on
    g_dist: str = "cfg1"       # "cfg1" | "uniform"
    g_low: float = 0.0         # for g_dist == "uniform": g ~ U(g_low, 0)
    s0_std: float = 0.0        # initial state ~ N(0, s0_std); 0 = zero state
    batch: int = 0             # decode: sequences per step
    steps: int = 0             # decode: number of steps
    conv_state_std: float = 1.0
    conv_kernel: int = 4

    @property
    def channels(self) -> int:
        return (2 * self.num_k_heads + self.num_v_heads) * self.head_dim

    @property
    def tokens(self) -> int:
        return int(sum(self.lengths))


def _varlen_lengths() -> tuple:
    return tuple(int(v) for v in np.random.default_rng(1002).integers(512, 8193, 8))


CONFIGS = [
    Workload("tiny_f32_T128_hk2_hv4", "prefill", 2, 4, 128, torch.float32, lengths=(128,),
             conv=False, norm=False, g_dist="uniform", g_low=-0.5),
    Workload("prefill_T4096_hk16_hv32", "prefill", 16, 32, 128, torch.bfloat16, lengths=(4096,)),
    Workload("varlen_8seq_hk16_hv32", "prefill", 16, 32, 128, torch.bfloat16,
             lengths=_varlen_lengths(), s0_std=0.1),
    Workload("decode_B256_hk16_hv32_64steps", "decode", 16, 32, 128, torch.bfloat16, batch=256,
             steps=64, s0_std=0.1),
    Workload("prefill_T262144_hk16_hv32", "prefill", 16, 32, 128, torch.bfloat16,
             lengths=(262144,), g_dist="uniform", g_low=-0.05),
]


def _children(seed: int):
    return dict(zip(_STREAMS, np.random.SeedSequence(seed).spawn(len(_STREAMS))))


def _normal_rows(ss, rows: int, cols: int, std: float, dtype: torch.dtype) -> torch.Tensor:
    """rows x cols of N(0, std) drawn in ROW_BLOCK-row blocks, rounded once to dtype."""
    rng = np.random.default_rng(ss)
    out = torch.empty((rows, cols), dtype=dtype)
    for r0 in range(0, rows, ROW_BLOCK):
        r1 = min(rows, r0 + ROW_BLOCK)
        blk = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            blk *= np.float32(std)
        out[r0:r1] = torch.from_numpy(blk).to(dtype)
    return out


def _sigmoid(a):
    return 1.0 / (1.0 + np.exp(-a))


def _softplus(a):
    return np.log1p(np.exp(-np.abs(a))) + np.maximum(a, 0.0)


def _gates(ss_beta, ss_g, rows: int, hv: int, g_dist: str, g_low: float):
    """beta = sigmoid(N(0,1)); g = log alpha per the workload; both fp32 [rows, hv]."""
    rb = np.random.default_rng(ss_beta)
    rg = np.random.default_rng(ss_g)
    beta = np.empty((rows, hv), np.float32)
    g = np.empty((rows, hv), np.float32)
    for r0 in range(0, rows, ROW_BLOCK):
        r1 = min(rows, r0 + ROW_BLOCK)
        beta[r0:r1] = _sigmoid(rb.standard_normal((r1 - r0, hv)))
        if g_dist == "uniform":
            g[r0:r1] = rg.uniform(g_low, 0.0, (r1 - r0, hv))
        else:
            a = rg.standard_normal((r1 - r0, hv)) * 0.5
            b = rg.standard_normal((r1 - r0, hv))
            g[r0:r1] = -np.exp(a) * _softplus(b)
    return torch.from_numpy(beta), torch.from_numpy(g)


def cu_seqlens_of(lengths) -> torch.Tensor:
    cu = np.zeros(len(lengths) + 1, np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, np.int64))
    return torch.from_numpy(cu.astype(np.int32))


def prefill_inputs(w: Workload, seed: int, lengths=None, with_conv0: bool = False) -> dict:
    """Inputs of one prefill call on CPU: x, conv_w, beta, g, z, norm_w, cu_seqlens, S0, conv0.

    ``lengths`` overrides the workload's sequence lengths (e.g. a bounded sample).
    Tensors the workload switches off are None.
    """
    lengths = tuple(int(v) for v in (w.lengths if lengths is None else lengths))
    T, N = int(sum(lengths)), len(lengths)
    ch = _children(seed)
    Hv, d, K = w.num_v_heads, w.head_dim, w.conv_kernel
    x = _normal_rows(ch["x"], T, w.channels, 1.0, w.dtype)
    z = _normal_rows(ch["z"], T, Hv * d, 1.0, w.dtype).view(T, Hv, d) if w.norm else None
    beta, g = _gates(ch["beta"], ch["g"], T, Hv, w.g_dist, w.g_low)
    conv_w = _normal_rows(ch["conv_w"], w.channels, K, 0.5, w.dtype) if w.conv else None
    norm_w = torch.ones(d, dtype=w.dtype) if w.norm else None
    S0 = (_normal_rows(ch["S0"], N * Hv * d, d, w.s0_std, torch.float32).view(N, Hv, d, d)
          if w.s0_std > 0 else None)
    conv0 = (_normal_rows(ch["conv0"], N * (K - 1), w.channels, 1.0, w.dtype).view(N, K - 1, w.channels)
             if with_conv0 else None)
    return dict(x=x, conv_w=conv_w, beta=beta, g=g, z=z, norm_w=norm_w,
                cu_seqlens=cu_seqlens_of(lengths), S0=S0, conv0=conv0)


def decode_state(w: Workload, seed: int) -> dict:
    """Initial decode state on CPU: S [B, Hv, d, d] fp32, conv_state [B, K-1, Cc], conv_w, norm_w."""
    ch = _children(seed)
    B, Hv, d, K = w.batch, w.num_v_heads, w.head_dim, w.conv_kernel
    S = _normal_rows(ch["S0"], B * Hv * d, d, w.s0_std, torch.float32).view(B, Hv, d, d)
    conv_state = _normal_rows(ch["conv0"], B * (K - 1), w.channels, w.conv_state_std,
                              w.dtype).view(B, K - 1, w.channels)
    conv_w = _normal_rows(ch["conv_w"], w.channels, K, 0.5, w.dtype)
    norm_w = torch.ones(d, dtype=w.dtype) if w.norm else None
    return dict(S=S, conv_state=conv_state, conv_w=conv_w, norm_w=norm_w)


def decode_step_inputs(w: Workload, seed: int, step: int) -> dict:
    """Fresh per-step decode inputs on CPU: x [B, Cc], z [B, Hv, d], beta, g [B, Hv]."""
    ch = _children(seed * 1000003 + step + 1)
    B, Hv, d = w.batch, w.num_v_heads, w.head_dim
    x = _normal_rows(ch["x"], B, w.channels, 1.0, w.dtype)
    z = _normal_rows(ch["z"], B, Hv * d, 1.0, w.dtype).view(B, Hv, d) if w.norm else None
    beta, g = _gates(ch["beta"], ch["g"], B, Hv, w.g_dist, w.g_low)
    return dict(x=x, z=z, beta=beta, g=g)


def block_inputs(w: Workload, seed: int, hidden: int, with_conv0: bool = False) -> dict:
    """Inputs of one token-mixer (projections + layer) call on CPU, bf16 unless stated:
    h [T, H] ~ N(0, 1); projection weights [in, out] ~ N(0, 1/in), so that x, z, b and a come
    out near unit variance; A_log ~ N(0, 0.5), dt_bias ~ N(0, 1) (fp32 [Hv]); conv_w ~
    N(0, 0.5); norm_w = 1; S0 ~ N(0, s0_std) when s0_std > 0."""
    lengths = tuple(int(v) for v in w.lengths)
    T, N = int(sum(lengths)), len(lengths)
    Hv, d, K, H, Cc = w.num_v_heads, w.head_dim, w.conv_kernel, hidden, w.channels
    ss = np.random.SeedSequence(seed).spawn(10)
    h = _normal_rows(ss[0], T, H, 1.0, w.dtype)
    w_qkv = _normal_rows(ss[1], H, Cc, H ** -0.5, w.dtype)
    w_z = _normal_rows(ss[2], H, Hv * d, H ** -0.5, w.dtype)
    w_ba = _normal_rows(ss[3], H, 2 * Hv, H ** -0.5, w.dtype)
    w_out = _normal_rows(ss[4], Hv * d, H, (Hv * d) ** -0.5, w.dtype)
    small = np.random.default_rng(ss[5])
    a_log = torch.from_numpy(small.normal(0.0, 0.5, Hv).astype(np.float32))
    dt_bias = torch.from_numpy(small.normal(0.0, 1.0, Hv).astype(np.float32))
    conv_w = _normal_rows(ss[6], Cc, K, 0.5, w.dtype)
    S0 = (_normal_rows(ss[7], N * Hv * d, d, w.s0_std, torch.float32).view(N, Hv, d, d)
          if w.s0_std > 0 else None)
    conv0 = (_normal_rows(ss[8], N * (K - 1), Cc, 1.0, w.dtype).view(N, K - 1, Cc)
             if with_conv0 else None)
    return dict(h=h, w_qkv=w_qkv, w_z=w_z, w_ba=w_ba, a_log=a_log, dt_bias=dt_bias, w_out=w_out,
                conv_w=conv_w, norm_w=torch.ones(d, dtype=w.dtype),
                cu_seqlens=cu_seqlens_of(lengths), S0=S0, conv0=conv0)


def config_seed(idx: int) -> int:
    return 1000 + idx


def custom(num_k_heads=2, num_v_heads=4, head_dim=128, dtype=torch.bfloat16, lengths=(128,),
           conv=True, norm=True, g_dist="cfg1", g_low=0.0, s0_std=0.0) -> Workload:
    """A small workload for tests, with the same distributions as the named configurations."""
    return Workload("custom", "prefill", num_k_heads, num_v_heads, head_dim, dtype,
                    lengths=tuple(lengths), conv=conv, norm=norm, g_dist=g_dist, g_low=g_low,
                    s0_std=s0_std)


__all__ = ["CONFIGS", "Workload", "prefill_inputs", "decode_state", "decode_step_inputs",
           "config_seed", "custom", "cu_seqlens_of", "block_inputs"]
