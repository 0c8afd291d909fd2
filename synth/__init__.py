"""Seeded synthetic inputs for the hybrid sparse attention forward.

This module only draws random tensors of the right shapes and distributions; it
holds none of the method's arithmetic.  It is the one piece of code that both
the CPU oracle's tests and the CUDA path's tests/benchmark use.

Distributions (the pages publish no data; these stand in for their long-context
prefill and decode workloads):
  * Q, K, V       : N(0, 1) * sigma, rounded to bf16 (sigma = 1/sqrt(d) for
                    prefill, 1 for the decode caches), drawn with torch's
                    seeded generator.
  * w (compressor): U(0, 2/blk) fp32.
  * q_idx, k_idx  : integers uniform on [-8, 8], int8.
  * w_idx         : integers uniform on [1, 4], int32.
Each tensor has its own stream: generator seed = base seed * 1000 + tensor id.
CPU generation is bit-reproducible and is what parity tests use; the benchmark
may draw the same distributions directly on the GPU (different values, same
law), which is stated in its output.
"""
from __future__ import annotations

import dataclasses
import math

import torch

SEED = 20261105

# tensor ids: one independent stream per tensor
TID = {"Q": 1, "K": 2, "V": 3, "w": 4, "q_idx": 5, "k_idx": 6, "w_idx": 7}


def _gen(seed: int, tensor: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + TID[tensor])
    return g


def normal_bf16(shape, sigma: float, seed: int, tensor: str, device="cpu") -> torch.Tensor:
    g = _gen(seed, tensor, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def uniform_f32(shape, lo: float, hi: float, seed: int, tensor: str, device="cpu") -> torch.Tensor:
    g = _gen(seed, tensor, device)
    x = torch.rand(*shape, generator=g, device=device, dtype=torch.float32)
    return x.mul_(hi - lo).add_(lo)


def randint(shape, lo: int, hi: int, seed: int, tensor: str, dtype, device="cpu") -> torch.Tensor:
    """Integers uniform on the closed range [lo, hi]."""
    g = _gen(seed, tensor, device)
    return torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device, dtype=torch.int64).to(dtype)


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class HcaConfig:
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    d: int = 512
    blk: int = 128
    W: int = 128
    sigma: float | None = None  # None -> 1/sqrt(d)

    @property
    def n_c(self) -> int:
        return self.L // self.blk


@dataclasses.dataclass(frozen=True)
class DsaConfig:
    name: str
    B: int
    L: int
    Hq: int
    d: int = 256
    H_idx: int = 4
    d_idx: int = 64
    k: int = 2048
    sigma: float | None = None


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    t: int                 # absolute position of the single query token
    hca_Hq: int = 16
    hca_d: int = 512
    blk: int = 128
    W: int = 128
    dsa_Hq: int = 64
    dsa_d: int = 256
    H_idx: int = 4
    d_idx: int = 64
    k: int = 2048

    @property
    def n_c(self) -> int:
        return (self.t + 1) // self.blk


HCA_TINY = HcaConfig("hca_tiny_L2048_h4_d512", B=1, L=2048, Hq=4, Hkv=4)
HCA_32K = HcaConfig("hca_prefill_L32768_hq16_hkv1_d512", B=1, L=32768, Hq=16, Hkv=1)
HCA_131K = HcaConfig("hca_prefill_L131072_hq16_hkv1_d512", B=1, L=131072, Hq=16, Hkv=1)
DSA_32K = DsaConfig("dsa_prefill_L32768_h64_d256_k2048", B=1, L=32768, Hq=64)
DECODE_1M = DecodeConfig("decode_B32_t1048575", B=32, t=1048575)

CONFIGS = {c.name: c for c in (HCA_TINY, HCA_32K, HCA_131K, DSA_32K, DECODE_1M)}


def sigma_of(cfg, d):
    return cfg.sigma if getattr(cfg, "sigma", None) is not None else 1.0 / math.sqrt(d)


def hca_inputs(cfg: HcaConfig, seed: int = SEED, device="cpu") -> dict:
    """K, V [B, L, Hkv, d]; Q [B, L, Hq, d]; w [blk]."""
    s = sigma_of(cfg, cfg.d)
    return {
        "Q": normal_bf16((cfg.B, cfg.L, cfg.Hq, cfg.d), s, seed, "Q", device),
        "K": normal_bf16((cfg.B, cfg.L, cfg.Hkv, cfg.d), s, seed, "K", device),
        "V": normal_bf16((cfg.B, cfg.L, cfg.Hkv, cfg.d), s, seed, "V", device),
        "w": uniform_f32((cfg.blk,), 0.0, 2.0 / cfg.blk, seed, "w", device),
    }


def dsa_inputs(cfg: DsaConfig, seed: int = SEED, device="cpu") -> dict:
    """Q [B, L, Hq, d]; K, V [B, L, d] (one shared head); q_idx [B, L, H_idx, d_idx];
    k_idx [B, L, d_idx]; w_idx [H_idx]."""
    s = sigma_of(cfg, cfg.d)
    return {
        "Q": normal_bf16((cfg.B, cfg.L, cfg.Hq, cfg.d), s, seed, "Q", device),
        "K": normal_bf16((cfg.B, cfg.L, cfg.d), s, seed, "K", device),
        "V": normal_bf16((cfg.B, cfg.L, cfg.d), s, seed, "V", device),
        "q_idx": randint((cfg.B, cfg.L, cfg.H_idx, cfg.d_idx), -8, 8, seed, "q_idx", torch.int8, device),
        "k_idx": randint((cfg.B, cfg.L, cfg.d_idx), -8, 8, seed, "k_idx", torch.int8, device),
        "w_idx": randint((cfg.H_idx,), 1, 4, seed, "w_idx", torch.int32, device),
    }
