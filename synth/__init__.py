"""Seeded synthetic inputs shared by the tests, the oracle checks and bench.py.

This module draws random numbers and casts them to bfloat16; it holds none of
the attention arithmetic.  The pages measure on no dataset: "BERT" and "GPT-2"
in the page "FlashAttention: The GPU Memory Hack That Changed Everything"
(section "Speed Improvements") supply only sequence lengths, and its
"Try It Yourself" script draws ``torch.randn`` Q, K, V of shape
(batch, heads, seq_len, head_dim).  The workloads below follow that recipe.

Recipe (one CPU ``torch.Generator`` per workload, seed 1220 + workload index):
draw Q, K, V in that order as float32 standard normals of shape (B, H, N, d),
multiply Q and K by ``qk_std`` (3.0 for the peaked long-context workload, so
the scaled scores have standard deviation 9), then round to bfloat16
(round-to-nearest-even, torch's cast).  Both the CUDA path and the oracle
consume these exact bf16 tensors.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    qk_std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return 1220 + self.index

    @property
    def flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the path's FLOP convention)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    @property
    def algorithmic_bytes(self) -> int:
        """Q, K, V read once and O written once (bf16) plus the fp32 LSE."""
        elems = self.B * self.H * self.N * self.d
        return 4 * elems * 2 + self.B * self.H * self.N * 4

    def describe(self) -> str:
        return (f"{self.name}: B={self.B} H={self.H} N={self.N} d={self.d} "
                f"{'causal' if self.causal else 'non-causal'}")


WORKLOADS = [
    Workload(1, "toy_single_head", 1, 1, 256, 64, False),
    Workload(2, "bert_base_encoder", 8, 12, 512, 64, False),
    Workload(3, "gpt2_small_decoder", 8, 12, 1024, 64, True),
    Workload(4, "long_context_causal", 2, 32, 8192, 128, True),
    Workload(5, "very_long_peaked_causal", 1, 16, 32768, 128, True, qk_std=3.0),
]


# The sequence-length sweep of the "Try It Yourself" script on the page
# "FlashAttention: The GPU Memory Hack That Changed Everything": batch 1,
# 32 heads, head dim 128, causal, seq_len 512..8192 (the page uses fp16;
# this path computes in bf16).
SWEEP_SEQ_LENS = (512, 1024, 2048, 4096, 8192)


def sweep_workload(N: int) -> Workload:
    return Workload(100 + SWEEP_SEQ_LENS.index(N), f"seq_sweep_{N}", 1, 32, N, 128, True)


@dataclass(frozen=True)
class DecodeWorkload:
    """Few queries (the newest Nq positions) against Nk keys per (batch, head)."""
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def kv_bytes(self) -> int:
        return 2 * self.B * self.H * self.Nk * self.d * 2

    @property
    def algorithmic_bytes(self) -> int:
        """K and V read once, Q read and O written (bf16), LSE written (fp32)."""
        qo = 2 * self.B * self.H * self.Nq * self.d * 2
        return self.kv_bytes + qo + self.B * self.H * self.Nq * 4

    def describe(self) -> str:
        return (f"{self.name}: B={self.B} H={self.H} Nq={self.Nq} Nk={self.Nk} d={self.d} "
                f"{'causal' if self.causal else 'non-causal'}")


# Decode-shaped workload: one new token per sequence against a 32K context.
DECODE_WORKLOAD = DecodeWorkload("decode_32k", 16, 32, 1, 32768, 128, False, 1240)


def draw_decode_qkv(B: int, H: int, Nq: int, Nk: int, d: int, seed: int):
    """Seeded bf16 q (B, H, Nq, d) and k, v (B, H, Nk, d), same recipe as draw_qkv."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def workload(index_or_name) -> Workload:
    for w in WORKLOADS:
        if w.index == index_or_name or w.name == index_or_name:
            return w
    raise KeyError(index_or_name)


def draw_qkv(B: int, H: int, N: int, d: int, seed: int, qk_std: float = 1.0):
    """Seeded bf16 Q, K, V on the CPU, shape (B, H, N, d), contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_std != 1.0:
        q.mul_(qk_std)
        k.mul_(qk_std)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def workload_qkv(w: Workload):
    return draw_qkv(w.B, w.H, w.N, w.d, w.seed, w.qk_std)


def draw_dout(B: int, H: int, N: int, d: int, seed: int):
    """Seeded upstream gradient dO for the backward pass: standard normals of
    shape (B, H, N, d) from a generator seeded with ``seed + 5000`` (so it
    differs from the Q, K, V draw of the same seed), rounded to bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 5000)
    return torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# FP8 (E4M3) inputs for the FP8 forward.  Per-tensor scaling: a tensor x is
# stored as codes x8 = e4m3(x / s) with s = amax(|x|) / 448 (448 is the
# largest finite E4M3 value), rounded to nearest even by torch's
# float8_e4m3fn cast; its value is x8 * s.  Both the CUDA path and the
# oracle consume the same codes and scales.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor):
    """(uint8 codes, float scale) of a float32 tensor, per-tensor scale."""
    amax = float(x.abs().max())
    scale = amax / E4M3_MAX if amax > 0 else 1.0
    codes = (x / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale


def draw_qkv_fp8(B: int, H: int, N: int, d: int, seed: int, qk_std: float = 1.0):
    """Seeded FP8 Q, K, V: the float32 draws of draw_qkv (same generator and
    order), each quantized per tensor.  Returns ((q8, k8, v8), (sq, sk, sv))."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_std != 1.0:
        q.mul_(qk_std)
        k.mul_(qk_std)
    (q8, sq), (k8, sk), (v8, sv) = quantize_e4m3(q), quantize_e4m3(k), quantize_e4m3(v)
    return (q8, k8, v8), (sq, sk, sv)
