"""Seeded synthetic inputs for SharQ linear layers.

This module only draws numbers; it holds none of the method's arithmetic, so
the CPU oracle's tests and the CUDA path's tests and benchmark can share it.

The pages evaluate on Llama-3.1-8B, Qwen2.5-7B, Qwen3-30B-A3B, Qwen3-VL-8B and
Wan2.2-T2V-A14B ("SharQ: Bridging Activation Sparsity and FP4 Quantization for
LLM Inference", Abstract) with wikitext2 / lm-eval suites (README, section
"Evaluation"). None of those weights or datasets exist here; these generators
stand in for them with the models' layer shapes and with activations that have
the property the abstract attributes to real ones: outliers, varying from input to
input, large enough to set the block scales -- here a few outlier channels scaled by
large factors, times a log-normal per-token scale.

Values are drawn in float32 with numpy's PCG64 (``default_rng(seed)``) and
rounded to bf16 (round to nearest even) by integer bit operations, so the
same bits go to the CPU oracle and to the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Linear:
    """One SharQ linear-layer problem: activations, optional RMSNorm weight, weight."""
    name: str
    x: np.ndarray            # uint16 bf16 bits [T, K]
    gamma: np.ndarray | None  # uint16 bf16 bits [K] or None (no fused RMSNorm)
    w: np.ndarray            # uint16 bf16 bits [N, K]
    eps: float = 1e-6

    @property
    def shape(self):
        T, K = self.x.shape
        return T, K, self.w.shape[0]


def outlier_activations(rng, T: int, K: int, n_outlier: int, scale_lo: float, scale_hi: float,
                        token_sigma: float) -> np.ndarray:
    """X = Z * (token_scale x channel_scale): Z ~ N(0,1); ``n_outlier`` channels
    scaled by U(scale_lo, scale_hi) (a fixed factor when lo == hi); token scale
    exp(N(0, token_sigma^2)) (1 when token_sigma == 0). Returns bf16 bits."""
    z = rng.standard_normal((T, K), dtype=np.float32)
    ch = np.ones(K, dtype=np.float32)
    idx = rng.choice(K, size=n_outlier, replace=False)
    ch[idx] = rng.uniform(scale_lo, scale_hi, size=n_outlier).astype(np.float32)
    tok = np.ones(T, dtype=np.float32)
    if token_sigma > 0:
        tok = np.exp(rng.normal(0.0, token_sigma, size=T)).astype(np.float32)
    return f32_to_bf16_bits(z * tok[:, None] * ch[None, :])


def swiglu_activations(rng, T: int, K: int) -> np.ndarray:
    """down_proj input: bf16(SiLU(g) * u) with g, u ~ N(0, 1) (heavy-tailed, no norm)."""
    g = rng.standard_normal((T, K), dtype=np.float32)
    u = rng.standard_normal((T, K), dtype=np.float32)
    silu = g / (np.float32(1.0) + np.exp(-g))
    return f32_to_bf16_bits(silu * u)


def gate_up_activations(rng, T: int, K: int) -> np.ndarray:
    """A gate/up projection's output [T, 2K] = [g | u] in bf16, g, u ~ N(0, 1) (the input of a
    down projection whose preparation fuses the gated activation)."""
    return f32_to_bf16_bits(rng.standard_normal((T, 2 * K), dtype=np.float32))


def rms_gamma(rng, K: int) -> np.ndarray:
    return f32_to_bf16_bits(rng.uniform(0.5, 1.5, size=K).astype(np.float32))


def weight(rng, N: int, K: int) -> np.ndarray:
    return f32_to_bf16_bits((rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)))


def tiny(seed: int = 0, T: int = 64) -> Linear:
    """X bf16 [64, 256] ~ N(0,1) with 4 fixed outlier channels x50; gamma ~ U(0.5,1.5);
    eps 1e-6; W bf16 [256, 256] ~ N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    K, N = 256, 256
    x = outlier_activations(rng, T, K, 4, 50.0, 50.0, 0.0)
    return Linear("tiny_64x256x256", x, rms_gamma(rng, K), weight(rng, N, K))


def llama_qkv(seed: int = 1, T: int = 2048) -> Linear:
    """Llama-3.1-8B QKV projection at prefill: X [T, 4096] with ~1% outlier channels
    x U(20,100) and a log-normal token scale (sigma 0.5), fused RMSNorm; W [6144, 4096]."""
    rng = np.random.default_rng(seed)
    K, N = 4096, 6144
    x = outlier_activations(rng, T, K, 41, 20.0, 100.0, 0.5)
    return Linear(f"llama31_8b_qkv_{T}x{K}x{N}", x, rms_gamma(rng, K), weight(rng, N, K))


def llama_gate_up(seed: int = 2, T: int = 4096) -> Linear:
    rng = np.random.default_rng(seed)
    K, N = 4096, 28672
    x = outlier_activations(rng, T, K, 41, 20.0, 100.0, 0.5)
    return Linear(f"llama31_8b_gate_up_{T}x{K}x{N}", x, rms_gamma(rng, K), weight(rng, N, K))


def llama_down(seed: int = 2, T: int = 4096) -> Linear:
    rng = np.random.default_rng(seed + 100)
    K, N = 14336, 4096
    return Linear(f"llama31_8b_down_{T}x{K}x{N}", swiglu_activations(rng, T, K), None, weight(rng, N, K))


def llama_down_gate_up(seed: int = 2, T: int = 2048) -> tuple[np.ndarray, np.ndarray]:
    """Llama-3.1-8B down projection fed by its gate/up output: ([T, 2*14336] bf16, W [4096, 14336])."""
    rng = np.random.default_rng(seed + 300)
    K, N = 14336, 4096
    return gate_up_activations(rng, T, K), weight(rng, N, K)


QWEN_LINEARS = {  # name: (K, N, fused RMSNorm)
    "qkv": (3584, 4608, True),
    "o": (3584, 3584, False),
    "gate_up": (3584, 37888, True),
    "down": (18944, 3584, False),
}


def qwen(which: str, T: int, seed: int = 3) -> Linear:
    """Qwen2.5-7B layer linears at T tokens (T in 1, 16, 128, 2048, 8192 in the sweep)."""
    K, N, norm = QWEN_LINEARS[which]
    rng = np.random.default_rng(seed)
    x = outlier_activations(rng, T, K, max(1, K // 100), 20.0, 100.0, 0.5)
    g = rms_gamma(rng, K) if norm else None
    return Linear(f"qwen25_7b_{which}_{T}x{K}x{N}", x, g, weight(rng, N, K))


def square(seed: int = 4, S: int = 8192) -> Linear:
    rng = np.random.default_rng(seed)
    x = outlier_activations(rng, S, S, S // 100, 20.0, 100.0, 0.5)
    return Linear(f"square_{S}", x, None, weight(rng, S, S))


def dit(seed: int = 4, T: int = 32760) -> Linear:
    """Video-DiT-like linear: M=32760, K=5120, N=5120 (Wan2.2-T2V-A14B width)."""
    rng = np.random.default_rng(seed)
    K, N = 5120, 5120
    x = outlier_activations(rng, T, K, K // 100, 20.0, 100.0, 0.5)
    return Linear(f"dit_{T}x{K}x{N}", x, None, weight(rng, N, K))


def moe_routing(seed: int, T: int, n_experts: int, top_k: int) -> np.ndarray:
    """Expert ids [T, top_k] of a mixture-of-experts router: the top_k of seeded N(0, 1)
    logits per token (distinct experts, token-major)."""
    rng = np.random.default_rng(seed + 500)
    logits = rng.standard_normal((T, n_experts), dtype=np.float32)
    return np.argsort(-logits, axis=1, kind="stable")[:, :top_k].astype(np.int64)


QWEN3_MOE = dict(hidden=2048, moe_intermediate=768, n_experts=128, top_k=8)  # Qwen3-30B-A3B expert layer


def crafted_row(values) -> np.ndarray:
    """bf16 bits of a hand-written row (for edge-case tests)."""
    return f32_to_bf16_bits(np.asarray(values, dtype=np.float32)[None, :])


def outlier_activations_device(seed: int, T: int, K: int, n_outlier: int, scale_lo: float, scale_hi: float,
                               token_sigma: float, device="cuda"):
    """The recipe of ``outlier_activations`` drawn on the device with torch's generator, for
    benchmark sizes whose host-side drawing would dominate the run (bf16 tensor [T, K]; the
    same distribution, not the same bits as the numpy stream)."""
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn(T, K, generator=g, device=device)
    ch = torch.ones(K, device=device)
    idx = torch.randperm(K, generator=g, device=device)[:n_outlier]
    ch[idx] = torch.empty(n_outlier, device=device).uniform_(scale_lo, scale_hi, generator=g)
    tok = torch.ones(T, device=device)
    if token_sigma > 0:
        tok = torch.exp(torch.randn(T, generator=g, device=device) * token_sigma)
    return (z * tok[:, None] * ch[None, :]).to(torch.bfloat16)


def swiglu_activations_device(seed: int, T: int, K: int, device="cuda"):
    """The recipe of ``swiglu_activations`` drawn on the device (bf16 tensor [T, K])."""
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    a = torch.randn(T, K, generator=g, device=device)
    u = torch.randn(T, K, generator=g, device=device)
    return (a / (1.0 + torch.exp(-a)) * u).to(torch.bfloat16)


def weight_device(seed: int, N: int, K: int, device="cuda"):
    """The recipe of ``weight`` drawn on the device (bf16 tensor [N, K], N(0, 0.02))."""
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(N, K, generator=g, device=device) * 0.02).to(torch.bfloat16)


def rms_gamma_device(seed: int, K: int, device="cuda"):
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.rand(K, generator=g, device=device) + 0.5).to(torch.bfloat16)
