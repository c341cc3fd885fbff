"""Seeded synthetic workloads for the SeerAttention prefill path.

This module only draws random numbers; it holds none of the method's
arithmetic.  The CUDA path and the fp64 oracle both consume what it returns
(the same bf16 bit patterns), so it is the single point where inputs are made.

Recipe (one CPU ``torch.Generator`` per workload, seed = 20250 + workload
number; every tensor drawn in fp32 then rounded to bf16 with
round-to-nearest-even):

1. Q ~ N(0, 1)                                   [B, Hq,  S, d]
2. K ~ N(0, 1)                                   [B, Hkv, S, d]
3. V ~ N(0, 1)                                   [B, Hkv, S, d]
4. block bias ~ N(0, 0.5^2) per (b, kv-head, key block, channel), added to
   every token of that key block of K ("some blocks dominate"); then the
   whole of key block 0 is multiplied by 3 (an attention sink).  Skipped for
   the tiny workload.
5. W_q ~ U(+-sqrt(6/(d+dg)))  [Hq, d, dg]; W_k likewise [Hkv, d, dg]
   (Xavier-uniform, random init: no trained AttnGate weights exist here).
6. tiny workload only: a causal block mask with the diagonal forced on and
   every strictly-lower block kept with probability 0.5.

The shapes follow the pages' models: a Llama-3.1-8B attention layer (32
query heads, 8 KV heads, head dim 128) and a Qwen2.5-14B layer (40/8, 128).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

BLOCK = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    number: int
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    d: int
    d_gate: int = 128
    rope_theta: float = 5e5
    block_bias: bool = True
    mask_source: str = "gate"          # "bernoulli" | "gate-threshold" | "gate-topk" | "dense-map"
    threshold: float | None = None
    densities: tuple = ()
    target_density: float | None = None

    @property
    def nb(self) -> int:
        return -(-self.S // BLOCK)      # the last block is partial when S % 64 != 0

    @property
    def seed(self) -> int:
        return 20250 + self.number


WORKLOADS = {
    "tiny": Workload(1, "tiny", 1, 2, 2, 512, 64, d_gate=64, block_bias=False,
                     mask_source="bernoulli"),
    "llama8b_8k": Workload(2, "llama8b_8k", 1, 32, 8, 8192, 128,
                           mask_source="gate-threshold", threshold=2e-3, target_density=0.7),
    "llama8b_32k": Workload(3, "llama8b_32k", 1, 32, 8, 32768, 128,
                            mask_source="gate-topk", densities=(1.0, 0.5, 0.3, 0.2, 0.1)),
    "llama8b_128k": Workload(4, "llama8b_128k", 1, 32, 8, 131072, 128,
                             mask_source="gate-threshold", target_density=0.17),
    "qwen14b_64k_map": Workload(5, "qwen14b_64k_map", 1, 40, 8, 65536, 128,
                                mask_source="dense-map"),
}


def custom(name: str, B: int, Hq: int, Hkv: int, S: int, d: int, number: int = 100,
           block_bias: bool = True, d_gate: int = 128, rope_theta: float = 5e5) -> Workload:
    """A workload of arbitrary shape with the same recipe (for tests)."""
    return Workload(number, name, B, Hq, Hkv, S, d, d_gate=d_gate, rope_theta=rope_theta,
                    block_bias=block_bias, mask_source="custom")


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bit patterns of a bf16 CPU tensor as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw Q, K, V, W_q, W_k (bf16, CPU) and, for the tiny workload, a mask."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    q = torch.randn((w.B, w.Hq, w.S, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.Hkv, w.S, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.Hkv, w.S, w.d), generator=g, dtype=torch.float32)
    if w.block_bias:
        bias = torch.randn((w.B, w.Hkv, w.nb, 1, w.d), generator=g, dtype=torch.float32) * 0.5
        k = k + bias[:, :, :, 0].repeat_interleave(BLOCK, dim=2)[:, :, : w.S]
        k[:, :, :BLOCK, :] *= 3.0
    bound = math.sqrt(6.0 / (w.d + w.d_gate))
    wq = (torch.rand((w.Hq, w.d, w.d_gate), generator=g, dtype=torch.float32) * 2 - 1) * bound
    wk = (torch.rand((w.Hkv, w.d, w.d_gate), generator=g, dtype=torch.float32) * 2 - 1) * bound
    out = {"q": _bf16(q), "k": _bf16(k), "v": _bf16(v), "wq": _bf16(wq), "wk": _bf16(wk)}
    del q, k, v
    if w.mask_source == "bernoulli":
        keep = torch.rand((w.B, w.Hq, w.nb, w.nb), generator=g) < 0.5
        lower = torch.ones(w.nb, w.nb, dtype=torch.bool).tril(-1)
        m = (keep & lower) | torch.eye(w.nb, dtype=torch.bool)
        out["mask"] = m.to(torch.uint8)
    return out


def random_mask(B: int, Hq: int, nb: int, p: float, seed: int, force_first: bool = True,
                force_diag: bool = True) -> torch.Tensor:
    """A seeded causal Bernoulli(p) block mask (u8 [B,Hq,nb,nb]) for tests."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    keep = torch.rand((B, Hq, nb, nb), generator=g) < p
    m = keep & torch.ones(nb, nb, dtype=torch.bool).tril()
    if force_first:
        m[..., 0] = True
    if force_diag:
        m |= torch.eye(nb, dtype=torch.bool)
    return m.to(torch.uint8)
