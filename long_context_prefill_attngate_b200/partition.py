"""Split of one attention layer across ranks by KV-head group.

The gate, the mask and the attention are computed per head ("Learning
Intrinsic Sparse Attention in Your LLMs", rebuttal Weakness 2: the AttnGate
scores and the TopK selection are per head), and every query head reads only
its own KV head.  A layer therefore partitions over KV heads: rank r of N
takes KV heads [r Hkv/N, (r+1) Hkv/N) together with the query heads that read
them, [r Hq/N, (r+1) Hq/N), and its slice of the layer is an independent
smaller layer.  No exchange is needed during the computation; the outputs
concatenate along the head axis.  This module only computes index ranges and
slices tensors (host logic, no arithmetic of the method).
"""
from __future__ import annotations


def head_range(Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int, int, int]:
    """(q-head begin, end, kv-head begin, end) owned by `rank` of `world`.

    Requires Hkv % world == 0 (whole GQA groups per rank); raises ValueError
    otherwise, and for a rank outside [0, world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if Hq % Hkv != 0:
        raise ValueError(f"Hq ({Hq}) must be a multiple of Hkv ({Hkv})")
    if Hkv % world != 0:
        raise ValueError(f"{Hkv} KV heads do not split evenly over {world} ranks")
    g = Hq // Hkv
    per = Hkv // world
    return rank * per * g, (rank + 1) * per * g, rank * per, (rank + 1) * per


def slice_layer(x: dict, Hq: int, Hkv: int, world: int, rank: int) -> dict:
    """This rank's slice of a layer's tensors (q, k, v: [B, H, S, d]; wq: [Hq, ...];
    wk: [Hkv, ...]; mask: [B, Hq, nb, nb] when present), as contiguous copies."""
    q0, q1, k0, k1 = head_range(Hq, Hkv, world, rank)
    out = {}
    for name, t in x.items():
        if name in ("q", "mask"):
            out[name] = t[:, q0:q1].contiguous()
        elif name in ("k", "v"):
            out[name] = t[:, k0:k1].contiguous()
        elif name == "wq":
            out[name] = t[q0:q1].contiguous()
        elif name == "wk":
            out[name] = t[k0:k1].contiguous()
        else:
            out[name] = t
    return out
