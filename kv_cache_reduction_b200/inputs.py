"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it draws random tensors, picks the
seeded full-head masks, describes the workload shapes, and converts bf16
tensors to the raw bit patterns the oracle reads.  The only transform it
applies is the per-head RMSNorm that the sliding-window workload asks for
*before* the attention kernel (eps 1e-6, unit weight), done once in float64
and rounded to bf16 so both sides see the same bf16 values.

Workloads (sizes from the Laguna-XS-2.1 geometry: 48 query heads, 8 KV
heads, window 512; DuoAttention sink 64 / recent 256; head_dim 128 assumed):

  decode_small   B=1, prompt 1024 then 16 one-token decode steps, full heads {0,3,5,6}
  decode_b32     B=32, one decode step at context 32768, 2 of 8 heads full (seeded)
  prefill_16k    B=1, prefill 16384 tokens, 2 of 8 heads full (seeded) + cache append
  sliding_32k    B=2, sliding-window prefill 32768 tokens, window 512, sink logits
  stack40        B=16, one decode step through 40 layers at context 131072
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

NUM_Q_HEADS = 48
NUM_KV_HEADS = 8
HEAD_DIM = 128
SINK = 64
RECENT = 256
WINDOW = 512


def seeded_full_mask(seed: int, n_full: int, num_kv_heads: int = NUM_KV_HEADS) -> Tuple[int, ...]:
    """A full/streaming head mask with exactly n_full full heads, drawn from a seed.

    Stands in for the trained ``full_attention_heads`` tensor, which is not
    available here.
    """
    chosen = np.random.default_rng(seed).choice(num_kv_heads, n_full, replace=False)
    mask = [0] * num_kv_heads
    for g in chosen:
        mask[int(g)] = 1
    return tuple(mask)


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) values rounded to bf16, from a seeded generator on `device`."""
    g = generator(seed, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def randn_bf16_into(out: torch.Tensor, seed: int, chunk_elems: int = 1 << 28) -> torch.Tensor:
    """Fills a large bf16 tensor with seeded N(0,1) values, chunk by chunk.

    Each chunk gets its own generator seeded from (seed, chunk index), so the
    fp32 temporary stays small however large the tensor is.
    """
    flat = out.view(-1)
    n = flat.numel()
    for c, start in enumerate(range(0, n, chunk_elems)):
        stop = min(n, start + chunk_elems)
        g = generator(seed * 1_000_003 + c, out.device)
        tmp = torch.randn((stop - start,), generator=g, device=out.device, dtype=torch.float32)
        flat[start:stop].copy_(tmp)
    return out


def randn_f32(shape, seed: int, device="cpu") -> torch.Tensor:
    g = generator(seed, device)
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)


def rmsnorm_bf16(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """Per-head RMSNorm with unit weight, in float64, rounded to bf16 (input prep)."""
    xd = x.to(torch.float64)
    y = xd * torch.rsqrt(xd.pow(2).mean(dim=-1, keepdim=True) + eps)
    return y.to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


@dataclass
class Workload:
    """Sizes, head layout and seeds of one synthetic workload."""
    name: str
    batch: int
    seq_len: int                      # prompt length (prefill) or context (decode)
    kind: str                         # "prefill", "decode", "prefill+decode", "stack"
    full_mask: Tuple[int, ...] = (0,) * NUM_KV_HEADS
    window: int = 0
    sink_logit: bool = False
    rmsnorm: bool = False
    decode_steps: int = 0
    layers: int = 1
    full_layers: Sequence[int] = field(default_factory=tuple)
    seed: int = 0
    mask_seed: int = 0
    random_ring_head: bool = False


def workload(name: str) -> Workload:
    if name == "decode_small":
        return Workload(name, 1, 1024, "prefill+decode", full_mask=(1, 0, 0, 1, 0, 1, 1, 0),
                        decode_steps=16, seed=1001)
    if name == "decode_b32":
        return Workload(name, 32, 32768, "decode", full_mask=seeded_full_mask(2002, 2),
                        seed=1002, mask_seed=2002, random_ring_head=True)
    if name == "prefill_16k":
        return Workload(name, 1, 16384, "prefill", full_mask=seeded_full_mask(2003, 2),
                        seed=1003, mask_seed=2003)
    if name == "sliding_32k":
        return Workload(name, 2, 32768, "prefill", window=WINDOW, sink_logit=True,
                        rmsnorm=True, seed=1004)
    if name == "stack40":
        return Workload(name, 16, 131072, "stack", layers=40,
                        full_layers=tuple(range(3, 40, 4)), sink_logit=True, seed=1005,
                        mask_seed=2005)
    raise KeyError(name)


def stack_layer_masks(w: Workload) -> List[Optional[Tuple[int, ...]]]:
    """Per layer of the 40-layer stack: a seeded 2-of-8 mask for a full-attention
    layer, None for a sliding-window layer."""
    return [seeded_full_mask(w.mask_seed + layer, 2) if layer in w.full_layers else None
            for layer in range(w.layers)]


WORKLOADS = ("decode_small", "decode_b32", "prefill_16k", "sliding_32k", "stack40")
