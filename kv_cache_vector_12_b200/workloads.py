"""Seeded synthetic workloads (shapes, value distributions, length mixes).

This module only draws inputs; it holds none of the method's arithmetic, so
both the CUDA path and the CPU oracle may consume what it produces.  Every
tensor comes from a seeded ``torch.Generator`` on the requested device (the
CUDA generator for the large shapes, so full-size inputs never cross PCIe);
the same call with the same seed and device returns the same values.

The five workloads are the ones the method is measured on:

* ``tiny``      1 KV head, 1 query head, d=128, 1024 tokens; K, V, q iid N(0,1)
                fp32 (rounded to bf16 where they enter the library); 3/3 bits.
* ``llama8b``   Llama-3-8B-shaped layer: 8 KV / 32 query heads, 32768 cached
                tokens, batch 1; x ~ N(0, I) times a LogNormal(0, 0.5) norm
                factor per (token, head); turbo3 for K and V; 64 decode steps
                that each append one token.
* ``qwen``      4 KV / 28 query heads, 16384 tokens; K norms U[172, 778],
                V norms U[2, 4], directions uniform on the sphere; q uniform
                on the unit sphere.
* ``llama70b``  8 KV / 64 query heads, 131072 tokens, batch 4; N(0,1) with
                round(1% of the 8*128 (head, channel) pairs) = 10 seeded pairs
                scaled by 20 in both K and V.
* ``serving``   32 sequences with lengths uniform on {1024, ..., 65536},
                8 KV / 32 query heads, N(0,1); 256 steps of append + decode.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    name: str
    n_seqs: int
    n_kv_heads: int
    n_q_heads: int
    seq_len: int                     # cached tokens (upper bound for ragged mixes)
    bits_k: int = 3
    bits_v: int = 3
    qjl: bool = False
    decode_steps: int = 1
    d: int = HEAD_DIM
    seed: int = 0
    pi_seed: int = 42
    settings: tuple = field(default_factory=tuple)   # extra (bits_k, bits_v, qjl) settings

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 1024, 3, 3, False, 1, seed=1001),
    "llama8b": Workload("llama8b", 1, 8, 32, 32768, 3, 3, False, 64, seed=1002),
    "qwen": Workload("qwen", 1, 4, 28, 16384, 4, 4, False, 1, seed=1003,
                     settings=((4, 2, False), (4, 4, False), (2, 2, True), (2, 4, True))),
    "llama70b": Workload("llama70b", 4, 8, 64, 131072, 3, 3, False, 1, seed=1004),
    "serving": Workload("serving", 32, 8, 32, 65536, 3, 3, False, 256, seed=1005,
                        settings=((2, 2, False), (3, 3, False), (4, 4, False),
                                  (2, 2, True), (3, 3, True), (4, 4, True))),
}


def generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def gaussian(shape, gen, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def unit_directions(shape, gen, device):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def kv_tokens(w: Workload, n_tok: int, gen, device, dtype=torch.bfloat16, outlier_mask=None):
    """K and V rows for n_tok tokens of one sequence: two [n_tok, H_kv, d] tensors."""
    shape = (n_tok, w.n_kv_heads, w.d)
    if w.name == "llama8b":
        k = gaussian(shape, gen, device) * torch.exp(0.5 * gaussian(shape[:2] + (1,), gen, device))
        v = gaussian(shape, gen, device) * torch.exp(0.5 * gaussian(shape[:2] + (1,), gen, device))
    elif w.name == "qwen":
        kn = 172.0 + 606.0 * torch.rand(shape[:2] + (1,), generator=gen, device=device)
        vn = 2.0 + 2.0 * torch.rand(shape[:2] + (1,), generator=gen, device=device)
        k = kn * unit_directions(shape, gen, device)
        v = vn * unit_directions(shape, gen, device)
    else:
        k = gaussian(shape, gen, device)
        v = gaussian(shape, gen, device)
        if outlier_mask is not None:
            k = k * outlier_mask
            v = v * outlier_mask
    return k.to(dtype), v.to(dtype)


def outlier_scale(w: Workload, device, seed: int):
    """[H_kv, d] multiplier: 1 everywhere except round(1% of H_kv*d) seeded
    (head, channel) pairs, which are 20."""
    n_pairs = round(0.01 * w.n_kv_heads * w.d)
    gen = generator("cpu", seed)
    flat = torch.randperm(w.n_kv_heads * w.d, generator=gen)[:n_pairs]
    m = torch.ones(w.n_kv_heads * w.d)
    m[flat] = 20.0
    return m.view(w.n_kv_heads, w.d).to(device)


def queries(w: Workload, n_seqs: int, gen, device, dtype=torch.bfloat16):
    """[n_seqs, H_q, d] query rows for one decode step."""
    shape = (n_seqs, w.n_q_heads, w.d)
    if w.name == "qwen":
        return unit_directions(shape, gen, device).to(dtype)
    return gaussian(shape, gen, device).to(dtype)


def serving_lengths(w: Workload, seed: int):
    """Sequence lengths uniform on {1024, ..., 65536} (host list)."""
    gen = generator("cpu", seed)
    return torch.randint(1024, 65536 + 1, (w.n_seqs,), generator=gen).tolist()
