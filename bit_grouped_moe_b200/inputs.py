"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws numbers and nothing else: it holds none of the method's
arithmetic (no quantiser, no decode, no routing sort, no GEMM).  Quantised
NF4 weights for parity tests are made by passing ``normal_weights`` through
the oracle's quantiser; the bench draws NF4 codes and block absmax values
directly (``nf4_direct``) so that the product path never runs oracle code.

The synthetic routing (``route_topk``) draws router logits and keeps each
token's k largest, which defines the workloads' expert-load distribution
(N(0,1) logits, optionally with a Zipf rank bias).  Its ids and weights are
inputs to the routing and combine steps on both sides alike.  The library's
router epilogue is never compared against it: its parity tests draw logits
here and compare the kernel with the oracle's own top-k.

Workload shapes follow the pages' models (OLMoE-1B-7B, Qwen3-30B-A3B,
gpt-oss-120b, a Kimi-class MoE); see ``WORKLOADS``.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def normal_weights(g: np.random.Generator, shape, std: float = 0.02) -> np.ndarray:
    """fp32 weights drawn N(0, std^2)."""
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def bf16_normal(g: np.random.Generator, shape) -> np.ndarray:
    """bf16 N(0,1) activations as raw uint16 bit patterns (fp32 draw rounded to bf16)."""
    x = torch.from_numpy(g.standard_normal(shape, dtype=np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 patterns -> fp32 values (bit placement only)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def mxfp4_random(g: np.random.Generator, E: int, N: int, K: int, e_lo: int = 118, e_hi: int = 130):
    """MXFP4 expert stack: every nibble uniform over the 16 e2m1 codes, every
    e8m0 scale byte uniform over [e_lo, e_hi] (inclusive)."""
    blocks = g.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = g.integers(e_lo, e_hi + 1, size=(E, N, K // 32), dtype=np.uint8)
    return blocks, scales


def nf4_direct(g: np.random.Generator, E: int, N: int, K: int, std: float = 0.02):
    """NF4 expert stack drawn directly (bench inputs): codes uniform over 16,
    absmax per 64-block = std * max|z| over 64 standard normal draws (the
    absmax a block of N(0, std^2) weights would carry)."""
    packed = g.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    nb = K // 64
    absmax = np.empty((E, N, nb), np.float32)
    # chunked so very large stacks do not need a [.., 64] temporary all at once
    flat = absmax.reshape(-1)
    step = 1 << 20
    for i in range(0, flat.size, step):
        n = min(step, flat.size - i)
        z = np.abs(g.standard_normal((n, 64), dtype=np.float32)).max(axis=1)
        flat[i:i + n] = z * np.float32(std)
    return packed, absmax


def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    return (p / p.sum(axis=1, keepdims=True)).astype(np.float32)


def route_uniform(g: np.random.Generator, T: int, k: int, E: int):
    """Each token picks k distinct experts uniformly at random; router weights
    are the softmax of k N(0,1) logits.  Returns (topk_ids [T,k] i32, w [T,k] f32)."""
    ids = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32) if T else np.zeros((0, k), np.int32)
    logits = g.standard_normal((T, k), dtype=np.float32)
    return ids, _softmax_rows(logits) if T else np.zeros((0, k), np.float32)


def route_topk(g: np.random.Generator, T: int, k: int, E: int, zipf_s: float | None = None):
    """Router logits N(0,1) [T,E], optionally plus a skew bias, then the k
    largest per token (distinct experts).  The skew bias ranks the experts by a
    seeded permutation and adds -s*ln(rank) to each expert's logit, so an
    expert's selection weight falls off as rank^-s (a Zipf(s) skew); with T in
    the thousands this leaves some experts with no rows.  Router weights are
    the softmax of the k selected raw logits."""
    logits = g.standard_normal((T, E), dtype=np.float32)
    score = logits
    if zipf_s is not None:
        rank = g.permutation(E).astype(np.float32) + 1.0
        score = logits + (-np.float32(zipf_s) * np.log(rank)).astype(np.float32)[None, :]
    ids = np.argsort(-score, axis=1, kind="stable")[:, :k].astype(np.int32)
    sel = np.take_along_axis(logits, ids, axis=1)
    return ids, _softmax_rows(sel)


@dataclass(frozen=True)
class Projection:
    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str  # "nf4" | "mxfp4"
    E: int
    k: int
    T: int
    projections: tuple
    routing: str  # "uniform" | "topk" | "zipf"
    zipf_s: float | None = None


WORKLOADS = {
    # Tiny NF4 case: the oracle finishes it in well under a second.
    "tiny-nf4": Workload("tiny-nf4", "nf4", E=8, k=2, T=16,
                         projections=(Projection("proj", 256, 512),), routing="uniform"),
    # NF4 decode, OLMoE-1B-7B shape (64 experts, hidden 2048, intermediate 1024).
    "olmoe-decode-t1": Workload("olmoe-decode-t1", "nf4", E=64, k=8, T=1,
                                projections=(Projection("gate_up", 2048, 2048), Projection("down", 1024, 2048)),
                                routing="topk"),
    "olmoe-decode-t8": Workload("olmoe-decode-t8", "nf4", E=64, k=8, T=8,
                                projections=(Projection("gate_up", 2048, 2048), Projection("down", 1024, 2048)),
                                routing="topk"),
    # NF4 prefill, Qwen3-30B-A3B shape (128 experts, hidden 2048, intermediate 768), Zipf(1.1) skew.
    "qwen3-30b-prefill": Workload("qwen3-30b-prefill", "nf4", E=128, k=8, T=2048,
                                  projections=(Projection("gate_up", 2048, 1536), Projection("down", 768, 2048)),
                                  routing="zipf", zipf_s=1.1),
    # MXFP4, gpt-oss-120b shape (128 experts, hidden 2880, intermediate 2880), top-4.
    "gptoss-t1": Workload("gptoss-t1", "mxfp4", E=128, k=4, T=1,
                          projections=(Projection("gate_up", 2880, 5760), Projection("down", 2880, 2880)),
                          routing="topk"),
    "gptoss-t64": Workload("gptoss-t64", "mxfp4", E=128, k=4, T=64,
                           projections=(Projection("gate_up", 2880, 5760), Projection("down", 2880, 2880)),
                           routing="topk"),
    "gptoss-t512": Workload("gptoss-t512", "mxfp4", E=128, k=4, T=512,
                            projections=(Projection("gate_up", 2880, 5760), Projection("down", 2880, 2880)),
                            routing="topk"),
    # MXFP4 large prefill, Kimi-class shape (384 experts, hidden 7168, intermediate 2048), Zipf(1.2) skew.
    "kimi-prefill": Workload("kimi-prefill", "mxfp4", E=384, k=8, T=4096,
                             projections=(Projection("gate_up", 7168, 4096), Projection("down", 2048, 7168)),
                             routing="zipf", zipf_s=1.2),
    # The same shapes scaled to 48 experts and 512 tokens (the same mean of 85
    # rows per expert, Zipf(1.2) skew): a device footprint of about 1 GB, for
    # profiler captures of the Kimi-class kernels.
    "kimi-prefill-e48": Workload("kimi-prefill-e48", "mxfp4", E=48, k=8, T=512,
                                 projections=(Projection("gate_up", 7168, 4096), Projection("down", 2048, 7168)),
                                 routing="zipf", zipf_s=1.2),
}


def routing_for(w: Workload, g: np.random.Generator, T: int | None = None):
    T = w.T if T is None else T
    if w.routing == "uniform":
        return route_uniform(g, T, w.k, w.E)
    if w.routing == "zipf":
        return route_topk(g, T, w.k, w.E, zipf_s=w.zipf_s)
    return route_topk(g, T, w.k, w.E)


def device_random_bytes(seed: int, shape, device="cuda", lo: int = 0, hi: int = 256):
    """uint8 tensor drawn uniformly in [lo, hi) directly on the device with a
    seeded torch generator (for expert stacks of several GB)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randint(lo, hi, tuple(shape), generator=gen, device=device, dtype=torch.int16).to(torch.uint8)


def device_bf16_normal(seed: int, shape, device="cuda"):
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def device_absmax(seed: int, shape, device="cuda", std: float = 0.02):
    """Block absmax values with the statistics of 64 N(0, std^2) draws."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = torch.empty(tuple(shape), dtype=torch.float32, device=device)
    flat = out.view(-1)
    step = 1 << 22
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        z = torch.randn((n, 64), generator=gen, device=device, dtype=torch.float32).abs().amax(dim=1)
        flat[i:i + n] = z * std
    return out
