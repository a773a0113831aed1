"""Seeded synthetic inputs for the W4A16 MoE layer workloads.

This module only draws random numbers and formats them (bf16 bit patterns as uint16); it
holds none of the layer's arithmetic. Both the CPU oracle (via the tests) and the CUDA path
(via the tests and bench.py) take their inputs from here, so the two sides see the same bits.

Workloads (shapes of the OLMoE-1B-7B model that the ExactMoE abstract evaluates on, plus a tiny
and a large-expert case):

    tiny          H=256  I=128   E=8  k=2 T=4      x~N(0,1), W~N(0,0.02), logits~N(0,1)
    olmoe_decode  H=2048 I=1024  E=64 k=8 T=1      16 layers, every expert resident
    olmoe_slots   H=2048 I=1024  E=64 k=8 T=16     16 layers, 16 slots, Zipf(1.1) routing
    olmoe_prefill H=2048 I=1024  E=64 k=8 T=2048   1 layer, Zipf(1.1) routing
    large_expert  H=4096 I=14336 E=8  k=2 T=512    W~N(0,0.01), logits~N(0,1)

Zipf(1.1) routing: expert popularity p_r proportional to r**-1.1 over ranks r=1..E, with the
rank -> expert map a seeded permutation per layer. Per token, logits = log p_e + Gumbel(0,1)
noise, rounded to bf16; the top-k of such logits is a draw of k distinct experts without
replacement with probabilities proportional to p, so the router still runs on every token.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    k: int
    T: int
    layers: int = 1
    slots: int = 0            # 0: every expert resident
    w_std: float = 0.02
    routing: str = "normal"   # "normal": logits ~ N(0,1); "zipf": Zipf(1.1) + Gumbel
    zipf_s: float = 1.1
    seed: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", H=256, I=128, E=8, k=2, T=4),
    "olmoe_decode": Workload("olmoe_decode", H=2048, I=1024, E=64, k=8, T=1, layers=16),
    "olmoe_slots": Workload("olmoe_slots", H=2048, I=1024, E=64, k=8, T=16, layers=16, slots=16,
                            routing="zipf"),
    "olmoe_prefill": Workload("olmoe_prefill", H=2048, I=1024, E=64, k=8, T=2048, routing="zipf"),
    "large_expert": Workload("large_expert", H=4096, I=14336, E=8, k=2, T=512, w_std=0.01),
}

_KIND = {"x": 1, "logits": 2, "w13": 3, "w2": 4, "zipf_perm": 5, "gumbel": 6}


def rng(wl: Workload, kind: str, layer: int = 0, step: int = 0, expert: int = 0) -> np.random.Generator:
    """Independent stream per (workload seed, kind, layer, step, expert)."""
    ss = np.random.SeedSequence([wl.seed, _KIND[kind], layer, step, expert])
    return np.random.Generator(np.random.PCG64(ss))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even, via torch) returned as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(wl: Workload, layer: int = 0, step: int = 0, T: int | None = None) -> np.ndarray:
    T = wl.T if T is None else T
    return to_bf16_bits(rng(wl, "x", layer, step).standard_normal((T, wl.H), dtype=np.float32))


def zipf_log_popularity(wl: Workload, layer: int) -> np.ndarray:
    ranks = np.arange(1, wl.E + 1, dtype=np.float64)
    p = ranks ** (-wl.zipf_s)
    p /= p.sum()
    perm = rng(wl, "zipf_perm", layer).permutation(wl.E)   # rank r -> expert perm[r]
    logp = np.empty(wl.E, np.float64)
    logp[perm] = np.log(p)
    return logp


def router_logits(wl: Workload, layer: int = 0, step: int = 0, T: int | None = None) -> np.ndarray:
    T = wl.T if T is None else T
    if wl.routing == "zipf":
        u = rng(wl, "gumbel", layer, step).random((T, wl.E))
        u = np.clip(u, 1e-300, 1.0 - 1e-16)
        g = -np.log(-np.log(u))
        return to_bf16_bits((zipf_log_popularity(wl, layer)[None, :] + g).astype(np.float32))
    return to_bf16_bits(rng(wl, "logits", layer, step).standard_normal((T, wl.E), dtype=np.float32))


def expert_weights(wl: Workload, layer: int, expert: int):
    """bf16 bits (w13 [2I][H] = [gate; up], w2 [H][I]) of one expert, N(0, w_std)."""
    w13 = rng(wl, "w13", layer, 0, expert).standard_normal((2 * wl.I, wl.H), dtype=np.float32)
    w2 = rng(wl, "w2", layer, 0, expert).standard_normal((wl.H, wl.I), dtype=np.float32)
    return to_bf16_bits(w13 * np.float32(wl.w_std)), to_bf16_bits(w2 * np.float32(wl.w_std))


def bank_weights(wl: Workload, layer: int = 0):
    """bf16 bits of every expert of a layer: (w13 [E][2I][H], w2 [E][H][I])."""
    w13 = np.empty((wl.E, 2 * wl.I, wl.H), np.uint16)
    w2 = np.empty((wl.E, wl.H, wl.I), np.uint16)
    for e in range(wl.E):
        w13[e], w2[e] = expert_weights(wl, layer, e)
    return w13, w2


def device_bank_weights(wl: Workload, layer: int, device) -> tuple:
    """Large-bank variant drawn on the device with torch's seeded generator (benchmarks only:
    the oracle never sees these). Returns bf16 tensors (w13 [E][2I][H], w2 [E][H][I])."""
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * (wl.seed + 1) + 7919 * layer + 17)
    w13 = torch.randn((wl.E, 2 * wl.I, wl.H), generator=g, device=device, dtype=torch.float32)
    w13 = (w13 * wl.w_std).to(torch.bfloat16)
    w2 = torch.randn((wl.E, wl.H, wl.I), generator=g, device=device, dtype=torch.float32)
    w2 = (w2 * wl.w_std).to(torch.bfloat16)
    return w13, w2
