"""Seeded synthetic inputs for the routed-expert FFN.

This module only draws random numbers: activations, expert weights, router
logits, permutations.  It holds none of the method's arithmetic (no
quantization, routing, sorting or matmul), so the oracle and the CUDA path
can both be fed from it without sharing any step of the computation.

Recipe (same shapes and distributions as the pages' workloads, synthetic):
  * activations x: N(0, 1), rounded to bf16 (round to nearest even);
  * expert weights: N(0, 0.02) fp32, per (bank row) sub-stream;
  * router logits: N(0, 1) + beta * (-s * ln rank_e), rank a per-layer seeded
    permutation of 1..E (a log-Zipf(s) popularity bias), beta = 0.55, s = 1.1;
  * guessed-prefetch workload: a unit-variance residual stream of hidden
    states, x_{l+1} = (x_l + sigma n_l) / sqrt(1 + sigma^2) with n_l ~ N(0, 1)
    and sigma = 0.5 (consecutive layers' states at correlation 0.89), and per
    layer router weights W ~ N(0, 1) [E, H] in bf16, so that
    x W^T / sqrt(H) + bias is N(0, 1) + the same popularity bias as above;
  * every stream is keyed by (seed, tensor kind, layer/row, ...).
"""
from __future__ import annotations

import numpy as np

KIND_X, KIND_LOGITS, KIND_RANK, KIND_WEIGHTS, KIND_BANKPERM, KIND_SLOTPERM, KIND_IDS, KIND_ROUTER, KIND_STREAM = \
    range(1, 10)


def rng(seed: int, *stream) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *[int(s) for s in stream]])))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(seed: int, layer: int, T: int, H: int, step: int = 0) -> np.ndarray:
    """bf16 bits [T, H] of N(0,1)."""
    return to_bf16_bits(rng(seed, KIND_X, layer, step).standard_normal((T, H), dtype=np.float32))


def popularity_rank(seed: int, layer: int, E: int) -> np.ndarray:
    """rank_e in 1..E (a seeded permutation)."""
    return rng(seed, KIND_RANK, layer).permutation(E).astype(np.int64) + 1


def router_logits(seed: int, layer: int, T: int, E: int, beta: float = 0.55, s: float = 1.1,
                  step: int = 0) -> np.ndarray:
    """fp32 [T, E]: N(0,1) + beta * (-s * ln rank_e)."""
    base = rng(seed, KIND_LOGITS, layer, step).standard_normal((T, E), dtype=np.float32)
    if beta == 0.0:
        return base
    bias = (beta * (-s * np.log(popularity_rank(seed, layer, E).astype(np.float64)))).astype(np.float32)
    return (base + bias[None, :]).astype(np.float32)


def router_bias(seed: int, layer: int, E: int, beta: float = 0.55, s: float = 1.1) -> np.ndarray:
    """fp32 [E]: the popularity bias of router_logits, beta * (-s * ln rank_e)."""
    return (beta * (-s * np.log(popularity_rank(seed, layer, E).astype(np.float64)))).astype(np.float32)


def router_weights(seed: int, layer: int, E: int, H: int) -> np.ndarray:
    """bf16 bits [E, H] of N(0, 1): a layer's router rows."""
    return to_bf16_bits(rng(seed, KIND_ROUTER, layer).standard_normal((E, H), dtype=np.float32))


def hidden_stream(seed: int, n_layers: int, T: int, H: int, sigma: float = 0.5, step: int = 0) -> np.ndarray:
    """bf16 bits [n_layers, T, H]: a unit-variance residual stream, each
    layer's state the previous one plus sigma * N(0, 1), rescaled."""
    r = rng(seed, KIND_STREAM, step)
    x = r.standard_normal((T, H), dtype=np.float32)
    out = np.empty((n_layers, T, H), np.uint16)
    c = np.float32(1.0 / np.sqrt(1.0 + sigma * sigma))
    for l in range(n_layers):
        out[l] = to_bf16_bits(x)
        x = ((x + np.float32(sigma) * r.standard_normal((T, H), dtype=np.float32)) * c).astype(np.float32)
    return out


def expert_weights(seed: int, bank_row: int, H: int, I: int, std: float = 0.02):
    """(w_gu [2I, H], w_d [H, I]) fp32 ~ N(0, std)."""
    r = rng(seed, KIND_WEIGHTS, bank_row)
    w_gu = (r.standard_normal((2 * I, H), dtype=np.float32) * np.float32(std)).astype(np.float32)
    w_d = (r.standard_normal((H, I), dtype=np.float32) * np.float32(std)).astype(np.float32)
    return w_gu, w_d


def expert_weights_torch(seed: int, bank_row: int, H: int, I: int, device, std: float = 0.02):
    """Same distribution drawn on a torch device (seeded torch generator)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(bank_row) * 7919 + 17) & 0x7FFFFFFFFFFFFFFF)
    w_gu = torch.randn((2 * I, H), generator=g, device=device, dtype=torch.float32) * std
    w_d = torch.randn((H, I), generator=g, device=device, dtype=torch.float32) * std
    return w_gu, w_d


def bank_permutation(seed: int, layer: int, E: int) -> np.ndarray:
    """Layer `layer`'s expert e uses bank row perm[e]."""
    return rng(seed, KIND_BANKPERM, layer).permutation(E).astype(np.int32)


def slot_permutation(seed: int, layer: int, n: int) -> np.ndarray:
    return rng(seed, KIND_SLOTPERM, layer).permutation(n).astype(np.int32)


def random_routing(seed: int, T: int, E: int, k: int):
    """Distinct expert ids per token and positive weights summing to ~1 (fp32)."""
    r = rng(seed, KIND_IDS, T, E, k)
    ids = np.stack([r.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32) if T else \
        np.zeros((0, k), np.int32)
    w = r.random((T, k)).astype(np.float32) + np.float32(0.05)
    w = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, w
