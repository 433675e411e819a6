"""Seeded synthetic inputs for the decode step: weights, KV cache, tokens.

This module only draws random numbers. It holds none of the decode step's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (shared by tests, the smoke check and the benchmark):
  * matrices: bf16 of N(0, 0.02) draws (the stated init of every config);
  * norm weights: exactly 1.0 unless ``norm_jitter`` > 0, then 1 + N(0, jitter);
  * KV cache: slots ``0 .. past-1`` of every (layer, sequence, kv head) hold
    bf16 of N(0, 1) draws; the remaining slots are zero;
  * tokens: uniform integers in ``[0, vocab)``.

Each tensor gets its own stream of numbers, derived from (seed, tensor id), and
is filled in fixed 4 Mi-element blocks, each with its own spawned child seed,
so the values do not depend on the thread count.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np
import torch

from .config import ModelConfig

_BLOCK = 1 << 22


def _normal_f32(n: int, seed: int, tensor_id: int, threads: int | None = None) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    kids = np.random.SeedSequence([seed, tensor_id]).spawn((n + _BLOCK - 1) // _BLOCK)

    def fill(i: int) -> None:
        g = np.random.Generator(np.random.PCG64(kids[i]))
        g.standard_normal(out=out[i * _BLOCK:(i + 1) * _BLOCK], dtype=np.float32)

    threads = threads or min(32, os.cpu_count() or 1)
    if len(kids) == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(len(kids))))
    return out


def normal_bf16(shape, std: float, seed: int, tensor_id: int, mean: float = 0.0) -> torch.Tensor:
    """bf16 tensor of N(mean, std) draws (rounded to nearest even by torch)."""
    n = int(np.prod(shape))
    a = torch.from_numpy(_normal_f32(n, seed, tensor_id))
    if std != 1.0:
        a.mul_(std)
    if mean != 0.0:
        a.add_(mean)
    return a.to(torch.bfloat16).reshape(shape)


@dataclasses.dataclass
class Weights:
    """Row-major bf16 CPU tensors; matrices are ``[out][in]``."""
    embed: torch.Tensor                 # [vocab][hidden]
    attn_norm: list[torch.Tensor]       # [hidden] per layer
    wq: list[torch.Tensor]              # [n_heads*head_dim][hidden]
    wk: list[torch.Tensor]              # [n_kv_heads*head_dim][hidden]
    wv: list[torch.Tensor]              # [n_kv_heads*head_dim][hidden]
    wo: list[torch.Tensor]              # [hidden][n_heads*head_dim]
    mlp_norm: list[torch.Tensor]        # [hidden]
    wgate: list[torch.Tensor]           # [ffn][hidden]
    wup: list[torch.Tensor]             # [ffn][hidden]
    wdown: list[torch.Tensor]           # [hidden][ffn]
    final_norm: torch.Tensor            # [hidden]

    def to(self, device) -> "Weights":
        f = lambda t: t.to(device)
        return Weights(f(self.embed), [f(t) for t in self.attn_norm], [f(t) for t in self.wq],
                       [f(t) for t in self.wk], [f(t) for t in self.wv], [f(t) for t in self.wo],
                       [f(t) for t in self.mlp_norm], [f(t) for t in self.wgate],
                       [f(t) for t in self.wup], [f(t) for t in self.wdown], f(self.final_norm))


def make_weights(cfg: ModelConfig, seed: int = 0, std: float = 0.02,
                 norm_jitter: float = 0.0) -> Weights:
    tid = iter(range(1, 1 << 30))
    H, Q, KV, F = cfg.hidden, cfg.q_dim, cfg.kv_dim, cfg.ffn

    def mat(rows, cols):
        return normal_bf16((rows, cols), std, seed, next(tid))

    def norm():
        i = next(tid)
        if norm_jitter > 0:
            return normal_bf16((H,), norm_jitter, seed, i, mean=1.0)
        return torch.ones(H, dtype=torch.bfloat16)

    embed = mat(cfg.vocab, H)
    L = cfg.n_layers
    attn_norm, wq, wk, wv, wo, mlp_norm, wg, wu, wd = ([] for _ in range(9))
    for _ in range(L):
        attn_norm.append(norm())
        wq.append(mat(Q, H))
        wk.append(mat(KV, H))
        wv.append(mat(KV, H))
        wo.append(mat(H, Q))
        mlp_norm.append(norm())
        wg.append(mat(F, H))
        wu.append(mat(F, H))
        wd.append(mat(H, F))
    final_norm = norm()
    return Weights(embed, attn_norm, wq, wk, wv, wo, mlp_norm, wg, wu, wd, final_norm)


def make_kv_cache(cfg: ModelConfig, batch: int, max_seq: int, past, seed: int = 1):
    """K and V caches, bf16 ``[n_layers][batch][n_kv_heads][max_seq][head_dim]``.

    ``past`` is an int or a per-sequence list: slots ``0..past[b]-1`` hold N(0,1)
    draws, every other slot is zero.
    """
    if isinstance(past, int):
        past = [past] * batch
    shape = (cfg.n_layers, batch, cfg.n_kv_heads, max_seq, cfg.head_dim)
    k = torch.zeros(shape, dtype=torch.bfloat16)
    v = torch.zeros(shape, dtype=torch.bfloat16)
    for b, p in enumerate(past):
        if p <= 0:
            continue
        sub = (cfg.n_layers, cfg.n_kv_heads, p, cfg.head_dim)
        k[:, b, :, :p, :] = normal_bf16(sub, 1.0, seed, 2 * b + 1)
        v[:, b, :, :p, :] = normal_bf16(sub, 1.0, seed, 2 * b + 2)
    return k, v


def make_tokens(cfg: ModelConfig, n: int, seed: int = 2) -> torch.Tensor:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0])))
    return torch.from_numpy(g.integers(0, cfg.vocab, size=n, dtype=np.int64).astype(np.int32))
