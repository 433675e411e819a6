"""fp64 NumPy brute force of the same decoder, used only to pin ``oracle.c``.

TEST INFRASTRUCTURE ONLY. Written separately from the C oracle (different
language, different loop structure: whole-matrix products, per-head slices), so
an indexing or sign slip in one is unlikely to be repeated in the other.

``decode_step(..., rounding=True)`` rounds the key and value written to the
cache to bf16, like the oracle, but from fp64 values and with torch's bf16
conversion; with ``rounding=False`` it is the exact fp64 decoder (the cache
then holds unrounded values). ``causal_forward`` runs a
whole prefix with no cache at all (every position attends to its own
prefix), which is what an incremental decode must reproduce.
"""
from __future__ import annotations

import numpy as np
import torch


def bf16_bits_to_f64(b) -> np.ndarray:
    if isinstance(b, torch.Tensor):
        return b.to(torch.float64).numpy()
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rb(x: np.ndarray, on: bool) -> np.ndarray:
    """Round an fp64 array to bf16 (via torch) and back to fp64, if ``on``."""
    if not on:
        return x
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _rms(x, w, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * w


def _rope_tables(d: int, pos: int, theta: float):
    i = np.arange(d // 2, dtype=np.float64)
    ang = pos * theta ** (-2.0 * i / d)
    return np.cos(ang), np.sin(ang)


def _rope_heads(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """v: [heads][d]; rotate-half pairs (i, i + d/2)."""
    d = v.shape[-1]
    c, s = _rope_tables(d, pos, theta)
    a, b = v[:, : d // 2], v[:, d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=1)


def _silu(g):
    return g / (1.0 + np.exp(-g))


class Brute:
    def __init__(self, cfg, weights):
        self.cfg = cfg
        f = bf16_bits_to_f64
        w = weights
        self.E = f(w.embed)
        self.layers = []
        for l in range(cfg.n_layers):
            self.layers.append(dict(
                an=f(w.attn_norm[l]), wq=f(w.wq[l]), wk=f(w.wk[l]), wv=f(w.wv[l]), wo=f(w.wo[l]),
                mn=f(w.mlp_norm[l]), wg=f(w.wgate[l]), wu=f(w.wup[l]), wd=f(w.wdown[l])))
        self.fn = f(w.final_norm)

    def decode_step(self, token: int, pos: int, K: list, V: list, rounding: bool = True):
        """One sequence. K, V: per layer fp64 arrays [nkv][max_seq][d], updated in place
        at slot ``pos``. Returns fp64 logits [vocab]."""
        c, r = self.cfg, rounding
        nq, nkv, d = c.n_heads, c.n_kv_heads, c.head_dim
        grp = nq // nkv
        x = self.E[token].copy()
        for l, P in enumerate(self.layers):
            xn = _rms(x, P["an"], c.rms_eps)
            q = (P["wq"] @ xn).reshape(nq, d)
            k = (P["wk"] @ xn).reshape(nkv, d)
            v = (P["wv"] @ xn).reshape(nkv, d)
            q = _rope_heads(q, pos, c.rope_theta)
            K[l][:, pos, :] = _rb(_rope_heads(k, pos, c.rope_theta), r)
            V[l][:, pos, :] = _rb(v, r)
            o = np.empty((nq, d))
            for h in range(nq):
                Kg, Vg = K[l][h // grp, : pos + 1], V[l][h // grp, : pos + 1]
                s = Kg @ q[h] / np.sqrt(d)
                p = np.exp(s - s.max())
                o[h] = (p / p.sum()) @ Vg
            x = x + P["wo"] @ o.reshape(-1)
            xn = _rms(x, P["mn"], c.rms_eps)
            h = _silu(P["wg"] @ xn) * (P["wu"] @ xn)
            x = x + P["wd"] @ h
        y = _rms(x, self.fn, c.rms_eps)
        return self.E @ y

    def causal_forward(self, tokens) -> np.ndarray:
        """Exact fp64 forward of a whole prefix (no cache, no rounding).
        Returns logits [len(tokens)][vocab]."""
        c = self.cfg
        nq, nkv, d = c.n_heads, c.n_kv_heads, c.head_dim
        grp = nq // nkv
        T = len(tokens)
        X = self.E[np.asarray(tokens)].copy()                    # [T][H]
        mask = np.tril(np.ones((T, T), dtype=bool))
        for P in self.layers:
            Xn = np.stack([_rms(X[t], P["an"], c.rms_eps) for t in range(T)])
            Q = (Xn @ P["wq"].T).reshape(T, nq, d)
            Kk = (Xn @ P["wk"].T).reshape(T, nkv, d)
            Vv = (Xn @ P["wv"].T).reshape(T, nkv, d)
            Q = np.stack([_rope_heads(Q[t], t, c.rope_theta) for t in range(T)])
            Kk = np.stack([_rope_heads(Kk[t], t, c.rope_theta) for t in range(T)])
            O = np.empty((T, nq, d))
            for h in range(nq):
                S = Q[:, h, :] @ Kk[:, h // grp, :].T / np.sqrt(d)   # [T][T]
                S = np.where(mask, S, -np.inf)
                Pm = np.exp(S - S.max(axis=1, keepdims=True))
                Pm /= Pm.sum(axis=1, keepdims=True)
                O[:, h, :] = Pm @ Vv[:, h // grp, :]
            X = X + O.reshape(T, -1) @ P["wo"].T
            Xn = np.stack([_rms(X[t], P["mn"], c.rms_eps) for t in range(T)])
            X = X + (_silu(Xn @ P["wg"].T) * (Xn @ P["wu"].T)) @ P["wd"].T
        Y = np.stack([_rms(X[t], self.fn, c.rms_eps) for t in range(T)])
        return Y @ self.E.T
