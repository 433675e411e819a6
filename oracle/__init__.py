"""Python view of the CPU oracle (``oracle.c``) plus an fp64 brute force.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may import this package; the product path never does. Nothing here
imports the CUDA library, and the CUDA library shares no code with it.

``decode_step`` is the oracle proper (fp32 over bf16 weights and the bf16 KV
cache; activations fp32; the key and value written to the cache rounded to bf16,
as documented in ``oracle.c``). ``brute`` holds an
independent fp64 NumPy restatement used to pin the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` with gcc into ``liboracle.so`` (no fast-math, no FMA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load(path: str) -> ctypes.CDLL:
    """Open a build of ``oracle.c`` at ``path`` and declare its entry points."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    L.orc_round_bf16.argtypes = [P, P, ctypes.c_int64]
    L.orc_bf16_to_f32.argtypes = [P, P, ctypes.c_int64]
    L.orc_rmsnorm.argtypes = [P, P, ctypes.c_int, ctypes.c_float, P]
    L.orc_rope.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_double]
    L.orc_matvec.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int]
    L.orc_attention.argtypes = [P, P, P] + [ctypes.c_int] * 5 + [P]
    L.orc_silu_mul.argtypes = [P, P, ctypes.c_int, P]
    L.orc_argmax.argtypes = [P, ctypes.c_int]
    L.orc_argmax.restype = ctypes.c_int
    L.orc_decode_step.argtypes = [P, ctypes.c_int, P, P, P, P, ctypes.c_int, P, ctypes.c_int]
    L.orc_decode_step.restype = ctypes.c_int
    L.orc_max_threads.restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def bits(t) -> np.ndarray:
    """bf16 torch tensor (or uint16 array) -> contiguous uint16 NumPy array of its bits."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.uint16)
    import torch
    return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))


def round_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_round_bf16(_p(x), _p(out), x.size)
    return out


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float32)
    lib().orc_bf16_to_f32(_p(b), _p(out), b.size)
    return out


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def rmsnorm(x: np.ndarray, w_bits: np.ndarray, eps: float) -> np.ndarray:
    """x fp32 [n], w bf16 bits [n] -> fp32 [n]."""
    x, w_bits = _f32(x), bits(w_bits)
    out = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), _p(w_bits), x.size, eps, _p(out))
    return out


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate one head vector (fp32, length d); returns the rotated copy."""
    v = np.array(v, dtype=np.float32, copy=True)
    lib().orc_rope(_p(v), v.size, pos, theta)
    return v


def matvec(W_bits: np.ndarray, x: np.ndarray, threads: int = 1) -> np.ndarray:
    """W bf16 bits [rows][cols], x fp32 [cols] -> fp32 [rows]."""
    W_bits, x = bits(W_bits), _f32(x)
    rows, cols = W_bits.shape
    y = np.empty(rows, dtype=np.float32)
    lib().orc_matvec(_p(W_bits), _p(x), rows, cols, _p(y), threads)
    return y


def attention(q: np.ndarray, K_bits, V_bits, n_keys: int) -> np.ndarray:
    """q fp32 [nq][d]; K, V bf16 bits [nkv][seq][d]. Returns fp32 [nq][d]."""
    q, K_bits, V_bits = _f32(q), bits(K_bits), bits(V_bits)
    nq, d = q.shape
    nkv, seq, _ = K_bits.shape
    out = np.empty((nq, d), dtype=np.float32)
    lib().orc_attention(_p(q), _p(K_bits), _p(V_bits), nq, nkv, d, n_keys, seq, _p(out))
    return out


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g, u = _f32(g), _f32(u)
    out = np.empty(g.shape, dtype=np.float32)
    lib().orc_silu_mul(_p(g), _p(u), g.size, _p(out))
    return out


def argmax(x: np.ndarray) -> int:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return int(lib().orc_argmax(_p(x), x.size))


def max_threads() -> int:
    return int(lib().orc_max_threads())


class _Model(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in ("n_layers", "hidden", "n_heads", "n_kv_heads",
                                           "head_dim", "ffn", "vocab")]
                + [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_double)]
                + [(n, ctypes.c_void_p) for n in ("embed", "attn_norm", "wq", "wk", "wv", "wo",
                                                 "mlp_norm", "wgate", "wup", "wdown",
                                                 "final_norm", "lm_head")])


class Model:
    """Host copy of a model's weights (uint16 bf16 bits) bound to the oracle."""

    def __init__(self, cfg, weights):
        self.cfg = cfg
        self._keep = []
        w = weights

        def arr(t):
            a = bits(t)
            self._keep.append(a)
            return a

        def ptrs(ts):
            arrs = [arr(t) for t in ts]
            tab = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
            self._keep.append(tab)
            return ctypes.cast(tab, ctypes.c_void_p)

        self.embed = arr(w.embed)
        m = _Model()
        m.n_layers, m.hidden, m.n_heads = cfg.n_layers, cfg.hidden, cfg.n_heads
        m.n_kv_heads, m.head_dim, m.ffn, m.vocab = cfg.n_kv_heads, cfg.head_dim, cfg.ffn, cfg.vocab
        m.rms_eps, m.rope_theta = cfg.rms_eps, cfg.rope_theta
        m.embed = self.embed.ctypes.data
        m.attn_norm, m.wq, m.wk, m.wv = ptrs(w.attn_norm), ptrs(w.wq), ptrs(w.wk), ptrs(w.wv)
        m.wo, m.mlp_norm, m.wgate = ptrs(w.wo), ptrs(w.mlp_norm), ptrs(w.wgate)
        m.wup, m.wdown = ptrs(w.wup), ptrs(w.wdown)
        m.final_norm = arr(w.final_norm).ctypes.data
        m.lm_head = None
        self._m = m

    def decode_step(self, tokens, positions, k_cache: np.ndarray, v_cache: np.ndarray,
                    threads: int = 0) -> np.ndarray:
        """One decode step for every sequence; updates the caches in place.

        ``k_cache``/``v_cache``: uint16 arrays [L][B][nkv][max_seq][d]. Returns
        fp32 logits [B][vocab]. Raises ValueError on an out-of-range token or
        position (nothing written then)."""
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        positions = np.ascontiguousarray(positions, dtype=np.int32)
        assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
        assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
        B = tokens.size
        max_seq = k_cache.shape[3]
        logits = np.empty((B, self.cfg.vocab), dtype=np.float32)
        rc = lib().orc_decode_step(ctypes.addressof(self._m), B, _p(tokens), _p(positions),
                                   _p(k_cache), _p(v_cache), max_seq, _p(logits),
                                   threads or max_threads())
        if rc != 0:
            raise ValueError("token or position out of range")
        return logits
