"""Weight packer: host packing equals the layout documented in include/mk.h,
re-derived here independently by unpacking (bit-exact round trip)."""
import dataclasses

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings

from persistent_megakernel_interpreter_b200.config import LLAMA_3B, TINY, ModelConfig
from persistent_megakernel_interpreter_b200.inputs import make_weights
from persistent_megakernel_interpreter_b200.model import pack_weights_host
from strategies import shapes


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _align(x, a=256):
    return (x + a - 1) // a * a


def unpack(cfg: ModelConfig, buf: np.ndarray):
    """Inverse of the documented layout, written from the header's description."""
    H, d, nq, nkv, F, V, L = cfg.hidden, cfg.head_dim, cfg.n_heads, cfg.n_kv_heads, cfg.ffn, cfg.vocab, cfg.n_layers
    grp = nq // nkv
    Q = nq * d
    b16 = buf.view(np.uint16)
    off = 0
    E = b16[off // 2: off // 2 + V * H].reshape(V, H)
    off = _align(V * H * 2)
    layers = []
    for l in range(L):
        out = {}
        # QKV
        qkv_rows = Q + 2 * nkv * d
        blk = b16[off // 2: off // 2 + qkv_rows * H].reshape(qkv_rows, H)
        wq = np.zeros((Q, H), np.uint16)
        wk = np.zeros((nkv * d, H), np.uint16)
        wv = np.zeros((nkv * d, H), np.uint16)
        r = 0
        for g in range(nkv):
            for hs in range(grp + 2):
                for j in range(d // 4):
                    for k in range(4):
                        if hs <= grp:
                            row = 2 * j + (k >> 1) + (d // 2 if k & 1 else 0)
                        else:
                            row = 4 * j + k
                        if hs < grp:
                            wq[(g * grp + hs) * d + row] = blk[r]
                        elif hs == grp:
                            wk[g * d + row] = blk[r]
                        else:
                            wv[g * d + row] = blk[r]
                        r += 1
        out.update(wq=wq, wk=wk, wv=wv)
        off = _align(off + qkv_rows * H * 2)
        out["wo"] = b16[off // 2: off // 2 + H * Q].reshape(H, Q)
        off = _align(off + H * Q * 2)
        gu = b16[off // 2: off // 2 + 2 * F * H].reshape(F // 2, 4, H)
        out["wgate"] = np.stack([gu[:, 0], gu[:, 2]], axis=1).reshape(F, H)
        out["wup"] = np.stack([gu[:, 1], gu[:, 3]], axis=1).reshape(F, H)
        off = _align(off + 2 * F * H * 2)
        dn = b16[off // 2: off // 2 + H * F].reshape(H // 4, 4, 4, F // 4)  # [rb][c][r][k]
        out["wdown"] = dn.transpose(0, 2, 1, 3).reshape(H, F)
        off = _align(off + H * F * 2)
        layers.append(out)
    norms = b16[off // 2: off // 2 + (2 * L + 1) * H].reshape(2 * L + 1, H)
    return E, layers, norms


# the 2-layer model, and the 3B-style head layout (head_dim 128, 3 query heads per KV
# head) on a small model
SHAPES = [TINY, dataclasses.replace(LLAMA_3B, name="3b-heads-small", n_layers=2, hidden=768, n_heads=6,
                                    n_kv_heads=2, ffn=2048, vocab=4096)]


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: c.name)
def test_pack_roundtrip_bit_exact(cfg):
    check_roundtrip(cfg)


@settings(max_examples=25, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(cfg=shapes())
def test_pack_roundtrip_bit_exact_random_shapes(cfg):
    """The same round trip on drawn shapes (head_dim 64 / 128, 1-4 query heads per KV
    head, 1-3 layers, hidden 256-1024, ffn 1024-3072, vocab any multiple of 4)."""
    check_roundtrip(cfg)


def check_roundtrip(cfg):
    w = make_weights(cfg, seed=7, norm_jitter=0.1)
    buf = pack_weights_host(cfg, w).numpy()
    E, layers, norms = unpack(cfg, buf)
    assert np.array_equal(E, _u16(w.embed))
    for l in range(cfg.n_layers):
        for name in ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown"):
            assert np.array_equal(layers[l][name], _u16(getattr(w, name)[l])), (l, name)
        assert np.array_equal(norms[2 * l], _u16(w.attn_norm[l]))
        assert np.array_equal(norms[2 * l + 1], _u16(w.mlp_norm[l]))
    assert np.array_equal(norms[2 * cfg.n_layers], _u16(w.final_norm))


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: c.name)
def test_pack_is_a_permutation_of_the_input_bytes(cfg):
    """Every input element appears exactly once; the rest of the buffer is zero padding."""
    w = make_weights(cfg, seed=8, norm_jitter=0.1)
    buf = pack_weights_host(cfg, w).numpy().view(np.uint16)
    parts = [_u16(w.embed).ravel(), _u16(w.final_norm)]
    for l in range(cfg.n_layers):
        for name in ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown", "attn_norm", "mlp_norm"):
            parts.append(_u16(getattr(w, name)[l]).ravel())
    src = np.concatenate(parts)
    assert buf.size >= src.size
    counts = np.bincount(buf, minlength=65536)
    counts[0] -= buf.size - src.size
    assert np.array_equal(counts, np.bincount(src, minlength=65536))


def test_host_packer_refuses_bad_arguments_without_writing():
    """Null pointers, a destination one byte short, an incomplete weight set and an
    unsupported shape are refused (MK_ERR_INVALID_ARG / MK_ERR_UNSUPPORTED) before
    any byte of the destination is written."""
    import ctypes
    from persistent_megakernel_interpreter_b200 import _lib
    L = _lib.lib()
    c = _lib.make_config(TINY, 1, 1)
    n = L.mk_packed_bytes(ctypes.byref(c))
    w = make_weights(TINY, seed=3)
    keep = []

    def tab(ts):
        ts = [t.contiguous() for t in ts]
        keep.extend(ts)
        arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
        keep.append(arr)
        return ctypes.cast(arr, ctypes.c_void_p)

    mw = _lib.MkWeights()
    mw.embed, mw.final_norm = w.embed.data_ptr(), w.final_norm.data_ptr()
    for name in ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wgate", "wup", "wdown"):
        setattr(mw, name, tab(getattr(w, name)))
    dst = np.full(n, 0xA5, np.uint8)
    p = dst.ctypes.data_as(ctypes.c_void_p)
    assert L.mk_pack_weights_host(None, ctypes.byref(mw), p, n) == 1
    assert L.mk_pack_weights_host(ctypes.byref(c), None, p, n) == 1
    assert L.mk_pack_weights_host(ctypes.byref(c), ctypes.byref(mw), None, n) == 1
    assert L.mk_pack_weights_host(ctypes.byref(c), ctypes.byref(mw), p, n - 1) == 1
    partial = _lib.MkWeights.from_buffer_copy(mw)
    partial.wdown = None
    assert L.mk_pack_weights_host(ctypes.byref(c), ctypes.byref(partial), p, n) == 1
    bad = _lib.make_config(dataclasses.replace(TINY, head_dim=96), 1, 1)
    assert L.mk_pack_weights_host(ctypes.byref(bad), ctypes.byref(mw), p, n) == 3
    assert np.all(dst == 0xA5)
    assert L.mk_pack_weights_host(ctypes.byref(c), ctypes.byref(mw), p, n) == 0
    assert not np.all(dst == 0xA5)
