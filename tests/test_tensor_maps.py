"""The tensor-core path's TMA views of the packed weights, checked on the host: for
every fill a schedule plans, the block its tensor map's box covers from the fill's
start coordinates must be exactly that fill's weight rows and 64-column K blocks in
the packed layout (restated here from mk_pack_weights_host's description: the
embedding rows, then per layer QKV [rows][hidden], O [hidden][Q], gate/up
[2 ffn][hidden] and down [row block][chunk][4][ffn/4], regions 256-byte aligned).
The start coordinates are the kernel's (issue_mma_fill): {0, row0, kb0, layer}
for QKV / O / gate-up, {0, row0, kb0} for the LM head, {0, 0, row0 / 4, kb0, layer}
for down chunk c. A wrong stride, dimension order or box size shows up as an
address mismatch, with no GPU."""
import ctypes
import dataclasses

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B, TINY
from persistent_megakernel_interpreter_b200.model import plan_schedule
from test_schedule import mma_fills
from strategies import shapes


def specs(cfg, stage_bytes):
    L = _lib.lib()
    c = _lib.make_config(cfg, 8, 129)
    n = ctypes.c_size_t(0)
    _lib.check(L.mk_tensor_map_specs_host(ctypes.byref(c), stage_bytes, None, 0, ctypes.byref(n)), "specs")
    out = (_lib.MkTmapSpec * n.value)()
    _lib.check(L.mk_tensor_map_specs_host(ctypes.byref(c), stage_bytes, out, n.value, ctypes.byref(n)), "specs")
    return {s.index: s for s in out}


def align(x, a=256):
    return (x + a - 1) // a * a


class Packed:
    """Byte offsets of the packed layout (restated from its description)."""

    def __init__(self, cfg):
        H, F, V, d = cfg.hidden, cfg.ffn, cfg.vocab, cfg.head_dim
        self.H, self.F, self.Q = H, F, cfg.n_heads * d
        self.qkv_rows = (cfg.n_heads + 2 * cfg.n_kv_heads) * d
        self.off_layer0 = align(V * H * 2)
        self.rel_o = align(self.qkv_rows * H * 2)
        self.rel_gu = align(self.rel_o + H * self.Q * 2)
        self.rel_down = align(self.rel_gu + 2 * F * H * 2)
        self.layer_stride = align(self.rel_down + H * F * 2)

    def addr(self, op, layer, chunk, row, k):
        lb = self.off_layer0 + layer * self.layer_stride
        if op == _lib.OP_QKV:
            return lb + (row * self.H + k) * 2
        if op == _lib.OP_OPROJ:
            return lb + self.rel_o + (row * self.Q + k) * 2
        if op == _lib.OP_GATEUP:
            return lb + self.rel_gu + (row * self.H + k) * 2
        if op == _lib.OP_DOWN:
            rb, r = row // 4, row % 4
            return lb + self.rel_down + ((rb * 4 + chunk) * 4 + r) * (self.F // 4) * 2 + k * 2
        return (row * self.H + k) * 2  # LM head: the embedding rows


def box_addr(s, coords):
    """Byte offset of the element at `coords` of a map (innermost first)."""
    a = s.base_offset + 2 * coords[0]
    for i in range(1, s.rank):
        a += coords[i] * s.strides[i - 1]
    return a


@pytest.mark.parametrize("cfg,batch,n_sm", [(TINY, 2, 37), (TINY, 8, 148), (LLAMA_1B, 8, 148),
                                            (LLAMA_3B, 8, 148), (LLAMA_3B, 3, 100)])
def test_every_fill_reads_its_rows(cfg, batch, n_sm):
    check_fills(cfg, batch, n_sm)


@settings(max_examples=80, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(cfg=shapes(), batch=st.integers(2, 8), n_sm=st.integers(1, 148))
def test_every_fill_reads_its_rows_random_shapes(cfg, batch, n_sm):
    """The same check on drawn shapes (head_dim 64 / 128, 1-4 query heads per KV head,
    hidden 256-1024, ffn 1024-3072), vocabularies rounded to whole 8-row units."""
    check_fills(dataclasses.replace(cfg, vocab=cfg.vocab // 8 * 8), batch, n_sm)


def check_fills(cfg, batch, n_sm):
    instrs, offs, info = plan_schedule(cfg, batch, 129, n_sm, max_batch=8, max_seq=129, proj=2)
    assert info.proj == _lib.PROJ_TENSOR_CORES
    sb = info.stage_bytes
    S = specs(cfg, sb)
    pk = Packed(cfg)
    rng = np.random.default_rng(0)
    checked = 0
    for ins in instrs:
        if ins.op == _lib.OP_ATTN:
            continue
        g, fills = mma_fills(ins, cfg, sb)
        for c, rg, seg, kf, boxes, rows, nb in fills:
            row0 = 4 * ((rg * (cfg.ffn // 8) if ins.op == _lib.OP_GATEUP else 0) + ins.first) + 128 * seg
            hk = rows // 8 - 1
            if ins.op == _lib.OP_DOWN:
                s = S[64 + c * 8 + hk]
                assert s.rank == 5 and s.box[0] == 64 and s.box[1] * s.box[2] == rows and s.box[3] == nb
            else:
                kind = {_lib.OP_QKV: 0, _lib.OP_OPROJ: 1, _lib.OP_GATEUP: 2, _lib.OP_LMHEAD: 3}[ins.op]
                s = S[kind * 16 + hk]
                assert s.box[0] == 64 and s.box[1] == rows and s.box[2] == nb
            # the box fits a ring stage; every stride and the base meet TMA's 16-byte rule
            assert nb * rows * 128 <= sb
            assert s.base_offset % 16 == 0 and all(s.strides[i] % 16 == 0 for i in range(s.rank - 1))
            kb0 = kf * nb
            # a sample of the box's elements (all corners, plus random ones), in range of K
            pts = [(ki, r, b) for ki in (0, 63) for r in (0, rows - 1) for b in (0, len(boxes) - 1)]
            pts += [(int(rng.integers(64)), int(rng.integers(rows)), int(rng.integers(len(boxes))))
                    for _ in range(4)]
            for ki, r, b in pts:
                k = (kb0 + b) * 64 + ki
                want = pk.addr(ins.op, ins.layer, c, row0 + r, k)
                if ins.op == _lib.OP_DOWN:
                    coords = (ki, r % 4, row0 // 4 + r // 4, kb0 + b, ins.layer)
                elif ins.op == _lib.OP_LMHEAD:
                    coords = (ki, row0 + r, kb0 + b)
                else:
                    coords = (ki, row0 + r, kb0 + b, ins.layer)
                assert all(coords[i] < s.dims[i] for i in range(s.rank)), (coords, list(s.dims))
                assert box_addr(s, coords) == want, (ins.op, ins.layer, c, row0 + r, k)
                checked += 1
    assert checked > 0


def test_specs_refuse_bad_arguments():
    L = _lib.lib()
    c = _lib.make_config(TINY, 2, 64)
    n = ctypes.c_size_t(0)
    assert L.mk_tensor_map_specs_host(ctypes.byref(c), 0, None, 0, ctypes.byref(n)) == 1
    assert L.mk_tensor_map_specs_host(None, 16384, None, 0, ctypes.byref(n)) == 1
    assert L.mk_tensor_map_specs_host(ctypes.byref(c), 16384, None, 0, None) == 1
    assert L.mk_tensor_map_specs_host(ctypes.byref(c), 16384, None, 0, ctypes.byref(n)) == 0
    out = (_lib.MkTmapSpec * 1)()
    assert L.mk_tensor_map_specs_host(ctypes.byref(c), 16384, out, 1, ctypes.byref(n)) == 1  # too small
