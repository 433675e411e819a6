"""The decode step for callers that cannot allocate device memory
(mk_baseline_decode_step_noalloc): an engine whose device memory is all handed
out by its own arena, or code running where cudaMalloc is not allowed, owns the
step's inputs and outputs but cannot give it scratch; the library keeps that
scratch in one fixed device array of its own.

Called through the C ABI, several times in a row (each step reads the keys and
values the steps before it wrote), with max_ctx changing between calls, it must
give exactly what the library's ordinary multi-kernel entry point gives
(mk_baseline_decode_step, the same kernels on a handle's allocated scratch):
the same logits and the same bits in every slot of both caches. It must also
match the CPU oracle within the parity tests' bounds, report a bad position
through its status word and then change nothing. This file is collected last,
so a run that stops at its first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import TINY
from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
from persistent_megakernel_interpreter_b200.model import Megakernel, pack_weights_host
from test_gpu_parity import TOL, bf16_ulp, reg_bar

pytestmark = pytest.mark.gpu

MK_ERR_BAD_POSITION = 7


def _noalloc_step(cfg_c, packed, tokens, positions, kd, vd, logits, batch, max_ctx, status):
    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = L.mk_baseline_decode_step_noalloc(ctypes.byref(cfg_c), packed.data_ptr(), tokens.data_ptr(),
                                             positions.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                             logits.data_ptr(), batch, max_ctx, status.data_ptr(), stream)
    _lib.check(code, "mk_baseline_decode_step_noalloc")


class Pair:
    """The same model and caches behind both entry points."""

    def __init__(self, batch=2, max_seq=320, past=(100, 37), seed=21):
        torch.cuda.set_device(0)
        self.cfg, self.batch, self.max_seq = TINY, batch, max_seq
        self.w = make_weights(TINY, seed=seed)
        self.k, self.v = make_kv_cache(TINY, batch, max_seq, past=list(past), seed=seed + 1)
        self.mk = Megakernel(TINY, self.w.to("cuda"), max_batch=batch, max_seq=max_seq)
        self.packed = pack_weights_host(TINY, self.w, max_batch=batch, max_seq=max_seq).cuda()
        self.cfg_c = _lib.make_config(TINY, batch, max_seq)
        self.k_ref, self.v_ref = self.k.cuda(), self.v.cuda()
        self.k_na, self.v_na = self.k.cuda(), self.v.cuda()
        self.out_ref = torch.empty(batch, TINY.vocab, dtype=torch.float32, device="cuda")
        self.out_na = torch.full((batch, TINY.vocab), float("nan"), dtype=torch.float32, device="cuda")
        self.status = torch.full((1,), -1, dtype=torch.int32, device="cuda")

    def step(self, toks, pos, max_ctx):
        self.mk.build_schedule(batch=self.batch, max_ctx=max_ctx)
        t = torch.as_tensor(np.asarray(toks), dtype=torch.int32).cuda()
        p = torch.as_tensor(np.asarray(pos), dtype=torch.int32).cuda()
        self.mk.baseline_decode_step(t, p, self.k_ref, self.v_ref, self.out_ref)
        _noalloc_step(self.cfg_c, self.packed, t, p, self.k_na, self.v_na, self.out_na, self.batch, max_ctx,
                      self.status)
        torch.cuda.synchronize()


def _bits(t):
    return t.cpu().view(torch.int16).numpy().copy()


def test_noalloc_step_matches_the_allocating_entry_point_bit_for_bit():
    """Five steps in a row, max_ctx 160 -> 320 -> 160 (the scratch array's layout
    does not depend on it), each step one position further: identical logits and
    identical caches, every layer, sequence and slot."""
    c = Pair()
    positions = np.array([100, 37])
    for step, max_ctx in enumerate((160, 160, 320, 320, 160)):
        toks = make_tokens(TINY, c.batch, seed=23 + step).numpy()
        c.step(toks, positions + step, max_ctx)
        assert int(c.status.item()) == 0
        assert np.array_equal(c.out_na.cpu().numpy(), c.out_ref.cpu().numpy()), (step, max_ctx)
        assert np.array_equal(_bits(c.k_na), _bits(c.k_ref)), step
        assert np.array_equal(_bits(c.v_na), _bits(c.v_ref)), step
    c.mk.close()


def test_noalloc_step_matches_the_oracle():
    """Two steps in a row against the CPU oracle: logits within the parity tests'
    pass line and regression bar, the written key/value within one bf16 ulp at the
    scale of its head, every other slot unchanged."""
    c = Pair(seed=31)
    orc = oracle.Model(TINY, c.w)
    kc = oracle.bits(c.k).copy()
    vc = oracle.bits(c.v).copy()
    positions = np.array([100, 37])
    for step in range(2):
        toks = make_tokens(TINY, c.batch, seed=33 + step).numpy()
        pos = positions + step
        c.step(toks, pos, 160)
        ref = orc.decode_step(toks, pos, kc, vc)
        got = c.out_na.cpu().numpy()
        for b in range(c.batch):
            err = np.max(np.abs(got[b] - ref[b]))
            top = np.max(np.abs(ref[b]))
            assert err <= TOL * top and err <= reg_bar(pos[b]) * top, (step, b, err / top)
            assert int(np.argmax(got[b])) == int(np.argmax(ref[b]))
        kg, vg = _bits(c.k_na), _bits(c.v_na)
        for got_c, ref_c in ((kg, kc), (vg, vc)):
            for b, p in enumerate(pos):
                g = oracle.bf16_to_f32(got_c[:, b, :, p].view(np.uint16)).astype(np.float64)
                r = oracle.bf16_to_f32(ref_c[:, b, :, p]).astype(np.float64)
                assert np.all(np.abs(g - r) <= bf16_ulp(np.max(np.abs(r), axis=-1, keepdims=True)))
                other = np.ones(c.max_seq, bool)
                other[p] = False
                assert np.array_equal(got_c[:, b][:, :, other].view(np.uint16), ref_c[:, b][:, :, other])
    c.mk.close()


def test_noalloc_bad_position_reports_and_writes_nothing():
    """A position at or past max_ctx: the status word says MK_ERR_BAD_POSITION and
    neither the logits buffer nor either cache changes."""
    c = Pair(seed=41)
    toks = torch.as_tensor(make_tokens(TINY, c.batch, seed=43).numpy(), dtype=torch.int32).cuda()
    pos = torch.as_tensor([100, 160], dtype=torch.int32).cuda()  # 160 >= max_ctx
    logits_before = c.out_na.clone()
    k_before, v_before = _bits(c.k_na), _bits(c.v_na)
    _noalloc_step(c.cfg_c, c.packed, toks, pos, c.k_na, c.v_na, c.out_na, c.batch, 160, c.status)
    torch.cuda.synchronize()
    assert int(c.status.item()) == MK_ERR_BAD_POSITION
    assert torch.equal(torch.isnan(c.out_na), torch.isnan(logits_before))
    assert np.array_equal(_bits(c.k_na), k_before) and np.array_equal(_bits(c.v_na), v_before)
    # the next call starts from a cleared error word
    c.step(toks.cpu().numpy(), [100, 37], 160)
    assert int(c.status.item()) == 0
    c.mk.close()


def test_noalloc_step_refuses_scratch_beyond_its_array():
    torch.cuda.set_device(0)
    cfg_c = _lib.make_config(TINY, 8, 16384)
    L = _lib.lib()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    # 16384 positions: beyond the RoPE table's 8192 at head_dim 64 (and more than 32
    # attention partitions)
    code = L.mk_baseline_decode_step_noalloc(ctypes.byref(cfg_c), dummy.data_ptr(), dummy.data_ptr(),
                                             dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                             dummy.data_ptr(), 8, 16384, None, None)
    assert code == 1  # MK_ERR_INVALID_ARG, before anything is launched
