"""The decode step for callers that cannot allocate device memory
(mk_baseline_decode_step_noalloc): an engine whose device memory is all handed
out by its own arena, or code running where cudaMalloc is not allowed, owns the
step's inputs and outputs but cannot give it scratch; the library keeps that
scratch in one fixed device array of its own.

Called through the C ABI, twice in a row (the second step reads the key/value
the first one wrote), its logits and KV writes must agree with the library's
ordinary multi-kernel entry point (mk_baseline_decode_step, which runs on a
handle's allocated scratch) within the tolerance of the other parity tests.
This file is collected last, so a run that stops at its first failure has run
every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import TINY
from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
from persistent_megakernel_interpreter_b200.model import Megakernel, pack_weights_host

pytestmark = pytest.mark.gpu

TOL = 1e-2  # max |d logit| <= TOL * max |logit|, as in the other parity tests


def _noalloc_step(cfg_c, packed, tokens, positions, kd, vd, logits, batch, max_ctx, status):
    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = L.mk_baseline_decode_step_noalloc(ctypes.byref(cfg_c), packed.data_ptr(), tokens.data_ptr(),
                                             positions.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                             logits.data_ptr(), batch, max_ctx, status.data_ptr(), stream)
    _lib.check(code, "mk_baseline_decode_step_noalloc")


def test_noalloc_step_matches_the_allocating_entry_point_twice():
    torch.cuda.set_device(0)
    cfg, batch, max_seq, max_ctx = TINY, 2, 160, 160
    w = make_weights(cfg, seed=21)
    k, v = make_kv_cache(cfg, batch, max_seq, past=[100, 37], seed=22)
    # the ordinary entry point, on a handle with its own scratch
    mk = Megakernel(cfg, w.to("cuda"), max_batch=batch, max_seq=max_seq)
    mk.build_schedule(batch=batch, max_ctx=max_ctx)
    # the caller's own buffers for the allocation-free step
    packed = pack_weights_host(cfg, w, max_batch=batch, max_seq=max_seq).cuda()
    cfg_c = _lib.make_config(cfg, batch, max_seq)
    k_ref, v_ref = k.cuda(), v.cuda()
    k_na, v_na = k.cuda(), v.cuda()
    out_ref = torch.empty(batch, cfg.vocab, dtype=torch.float32, device="cuda")
    out_na = torch.full((batch, cfg.vocab), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    positions = [100, 37]
    for step in range(2):  # the second call reads what the first one wrote
        toks = torch.as_tensor(make_tokens(cfg, batch, seed=23 + step).numpy(), dtype=torch.int32).cuda()
        pos = torch.as_tensor(np.asarray(positions) + step, dtype=torch.int32).cuda()
        mk.baseline_decode_step(toks, pos, k_ref, v_ref, out_ref)
        _noalloc_step(cfg_c, packed, toks, pos, k_na, v_na, out_na, batch, max_ctx, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref, got = out_ref.cpu().numpy(), out_na.cpu().numpy()
        for b in range(batch):
            err = np.max(np.abs(got[b] - ref[b]))
            assert err <= TOL * np.max(np.abs(ref[b])), (step, b, err)
            assert int(np.argmax(got[b])) == int(np.argmax(ref[b]))
        # the key/value slots written by the step agree too (bf16 bits)
        kr, kn = k_ref.cpu().view(torch.int16).numpy(), k_na.cpu().view(torch.int16).numpy()
        vr, vn = v_ref.cpu().view(torch.int16).numpy(), v_na.cpu().view(torch.int16).numpy()
        for b, p in enumerate(np.asarray(positions) + step):
            kf = kr[:, b, :, p].astype(np.int32) - kn[:, b, :, p].astype(np.int32)
            vf = vr[:, b, :, p].astype(np.int32) - vn[:, b, :, p].astype(np.int32)
            assert np.max(np.abs(kf)) <= 1 and np.max(np.abs(vf)) <= 1  # at most one bf16 ulp
    mk.close()


def test_noalloc_step_refuses_scratch_beyond_its_array():
    torch.cuda.set_device(0)
    cfg = TINY
    cfg_c = _lib.make_config(cfg, 8, 16384)
    L = _lib.lib()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    # 16384 positions need more than 32 attention partitions and a 4 MiB+ RoPE table
    code = L.mk_baseline_decode_step_noalloc(ctypes.byref(cfg_c), dummy.data_ptr(), dummy.data_ptr(),
                                             dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                             dummy.data_ptr(), 8, 16384, None, None)
    assert code == 1  # MK_ERR_INVALID_ARG, before anything is launched
