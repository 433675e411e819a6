"""Python binding of the megakernel library: a thin wrapper over the C ABI.

``Megakernel(cfg, weights, max_batch, max_seq)`` packs device weights into a
library handle; ``build_schedule``; ``decode_step`` (one persistent kernel
launch), ``baseline_decode_step`` (the multi-kernel baseline) and
``decode_step_host`` (host buffers in and out) run one step; ``greedy_select``
picks the next tokens from a step's logits on the device. PyTorch supplies
device memory and streams only.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from .config import ModelConfig


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Megakernel:
    def __init__(self, cfg: ModelConfig, weights, max_batch: int = 1, max_seq: int = 256,
                 device: int | None = None):
        """``weights``: an ``inputs.Weights`` whose tensors are bf16 on the CUDA device."""
        L = _lib.lib()
        self.cfg = cfg
        self.max_batch, self.max_seq = max_batch, max_seq
        self.device = torch.cuda.current_device() if device is None else device
        self._cfg = _lib.make_config(cfg, max_batch, max_seq)
        w = weights
        keep = []

        def tab(ts):
            for t in ts:
                assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
            arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
            keep.append(arr)
            return ctypes.cast(arr, ctypes.c_void_p)

        mw = _lib.MkWeights(_ptr(w.embed), tab(w.attn_norm), tab(w.wq), tab(w.wk), tab(w.wv),
                            tab(w.wo), tab(w.mlp_norm), tab(w.wgate), tab(w.wup), tab(w.wdown),
                            _ptr(w.final_norm))
        h = ctypes.c_void_p()
        torch.cuda.synchronize(self.device)
        _lib.check(L.mk_create(ctypes.byref(self._cfg), ctypes.byref(mw), self.device,
                               ctypes.byref(h)), "mk_create")
        self._h = h
        self.batch = None

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.lib().mk_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def build_schedule(self, batch: int, max_ctx: int, **opts) -> _lib.MkScheduleInfo:
        o = _lib.make_opts(**opts) if opts else None
        _lib.check(_lib.lib().mk_build_schedule(self._h, batch, max_ctx,
                                                ctypes.byref(o) if o is not None else None),
                   "mk_build_schedule")
        self.batch = batch
        return self.schedule_info()

    def schedule_info(self) -> _lib.MkScheduleInfo:
        info = _lib.MkScheduleInfo()
        _lib.check(_lib.lib().mk_get_schedule_info(self._h, ctypes.byref(info)), "schedule info")
        return info

    def _step(self, fn, tokens, positions, k_cache, v_cache, logits, stream):
        for t, dt in ((tokens, torch.int32), (positions, torch.int32), (logits, torch.float32)):
            assert t.is_cuda and t.dtype == dt and t.is_contiguous()
        assert k_cache.dtype == torch.bfloat16 and v_cache.dtype == torch.bfloat16
        _lib.check(fn(self._h, _ptr(tokens), _ptr(positions), _ptr(k_cache), _ptr(v_cache),
                      _ptr(logits), _stream(stream)), fn.__name__)

    def decode_step(self, tokens, positions, k_cache, v_cache, logits, stream=None) -> None:
        """One step of the persistent megakernel, asynchronous on ``stream``."""
        self._step(_lib.lib().mk_decode_step, tokens, positions, k_cache, v_cache, logits, stream)

    def decode_steps_greedy(self, tokens, positions, k_cache, v_cache, logits, n_steps: int,
                            generated=None, stream=None) -> None:
        """``n_steps`` greedy steps back to back (the choice fused into each step's LM
        head): tokens and positions are overwritten with the next ones after every
        step; ``generated`` (int32 [n_steps][batch], optional) receives the tokens."""
        for t, dt in ((tokens, torch.int32), (positions, torch.int32), (logits, torch.float32)):
            assert t.is_cuda and t.dtype == dt and t.is_contiguous()
        assert k_cache.dtype == torch.bfloat16 and v_cache.dtype == torch.bfloat16
        if generated is not None:
            assert generated.is_cuda and generated.dtype == torch.int32 and generated.is_contiguous()
            assert generated.numel() >= n_steps * tokens.numel()
        _lib.check(_lib.lib().mk_decode_steps_greedy(
            self._h, _ptr(tokens), _ptr(positions), _ptr(k_cache), _ptr(v_cache), _ptr(logits),
            _ptr(generated) if generated is not None else None, int(n_steps), _stream(stream)),
            "mk_decode_steps_greedy")

    def baseline_decode_step(self, tokens, positions, k_cache, v_cache, logits, stream=None) -> None:
        """The same step as one kernel per op and layer."""
        self._step(_lib.lib().mk_baseline_decode_step, tokens, positions, k_cache, v_cache, logits,
                   stream)

    def decode_step_host(self, tokens_host, positions_host, k_cache, v_cache, logits_host,
                         stream=None) -> None:
        """Host int32 tokens/positions in, host fp32 logits out (pinned memory preferred)."""
        for t in (tokens_host, positions_host, logits_host):
            assert not t.is_cuda and t.is_contiguous()
        _lib.check(_lib.lib().mk_decode_step_host(
            self._h, _ptr(tokens_host), _ptr(positions_host), _ptr(k_cache), _ptr(v_cache),
            _ptr(logits_host), _stream(stream)), "mk_decode_step_host")

    def status(self) -> tuple[int, str]:
        """Synchronise, then return and clear the device status: (code, message)."""
        code = ctypes.c_int(0)
        buf = ctypes.create_string_buffer(512)
        _lib.check(_lib.lib().mk_get_status(self._h, ctypes.byref(code), buf, 512), "mk_get_status")
        return code.value, buf.value.decode()

    def trace(self):
        """Per-job timestamps of the last step: uint64 array [n_sm][jobs][16] (see mk.h)."""
        import numpy as np
        L = _lib.lib()
        jobs = ctypes.c_int32(0)
        _lib.check(L.mk_read_trace(self._h, None, 0, ctypes.byref(jobs)), "mk_read_trace")
        n_sm = self.schedule_info().n_sm
        out = np.zeros((n_sm, jobs.value, 16), dtype=np.uint64)
        if jobs.value:
            _lib.check(L.mk_read_trace(self._h, out.ctypes.data, out.nbytes, ctypes.byref(jobs)),
                       "mk_read_trace")
        return out

    def counters(self) -> list[int]:
        L = _lib.lib()
        n = ctypes.c_size_t(0)
        _lib.check(L.mk_read_counters(self._h, None, 0, ctypes.byref(n)), "mk_read_counters")
        arr = (ctypes.c_uint32 * n.value)()
        _lib.check(L.mk_read_counters(self._h, arr, n.value, ctypes.byref(n)), "mk_read_counters")
        return list(arr)


def greedy_select(logits: torch.Tensor, next_tokens: torch.Tensor, positions=None, stream=None) -> None:
    """next_tokens[b] = argmax of logits[b] (lowest index among equal maxima), on the
    device and asynchronous on ``stream``; ``positions`` (optional) is advanced by one."""
    assert logits.is_cuda and logits.dtype == torch.float32 and logits.is_contiguous() and logits.dim() == 2
    assert next_tokens.is_cuda and next_tokens.dtype == torch.int32 and next_tokens.numel() >= logits.shape[0]
    if positions is not None:
        assert positions.is_cuda and positions.dtype == torch.int32 and positions.numel() >= logits.shape[0]
    _lib.check(_lib.lib().mk_greedy_select(_ptr(logits), logits.shape[0], logits.shape[1], _ptr(next_tokens),
                                           _ptr(positions) if positions is not None else None,
                                           _stream(stream)), "mk_greedy_select")


def plan_schedule(cfg: ModelConfig, batch: int, max_ctx: int, n_sm: int, max_batch: int = 8,
                  max_seq: int | None = None, **opts):
    """Host-only schedule plan: (list of MkInstr, per-SM offsets, MkScheduleInfo)."""
    L = _lib.lib()
    c = _lib.make_config(cfg, max_batch, max_seq or max_ctx)
    o = _lib.make_opts(**opts) if opts else None
    info = _lib.MkScheduleInfo()
    po = ctypes.byref(o) if o is not None else None
    _lib.check(L.mk_plan_schedule_host(ctypes.byref(c), batch, max_ctx, n_sm, po, None, 0, None,
                                       ctypes.byref(info)), "plan")
    instrs = (_lib.MkInstr * info.n_instr)()
    offs = (ctypes.c_int32 * (n_sm + 1))()
    _lib.check(L.mk_plan_schedule_host(ctypes.byref(c), batch, max_ctx, n_sm, po, instrs,
                                       info.n_instr, offs, ctypes.byref(info)), "plan")
    return list(instrs), list(offs), info


def pack_weights_host(cfg: ModelConfig, weights, max_batch: int = 1, max_seq: int = 1):
    """Host packing (the same layout mk_create builds on the device): uint8 tensor."""
    L = _lib.lib()
    c = _lib.make_config(cfg, max_batch, max_seq)
    n = L.mk_packed_bytes(ctypes.byref(c))
    if n == 0:
        raise _lib.MkError(3, "mk_packed_bytes")
    w = weights
    keep = []

    def tab(ts):
        ts = [t.contiguous() for t in ts]
        keep.extend(ts)
        arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
        keep.append(arr)
        return ctypes.cast(arr, ctypes.c_void_p)

    mw = _lib.MkWeights(w.embed.data_ptr(), tab(w.attn_norm), tab(w.wq), tab(w.wk), tab(w.wv),
                        tab(w.wo), tab(w.mlp_norm), tab(w.wgate), tab(w.wup), tab(w.wdown),
                        w.final_norm.data_ptr())
    out = torch.empty(n, dtype=torch.uint8)
    _lib.check(L.mk_pack_weights_host(ctypes.byref(c), ctypes.byref(mw), out.data_ptr(), n),
               "mk_pack_weights_host")
    return out
