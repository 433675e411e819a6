"""ctypes declarations for libmk.so (the C ABI in include/mk.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels. Loading fails loudly when the library is missing; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

P = ctypes.c_void_p
I32 = ctypes.c_int32


class MkConfig(ctypes.Structure):
    _fields_ = [("n_layers", I32), ("hidden", I32), ("n_heads", I32), ("n_kv_heads", I32),
                ("head_dim", I32), ("ffn", I32), ("vocab", I32), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_double), ("max_batch", I32), ("max_seq", I32)]


class MkWeights(ctypes.Structure):
    _fields_ = [(n, P) for n in ("embed", "attn_norm", "wq", "wk", "wv", "wo", "mlp_norm",
                                 "wgate", "wup", "wdown", "final_norm")]


class MkScheduleOpts(ctypes.Structure):
    _fields_ = [("n_sm", I32), ("part_keys", I32), ("rowblocks_down", I32),
                ("seed", ctypes.c_uint32), ("wait_timeout_ms", I32), ("test_drop_item", I32),
                ("trace", I32), ("proj", I32)]


class MkInstr(ctypes.Structure):
    _fields_ = [("op", ctypes.c_uint16), ("layer", ctypes.c_uint16), ("batch", ctypes.c_uint16),
                ("group", ctypes.c_uint16)] + [(n, ctypes.c_uint32) for n in (
                    "first", "count", "seq", "nfill", "wait_ctr", "wait_n", "signal_ctr",
                    "job_items", "aux0", "aux1")]


class MkScheduleInfo(ctypes.Structure):
    _fields_ = [(n, I32) for n in ("n_sm", "batch", "max_ctx", "part_keys", "n_parts",
                                   "keys_per_stage", "stage_bytes", "n_stages", "n_counters",
                                   "n_instr")] + [
        ("bytes_per_step", ctypes.c_uint64), ("max_sm_bytes", ctypes.c_uint64),
        ("min_sm_bytes", ctypes.c_uint64), ("proj", I32), ("reserved0", I32)]


class MkTmapSpec(ctypes.Structure):
    _fields_ = [("index", I32), ("rank", I32), ("base_offset", ctypes.c_uint64),
                ("dims", ctypes.c_uint64 * 5), ("strides", ctypes.c_uint64 * 4), ("box", ctypes.c_uint32 * 5)]


OP_QKV, OP_ATTN, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LMHEAD = 1, 2, 3, 4, 5, 6
PROJ_AUTO, PROJ_CUDA_CORES, PROJ_TENSOR_CORES = 0, 1, 2
NO_COUNTER = 0xFFFFFFFF

STATUS = {0: "MK_OK", 1: "MK_ERR_INVALID_ARG", 2: "MK_ERR_CUDA", 3: "MK_ERR_UNSUPPORTED",
          4: "MK_ERR_NO_SCHEDULE", 5: "MK_ERR_TIMEOUT", 6: "MK_ERR_BAD_TOKEN",
          7: "MK_ERR_BAD_POSITION", 8: "MK_ERR_OUT_OF_MEMORY"}


class MkError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmk.so (raises if it was not built: run the package's build first)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m persistent_megakernel_interpreter_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    st = ctypes.c_int
    L.mk_create.argtypes = [ctypes.POINTER(MkConfig), ctypes.POINTER(MkWeights), ctypes.c_int,
                            ctypes.POINTER(P)]
    L.mk_build_schedule.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.POINTER(MkScheduleOpts)]
    step = [P, P, P, P, P, P, P]
    L.mk_decode_step.argtypes = step
    L.mk_baseline_decode_step.argtypes = step
    L.mk_decode_step_host.argtypes = step
    L.mk_get_status.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.c_char_p, ctypes.c_size_t]
    L.mk_destroy.argtypes = [P]
    L.mk_destroy.restype = None
    L.mk_status_str.argtypes = [ctypes.c_int]
    L.mk_status_str.restype = ctypes.c_char_p
    L.mk_plan_schedule_host.argtypes = [ctypes.POINTER(MkConfig), ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.POINTER(MkScheduleOpts),
                                        ctypes.POINTER(MkInstr), ctypes.c_size_t,
                                        ctypes.POINTER(I32), ctypes.POINTER(MkScheduleInfo)]
    L.mk_get_schedule_info.argtypes = [P, ctypes.POINTER(MkScheduleInfo)]
    L.mk_read_counters.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_size_t,
                                   ctypes.POINTER(ctypes.c_size_t)]
    L.mk_read_trace.argtypes = [P, P, ctypes.c_size_t, ctypes.POINTER(I32)]
    L.mk_packed_bytes.argtypes = [ctypes.POINTER(MkConfig)]
    L.mk_packed_bytes.restype = ctypes.c_size_t
    L.mk_pack_weights_host.argtypes = [ctypes.POINTER(MkConfig), ctypes.POINTER(MkWeights), P,
                                       ctypes.c_size_t]
    L.mk_baseline_decode_step_noalloc.argtypes = [ctypes.POINTER(MkConfig), P, P, P, P, P, P, ctypes.c_int,
                                                  ctypes.c_int, P, P]
    L.mk_greedy_select.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P]
    L.mk_decode_steps_greedy.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P]
    L.mk_tensor_map_specs_host.argtypes = [ctypes.POINTER(MkConfig), ctypes.c_uint32, ctypes.POINTER(MkTmapSpec),
                                           ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]
    for f in ("mk_create", "mk_build_schedule", "mk_decode_step", "mk_decode_steps_greedy", "mk_baseline_decode_step",
              "mk_decode_step_host", "mk_get_status", "mk_plan_schedule_host",
              "mk_get_schedule_info", "mk_read_counters", "mk_pack_weights_host", "mk_read_trace",
              "mk_baseline_decode_step_noalloc", "mk_greedy_select", "mk_tensor_map_specs_host"):
        getattr(L, f).restype = st
    _lib = L
    return L


def check(code: int, what: str) -> None:
    if code != 0:
        raise MkError(code, what)


def make_config(cfg, max_batch: int, max_seq: int) -> MkConfig:
    return MkConfig(cfg.n_layers, cfg.hidden, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn,
                    cfg.vocab, cfg.rms_eps, cfg.rope_theta, max_batch, max_seq)


def make_opts(**kw) -> MkScheduleOpts:
    o = MkScheduleOpts()
    for k, v in kw.items():
        setattr(o, k, v)
    return o
