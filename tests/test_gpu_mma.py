"""The tensor-core projections at batch > 1 (MK_PROJ_TENSOR_CORES, the default
there; MK_PROJ_CUDA_CORES selects the batched CUDA-core dot): every projection's weight rows stream as 64-column boxes into the ring
and one thread issues tcgen05.mma (128 weight rows x 16 input rows: each
sequence's fp32 input split into a bf16 high part and the bf16 rounding of the
remainder) into fp32 accumulators in Tensor Memory, read back for the fused
epilogues. Its accumulation order is the tensor cores', so it is held to the
oracle's bars (the pass line and the regression bar of the parity tests) rather
than to the CUDA-core path's bits; the two paths must also agree with each other
within the regression bar."""
import dataclasses

import numpy as np
import pytest

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import LLAMA_1B, TINY
from persistent_megakernel_interpreter_b200.inputs import make_tokens
from test_gpu_parity import Case, assert_kv_ok, assert_logits_close, reg_bar

pytestmark = pytest.mark.gpu


def _both_paths(c, batch, max_ctx, toks, pos):
    """Logits of one step on each path, from the same caches."""
    info = c.mk.build_schedule(batch, max_ctx, proj=_lib.PROJ_TENSOR_CORES)
    assert info.proj == _lib.PROJ_TENSOR_CORES
    tc = c.gpu_step(toks, pos)
    assert c.mk.status()[0] == 0, c.mk.status()
    c.reset_kv()
    info = c.mk.build_schedule(batch, max_ctx, proj=_lib.PROJ_CUDA_CORES)
    assert info.proj == _lib.PROJ_CUDA_CORES
    cc = c.gpu_step(toks, pos)
    assert c.mk.status()[0] == 0
    c.reset_kv()
    return tc, cc


def _paths_agree(tc, cc, positions):
    """Within the regression bar of each sequence's position (each path rounds the
    step's new key and value to bf16 from its own fp32 value)."""
    for b in range(tc.shape[0]):
        assert np.max(np.abs(tc[b] - cc[b])) <= reg_bar(positions[b]) * np.max(np.abs(cc[b])), b


@pytest.mark.parametrize("batch,past", [
    (2, [128, 57]), (3, [0, 1, 159]), (5, [7, 64, 100, 3, 150]), (8, [159, 0, 31, 32, 33, 120, 64, 1]),
])
def test_tiny_tensor_core_step_matches_oracle(batch, past):
    """Ragged positions (a single key, the last slot of the cache), odd batches (the
    operand's unused rows are never read), both warp halves of the sequences."""
    c = Case(TINY, batch=batch, max_seq=160, past=past, seed=70 + batch)
    toks = make_tokens(TINY, batch, seed=80 + batch).numpy()
    tc, cc = _both_paths(c, batch, 160, toks, past)
    ref, kc, vc = c.oracle_step(toks, past)
    assert_logits_close(tc, ref, past)
    _paths_agree(tc, cc, past)
    c.mk.build_schedule(batch, 160, proj=_lib.PROJ_TENSOR_CORES)
    c.gpu_step(toks, past)
    assert_kv_ok(c, kc, vc, past)
    c.mk.close()


def test_tiny_tensor_core_repeated_steps_identical():
    """The same step three times gives the same bits (a fixed order of MMAs and
    accumulators, whatever the timing)."""
    c = Case(TINY, batch=4, max_seq=160, past=[10, 20, 30, 40], seed=91)
    c.mk.build_schedule(4, 160, proj=_lib.PROJ_TENSOR_CORES)
    toks = make_tokens(TINY, 4, seed=92).numpy()
    outs = []
    for _ in range(3):
        c.reset_kv()
        outs.append(c.gpu_step(toks, [10, 20, 30, 40]))
    assert c.mk.status()[0] == 0
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
    c.mk.close()


def test_1b_shape_batch8_two_layers_tensor_core():
    """The 1B shape (head_dim 64, 4 query heads per KV head) cut to two layers at
    batch 8: the LM head's 128256 rows run as segments of 128 rows."""
    cfg = dataclasses.replace(LLAMA_1B, n_layers=2, name="1b-shape-2l")
    past = [128, 1, 77, 127, 0, 64, 100, 33]
    c = Case(cfg, batch=8, max_seq=129, past=past, seed=41)
    toks = make_tokens(cfg, 8, seed=42).numpy()
    tc, cc = _both_paths(c, 8, 129, toks, past)
    ref, kc, vc = c.oracle_step(toks, past)
    assert_logits_close(tc, ref, past)
    _paths_agree(tc, cc, past)
    c.mk.close()


def test_tensor_core_schedule_options_do_not_change_results():
    """Fewer SMs, a shuffled placement, smaller down-projection instructions: each
    row's accumulation runs over the same K boxes in the same order, so the bits
    stay the same."""
    c = Case(TINY, batch=3, max_seq=160, past=[100, 37, 5], seed=93)
    toks = make_tokens(TINY, 3, seed=94).numpy()
    info = c.mk.build_schedule(3, 160, proj=_lib.PROJ_TENSOR_CORES)
    ref = c.gpu_step(toks, [100, 37, 5])
    for opts in (dict(n_sm=37), dict(seed=5), dict(n_sm=5, rowblocks_down=1), dict(rowblocks_down=3)):
        c.reset_kv()
        c.mk.build_schedule(3, 160, part_keys=info.part_keys, proj=_lib.PROJ_TENSOR_CORES, **opts)
        assert np.array_equal(c.gpu_step(toks, [100, 37, 5]), ref), opts
    assert c.mk.status()[0] == 0
    c.mk.close()
