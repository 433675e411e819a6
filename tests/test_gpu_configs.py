"""Parity of the megakernel with the CPU oracle on the full-size workloads beyond
the single 128-position step: the Llama-1B shape over long contexts (where the
attention is split into several key partitions per KV group and merged), a
greedy decode of 256 tokens after a 32-token prompt with the cache growing
step by step, and the 3B-style shape at batch 8 with 2048-position caches.

Tolerance as in the other parity tests: max |logit_gpu - logit_oracle| <=
1e-2 * max |logit_oracle| per sequence and step, argmax agreement (on at least
99% of the greedy steps, teacher-forced), and the KV slots each step writes
within the same bound while every other slot stays bit-identical."""
import numpy as np
import pytest

from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B
from persistent_megakernel_interpreter_b200.inputs import make_tokens, make_weights

from test_gpu_parity import Case, assert_kv_ok, assert_logits_close, greedy_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w1b():
    return make_weights(LLAMA_1B, seed=0)


def test_llama1b_long_contexts(w1b):
    """1B at 1024 / 4096 / 8192 cached positions: several key partitions per
    (sequence, KV group), each finished by the merge of the last arriving item."""
    c = Case(LLAMA_1B, batch=1, max_seq=8193, past=8192, seed=0, weights=w1b)
    for past in (1024, 4096, 8192):
        c.reset_kv()
        info = c.mk.build_schedule(1, past + 1)
        assert info.n_parts > 1
        toks, pos = make_tokens(LLAMA_1B, 1, seed=40 + past).numpy(), [past]
        gpu = c.gpu_step(toks, pos)
        assert c.mk.status()[0] == 0
        ref, kc, vc = c.oracle_step(toks, pos)
        assert_logits_close(gpu, ref, pos)
        assert_kv_ok(c, kc, vc, pos)
    c.mk.close()


def test_llama1b_greedy_256_after_32_token_prompt(w1b):
    """A 32-token random prompt fed as decode steps into an empty cache, then 256
    greedy tokens, the oracle teacher-forced on the GPU's tokens and cache
    (greedy_teacher_forced): the argmax agrees on at least 99% of the steps."""
    n_prompt, n_gen = 32, 256
    steps = n_prompt + n_gen
    c = Case(LLAMA_1B, batch=1, max_seq=steps, past=0, seed=0, weights=w1b)
    c.mk.build_schedule(1, steps)
    prompt = make_tokens(LLAMA_1B, n_prompt, seed=50).numpy()
    assert greedy_teacher_forced(c, prompt, steps) >= 0.99 * steps
    c.mk.close()


def test_3b_shape_batch8_full_depth():
    """All 28 layers of the 3B-style shape at batch 8, every sequence with 2048
    cached positions, on the tensor-core path (the default) and the CUDA-core path
    against the oracle; the CUDA-core megakernel and the multi-kernel baseline agree
    bit for bit."""
    past = [2048] * 8
    c = Case(LLAMA_3B, batch=8, max_seq=2049, past=past, seed=60)
    c.mk.build_schedule(8, 2049, proj=2)  # the tensor-core path first
    toks = make_tokens(LLAMA_3B, 8, seed=61).numpy()
    gpu = c.gpu_step(toks, past)
    assert c.mk.status()[0] == 0
    ref, kc, vc = c.oracle_step(toks, past)
    assert_logits_close(gpu, ref, past)
    assert_kv_ok(c, kc, vc, past)
    # the CUDA-core path: within the same bars, and bit for bit the baseline's
    c.reset_kv()
    c.mk.build_schedule(8, 2049, proj=1)
    cc = c.gpu_step(toks, past)
    assert c.mk.status()[0] == 0
    assert_logits_close(cc, ref, past)
    c.reset_kv()
    assert np.array_equal(c.gpu_step(toks, past, baseline=True), cc)
    c.mk.close()
