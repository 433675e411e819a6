"""Parity of the CUDA path (called through the C ABI) with the CPU oracle, plus
the integer/protocol properties that must hold bit for bit.

Tolerance (stated in the decode-step target): max |logit_gpu - logit_oracle|
<= 1e-2 * max |logit_oracle| per step, and greedy argmax agreement. A second,
tighter bar catches regressions the pass line would let through (one wrong head,
a dropped residual row): 1e-4 * max |logit_oracle| for a sequence with many keys
(fp32 arithmetic in two summation orders; measured about 2e-5 on the 1B step at
128 positions). A sequence with few keys gets 2^-7 / (position + 1) instead when
that is larger: the step's own key and value are rounded to bf16 on each side,
and where the fp32 values sit near a rounding boundary the two roundings differ by
one ulp (2^-8 relative); that key weighs up to 1 / (position + 1) in the softmax
(measured: 6e-4 with 2 keys on the 3B-style shape). Greedy decoding from an
empty cache attends over the model's own keys, where that weight can reach 1: each
step is held to 2^-8 there and the median step to 1e-4 (measured: 1.5e-4 at 99
keys on the 1B shape). The new key and value
themselves are within one bf16 ulp at the scale of their head (the largest
magnitude of the head's row): RoPE's a*c - b*s and the value's dot product can
cancel, so a small element's own ulp is no bound. Integer work is exact:
untouched KV slots, counters, token ids."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B, TINY
from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights

pytestmark = pytest.mark.gpu

TOL = 1e-2   # pass line
REG = 1e-4   # regression bar


def _bits(t):
    return oracle.bits(t.cpu()).copy()


class Case:
    """One model on the GPU and on the oracle, with a KV cache on each side."""

    def __init__(self, cfg, batch, max_seq, past, seed=0, norm_jitter=0.0, weights=None):
        from persistent_megakernel_interpreter_b200.model import Megakernel
        self.cfg, self.batch, self.max_seq = cfg, batch, max_seq
        w = weights or make_weights(cfg, seed=seed, norm_jitter=norm_jitter)
        self.orc = oracle.Model(cfg, w)
        self.k, self.v = make_kv_cache(cfg, batch, max_seq, past, seed=seed + 1)
        dev = w.to("cuda")
        self.mk = Megakernel(cfg, dev, max_batch=batch, max_seq=max_seq)
        del dev
        self.kd, self.vd = self.k.cuda(), self.v.cuda()
        self.logits = torch.empty(batch, cfg.vocab, dtype=torch.float32, device="cuda")

    def reset_kv(self):
        """Restore the GPU caches to the generated contents (earlier steps wrote slots)."""
        self.kd.copy_(self.k)
        self.vd.copy_(self.v)
        torch.cuda.synchronize()

    def gpu_step(self, tokens, positions, baseline=False):
        t = torch.as_tensor(np.asarray(tokens), dtype=torch.int32).cuda()
        p = torch.as_tensor(np.asarray(positions), dtype=torch.int32).cuda()
        fn = self.mk.baseline_decode_step if baseline else self.mk.decode_step
        fn(t, p, self.kd, self.vd, self.logits)
        torch.cuda.synchronize()
        return self.logits.cpu().numpy().copy()

    def oracle_step(self, tokens, positions, kc=None, vc=None):
        kc = _bits(self.k) if kc is None else kc
        vc = _bits(self.v) if vc is None else vc
        return self.orc.decode_step(np.asarray(tokens), np.asarray(positions), kc, vc), kc, vc


def reg_bar(position, floor=REG):
    """The regression bar of a sequence decoding at `position` (see the module notes)."""
    return max(floor, 2.0 ** -7 / (int(position) + 1))


def assert_logits_close(gpu, ref, positions=None, floor=REG):
    for b in range(ref.shape[0]):
        err = np.max(np.abs(gpu[b] - ref[b]))
        top = np.max(np.abs(ref[b]))
        assert err <= TOL * top, (b, err, top)
        bar = reg_bar(positions[b], floor) if positions is not None else floor
        assert err <= bar * top, ("regression bar", b, err / top, bar)
        assert int(np.argmax(gpu[b])) == int(np.argmax(ref[b]))


def bf16_ulp(x):
    """The spacing of bf16 values at |x| (8 significant bits); the smallest normal's
    at 0."""
    a = np.maximum(np.abs(x), np.float64(2.0 ** -126))
    return np.exp2(np.floor(np.log2(a)) - 7)


def assert_slot_close(kg, vg, kc_ref, vc_ref, b, p):
    """Slot p of sequence b (bf16 bits, [layer][seq][kv head][slot][dim]) within one
    bf16 ulp of the oracle's at the scale of each head row."""
    for got, ref in ((kg, kc_ref), (vg, vc_ref)):
        g = oracle.bf16_to_f32(got[:, b, :, p]).astype(np.float64)  # [layer][kv head][dim]
        r = oracle.bf16_to_f32(ref[:, b, :, p]).astype(np.float64)
        scale = bf16_ulp(np.max(np.abs(r), axis=-1, keepdims=True))
        assert np.all(np.abs(g - r) <= scale), np.max(np.abs(g - r) / scale)


def greedy_teacher_forced(c, prompt, steps):
    """Greedy decoding at batch 1 from an empty cache: the prompt's tokens, then the
    GPU's argmax. Every step the oracle decodes the GPU's token from the GPU's own
    cache as it stood before the step (teacher forcing on tokens and cache), so the
    two differ only by the step's arithmetic: the logits are held to the single-step
    bars, with one difference: the cache here is the model's own, whose attention
    can rest on a few keys, so the step's own key and value (rounded to bf16 on
    each side, one ulp apart where the fp32 value sits near a rounding boundary)
    can carry up to all of a head's softmax weight. A step is held to one bf16 ulp
    (2^-8) relative, and the median step to the regression bar. The written slot is
    within one ulp at its head's scale. Returns the number of steps whose argmaxes
    agree."""
    tok, agree, errs = int(prompt[0]), 0, []
    for p in range(steps):
        kc, vc = _bits(c.kd), _bits(c.vd)
        gpu = c.gpu_step([tok], [p])
        ref, kc, vc = c.oracle_step([tok], [p], kc, vc)
        err = np.max(np.abs(gpu[0] - ref[0])) / np.max(np.abs(ref[0]))
        errs.append(err)
        assert err <= TOL and err <= 2.0 ** -8, (p, err)
        assert_slot_close(_bits(c.kd), _bits(c.vd), kc, vc, 0, p)
        agree += int(np.argmax(gpu[0]) == np.argmax(ref[0]))
        tok = int(prompt[p + 1]) if p + 1 < len(prompt) else int(np.argmax(gpu[0]))
    assert c.mk.status()[0] == 0
    print(f"greedy: max relative error {max(errs):.3g}, median {np.median(errs):.3g} over {steps} steps")
    assert np.median(errs) <= REG, np.median(errs)
    return agree


def assert_kv_ok(case, kc_ref, vc_ref, positions):
    """New slots close to the oracle's; every other slot bit-identical to before."""
    kg, vg = _bits(case.kd), _bits(case.vd)
    k0, v0 = _bits(case.k), _bits(case.v)
    for b, p in enumerate(positions):
        mask = np.ones(case.max_seq, bool)
        mask[p] = False
        assert np.array_equal(kg[:, b][:, :, mask], k0[:, b][:, :, mask])
        assert np.array_equal(vg[:, b][:, :, mask], v0[:, b][:, :, mask])
        assert_slot_close(kg, vg, kc_ref, vc_ref, b, p)


@pytest.fixture(scope="module")
def tiny_case():
    c = Case(TINY, batch=2, max_seq=160, past=[128, 57])
    c.mk.build_schedule(batch=2, max_ctx=160)
    yield c
    c.mk.close()


@pytest.fixture
def tiny(tiny_case):
    tiny_case.reset_kv()
    return tiny_case


def test_tiny_step_matches_oracle(tiny):
    toks = make_tokens(TINY, 2, seed=2).numpy()
    pos = [128, 57]
    gpu = tiny.gpu_step(toks, pos)
    code, msg = tiny.mk.status()
    assert code == 0, msg
    ref, kc, vc = tiny.oracle_step(toks, pos)
    assert_logits_close(gpu, ref, pos)
    assert_kv_ok(tiny, kc, vc, pos)


def test_megakernel_equals_baseline_bit_for_bit(tiny):
    """The megakernel on the CUDA cores and the multi-kernel baseline share every
    order of arithmetic (the tensor-core path accumulates in its own order: it is
    held to the oracle instead, test_gpu_mma.py)."""
    toks = make_tokens(TINY, 2, seed=3).numpy()
    pos = [100, 3]
    tiny.mk.build_schedule(2, 160, proj=1)
    a = tiny.gpu_step(toks, pos)
    ka, va = _bits(tiny.kd), _bits(tiny.vd)
    b = tiny.gpu_step(toks, pos, baseline=True)
    tiny.mk.build_schedule(2, 160)
    assert tiny.mk.status()[0] == 0
    assert np.array_equal(a, b)
    assert np.array_equal(ka, _bits(tiny.kd)) and np.array_equal(va, _bits(tiny.vd))


def test_repeated_steps_are_identical_and_counters_exact(tiny):
    toks = make_tokens(TINY, 2, seed=4).numpy()
    pos = [128, 57]
    tiny.gpu_step(toks, pos)
    base = tiny.mk.counters()
    outs = [tiny.gpu_step(toks, pos) for _ in range(3)]
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
    after = tiny.mk.counters()
    n = len(after) - 2
    epoch0, epoch1 = base[n], after[n]
    assert epoch1 == epoch0 + 3 and after[n + 1] == 0
    for c in range(n):  # every counter advanced by exactly 3 steps' worth of signals
        per_step = base[c] // epoch0 if epoch0 else None
        assert after[c] == per_step * epoch1


def test_schedule_placement_does_not_change_results(tiny):
    toks = make_tokens(TINY, 2, seed=5).numpy()
    pos = [128, 57]
    info = tiny.mk.schedule_info()
    ref = tiny.gpu_step(toks, pos)
    for opts in (dict(n_sm=37), dict(seed=99), dict(n_sm=5), dict(n_sm=5, seed=7, rowblocks_down=1),
                 dict(rowblocks_down=3)):
        tiny.mk.build_schedule(2, 160, part_keys=info.part_keys, **opts)
        assert np.array_equal(tiny.gpu_step(toks, pos), ref), opts
    tiny.mk.build_schedule(2, 160)


def test_split_k_partitions_agree_with_oracle(tiny):
    """Any partition size gives the oracle's logits (the merge is exact up to rounding)."""
    toks = make_tokens(TINY, 2, seed=6).numpy()
    pos = [150, 20]
    ref, _, _ = tiny.oracle_step(toks, pos)
    kps = tiny.mk.schedule_info().keys_per_stage
    for pk in (kps, 2 * kps, 160 // kps * kps + kps):
        tiny.mk.build_schedule(2, 160, part_keys=pk)
        tiny.reset_kv()
        assert_logits_close(tiny.gpu_step(toks, pos), ref, pos)
    tiny.mk.build_schedule(2, 160)


def test_host_buffer_entry_point(tiny):
    toks = make_tokens(TINY, 2, seed=7).numpy()
    pos = [128, 57]
    dev = tiny.gpu_step(toks, pos)
    th = torch.as_tensor(toks, dtype=torch.int32).pin_memory()
    ph = torch.as_tensor(pos, dtype=torch.int32).pin_memory()
    out = torch.empty(2, TINY.vocab, dtype=torch.float32).pin_memory()
    tiny.mk.decode_step_host(th, ph, tiny.kd, tiny.vd, out)
    assert np.array_equal(out.numpy(), dev)


def test_bad_token_and_position_are_reported_and_write_nothing(tiny):
    kb, vb = _bits(tiny.kd), _bits(tiny.vd)
    for baseline in (False, True):
        tiny.gpu_step([TINY.vocab, 1], [10, 10], baseline=baseline)
        code, msg = tiny.mk.status()
        assert code == 6, msg
        tiny.gpu_step([1, 2], [10, 160], baseline=baseline)
        code, msg = tiny.mk.status()
        assert code == 7, msg
    assert np.array_equal(kb, _bits(tiny.kd)) and np.array_equal(vb, _bits(tiny.vd))
    # the handle keeps working
    tiny.reset_kv()
    toks, pos = make_tokens(TINY, 2, seed=8).numpy(), [128, 57]
    ref, _, _ = tiny.oracle_step(toks, pos)
    assert_logits_close(tiny.gpu_step(toks, pos), ref, pos)
    assert tiny.mk.status()[0] == 0


def test_wait_timeout_is_reported_without_hanging(tiny):
    """A schedule missing one producer (host-side injection): the waits give up
    after their budget, the step reports MK_ERR_TIMEOUT, and the next step runs."""
    tiny.mk.build_schedule(2, 160, test_drop_item=3, wait_timeout_ms=200)
    tiny.gpu_step([1, 2], [5, 6])
    code, msg = tiny.mk.status()
    assert code == 5, msg
    counters = tiny.mk.counters()
    assert all(c == 0 for c in counters)  # reset by the last CTA of the failed step
    tiny.mk.build_schedule(2, 160)
    tiny.reset_kv()
    toks, pos = make_tokens(TINY, 2, seed=9).numpy(), [128, 57]
    ref, _, _ = tiny.oracle_step(toks, pos)
    assert_logits_close(tiny.gpu_step(toks, pos), ref, pos)
    assert tiny.mk.status()[0] == 0


def test_tiny_greedy_decode_teacher_forced():
    """32-token prompt from an empty cache, then greedy decoding (greedy_teacher_forced);
    the argmax agrees on every step."""
    c = Case(TINY, batch=1, max_seq=64, past=0, seed=11)
    c.mk.build_schedule(1, 64)
    prompt = make_tokens(TINY, 32, seed=12).numpy()
    assert greedy_teacher_forced(c, prompt, 56) >= 0.99 * 56
    c.mk.close()


def test_tiny_with_non_unit_norm_weights():
    c = Case(TINY, batch=1, max_seq=140, past=130, seed=21, norm_jitter=0.1)
    c.mk.build_schedule(1, 140)
    toks, pos = make_tokens(TINY, 1, seed=22).numpy(), [130]
    ref, kc, vc = c.oracle_step(toks, pos)
    assert_logits_close(c.gpu_step(toks, pos), ref, pos)
    assert_kv_ok(c, kc, vc, pos)
    c.mk.close()


def test_3b_shape_batch8_two_layers():
    """The 3B-style shape (hidden 3072, head_dim 128, 3 query heads per KV head) at
    batch 8 with ragged positions, cut to two layers so the oracle stays quick."""
    cfg = dataclasses.replace(LLAMA_3B, n_layers=2, name="3b-shape-2l")
    past = [2048, 1, 700, 2047, 0, 64, 1500, 333]
    c = Case(cfg, batch=8, max_seq=2049, past=past, seed=31)
    c.mk.build_schedule(8, 2049, proj=2)  # the tensor-core path first
    toks = make_tokens(cfg, 8, seed=32).numpy()
    ref, kc, vc = c.oracle_step(toks, past)
    gpu = c.gpu_step(toks, past)
    assert c.mk.status()[0] == 0
    assert_logits_close(gpu, ref, past)
    assert_kv_ok(c, kc, vc, past)
    # the CUDA-core path: the oracle's bars too, and the baseline's bits
    c.reset_kv()
    c.mk.build_schedule(8, 2049, proj=1)
    cc = c.gpu_step(toks, past)
    assert c.mk.status()[0] == 0
    assert_logits_close(cc, ref, past)
    c.reset_kv()
    assert np.array_equal(c.gpu_step(toks, past, baseline=True), cc)
    c.mk.close()


@pytest.fixture(scope="module")
def llama1b_case():
    c = Case(LLAMA_1B, batch=1, max_seq=129, past=128, seed=0)
    c.mk.build_schedule(1, 129)
    yield c
    c.mk.close()


@pytest.fixture
def llama1b(llama1b_case):
    llama1b_case.reset_kv()
    return llama1b_case


def test_llama1b_step_matches_oracle(llama1b):
    """The benchmark's workload and launch configuration (148 SMs, ctx 128)."""
    toks, pos = make_tokens(LLAMA_1B, 1, seed=2).numpy(), [128]
    gpu = llama1b.gpu_step(toks, pos)
    assert llama1b.mk.status()[0] == 0
    ref, kc, vc = llama1b.oracle_step(toks, pos)
    assert_logits_close(gpu, ref, pos)
    assert_kv_ok(llama1b, kc, vc, pos)


def test_llama1b_megakernel_equals_baseline(llama1b):
    toks, pos = make_tokens(LLAMA_1B, 1, seed=3).numpy(), [128]
    a = llama1b.gpu_step(toks, pos)
    b = llama1b.gpu_step(toks, pos, baseline=True)
    assert np.array_equal(a, b)
