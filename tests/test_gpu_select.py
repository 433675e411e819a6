"""Greedy selection on the device (mk_greedy_select) and a decode loop that never
returns to the host between steps.

The selection is integer work on given fp32 logits, so it is checked exactly:
the chosen id must be the lowest index of the row's maximum (numpy's nanargmax,
with a row of NaNs giving 0), for ragged vocabularies, rows that start off a
16-byte boundary, planted ties, -inf rows and NaN entries."""
import numpy as np
import pytest
import torch

from persistent_megakernel_interpreter_b200.config import TINY
from persistent_megakernel_interpreter_b200.inputs import make_tokens
from persistent_megakernel_interpreter_b200.model import greedy_select

from test_gpu_parity import TOL, Case, _bits

pytestmark = pytest.mark.gpu


def expected(x: np.ndarray) -> np.ndarray:
    out = np.zeros(x.shape[0], dtype=np.int32)
    for b, row in enumerate(x):
        if not np.all(np.isnan(row)):
            out[b] = int(np.nanargmax(row))
    return out


def planted_logits(batch: int, vocab: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, vocab)).astype(np.float32)
    if vocab >= 3:
        j = rng.choice(vocab, size=2, replace=False)
        x[1, j] = 9.0                                      # a tie: the lower index wins
        x[2, :] = -np.inf                                  # every entry -inf: index 0
        x[3, rng.choice(vocab, size=max(1, vocab // 10), replace=False)] = np.nan
        x[3, vocab // 2] = 7.0                             # NaNs beside the maximum
        x[4, :] = np.nan                                   # nothing selectable: 0
        x[5, -1] = 8.0                                     # the maximum in the ragged tail
    return x


@pytest.mark.parametrize("vocab", [1, 7, 1001, 4096, 128256])
@pytest.mark.parametrize("offset", [0, 1, 3])
def test_greedy_select_is_the_lowest_index_of_the_maximum(vocab, offset):
    batch = 6
    x = planted_logits(batch, vocab, seed=vocab + offset)
    buf = torch.full((batch * vocab + 4,), float("nan"), dtype=torch.float32, device="cuda")
    logits = buf[offset:offset + batch * vocab].view(batch, vocab)
    logits.copy_(torch.from_numpy(x))
    tok = torch.full((batch,), -1, dtype=torch.int32, device="cuda")
    pos = torch.arange(batch, dtype=torch.int32, device="cuda") * 5
    greedy_select(logits, tok, pos)
    torch.cuda.synchronize()
    assert np.array_equal(tok.cpu().numpy(), expected(x))
    assert np.array_equal(pos.cpu().numpy(), np.arange(batch) * 5 + 1)
    greedy_select(logits, tok)                              # without positions
    torch.cuda.synchronize()
    assert np.array_equal(tok.cpu().numpy(), expected(x))


def test_decode_loop_selects_on_the_device():
    """TINY, two sequences from an empty cache, 24 steps of decode_step followed by
    greedy_select into the same token and position buffers. Each chosen id equals
    the argmax of that step's logits exactly; the logits follow the oracle fed the
    same tokens within the decode-step tolerance, and where the argmaxes differ the
    oracle's top two are within that tolerance of each other."""
    batch, steps = 2, 24
    c = Case(TINY, batch=batch, max_seq=steps, past=0, seed=70)
    c.mk.build_schedule(batch, steps)
    tok = make_tokens(TINY, batch, seed=71).to(torch.int32).cuda()
    pos = torch.zeros(batch, dtype=torch.int32, device="cuda")
    hist_logits = torch.empty(steps, batch, TINY.vocab, dtype=torch.float32, device="cuda")
    hist_tok = torch.empty(steps + 1, batch, dtype=torch.int32, device="cuda")
    hist_tok[0].copy_(tok)
    for p in range(steps):
        c.mk.decode_step(tok, pos, c.kd, c.vd, c.logits)
        hist_logits[p].copy_(c.logits)
        greedy_select(c.logits, tok, pos)
        hist_tok[p + 1].copy_(tok)
    torch.cuda.synchronize()
    assert c.mk.status()[0] == 0
    assert np.array_equal(pos.cpu().numpy(), [steps] * batch)
    lg, tk = hist_logits.cpu().numpy(), hist_tok.cpu().numpy()
    kc, vc = _bits(c.k), _bits(c.v)
    for p in range(steps):
        assert np.array_equal(tk[p + 1], np.argmax(lg[p], axis=1))
        ref, kc, vc = c.oracle_step(tk[p], [p] * batch, kc, vc)
        for b in range(batch):
            scale = np.max(np.abs(ref[b]))
            assert np.max(np.abs(lg[p, b] - ref[b])) <= TOL * scale, (p, b)
            if tk[p + 1, b] != np.argmax(ref[b]):
                top2 = np.sort(ref[b])[-2:]
                assert top2[1] - top2[0] <= 2 * TOL * scale, (p, b)
    c.mk.close()


@pytest.mark.parametrize("batch", [1, 3])
def test_fused_greedy_steps_equal_select_between_steps(batch):
    """mk_decode_steps_greedy (the choice fused into each step's LM head, N launches
    with no host work) against mk_decode_step + mk_greedy_select per step on a
    copy of the same caches: the same tokens at every step, the same positions,
    the last step's logits bit for bit, and identical caches. Batch 3 runs the
    batched kernel (its LM-head rows shared by two warps per tile)."""
    n = 24
    c = Case(TINY, batch=batch, max_seq=64, past=0, seed=5)
    c.mk.build_schedule(batch, 64)
    k2, v2 = c.kd.clone(), c.vd.clone()
    t0 = torch.as_tensor(make_tokens(TINY, batch, seed=6).numpy(), dtype=torch.int32).cuda()
    # the fused loop
    tok_f, pos_f = t0.clone(), torch.zeros(batch, dtype=torch.int32, device="cuda")
    gen = torch.full((n, batch), -1, dtype=torch.int32, device="cuda")
    logits_f = torch.empty(batch, TINY.vocab, dtype=torch.float32, device="cuda")
    c.mk.decode_steps_greedy(tok_f, pos_f, c.kd, c.vd, logits_f, n, generated=gen)
    torch.cuda.synchronize()
    assert c.mk.status()[0] == 0
    # the step-by-step loop with the separate selection kernel
    tok_s, pos_s = t0.clone(), torch.zeros(batch, dtype=torch.int32, device="cuda")
    logits_s = torch.empty(batch, TINY.vocab, dtype=torch.float32, device="cuda")
    seq = []
    for _ in range(n):
        c.mk.decode_step(tok_s, pos_s, k2, v2, logits_s)
        greedy_select(logits_s, tok_s, pos_s)
        seq.append(tok_s.clone())
    torch.cuda.synchronize()
    assert np.array_equal(gen.cpu().numpy(), torch.stack(seq).cpu().numpy())
    assert np.array_equal(tok_f.cpu().numpy(), tok_s.cpu().numpy())
    assert np.array_equal(pos_f.cpu().numpy(), np.full(batch, n))
    assert np.array_equal(logits_f.cpu().numpy(), logits_s.cpu().numpy())
    assert np.array_equal(_bits(c.kd), _bits(k2)) and np.array_equal(_bits(c.vd), _bits(v2))
    c.mk.close()


def test_fused_greedy_steps_1b():
    """The same equality on the Llama-3.2-1B shape for 6 steps from 128 cached
    positions (the LM head spread over every SM)."""
    from persistent_megakernel_interpreter_b200.config import LLAMA_1B
    n = 6
    c = Case(LLAMA_1B, batch=1, max_seq=136, past=128, seed=0)
    c.mk.build_schedule(1, 136)
    k2, v2 = c.kd.clone(), c.vd.clone()
    t0 = torch.as_tensor(make_tokens(LLAMA_1B, 1, seed=2).numpy(), dtype=torch.int32).cuda()
    tok_f, pos_f = t0.clone(), torch.full((1,), 128, dtype=torch.int32, device="cuda")
    gen = torch.full((n, 1), -1, dtype=torch.int32, device="cuda")
    logits_f = torch.empty(1, LLAMA_1B.vocab, dtype=torch.float32, device="cuda")
    c.mk.decode_steps_greedy(tok_f, pos_f, c.kd, c.vd, logits_f, n, generated=gen)
    tok_s, pos_s = t0.clone(), torch.full((1,), 128, dtype=torch.int32, device="cuda")
    logits_s = torch.empty(1, LLAMA_1B.vocab, dtype=torch.float32, device="cuda")
    seq = []
    for _ in range(n):
        c.mk.decode_step(tok_s, pos_s, k2, v2, logits_s)
        greedy_select(logits_s, tok_s, pos_s)
        seq.append(tok_s.clone())
    torch.cuda.synchronize()
    assert c.mk.status()[0] == 0
    assert np.array_equal(gen.cpu().numpy(), torch.stack(seq).cpu().numpy())
    assert int(pos_f.item()) == 128 + n
    assert np.array_equal(logits_f.cpu().numpy(), logits_s.cpu().numpy())
    c.mk.close()
