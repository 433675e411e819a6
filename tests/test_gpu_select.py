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
