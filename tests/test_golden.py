"""The oracle against its stored decode step (tests/golden/tiny_decode.txt).

The fixture is written by tests/golden/make_golden.py from the oracle alone; it
guards the oracle's arithmetic against silent change (a change to it, or to the
fixture, names in its commit message the passage that justifies it). The same
step on every host thread count must give the same bits: each output row is
summed in one fixed order whatever the threading."""
import numpy as np

import oracle
from golden import make_golden as mg


def test_oracle_reproduces_the_stored_step():
    want = mg.read()
    toks, logits, kslot, vslot = mg.compute()
    assert [int(t) for t in want["tokens"]] == [int(t) for t in toks]
    assert [int(p) for p in want["positions"]] == mg.PAST
    for b in range(len(mg.PAST)):
        head = want[(b, "argmax")]
        assert int(head[0]) == int(np.argmax(logits[b]))
        max_abs = float(head[2])
        assert abs(float(np.max(np.abs(logits[b]))) - max_abs) <= 1e-6 * max_abs
        assert abs(float(np.sum(logits[b].astype(np.float64))) - float(head[4])) <= 1e-5 * max_abs
        stored = np.array([float(x) for x in want[(b, "logits_head")]], dtype=np.float64)
        assert np.max(np.abs(logits[b, :mg.N_STORED] - stored)) <= 1e-6 * max_abs
        assert [int(x) for x in want[(b, "k_slot_layer0_head0")]] == [int(x) for x in kslot[0, b, 0, :16]]
        assert [int(x) for x in want[(b, "v_slot_layer1_head1")]] == [int(x) for x in vslot[1, b, 1, :16]]


def test_oracle_is_independent_of_the_thread_count():
    from persistent_megakernel_interpreter_b200.config import TINY
    from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
    w = make_weights(TINY, seed=0)
    k, v = make_kv_cache(TINY, 2, mg.MAX_SEQ, mg.PAST, seed=1)
    toks = make_tokens(TINY, 2, seed=2).numpy()
    model = oracle.Model(TINY, w)
    out = []
    for threads in (1, max(2, oracle.max_threads())):
        kc, vc = oracle.bits(k).copy(), oracle.bits(v).copy()
        out.append((model.decode_step(toks, np.array(mg.PAST), kc, vc, threads=threads), kc, vc))
    (l1, k1, v1), (l2, k2, v2) = out
    assert np.array_equal(l1.view(np.uint32), l2.view(np.uint32))
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2)
