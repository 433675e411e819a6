"""Schedule builder (host only): coverage of every tile exactly once, counter
targets, per-SM byte balance, and a CPU simulation of the megakernel's
synchronisation protocol (loader ring of S stages, 8 consumer warps taking
instructions round-robin, counters with targets) that must run to completion --
i.e. the schedule cannot deadlock -- and end with every counter at its target."""
import collections

import pytest

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B, TINY
from persistent_megakernel_interpreter_b200.model import plan_schedule

W = 8  # consumer warps per CTA
NO = _lib.NO_COUNTER


def simulate(instrs, offs, n_counters, S):
    n_sm = len(offs) - 1
    ctr = [0] * n_counters
    lists = [instrs[offs[s]:offs[s + 1]] for s in range(n_sm)]
    total_fills = [sum(i.nfill for i in L) for L in lists]
    issued = [0] * n_sm
    released = [bytearray(t) for t in total_fills]
    pos = [[w for w in range(W)] for _ in range(n_sm)]       # next instruction index per warp
    fill = [[0] * W for _ in range(n_sm)]
    done = 0
    n_total = len(instrs)
    changed = True
    rounds = 0
    while changed:
        changed = False
        rounds += 1
        for s in range(n_sm):
            L = lists[s]
            while issued[s] < total_fills[s] and (issued[s] < S or released[s][issued[s] - S]):
                issued[s] += 1
                changed = True
            for w in range(W):
                while pos[s][w] < len(L):
                    ins = L[pos[s][w]]
                    f = fill[s][w]
                    if ins.op == _lib.OP_DOWN:
                        c = min(f, ins.nfill - 1) // ins.count
                        need = (ins.wait_ctr + c, ins.wait_n)
                    elif ins.wait_ctr != NO:
                        need = (ins.wait_ctr, ins.wait_n)
                    else:
                        need = None
                    if need and f < ins.nfill and ctr[need[0]] < need[1]:
                        break
                    if f < ins.nfill:
                        seq = ins.seq + f
                        if seq >= issued[s]:
                            break
                        released[s][seq] = 1
                        fill[s][w] += 1
                        changed = True
                        continue
                    # complete
                    if ins.signal_ctr != NO:
                        ctr[ins.signal_ctr] += 1
                    if ins.op == _lib.OP_ATTN and ctr[ins.signal_ctr] == ins.aux_n:
                        ctr[ins.aux_ctr] += 1
                    done += 1
                    pos[s][w] += W
                    fill[s][w] = 0
                    changed = True
    return done == n_total, ctr, rounds


def check_plan(cfg, batch, max_ctx, n_sm, **opts):
    instrs, offs, info = plan_schedule(cfg, batch, max_ctx, n_sm, max_batch=8, max_seq=max_ctx, **opts)
    assert info.n_instr == len(instrs) and offs[-1] == len(instrs)
    # per-SM fill numbering is the prefix sum of fills
    for s in range(n_sm):
        seq = 0
        for ins in instrs[offs[s]:offs[s + 1]]:
            assert ins.seq == seq
            seq += ins.nfill
    # coverage: every tile / row block / key exactly once
    tpg = (cfg.group + 2) * cfg.head_dim // 4
    cov = collections.Counter()
    for ins in instrs:
        if ins.op == _lib.OP_ATTN:
            for k in range(ins.first, ins.first + ins.count):
                cov[(ins.op, ins.layer, ins.batch, ins.group, k)] += 1
            assert ins.nfill == -(-ins.count // info.keys_per_stage)
        else:
            for t in range(ins.first, ins.first + ins.count):
                cov[(ins.op, ins.layer, t)] += 1
    assert all(v == 1 for v in cov.values())
    for l in range(cfg.n_layers):
        assert all(cov[(_lib.OP_QKV, l, t)] for t in range(cfg.n_kv_heads * tpg))
        assert all(cov[(_lib.OP_OPROJ, l, t)] for t in range(cfg.hidden // 4))
        assert all(cov[(_lib.OP_GATEUP, l, t)] for t in range(cfg.ffn // 2))
        assert all(cov[(_lib.OP_DOWN, l, t)] for t in range(cfg.hidden // 4))
        for b in range(batch):
            for g in range(cfg.n_kv_heads):
                assert all(cov[(_lib.OP_ATTN, l, b, g, k)] for k in range(max_ctx))
    assert all(cov[(_lib.OP_LMHEAD, cfg.n_layers - 1, t)] for t in range(cfg.vocab // 4))
    assert len(cov) == (cfg.n_layers * (cfg.n_kv_heads * tpg + cfg.hidden // 2 + cfg.ffn // 2
                                        + batch * cfg.n_kv_heads * max_ctx) + cfg.vocab // 4)
    # every signalled counter is waited for with the right count
    signals = collections.Counter(i.signal_ctr for i in instrs)
    for ins in instrs:
        if ins.wait_ctr == NO:
            continue
        if ins.op == _lib.OP_OPROJ:
            assert ins.wait_n == batch * cfg.n_kv_heads
        elif ins.op == _lib.OP_DOWN:
            for c in range(4):
                assert signals[ins.wait_ctr + c] == ins.wait_n
        else:
            assert signals[ins.wait_ctr] == ins.wait_n
    return instrs, offs, info


@pytest.mark.parametrize("cfg,batch,ctx,n_sm", [
    (TINY, 1, 129, 148), (TINY, 2, 200, 37), (TINY, 3, 64, 7), (TINY, 1, 1, 148),
    (LLAMA_1B, 1, 129, 148), (LLAMA_1B, 1, 8193, 148), (LLAMA_3B, 8, 2049, 148),
])
def test_plan_valid_and_deadlock_free(cfg, batch, ctx, n_sm):
    instrs, offs, info = check_plan(cfg, batch, ctx, n_sm)
    ok, ctr, rounds = simulate(instrs, offs, info.n_counters, info.n_stages)
    assert ok, "simulated step did not complete"
    signals = collections.Counter(i.signal_ctr for i in instrs if i.signal_ctr != NO)
    for c in range(info.n_counters):
        expect = signals.get(c, 0)
        if any(i.op == _lib.OP_ATTN and i.aux_ctr == c for i in instrs):
            expect = batch * cfg.n_kv_heads
        assert ctr[c] == expect, c


def test_balance_1b():
    _, _, info = plan_schedule(LLAMA_1B, 1, 129, 148, max_seq=129)
    mean = info.bytes_per_step / 148
    assert info.max_sm_bytes <= mean * 1.02
    assert info.min_sm_bytes >= mean * 0.98
    assert info.stage_bytes == 16384 and info.n_stages >= 9


def test_seeded_placement_is_also_valid():
    instrs, offs, info = check_plan(TINY, 2, 100, 20, seed=1234)
    ok, _, _ = simulate(instrs, offs, info.n_counters, info.n_stages)
    assert ok


def test_dropped_item_cannot_complete():
    """The failure-injection hook removes one producer: the protocol must stall
    (on the GPU the bounded waits then end the step with MK_ERR_TIMEOUT)."""
    instrs, offs, info = plan_schedule(TINY, 1, 64, 16, max_seq=64, test_drop_item=5)
    ok, _, _ = simulate(instrs, offs, info.n_counters, info.n_stages)
    assert not ok
