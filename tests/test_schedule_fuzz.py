"""Randomised schedules: decoder shapes, batches, contexts, SM counts, projection
paths and schedule options drawn inside the ranges mk.h accepts (hypothesis, with a
fixed seed so that every run draws the same cases). For each draw the host planner
either refuses an explicit attention partition size exactly when mk.h's rule makes it
illegal (MK_ERR_INVALID_ARG), or returns a plan that passes the same checks as the
hand-picked cases in test_schedule.py: every weight tile, row block and cached key
covered exactly once, every waited count equal to the signals that counter receives,
and a simulated step of the megakernel's synchronisation protocol that runs to
completion with every counter at its target."""
from hypothesis import HealthCheck, event, given, settings, strategies as st

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.model import plan_schedule
from strategies import shapes
from test_schedule import check_plan, sim, static_signals


@settings(max_examples=150, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(cfg=shapes(), batch=st.integers(1, 8), ctx=st.integers(1, 700), n_sm=st.integers(1, 148),
       proj=st.sampled_from([0, 1, 2]),
       part_keys=st.one_of(st.just(0), st.integers(1, 8).map(lambda k: 8 * k),
                           st.integers(1, 16).map(lambda k: 32 * k)),
       rowblocks_down=st.integers(0, 16), seed=st.one_of(st.just(0), st.integers(1, 2**31)))
def test_random_plans_are_valid_or_refused(cfg, batch, ctx, n_sm, proj, part_keys, rowblocks_down, seed):
    assert cfg.n_heads <= 32 and cfg.group <= 4 and (cfg.n_heads * cfg.head_dim) % 256 == 0
    # the automatic partitioning is always accepted at these sizes; it fixes the ring
    # geometry that decides whether an explicit part_keys is legal
    _, _, auto = plan_schedule(cfg, batch, ctx, n_sm, max_batch=8, max_seq=ctx, proj=proj,
                               rowblocks_down=rowblocks_down, seed=seed)
    kps, max_item = auto.keys_per_stage, min(512, auto.n_stages * auto.keys_per_stage)
    legal = part_keys == 0 or ((part_keys <= kps or part_keys % kps == 0) and part_keys <= max_item
                               and -(-ctx // part_keys) <= 32)
    try:
        instrs, offs, info = check_plan(cfg, batch, ctx, n_sm, proj=proj, part_keys=part_keys,
                                        rowblocks_down=rowblocks_down, seed=seed)
    except _lib.MkError as e:
        # mk.h: a partition is a multiple of 8 keys up to one ring stage, else whole
        # stages, at most what an item holds, and at most 32 per (sequence, group)
        assert e.code == 1 and not legal, (e, part_keys, kps, max_item)
        event("part_keys refused")
        return
    assert legal, (part_keys, kps, max_item)
    assert part_keys == 0 or info.part_keys == part_keys
    event("planned on " + ("tensor cores" if info.proj == _lib.PROJ_TENSOR_CORES else "CUDA cores"))
    # tensor cores only at batch > 1, with a vocabulary of whole 8-row units, unless declined
    assert (info.proj == _lib.PROJ_TENSOR_CORES) == (batch > 1 and cfg.vocab % 8 == 0 and proj != 1)
    ok, ctr = sim(instrs, offs, info, 1 + seed % 3, cfg)
    assert ok, "simulated step did not complete"
    signals = static_signals(instrs, offs, cfg.group, info.n_parts)
    for c in range(info.n_counters):
        assert ctr[c] == signals.get(c, 0), c
