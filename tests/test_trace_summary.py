"""The trace summary (trace.py) on a hand-built trace: two SMs, three job rows,
stamps in nanoseconds chosen so every reported figure is known in advance."""
import numpy as np

from persistent_megakernel_interpreter_b200 import trace as tr


def _job(stamps, op, layer, chunk=0, fill=0):
    row = np.zeros(16, np.uint64)
    row[:6] = stamps
    row[tr.META] = op | (layer << 8) | (chunk << 24)
    row[tr.FILL] = fill
    return row


def test_summary_of_a_hand_built_trace():
    t = np.zeros((2, 3, 16), np.uint64)
    # slot wait, counter wait, counter done, ready, start, done
    t[0, 0] = _job([1000, 1000, 3000, 4000, 4000, 9000], op=1, layer=0, fill=5000)
    t[1, 0] = _job([1000, 2000, 4000, 4000, 5000, 11000], op=1, layer=0)
    t[1, 1] = _job([11000, 12000, 13000, 15000, 15000, 21000], op=4, layer=1)
    # t[0, 1], t[0, 2], t[1, 2] stay empty and are skipped
    s = tr.summarize(t)
    assert s["jobs"] == 3
    assert s["step_us"] == (21000 - 1000) / 1e3
    q = s["ops"]["qkv"]
    assert q["jobs"] == 2
    assert q["counter_wait_us"] == {"mean": 2.0, "max": 2.0}
    assert q["prep_us"] == {"mean": 0.5, "max": 1.0}
    assert q["compute_us"] == {"mean": 5.5, "max": 6.0}
    assert q["slot_wait_us"] == {"mean": 0.5, "max": 1.0}
    assert q["first_fill_wait_us"] == {"mean": 1.0, "max": 1.0}
    assert set(s["ops"]) == {"qkv", "gateup"}
    l0, l1 = s["layers"]
    assert l0["layer"] == 0 and l0["qkv_done_last_us"] == 10.0 and l0["qkv_ready_first_us"] == 2.0
    assert l1["gateup_done_last_us"] == 20.0
    text = tr.format_summary(s)
    assert text.startswith("step 20.0 us, 3 jobs") and "L 1 gateup=20.0" in text


def test_empty_trace_gives_empty_summary():
    assert tr.summarize(np.zeros((4, 2, 16), np.uint64)) == {}
