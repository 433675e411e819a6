"""Writes tiny_decode.txt: the oracle's decode step on the small two-layer model,
stored so that any later change to the oracle's arithmetic shows up as a failing
test (the pages print no worked example with values, so no fixture quotes them).

Run from the repository root: ``python tests/golden/make_golden.py``. It calls
only ``oracle/`` and the seeded input generators; nothing here touches the CUDA
library. Workload: the 2-layer, 512-wide model (8 query heads, 2 KV heads, head
size 64, FFN 2048, vocabulary 4096), weights seed 0, two sequences with 128 and
77 cached positions (KV seed 1), tokens seed 2, decoded at positions 128 and 77.
"""
from __future__ import annotations

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FIXTURE = os.path.join(HERE, "tiny_decode.txt")
PAST = [128, 77]
MAX_SEQ = 160
N_STORED = 32  # logits stored per sequence, besides the argmax, the max and the sum


def compute():
    """(logits fp32 [2][vocab], k slot bits, v slot bits) from the oracle."""
    import oracle
    from persistent_megakernel_interpreter_b200.config import TINY
    from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
    w = make_weights(TINY, seed=0)
    k, v = make_kv_cache(TINY, len(PAST), MAX_SEQ, PAST, seed=1)
    toks = make_tokens(TINY, len(PAST), seed=2).numpy()
    kc, vc = oracle.bits(k).copy(), oracle.bits(v).copy()
    logits = oracle.Model(TINY, w).decode_step(toks, np.array(PAST), kc, vc, threads=1)
    kslot = np.stack([kc[:, b, :, p] for b, p in enumerate(PAST)], axis=1)  # [L][B][nkv][d]
    vslot = np.stack([vc[:, b, :, p] for b, p in enumerate(PAST)], axis=1)
    return toks, logits, kslot, vslot


def write():
    toks, logits, kslot, vslot = compute()
    lines = ["# oracle decode step, 2-layer 512-wide model; written by make_golden.py (oracle only)",
             f"tokens {' '.join(str(int(t)) for t in toks)}",
             f"positions {' '.join(str(p) for p in PAST)}"]
    for b in range(logits.shape[0]):
        row = logits[b]
        lines.append(f"seq {b} argmax {int(np.argmax(row))} max_abs {float(np.max(np.abs(row))):.9e} "
                     f"sum {float(np.sum(row.astype(np.float64))):.9e}")
        lines.append(f"seq {b} logits_head " + " ".join(f"{float(x):.9e}" for x in row[:N_STORED]))
        lines.append(f"seq {b} k_slot_layer0_head0 " + " ".join(str(int(x)) for x in kslot[0, b, 0, :16]))
        lines.append(f"seq {b} v_slot_layer1_head1 " + " ".join(str(int(x)) for x in vslot[1, b, 1, :16]))
    with open(FIXTURE, "w") as f:
        f.write("\n".join(lines) + "\n")


def read():
    """The fixture as {key: list of tokens after the key}."""
    out = {}
    with open(FIXTURE) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "seq":
                out[(int(parts[1]), parts[2])] = parts[3:]
            else:
                out[parts[0]] = parts[1:]
    return out


if __name__ == "__main__":
    write()
    print(FIXTURE)
