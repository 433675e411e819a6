"""Planted mistakes in the CPU oracle, each of which a pin must catch.

Every case copies ``oracle.c``, plants one plausible mistake in the copy (a dropped
term, a flipped sign, a wrong index or pairing, a transposed operand, a wrong
rounding rule, a skipped step of the decoder), builds it with the oracle's own
compiler flags and runs the oracle's pins (``test_oracle_pins.py`` and
``test_oracle_model.py``: closed forms, invariants, brute force and independent
libraries; the fp64 brute force is set aside) against that build in a child
process. Each mutant must fail at least one pin; the unmodified oracle must pass
them all. The stored regression fixture
(``tests/golden``) is left out on purpose: it was written by the oracle, so it
would catch any change and prove nothing about the pins.

All of this runs on the CPU. The planted mistakes live only in temporary copies;
``oracle.c`` itself is never modified."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
PINS = ["tests/test_oracle_pins.py", "tests/test_oracle_model.py"]

KV_WRITE = ("orc_round_bf16(kf + (size_t)h * d, Kl + (size_t)h * slot_stride + (size_t)pos * d, d);\n"
            "                orc_round_bf16(vf + (size_t)h * d, Vl + (size_t)h * slot_stride + (size_t)pos * d, d);")

# name -> list of (text in oracle.c, replacement); each text occurs exactly once
MUTANTS = {
    "bf16 rounding truncates": [("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0u;")],
    "bf16 ties round away from zero": [("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;")],
    "RMSNorm eps outside the root": [("1.0f / sqrtf(ss / (float)n + eps)",
                                      "1.0f / (sqrtf(ss / (float)n) + eps)")],
    "RMSNorm sum of squares not averaged": [("sqrtf(ss / (float)n + eps)", "sqrtf(ss + eps)")],
    "RMSNorm weight dropped": [("out[i] = (x[i] * r) * bf2f(w[i]);", "out[i] = x[i] * r;")],
    "RoPE first half sign flipped": [("v[i] = a * c - b * s;", "v[i] = a * c + b * s;")],
    "RoPE second half sign flipped": [("v[i + half] = b * c + a * s;", "v[i + half] = b * c - a * s;")],
    "RoPE frequency exponent halved": [("-(2.0 * (double)i) / (double)d", "-(double)i / (double)d")],
    "RoPE adjacent pairs instead of rotate-half": [
        ("float a = v[i], b = v[i + half];\n        v[i] = a * c - b * s;\n        v[i + half] = b * c + a * s;",
         "float a = v[2 * i], b = v[2 * i + 1];\n        v[2 * i] = a * c - b * s;\n"
         "        v[2 * i + 1] = b * c + a * s;")],
    "matvec operand transposed": [("acc += bf2f(wr[k]) * x[k];",
                                   "acc += bf2f(W[(size_t)k * (size_t)rows + (size_t)r]) * x[k];")],
    "attention heads mapped round-robin": [("int g = h / group;", "int g = h % nkv;")],
    "attention scale dropped": [("float scale = 1.0f / sqrtf((float)d);", "float scale = 1.0f;")],
    "attention scale 1/d": [("float scale = 1.0f / sqrtf((float)d);", "float scale = 1.0f / (float)d;")],
    "attention not normalised": [("o[i] = o[i] / l;", "o[i] = o[i];")],
    "new token does not attend to itself": [("pos + 1, max_seq, attn", "pos, max_seq, attn")],
    "keys and values swapped in the cache": [
        (KV_WRITE, KV_WRITE.replace("d, Kl +", "d, TMP +").replace("d, Vl +", "d, Kl +")
         .replace("d, TMP +", "d, Vl +"))],
    "new key written one slot early": [(KV_WRITE, KV_WRITE.replace(
        "(size_t)pos * d", "(size_t)(pos > 0 ? pos - 1 : 0) * d"))],
    "RoPE not applied to keys": [
        ("for (int h = 0; h < nkv; ++h) orc_rope(kf + (size_t)h * d, d, pos, m->rope_theta);", "")],
    "RoPE not applied to queries": [
        ("for (int h = 0; h < nq; ++h) orc_rope(q + (size_t)h * d, d, pos, m->rope_theta);", "")],
    "cache layers overlap across sequences": [
        ("uint16_t* Kl = k_cache + (size_t)l * layer_stride", "uint16_t* Kl = k_cache + (size_t)l * seq_stride"),
        ("uint16_t* Vl = v_cache + (size_t)l * layer_stride", "uint16_t* Vl = v_cache + (size_t)l * seq_stride")],
    "attention residual dropped": [
        ("orc_matvec(m->wo[l], attn, H, Q, y, threads);\n            for (int i = 0; i < H; ++i) x[i] += y[i];",
         "orc_matvec(m->wo[l], attn, H, Q, y, threads);\n            for (int i = 0; i < H; ++i) x[i] = y[i];")],
    "MLP residual dropped": [
        ("orc_matvec(m->wdown[l], hb, H, F, y, threads);\n            for (int i = 0; i < H; ++i) x[i] += y[i];",
         "orc_matvec(m->wdown[l], hb, H, F, y, threads);\n            for (int i = 0; i < H; ++i) x[i] = y[i];")],
    "MLP normalised with the attention norm": [("orc_rmsnorm(x, m->mlp_norm[l]", "orc_rmsnorm(x, m->attn_norm[l]")],
    "gate and up swapped": [("orc_silu_mul(g, u, F, hb);", "orc_silu_mul(u, g, F, hb);")],
    "SiLU sign flipped": [("(1.0f + expf(-g[i]))", "(1.0f + expf(g[i]))")],
    "final norm skipped": [("m->lm_head ? m->lm_head : m->embed, xn,", "m->lm_head ? m->lm_head : m->embed, x,")],
    "embedding row offset not scaled": [("m->embed + (size_t)tokens[b] * H, x, H", "m->embed + (size_t)tokens[b], x, H")],
    "argmax keeps the last of equal logits": [("if (x[i] > x[best]) best = i;", "if (x[i] >= x[best]) best = i;")],
}

# Runs the pins once per build in one process (the imports are paid once), up to the
# first failure, with the fp64 restatement of the decoder (brute.py) set aside so that
# every catch comes from mathematics or an independent library; prints one JSON line:
# build name -> node ids of the pins that failed.
CHILD = r"""
import json, sys
import pytest
import oracle
builds = json.loads(sys.stdin.read())
out = {}
class Failed:
    def __init__(self): self.ids = []
    def pytest_runtest_logreport(self, report):
        if report.failed: self.ids.append(report.nodeid)
for name, path in builds:
    oracle._lib = oracle.load(path)
    f = Failed()
    pytest.main(["-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu", "-k", "not brute",
                 "-W", "ignore"] + PINS, plugins=[f])
    out[name] = f.ids
print("MUTANT-RESULTS " + json.dumps(out))
"""


def build(text: str, path: str) -> None:
    src = path[:-3] + ".c"
    with open(src, "w") as fh:
        fh.write(text)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                           "-shared", "-fPIC", "-o", path, src, "-lm"])


def test_every_planted_mistake_fails_a_pin(tmp_path):
    import oracle
    with open(SRC) as fh:
        base = fh.read()
    builds = [("unmodified", oracle.build())]
    for i, (name, edits) in enumerate(MUTANTS.items()):
        text = base
        for old, new in edits:
            assert text.count(old) == 1, (name, old)
            text = text.replace(old, new)
        assert text != base, name
        path = str(tmp_path / f"mutant{i}.so")
        build(text, path)
        builds.append((name, path))
    child = CHILD.replace("PINS", json.dumps(PINS))
    r = subprocess.run([sys.executable, "-c", child], input=json.dumps(builds), cwd=ROOT,
                       capture_output=True, text=True, timeout=900,
                       env=dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.path.join(ROOT, "tests")))
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("MUTANT-RESULTS ")]
    assert r.returncode == 0 and line, r.stdout[-3000:] + r.stderr[-3000:]
    failed = json.loads(line[-1][len("MUTANT-RESULTS "):])
    assert failed["unmodified"] == [], failed["unmodified"]
    for name in MUTANTS:
        print(f"{name:45s} caught by", ", ".join(failed[name]) or "NOTHING")
    missed = [name for name in MUTANTS if not failed[name]]
    assert not missed, missed
