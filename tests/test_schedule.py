"""Schedule builder (host only): coverage of every tile exactly once, counter
targets, per-SM byte balance, and a CPU simulation of the megakernel's
synchronisation protocol that must run to completion (the schedule cannot
deadlock) and leave every counter at its target. The simulated protocol: a
loader issuing the SM's fills in order into a ring of S stages, each once the
stage's previous fill is released; four mover warps, mover q taking the fills
seq = q (mod 4) in order and moving each landed weight tile into Tensor Memory
slot seq mod NT once that slot's previous tile is released (which frees the
tile's stage; a cached-KV fill stays in the ring and only passes its slot over);
an activation warp preparing each job's input in one of NS slots once its
counters are met; 8 compute warps, warp w taking the job's tiles with
seq = w (mod 8) (batch > 1: seq = w (mod 4), two warps per tile), and an
attention item waiting for all of its fills and freeing their stages when every
warp is done. Attention items signal per query head: a (sequence, KV group)
pair's heads are signalled once its last partition has arrived (with one
partition, at once)."""
import collections

import numpy as np

import pytest

from persistent_megakernel_interpreter_b200 import _lib
from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B, TINY
from persistent_megakernel_interpreter_b200.model import plan_schedule

W = 8  # compute warps per CTA
NO = _lib.NO_COUNTER


def jobs_of(lst):
    """The kernel's job sequence for one SM list: (first instr index, chunk, n items)."""
    jobs, i = [], 0
    while i < len(lst):
        ins = lst[i]
        items = ins.job_items if ins.op == _lib.OP_ATTN else 1
        assert items >= 1
        for c in range(4 if ins.op == _lib.OP_DOWN else 1):
            jobs.append((i, c, items))
        i += items
    return jobs


def job_waits(lst, job):
    i, c, items = job
    ins = lst[i]
    if ins.op == _lib.OP_ATTN:
        return [(lst[i + k].wait_ctr, lst[i + k].wait_n) for k in range(items)]
    if ins.op == _lib.OP_DOWN:
        t = [ins.wait_n, ins.aux0 & 0xFFFF, ins.aux0 >> 16, ins.aux1]
        return [(ins.wait_ctr + c, t[c])]
    return [] if ins.wait_ctr == NO else [(ins.wait_ctr, ins.wait_n)]


def job_fills(lst, job):
    """Fills of the job: (weight tiles, cached-KV fills)."""
    i, c, items = job
    ins = lst[i]
    if ins.op == _lib.OP_ATTN:
        kv = []
        for k in range(items):
            a = lst[i + k]
            kv += list(range(a.seq, a.seq + a.nfill))
        return [], kv
    if ins.op == _lib.OP_DOWN:
        return [ins.seq + c * ins.count + r for r in range(ins.count)], []
    return [ins.seq + t for t in range(ins.count)], []


def tmem_slots(stage_bytes):
    """Tensor Memory slots of a plan (as the library sets them): four lane quarters
    of 512 columns, one slot per stage_bytes / 128 columns, at most 16 a quarter."""
    return 4 * min(16, 512 // (stage_bytes // 128))


def job_done_signals(L, job, group, n_parts, arr, ctr):
    """Counter increments when all compute warps finished `job` (arr: arrival
    counts per (sequence, group) pair)."""
    i, c, items = job
    ins = L[i]
    if ins.op == _lib.OP_ATTN:
        for k in range(items):
            a = L[i + k]
            if a.signal_ctr == NO:
                continue
            arr[a.aux0] += group
            if arr[a.aux0] == n_parts * group:
                ctr[a.signal_ctr] += group
    elif ins.signal_ctr != NO and (ins.op != _lib.OP_DOWN or c == 3):
        span = max(1, ins.aux1) if ins.op in (_lib.OP_QKV, _lib.OP_GATEUP) else 1
        for k in range(span):
            ctr[ins.signal_ctr + k] += 1


def static_signals(instrs, offs, group, n_parts):
    ctr, arr = collections.Counter(), collections.Counter()
    for s_ in range(len(offs) - 1):
        L = instrs[offs[s_]:offs[s_ + 1]]
        for job in jobs_of(L):
            job_done_signals(L, job, group, n_parts, arr, ctr)
    return ctr


def simulate(instrs, offs, n_counters, S, NS=2, group=1, n_parts=1, NT=16, batched=False):
    assert S % 4 == 0 and NT % 4 == 0
    n_sm = len(offs) - 1
    ctr = [0] * n_counters
    arr = collections.Counter()
    users = 2 if batched else 1  # compute warps reading each weight tile
    lists = [instrs[offs[s]:offs[s + 1]] for s in range(n_sm)]
    jobs = [jobs_of(L) for L in lists]
    kv_fill = []
    for L in lists:
        k = []
        for ins in L:
            k += [ins.op == _lib.OP_ATTN] * ins.nfill
        kv_fill.append(k)
    total = [len(k) for k in kv_fill]
    n_iss = [0] * n_sm                         # fills the loader has issued
    n_mov = [[0] * 4 for _ in range(n_sm)]     # per mover: its fills moved (or passed over)
    issued = [bytearray(t) for t in total]
    freed = [bytearray(t) for t in total]      # ring stage released
    moved = [bytearray(t) for t in total]      # Tensor Memory slot holds the tile
    reads = [[0] * t for t in total]           # compute warps done with the slot
    prepared = [0] * n_sm                       # jobs whose input is ready
    done = [[0] * len(j) for j in jobs]         # warps finished per job
    wjob = [[0] * W for _ in range(n_sm)]       # job each warp is on
    wpos = [[0] * W for _ in range(n_sm)]       # tiles consumed in that job
    changed = True
    while changed:
        changed = False
        for s in range(n_sm):
            L, J = lists[s], jobs[s]
            while True:  # the loader: fills in order, each once its stage is free
                f = n_iss[s]
                if f >= total[s] or (f >= S and not freed[s][f - S]):
                    break
                issued[s][f] = 1
                n_iss[s] += 1
                changed = True
            for q in range(4):  # mover q: its fills in order, blocking on each
                while True:
                    f = q + 4 * n_mov[s][q]
                    if f >= total[s] or not issued[s][f]:
                        break
                    if f >= NT and reads[s][f - NT] < users:
                        break
                    moved[s][f] = 1
                    if kv_fill[s][f]:
                        reads[s][f] = users  # the slot is passed over
                    else:
                        freed[s][f] = 1
                    n_mov[s][q] += 1
                    changed = True
            while prepared[s] < len(J):
                j = prepared[s]
                if j >= NS and done[s][j - NS] < W:
                    break
                if any(ctr[c] < t for c, t in job_waits(L, J[j])):
                    break
                prepared[s] += 1
                changed = True
            for w in range(W):
                while wjob[s][w] < len(J) and wjob[s][w] < prepared[s]:
                    j = wjob[s][w]
                    tiles, kv = job_fills(L, J[j])
                    mine = [f for f in tiles if (f % 4 == w % 4 if batched else f % 8 == w)]
                    k = wpos[s][w]
                    if k < len(mine):
                        if not moved[s][mine[k]]:
                            break
                        reads[s][mine[k]] += 1
                        wpos[s][w] += 1
                        changed = True
                        continue
                    if not all(issued[s][f] for f in kv):
                        break
                    done[s][j] += 1
                    if done[s][j] == W:
                        for f in kv:
                            freed[s][f] = 1
                        job_done_signals(L, J[j], group, n_parts, arr, ctr)
                    wjob[s][w] += 1
                    wpos[s][w] = 0
                    changed = True
    ok = all(all(d == W for d in dj) for dj in done)
    return ok, ctr


# ---- the tensor-core path (batch > 1): fill geometry and protocol

def mma_geom(ins, cfg, stage_bytes):
    """Fills of a matvec instruction on the tensor-core path (restated from the
    library's header): rows (a multiple of 8) cut into segments of <= 128 per range
    (gate/up: one range per MLP chunk); a segment of R rows streams in fills of
    nb(R) 64-column boxes, as many as a ring stage holds."""
    jobs, nrange, rows, k64 = 1, 1, 4 * ins.count, cfg.hidden // 64
    if ins.op == _lib.OP_OPROJ:
        k64 = cfg.n_heads * cfg.head_dim // 64
    elif ins.op == _lib.OP_DOWN:
        k64, jobs = cfg.ffn // 4 // 64, 4
    elif ins.op == _lib.OP_GATEUP:
        rows, nrange = 4 * ins.aux0, 4
    segs = -(-rows // 128)
    seg_rows = [128] * (segs - 1) + [rows - 128 * (segs - 1)]
    nb = [max(1, min(k64, stage_bytes // (r * 128))) for r in seg_rows]
    fps = [-(-k64 // n) for n in nb]
    return dict(jobs=jobs, nrange=nrange, rows=rows, k64=k64, segs=segs, seg_rows=seg_rows, nb=nb, fps=fps)


def mma_fills(ins, cfg, stage_bytes):
    """Per fill of the instruction, in order: (job c, range, segment, fill index kf,
    K boxes it uses, segment rows, boxes the copy spans)."""
    g = mma_geom(ins, cfg, stage_bytes)
    out = []
    for c in range(g["jobs"]):
        for rg in range(g["nrange"]):
            for seg in range(g["segs"]):
                nb = g["nb"][seg]
                for kf in range(g["fps"][seg]):
                    boxes = range(kf * nb, min(kf * nb + nb, g["k64"]))
                    out.append((c, rg, seg, kf, boxes, g["seg_rows"][seg], nb))
    return g, out


def simulate_mma(instrs, offs, n_counters, S, NS, group, n_parts, cfg, stage_bytes, n_acc=8):
    """The tensor-core protocol: the loader as above; an activation warp preparing
    each job once its slot is free and its counters are met; the compute warps (as
    one) writing a matvec job's operand, then reading out each of its segments'
    accumulators once final (the down-projection: after its last chunk), then
    waiting for the job's MMAs before freeing the slot; an attention item as
    above; the issuer (the kernel's four issuer warps wait for the same things in
    the same order, so they are one here) walking the jobs in order, each once its
    operand is written:
    each fill once it has landed and, for a segment's first fill, once the
    segment n_acc earlier (same accumulator) has been read out; the fill's MMAs
    free its stage, a segment's last fill makes its accumulator final, a job's
    last marks the job's MMAs done."""
    n_sm = len(offs) - 1
    ctr = [0] * n_counters
    arr = collections.Counter()
    ok_all = True
    lists = [instrs[offs[s]:offs[s + 1]] for s in range(n_sm)]
    jobs = [jobs_of(L) for L in lists]
    # per SM: each job's fills (seq, segment number, first of segment, last of segment)
    # and the segments its epilogue reads
    plan = []
    for L, J in zip(lists, jobs):
        sn0, per_job, reads = 0, [], []
        for (i, c, items) in J:
            ins = L[i]
            if ins.op == _lib.OP_ATTN:
                per_job.append(None)
                reads.append([])
                continue
            g, fl = mma_fills(ins, cfg, stage_bytes)
            per = len(fl) // g["jobs"]
            mine = []
            for r in range(per):
                cc, rg, seg, kf, boxes, rows, nb = fl[c * per + r]
                assert cc == c
                sn = sn0 + rg * g["segs"] + seg
                mine.append((ins.seq + c * per + r, sn, c == 0 and kf == 0,
                             c == g["jobs"] - 1 and kf == g["fps"][seg] - 1))
            per_job.append(mine)
            reads.append([sn0 + k for k in range(g["nrange"] * g["segs"])] if c == g["jobs"] - 1 else [])
            if c == g["jobs"] - 1:
                sn0 += g["nrange"] * g["segs"]
        plan.append((per_job, reads))
    total = [sum(ins.nfill for ins in L) for L in lists]
    kv_of = []
    for L, J in zip(lists, jobs):
        kv_of.append([job_fills(L, job)[1] for job in J])
    n_iss = [0] * n_sm
    issued = [bytearray(t) for t in total]
    freed = [bytearray(t) for t in total]
    prepared = [0] * n_sm
    opnd = [bytearray(len(J)) for J in jobs]
    mdone = [bytearray(len(J)) for J in jobs]
    afull, aread = [set() for _ in range(n_sm)], [set() for _ in range(n_sm)]
    done = [bytearray(len(J)) for J in jobs]
    ij, ip = [0] * n_sm, [0] * n_sm     # issuer: job, fill within it
    cj, cr = [0] * n_sm, [0] * n_sm     # compute warps: job, segments read in it
    changed = True
    while changed:
        changed = False
        for s in range(n_sm):
            L, J = lists[s], jobs[s]
            per_job, reads = plan[s]
            while True:
                f = n_iss[s]
                if f >= total[s] or (f >= S and not freed[s][f - S]):
                    break
                issued[s][f] = 1
                n_iss[s] += 1
                changed = True
            while prepared[s] < len(J):
                j = prepared[s]
                if j >= NS and not done[s][j - NS]:
                    break
                if any(ctr[c] < t for c, t in job_waits(L, J[j])):
                    break
                prepared[s] += 1
                changed = True
            while ij[s] < len(J):  # the issuer
                j = ij[s]
                if per_job[j] is None:
                    ij[s] += 1
                    changed = True
                    continue
                if not opnd[s][j]:
                    break
                if ip[s] < len(per_job[j]):
                    f, sn, first, last = per_job[j][ip[s]]
                    if first and sn >= n_acc and (sn - n_acc) not in aread[s]:
                        break
                    if not issued[s][f]:
                        break
                    freed[s][f] = 1
                    if last:
                        afull[s].add(sn)
                    ip[s] += 1
                    changed = True
                    continue
                mdone[s][j] = 1
                ij[s] += 1
                ip[s] = 0
                changed = True
            while cj[s] < len(J) and cj[s] < prepared[s]:  # the compute warps
                j = cj[s]
                if per_job[j] is None:
                    if not all(issued[s][f] for f in kv_of[s][j]):
                        break
                    for f in kv_of[s][j]:
                        freed[s][f] = 1
                else:
                    opnd[s][j] = 1
                    if cr[s] < len(reads[j]):
                        sn = reads[j][cr[s]]
                        if sn not in afull[s]:
                            break
                        aread[s].add(sn)
                        cr[s] += 1
                        changed = True
                        continue
                    if not mdone[s][j]:
                        break
                done[s][j] = 1
                job_done_signals(L, J[j], group, n_parts, arr, ctr)
                cj[s] += 1
                cr[s] = 0
                changed = True
        ok_all = all(all(d for d in dj) for dj in done)
    return ok_all, ctr


def sim(instrs, offs, info, ns, cfg):
    if info.proj == _lib.PROJ_TENSOR_CORES:
        return simulate_mma(instrs, offs, info.n_counters, info.n_stages, ns, cfg.group, info.n_parts, cfg,
                            info.stage_bytes)
    return simulate(instrs, offs, info.n_counters, info.n_stages, ns, cfg.group, info.n_parts,
                    NT=tmem_slots(info.stage_bytes), batched=info.batch > 1)


def check_plan(cfg, batch, max_ctx, n_sm, **opts):
    instrs, offs, info = plan_schedule(cfg, batch, max_ctx, n_sm, max_batch=8, max_seq=max_ctx, **opts)
    check_lists(cfg, batch, max_ctx, instrs, offs, info)
    return instrs, offs, info


def check_lists(cfg, batch, max_ctx, instrs, offs, info):
    """The static checks of a plan's per-SM lists (raise AssertionError on a fault)."""
    n_sm = len(offs) - 1
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
        elif ins.op == _lib.OP_GATEUP:  # chunk-major: the same slice of each chunk
            assert ins.count == 4 * ins.aux0
            for i in range(ins.count):
                t = (i // ins.aux0) * (cfg.ffn // 8) + ins.first + i % ins.aux0
                cov[(ins.op, ins.layer, t)] += 1
        else:
            for t in range(ins.first, ins.first + ins.count):
                cov[(ins.op, ins.layer, t)] += 1
    assert all(v == 1 for v in cov.values())
    # one QKV and one gate/up job per SM and layer (one RMSNorm each); a job whose
    # tiles cross a KV-group / MLP-chunk boundary signals every counter it touched
    for s in range(n_sm):
        per = collections.Counter((ins.op, ins.layer) for ins in instrs[offs[s]:offs[s + 1]]
                                  if ins.op in (_lib.OP_QKV, _lib.OP_GATEUP))
        assert all(v == 1 for v in per.values()), per
    for ins in instrs:
        if ins.op == _lib.OP_QKV:
            assert ins.group == ins.first // tpg
            assert ins.aux1 == (ins.first + ins.count - 1) // tpg - ins.group + 1
        if ins.op == _lib.OP_GATEUP:  # every chunk counter, once
            assert ins.aux1 == 4 and ins.first + ins.aux0 <= cfg.ffn // 8
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
    # arrival counters: one per (layer, sequence, group), shared by exactly that
    # pair's items, never waited on
    arr_of = collections.defaultdict(set)
    for ins in instrs:
        if ins.op == _lib.OP_ATTN:
            arr_of[ins.aux0].add((ins.layer, ins.batch, ins.group))
            assert ins.aux0 < info.n_counters
    assert all(len(v) == 1 for v in arr_of.values())
    assert len(arr_of) == cfg.n_layers * batch * cfg.n_kv_heads
    waited = {ins.wait_ctr for ins in instrs}
    assert not waited & set(arr_of)
    # every waited counter's target is the number of signals it receives
    signals = static_signals(instrs, offs, cfg.group, info.n_parts)
    for l in range(cfg.n_layers):
        c = {ins.signal_ctr for ins in instrs if ins.op == _lib.OP_ATTN and ins.layer == l}
        assert len(c) == 1 and signals[c.pop()] == batch * cfg.n_heads
    for s_ in range(n_sm):
        L = instrs[offs[s_]:offs[s_ + 1]]
        for job in jobs_of(L):
            for c, t in job_waits(L, job):
                assert signals[c] == t, (c, t, signals[c])


@pytest.mark.parametrize("cfg,batch,ctx,n_sm,proj", [
    (TINY, 1, 129, 148, 0), (TINY, 2, 200, 37, 0), (TINY, 2, 200, 37, 1), (TINY, 3, 64, 7, 0),
    (TINY, 3, 64, 7, 1), (TINY, 1, 1, 148, 2), (LLAMA_1B, 1, 129, 148, 0), (LLAMA_1B, 1, 8193, 148, 0),
    (LLAMA_3B, 8, 2049, 148, 0), (LLAMA_3B, 8, 2049, 148, 1),
])
def test_plan_valid_and_deadlock_free(cfg, batch, ctx, n_sm, proj):
    """Both projection paths at batch > 1 (proj 0: the default, tensor cores; 1:
    CUDA cores); batch 1 always runs on the CUDA cores."""
    instrs, offs, info = check_plan(cfg, batch, ctx, n_sm, proj=proj)
    assert info.proj == (_lib.PROJ_TENSOR_CORES if batch > 1 and proj != 1 else _lib.PROJ_CUDA_CORES)
    for ns in (1, 2, 3):
        ok, ctr = sim(instrs, offs, info, ns, cfg)
        assert ok, "simulated step did not complete"
    signals = static_signals(instrs, offs, cfg.group, info.n_parts)
    for c in range(info.n_counters):
        assert ctr[c] == signals.get(c, 0), c


def test_balance_1b():
    """Streamed bytes per SM within 3% of the mean: placement balances bytes plus a
    fixed charge per attention item (the SMs that run attention take fewer gate/up
    tiles of that layer), so the bytes alone are not exactly even."""
    _, _, info = plan_schedule(LLAMA_1B, 1, 129, 148, max_seq=129)
    mean = info.bytes_per_step / 148
    assert info.max_sm_bytes <= mean * 1.03
    assert info.min_sm_bytes >= mean * 0.97
    # 12 stages: the most that fit beside 3 job slots, a multiple of the 4 mover warps
    assert info.stage_bytes == 16384 and info.n_stages == 12


def test_seeded_placement_is_also_valid():
    instrs, offs, info = check_plan(TINY, 2, 100, 20, seed=1234)
    ok, _ = sim(instrs, offs, info, 2, TINY)
    assert ok


def test_dropped_item_cannot_complete():
    """The failure-injection hook removes one producer: the protocol must stall
    (on the GPU the bounded waits then end the step with MK_ERR_TIMEOUT)."""
    for drop in range(1, 12):
        instrs, offs, info = plan_schedule(TINY, 1, 64, 16, max_seq=64, test_drop_item=drop)
        if instrs[drop - 1].op == _lib.OP_LMHEAD:
            continue  # nothing in the step waits for the logits
        ok, _ = sim(instrs, offs, info, 2, TINY)
        assert not ok, drop


def _copy(ins):
    return _lib.MkInstr.from_buffer_copy(ins)


def _renumber(instrs, offs):
    """Recompute each SM's fill numbering (seq) after a list was edited."""
    for s_ in range(len(offs) - 1):
        seq = 0
        for ins in instrs[offs[s_]:offs[s_ + 1]]:
            ins.seq = seq
            seq += ins.nfill


def _plant(instrs, offs, kind):
    """A copy of the plan with one planted mistake of the given kind."""
    L = [_copy(i) for i in instrs]
    if kind == "waited count one too high":
        next(i for i in L if i.op == _lib.OP_OPROJ).wait_n += 1
    elif kind == "a tile computed twice, another never":
        next(i for i in L if i.op == _lib.OP_OPROJ and i.count > 1).first += 1
    elif kind == "fill numbering off by one":
        next(i for i in L if i.op == _lib.OP_GATEUP).seq += 1
    elif kind == "attention item signals the wrong layer":
        a = [i for i in L if i.op == _lib.OP_ATTN]
        a[0].signal_ctr = next(i.signal_ctr for i in a if i.layer != a[0].layer)
    elif kind == "consumer ahead of its producer on one SM":
        # an attention item moved in front of the QKV job of its own layer on the
        # same SM, whose group counter it waits on
        for s_ in range(len(offs) - 1):
            lst = L[offs[s_]:offs[s_ + 1]]
            q = [k for k, i in enumerate(lst) if i.op == _lib.OP_QKV]
            a = [k for k, i in enumerate(lst) if i.op == _lib.OP_ATTN and i.job_items == 1
                 and any(lst[j].layer == i.layer and lst[j].signal_ctr <= i.wait_ctr
                         < lst[j].signal_ctr + max(1, lst[j].aux1) for j in q if j < k)]
            if a:
                k = a[0]
                j = next(j for j in q if j < k and lst[j].layer == lst[k].layer)
                lst.insert(j, lst.pop(k))
                L[offs[s_]:offs[s_ + 1]] = lst
                _renumber(L, offs)
                return L
        raise AssertionError("no attention item shares an SM with its QKV producer")
    return L


@pytest.mark.parametrize("proj", [1, 2])
@pytest.mark.parametrize("kind", ["waited count one too high", "a tile computed twice, another never",
                                  "fill numbering off by one", "attention item signals the wrong layer",
                                  "consumer ahead of its producer on one SM"])
def test_checks_catch_planted_plan_errors(kind, proj):
    """The plan checks and the protocol simulators (CUDA-core and tensor-core paths) are
    themselves tested: each planted mistake in a valid plan fails a static check or
    leaves the simulated step stuck (an ordering mistake passes every static check;
    only the simulation sees it)."""
    instrs, offs, info = check_plan(TINY, 2, 129, 37, proj=proj)
    assert info.proj == (_lib.PROJ_CUDA_CORES if proj == 1 else _lib.PROJ_TENSOR_CORES)
    bad = _plant(instrs, offs, kind)
    try:
        check_lists(TINY, 2, 129, bad, offs, info)
    except AssertionError:
        static = True
    else:
        static = False
    ok, _ = sim(bad, offs, info, 2, TINY)
    assert static or not ok, kind
    if kind == "consumer ahead of its producer on one SM":
        assert not static and not ok


@pytest.mark.parametrize("cfg,batch,ctx,parts", [
    (LLAMA_1B, 1, 129, 1), (LLAMA_1B, 1, 288, 1), (LLAMA_1B, 1, 512, 16), (LLAMA_1B, 1, 1025, 17),
    (LLAMA_1B, 1, 2048, 16), (LLAMA_1B, 1, 8193, 17), (LLAMA_3B, 8, 2049, 10), (TINY, 1, 129, 1),
])
def test_partition_count(cfg, batch, ctx, parts):
    """One partition per (sequence, group) up to 320 keys; for longer contexts as
    many as fit one item per SM; more items than SMs only when a partition is
    already as long as an item may be (all its fills in the ring at once, at most
    512 keys)."""
    _, _, info = plan_schedule(cfg, batch, ctx, 148, max_batch=8, max_seq=ctx)
    assert info.n_parts == parts
    max_item = min(512, info.n_stages * info.keys_per_stage)
    assert info.part_keys <= max_item
    assert (info.n_parts * batch * cfg.n_kv_heads <= 148
            or info.part_keys == max_item // info.keys_per_stage * info.keys_per_stage)


@pytest.mark.parametrize("cfg,batch,ctx", [
    (LLAMA_1B, 1, 129), (LLAMA_1B, 1, 4097), (LLAMA_1B, 1, 8193), (LLAMA_3B, 8, 2049), (TINY, 3, 200),
])
def test_attention_items_spread_over_sms(cfg, batch, ctx):
    """An SM runs its attention items one after the other, so within a layer no
    SM gets a second item before every SM has one (the layer's attention ends
    with its slowest SM)."""
    instrs, offs, info = plan_schedule(cfg, batch, ctx, 148, max_batch=8, max_seq=ctx)
    per_layer = collections.defaultdict(lambda: collections.Counter())
    for s in range(148):
        for ins in instrs[offs[s]:offs[s + 1]]:
            if ins.op == _lib.OP_ATTN:
                per_layer[ins.layer][s] += 1
    items = batch * cfg.n_kv_heads * info.n_parts
    for layer, cnt in per_layer.items():
        assert sum(cnt.values()) == items
        assert max(cnt.values()) == -(-items // 148), (layer, max(cnt.values()))
        if items >= 148:
            assert len(cnt) == 148


@pytest.mark.parametrize("cfg,batch", [(LLAMA_1B, 1), (LLAMA_3B, 8), (TINY, 2)])
def test_down_instructions_cover_row_block_ranges(cfg, batch):
    """Down-projection instructions take contiguous ranges of up to 16 row blocks
    at every batch size (each chunk's input is loaded once per instruction), and
    together cover every row block of every layer exactly once."""
    instrs, offs, _ = plan_schedule(cfg, batch, 129, 148, max_batch=8, max_seq=129, proj=1)
    for layer in range(cfg.n_layers):
        seen = []
        for ins in instrs:
            if ins.op == _lib.OP_DOWN and ins.layer == layer:
                assert 1 <= ins.count <= 16 and ins.nfill == 4 * ins.count
                seen.extend(range(ins.first, ins.first + ins.count))
        assert sorted(seen) == list(range(cfg.hidden // 4))
    n_down = sum(1 for ins in instrs if ins.op == _lib.OP_DOWN)
    assert n_down <= cfg.n_layers * 148 + cfg.n_layers * (cfg.hidden // 4) // 16


def test_attention_sms_take_fewer_gateup_tiles_when_items_are_few():
    """With few attention items per layer (1B, 128 positions: 8 items on 148 SMs)
    each item is charged extra load, so the SMs that run a layer's attention take
    fewer of that layer's gate/up tiles than the other SMs; with an item on nearly
    every SM (8192 positions) no such charge applies."""
    for ctx, charged in ((129, True), (8193, False)):
        instrs, offs, _ = plan_schedule(LLAMA_1B, 1, ctx, 148, max_batch=1, max_seq=ctx)
        fewer = 0
        layers = 0
        for layer in range(1, LLAMA_1B.n_layers):
            att, gu = set(), collections.Counter()
            for s in range(148):
                for ins in instrs[offs[s]:offs[s + 1]]:
                    if ins.layer != layer:
                        continue
                    if ins.op == _lib.OP_ATTN:
                        att.add(s)
                    elif ins.op == _lib.OP_GATEUP:
                        gu[s] += ins.count
            others = [gu[s] for s in range(148) if s not in att]
            if not att or not others:
                continue
            layers += 1
            fewer += max(gu[s] for s in att) < min(others)
        if charged:
            assert fewer == layers, (fewer, layers)
        else:
            assert fewer < layers


def test_planner_refuses_degenerate_arguments():
    """Zero or negative sizes, a batch above the cache's, a context above max_seq,
    an SM count far above any GPU's and a too-small output array are refused with
    MK_ERR_INVALID_ARG; nothing throws through the C boundary."""
    import ctypes
    L = _lib.lib()
    c = _lib.make_config(TINY, 2, 64)
    info = _lib.MkScheduleInfo()

    def rc(batch, ctx, n_sm):
        return L.mk_plan_schedule_host(ctypes.byref(c), batch, ctx, n_sm, None, None, 0, None,
                                       ctypes.byref(info))
    assert rc(1, 64, 148) == 0
    for args in ((0, 64, 148), (-1, 64, 148), (3, 64, 148), (1, 0, 148), (1, 65, 148),
                 (1, 64, 0), (1, 64, -5), (1, 64, 1 << 30)):
        assert rc(*args) == 1, args
    instrs = (_lib.MkInstr * 1)()
    assert L.mk_plan_schedule_host(ctypes.byref(c), 1, 64, 148, None, instrs, 1, None,
                                   ctypes.byref(info)) == 1


@pytest.mark.parametrize("cfg,batch,ctx,n_sm", [
    (TINY, 5, 77, 148), (TINY, 7, 321, 100), (TINY, 8, 1, 148), (TINY, 4, 2048, 132),
    (LLAMA_1B, 2, 1025, 148), (LLAMA_1B, 3, 4097, 148), (LLAMA_1B, 8, 129, 132),
    (LLAMA_3B, 1, 129, 148), (LLAMA_3B, 5, 700, 148), (LLAMA_3B, 6, 1500, 148),
])
def test_plan_valid_across_batches_contexts_and_sm_counts(cfg, batch, ctx, n_sm):
    """Odd batches, a single key, contexts just past a partition boundary, and SM
    counts other than the B200's: the plan covers every tile once, every waited
    count equals the signals it receives, and a simulated step completes."""
    instrs, offs, info = check_plan(cfg, batch, ctx, n_sm)
    ok, ctr = sim(instrs, offs, info, 1, cfg)
    assert ok, "simulated step did not complete"


@pytest.mark.parametrize("cfg,batch,proj,limit", [
    (LLAMA_1B, 1, 0, 16384), (LLAMA_1B, 4, 0, 16384), (LLAMA_1B, 8, 0, 16384),
    (LLAMA_3B, 1, 0, 12288), (LLAMA_3B, 2, 0, 7168), (LLAMA_3B, 5, 0, 7168), (LLAMA_3B, 8, 0, 7168),
    (LLAMA_3B, 2, 1, 12288), (LLAMA_3B, 3, 1, 6144), (LLAMA_3B, 8, 1, 6144), (LLAMA_1B, 8, 1, 16384),
])
def test_context_ceiling_is_the_documented_one(cfg, batch, proj, limit):
    """The largest max_ctx the planner accepts (32 partitions of at most one ring's
    keys, and 512) is the one the header states; one key more is refused."""
    _, _, info = plan_schedule(cfg, batch, limit, 148, max_batch=8, max_seq=limit + 1, proj=proj)
    assert info.n_parts <= 32 and info.n_parts * info.part_keys >= limit
    with pytest.raises(_lib.MkError):
        plan_schedule(cfg, batch, limit + 1, 148, max_batch=8, max_seq=limit + 1, proj=proj)


@pytest.mark.parametrize("cfg,batch,ctx", [(LLAMA_1B, 1, 16384), (LLAMA_3B, 1, 12288), (LLAMA_3B, 8, 7168)])
def test_plans_at_the_context_ceiling_simulate_to_completion(cfg, batch, ctx):
    """At the longest context each shape takes (32 partitions per (sequence, KV
    group)) the plan passes the static checks and its simulated step completes."""
    instrs, offs, info = check_plan(cfg, batch, ctx, 148)
    assert info.n_parts == 32
    ok, _ = sim(instrs, offs, info, 1, cfg)
    assert ok, "simulated step did not complete"


@pytest.mark.parametrize("cfg,batch,n_sm", [(TINY, 2, 37), (TINY, 8, 148), (LLAMA_1B, 8, 148),
                                            (LLAMA_3B, 8, 148), (LLAMA_3B, 3, 100)])
def test_tensor_core_fills_cover_every_weight_once(cfg, batch, n_sm):
    """On the tensor-core path every matvec instruction's fills (one copy of nb
    64-column boxes of a <= 128-row segment) cover each (row, 64-column block) of
    its weight rows exactly once, each fill fits one ring stage, every segment is
    whole 8-row swizzle atoms (the down-projection's at most 64 rows: its tensor
    maps), and the planner's fill counts are these. The bytes streamed are the
    CUDA-core path's, row for row."""
    instrs, offs, info = plan_schedule(cfg, batch, 129, n_sm, max_batch=8, max_seq=129, proj=2)
    assert info.proj == _lib.PROJ_TENSOR_CORES
    _, _, info_cc = plan_schedule(cfg, batch, 129, n_sm, max_batch=8, max_seq=129, proj=1)
    assert info.bytes_per_step == info_cc.bytes_per_step
    sb = info.stage_bytes
    assert sb % 1024 == 0
    k_h, k_o, k_f = cfg.hidden // 64, cfg.n_heads * cfg.head_dim // 64, cfg.ffn // 4 // 64
    qkv_rows = (cfg.n_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    shape = {_lib.OP_QKV: (qkv_rows, k_h), _lib.OP_OPROJ: (cfg.hidden, k_o), _lib.OP_GATEUP: (2 * cfg.ffn, k_h),
             _lib.OP_DOWN: (cfg.hidden, k_f), _lib.OP_LMHEAD: (cfg.vocab, k_h)}
    cov = {}  # (op, layer, chunk) -> hits per (row, 64-column block)
    for ins in instrs:
        if ins.op == _lib.OP_ATTN:
            continue
        g, fills = mma_fills(ins, cfg, sb)
        assert ins.nfill == len(fills)
        for c, rg, seg, kf, boxes, rows, nb in fills:
            # one copy of nb boxes of whole 8-row swizzle atoms, within a stage
            assert nb * rows * 128 <= sb and 8 <= rows <= 128 and rows % 8 == 0
            assert ins.op != _lib.OP_DOWN or rows <= 64
            if ins.op == _lib.OP_GATEUP:
                row0 = 4 * (rg * (cfg.ffn // 8) + ins.first)
            else:
                row0 = 4 * ins.first
            row0 += 128 * seg
            key = (ins.op, ins.layer, c)
            if key not in cov:
                cov[key] = np.zeros(shape[ins.op], np.int32)
            cov[key][row0:row0 + rows, boxes.start:boxes.stop] += 1
    assert all(np.all(v == 1) for v in cov.values())
    want = cfg.n_layers * 4 + 1 + cfg.n_layers * 3  # QKV, O, gate/up, down chunk 0; LM head; down chunks 1-3
    assert len(cov) == want
