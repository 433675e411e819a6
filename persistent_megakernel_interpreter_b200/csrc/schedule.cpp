// Schedule builder: turns one decode step into per-SM instruction lists.
//
// The write-ups arrange every dependency before the run ("Look Ma, No Bubbles"
// summaries: instructions statically ordered per SM) and cut the work into
// tile-sized tasks whose inputs are tracked by counters (Cohere's task list:
// "one tile of one operator" as the scheduling unit, each task waiting only for
// the producers it reads). Here:
//
//  * Each op is cut into units (4-row tiles, down-projection row blocks,
//    attention items); every unit goes to the SM whose running byte total is
//    smallest, so every prefix of the step is balanced across SMs to within one
//    unit (the wave-quantisation holes of a kernel-per-op engine are filled by
//    the next op's units). An SM's units of one op form one contiguous range,
//    split only where a counter boundary (KV group, MLP chunk) falls.
//  * Ops are appended in one global topological order: per layer QKV (per KV
//    group) -> attention items -> O-proj -> gate/up (per MLP chunk) -> down,
//    then the LM head. Each SM's list keeps that order, so every wait refers to
//    work that comes earlier everywhere: with all CTAs resident the step cannot
//    deadlock.
//  * Counter targets are the number of jobs that signal each counter, except the
//    attention counter of a layer: it counts query heads whose output is final
//    (batch * n_heads). Each (sequence, KV group) pair also has an arrival
//    counter that its items' heads increment after storing a split-K partial;
//    the item that completes it merges the pair. No instruction waits on it.
#include <algorithm>
#include <new>
#include <numeric>
#include <queue>
#include <random>
#include <vector>

#include "pack.h"

namespace mk {

uint32_t default_stage_bytes(const Layout& L, bool mma) {
    // the tensor-core path streams 64-column boxes, not 4-row tiles: a stage holds
    // one box of a full 128-row segment (16 KB; as many boxes of a shorter one)
    if (mma) return kMmaRows * kBoxK * 2u;
    const uint32_t s = std::max(L.tile_h, std::max(L.tile_o, L.tile_f));
    return (uint32_t)align_up(s, 128);
}

SlotPlan slot_plan(const Layout& L, int batch, uint32_t stage_bytes, bool mma) {
    SlotPlan sp{};
    sp.keys_per_stage = (int)(stage_bytes / (4u * (uint32_t)L.d));
    sp.vec_floats = (uint32_t)align_up((size_t)std::max(std::max(L.H, L.Q), L.F / 4), 64);
    sp.item_bytes = attn_item_bytes(L.group, L.d) + 4u * attn_scratch_floats(L.d);
    // per sequence: the input vector; then per sequence (QKV jobs) the RoPE row
    // cos[d/2], sin[d/2] and the position; then per sequence (O-proj and down
    // jobs) the residual rows the job updates. An attention job: its item's q and
    // new key/value, then the item's scratch. On the tensor-core path the input
    // vectors are the MMA operand instead: 16 rows (each sequence's high and low
    // bf16 parts) of vec_floats bf16 each, whatever the batch.
    const uint32_t aux = (uint32_t)batch * ((uint32_t)L.d + 4u + (uint32_t)kMaxResidRows) * 4u;
    if (mma) {
        sp.aux_floats = sp.vec_floats * 8u;
        sp.slot_bytes = (uint32_t)align_up(std::max(sp.vec_floats * 32u + aux, sp.item_bytes), 1024);
    } else {
        sp.aux_floats = (uint32_t)batch * sp.vec_floats;
        sp.slot_bytes = align16(std::max((uint32_t)batch * sp.vec_floats * 4u + aux, sp.item_bytes));
    }
    // the most job slots that leave at least 8 stages (an attention item's keys all
    // sit in the ring at once), else at least 4; on the CUDA-core path the stage
    // count is a multiple of 4, so each stage's fills belong to one mover warp
    sp.xs_slots = 0;
    for (int min_s = 8; min_s >= kMoveWarps && sp.xs_slots == 0; min_s -= 4) {
        for (int ns = 3; ns >= 1; --ns) {
            int S = 0;
            while (smem_layout(S + 1, stage_bytes, ns, sp.slot_bytes, mma).total + 1024 <= kSmemBudget)
                ++S;
            if (!mma) S -= S % kMoveWarps;
            if (S >= min_s) {
                sp.xs_slots = ns;
                sp.stages = S;
                break;
            }
        }
    }
    if (sp.xs_slots == 0) {  // nothing fits: reported by the caller (fewer than 4 stages)
        sp.xs_slots = 1;
        sp.stages = 0;
    }
    sp.smem_bytes = smem_layout(sp.stages, stage_bytes, sp.xs_slots, sp.slot_bytes, mma).total;
    return sp;
}

bool use_mma(const Layout& L, int batch, const mk_schedule_opts* opts) {
    // The default at batch > 1: measured on the 3B-style shape at batch 8 and 2048
    // positions the tensor-core step takes 6.30 ms against 6.63 ms on the CUDA cores
    // (same B200). The path takes rows in pairs of 4-row tiles (segments of a
    // multiple of 8 rows), so the LM head's vocabulary must be a multiple of 8.
    return batch > 1 && L.V % 8 == 0 && !(opts && opts->proj == MK_PROJ_CUDA_CORES);
}

// the most SMs a plan may spread over (a B200 has 148)
constexpr int kMaxPlanSms = 1024;

mk_status plan_schedule(const Layout& L, int batch, int max_ctx, int n_sm,
                        const mk_schedule_opts* opts, uint32_t stage_bytes, Plan* out) {
    mk_schedule_opts o{};
    if (opts) o = *opts;
    if (batch < 1 || batch > kMaxBatch || max_ctx < 1 || n_sm < 1 || n_sm > kMaxPlanSms)
        return MK_ERR_INVALID_ARG;
    if (o.proj < MK_PROJ_AUTO || o.proj > MK_PROJ_TENSOR_CORES) return MK_ERR_INVALID_ARG;
    const bool mma = use_mma(L, batch, &o);
    // units of work: single 4-row tiles, or pairs of them on the tensor-core path
    // (every segment a multiple of 8 rows: whole 1024-byte swizzle atoms)
    const int gran = mma ? 2 : 1;
    if (stage_bytes == 0) stage_bytes = default_stage_bytes(L, mma);
    if (stage_bytes % (mma ? 1024 : 128) || stage_bytes < default_stage_bytes(L, mma)) return MK_ERR_INVALID_ARG;
    const SlotPlan sp = slot_plan(L, batch, stage_bytes, mma);
    const int kps = sp.keys_per_stage;
    if (kps < 1 || sp.stages < kMoveWarps) return MK_ERR_UNSUPPORTED;
    // an attention item reads each pass of 256 / head_dim keys from one fill, so a
    // ring stage holds whole passes
    const int attn_pass = std::max(1, 256 / L.d);
    if (kps % attn_pass) return MK_ERR_UNSUPPORTED;

    // attention partitions: one per (sequence, KV group) up to kSingleItemKeys
    // keys; for longer contexts as many as there are SMs for (an item's time is
    // mostly per key, and the merge of several partitions costs about as much as
    // ~340 keys of one item, measured), but no more items than SMs and at most
    // kMaxParts per pair, the merge's limit. An item's fills must all sit in the
    // ring at once and its scores in the item scratch, so a partition holds at
    // most min(kMaxItemKeys, stages * keys_per_stage) keys. A partition is a
    // multiple of 8 keys up to one ring stage, then a multiple of whole stages.
    constexpr int kSingleItemKeys = 320;
    const int max_item = std::min(kMaxItemKeys, sp.stages * kps);
    int part_keys;
    if (o.part_keys > 0) {
        if (o.part_keys > kps && o.part_keys % kps) return MK_ERR_INVALID_ARG;
        if (o.part_keys > max_item) return MK_ERR_INVALID_ARG;
        part_keys = o.part_keys;
    } else {
        const int pairs = batch * L.nkv;
        const int cap = std::max(1, std::min(kMaxParts, n_sm / pairs));
        int parts = max_ctx > kSingleItemKeys ? cap : 1;
        parts = std::max(parts, (max_ctx + max_item - 1) / max_item);
        const int want = std::max((max_ctx + parts - 1) / parts, (max_ctx + kMaxParts - 1) / kMaxParts);
        part_keys = want <= kps ? (want + 7) / 8 * 8 : (want + kps - 1) / kps * kps;
        if (part_keys > max_item) part_keys = max_item / kps * kps;
    }
    const int n_parts = (max_ctx + part_keys - 1) / part_keys;
    if (n_parts > kMaxParts) return MK_ERR_INVALID_ARG;
    int down_cap = std::max(1, std::min(o.rowblocks_down > 0 ? o.rowblocks_down : kMaxDownRows, kMaxDownRows));
    down_cap = (down_cap + gran - 1) / gran * gran;

    // counters
    int nc = 0;
    std::vector<int> c_qkv(L.L), c_part(L.L), c_arr(L.L), c_o(L.L), c_h(L.L), c_down(L.L);
    for (int l = 0; l < L.L; ++l) {
        c_qkv[l] = nc; nc += L.nkv;
        c_part[l] = nc++;
        c_arr[l] = nc; nc += batch * L.nkv;  // per (sequence, group): heads' partials stored
        c_o[l] = nc++;
        c_h[l] = nc; nc += 4;
        c_down[l] = nc++;
    }
    const int c_lm = nc++;

    // placement state
    std::vector<std::vector<mk_instr>> lists(n_sm);
    std::vector<uint64_t> load(n_sm, 0);
    std::vector<uint32_t> rank(n_sm);
    std::iota(rank.begin(), rank.end(), 0u);
    if (o.seed) {
        std::mt19937 rng(o.seed);
        std::shuffle(rank.begin(), rank.end(), rng);
    }
    constexpr uint64_t kJobOverhead = 4096;  // byte-equivalent cost of one job's sync and prep
    // Byte-equivalent cost of running an attention item, besides its KV bytes, when
    // a layer has few items: while the item's SM computes it (and its ring holds KV
    // fills), the other SMs' rings fill with the layer's gate/up weights, so the
    // item's SM should take fewer of them. Measured on the 1B step at 128 positions
    // (8 items): 0 / 32 / 64 / 128 / 160 / 192 / 256 KB -> 692 / 682 / 683 / 680 /
    // 682 / 682 / 688 us. With an item on (nearly) every SM the charge only
    // overloads the SMs without one (1B at 8192 positions: 900 -> 987 us), so it
    // applies to few items only.
    const uint64_t attn_item_cost = (uint64_t)batch * L.nkv * n_parts * 8 <= (uint64_t)n_sm ? 128 * 1024 : 0;
    using Key = std::pair<uint64_t, uint32_t>;  // (load, rank)
    std::vector<int> sm_of_rank(n_sm);
    for (int s = 0; s < n_sm; ++s) sm_of_rank[rank[s]] = s;
    // Units of one op, each costing `unit_cost`: how many each SM takes (the SM
    // with the smallest running total takes the next unit).
    auto share = [&](int units, uint64_t unit_cost) {
        std::priority_queue<Key, std::vector<Key>, std::greater<Key>> pq;
        for (int s = 0; s < n_sm; ++s) pq.push({load[s], rank[s]});
        std::vector<int> cnt(n_sm, 0);
        for (int u = 0; u < units; ++u) {
            Key k = pq.top();
            pq.pop();
            const int s = sm_of_rank[k.second];
            cnt[s]++;
            const uint64_t add = unit_cost + (cnt[s] == 1 ? kJobOverhead : 0);
            load[s] += add;
            pq.push({k.first + add, k.second});
        }
        return cnt;
    };
    // the same in units of `gran` tiles (every total here is a multiple of 2); counts in tiles
    auto share_g = [&](int tiles, uint64_t tile_cost) {
        std::vector<int> cnt = share(tiles / gran, tile_cost * gran);
        for (int& c : cnt) c *= gran;
        return cnt;
    };
    auto mk_in = [](uint16_t op, int l) {
        mk_instr in{};
        in.op = op;
        in.layer = (uint16_t)l;
        in.wait_ctr = MK_NO_COUNTER;
        in.signal_ctr = MK_NO_COUNTER;
        in.job_items = 1;
        return in;
    };
    // Contiguous ranges [start, start+cnt) in SM order, cut at multiples of `cut`
    // (counter boundaries) and at `cap` units per instruction.
    auto emit_ranges = [&](const std::vector<int>& cnt, int cut, int cap, auto&& make) {
        int start = 0;
        for (int s = 0; s < n_sm; ++s) {
            int a = start, e = start + cnt[s];
            while (a < e) {
                int b = std::min(e, (a / cut + 1) * cut);
                b = std::min(b, a + cap);
                lists[s].push_back(make(a, b - a));
                a = b;
            }
            start = e;
        }
    };
    std::vector<uint32_t> signals(nc, 0);
    std::vector<int> att_sm;  // the SM of each attention item, chosen in layer 0
    const uint32_t kv_key_bytes = 2u * (uint32_t)L.d * 2u;
    const int gu_chunk = L.F / 8;
    for (int l = 0; l < L.L; ++l) {
        // QKV: tiles grouped by KV group
        // One job per SM even where its range crosses a KV-group boundary (one
        // RMSNorm of x); the job then signals each group it touched.
        emit_ranges(share_g(L.nkv * L.tiles_per_group, L.tile_h), 1 << 30, 1 << 30,
                    [&](int a, int n) {
                        mk_instr in = mk_in(MK_OP_QKV, l);
                        in.group = (uint16_t)(a / L.tiles_per_group);
                        in.first = (uint32_t)a;
                        in.count = in.nfill = (uint32_t)n;
                        if (l > 0) in.wait_ctr = (uint32_t)c_down[l - 1];
                        in.signal_ctr = (uint32_t)(c_qkv[l] + in.group);
                        in.aux1 = (uint32_t)((a + n - 1) / L.tiles_per_group - in.group + 1);
                        for (uint32_t k = 0; k < in.aux1; ++k) signals[in.signal_ctr + k]++;
                        return in;
                    });
        // attention items, each its own job on the SM with the fewest items of
        // this layer so far, then the least-loaded one: an SM that runs two items
        // runs them one after the other, on the layer's critical path. Later
        // layers put each item on the SM the first layer chose for it: the
        // attention code then stays in those SMs' instruction caches, where a
        // new SM each layer would fetch it from L2 on the critical path.
        std::vector<int> n_att(n_sm, 0);
        int item = 0;
        for (int b = 0; b < batch; ++b)
            for (int g = 0; g < L.nkv; ++g)
                for (int j = 0; j < n_parts; ++j, ++item) {
                    int best = 0;
                    if (l > 0) {
                        best = att_sm[item];
                    } else {
                        for (int s = 1; s < n_sm; ++s)
                            if (n_att[s] < n_att[best] ||
                                (n_att[s] == n_att[best] &&
                                 (load[s] < load[best] || (load[s] == load[best] && rank[s] < rank[best]))))
                                best = s;
                        att_sm.push_back(best);
                    }
                    n_att[best]++;
                    mk_instr in = mk_in(MK_OP_ATTN, l);
                    in.batch = (uint16_t)b;
                    in.group = (uint16_t)g;
                    in.first = (uint32_t)(j * part_keys);
                    in.count = (uint32_t)std::min(part_keys, max_ctx - j * part_keys);
                    in.nfill = (in.count + kps - 1) / kps;
                    in.wait_ctr = (uint32_t)(c_qkv[l] + g);
                    in.signal_ctr = (uint32_t)c_part[l];
                    in.aux0 = (uint32_t)(c_arr[l] + b * L.nkv + g);
                    lists[best].push_back(in);
                    load[best] += (uint64_t)in.count * kv_key_bytes + kJobOverhead + attn_item_cost;
                }
        // each (sequence, group) pair signals each of its query heads once, when
        // the head's output is final
        signals[c_part[l]] += (uint32_t)(batch * L.nq);
        emit_ranges(share_g(L.H / 4, L.tile_o), 1 << 30, kMaxResidRows / 4, [&](int a, int n) {
            mk_instr in = mk_in(MK_OP_OPROJ, l);
            in.first = (uint32_t)a;
            in.count = in.nfill = (uint32_t)n;
            in.wait_ctr = (uint32_t)c_part[l];
            in.signal_ctr = (uint32_t)c_o[l];
            signals[in.signal_ctr]++;
            return in;
        });
        // gate/up, chunk-major: every SM takes the same slice [a, a + n) of each of
        // the four MLP chunks and works through the chunks in order, so chunks 0..2
        // of h are complete well before the layer's last gate/up tile; one job per SM,
        // which counts once on each chunk counter
        {
            const std::vector<int> cnt = share_g(gu_chunk, 4ull * L.tile_h);
            int start = 0;
            for (int s = 0; s < n_sm; ++s) {
                const int n = cnt[s];
                if (n == 0) continue;
                mk_instr in = mk_in(MK_OP_GATEUP, l);
                in.first = (uint32_t)start;
                in.count = in.nfill = 4u * (uint32_t)n;
                in.aux0 = (uint32_t)n;
                in.wait_ctr = (uint32_t)c_o[l];
                in.signal_ctr = (uint32_t)c_h[l];
                in.aux1 = 4;
                for (uint32_t k = 0; k < 4; ++k) signals[in.signal_ctr + k]++;
                lists[s].push_back(in);
                start += n;
            }
        }
        emit_ranges(share_g(L.H / 4, 4ull * L.tile_f), 1 << 30, down_cap,
                    [&](int a, int n) {
                        mk_instr in = mk_in(MK_OP_DOWN, l);
                        in.first = (uint32_t)a;
                        in.count = (uint32_t)n;
                        in.nfill = 4u * (uint32_t)n;
                        in.wait_ctr = (uint32_t)c_h[l];
                        in.signal_ctr = (uint32_t)c_down[l];
                        signals[in.signal_ctr]++;
                        return in;
                    });
    }
    uint32_t lm_ord = 0;  // LM-head instructions, numbered in SM order (greedy selection slots)
    emit_ranges(share_g(L.V / 4, L.tile_h), 1 << 30, 1 << 30, [&](int a, int n) {
        mk_instr in = mk_in(MK_OP_LMHEAD, L.L - 1);
        in.aux0 = lm_ord++;
        in.first = (uint32_t)a;
        in.count = in.nfill = (uint32_t)n;
        in.wait_ctr = (uint32_t)c_down[L.L - 1];
        in.signal_ctr = (uint32_t)c_lm;
        signals[in.signal_ctr]++;
        return in;
    });

    // wait targets; fill numbering; the failure-injection hook
    Plan P;
    P.sm_off.push_back(0);
    uint64_t total = 0;
    for (int s = 0; s < n_sm; ++s) {
        uint32_t seq = 0;
        for (mk_instr in : lists[s]) {
            if (in.wait_ctr != MK_NO_COUNTER) in.wait_n = signals[in.wait_ctr];
            if (mma && in.op != MK_OP_ATTN)  // the same rows, streamed as 64-column boxes
                in.nfill = mma_geom(in.op, in.count, in.aux0, L.H, L.Q, L.F, stage_bytes).nfill();
            in.seq = seq;
            seq += in.nfill;
            P.instrs.push_back(in);
        }
        P.sm_off.push_back((int32_t)P.instrs.size());
    }
    for (mk_instr& in : P.instrs)
        if (in.op == MK_OP_DOWN) {
            // each MLP chunk may have a different number of gate/up jobs
            in.wait_n = signals[in.wait_ctr];
            in.aux0 = signals[in.wait_ctr + 1] | (signals[in.wait_ctr + 2] << 16);
            in.aux1 = signals[in.wait_ctr + 3];
        }
    if (o.test_drop_item > 0) {
        if ((size_t)o.test_drop_item > P.instrs.size()) return MK_ERR_INVALID_ARG;
        // the job's work still runs, but its completion is never signalled
        mk_instr& in = P.instrs[o.test_drop_item - 1];
        in.signal_ctr = MK_NO_COUNTER;
    }
    for (int s = 0; s < n_sm; ++s) total += load[s];
    mk_schedule_info& I = P.info;
    I = mk_schedule_info{};
    I.n_sm = n_sm;
    I.batch = batch;
    I.max_ctx = max_ctx;
    I.part_keys = part_keys;
    I.n_parts = n_parts;
    I.keys_per_stage = kps;
    I.stage_bytes = (int32_t)stage_bytes;
    I.n_stages = sp.stages;
    I.n_counters = nc;
    I.n_instr = (int32_t)P.instrs.size();
    uint64_t bytes = 0;
    for (const mk_instr& in : P.instrs) {
        if (in.op == MK_OP_ATTN) bytes += (uint64_t)in.count * kv_key_bytes;
        else if (in.op == MK_OP_DOWN) bytes += 4ull * in.count * L.tile_f;
        else if (in.op == MK_OP_OPROJ) bytes += (uint64_t)in.count * L.tile_o;
        else bytes += (uint64_t)in.count * L.tile_h;
    }
    I.bytes_per_step = bytes;
    I.proj = mma ? MK_PROJ_TENSOR_CORES : MK_PROJ_CUDA_CORES;
    I.max_sm_bytes = *std::max_element(load.begin(), load.end());
    I.min_sm_bytes = *std::min_element(load.begin(), load.end());
    (void)total;
    *out = std::move(P);
    return MK_OK;
}

// mk_plan_schedule_host's body (the C entry point below keeps exceptions inside)
mk_status plan_schedule_host(const mk_config* cfg, int batch, int max_ctx, int n_sm, const mk_schedule_opts* opts,
                             mk_instr* instr_out, size_t cap, int32_t* sm_offsets, mk_schedule_info* info) {
    if (!cfg) return MK_ERR_INVALID_ARG;
    mk::Layout L;
    if (!mk::make_layout(*cfg, &L, nullptr)) return MK_ERR_UNSUPPORTED;
    if (batch > cfg->max_batch || max_ctx > cfg->max_seq) return MK_ERR_INVALID_ARG;
    mk::Plan P;
    const mk_status st = mk::plan_schedule(L, batch, max_ctx, n_sm, opts, 0, &P);
    if (st != MK_OK) return st;
    if (info) *info = P.info;
    if (sm_offsets) std::copy(P.sm_off.begin(), P.sm_off.end(), sm_offsets);
    if (instr_out) {
        if (cap < P.instrs.size()) return MK_ERR_INVALID_ARG;
        std::copy(P.instrs.begin(), P.instrs.end(), instr_out);
    }
    return MK_OK;
}
}  // namespace mk

extern "C" mk_status mk_plan_schedule_host(const mk_config* cfg, int batch, int max_ctx, int n_sm,
                                           const mk_schedule_opts* opts, mk_instr* instr_out,
                                           size_t cap, int32_t* sm_offsets, mk_schedule_info* info) {
    try {
        return mk::plan_schedule_host(cfg, batch, max_ctx, n_sm, opts, instr_out, cap, sm_offsets, info);
    } catch (const std::bad_alloc&) {
        return MK_ERR_OUT_OF_MEMORY;
    } catch (...) {
        return MK_ERR_INVALID_ARG;
    }
}
