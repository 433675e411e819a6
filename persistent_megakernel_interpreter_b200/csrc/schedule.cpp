// Schedule builder: turns one decode step into per-SM instruction lists.
//
// The write-ups arrange every dependency before the run ("Look Ma, No Bubbles"
// summaries: instructions statically ordered per SM) and cut the work into
// tile-sized tasks whose inputs are tracked by counters (Cohere's task list:
// "one tile of one operator" as the scheduling unit, each task waiting only for
// the producers it reads). Here:
//
//  * Work items are emitted in one global order that is a topological order of
//    the step: per layer QKV (per KV group) -> attention partitions -> O-proj ->
//    gate/up (per MLP chunk) -> down (per row block), then the LM head.
//  * Each item goes to the SM whose running byte total is smallest, so every
//    prefix of the step is balanced across SMs to within one item (the
//    wave-quantisation holes of a kernel-per-op engine are filled by the next
//    op's items).
//  * Each SM's list keeps the global order, so every wait refers to work that
//    comes earlier everywhere: with all CTAs resident the step cannot deadlock.
//  * Counter targets are the number of items that signal each counter.
#include <algorithm>
#include <numeric>
#include <queue>
#include <random>
#include <vector>

#include "pack.h"

namespace mk {

uint32_t default_stage_bytes(const Layout& L) {
    uint32_t s = std::max(L.tile_h, std::max(L.tile_o, L.tile_f));
    return (uint32_t)align_up(s, 128);
}

int warp_scratch_floats(const Layout& L, uint32_t stage_bytes) {
    const int kps = (int)(stage_bytes / (4u * (uint32_t)L.d));
    int n = std::max(L.H, L.Q);                 // a matvec input vector
    n = std::max(n, L.F / 4 + 32);              // a down chunk + the running sums
    n = std::max(n, 4 * kps);                   // attention scores
    return (n + 3) / 4 * 4;
}

int stages_for(const Layout& L, uint32_t stage_bytes) {
    const size_t scratch = (size_t)kConsumerWarps * warp_scratch_floats(L, stage_bytes) * sizeof(float);
    const size_t budget = kSmemBudget - 1024 - 16 - scratch;
    return (int)(budget / (stage_bytes + 20));
}

mk_status plan_schedule(const Layout& L, int batch, int max_ctx, int n_sm,
                        const mk_schedule_opts* opts, uint32_t stage_bytes, Plan* out) {
    mk_schedule_opts o{};
    if (opts) o = *opts;
    if (batch < 1 || batch > 8 || max_ctx < 1 || n_sm < 1) return MK_ERR_INVALID_ARG;
    if (stage_bytes == 0) stage_bytes = default_stage_bytes(L);
    if (stage_bytes % 128 || stage_bytes < default_stage_bytes(L)) return MK_ERR_INVALID_ARG;
    const int kps = (int)(stage_bytes / (4u * (uint32_t)L.d));
    const int S = stages_for(L, stage_bytes);
    if (kps < 1 || S < 2) return MK_ERR_UNSUPPORTED;

    // attention partitions
    const int fills_per_seq = (max_ctx + kps - 1) / kps;
    int part_keys;
    if (o.part_keys > 0) {
        if (o.part_keys % kps) return MK_ERR_INVALID_ARG;
        part_keys = o.part_keys;
    } else {
        const int want = std::max(1, (2 * n_sm + batch * L.nkv - 1) / (batch * L.nkv));
        part_keys = kps * ((fills_per_seq + want - 1) / want);
    }
    const int n_parts = (max_ctx + part_keys - 1) / part_keys;

    const int tq = o.tiles_qkv > 0 ? o.tiles_qkv : 2;
    const int to = o.tiles_o > 0 ? o.tiles_o : 2;
    const int tg = o.tiles_gateup > 0 ? o.tiles_gateup : 4;
    int rd = o.rowblocks_down > 0 ? o.rowblocks_down : 1;
    const int tl = o.tiles_lm > 0 ? o.tiles_lm : 8;
    if (batch > 1) rd = 1;
    if (rd > 8) return MK_ERR_INVALID_ARG;
    const int gu_tiles_chunk = L.F / 8;  // gate/up tiles (2 outputs each) per MLP chunk
    if (gu_tiles_chunk % tg) return MK_ERR_INVALID_ARG;

    // counters
    int nc = 0;
    std::vector<int> c_qkv(L.L), c_part(L.L), c_attn(L.L), c_o(L.L), c_h(L.L), c_down(L.L);
    for (int l = 0; l < L.L; ++l) {
        c_qkv[l] = nc; nc += L.nkv;
        c_part[l] = nc; nc += batch * L.nkv;
        c_attn[l] = nc++;
        c_o[l] = nc++;
        c_h[l] = nc; nc += 4;
        c_down[l] = nc++;
    }
    const int c_lm = nc++;

    struct Unit {
        mk_instr in;
        uint64_t bytes;
    };
    std::vector<Unit> units;
    auto mk_in = [](uint16_t op, int l) {
        mk_instr in{};
        in.op = op;
        in.layer = (uint16_t)l;
        in.wait_ctr = MK_NO_COUNTER;
        in.signal_ctr = MK_NO_COUNTER;
        in.aux_ctr = MK_NO_COUNTER;
        return in;
    };
    const uint32_t kv_key_bytes = 2u * (uint32_t)L.d * 2u;  // K and V of one key
    for (int l = 0; l < L.L; ++l) {
        for (int g = 0; g < L.nkv; ++g)
            for (int t = 0; t < L.tiles_per_group; t += tq) {
                mk_instr in = mk_in(MK_OP_QKV, l);
                in.group = (uint16_t)g;
                in.first = (uint32_t)(g * L.tiles_per_group + t);
                in.count = (uint32_t)std::min(tq, L.tiles_per_group - t);
                in.nfill = in.count;
                if (l > 0) in.wait_ctr = (uint32_t)c_down[l - 1];
                in.signal_ctr = (uint32_t)(c_qkv[l] + g);
                units.push_back({in, (uint64_t)in.count * L.tile_h});
            }
        for (int b = 0; b < batch; ++b)
            for (int g = 0; g < L.nkv; ++g)
                for (int j = 0; j < n_parts; ++j) {
                    mk_instr in = mk_in(MK_OP_ATTN, l);
                    in.batch = (uint16_t)b;
                    in.group = (uint16_t)g;
                    in.first = (uint32_t)(j * part_keys);
                    in.count = (uint32_t)std::min(part_keys, max_ctx - j * part_keys);
                    in.nfill = (in.count + kps - 1) / kps;
                    in.wait_ctr = (uint32_t)(c_qkv[l] + g);
                    in.signal_ctr = (uint32_t)(c_part[l] + b * L.nkv + g);
                    in.aux_ctr = (uint32_t)c_attn[l];
                    in.aux_n = (uint32_t)n_parts;
                    units.push_back({in, (uint64_t)in.count * kv_key_bytes});
                }
        for (int t = 0; t < L.H / 4; t += to) {
            mk_instr in = mk_in(MK_OP_OPROJ, l);
            in.first = (uint32_t)t;
            in.count = (uint32_t)std::min(to, L.H / 4 - t);
            in.nfill = in.count;
            in.wait_ctr = (uint32_t)c_attn[l];
            in.signal_ctr = (uint32_t)c_o[l];
            units.push_back({in, (uint64_t)in.count * L.tile_o});
        }
        for (int c = 0; c < 4; ++c)
            for (int t = 0; t < gu_tiles_chunk; t += tg) {
                mk_instr in = mk_in(MK_OP_GATEUP, l);
                in.group = (uint16_t)c;
                in.first = (uint32_t)(c * gu_tiles_chunk + t);
                in.count = (uint32_t)tg;
                in.nfill = in.count;
                in.wait_ctr = (uint32_t)c_o[l];
                in.signal_ctr = (uint32_t)(c_h[l] + c);
                units.push_back({in, (uint64_t)in.count * L.tile_h});
            }
        for (int r = 0; r < L.H / 4; r += rd) {
            mk_instr in = mk_in(MK_OP_DOWN, l);
            in.first = (uint32_t)r;
            in.count = (uint32_t)std::min(rd, L.H / 4 - r);
            in.nfill = 4 * in.count;
            in.wait_ctr = (uint32_t)c_h[l];
            in.signal_ctr = (uint32_t)c_down[l];
            units.push_back({in, (uint64_t)in.nfill * L.tile_f});
        }
    }
    for (int t = 0; t < L.V / 4; t += tl) {
        mk_instr in = mk_in(MK_OP_LMHEAD, L.L - 1);
        in.first = (uint32_t)t;
        in.count = (uint32_t)std::min(tl, L.V / 4 - t);
        in.nfill = in.count;
        in.wait_ctr = (uint32_t)c_down[L.L - 1];
        in.signal_ctr = (uint32_t)c_lm;
        units.push_back({in, (uint64_t)in.count * L.tile_h});
    }

    // targets: how many items signal each counter per step
    std::vector<uint32_t> signals(nc, 0);
    for (const Unit& u : units)
        if (u.in.signal_ctr != MK_NO_COUNTER) signals[u.in.signal_ctr]++;
    for (int l = 0; l < L.L; ++l) signals[c_attn[l]] = (uint32_t)(batch * L.nkv);  // merges
    for (Unit& u : units) {
        if (u.in.wait_ctr == MK_NO_COUNTER) continue;
        u.in.wait_n = signals[u.in.wait_ctr];
        if (u.in.op == MK_OP_DOWN)
            for (int c = 1; c < 4; ++c)
                if (signals[u.in.wait_ctr + c] != u.in.wait_n) return MK_ERR_UNSUPPORTED;
    }

    if (o.test_drop_item > 0) {
        if ((size_t)o.test_drop_item > units.size()) return MK_ERR_INVALID_ARG;
        units.erase(units.begin() + (o.test_drop_item - 1));
    }

    // placement: smallest running total first
    constexpr uint64_t kItemOverhead = 2048;  // byte-equivalent cost of one item's sync
    std::vector<std::vector<mk_instr>> lists(n_sm);
    std::vector<uint64_t> load(n_sm, 0);
    std::vector<uint32_t> tiebreak(n_sm);
    std::iota(tiebreak.begin(), tiebreak.end(), 0u);
    if (o.seed) {
        std::mt19937 rng(o.seed);
        std::shuffle(tiebreak.begin(), tiebreak.end(), rng);
    }
    using Key = std::pair<uint64_t, uint32_t>;  // (load, tiebreak rank)
    std::priority_queue<Key, std::vector<Key>, std::greater<Key>> pq;
    std::vector<int> sm_of_rank(n_sm);
    for (int s = 0; s < n_sm; ++s) {
        sm_of_rank[tiebreak[s]] = s;
        pq.push({0, tiebreak[s]});
    }
    uint64_t total = 0;
    for (const Unit& u : units) {
        Key k = pq.top();
        pq.pop();
        const int s = sm_of_rank[k.second];
        lists[s].push_back(u.in);
        load[s] += u.bytes;
        total += u.bytes;
        pq.push({k.first + u.bytes + kItemOverhead, k.second});
    }

    Plan P;
    P.sm_off.push_back(0);
    for (int s = 0; s < n_sm; ++s) {
        uint32_t seq = 0;
        for (mk_instr in : lists[s]) {
            in.seq = seq;
            seq += in.nfill;
            P.instrs.push_back(in);
        }
        P.sm_off.push_back((int32_t)P.instrs.size());
    }
    mk_schedule_info& I = P.info;
    I = mk_schedule_info{};
    I.n_sm = n_sm;
    I.batch = batch;
    I.max_ctx = max_ctx;
    I.part_keys = part_keys;
    I.n_parts = n_parts;
    I.keys_per_stage = kps;
    I.stage_bytes = (int32_t)stage_bytes;
    I.n_stages = S;
    I.n_counters = nc;
    I.n_instr = (int32_t)P.instrs.size();
    I.bytes_per_step = total;
    I.max_sm_bytes = *std::max_element(load.begin(), load.end());
    I.min_sm_bytes = *std::min_element(load.begin(), load.end());
    *out = std::move(P);
    return MK_OK;
}

}  // namespace mk

extern "C" mk_status mk_plan_schedule_host(const mk_config* cfg, int batch, int max_ctx, int n_sm,
                                           const mk_schedule_opts* opts, mk_instr* instr_out,
                                           size_t cap, int32_t* sm_offsets, mk_schedule_info* info) {
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
