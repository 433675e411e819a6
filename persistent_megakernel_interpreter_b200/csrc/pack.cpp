// Weight packer: the row order and tiling of every matrix as the kernels read
// it (documented with mk_pack_weights_host in mk.h). The packer is a list of
// (destination offset, source pointer, bytes) copies -- a pure bit copy -- run
// by a gather kernel on the device (mk_create) or by memcpy on the host.
#include <string.h>

#include <initializer_list>
#include <vector>

#include "pack.h"

namespace mk {

namespace {
// the largest hidden size, ffn, vocabulary and max_seq a configuration may give (the
// kernels further limit hidden and ffn to their instantiated shapes); they keep every
// host-side product of dimensions far from int overflow
constexpr int kMaxHidden = 1 << 16;
constexpr int kMaxFfn = 1 << 18;
constexpr int kMaxVocab = 1 << 24;
constexpr int kMaxSeq = 1 << 20;
}  // namespace

bool make_layout(const mk_config& c, Layout* out, const char** why) {
    auto fail = [&](const char* m) {
        if (why) *why = m;
        return false;
    };
    if (c.n_layers <= 0 || c.n_layers > kMaxLayers) return fail("n_layers out of range");
    if (c.hidden <= 0 || c.n_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim <= 0 || c.ffn <= 0 ||
        c.vocab <= 0)
        return fail("non-positive dimension");
    if (c.n_heads % c.n_kv_heads) return fail("n_heads must be a multiple of n_kv_heads");
    if (c.head_dim != 64 && c.head_dim != 128) return fail("head_dim must be 64 or 128");
    const int group = c.n_heads / c.n_kv_heads;
    if (group > 4) return fail("more than 4 query heads per KV head");
    if (c.n_heads > 32) return fail("more than 32 query heads");
    if (c.hidden % 256) return fail("hidden must be a multiple of 256");
    if ((c.n_heads * c.head_dim) % 256) return fail("n_heads*head_dim must be a multiple of 256");
    if (c.ffn % 1024) return fail("ffn must be a multiple of 1024");
    if (c.vocab % 4) return fail("vocab must be a multiple of 4");
    if (c.max_batch < 1 || c.max_batch > 8) return fail("max_batch must be in [1, 8]");
    if (c.max_seq < 1) return fail("max_seq must be positive");
    if (c.hidden > kMaxHidden || c.ffn > kMaxFfn || c.vocab > kMaxVocab || c.max_seq > kMaxSeq)
        return fail("a dimension is above the supported maximum");
    if (!(c.rms_eps >= 0.0f) || !(c.rope_theta > 0.0)) return fail("bad eps or rope_theta");
    Layout L{};
    L.L = c.n_layers; L.H = c.hidden; L.nq = c.n_heads; L.nkv = c.n_kv_heads; L.d = c.head_dim;
    L.F = c.ffn; L.V = c.vocab; L.group = group;
    L.Q = c.n_heads * c.head_dim;
    L.KVD = c.n_kv_heads * c.head_dim;
    L.qkv_rows = L.Q + 2 * L.KVD;
    L.tiles_per_group = (group + 2) * (c.head_dim / 4);
    L.tile_h = (uint32_t)(4 * L.H * 2);
    L.tile_o = (uint32_t)(4 * L.Q * 2);
    L.tile_f = (uint32_t)(4 * (L.F / 4) * 2);
    size_t off = 0;
    L.off_embed = off;
    off = align_up(off + (size_t)L.V * L.H * 2, 256);
    L.off_layer0 = off;
    size_t rel = 0;
    L.rel_qkv = rel;
    rel = align_up(rel + (size_t)L.qkv_rows * L.H * 2, 256);
    L.rel_o = rel;
    rel = align_up(rel + (size_t)L.H * L.Q * 2, 256);
    L.rel_gu = rel;
    rel = align_up(rel + (size_t)2 * L.F * L.H * 2, 256);
    L.rel_down = rel;
    rel = align_up(rel + (size_t)L.H * L.F * 2, 256);
    L.layer_stride = rel;
    off += (size_t)L.L * L.layer_stride;
    L.off_norms = off;
    off = align_up(off + (size_t)(2 * L.L + 1) * L.H * 2, 256);
    L.total = off;
    *out = L;
    return true;
}

namespace {
constexpr size_t kMaxSeg = 1 << 20;  // split long copies so the gather kernel spreads them

void add(std::vector<Segment>& v, size_t dst, const void* src, size_t bytes) {
    const uint8_t* s = static_cast<const uint8_t*>(src);
    while (bytes > 0) {
        const size_t n = bytes < kMaxSeg ? bytes : kMaxSeg;
        v.push_back(Segment{dst, s, (uint32_t)n, 0});
        dst += n;
        s += n;
        bytes -= n;
    }
}
}  // namespace

std::vector<Segment> pack_segments(const Layout& L, const mk_weights& w) {
    std::vector<Segment> v;
    const size_t row_h = (size_t)L.H * 2;
    add(v, L.off_embed, w.embed, (size_t)L.V * row_h);
    for (int l = 0; l < L.L; ++l) {
        const size_t lb = L.off_layer0 + (size_t)l * L.layer_stride;
        // QKV, grouped by KV head; RoPE pairs kept inside one tile
        size_t dst = lb + L.rel_qkv;
        const uint8_t* wq = static_cast<const uint8_t*>(w.wq[l]);
        const uint8_t* wk = static_cast<const uint8_t*>(w.wk[l]);
        const uint8_t* wv = static_cast<const uint8_t*>(w.wv[l]);
        for (int g = 0; g < L.nkv; ++g) {
            for (int hs = 0; hs < L.group + 2; ++hs) {
                const uint8_t* head;
                if (hs < L.group) head = wq + (size_t)(g * L.group + hs) * L.d * row_h;
                else if (hs == L.group) head = wk + (size_t)g * L.d * row_h;
                else head = wv + (size_t)g * L.d * row_h;
                for (int j = 0; j < L.d / 4; ++j) {
                    for (int r = 0; r < 4; ++r) {
                        int row;
                        if (hs <= L.group) {
                            const int pair = r >> 1, second = r & 1;
                            row = 2 * j + pair + (second ? L.d / 2 : 0);
                        } else {
                            row = 4 * j + r;
                        }
                        add(v, dst, head + (size_t)row * row_h, row_h);
                        dst += row_h;
                    }
                }
            }
        }
        add(v, lb + L.rel_o, w.wo[l], (size_t)L.H * L.Q * 2);
        // gate/up interleaved in pairs of rows
        dst = lb + L.rel_gu;
        const uint8_t* wg = static_cast<const uint8_t*>(w.wgate[l]);
        const uint8_t* wu = static_cast<const uint8_t*>(w.wup[l]);
        for (int j = 0; j < L.F / 2; ++j) {
            const uint8_t* rows[4] = {wg + (size_t)(2 * j) * row_h, wu + (size_t)(2 * j) * row_h,
                                      wg + (size_t)(2 * j + 1) * row_h, wu + (size_t)(2 * j + 1) * row_h};
            for (int r = 0; r < 4; ++r) {
                add(v, dst, rows[r], row_h);
                dst += row_h;
            }
        }
        // down: [row block][chunk][4][ffn/4]
        dst = lb + L.rel_down;
        const uint8_t* wd = static_cast<const uint8_t*>(w.wdown[l]);
        const size_t fc = (size_t)(L.F / 4) * 2;
        for (int rb = 0; rb < L.H / 4; ++rb)
            for (int c = 0; c < 4; ++c)
                for (int r = 0; r < 4; ++r) {
                    add(v, dst, wd + (size_t)(4 * rb + r) * L.F * 2 + c * fc, fc);
                    dst += fc;
                }
    }
    for (int l = 0; l < L.L; ++l) {
        add(v, L.off_norms + (size_t)(2 * l) * row_h, w.attn_norm[l], row_h);
        add(v, L.off_norms + (size_t)(2 * l + 1) * row_h, w.mlp_norm[l], row_h);
    }
    add(v, L.off_norms + (size_t)(2 * L.L) * row_h, w.final_norm, row_h);
    return v;
}

// One map per (matrix, segment rows R = 8 (h + 1)), whose box is one fill of such a
// segment: {64 columns, R rows, nb(R) 64-column blocks}, K viewed as (64, K / 64):
//   QKV / O / gate-up: {64, rows, K / 64, layer}; LM head (the embedding rows):
//   {64, rows, K / 64}; down chunk c: {64, 4 rows of a block, hidden / 4 row blocks,
//   (ffn / 4) / 64, layer}, R <= 64 (a down instruction has at most 64 rows).
std::vector<mk_tmap_spec> tmap_specs(const Layout& L, uint32_t stage_bytes) {
    std::vector<mk_tmap_spec> v;
    const uint64_t ls = (uint64_t)L.layer_stride;
    const uint32_t kh = (uint32_t)L.H / kBoxK, kq = (uint32_t)L.Q / kBoxK, kf = (uint32_t)(L.F / 4) / kBoxK;
    auto add_spec = [&](int idx, size_t base, int rank, std::initializer_list<uint64_t> dims,
                        std::initializer_list<uint64_t> strides, std::initializer_list<uint32_t> box) {
        mk_tmap_spec t{};
        t.index = idx;
        t.rank = rank;
        t.base_offset = base;
        int i = 0;
        for (uint64_t d : dims) t.dims[i++] = d;
        i = 0;
        for (uint64_t st : strides) t.strides[i++] = st;
        i = 0;
        for (uint32_t b : box) t.box[i++] = b;
        v.push_back(t);
    };
    for (int hk = 0; hk < kTmPerKind; ++hk) {
        const uint32_t R = 8u * (uint32_t)(hk + 1);
        add_spec(kTmQKV * kTmPerKind + hk, L.off_layer0 + L.rel_qkv, 4,
                 {kBoxK, (uint64_t)L.qkv_rows, kh, (uint64_t)L.L}, {(uint64_t)L.H * 2, 128, ls},
                 {kBoxK, R, mma_nb(R, kh, stage_bytes), 1});
        add_spec(kTmO * kTmPerKind + hk, L.off_layer0 + L.rel_o, 4, {kBoxK, (uint64_t)L.H, kq, (uint64_t)L.L},
                 {(uint64_t)L.Q * 2, 128, ls}, {kBoxK, R, mma_nb(R, kq, stage_bytes), 1});
        add_spec(kTmGU * kTmPerKind + hk, L.off_layer0 + L.rel_gu, 4,
                 {kBoxK, (uint64_t)(2 * L.F), kh, (uint64_t)L.L}, {(uint64_t)L.H * 2, 128, ls},
                 {kBoxK, R, mma_nb(R, kh, stage_bytes), 1});
        add_spec(kTmLM * kTmPerKind + hk, L.off_embed, 3, {kBoxK, (uint64_t)L.V, kh}, {(uint64_t)L.H * 2, 128},
                 {kBoxK, R, mma_nb(R, kh, stage_bytes)});
        if (R <= 64) {
            const uint64_t f4 = (uint64_t)(L.F / 4);
            for (int c = 0; c < 4; ++c)
                add_spec(kTmDown0 + c * 8 + hk, L.off_layer0 + L.rel_down + (size_t)c * f4 * 2 * 4, 5,
                         {kBoxK, 4, (uint64_t)(L.H / 4), kf, (uint64_t)L.L}, {f4 * 2, f4 * 2 * 16, 128, ls},
                         {kBoxK, 4, R / 4, mma_nb(R, kf, stage_bytes), 1});
        }
    }
    return v;
}

bool weights_complete(const Layout& L, const mk_weights& w) {
    if (!w.embed || !w.final_norm || !w.attn_norm || !w.wq || !w.wk || !w.wv || !w.wo ||
        !w.mlp_norm || !w.wgate || !w.wup || !w.wdown)
        return false;
    for (int l = 0; l < L.L; ++l)
        if (!w.attn_norm[l] || !w.wq[l] || !w.wk[l] || !w.wv[l] || !w.wo[l] || !w.mlp_norm[l] ||
            !w.wgate[l] || !w.wup[l] || !w.wdown[l])
            return false;
    return true;
}

}  // namespace mk

extern "C" size_t mk_packed_bytes(const mk_config* cfg) {
    mk::Layout L;
    if (!cfg || !mk::make_layout(*cfg, &L, nullptr)) return 0;
    return L.total;
}

extern "C" mk_status mk_tensor_map_specs_host(const mk_config* cfg, uint32_t stage_bytes, mk_tmap_spec* out,
                                               size_t cap, size_t* n) {
    mk::Layout L;
    if (!cfg || !n || stage_bytes == 0) return MK_ERR_INVALID_ARG;
    if (!mk::make_layout(*cfg, &L, nullptr)) return MK_ERR_UNSUPPORTED;
    try {
        const std::vector<mk_tmap_spec> v = mk::tmap_specs(L, stage_bytes);
        *n = v.size();
        if (out) {
            if (cap < v.size()) return MK_ERR_INVALID_ARG;
            for (size_t i = 0; i < v.size(); ++i) out[i] = v[i];
        }
    } catch (...) {
        return MK_ERR_OUT_OF_MEMORY;
    }
    return MK_OK;
}

extern "C" mk_status mk_pack_weights_host(const mk_config* cfg, const mk_weights* w, void* dst,
                                          size_t dst_bytes) {
    mk::Layout L;
    if (!cfg || !w || !dst) return MK_ERR_INVALID_ARG;
    if (!mk::make_layout(*cfg, &L, nullptr)) return MK_ERR_UNSUPPORTED;
    if (dst_bytes < L.total || !mk::weights_complete(L, *w)) return MK_ERR_INVALID_ARG;
    std::vector<mk::Segment> segs;
    try {
        segs = mk::pack_segments(L, *w);
    } catch (...) {  // the segment list could not be allocated; nothing is written
        return MK_ERR_OUT_OF_MEMORY;
    }
    memset(dst, 0, L.total);
    for (const mk::Segment& s : segs) memcpy(static_cast<uint8_t*>(dst) + s.dst, s.src, s.bytes);
    return MK_OK;
}
