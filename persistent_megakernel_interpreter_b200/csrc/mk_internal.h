// Internal definitions shared by the host code and the kernels of libmk.so:
// the packed-weight layout, the kernel parameter block, the control block.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "mk.h"

#ifdef __CUDACC__
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif

namespace mk {

constexpr int kConsumerWarps = 8;                    // compute warps
// Mover warps kConsumerWarps .. +3: mover q (its warp index mod 4 is q, the Tensor
// Memory lane quarter it may access) moves each landed weight tile of the ring
// fills seq = q (mod 4) into Tensor Memory.
constexpr int kMoveWarps = 4;
constexpr int kPrepWarp = kConsumerWarps + kMoveWarps;   // stages RoPE rows and down-projection inputs
constexpr int kLoaderWarp = kPrepWarp + 1;               // lane 0 issues every ring fill
// Stage warps: at batch 1, stage warp h stages the h chunk of every down-projection
// chunk-h job (h < kStageWarps), in parallel with the activation warp's other jobs.
constexpr int kStageWarps = 2;
constexpr int kStageWarp0 = kLoaderWarp + 1;
constexpr int kThreads = 32 * (kStageWarp0 + kStageWarps);
// 16 warps: each of the SM's four schedulers (16384 registers each) hosts four of
// them, so a thread gets at most 16384 / (4 * 32) = 128 registers.
constexpr uint32_t kTmemCols = 512;                  // all of an SM's Tensor Memory (256 KB)
constexpr int kMaxTmemSlots = 64;                    // weight tiles Tensor Memory holds at most
constexpr int kRowsPerTile = 4;                      // every matvec tile holds 4 rows
constexpr int kMaxDownRows = 16;                     // row blocks per down instruction
constexpr int kMaxResidRows = 64;                    // residual rows per O-proj / down job
constexpr int kMaxBatch = 8;
constexpr int kMaxGroupHeads = 4;                    // query heads per KV head
constexpr int kMaxParts = 32;                        // split-K partitions per (sequence, group)
constexpr int kMaxItemKeys = 512;                    // keys of one attention item at most
// Shared-memory scratch of one attention item (inside its job slot, after the
// item's q and new key/value), in floats: per compute warp a region of 4 * hd
// (a block's weights while the warp runs, then its value sums for up to 4 heads
// of hd dims), the warps' maxima and sums, a flag word.
MK_HD constexpr uint32_t attn_scratch_floats(int hd) {
    return 4u * (uint32_t)hd * kConsumerWarps + 8u * kConsumerWarps + 4u;
}
// An attention item's q (fp32 [group][hd]) and new key and value (bf16 [2][hd]) at
// the start of its job slot, 16-byte aligned; the scratch follows.
MK_HD constexpr uint32_t attn_item_bytes(int group, int hd) {
    return ((uint32_t)(group * hd * 4 + 2 * hd * 2) + 15u) & ~15u;
}
// Tensor-core projections at batch > 1 (MK_PROJ_TENSOR_CORES). An instruction's
// weight rows (a multiple of 8 on this path) are cut into segments of at most 128
// rows (gate/up: per MLP chunk). A segment of R rows streams in fills of nb(R)
// 64-column boxes (128 bytes: the swizzle span), each fill one TMA copy of a
// {64 columns, R rows, nb boxes} block that lands as nb boxes of R rows side by
// side, and accumulates in its own Tensor Memory accumulator over lanes = rows:
// kSubAcc partial sums of 16 fp32 columns each (8 sequences, high and low bf16
// parts of the input), the K = 16 steps taken in turn.
constexpr uint32_t kAccCols = 16;
constexpr uint32_t kSubAcc = 4;
// Issuing warps of the tensor-core path (the mover warps' places): issuer u issues
// the MMAs of partial sum u, so the four K steps of a box go out from four threads.
constexpr int kIssuers = 4;
static_assert(kIssuers == (int)kSubAcc, "one issuer per partial sum");
constexpr int kMaxAcc = (int)(kTmemCols / (kAccCols * kSubAcc));  // segment accumulators in use at once
constexpr uint32_t kMmaRows = 128;                   // M of every MMA: rows of a full segment
constexpr uint32_t kBoxK = 64;                        // K columns of one box
// Tensor maps, one per (weight matrix, segment rows R = 8 (h + 1)): QKV, O, gate/up
// and the LM head at kind * 16 + h; the down-projection's chunk c at 64 + c * 8 + h
// (its segments are at most 64 rows).
enum TmapKind { kTmQKV = 0, kTmO = 1, kTmGU = 2, kTmLM = 3 };
constexpr int kTmPerKind = 16;
constexpr int kTmDown0 = 4 * kTmPerKind;
constexpr int kTmCount = kTmDown0 + 4 * 8;
constexpr uint32_t kTmBytes = 128;                    // sizeof(CUtensorMap)

// Boxes per fill of a segment of R rows: as many as a ring stage holds, at most
// the row's k64 boxes.
MK_HD inline uint32_t mma_nb(uint32_t R, uint32_t k64, uint32_t stage_bytes) {
    uint32_t nb = stage_bytes / (R * 128u);
    if (nb < 1) nb = 1;
    return nb > k64 ? k64 : nb;
}

// Fills of a matvec instruction on the tensor-core path, in the order job c (the
// down-projection's chunk), range, segment, K-fill. Every segment but the last
// of a range is full (128 rows).
struct MmaGeom {
    uint32_t k64;           // 64-column boxes along K
    uint32_t rows;          // weight rows of one range
    uint32_t nrange;        // 4 for gate/up (one per MLP chunk), else 1
    uint32_t segs;          // segments per range
    uint32_t jobs;          // 4 chunk jobs for the down-projection, else 1
    uint32_t nb_f, fps_f;   // a full segment: boxes per fill, fills
    uint32_t rows_l, nb_l, fps_l;  // the last segment
    MK_HD uint32_t per_range() const { return (segs - 1u) * fps_f + fps_l; }
    MK_HD uint32_t per_job() const { return nrange * per_range(); }
    MK_HD uint32_t nfill() const { return jobs * per_job(); }
};

MK_HD inline MmaGeom mma_geom(uint32_t op, uint32_t count, uint32_t aux0, int H, int Q, int F,
                              uint32_t stage_bytes) {
    MmaGeom g{};
    g.jobs = 1;
    g.nrange = 1;
    g.rows = 4u * count;
    g.k64 = (uint32_t)H / kBoxK;
    if (op == MK_OP_OPROJ) {
        g.k64 = (uint32_t)Q / kBoxK;
    } else if (op == MK_OP_DOWN) {
        g.k64 = (uint32_t)(F / 4) / kBoxK;
        g.jobs = 4;
    } else if (op == MK_OP_GATEUP) {
        g.rows = 4u * aux0;
        g.nrange = 4;
    }
    g.segs = (g.rows + kMmaRows - 1) / kMmaRows;
    g.nb_f = mma_nb(kMmaRows, g.k64, stage_bytes);
    g.fps_f = (g.k64 + g.nb_f - 1) / g.nb_f;
    g.rows_l = g.rows - (g.segs - 1u) * kMmaRows;
    g.nb_l = mma_nb(g.rows_l, g.k64, stage_bytes);
    g.fps_l = (g.k64 + g.nb_l - 1) / g.nb_l;
    return g;
}

constexpr int kMaxLayers = 64;
constexpr int kCounterStride = 32;                   // uint32 per counter: one per 128 B line
constexpr size_t kSmemBudget = 227 * 1024;           // dynamic shared memory per CTA
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Byte offsets of every packed region (see mk_pack_weights_host in mk.h).
struct Layout {
    int L, H, nq, nkv, d, F, V;
    int group;            // query heads per KV head
    int Q, KVD;           // n_heads*head_dim, n_kv_heads*head_dim
    int qkv_rows;         // Q + 2*KVD
    int tiles_per_group;  // 4-row QKV tiles per KV group
    // tile sizes in bytes
    uint32_t tile_h;      // 4 x hidden (QKV, gate/up, LM head)
    uint32_t tile_o;      // 4 x Q (O-projection)
    uint32_t tile_f;      // 4 x ffn/4 (down, one chunk)
    size_t off_embed, off_layer0, layer_stride;
    size_t rel_qkv, rel_o, rel_gu, rel_down;  // within a layer
    size_t off_norms, total;

    size_t qkv(int l) const { return off_layer0 + (size_t)l * layer_stride + rel_qkv; }
    size_t o(int l) const { return off_layer0 + (size_t)l * layer_stride + rel_o; }
    size_t gu(int l) const { return off_layer0 + (size_t)l * layer_stride + rel_gu; }
    size_t down(int l) const { return off_layer0 + (size_t)l * layer_stride + rel_down; }
    size_t attn_norm(int l) const { return off_norms + (size_t)(2 * l) * H * 2; }
    size_t mlp_norm(int l) const { return off_norms + (size_t)(2 * l + 1) * H * 2; }
    size_t final_norm() const { return off_norms + (size_t)(2 * L) * H * 2; }
};

// Shared-memory map of the megakernel (byte offsets from the dynamic base).
struct SmemLayout {
    uint32_t ring, full, empty, armed;        // weight / cached-KV ring of S stages
    uint32_t xs, xs_full, xs_empty, xs_done;  // NS activation slots
    uint32_t xs_job;                          // the job each slot was last prepared for
    uint32_t tot;                             // down-projection running sums
    uint32_t red;                             // per-warp partial sums of a job input
    uint32_t cbar;                            // barrier of the compute warps
    uint32_t sel;                             // [warps][kMaxBatch] LM-head best per warp (greedy)
    uint32_t tfull, tempty, tarmed;           // Tensor Memory slots: landed / released / fill held
    uint32_t tbase;                           // Tensor Memory address of the allocation
    // tensor-core path only (zero bytes otherwise)
    uint32_t opnd;                            // [NS] a job's MMA operand is in its slot
    uint32_t mdone;                           // [NS] the job's MMAs have completed
    uint32_t afull, aempty;                   // [kMaxAcc] accumulator written / read
    uint32_t fin;                             // every MMA issued has completed
    uint32_t total;
};

MK_HD inline uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// With `mma` (the tensor-core path) the slots start on a 1024-byte boundary (each
// holds its MMA operand in 128-byte-swizzled atoms of 8 rows) and the MMA
// barriers are added.
MK_HD inline SmemLayout smem_layout(int S, uint32_t stage_bytes, int NS, uint32_t slot_bytes, bool mma = false) {
    SmemLayout m;
    uint32_t o = 0;
    m.ring = o;      o += (uint32_t)S * stage_bytes;
    m.full = o;      o += 8u * S;
    m.empty = o;     o += 8u * S;
    m.armed = o;     o = align16(o + 4u * S);
    if (mma) o = (o + 1023u) & ~1023u;
    m.xs = o;        o += (uint32_t)NS * slot_bytes;
    m.xs_full = o;   o += 8u * NS;
    m.xs_empty = o;  o += 8u * NS;
    m.xs_done = o;   o += 4u * NS;
    m.xs_job = o;    o = align16(o + 4u * NS);
    m.tot = o;       o += 4u * kMaxDownRows * kMaxBatch * 4u;
    m.red = o;       o += 4u * 32u;
    m.cbar = o;      o += 8u;
    m.sel = o;       o += 8u * kConsumerWarps * kMaxBatch;
    o = (o + 7u) & ~7u;
    m.tfull = o;     o += 8u * kMaxTmemSlots;
    m.tempty = o;    o += 8u * kMaxTmemSlots;
    m.tarmed = o;    o += 4u * kMaxTmemSlots;
    m.tbase = o;     o += 4u;
    o = (o + 7u) & ~7u;
    const uint32_t nacc = mma ? (uint32_t)kMaxAcc : 0u, nsl = mma ? (uint32_t)NS : 0u;
    m.opnd = o;      o += 8u * nsl;
    m.mdone = o;     o += 8u * nsl;
    m.afull = o;     o += 8u * nacc;
    m.aempty = o;    o += 8u * nacc;
    m.fin = o;       o += mma ? 8u : 0u;
    m.total = align16(o);
    return m;
}

// Returns false if the shape is not one the kernels handle.
bool make_layout(const mk_config& c, Layout* out, const char** why);

// Control words, one 128-byte line each (see the megakernel for their protocol).
struct Ctl {
    uint32_t epoch;     uint32_t pad0[31];
    uint32_t done;      uint32_t pad1[31];
    uint32_t status;    uint32_t abort;  uint32_t info[6]; uint32_t pad2[24];
};

// Kernel parameter block (passed by value, __grid_constant__).
struct Params {
    // shape
    int L, H, nq, nkv, d, F, V, group, Q, KVD;
    int B, max_batch, max_seq, max_ctx;
    float eps;
    // packed weights
    const uint8_t* packed;
    size_t off_layer0, layer_stride, rel_qkv, rel_o, rel_gu, rel_down, off_norms;
    uint32_t tile_h, tile_o, tile_f;
    const float* rope_cos;   // [max_seq][d/2]
    const float* rope_sin;
    // per step
    const int32_t* tokens;
    const int32_t* positions;
    uint16_t* kc;
    uint16_t* vc;
    float* logits;
    // greedy selection fused into the LM head (all NULL: off): the next token of
    // sequence b goes to next_tokens[b], its position + 1 to next_positions[b], and
    // the token also to gen_tokens[b] when that is set
    int32_t* next_tokens;
    int32_t* next_positions;
    int32_t* gen_tokens;
    uint32_t* sel_best;  // [B][n_lm_jobs][2] each LM-head job's best (value bits, index)
    int n_lm_jobs;
    // scratch
    float* x;          // [B][H]   residual stream (fp32)
    float* q;          // [B][Q]
    float* attn;       // [B][Q]
    float* hbuf;       // [B][F]
    float* part_ml;    // [B][nq][P][2]  (m, l)
    float* part_o;     // [B][nq][P][d]
    // the megakernel's tagged activations (value | tag << 32, see act_tag)
    uint64_t* x_t;     // [B][H]   residual stream
    uint64_t* q_t;     // [B][Q]   queries
    uint64_t* kv_t;    // [B][nkv][2][d] the step's new key and value (bf16 values)
    uint64_t* attn_t;  // [B][Q]   attention output
    uint64_t* h_t;     // [B][F]   gated MLP activations
    size_t tagged_words;  // total words of the five (contiguous from x_t)
    uint32_t* counters;
    Ctl* ctl;
    // schedule
    const mk_instr* instrs;
    const int32_t* sm_off;
    int n_sm;
    int part_keys, n_parts, keys_per_stage;
    uint32_t stage_bytes;
    int n_stages;              // ring stages (a multiple of 4)
    int n_tslots;              // Tensor Memory slots (a multiple of 4; slot k in lane quarter k % 4)
    uint32_t tslot_cols;       // columns of one slot: a stage's bytes / (32 lanes * 4 bytes)
    int xs_slots;              // activation slots (1..3)
    uint32_t xs_slot_bytes;
    uint32_t xs_vec_floats;    // stride of one sequence's vector inside a slot
    uint32_t xs_aux_floats;    // offset of the slot's RoPE rows and residual rows
    // tensor-core projections (batch > 1): MK_PROJ_TENSOR_CORES, else 0
    int mma;
    const void* tmaps;         // [kTmCount] CUtensorMap (64-byte aligned, global)
    int n_counters;
    uint64_t timeout_ns;
    // optional per-job timestamps: [n_sm][trace_jobs][kTraceWords] (nullptr = off)
    uint64_t* trace;
    int trace_jobs;
};

// Trace record of one job (globaltimer nanoseconds).
enum TraceWord {
    kTrSlotWait = 0,   // activation warp starts waiting for a free slot
    kTrCtrWait = 1,    // slot free; starts waiting for the input counter
    kTrCtrDone = 2,    // input counter reached
    kTrReady = 3,      // input prepared, slot handed to the compute warps
    kTrStart = 4,      // compute warp 0 starts the job
    kTrDone = 5,       // last compute warp finished (job counter signalled)
    kTrMeta = 6,       // op | layer << 8 | chunk << 24
    kTrFill = 7,       // compute warp 0 has its first ring fill of the job
    kTrSub0 = 8,       // 8..15: op-specific stamps of compute warp 0 (see the kernel)
    kTraceWords = 16
};

// Device status codes live in Ctl::status (values of mk_status).

}  // namespace mk
