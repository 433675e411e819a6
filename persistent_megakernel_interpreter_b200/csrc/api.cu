// The C ABI of libmk.so (declarations and contracts in include/mk.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <stdexcept>
#include <string>
#include <vector>

#include "pack.h"

namespace mk {
// megakernel.cu
bool megakernel_supported(int H, int Q, int F, int d);
cudaError_t megakernel_prepare(const Params& p);
cudaError_t megakernel_occupancy(const Params& p, int* blocks_per_sm);
cudaError_t megakernel_launch(const Params& p, cudaStream_t stream);
size_t megakernel_smem_bytes(const Params& p);
// baseline.cu
cudaError_t baseline_launch(const Params& p, cudaStream_t stream, int n_sm);
cudaError_t baseline_prepare(const Params& p);

// Device gather used by the packer: one warp per segment, 16-byte words.
__global__ void k_gather(const Segment* segs, size_t n, uint8_t* dst) {
    const size_t w = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const size_t nw = ((size_t)gridDim.x * blockDim.x) >> 5;
    for (size_t i = w; i < n; i += nw) {
        const Segment s = segs[i];
        const uint4* src = static_cast<const uint4*>(s.src);
        uint4* d = reinterpret_cast<uint4*>(dst + s.dst);
        for (uint32_t k = lane; k < s.bytes / 16; k += 32) d[k] = src[k];
    }
}
}  // namespace mk

struct mk_handle {
    int device = 0;
    int dev_sms = 0;
    mk_config cfg{};
    mk::Layout lay{};
    uint8_t* packed = nullptr;
    float* rope = nullptr;          // cos table then sin table
    void* d_tmaps = nullptr;        // tensor maps of the packed weights (tensor-core path)
    uint32_t tmap_stage_bytes = 0;  // the ring stage size they were built for
    // scratch (sized by mk_build_schedule)
    void* scratch = nullptr;
    size_t scratch_bytes = 0;
    uint32_t* counters = nullptr;   // inside `scratch`
    mk::Ctl* ctl = nullptr;
    // schedule
    bool has_schedule = false;
    mk_instr* d_instrs = nullptr;
    int32_t* d_sm_off = nullptr;
    mk_schedule_info info{};
    mk::Params params{};
    // staging for the host-buffer entry point
    uint64_t* d_trace = nullptr;    // per-job timestamps (traced schedules only)
    int trace_jobs = 0;
    int32_t* d_io = nullptr;        // tokens [max_batch], positions [max_batch]
    int32_t* h_io = nullptr;        // pinned host staging of the same, for mk_decode_step_host
    float* d_logits = nullptr;
    std::string msg;
};

namespace {

mk_status cuda_fail(mk_handle* h, cudaError_t e, const char* what) {
    if (h) h->msg = std::string(what) + ": " + cudaGetErrorString(e);
    return e == cudaErrorMemoryAllocation ? MK_ERR_OUT_OF_MEMORY : MK_ERR_CUDA;
}

#define MK_CUDA(h, call)                                  \
    do {                                                  \
        cudaError_t e_ = (call);                          \
        if (e_ != cudaSuccess) return cuda_fail(h, e_, #call); \
    } while (0)

// Makes the handle's device current for the calls of one entry point and gives
// the caller's current device back when the entry point returns.
struct DeviceScope {
    int prev = -1;
    cudaError_t enter(int device) {
        const cudaError_t e = cudaGetDevice(&prev);
        if (e != cudaSuccess) {
            prev = -1;
            return e;
        }
        return prev == device ? cudaSuccess : cudaSetDevice(device);
    }
    ~DeviceScope() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

// Runs an entry point's body so that no C++ exception leaves the C ABI: a failed
// host allocation reads as MK_ERR_OUT_OF_MEMORY, anything else as MK_ERR_INVALID_ARG.
template <class F>
mk_status no_throw(F&& body) {
    try {
        return body();
    } catch (const std::bad_alloc&) {
        return MK_ERR_OUT_OF_MEMORY;
    } catch (const std::length_error&) {
        return MK_ERR_OUT_OF_MEMORY;
    } catch (...) {
        return MK_ERR_INVALID_ARG;
    }
}

void free_schedule(mk_handle* h) {
    cudaFree(h->scratch);
    cudaFree(h->d_instrs);
    cudaFree(h->d_sm_off);
    cudaFree(h->d_io);
    cudaFreeHost(h->h_io);
    cudaFree(h->d_logits);
    cudaFree(h->d_trace);
    h->d_trace = nullptr;
    h->trace_jobs = 0;
    h->scratch = nullptr;
    h->d_instrs = nullptr;
    h->d_sm_off = nullptr;
    h->d_io = nullptr;
    h->h_io = nullptr;
    h->d_logits = nullptr;
    h->has_schedule = false;
}

}  // namespace

extern "C" const char* mk_status_str(mk_status s) {
    switch (s) {
        case MK_OK: return "ok";
        case MK_ERR_INVALID_ARG: return "invalid argument";
        case MK_ERR_CUDA: return "CUDA error";
        case MK_ERR_UNSUPPORTED: return "unsupported";
        case MK_ERR_NO_SCHEDULE: return "no schedule built";
        case MK_ERR_TIMEOUT: return "device wait timed out";
        case MK_ERR_BAD_TOKEN: return "token out of range";
        case MK_ERR_BAD_POSITION: return "position out of range";
        case MK_ERR_OUT_OF_MEMORY: return "out of memory";
    }
    return "unknown status";
}

static mk_status create_impl(const mk_config* cfg, const mk_weights* w, int device, mk_handle** out) {
    if (!out) return MK_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !w) return MK_ERR_INVALID_ARG;
    mk::Layout L;
    const char* why = nullptr;
    if (!mk::make_layout(*cfg, &L, &why)) return MK_ERR_UNSUPPORTED;
    if (!mk::megakernel_supported(L.H, L.Q, L.F, L.d)) return MK_ERR_UNSUPPORTED;
    if (!mk::weights_complete(L, *w)) return MK_ERR_INVALID_ARG;
    // the handle is destroyed on every way out but success, a thrown one included
    struct Owner {
        mk_handle* h;
        ~Owner() { mk_destroy(h); }
    } owner{new mk_handle()};
    mk_handle* h = owner.h;
    h->device = device;
    h->cfg = *cfg;
    h->lay = L;
    DeviceScope scope;
    cudaError_t e = scope.enter(device);
    if (e != cudaSuccess) return MK_ERR_CUDA;
    if (cudaDeviceGetAttribute(&h->dev_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
        return MK_ERR_CUDA;
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device);
    if (!coop) return MK_ERR_UNSUPPORTED;

    if (cudaMalloc(&h->packed, L.total) != cudaSuccess) return MK_ERR_OUT_OF_MEMORY;
    // pack: gather segments on the device (bit copy)
    {
        std::vector<mk::Segment> segs = mk::pack_segments(L, *w);
        for (const mk::Segment& s : segs)
            if ((reinterpret_cast<uintptr_t>(s.src) | s.dst | s.bytes) & 15) return MK_ERR_INVALID_ARG;
        mk::Segment* d_segs = nullptr;
        if (cudaMalloc(&d_segs, segs.size() * sizeof(mk::Segment)) != cudaSuccess)
            return MK_ERR_OUT_OF_MEMORY;
        e = cudaMemcpy(d_segs, segs.data(), segs.size() * sizeof(mk::Segment), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemset(h->packed, 0, L.total);
        if (e == cudaSuccess) {
            mk::k_gather<<<h->dev_sms * 8, 256>>>(d_segs, segs.size(), h->packed);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        cudaFree(d_segs);
        if (e != cudaSuccess) return MK_ERR_CUDA;
    }
    // RoPE table: angle pos * theta^(-2i/d) in double, cos/sin stored as float
    {
        const int half = L.d / 2;
        std::vector<float> tab((size_t)2 * cfg->max_seq * half);
        for (int pos = 0; pos < cfg->max_seq; ++pos)
            for (int i = 0; i < half; ++i) {
                const double inv_freq = pow(cfg->rope_theta, -(2.0 * i) / (double)L.d);
                const double ang = (double)pos * inv_freq;
                tab[(size_t)pos * half + i] = (float)cos(ang);
                tab[(size_t)cfg->max_seq * half + (size_t)pos * half + i] = (float)sin(ang);
            }
        if (cudaMalloc(&h->rope, tab.size() * sizeof(float)) != cudaSuccess)
            return MK_ERR_OUT_OF_MEMORY;
        if (cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float), cudaMemcpyHostToDevice) !=
            cudaSuccess)
            return MK_ERR_CUDA;
    }
    owner.h = nullptr;
    *out = h;
    return MK_OK;
}

extern "C" mk_status mk_create(const mk_config* cfg, const mk_weights* w, int device,
                               mk_handle** out) {
    return no_throw([&] { return create_impl(cfg, w, device, out); });
}

// Tensor maps of the packed weights for the tensor-core path (mk::tmap_specs: one
// per matrix and segment height, the box one fill of such a segment), encoded with
// the 128-byte swizzle the MMA's shared-memory descriptors read. nb depends on the
// ring's stage size, so the maps are rebuilt when it changes.
static mk_status make_tmaps(mk_handle* h, uint32_t stage_bytes) {
    if (h->d_tmaps && h->tmap_stage_bytes == stage_bytes) return MK_OK;
    typedef CUresult (*Encode)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        h->msg = "cuTensorMapEncodeTiled is not available";
        return MK_ERR_UNSUPPORTED;
    }
    static_assert(sizeof(CUtensorMap) == mk::kTmBytes, "tensor map size");
    const Encode encode = reinterpret_cast<Encode>(fn);
    const mk::Layout& L = h->lay;
    std::vector<CUtensorMap> maps((size_t)mk::kTmCount);
    memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
    const cuuint32_t unit[5] = {1, 1, 1, 1, 1};
    auto enc = [&](int idx, uint8_t* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                   const cuuint32_t* box) {
        const CUresult r = encode(&maps[(size_t)idx], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, base, dims,
                                  strides, box, unit, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        return r == CUDA_SUCCESS;
    };
    bool ok = true;
    for (const mk_tmap_spec& t : mk::tmap_specs(L, stage_bytes)) {
        cuuint64_t dims[5], strides[4];
        cuuint32_t box[5];
        for (int i = 0; i < t.rank; ++i) {
            dims[i] = (cuuint64_t)t.dims[i];
            box[i] = (cuuint32_t)t.box[i];
            if (i + 1 < t.rank) strides[i] = (cuuint64_t)t.strides[i];
        }
        ok = ok && enc(t.index, h->packed + t.base_offset, t.rank, dims, strides, box);
    }
    if (!ok) {
        h->msg = "cuTensorMapEncodeTiled refused a weight tensor map";
        return MK_ERR_UNSUPPORTED;
    }
    if (!h->d_tmaps) MK_CUDA(h, cudaMalloc(&h->d_tmaps, maps.size() * sizeof(CUtensorMap)));
    MK_CUDA(h, cudaMemcpy(h->d_tmaps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice));
    h->tmap_stage_bytes = stage_bytes;
    return MK_OK;
}

static mk_status build_schedule_impl(mk_handle* h, int batch, int max_ctx, const mk_schedule_opts* opts) {
    if (!h) return MK_ERR_INVALID_ARG;
    const mk_config& c = h->cfg;
    const mk::Layout& L = h->lay;
    if (batch < 1 || batch > c.max_batch || max_ctx < 1 || max_ctx > c.max_seq)
        return MK_ERR_INVALID_ARG;
    const int n_sm = (opts && opts->n_sm > 0) ? opts->n_sm : h->dev_sms;
    if (n_sm > h->dev_sms) return MK_ERR_INVALID_ARG;
    DeviceScope scope;
    MK_CUDA(h, scope.enter(h->device));
    mk::Plan P;
    mk_status st = mk::plan_schedule(L, batch, max_ctx, n_sm, opts, 0, &P);
    if (st != MK_OK) return st;
    const bool mma = P.info.proj == MK_PROJ_TENSOR_CORES;
    MK_CUDA(h, cudaDeviceSynchronize());
    if (mma) {
        st = make_tmaps(h, (uint32_t)P.info.stage_bytes);
        if (st != MK_OK) return st;
    }
    free_schedule(h);

    // scratch: activations, attention partials, counters, control block
    const mk_schedule_info& I = P.info;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = mk::align_up(off + bytes, 256);
        return o;
    };
    const size_t o_x = take((size_t)batch * L.H * 4);
    const size_t o_q = take((size_t)batch * L.Q * 4);
    const size_t o_attn = take((size_t)batch * L.Q * 4);
    const size_t o_h = take((size_t)batch * L.F * 4);
    const size_t o_ml = take((size_t)batch * L.nq * I.n_parts * 2 * sizeof(float));
    const size_t o_po = take((size_t)batch * L.nq * I.n_parts * L.d * sizeof(float));
    // tagged activations of the megakernel, contiguous (cleared as one range)
    const size_t tw_x = (size_t)batch * L.H, tw_q = (size_t)batch * L.Q,
                 tw_kv = (size_t)batch * L.nkv * 2 * L.d, tw_a = (size_t)batch * L.Q, tw_h = (size_t)batch * L.F;
    const size_t tagged_words = tw_x + tw_q + tw_kv + tw_a + tw_h;
    const size_t o_tag = take(tagged_words * sizeof(uint64_t));
    const size_t o_ctr = take((size_t)I.n_counters * mk::kCounterStride * sizeof(uint32_t));
    const size_t o_ctl = take(sizeof(mk::Ctl));
    int n_lm = 0;  // LM-head instructions: one greedy-selection entry each per sequence
    for (const mk_instr& in : P.instrs) n_lm += in.op == MK_OP_LMHEAD;
    const size_t o_sel = take((size_t)batch * n_lm * 2 * sizeof(uint32_t));
    MK_CUDA(h, cudaMalloc(&h->scratch, off));
    MK_CUDA(h, cudaMemset(h->scratch, 0, off));
    h->scratch_bytes = off;
    uint8_t* sb = static_cast<uint8_t*>(h->scratch);
    h->counters = reinterpret_cast<uint32_t*>(sb + o_ctr);
    h->ctl = reinterpret_cast<mk::Ctl*>(sb + o_ctl);

    MK_CUDA(h, cudaMalloc(&h->d_instrs, P.instrs.size() * sizeof(mk_instr)));
    MK_CUDA(h, cudaMemcpy(h->d_instrs, P.instrs.data(), P.instrs.size() * sizeof(mk_instr),
                          cudaMemcpyHostToDevice));
    MK_CUDA(h, cudaMalloc(&h->d_sm_off, P.sm_off.size() * sizeof(int32_t)));
    MK_CUDA(h, cudaMemcpy(h->d_sm_off, P.sm_off.data(), P.sm_off.size() * sizeof(int32_t),
                          cudaMemcpyHostToDevice));
    MK_CUDA(h, cudaMalloc(&h->d_io, 2 * (size_t)c.max_batch * sizeof(int32_t)));
    MK_CUDA(h, cudaMallocHost(&h->h_io, 2 * (size_t)c.max_batch * sizeof(int32_t)));
    memset(h->h_io, 0, 2 * (size_t)c.max_batch * sizeof(int32_t));
    MK_CUDA(h, cudaMalloc(&h->d_logits, (size_t)batch * L.V * sizeof(float)));

    mk::Params& p = h->params;
    p = mk::Params{};
    p.L = L.L; p.H = L.H; p.nq = L.nq; p.nkv = L.nkv; p.d = L.d; p.F = L.F; p.V = L.V;
    p.group = L.group; p.Q = L.Q; p.KVD = L.KVD;
    p.B = batch; p.max_batch = c.max_batch; p.max_seq = c.max_seq; p.max_ctx = max_ctx;
    p.eps = c.rms_eps;
    p.packed = h->packed;
    p.off_layer0 = L.off_layer0; p.layer_stride = L.layer_stride;
    p.rel_qkv = L.rel_qkv; p.rel_o = L.rel_o; p.rel_gu = L.rel_gu; p.rel_down = L.rel_down;
    p.off_norms = L.off_norms;
    p.tile_h = L.tile_h; p.tile_o = L.tile_o; p.tile_f = L.tile_f;
    p.rope_cos = h->rope;
    p.rope_sin = h->rope + (size_t)c.max_seq * (L.d / 2);
    p.x = reinterpret_cast<float*>(sb + o_x);
    p.q = reinterpret_cast<float*>(sb + o_q);
    p.attn = reinterpret_cast<float*>(sb + o_attn);
    p.hbuf = reinterpret_cast<float*>(sb + o_h);
    p.part_ml = reinterpret_cast<float*>(sb + o_ml);
    p.part_o = reinterpret_cast<float*>(sb + o_po);
    p.x_t = reinterpret_cast<uint64_t*>(sb + o_tag);
    p.q_t = p.x_t + tw_x;
    p.kv_t = p.q_t + tw_q;
    p.attn_t = p.kv_t + tw_kv;
    p.h_t = p.attn_t + tw_a;
    p.tagged_words = tagged_words;
    p.counters = h->counters;
    p.ctl = h->ctl;
    p.sel_best = reinterpret_cast<uint32_t*>(sb + o_sel);
    p.n_lm_jobs = n_lm;
    p.instrs = h->d_instrs;
    p.sm_off = h->d_sm_off;
    p.n_sm = n_sm;
    p.part_keys = I.part_keys;
    p.n_parts = I.n_parts;
    p.keys_per_stage = I.keys_per_stage;
    p.stage_bytes = (uint32_t)I.stage_bytes;
    p.n_stages = I.n_stages;
    // Tensor Memory: one slot per weight tile of up to a stage's bytes, in one lane
    // quarter (32 lanes of stage_bytes / 32 bytes each); as many as 512 columns hold
    // per quarter, four quarters
    p.tslot_cols = (uint32_t)I.stage_bytes / 128u;
    if (mma) {
        // Tensor Memory holds the MMA accumulators instead of weight tiles
        p.mma = MK_PROJ_TENSOR_CORES;
        p.tmaps = h->d_tmaps;
        p.n_tslots = 0;
    } else {
        int per_q = p.tslot_cols ? (int)(mk::kTmemCols / p.tslot_cols) : 0;
        if (per_q > mk::kMaxTmemSlots / 4) per_q = mk::kMaxTmemSlots / 4;
        p.n_tslots = 4 * per_q;
        if (p.n_tslots < 4 || I.stage_bytes % 128 != 0) {
            h->msg = "a weight tile does not fit the SM's Tensor Memory";
            free_schedule(h);
            return MK_ERR_UNSUPPORTED;
        }
    }
    {
        const mk::SlotPlan sp = mk::slot_plan(L, batch, (uint32_t)I.stage_bytes, mma);
        p.xs_slots = sp.xs_slots;
        p.xs_slot_bytes = sp.slot_bytes;
        p.xs_vec_floats = sp.vec_floats;
        p.xs_aux_floats = sp.aux_floats;
        // an MMA reads 128 rows from each box's start, rows past the segment's own
        // (never used) included: the shared memory after the ring must cover them
        const mk::SmemLayout m = mk::smem_layout(p.n_stages, p.stage_bytes, p.xs_slots, p.xs_slot_bytes, mma);
        if (mma && m.total < m.ring + (uint32_t)p.n_stages * p.stage_bytes + mk::kMmaRows * 128u) {
            h->msg = "shared memory too small for the tensor-core path";
            free_schedule(h);
            return MK_ERR_UNSUPPORTED;
        }
    }
    p.n_counters = I.n_counters;
    if (opts && opts->trace) {
        int most = 0;
        for (int s = 0; s < n_sm; ++s) {
            int jobs = 0;
            for (int i = P.sm_off[s]; i < P.sm_off[s + 1]; ++i)
                jobs += P.instrs[i].op == MK_OP_DOWN ? 4 : 1;
            most = jobs > most ? jobs : most;
        }
        h->trace_jobs = most;
        const size_t tb = (size_t)n_sm * most * mk::kTraceWords * sizeof(uint64_t);
        MK_CUDA(h, cudaMalloc(&h->d_trace, tb));
        MK_CUDA(h, cudaMemset(h->d_trace, 0, tb));
    }
    p.trace = h->d_trace;
    p.trace_jobs = h->trace_jobs;
    p.timeout_ns = mk::kDefaultTimeoutNs;
    if (opts && opts->wait_timeout_ms > 0) p.timeout_ns = (uint64_t)opts->wait_timeout_ms * 1000000ull;

    MK_CUDA(h, mk::megakernel_prepare(p));
    MK_CUDA(h, mk::baseline_prepare(p));
    int per_sm = 0;
    MK_CUDA(h, mk::megakernel_occupancy(p, &per_sm));
    if (per_sm < 1) {
        h->msg = "megakernel does not fit on an SM";
        free_schedule(h);
        return MK_ERR_UNSUPPORTED;
    }
    h->info = I;
    h->has_schedule = true;
    return MK_OK;
}

extern "C" mk_status mk_build_schedule(mk_handle* h, int batch, int max_ctx,
                                       const mk_schedule_opts* opts) {
    return no_throw([&] { return build_schedule_impl(h, batch, max_ctx, opts); });
}

// A step is enqueued on the calling thread's current device; one whose handle
// lives on another device is refused (its buffers are not that device's memory).
static mk_status current_device_is(mk_handle* h) {
    int cur = -1;
    MK_CUDA(h, cudaGetDevice(&cur));
    if (cur != h->device) {
        h->msg = "the calling thread's current device is not the handle's device";
        return MK_ERR_INVALID_ARG;
    }
    return MK_OK;
}

static mk_status step_args(mk_handle* h, const int32_t* tokens, const int32_t* positions,
                           void* k_cache, void* v_cache, float* logits) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->has_schedule) return MK_ERR_NO_SCHEDULE;
    if (!tokens || !positions || !k_cache || !v_cache || !logits) return MK_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
        return MK_ERR_INVALID_ARG;
    return current_device_is(h);
}

extern "C" mk_status mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions,
                                    void* k_cache, void* v_cache, float* logits, void* stream) {
    mk_status st = step_args(h, tokens, positions, k_cache, v_cache, logits);
    if (st != MK_OK) return st;
    mk::Params p = h->params;
    p.tokens = tokens;
    p.positions = positions;
    p.kc = static_cast<uint16_t*>(k_cache);
    p.vc = static_cast<uint16_t*>(v_cache);
    p.logits = logits;
    MK_CUDA(h, mk::megakernel_launch(p, static_cast<cudaStream_t>(stream)));
    return MK_OK;
}

extern "C" mk_status mk_decode_steps_greedy(mk_handle* h, int32_t* tokens, int32_t* positions, void* k_cache,
                                            void* v_cache, float* logits, int32_t* generated, int n_steps,
                                            void* stream) {
    mk_status st = step_args(h, tokens, positions, k_cache, v_cache, logits);
    if (st != MK_OK) return st;
    if (n_steps < 1) return MK_ERR_INVALID_ARG;
    mk::Params p = h->params;
    p.tokens = tokens;
    p.positions = positions;
    p.kc = static_cast<uint16_t*>(k_cache);
    p.vc = static_cast<uint16_t*>(v_cache);
    p.logits = logits;
    // the step's selection overwrites the tokens and advances the positions it read
    // (their last reads come long before the LM head), so the next launch decodes
    // the chosen tokens with no host work in between
    p.next_tokens = tokens;
    p.next_positions = positions;
    for (int s = 0; s < n_steps; ++s) {
        p.gen_tokens = generated ? generated + (size_t)s * p.B : nullptr;
        MK_CUDA(h, mk::megakernel_launch(p, static_cast<cudaStream_t>(stream)));
    }
    return MK_OK;
}

extern "C" mk_status mk_baseline_decode_step(mk_handle* h, const int32_t* tokens,
                                             const int32_t* positions, void* k_cache,
                                             void* v_cache, float* logits, void* stream) {
    mk_status st = step_args(h, tokens, positions, k_cache, v_cache, logits);
    if (st != MK_OK) return st;
    mk::Params p = h->params;
    p.tokens = tokens;
    p.positions = positions;
    p.kc = static_cast<uint16_t*>(k_cache);
    p.vc = static_cast<uint16_t*>(v_cache);
    p.logits = logits;
    MK_CUDA(h, mk::baseline_launch(p, static_cast<cudaStream_t>(stream), h->dev_sms));
    return MK_OK;
}

extern "C" mk_status mk_decode_step_host(mk_handle* h, const int32_t* tokens_host,
                                         const int32_t* positions_host, void* k_cache,
                                         void* v_cache, float* logits_host, void* stream) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->has_schedule) return MK_ERR_NO_SCHEDULE;
    if (!tokens_host || !positions_host || !logits_host) return MK_ERR_INVALID_ARG;
    if (const mk_status st = current_device_is(h); st != MK_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int B = h->params.B, MB = h->cfg.max_batch;
    // tokens and positions travel in one copy, through the handle's pinned staging
    // (the previous call's copy has completed: every call ends with a stream sync)
    memcpy(h->h_io, tokens_host, B * sizeof(int32_t));
    memcpy(h->h_io + MB, positions_host, B * sizeof(int32_t));
    MK_CUDA(h, cudaMemcpyAsync(h->d_io, h->h_io, 2 * (size_t)MB * sizeof(int32_t), cudaMemcpyHostToDevice, s));
    mk_status st = mk_decode_step(h, h->d_io, h->d_io + h->cfg.max_batch, k_cache, v_cache,
                                  h->d_logits, stream);
    if (st != MK_OK) return st;
    MK_CUDA(h, cudaMemcpyAsync(logits_host, h->d_logits, (size_t)B * h->lay.V * sizeof(float),
                               cudaMemcpyDeviceToHost, s));
    MK_CUDA(h, cudaStreamSynchronize(s));
    return MK_OK;
}

extern "C" mk_status mk_get_status(mk_handle* h, mk_status* device_status, char* msg,
                                   size_t msg_len) {
    if (!h) return MK_ERR_INVALID_ARG;
    DeviceScope scope;
    MK_CUDA(h, scope.enter(h->device));
    MK_CUDA(h, cudaDeviceSynchronize());
    mk_status dev = MK_OK;
    std::string text = h->msg;
    if (h->ctl) {
        mk::Ctl c;
        MK_CUDA(h, cudaMemcpy(&c, h->ctl, sizeof(c), cudaMemcpyDeviceToHost));
        dev = static_cast<mk_status>(c.status);
        if (dev != MK_OK) {
            char buf[256];
            snprintf(buf, sizeof buf, "%s (sm %d, where %u, counter %u, seen %u, target %u, site %u)",
                     mk_status_str(dev), (int)c.info[0], c.info[1], c.info[2], c.info[3], c.info[4],
                     c.info[5]);
            text = buf;
            // clear: counters were reset by the last CTA of the failed step
            MK_CUDA(h, cudaMemset(&h->ctl->status, 0, sizeof(uint32_t) * 8));
        }
    }
    if (device_status) *device_status = dev;
    if (msg && msg_len) {
        strncpy(msg, text.c_str(), msg_len - 1);
        msg[msg_len - 1] = 0;
    }
    h->msg.clear();
    return MK_OK;
}

extern "C" mk_status mk_get_schedule_info(mk_handle* h, mk_schedule_info* info) {
    if (!h || !info) return MK_ERR_INVALID_ARG;
    if (!h->has_schedule) return MK_ERR_NO_SCHEDULE;
    *info = h->info;
    return MK_OK;
}

static mk_status read_counters_impl(mk_handle* h, uint32_t* host, size_t n, size_t* n_total) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->has_schedule) return MK_ERR_NO_SCHEDULE;
    const size_t nc = (size_t)h->info.n_counters;
    if (n_total) *n_total = nc + 2;
    if (!host || n == 0) return MK_OK;
    DeviceScope scope;
    MK_CUDA(h, scope.enter(h->device));
    MK_CUDA(h, cudaDeviceSynchronize());
    std::vector<uint32_t> raw(nc * mk::kCounterStride);
    MK_CUDA(h, cudaMemcpy(raw.data(), h->counters, raw.size() * sizeof(uint32_t), cudaMemcpyDeviceToHost));
    mk::Ctl c;
    MK_CUDA(h, cudaMemcpy(&c, h->ctl, sizeof(c), cudaMemcpyDeviceToHost));
    for (size_t i = 0; i < nc + 2 && i < n; ++i)
        host[i] = i < nc ? raw[i * mk::kCounterStride] : (i == nc ? c.epoch : c.done);
    return MK_OK;
}

extern "C" mk_status mk_read_counters(mk_handle* h, uint32_t* host, size_t n, size_t* n_total) {
    return no_throw([&] { return read_counters_impl(h, host, n, n_total); });
}

extern "C" mk_status mk_read_trace(mk_handle* h, uint64_t* host, size_t bytes, int32_t* jobs) {
    if (!h) return MK_ERR_INVALID_ARG;
    if (!h->has_schedule) return MK_ERR_NO_SCHEDULE;
    if (jobs) *jobs = h->trace_jobs;
    if (!h->d_trace || !host || bytes == 0) return MK_OK;
    const size_t tb = (size_t)h->params.n_sm * h->trace_jobs * mk::kTraceWords * sizeof(uint64_t);
    DeviceScope scope;
    MK_CUDA(h, scope.enter(h->device));
    MK_CUDA(h, cudaDeviceSynchronize());
    MK_CUDA(h, cudaMemcpy(host, h->d_trace, bytes < tb ? bytes : tb, cudaMemcpyDeviceToHost));
    return MK_OK;
}

extern "C" void mk_destroy(mk_handle* h) {
    if (!h) return;
    {
        DeviceScope scope;
        if (scope.enter(h->device) == cudaSuccess) cudaDeviceSynchronize();
        free_schedule(h);
        cudaFree(h->packed);
        cudaFree(h->rope);
        cudaFree(h->d_tmaps);
    }
    delete h;
}
