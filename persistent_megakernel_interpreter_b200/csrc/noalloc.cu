// A decode step for callers that cannot allocate device memory.
//
// Some hosts of this library cannot call cudaMalloc at the point where they
// decode: an engine whose device memory is reserved up front by an arena it
// controls, or a caller replaying work where allocation is not allowed. They
// can own their inputs and outputs (packed weights, KV cache, tokens,
// positions, logits) but not the step's scratch. For them,
// mk_baseline_decode_step_noalloc runs the multi-kernel decode step with every
// scratch buffer -- activations, attention partials, the RoPE table, the
// control block -- carved out of one file-scope device array of fixed size,
// reached through its symbol address. It allocates nothing, on the device or
// through any library. The array is this library's, per device, for the life
// of the process.
#include <cuda_runtime.h>

#include <math.h>
#include <mutex>

#include "mk_internal.h"

namespace mk {
cudaError_t baseline_launch(const Params& p, cudaStream_t stream, int n_sm);
cudaError_t baseline_prepare(const Params& p);
}  // namespace mk

namespace {

// The scratch of every no-allocation step on a device: 4 MiB. Its layout does not
// depend on the call's max_ctx: the control block (cleared by every call), then
// the RoPE table in a fixed 2 MiB region -- cos [kRopeRows(d)][d/2], then sin, for
// as many positions as the region holds at that head_dim (8192 at 64, 4096 at
// 128) -- then the step's activations and attention partials.
constexpr size_t kScratchBytes = 4u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
constexpr size_t kCtlBytes = 512;
constexpr size_t kRopeOff = kCtlBytes;
constexpr size_t kRopeBytes = 2u << 20;
constexpr size_t kActOff = kRopeOff + kRopeBytes;

// Positions the RoPE region holds at head dim d (cos and sin, d/2 floats each).
int rope_rows(int d) { return (int)(kRopeBytes / ((size_t)d * sizeof(float))); }

struct DeviceState {
    unsigned char* base = nullptr;  // device address of g_noalloc_scratch
    int n_sm = 0;
    // the RoPE table in the array (rebuilt when either changes)
    double theta = 0.0;
    int head_dim = 0;
};

std::mutex g_mutex;
DeviceState g_state[kMaxDevices];

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" mk_status mk_baseline_decode_step_noalloc(const mk_config* cfg, const void* packed,
                                                     const int32_t* tokens, const int32_t* positions,
                                                     void* k_cache, void* v_cache, float* logits, int batch,
                                                     int max_ctx, int32_t* status_out, void* stream) {
    if (!cfg || !packed || !tokens || !positions || !k_cache || !v_cache || !logits) return MK_ERR_INVALID_ARG;
    mk::Layout L;
    if (!mk::make_layout(*cfg, &L, nullptr)) return MK_ERR_UNSUPPORTED;
    if (batch < 1 || batch > cfg->max_batch || max_ctx < 1 || max_ctx > cfg->max_seq) return MK_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MK_ERR_CUDA;

    // split-K partitions of the attention: at most 320 keys each (16-key rounding)
    const int n_parts = (max_ctx + 319) / 320;
    if (n_parts > mk::kMaxParts) return MK_ERR_INVALID_ARG;
    const int part_keys = ((max_ctx + n_parts - 1) / n_parts + 15) / 16 * 16;

    // the scratch plan; calls whose scratch exceeds the array are refused
    const int half = L.d / 2;
    const int rows = rope_rows(L.d);
    if (max_ctx > rows) return MK_ERR_INVALID_ARG;
    size_t off = kActOff;
    const size_t o_x = off;
    off = up256(off + (size_t)batch * L.H * sizeof(float));
    const size_t o_q = off;
    off = up256(off + (size_t)batch * L.Q * sizeof(float));
    const size_t o_attn = off;
    off = up256(off + (size_t)batch * L.Q * sizeof(float));
    const size_t o_h = off;
    off = up256(off + (size_t)batch * L.F * sizeof(float));
    const size_t o_ml = off;
    off = up256(off + (size_t)batch * L.nq * n_parts * 2 * sizeof(float));
    const size_t o_po = off;
    off = up256(off + (size_t)batch * L.nq * n_parts * L.d * sizeof(float));
    if (off > kScratchBytes) return MK_ERR_INVALID_ARG;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& ds = g_state[dev];
    if (ds.base == nullptr) {
        // once per device, with the device current: the array's device address (in
        // host code the symbol itself is only a stand-in, not a device address)
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return MK_ERR_CUDA;
        if (cudaDeviceGetAttribute(&ds.n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MK_ERR_CUDA;
        ds.base = static_cast<unsigned char*>(ptr);
    }
    unsigned char* sb = ds.base;

    // the RoPE table of positions 0..rows-1 (angle pos * theta^(-2i/d) in double,
    // cos and sin stored as float), uploaded in pieces from the stack when theta or
    // the head dim differs from the table in the array. A capture cannot take the
    // upload (its source is on the stack): refused while the stream captures.
    float* cos_dst = reinterpret_cast<float*>(sb + kRopeOff);
    float* sin_dst = cos_dst + (size_t)rows * half;
    if (ds.theta != cfg->rope_theta || ds.head_dim != L.d) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return MK_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return MK_ERR_INVALID_ARG;
        constexpr int kChunk = 2048;
        float buf[kChunk];
        for (int table = 0; table < 2; ++table) {
            const size_t total = (size_t)rows * half;
            for (size_t e0 = 0; e0 < total; e0 += kChunk) {
                const size_t n = total - e0 < (size_t)kChunk ? total - e0 : (size_t)kChunk;
                for (size_t k = 0; k < n; ++k) {
                    const size_t e = e0 + k;
                    const int pos = (int)(e / half), i = (int)(e % half);
                    const double ang = (double)pos * pow(cfg->rope_theta, -(2.0 * i) / (double)L.d);
                    buf[k] = (float)(table == 0 ? cos(ang) : sin(ang));
                }
                // pageable source: the copy has read `buf` when the call returns
                if (cudaMemcpyAsync((table == 0 ? cos_dst : sin_dst) + e0, buf, n * sizeof(float),
                                    cudaMemcpyHostToDevice, st) != cudaSuccess)
                    return MK_ERR_CUDA;
            }
        }
        ds.theta = cfg->rope_theta;
        ds.head_dim = L.d;
    }
    // the control block must start at zero (the step's error word)
    if (cudaMemsetAsync(sb, 0, kCtlBytes, st) != cudaSuccess) return MK_ERR_CUDA;

    mk::Params p{};
    p.L = L.L; p.H = L.H; p.nq = L.nq; p.nkv = L.nkv; p.d = L.d; p.F = L.F; p.V = L.V;
    p.group = L.group; p.Q = L.Q; p.KVD = L.KVD;
    p.B = batch; p.max_batch = cfg->max_batch; p.max_seq = cfg->max_seq; p.max_ctx = max_ctx;
    p.eps = cfg->rms_eps;
    p.packed = static_cast<const uint8_t*>(packed);
    p.off_layer0 = L.off_layer0; p.layer_stride = L.layer_stride;
    p.rel_qkv = L.rel_qkv; p.rel_o = L.rel_o; p.rel_gu = L.rel_gu; p.rel_down = L.rel_down;
    p.off_norms = L.off_norms;
    p.tile_h = L.tile_h; p.tile_o = L.tile_o; p.tile_f = L.tile_f;
    p.rope_cos = cos_dst;
    p.rope_sin = sin_dst;
    p.tokens = tokens;
    p.positions = positions;
    p.kc = static_cast<uint16_t*>(k_cache);
    p.vc = static_cast<uint16_t*>(v_cache);
    p.logits = logits;
    p.x = reinterpret_cast<float*>(sb + o_x);
    p.q = reinterpret_cast<float*>(sb + o_q);
    p.attn = reinterpret_cast<float*>(sb + o_attn);
    p.hbuf = reinterpret_cast<float*>(sb + o_h);
    p.part_ml = reinterpret_cast<float*>(sb + o_ml);
    p.part_o = reinterpret_cast<float*>(sb + o_po);
    p.ctl = reinterpret_cast<mk::Ctl*>(sb);
    p.part_keys = part_keys;
    p.n_parts = n_parts;
    if (mk::baseline_prepare(p) != cudaSuccess) return MK_ERR_CUDA;
    if (mk::baseline_launch(p, st, ds.n_sm) != cudaSuccess) return MK_ERR_CUDA;
    // the step's device error word (MK_OK, MK_ERR_BAD_TOKEN, MK_ERR_BAD_POSITION)
    if (status_out != nullptr &&
        cudaMemcpyAsync(status_out, &p.ctl->status, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MK_ERR_CUDA;
    return MK_OK;
}
