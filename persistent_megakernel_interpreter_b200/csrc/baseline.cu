// The multi-kernel "bubble" baseline: the same decode step as one ordinary
// kernel per op and layer (about six launches per layer), the structure the
// megakernel write-ups measure against (the "Look Ma, No Bubbles" summaries,
// section "Memory Pipeline Bubbles Explained": every kernel boundary waits for
// stragglers, pays launch and teardown, and cannot prefetch the next op's
// weights). It uses the very same tile, epilogue and attention routines as the
// megakernel, with weights read straight from global memory, so the two give
// bit-identical results. Capturable in a CUDA graph.
#include <cuda_runtime.h>

#include "mk_device.cuh"

namespace mk {

constexpr int kBaseWarps = 8;
constexpr int kBaseThreads = 32 * kBaseWarps;
static_assert(kBaseThreads == kNT, "the block-level input routines assume the megakernel's compute warps");

__device__ __forceinline__ bool step_failed(const Params& p) {
    return ld_volatile_u32(&p.ctl->status) != 0u;
}

// Token and position checks, once per step, before any other kernel.
__global__ void k_validate(const __grid_constant__ Params p) {
    if (threadIdx.x != 0 || step_failed(p)) return;
    for (int b = 0; b < p.B; ++b) {
        const int tok = p.tokens[b], pos = p.positions[b];
        uint32_t code = 0;
        if (tok < 0 || tok >= p.V) code = MK_ERR_BAD_TOKEN;
        else if (pos < 0 || pos >= p.max_seq || pos + 1 > p.max_ctx) code = MK_ERR_BAD_POSITION;
        if (code) {
            if (atomicCAS(&p.ctl->status, 0u, code) == 0u) {
                p.ctl->info[0] = 0xffffffffu;
                p.ctl->info[1] = b;
                p.ctl->info[2] = (uint32_t)tok;
                p.ctl->info[3] = (uint32_t)pos;
            }
            return;
        }
    }
}

__device__ __forceinline__ const uint8_t* op_tiles(const Params& p, int op, int l) {
    const size_t lb = p.off_layer0 + (size_t)l * p.layer_stride;
    switch (op) {
        case MK_OP_QKV: return p.packed + lb + p.rel_qkv;
        case MK_OP_OPROJ: return p.packed + lb + p.rel_o;
        case MK_OP_GATEUP: return p.packed + lb + p.rel_gu;
        default: return p.packed;  // LM head: the embedding table
    }
}

// One matvec op of one layer. The CTA first builds each sequence's input vector
// in shared memory (RMSNorm where the op has one) with the same block routine as
// the megakernel; then each warp takes tiles.
template <int OP, int KC, int HD>
__global__ void __launch_bounds__(kBaseThreads) k_tiles(const __grid_constant__ Params p, int l,
                                                        uint32_t ntiles, uint32_t tile_bytes) {
    if (step_failed(p)) return;
    extern __shared__ __align__(16) float xs_all[];  // [B][KC*256], then kConsumerWarps floats
    constexpr int N = KC * 256;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    float* red = xs_all + (size_t)p.B * N;
    auto bar = []() {
        __syncthreads();
        return true;
    };
    for (int b = 0; b < p.B; ++b) {
        const float* sf = nullptr;
        const uint16_t* sh = nullptr;
        const uint16_t* w = nullptr;
        if (OP == MK_OP_QKV) {
            w = norm_ptr(p, p.off_norms + (size_t)(2 * l) * p.H * 2);
            if (l == 0) sh = embed_row(p, b);
            else sf = p.x + (size_t)b * p.H;
        } else if (OP == MK_OP_GATEUP) {
            w = norm_ptr(p, p.off_norms + (size_t)(2 * l + 1) * p.H * 2);
            sf = p.x + (size_t)b * p.H;
        } else if (OP == MK_OP_OPROJ) {
            sf = p.attn + (size_t)b * p.Q;
        } else {
            w = norm_ptr(p, p.off_norms + (size_t)(2 * p.L) * p.H * 2);
            sf = p.x + (size_t)b * p.H;
        }
        block_input_plain(sf, sh, w, p.eps, N, xs_all + (size_t)b * N, red, t, warp, lane, bar);
    }
    const uint32_t gw = blockIdx.x * kBaseWarps + warp;
    const uint32_t nw = gridDim.x * kBaseWarps;
    const uint64_t pol = l2_evict_first_policy();
    const uint8_t* base = op_tiles(p, OP, l);
    for (uint32_t tl = gw; tl < ntiles; tl += nw) {
        for (int b = 0; b < p.B; ++b) {
            float4* v = reinterpret_cast<float4*>(xs_all + (size_t)b * N);
            const XSmem<KC> x{v, v + KC * 32};
            float acc[4];
            dot4<KC, false>(base + (size_t)tl * tile_bytes, x, acc, lane, pol);
            RopeRow rr{nullptr, nullptr, 0};
            if constexpr (OP == MK_OP_QKV) rr = rope_row_global(p, b);
            tile_epilogue<OP, HD>(p, l, b, tl, acc, lane, rr);
        }
    }
}

template <int KF>
__global__ void __launch_bounds__(kBaseThreads) k_down(const __grid_constant__ Params p, int l) {
    if (step_failed(p)) return;
    const int lane = threadIdx.x & 31;
    const uint32_t gw = blockIdx.x * kBaseWarps + (threadIdx.x >> 5);
    const uint32_t nw = gridDim.x * kBaseWarps;
    const uint64_t pol = l2_evict_first_policy();
    const uint8_t* base = p.packed + p.off_layer0 + (size_t)l * p.layer_stride + p.rel_down;
    const uint32_t nrb = p.H / 4;
    for (uint32_t rb = gw; rb < nrb; rb += nw) {
        for (int b = 0; b < p.B; ++b) {
            float tot[4];
            XRegs<KF> x;
            for (int c = 0; c < 4; ++c) {
                load_vec<KF>(p.hbuf + (size_t)b * p.F + (size_t)c * (p.F / 4), x, lane);
                float acc[4];
                dot4<KF, false>(base + ((size_t)rb * 4 + c) * p.tile_f, x, acc, lane, pol);
#pragma unroll
                for (int k = 0; k < 4; ++k) tot[k] = (c == 0) ? acc[k] : tot[k] + acc[k];
            }
            residual_epilogue(p, false, b, rb, tot, lane);
        }
    }
}

// Rows of one item in the baseline's shared memory: kpad is the partition
// length rounded up to 16 keys (a multiple of every key-class count). All rows,
// the key at pos included, are read from the cache, in the same order of
// arithmetic as the megakernel's rows (whose last row, the key at pos, comes
// from the step's own k/v).
__host__ __device__ inline int attn_kpad(int part_keys) { return (part_keys + 15) / 16 * 16; }

template <int HD>
__host__ __device__ inline size_t attn_item_smem(int G, int kpad) {
    return (size_t)align16((uint32_t)(G * HD * 4)) + 2 * (size_t)kpad * HD * 2 + (size_t)attn_scratch_floats(HD) * 4;
}

// One attention item per CTA: the item's rows (keys first .. first + n - 1, the
// key at pos included, which the QKV kernel has written) are copied into shared
// memory as one fill, then the same four phases as the megakernel run on them.
template <int HD>
__global__ void __launch_bounds__(kBaseThreads) k_attn_item(const __grid_constant__ Params p, int l) {
    if (step_failed(p)) return;
    extern __shared__ __align__(16) uint8_t sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x % p.n_parts, g = (blockIdx.x / p.n_parts) % p.nkv;
    const int b = blockIdx.x / (p.n_parts * p.nkv);
    const int G = p.group, kpad = attn_kpad(p.part_keys);
    float* qs = reinterpret_cast<float*>(sm);
    uint16_t* rows = reinterpret_cast<uint16_t*>(sm + align16((uint32_t)(G * HD * 4)));
    float* sc = reinterpret_cast<float*>(rows + 2 * (size_t)kpad * HD);
    const int pos = p.positions[b];
    const int first = j * p.part_keys;
    const int count = min(p.part_keys, p.max_ctx - first);
    const int n = min(count, pos + 1 - first);
    const float* qsrc = p.q + (size_t)b * p.Q + (size_t)g * G * HD;
    for (int e = threadIdx.x * 4; e < G * HD; e += kBaseThreads * 4)
        *reinterpret_cast<uint4*>(qs + e) = ld_cg_v4(qsrc + e);
    const size_t base = kv_off(p, l, b, g, first);
    for (int i = threadIdx.x; i < n * (HD / 8); i += kBaseThreads) {
        reinterpret_cast<uint4*>(rows)[i] = ld_cg_v4(p.kc + base + (size_t)i * 8);
        reinterpret_cast<uint4*>(rows + (size_t)kpad * HD)[i] = ld_cg_v4(p.vc + base + (size_t)i * 8);
    }
    __syncthreads();
    // one fill of kpad rows; no row is special (knew / vnew only stand in for
    // rows past the item)
    const AttnRows<HD> R{reinterpret_cast<const uint8_t*>(rows), 0u, 1, 0, kpad, n, -1, rows,
                         rows + (size_t)kpad * HD};
    auto bar = []() {
        __syncthreads();
        return true;
    };
    if (p.n_parts == 1) {
        float* out = p.attn + (size_t)b * p.Q + (size_t)g * G * HD;
        attn_item_block<HD>(R, qs, G, sc, warp, lane, bar, [](int) {},
                            [&](int h, int d, float o, float, float l) { out[h * HD + d] = __fdiv_rn(o, l); });
    } else {
        attn_item_block<HD>(R, qs, G, sc, warp, lane, bar, [](int) {}, [&](int h, int d, float o, float m, float l) {
            const size_t hp = ((size_t)b * p.nq + (size_t)(g * G + h)) * p.n_parts + j;
            p.part_o[hp * HD + d] = o;
            if (d == 0) {
                p.part_ml[hp * 2] = m;
                p.part_ml[hp * 2 + 1] = l;
            }
        });
    }
}

template <int HD>
__global__ void __launch_bounds__(kBaseThreads) k_attn_merge(const __grid_constant__ Params p) {
    if (step_failed(p)) return;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kBaseWarps + (threadIdx.x >> 5);
    if (gw >= p.B * p.nq) return;
    const int b = gw / p.nq, head = gw % p.nq;
    float* out = p.attn + (size_t)b * p.Q;
    attn_merge_heads<HD, 1>(p, b, head, 1, p.nq, lane, [&](int e, float x) { out[e] = x; });
}

// ------------------------------------------------------------------ host-side launch

template <int KH, int KO, int KF, int HD>
static cudaError_t launch_all(const Params& p, cudaStream_t st, int n_sm) {
    const uint32_t warps_cap = (uint32_t)n_sm * 16;
    auto blocks_for = [&](uint32_t units) {
        const uint32_t w = units < warps_cap ? units : warps_cap;
        return (w + kBaseWarps - 1) / kBaseWarps;
    };
    const size_t attn_smem = attn_item_smem<HD>(p.group, attn_kpad(p.part_keys));
    const size_t in_h = (size_t)p.B * KH * 256 * 4 + 4 * kConsumerWarps;
    const size_t in_o = (size_t)p.B * KO * 256 * 4 + 4 * kConsumerWarps;
    k_validate<<<1, 32, 0, st>>>(p);
    const uint32_t tpg = (uint32_t)(p.group + 2) * (HD / 4);
    for (int l = 0; l < p.L; ++l) {
        const uint32_t nq = (uint32_t)p.nkv * tpg;
        k_tiles<MK_OP_QKV, KH, HD><<<blocks_for(nq), kBaseThreads, in_h, st>>>(p, l, nq, p.tile_h);
        const uint32_t na = (uint32_t)(p.B * p.nkv * p.n_parts);
        k_attn_item<HD><<<na, kBaseThreads, attn_smem, st>>>(p, l);
        if (p.n_parts > 1) {
            const uint32_t nm = (uint32_t)(p.B * p.nq);
            k_attn_merge<HD><<<(nm + kBaseWarps - 1) / kBaseWarps, kBaseThreads, 0, st>>>(p);
        }
        const uint32_t no = (uint32_t)p.H / 4;
        k_tiles<MK_OP_OPROJ, KO, HD><<<blocks_for(no), kBaseThreads, in_o, st>>>(p, l, no, p.tile_o);
        const uint32_t ng = (uint32_t)p.F / 2;
        k_tiles<MK_OP_GATEUP, KH, HD><<<blocks_for(ng), kBaseThreads, in_h, st>>>(p, l, ng, p.tile_h);
        k_down<KF><<<blocks_for((uint32_t)p.H / 4), kBaseThreads, 0, st>>>(p, l);
    }
    const uint32_t nl = (uint32_t)p.V / 4;
    k_tiles<MK_OP_LMHEAD, KH, HD><<<blocks_for(nl), kBaseThreads, in_h, st>>>(p, 0, nl, p.tile_h);
    return cudaGetLastError();
}

// Shared memory of the attention kernel for the current schedule (set once per
// schedule, outside any stream capture).
template <int KH, int KO, int HD>
static cudaError_t prepare_tiles(const Params& p) {
    const int in_h = (int)((size_t)p.B * KH * 256 * 4 + 4 * kConsumerWarps);
    const int in_o = (int)((size_t)p.B * KO * 256 * 4 + 4 * kConsumerWarps);
    cudaError_t e = cudaFuncSetAttribute(k_tiles<MK_OP_QKV, KH, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, in_h);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_tiles<MK_OP_GATEUP, KH, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, in_h);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_tiles<MK_OP_LMHEAD, KH, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, in_h);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_tiles<MK_OP_OPROJ, KO, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, in_o);
    return e;
}

cudaError_t baseline_prepare(const Params& p) {
    const int KH = p.H / 256, KO = p.Q / 256;
    cudaError_t e = cudaErrorInvalidValue;
    if (KH == 2 && KO == 2 && p.d == 64) e = prepare_tiles<2, 2, 64>(p);
    else if (KH == 8 && KO == 8 && p.d == 64) e = prepare_tiles<8, 8, 64>(p);
    else if (KH == 12 && KO == 12 && p.d == 128) e = prepare_tiles<12, 12, 128>(p);
    if (e != cudaSuccess) return e;
    const int kpad = attn_kpad(p.part_keys);
    if (p.d == 64)
        return cudaFuncSetAttribute(k_attn_item<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)attn_item_smem<64>(p.group, kpad));
    if (p.d == 128)
        return cudaFuncSetAttribute(k_attn_item<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)attn_item_smem<128>(p.group, kpad));
    return cudaErrorInvalidValue;
}

cudaError_t baseline_launch(const Params& p, cudaStream_t stream, int n_sm) {
    const int KH = p.H / 256, KO = p.Q / 256, KF = p.F / 1024;
    if (KH == 2 && KO == 2 && KF == 2 && p.d == 64) return launch_all<2, 2, 2, 64>(p, stream, n_sm);
    if (KH == 8 && KO == 8 && KF == 8 && p.d == 64) return launch_all<8, 8, 8, 64>(p, stream, n_sm);
    if (KH == 12 && KO == 12 && KF == 8 && p.d == 128) return launch_all<12, 12, 8, 128>(p, stream, n_sm);
    return cudaErrorInvalidValue;
}

}  // namespace mk
