// Device building blocks shared by the persistent megakernel and the
// multi-kernel baseline: PTX wrappers, the 4-row matvec tile, the fused
// epilogues (RoPE + KV append, residual add, SiLU-gated product, logits) and
// split-K decode attention with its merge.
//
// Precision: bf16 weights and KV cache, fp32 arithmetic and fp32 activations;
// the only rounding to bf16 is the key/value written to the cache.
//
// Work split inside a warp (batch-1 matvec, the memory-bound case the
// megakernel write-ups target): lane `ln` owns input elements
// (kc*32 + ln)*8 .. +7 for kc = 0..KC-1 (KC = in_dim / 256), holds them as fp32
// in registers and reads the matching 16-byte pieces of each weight row, so
// one warp-wide load covers 512 contiguous bytes of a row. Partial sums are
// combined with an xor butterfly, which leaves the identical total in every
// lane (each step adds the same two values in either order).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "mk_internal.h"

namespace mk {

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Same, but the thread sleeps (up to `ns` nanoseconds) until the phase
// completes instead of returning at once: waiting warps then leave their
// scheduler's issue slots to the warps that work.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// One-dimensional bulk copy global -> this CTA's shared memory, completion
// counted on `bar` (transaction bytes). No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_volatile_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Shared-memory counter of a CTA: acquire-release at CTA scope.
__device__ __forceinline__ uint32_t atom_shared_acq_rel_add(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "r"(smem_addr(p)), "r"(v)
                 : "memory");
    return old;
}

// Pull a byte range into L2 ahead of its use (no completion tracking).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes, uint64_t policy) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(src),
                 "r"(bytes), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_evict_normal_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Activations written earlier in the same kernel by other SMs: read at L2 (.cg).
// Plain intrinsics (not volatile asm), so independent loads issue together; the
// acquire loads that guard them clobber memory, so none is hoisted above its wait.
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
    return __ldcg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ uint2 ld_cg_v2(const void* p) {
    return __ldcg(reinterpret_cast<const uint2*>(p));
}
__device__ __forceinline__ uint32_t ld_cg_u32(const void* p) {
    return __ldcg(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ float ld_cg_f32(const float* p) { return __ldcg(p); }

// Weights streamed once per step: read-only path, no L1 allocation, evict-first in L2.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}

__device__ __forceinline__ uint4 lds_v4(const void* p) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(smem_addr(p)));
    return r;
}

// ------------------------------------------------------------------ bf16 helpers

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ float bf2f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float round_bf(float f) { return bf2f(f2bf(f)); }

__device__ __forceinline__ void unpack8(uint4 u, float* v) {
    v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
    v[4] = bf_lo(u.z); v[5] = bf_hi(u.z); v[6] = bf_lo(u.w); v[7] = bf_hi(u.w);
}

// Element `lane` (0..3) of a 4-vector without a dynamically indexed array.
__device__ __forceinline__ float pick4(const float (&a)[4], int i) {
    return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
    return v;
}

// ------------------------------------------------------------------ vectors in registers

// Input vectors of a matvec live either in registers (XRegs, the baseline
// kernels) or in the warp's slot of shared memory (XSmem, the megakernel, whose
// register file is shared with a deep instruction loop). Both hold lane `ln`'s
// elements (kc*32 + ln)*8 .. +7 and feed the same FMA sequence, so the two give
// identical sums. In XSmem the 8 elements sit as two float4 halves in separate
// arrays, so a warp-wide 16-byte load is conflict-free.
template <int KC>
struct XRegs {
    static constexpr int kUnroll = KC;  // register arrays need compile-time indices
    float v[KC][8];
    __device__ __forceinline__ void put(int kc, int lane, const float* e) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[kc][i] = e[i];
    }
    __device__ __forceinline__ void get(int kc, int lane, float* e) const {
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = v[kc][i];
    }
};

template <int KC>
struct XSmem {
    static constexpr int kUnroll = 2;   // short loop body: the megakernel's code stays small
    float4* a;  // [KC*32] elements 0..3 of each 8-element piece
    float4* b;  // [KC*32] elements 4..7
    __device__ __forceinline__ void put(int kc, int lane, const float* e) {
        a[kc * 32 + lane] = make_float4(e[0], e[1], e[2], e[3]);
        b[kc * 32 + lane] = make_float4(e[4], e[5], e[6], e[7]);
    }
    __device__ __forceinline__ void get(int kc, int lane, float* e) const {
        const float4 u = a[kc * 32 + lane], w = b[kc * 32 + lane];
        e[0] = u.x; e[1] = u.y; e[2] = u.z; e[3] = u.w;
        e[4] = w.x; e[5] = w.y; e[6] = w.z; e[7] = w.w;
    }
};

// Load an fp32 vector of KC*256 elements.
template <int KC, class X>
__device__ __forceinline__ void load_vec(const float* src, X& x, int lane) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        const uint4 a = ld_cg_v4(s + (kc * 32 + lane) * 2);
        const uint4 b = ld_cg_v4(s + (kc * 32 + lane) * 2 + 1);
        const float e[8] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z),
                            __uint_as_float(a.w), __uint_as_float(b.x), __uint_as_float(b.y),
                            __uint_as_float(b.z), __uint_as_float(b.w)};
        x.put(kc, lane, e);
    }
}

// The same from a bf16 vector (the embedding row).
template <int KC, class X>
__device__ __forceinline__ void load_vec_bf16(const uint16_t* src, X& x, int lane) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float e[8];
        unpack8(ld_cg_v4(s + kc * 32 + lane), e);
        x.put(kc, lane, e);
    }
}

// RMSNorm in place: x <- (x * r) * w with r = 1 / sqrt(mean(x^2) + eps), mean
// over the KC*256 elements.
template <int KC, class X>
__device__ __forceinline__ void rmsnorm_vec(X& x, const uint16_t* w, float eps, int lane) {
    float ss = 0.f;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float e[8];
        x.get(kc, lane, e);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(e[i], e[i], ss);
    }
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)(KC * 256) + eps);
    const uint4* wp = reinterpret_cast<const uint4*>(w);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float e[8], wv[8];
        x.get(kc, lane, e);
        unpack8(ld_cg_v4(wp + kc * 32 + lane), wv);
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = __fmul_rn(__fmul_rn(e[i], r), wv[i]);
        x.put(kc, lane, e);
    }
}

// RMSNorm of a vector read from global memory (fp32, or bf16 when SRC_BF16),
// with every load -- the vector and the norm weights -- issued before the
// reduction. The arithmetic (per-lane sum of squares in element order, the
// butterfly, (x * r) * w) is the same as load_vec + rmsnorm_vec.
template <int KC, bool SRC_BF16, class X>
__device__ __forceinline__ void load_rmsnorm(const void* src, const uint16_t* w, float eps, X& x,
                                             int lane) {
    uint4 ra[KC], rb[KC], wv[KC];
    const uint4* sp = reinterpret_cast<const uint4*>(src);
    const uint4* wp = reinterpret_cast<const uint4*>(w);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        if (SRC_BF16) {
            ra[kc] = ld_cg_v4(sp + kc * 32 + lane);
        } else {
            ra[kc] = ld_cg_v4(sp + (kc * 32 + lane) * 2);
            rb[kc] = ld_cg_v4(sp + (kc * 32 + lane) * 2 + 1);
        }
        wv[kc] = ld_cg_v4(wp + kc * 32 + lane);
    }
    float ss = 0.f;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float e[8];
        if (SRC_BF16) {
            unpack8(ra[kc], e);
        } else {
            e[0] = __uint_as_float(ra[kc].x); e[1] = __uint_as_float(ra[kc].y);
            e[2] = __uint_as_float(ra[kc].z); e[3] = __uint_as_float(ra[kc].w);
            e[4] = __uint_as_float(rb[kc].x); e[5] = __uint_as_float(rb[kc].y);
            e[6] = __uint_as_float(rb[kc].z); e[7] = __uint_as_float(rb[kc].w);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(e[i], e[i], ss);
    }
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)(KC * 256) + eps);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float e[8], wf[8];
        if (SRC_BF16) {
            unpack8(ra[kc], e);
        } else {
            e[0] = __uint_as_float(ra[kc].x); e[1] = __uint_as_float(ra[kc].y);
            e[2] = __uint_as_float(ra[kc].z); e[3] = __uint_as_float(ra[kc].w);
            e[4] = __uint_as_float(rb[kc].x); e[5] = __uint_as_float(rb[kc].y);
            e[6] = __uint_as_float(rb[kc].z); e[7] = __uint_as_float(rb[kc].w);
        }
        unpack8(wv[kc], wf);
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = __fmul_rn(__fmul_rn(e[i], r), wf[i]);
        x.put(kc, lane, e);
    }
}

// ------------------------------------------------------------------ the 4-row tile

__device__ __forceinline__ void fma8(float& acc, uint4 w, const float* x) {
    acc = fmaf(bf_lo(w.x), x[0], acc);
    acc = fmaf(bf_hi(w.x), x[1], acc);
    acc = fmaf(bf_lo(w.y), x[2], acc);
    acc = fmaf(bf_hi(w.y), x[3], acc);
    acc = fmaf(bf_lo(w.z), x[4], acc);
    acc = fmaf(bf_hi(w.z), x[5], acc);
    acc = fmaf(bf_lo(w.w), x[6], acc);
    acc = fmaf(bf_hi(w.w), x[7], acc);
}

// acc[r] = W_tile[r] . x for the 4 rows of a [4][KC*256] bf16 tile. The tile is
// in shared memory (SMEM) or read straight from global memory. Every lane
// returns the same four totals.
template <int KC, bool SMEM, class X>
__device__ __forceinline__ void dot4(const uint8_t* tile, const X& x, float (&acc)[4], int lane,
                                     uint64_t pol) {
    const uint4* t = reinterpret_cast<const uint4*>(tile);
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r] = 0.f;
#pragma unroll (X::kUnroll)
    for (int kc = 0; kc < KC; ++kc) {
        uint4 w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint4* a = t + r * KC * 32 + kc * 32 + lane;
            w[r] = SMEM ? lds_v4(a) : ld_stream_v4(a, pol);
        }
        float e[8];
        x.get(kc, lane, e);
#pragma unroll
        for (int r = 0; r < 4; ++r) fma8(acc[r], w[r], e);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r] = warp_sum(acc[r]);
}

// ------------------------------------------------------------------ per-op helpers

__device__ __forceinline__ const uint16_t* norm_ptr(const Params& p, size_t off) {
    return reinterpret_cast<const uint16_t*>(p.packed + off);
}

// The embedding row of sequence b's token (the residual stream before layer 0).
__device__ __forceinline__ const uint16_t* embed_row(const Params& p, int b) {
    return reinterpret_cast<const uint16_t*>(p.packed) + (size_t)p.tokens[b] * p.H;
}

__device__ __forceinline__ size_t kv_off(const Params& p, int l, int b, int g, int slot) {
    return ((((size_t)l * p.max_batch + b) * p.nkv + g) * p.max_seq + slot) * p.d;
}

// Per-sequence context of a tile epilogue: the position and its RoPE row
// (cos[HD/2], sin[HD/2]), in global memory (baseline) or staged in shared
// memory by the megakernel's activation warp -- the same values either way.
struct RopeRow {
    const float* cos;
    const float* sin;
    int pos;
};

__device__ __forceinline__ RopeRow rope_row_global(const Params& p, int b) {
    const int pos = p.positions[b];
    return {p.rope_cos + (size_t)pos * (p.d / 2), p.rope_sin + (size_t)pos * (p.d / 2), pos};
}

// QKV tile epilogue: RoPE on query/key pairs; q stays fp32, the key and value are
// rounded to bf16 into the cache slot. `tile` is the tile index inside the
// layer's QKV block.
template <int HD>
__device__ __forceinline__ void qkv_epilogue(const Params& p, int l, int b, uint32_t tile,
                                             const float (&acc)[4], int lane, const RopeRow& rr) {
    if (lane >= 4) return;
    constexpr int TPH = HD / 4;  // tiles per head
    const int g = tile / (uint32_t)((p.group + 2) * TPH);
    const int u = tile % (uint32_t)((p.group + 2) * TPH);
    const int hs = u / TPH, j = u % TPH;
    const int pos = rr.pos;
    if (hs <= p.group) {
        // query head (hs < group) or key head (hs == group): rows {2j, 2j+d/2, 2j+1, 2j+1+d/2}
        const int pair = lane >> 1;          // 0: freq 2j, 1: freq 2j+1
        const int i = 2 * j + pair;
        const float a = pair ? acc[2] : acc[0], bb = pair ? acc[3] : acc[1];
        const float c = rr.cos[i];
        const float s = rr.sin[i];
        float out;
        int dim;
        if ((lane & 1) == 0) {
            out = __fsub_rn(__fmul_rn(a, c), __fmul_rn(bb, s));
            dim = i;
        } else {
            out = __fadd_rn(__fmul_rn(bb, c), __fmul_rn(a, s));
            dim = i + HD / 2;
        }
        if (hs < p.group) {
            const int head = g * p.group + hs;
            p.q[(size_t)b * p.Q + (size_t)head * HD + dim] = out;
        } else {
            p.kc[kv_off(p, l, b, g, pos) + dim] = f2bf(out);   // the cache is bf16
        }
    } else {
        p.vc[kv_off(p, l, b, g, pos) + 4 * j + lane] = f2bf(pick4(acc, lane));
    }
}

// x[b][row] = xin[row] + y. The residual input is x itself, except for the
// first O-projection, whose input is the embedding row (`from_embed`).
__device__ __forceinline__ void residual_one(const Params& p, bool from_embed, int b, uint32_t row,
                                             float y) {
    const float xv = from_embed ? bf2f(embed_row(p, b)[row]) : ld_cg_f32(p.x + (size_t)b * p.H + row);
    p.x[(size_t)b * p.H + row] = __fadd_rn(xv, y);
}

// The tile's 4 consecutive rows; lanes 0..3 write one each.
__device__ __forceinline__ void residual_epilogue(const Params& p, bool from_embed, int b,
                                                  uint32_t tile, const float (&acc)[4], int lane) {
    if (lane >= 4) return;
    residual_one(p, from_embed, b, tile * 4 + lane, pick4(acc, lane));
}

// gate/up tile rows {g 2j, u 2j, g 2j+1, u 2j+1}: h = (g / (1 + e^-g)) * u.
__device__ __forceinline__ void gateup_epilogue(const Params& p, int b, uint32_t tile,
                                                const float (&acc)[4], int lane) {
    if (lane >= 2) return;
    const float g = lane ? acc[2] : acc[0], u = lane ? acc[3] : acc[1];
    const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
    p.hbuf[(size_t)b * p.F + 2 * tile + lane] = __fmul_rn(silu, u);
}

__device__ __forceinline__ void logits_epilogue(const Params& p, int b, uint32_t tile,
                                                const float (&acc)[4], int lane) {
    if (lane >= 4) return;
    p.logits[(size_t)b * p.V + tile * 4 + lane] = pick4(acc, lane);
}

// ------------------------------------------------------------------ matvec op inputs/outputs

// Input vector of a matvec op for sequence b.
template <int OP, int KC, class X>
__device__ __forceinline__ void prep_input(const Params& p, int l, int b, X& x, int lane) {
    if constexpr (OP == MK_OP_QKV) {
        const uint16_t* w = norm_ptr(p, p.off_norms + (size_t)(2 * l) * p.H * 2);
        if (l == 0) load_rmsnorm<KC, true>(embed_row(p, b), w, p.eps, x, lane);
        else load_rmsnorm<KC, false>(p.x + (size_t)b * p.H, w, p.eps, x, lane);
    } else if constexpr (OP == MK_OP_GATEUP) {
        load_rmsnorm<KC, false>(p.x + (size_t)b * p.H,
                                norm_ptr(p, p.off_norms + (size_t)(2 * l + 1) * p.H * 2), p.eps, x, lane);
    } else if constexpr (OP == MK_OP_OPROJ) {
        load_vec<KC>(p.attn + (size_t)b * p.Q, x, lane);
    } else {  // LM head
        load_rmsnorm<KC, false>(p.x + (size_t)b * p.H,
                                norm_ptr(p, p.off_norms + (size_t)(2 * p.L) * p.H * 2), p.eps, x, lane);
    }
}

template <int OP, int HD>
__device__ __forceinline__ void tile_epilogue(const Params& p, int l, int b, uint32_t tile,
                                              const float (&acc)[4], int lane, const RopeRow& rr) {
    if constexpr (OP == MK_OP_QKV) qkv_epilogue<HD>(p, l, b, tile, acc, lane, rr);
    else if constexpr (OP == MK_OP_GATEUP) gateup_epilogue(p, b, tile, acc, lane);
    else if constexpr (OP == MK_OP_OPROJ) residual_epilogue(p, l == 0, b, tile, acc, lane);
    else logits_epilogue(p, b, tile, acc, lane);
}

// ------------------------------------------------------------------ decode attention

// Lane layout for the scores: LPK lanes share one key (8 dims each); KPI keys per
// warp-wide step. For the value sum each lane owns DPL consecutive dims.
template <int HD>
struct AttnShape {
    static constexpr int LPK = HD / 8;
    static constexpr int KPI = 32 / LPK;
    static constexpr int DPL = HD / 32;
};

constexpr int kMaxGroup = 4;  // query heads per KV head handled by one instruction

template <int HD>
struct AttnState {
    float q[kMaxGroup][8];                        // this lane's 8 query dims, per head
    float m[kMaxGroup], l[kMaxGroup];             // running max and sum
    float o[kMaxGroup][AttnShape<HD>::DPL];       // running unnormalised output
};

// q for the group's heads: 8 dims per lane from qh (fp32 [group][HD]), read from
// shared memory (SMEM) or global memory.
template <int HD, bool SMEM>
__device__ __forceinline__ void attn_init(const Params& p, const float* qg, AttnState<HD>& st,
                                          int lane) {
    using S = AttnShape<HD>;
    const int dc = lane % S::LPK;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h < p.group) {
            const float* qh = qg + (size_t)h * HD + dc * 8;
            uint4 a, c;
            if (SMEM) {
                a = lds_v4(qh);
                c = lds_v4(qh + 4);
            } else {
                a = ld_cg_v4(qh);
                c = ld_cg_v4(qh + 4);
            }
            st.q[h][0] = __uint_as_float(a.x); st.q[h][1] = __uint_as_float(a.y);
            st.q[h][2] = __uint_as_float(a.z); st.q[h][3] = __uint_as_float(a.w);
            st.q[h][4] = __uint_as_float(c.x); st.q[h][5] = __uint_as_float(c.y);
            st.q[h][6] = __uint_as_float(c.z); st.q[h][7] = __uint_as_float(c.w);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) st.q[h][e] = 0.f;
        }
        st.m[h] = -INFINITY;
        st.l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < S::DPL; ++e) st.o[h][e] = 0.f;
    }
}

// One chunk of keys [ka, kend) (kend <= pos + 1, ka < kend). Rows of keys < pos
// come from Kc/Vc (row 0 = key ka); the key at `pos`, written earlier in this
// step, from Kpos/Vpos. All four are bf16 rows in shared memory when SMEM, else
// in global memory. `s` is this warp's score scratch in shared memory,
// [kMaxGroup][ks] floats. Independent passes are unrolled and the heads'
// reductions interleaved, so the chunk's latency is a few dependent steps.
template <int HD, bool SMEM>
__device__ __forceinline__ void attn_chunk(const Params& p, AttnState<HD>& st, const uint16_t* Kc,
                                           const uint16_t* Vc, const uint16_t* Kpos,
                                           const uint16_t* Vpos, int ka, int kend, int pos,
                                           float* s, int ks, int lane) {
    using S = AttnShape<HD>;
    const int n = kend - ka;
    const int dc = lane % S::LPK, kk = lane / S::LPK;
    const float scale = 1.0f / sqrtf((float)HD);
    // scores: S::KPI keys per pass, LPK lanes per key
#pragma unroll 2
    for (int base = 0; base < n; base += S::KPI) {
        const int j = base + kk;
        float part[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) part[h] = 0.f;
        if (j < n) {
            const int key = ka + j;
            const uint16_t* kr = (key < pos ? Kc + (size_t)j * HD : Kpos) + dc * 8;
            const uint4 raw = SMEM ? lds_v4(kr) : ld_cg_v4(kr);
            float kv[8];
            unpack8(raw, kv);
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) part[h] = fmaf(st.q[h][e], kv[e], part[h]);
        }
#pragma unroll
        for (int m = S::LPK / 2; m > 0; m >>= 1)
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) part[h] += __shfl_xor_sync(0xffffffffu, part[h], m);
        if (j < n && dc < p.group) {
            float mine = 0.f;
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h)
                if (dc == h) mine = part[h];
            s[dc * ks + j] = mine * scale;
        }
    }
    __syncwarp();
    // online softmax update, all heads together
    float cm[kMaxGroup], cs[kMaxGroup], m_new[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) cm[h] = -INFINITY;
    for (int j = lane; j < n; j += 32)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
            if (h < p.group) cm[h] = fmaxf(cm[h], s[h * ks + j]);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) cm[h] = fmaxf(cm[h], __shfl_xor_sync(0xffffffffu, cm[h], m));
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        m_new[h] = fmaxf(st.m[h], cm[h]);
        cs[h] = 0.f;
    }
    for (int j = lane; j < n; j += 32)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
            if (h < p.group) {
                const float e = expf(s[h * ks + j] - m_new[h]);
                s[h * ks + j] = e;
                cs[h] += e;
            }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) cs[h] += __shfl_xor_sync(0xffffffffu, cs[h], m);
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= p.group) continue;
        const float alpha = expf(st.m[h] - m_new[h]);   // 0 on the first chunk (m = -inf)
        st.l[h] = fmaf(st.l[h], alpha, cs[h]);
#pragma unroll
        for (int e = 0; e < S::DPL; ++e) st.o[h][e] *= alpha;
        st.m[h] = m_new[h];
    }
    __syncwarp();
    // values: keys in order, unrolled so the loads of several keys are in flight
#pragma unroll 2
    for (int j = 0; j < n; ++j) {
        const int key = ka + j;
        float v[S::DPL];
        const uint16_t* vr = (key < pos ? Vc + (size_t)j * HD : Vpos) + lane * S::DPL;
        if constexpr (S::DPL == 2) {
            const uint32_t w = SMEM ? *reinterpret_cast<const uint32_t*>(vr) : ld_cg_u32(vr);
            v[0] = bf_lo(w);
            v[1] = bf_hi(w);
        } else {
            static_assert(S::DPL == 4, "head_dim 64 or 128");
            const uint2 w = SMEM ? *reinterpret_cast<const uint2*>(vr) : ld_cg_v2(vr);
            v[0] = bf_lo(w.x);
            v[1] = bf_hi(w.x);
            v[2] = bf_lo(w.y);
            v[3] = bf_hi(w.y);
        }
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h >= p.group) continue;
            const float e = s[h * ks + j];
#pragma unroll
            for (int d = 0; d < S::DPL; ++d) st.o[h][d] = fmaf(e, v[d], st.o[h][d]);
        }
    }
    __syncwarp();
}

// ------------------------------------------------------------------ attention items
//
// An item is one (sequence, KV group, key range [first, first+count)) of the
// split-K attention. Its keys are cut into kSubRanges contiguous sub-ranges of
// ceil(count / kSubRanges) keys; each sub-range gets its own online-softmax
// partial (chunks cut at ring-stage boundaries, keys_per_stage apart from
// `first`), and the item's partial is the ordered combination of the
// sub-range partials, sub-range 0 first. Whether the sub-ranges run in
// parallel on several warps or one after another on one warp, every value is
// computed the same way.
constexpr int kSubRanges = kSubRangeCount;

__device__ __forceinline__ void sub_range(uint32_t first, uint32_t count, int u, int* lo, int* hi) {
    const int sub = (int)((count + kSubRanges - 1) / kSubRanges);
    *lo = (int)first + min(u * sub, (int)count);
    *hi = (int)first + min((u + 1) * sub, (int)count);
}

// Fold one head's partial (bm, bl, bo) into the running (M, L, O): rescale both
// to the larger max; an empty partial (m = -inf) leaves the other unchanged.
template <int HD>
__device__ __forceinline__ void fold_one(float& M, float& L, float (&O)[AttnShape<HD>::DPL], float bm,
                                         float bl, const float (&bo)[AttnShape<HD>::DPL]) {
    if (bm == -INFINITY) return;
    if (M == -INFINITY) {
        M = bm;
        L = bl;
#pragma unroll
        for (int d = 0; d < AttnShape<HD>::DPL; ++d) O[d] = bo[d];
        return;
    }
    const float Mn = fmaxf(M, bm);
    const float wa = expf(M - Mn), wb = expf(bm - Mn);
    L = fmaf(L, wa, bl * wb);
#pragma unroll
    for (int d = 0; d < AttnShape<HD>::DPL; ++d) O[d] = fmaf(O[d], wa, bo[d] * wb);
    M = Mn;
}

// Fold partial `b` into the running partial `a` (a = a (+) b) for every head:
// rescale both to the larger max. Empty partials (m = -inf) leave the other
// unchanged.
template <int HD>
__device__ __forceinline__ void fold_partial(float (&am)[kMaxGroup], float (&al)[kMaxGroup],
                                             float (&ao)[kMaxGroup][AttnShape<HD>::DPL],
                                             const float (&bm)[kMaxGroup], const float (&bl)[kMaxGroup],
                                             const float (&bo)[kMaxGroup][AttnShape<HD>::DPL]) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) fold_one<HD>(am[h], al[h], ao[h], bm[h], bl[h], bo[h]);
}

// One sub-range [lo, hi) of an item, keys < pos + 1 only. `rows(f, K, V)` gives
// the bf16 K/V rows of the item's fill f (row 0 = key first + f*kps) and may wait
// for it; `done(f)` is called once the warp no longer needs fill f.
template <int HD, bool SMEM, class Rows, class Done>
__device__ __forceinline__ bool attn_sub(const Params& p, AttnState<HD>& st, uint32_t first, int lo,
                                         int hi, int pos, const uint16_t* Kpos, const uint16_t* Vpos,
                                         float* s, int lane, Rows&& rows, Done&& done) {
    using S = AttnShape<HD>;
    const int kps = p.keys_per_stage;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        st.m[h] = -INFINITY;
        st.l[h] = 0.f;
#pragma unroll
        for (int d = 0; d < S::DPL; ++d) st.o[h][d] = 0.f;
    }
    hi = min(hi, pos + 1);
    if (lo >= hi) return true;
    const int f0 = (lo - (int)first) / kps, f1 = (hi - 1 - (int)first) / kps;
    for (int f = f0; f <= f1; ++f) {
        const int fa = (int)first + f * kps;
        const uint16_t *K, *V;
        if (!rows(f, K, V)) return false;
        const int ka = max(lo, fa), kb = min(hi, fa + kps);
        attn_chunk<HD, SMEM>(p, st, K + (size_t)(ka - fa) * HD, V + (size_t)(ka - fa) * HD, Kpos, Vpos,
                             ka, kb, pos, s, kps, lane);
        done(f);
    }
    return true;
}

// Write one head's partial (m, l, o) of partition `part`.
template <int HD>
__device__ __forceinline__ void attn_store_partial_head(const Params& p, float m, float l,
                                                        const float (&o)[AttnShape<HD>::DPL], int b,
                                                        int head, int part, int lane) {
    using S = AttnShape<HD>;
    const size_t hp = ((size_t)b * p.nq + (size_t)head) * p.n_parts + part;
    if (lane == 0) {
        p.part_ml[hp * 2] = m;
        p.part_ml[hp * 2 + 1] = l;
    }
#pragma unroll
    for (int d = 0; d < S::DPL; ++d) p.part_o[hp * HD + lane * S::DPL + d] = o[d];
}

// Write an item's (m, l, o) for the group's heads.
template <int HD>
__device__ __forceinline__ void attn_store_partial(const Params& p, const float (&m)[kMaxGroup],
                                                   const float (&l)[kMaxGroup],
                                                   const float (&o)[kMaxGroup][AttnShape<HD>::DPL],
                                                   int b, int g, int part, int lane) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
        if (h < p.group) attn_store_partial_head<HD>(p, m[h], l[h], o[h], b, g * p.group + h, part, lane);
}

// The attention output of one head from a partial that covers all its keys:
// o / l, the same value the merge of a single partition gives (weight e^0 = 1).
template <int HD>
__device__ __forceinline__ void attn_store_final_head(const Params& p, float l,
                                                      const float (&o)[AttnShape<HD>::DPL], int b,
                                                      int head, int lane) {
    using S = AttnShape<HD>;
    float* out = p.attn + (size_t)b * p.Q + (size_t)head * HD + lane * S::DPL;
#pragma unroll
    for (int d = 0; d < S::DPL; ++d) out[d] = __fdiv_rn(o[d], l);
}

// One whole item on one warp: the sub-ranges in order, each folded into the
// running partial as soon as it is done; the item's partial is left in
// (rm, rl, ro). `rows`/`done` as for attn_sub.
template <int HD, bool SMEM, class Rows, class Done>
__device__ __forceinline__ bool attn_item_serial(const Params& p, AttnState<HD>& st, uint32_t first,
                                                 uint32_t count, int pos, const uint16_t* Kpos,
                                                 const uint16_t* Vpos, float* s, int lane, Rows&& rows,
                                                 Done&& done, float (&rm)[kMaxGroup],
                                                 float (&rl)[kMaxGroup],
                                                 float (&ro)[kMaxGroup][AttnShape<HD>::DPL]) {
    using S = AttnShape<HD>;
    for (int u = 0; u < kSubRanges; ++u) {
        int lo, hi;
        sub_range(first, count, u, &lo, &hi);
        if (!attn_sub<HD, SMEM>(p, st, first, lo, hi, pos, Kpos, Vpos, s, lane, rows, done)) return false;
        if (u == 0) {
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                rm[h] = st.m[h];
                rl[h] = st.l[h];
#pragma unroll
                for (int d = 0; d < S::DPL; ++d) ro[h][d] = st.o[h][d];
            }
        } else {
            fold_partial<HD>(rm, rl, ro, st.m, st.l, st.o);
        }
    }
    return true;
}

// Merge the n_parts partials of NH heads h = h0 + i*hstep (i < NH; heads >=
// h_end are skipped) of sequence b, in partition order:
// attn = (sum_j e^(m_j - M) o_j) / (sum_j e^(m_j - M) l_j), M = max_j m_j.
// Lane j holds partition j's (m, l) and computes its weight (n_parts <= 32);
// the outputs of kMergeBatch partitions per head are loaded in one batch. The
// lane's DPL dims of head h go to out[h*HD + lane*DPL + d] through `put`.
constexpr int kMergeBatch = 8;

template <int HD, int NH, class Put>
__device__ __forceinline__ void attn_merge_heads(const Params& p, int b, int h0, int hstep, int h_end,
                                                 int lane, Put&& put) {
    using S = AttnShape<HD>;
    const int P = p.n_parts;
    float w[NH], l[NH], L[NH], O[NH][S::DPL], ov[NH][kMergeBatch][S::DPL];
    const float* po[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const int h = h0 + i * hstep;
        const size_t base = ((size_t)b * p.nq + h) * P;
        po[i] = p.part_o + base * HD + lane * S::DPL;
        w[i] = -INFINITY;
        l[i] = 0.f;
        if (h < h_end && lane < P) {
            w[i] = ld_cg_f32(p.part_ml + (base + lane) * 2);
            l[i] = ld_cg_f32(p.part_ml + (base + lane) * 2 + 1);
        }
    }
    auto load_o = [&](int j0) {
#pragma unroll
        for (int i = 0; i < NH; ++i) {
            const bool ok = h0 + i * hstep < h_end;
#pragma unroll
            for (int j = 0; j < kMergeBatch; ++j)
#pragma unroll
                for (int d = 0; d < S::DPL; ++d)
                    ov[i][j][d] = (ok && j0 + j < P) ? ld_cg_f32(po[i] + (j0 + j) * HD + d) : 0.f;
        }
    };
    load_o(0);
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const float M = warp_max(w[i]);
        w[i] = (lane < P && h0 + i * hstep < h_end) ? expf(w[i] - M) : 0.f;  // empty: e^-inf = 0
        L[i] = 0.f;
#pragma unroll
        for (int d = 0; d < S::DPL; ++d) O[i][d] = 0.f;
    }
    // partitions past P contribute w = 0 times o = 0 (exact no-ops)
#pragma unroll 1
    for (int j0 = 0; j0 < P; j0 += kMergeBatch) {
        if (j0 > 0) load_o(j0);
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
#pragma unroll
            for (int i = 0; i < NH; ++i) {
                const float wj = __shfl_sync(0xffffffffu, w[i], j0 + j);
                const float lj = __shfl_sync(0xffffffffu, l[i], j0 + j);
                L[i] = fmaf(wj, lj, L[i]);
#pragma unroll
                for (int d = 0; d < S::DPL; ++d) O[i][d] = fmaf(wj, ov[i][j][d], O[i][d]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NH; ++i) {
        const int h = h0 + i * hstep;
        if (h >= h_end) continue;
#pragma unroll
        for (int d = 0; d < S::DPL; ++d) put(h * HD + lane * S::DPL + d, __fdiv_rn(O[i][d], L[i]));
    }
}

}  // namespace mk
