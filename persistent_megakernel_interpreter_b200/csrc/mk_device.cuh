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

// Non-blocking probe of phase `parity` (acquire at CTA scope when it has completed).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
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

// Tiled TMA loads (global -> this CTA's shared memory) through a tensor map in
// global memory, completion counted on `bar`. Coordinates innermost first; the
// innermost is a multiple of 64 elements here (128 bytes). No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int c0, int c1, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int c0, int c1, int c2, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const void* map, int c0, int c1, int c2, int c3, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const void* map, int c0, int c1, int c2, int c3, int c4,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_addr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Generic-proxy writes to shared memory by this thread become visible to the
// async proxy (the tensor cores' operand reads) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tagged activations
//
// Inside one megakernel launch, activations that cross SMs (residual stream x,
// q and the new key/value, attention output, MLP activations) travel as 64-bit
// words: the fp32 value in the low half and a tag in the high half naming the
// step, layer and producer. A single 64-bit access is indivisible, so a reader
// that sees the expected tag sees the value that goes with it; no fence orders
// the data before the dependency counter, and the counter becomes a hint of
// when to look. (A GPU-scope release fence waits for every memory operation
// the SM has in flight, bulk weight copies included: microseconds when the ring
// is full, on every signal.)
enum TagKind : uint32_t { kTagQKV = 1, kTagAttn = 2, kTagXAttn = 3, kTagH = 4, kTagXMlp = 5 };

__host__ __device__ __forceinline__ uint32_t act_tag(uint32_t epoch, int layer, uint32_t kind) {
    return (((epoch + 1u) & 0x3fffffu) << 10) | ((uint32_t)layer << 3) | kind;
}

__device__ __forceinline__ void st_tagged(uint64_t* p, float v, uint32_t tag) {
    const uint64_t w = ((uint64_t)tag << 32) | __float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ void ld_tagged2(const uint64_t* p, uint64_t& a, uint64_t& b) {
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

__device__ __forceinline__ uint64_t ld_tagged(const uint64_t* p) {
    uint64_t a;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(a) : "l"(p) : "memory");
    return a;
}

__device__ __forceinline__ bool tag_ok(uint64_t w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float tag_val(uint64_t w) { return __uint_as_float((uint32_t)w); }

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_relaxed_add(uint32_t* p, uint32_t v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// RMSNorm of the lane's KC x 8 input elements e (fp32) with norm weights w
// (bf16, the same layout): per-lane sum of squares in element order, the
// butterfly, then (x * r) * w into x. Every RMSNorm of the step goes through
// here, whatever the input's source.
template <int KC, class X>
__device__ __forceinline__ void rmsnorm_core(const float (&e)[KC][8], const uint4 (&wv)[KC], float eps, X& x,
                                             int lane) {
    float ss = 0.f;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc)
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(e[kc][i], e[kc][i], ss);
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)(KC * 256) + eps);
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        float wf[8], o[8];
        unpack8(wv[kc], wf);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = __fmul_rn(__fmul_rn(e[kc][i], r), wf[i]);
        x.put(kc, lane, o);
    }
}

// RMSNorm of a vector read from global memory (fp32, or bf16 when SRC_BF16),
// with every load -- the vector and the norm weights -- issued before the
// reduction.
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
    float e[KC][8];
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
        if (SRC_BF16) {
            unpack8(ra[kc], e[kc]);
        } else {
            e[kc][0] = __uint_as_float(ra[kc].x); e[kc][1] = __uint_as_float(ra[kc].y);
            e[kc][2] = __uint_as_float(ra[kc].z); e[kc][3] = __uint_as_float(ra[kc].w);
            e[kc][4] = __uint_as_float(rb[kc].x); e[kc][5] = __uint_as_float(rb[kc].y);
            e[kc][6] = __uint_as_float(rb[kc].z); e[kc][7] = __uint_as_float(rb[kc].w);
        }
    }
    rmsnorm_core<KC>(e, wv, eps, x, lane);
}

// ------------------------------------------------------------------ block-level job inputs
//
// A matvec job's input vector (n elements, n a multiple of 2 * kNT... or less)
// is loaded, and normalised where the op needs it, by all kConsumerWarps
// compute warps of the CTA together, into the XSmem order in shared memory.
// Thread t owns the element pairs j = i * kNT + t (i ascending). RMSNorm: each
// thread's sum of squares over its pairs in order, the warp butterfly, the warp
// sums added in warp order; then (x * r) * w for the thread's own elements. The
// megakernel and the baseline both go through here, so they agree bit for bit.
constexpr int kNT = 32 * kConsumerWarps;
constexpr int kMaxPairs = 8;  // vectors of up to 2 * 8 * kNT = 4096 elements

// Float index, inside an XSmem vector of n elements, of element e (its half, its
// group of 8, its place): elements e and e + 1 (e even) are adjacent.
__device__ __forceinline__ int xs_index(int n, int e) {
    return ((e & 4) ? n / 2 : 0) + (e >> 3) * 4 + (e & 3);
}

// The thread's pairs (v0[i], v1[i]) = elements 2j, 2j + 1 into the XSmem vector
// at xs; with w (bf16 norm weights of the pairs, pre-loaded in wv), RMSNorm
// first. `red`: kConsumerWarps floats of shared scratch. Ends with a barrier.
// The tensor cores' input operand (the megakernel's tensor-core path): row `row`
// (a sequence's high bf16 part; its low part is row 8 + row) of a K-major operand
// of 16 rows, stored as 64-column chunks of two 8-row atoms (2048 bytes a chunk),
// each 128-byte row with its 16-byte pieces swizzled by the row index (piece i at
// i ^ row). Elements k, k + 1 (k even) of x: the high parts round x to bf16, the
// low parts the exact fp32 remainder x - high, so high + low carries x to about
// 2^-17 relative.
__device__ __forceinline__ void mma_opnd_store(float* base, int row, int k, float x0, float x1) {
    uint8_t* p8 = reinterpret_cast<uint8_t*>(base) + (size_t)(k >> 6) * 2048 + row * 128 +
                  ((((k >> 3) & 7) ^ row) << 4) + (k & 7) * 2;
    const uint16_t h0 = f2bf(x0), h1 = f2bf(x1);
    const uint16_t l0 = f2bf(__fsub_rn(x0, bf2f(h0))), l1 = f2bf(__fsub_rn(x1, bf2f(h1)));
    *reinterpret_cast<uint32_t*>(p8) = (uint32_t)h0 | ((uint32_t)h1 << 16);
    *reinterpret_cast<uint32_t*>(p8 + 1024) = (uint32_t)l0 | ((uint32_t)l1 << 16);
}

// With MMAOP the pairs go into the tensor cores' operand at xs, row `orow`
// (mma_opnd_store) instead of an XSmem vector.
template <bool MMAOP = false, class Bar>
__device__ __forceinline__ bool block_store_input(const float (&v0)[kMaxPairs], const float (&v1)[kMaxPairs],
                                                  const uint32_t (&wv)[kMaxPairs], bool norm, float eps,
                                                  int n, float* xs, float* red, int t, int warp, int lane,
                                                  Bar&& bar, int orow = 0) {
    const int np = n / 2;
    float r = 1.f;
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxPairs; ++i)
            if (i * kNT + t < np) {
                ss = fmaf(v0[i], v0[i], ss);
                ss = fmaf(v1[i], v1[i], ss);
            }
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        if (!bar()) return false;
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) tot += red[w];
        r = 1.0f / sqrtf(tot / (float)n + eps);
    }
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int j = i * kNT + t;
        if (j < np) {
            float a = v0[i], b = v1[i];
            if (norm) {
                a = __fmul_rn(__fmul_rn(a, r), bf_lo(wv[i]));
                b = __fmul_rn(__fmul_rn(b, r), bf_hi(wv[i]));
            }
            if constexpr (MMAOP) mma_opnd_store(xs, orow, 2 * j, a, b);
            else *reinterpret_cast<float2*>(xs + xs_index(n, 2 * j)) = make_float2(a, b);
        }
    }
    return bar();
}

// The same from a plain source: fp32 (src_f) or bf16 (src_h) in global memory.
template <bool MMAOP = false, class Bar>
__device__ __forceinline__ bool block_input_plain(const float* src_f, const uint16_t* src_h, const uint16_t* w,
                                                  float eps, int n, float* xs, float* red, int t, int warp,
                                                  int lane, Bar&& bar, int orow = 0) {
    const int np = n / 2;
    float v0[kMaxPairs], v1[kMaxPairs];
    uint32_t wv[kMaxPairs];
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int j = i * kNT + t;
        v0[i] = v1[i] = 0.f;
        wv[i] = 0u;
        if (j < np) {
            if (w) wv[i] = ld_cg_u32(w + 2 * j);
            if (src_f) {
                const uint2 u = ld_cg_v2(src_f + 2 * j);
                v0[i] = __uint_as_float(u.x);
                v1[i] = __uint_as_float(u.y);
            } else {
                const uint32_t u = ld_cg_u32(src_h + 2 * j);
                v0[i] = bf_lo(u);
                v1[i] = bf_hi(u);
            }
        }
    }
    return block_store_input<MMAOP>(v0, v1, wv, w != nullptr, eps, n, xs, red, t, warp, lane, bar, orow);
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

// The 4-row tile in shared memory against the input vectors of B <= kMaxBatch
// sequences (XSmem layout, sequence b at xs + b * vec_floats): each 16-byte
// weight piece is read and unpacked once and applied to every sequence. Each
// (sequence, row) total comes from the same lane chains as dot4's and the same
// xor tree (16, 8, 4, 2, 1) as warp_sum, so it equals dot4's total for that
// sequence bit for bit; the tree is run as a reduce-scatter, after which lane l
// holds the total of sequence l / 4, row l % 4 (sequences >= B: zero).
template <int KC>
__device__ __forceinline__ float dot4_batch(const uint8_t* tile, const float* xs, uint32_t vec_floats, int B,
                                            int lane) {
    const uint4* t = reinterpret_cast<const uint4*>(tile) + lane;
    float v[kMaxBatch * 4];
#pragma unroll
    for (int i = 0; i < kMaxBatch * 4; ++i) v[i] = 0.f;
#pragma unroll 1
    for (int kc = 0; kc < KC; ++kc) {
        float w[4][8];
#pragma unroll
        for (int r = 0; r < 4; ++r) unpack8(lds_v4(t + r * KC * 32 + kc * 32), w[r]);
#pragma unroll
        for (int b = 0; b < kMaxBatch; ++b) {
            if (b < B) {
                const float4* x = reinterpret_cast<const float4*>(xs + (size_t)b * vec_floats);
                const float4 lo = x[kc * 32 + lane], hi = x[KC * 32 + kc * 32 + lane];
                const float e[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[b * 4 + r] = fmaf(w[r][i], e[i], v[b * 4 + r]);
            }
        }
    }
    // reduce-scatter: at mask m the lane keeps the half of its values whose index
    // bit matches its lane bit, adding the partner lane's partial of each
#pragma unroll
    for (int m = 16, n = 16; m > 0; m >>= 1, n >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float keep = up ? v[n + i] : v[i];
            const float send = up ? v[i] : v[n + i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0];
}

// The batched tile's reduction for at most 4 sequences: each lane holds 16
// partial sums v[b * 4 + r] (sequence b, row r) of its own input pieces, in dot4's
// lane order. They are reduce-scattered with warp_sum's masks 16, 8, 4, 2 and
// summed across the last pair with mask 1, so each total equals dot4's for its
// sequence bit for bit; lanes l and l ^ 1 hold the total of sequence l / 8, row
// (l / 2) % 4.
__device__ __forceinline__ float reduce_batch4(float (&v)[16], int lane) {
#pragma unroll
    for (int m = 16, n = 8; m > 1; m >>= 1, n >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float keep = up ? v[n + i] : v[i];
            const float send = up ? v[i] : v[n + i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
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
// layer's QKV block. TAGGED (the megakernel): q, and the new key and value as
// the bf16 values written to the cache, also go out as tagged words (q_t, kv_t)
// for the attention items of this step; otherwise q goes to the plain buffer.
template <int HD, bool TAGGED>
__device__ __forceinline__ void qkv_epilogue(const Params& p, int l, int b, uint32_t tile,
                                             const float (&acc)[4], int lane, const RopeRow& rr,
                                             uint32_t tag) {
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
            if (TAGGED) st_tagged(p.q_t + (size_t)b * p.Q + (size_t)head * HD + dim, out, tag);
            else p.q[(size_t)b * p.Q + (size_t)head * HD + dim] = out;
        } else {
            const uint16_t kb = f2bf(out);   // the cache is bf16
            p.kc[kv_off(p, l, b, g, pos) + dim] = kb;
            if (TAGGED) st_tagged(p.kv_t + ((size_t)(b * p.nkv + g) * 2) * HD + dim, bf2f(kb), tag);
        }
    } else {
        const uint16_t vb = f2bf(pick4(acc, lane));
        p.vc[kv_off(p, l, b, g, pos) + 4 * j + lane] = vb;
        if (TAGGED) st_tagged(p.kv_t + ((size_t)(b * p.nkv + g) * 2 + 1) * HD + 4 * j + lane, bf2f(vb), tag);
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
template <bool TAGGED>
__device__ __forceinline__ void gateup_epilogue(const Params& p, int b, uint32_t tile,
                                                const float (&acc)[4], int lane, uint32_t tag) {
    if (lane >= 2) return;
    const float g = lane ? acc[2] : acc[0], u = lane ? acc[3] : acc[1];
    const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
    const float h = __fmul_rn(silu, u);
    if (TAGGED) st_tagged(p.h_t + (size_t)b * p.F + 2 * tile + lane, h, tag);
    else p.hbuf[(size_t)b * p.F + 2 * tile + lane] = h;
}

__device__ __forceinline__ void logits_epilogue(const Params& p, int b, uint32_t tile,
                                                const float (&acc)[4], int lane) {
    if (lane >= 4) return;
    p.logits[(size_t)b * p.V + tile * 4 + lane] = pick4(acc, lane);
}

// ------------------------------------------------------------------ matvec op inputs/outputs

template <int OP, int HD>
__device__ __forceinline__ void tile_epilogue(const Params& p, int l, int b, uint32_t tile,
                                              const float (&acc)[4], int lane, const RopeRow& rr) {
    if constexpr (OP == MK_OP_QKV) qkv_epilogue<HD, false>(p, l, b, tile, acc, lane, rr, 0u);
    else if constexpr (OP == MK_OP_GATEUP) gateup_epilogue<false>(p, b, tile, acc, lane, 0u);
    else if constexpr (OP == MK_OP_OPROJ) residual_epilogue(p, l == 0, b, tile, acc, lane);
    else logits_epilogue(p, b, tile, acc, lane);
}

// ------------------------------------------------------------------ decode attention
//
// One attention item is one (sequence b, KV group g, key range [first,
// first + count)) of the split-K decode attention, restricted to keys <= pos
// (the key at pos is the one this step writes). The whole item runs on the
// compute warps of one CTA (256 threads), in one pass per warp and one merge:
//
//  * The keys are cut into passes of KPW keys (4 at head_dim 64, 2 at 128);
//    warp w takes passes w, w + 8, w + 16, ... and runs an online softmax over
//    them, NB passes at a time, for all of the group's query heads at once.
//  * Scores: LPK lanes per key (8 dims each), the group's query heads held in
//    registers. The partial dot products meet in a reduce-scatter butterfly
//    that leaves head 2*b2 + b1 on the lanes with lane bits (b2, b1), as
//    s_h(j) = (q_h . k_j) * (log2(e) / sqrt(HD)) (head_dim 128: bit 3 folded
//    first): the softmax runs in base 2, 2^(s - m) being e^((q . k) / sqrt(HD) - m')
//    for the same maximum.
//  * After each block of NB passes the warp's running maximum m_h becomes
//    max(m_h, block maximum), the running sums are scaled by 2^(m_old - m_new),
//    the block's weights e_h(j) = 2^(s_h(j) - m_h) are published to the warp's
//    scratch, and every lane adds e_h(j) * v_j over its DPL dims for every head.
//  * One CTA barrier; then thread (h, d) merges the warps in warp order:
//    M_h = max_w m_w,h, f_w = 2^(m_w,h - M_h), l_h = sum_w f_w l_w,h,
//    o_h[d] = sum_w f_w o_w,h[d]. Partials of several partitions (M_h in the same
//    base-2 units) merge the same way.
// With one partition per (sequence, group) the output is o_h / l_h; otherwise
// (M_h, l_h, o_h) is the partition's partial, merged in partition order. Every
// order of summation depends only on the key indices and the shape, not on
// where a row sits, so the megakernel (rows in its ring) and the multi-kernel
// baseline (rows copied to shared memory) give identical results.

// DPL: dims per lane in the values and the partial merge; LPK lanes per key in
// the scores; KPW keys per warp pass.
template <int HD>
struct AttnShape {
    static constexpr int DPL = HD / 32;
    static constexpr int LPK = HD / 8;
    static constexpr int KPW = 32 / LPK;
    static constexpr int NB = 5;                 // passes per online-softmax block (129 keys: one block per warp)
    static constexpr int BK = NB * KPW;          // keys per block
};

constexpr int kMaxGroup = kMaxGroupHeads;  // query heads per KV head handled by one item

// Offsets inside an item's scratch (attn_scratch_floats(HD) floats of shared
// memory): per warp a region of 4 * HD floats, holding a block's weights [BK][4]
// while the warp runs, then the warp's value sums [4][HD]; the warps' maxima and
// sums [warps][4] each; a flag word.
template <int HD>
struct AttnScratch {
    static constexpr uint32_t kWarp = 4 * HD;
    static constexpr uint32_t kWM = kConsumerWarps * kWarp;       // [warps][4]
    static constexpr uint32_t kWL = kWM + 4 * kConsumerWarps;    // [warps][4]
    static constexpr uint32_t kFlag = kWL + 4 * kConsumerWarps;
    static_assert(kFlag + 4 == attn_scratch_floats(HD), "attention scratch");
};

// The rows of an item in shared memory (knew and vnew always point at a valid
// row: they also stand in for rows past the item, whose results are masked). Row j (0 <= j < n) is key first + j. The
// rows sit in fills of kps rows: fill f is stage (s0 + f) mod S of a ring of S
// stages of `stage_bytes` at `base`, K rows first, V rows kps rows further on.
// Row jnew = n - 1, when the item holds the key at pos, is the exception: its
// key and value come from knew / vnew. n counts the item's keys at or before pos
// (<= 0: none).
template <int HD>
struct AttnRows {
    const uint8_t* base;
    uint32_t stage_bytes;
    int S, s0, kps;
    int n;
    int jnew;  // n - 1 or -1
    const uint16_t* knew;
    const uint16_t* vnew;
};

// Branch-free address of row j < R.n of the fills (key rows; V rows are kps
// rows further on): fill f = j / kps by a multiply-high with m = 2^32 / kps
// rounded up (exact for the few thousand rows an item can have), stage
// (s0 + f) mod S by one conditional subtraction (f < S).
template <int HD>
__device__ __forceinline__ const uint16_t* attn_row(const AttnRows<HD>& R, uint32_t m, int j) {
    const int f = (int)__umulhi((uint32_t)j, m);
    const int r = j - f * R.kps;
    int s = R.s0 + f;
    s = s >= R.S ? s - R.S : s;
    return reinterpret_cast<const uint16_t*>(R.base + (size_t)s * R.stage_bytes) + (size_t)r * HD;
}

// e^(a - b) for a running maximum a that may still be -inf (no key yet): 0.
__device__ __forceinline__ float exp_rel(float a, float b) { return a == -INFINITY ? 0.f : exp2f(a - b); }

// The item on all compute warps (warp < kConsumerWarps). qs: the group's G query
// heads, fp32 [G][HD], in shared memory; sc: attn_scratch_floats(HD) of shared
// memory; bar(): barrier of the compute warps (false: give up); mark(k): trace
// hook. R.jnew must be -1 or n - 1. On success emit(h, d, o, M_h, l_h) runs once
// for every output dim d < HD of every head h < G, on the thread that holds it.
template <int HD, class Bar, class Mark, class Emit>
__device__ __forceinline__ bool attn_item_block(const AttnRows<HD>& R, const float* qs, int G, float* sc,
                                                int warp, int lane, Bar&& bar, Mark&& mark, Emit&& emit) {
    using S = AttnShape<HD>;
    constexpr int NT = 32 * kConsumerWarps;
    constexpr int DPL = S::DPL, KPW = S::KPW, NB = S::NB;
    using SC = AttnScratch<HD>;
    static_assert(4 * S::BK <= (int)SC::kWarp && kMaxGroup * HD <= (int)SC::kWarp, "attention scratch");
    const int n = R.n, t = warp * 32 + lane;
    const int nc = R.jnew >= 0 ? n - 1 : n;  // rows read from the fills
    // scores in base 2: s = (q . k) * log2(e) / sqrt(HD), weights 2^(s - m) = e^((q . k) / sqrt(HD) - m')
    const float scale = 1.44269504088896341f / sqrtf((float)HD);
    float* ew = sc + (size_t)warp * SC::kWarp;  // this warp's region
    const int dc = lane % S::LPK, kk = lane / S::LPK;
    const int hh = ((lane & 4) ? 2 : 0) + ((lane & 2) ? 1 : 0);  // head this lane's scores belong to
    const bool writer = (lane & (S::LPK == 8 ? 1 : 9)) == 0;    // one lane per (key, head)
    const uint32_t m = 0xffffffffu / (uint32_t)R.kps + 1u;
    const size_t vofs = (size_t)R.kps * HD;
    float q[kMaxGroup][8];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h < G) {
            const float4 a = *reinterpret_cast<const float4*>(qs + h * HD + dc * 8);
            const float4 c = *reinterpret_cast<const float4*>(qs + h * HD + dc * 8 + 4);
            q[h][0] = a.x; q[h][1] = a.y; q[h][2] = a.z; q[h][3] = a.w;
            q[h][4] = c.x; q[h][5] = c.y; q[h][6] = c.z; q[h][7] = c.w;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) q[h][e] = 0.f;
        }
    }
    // running state: the maximum of head hh (lane's scores), the lane's share of
    // l_hh, and the value sums o[h][dd] of dims lane * DPL + dd for every head
    float mrun = -INFINITY, lpart = 0.f;
    float o[kMaxGroup][DPL];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) o[h][dd] = 0.f;
    const int npass = (n + KPW - 1) / KPW;
#pragma unroll 1
    for (int p0 = warp; p0 < npass; p0 += NB * kConsumerWarps) {
        // scores of NB passes: pass i covers keys (p0 + 8 i) * KPW + kk
        float s[NB];
        {
            float acc[NB][kMaxGroup];
            float kv[NB][8];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int j = (p0 + i * kConsumerWarps) * KPW + kk;
                // rows past the fills read the new key (a valid stand-in; masked below)
                const uint16_t* kr = j < nc ? attn_row<HD>(R, m, j) : R.knew;
                unpack8(lds_v4(kr + dc * 8), kv[i]);
            }
#pragma unroll
            for (int i = 0; i < NB; ++i)
#pragma unroll
                for (int h = 0; h < kMaxGroup; ++h) {
                    acc[i][h] = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[i][h] = fmaf(q[h][e], kv[i][e], acc[i][h]);
                }
            if (S::LPK == 16) {
#pragma unroll
                for (int i = 0; i < NB; ++i)
#pragma unroll
                    for (int h = 0; h < kMaxGroup; ++h) acc[i][h] += __shfl_xor_sync(0xffffffffu, acc[i][h], 8);
            }
            const bool b2 = lane & 4, b1 = lane & 2;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const float k0 = b2 ? acc[i][2] : acc[i][0], k1 = b2 ? acc[i][3] : acc[i][1];
                const float s0 = b2 ? acc[i][0] : acc[i][2], s1 = b2 ? acc[i][1] : acc[i][3];
                const float m0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 4);
                const float m1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 4);
                const float kp = b1 ? m1 : m0, sp = b1 ? m0 : m1;
                const float v = kp + __shfl_xor_sync(0xffffffffu, sp, 2);
                const float tot = v + __shfl_xor_sync(0xffffffffu, v, 1);
                const int j = (p0 + i * kConsumerWarps) * KPW + kk;
                s[i] = (j < n && hh < G) ? __fmul_rn(tot, scale) : -INFINITY;
            }
        }
        // the block's maximum per head: lanes holding the same head differ in bits 0, 3, 4
        float bm = s[0];
#pragma unroll
        for (int i = 1; i < NB; ++i) bm = fmaxf(bm, s[i]);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        const float mnew = fmaxf(mrun, bm);
        const float f = exp_rel(mrun, mnew);  // rescale of what the warp summed so far
        mrun = mnew;
        __syncwarp();  // the previous block's weights have been read
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            const float e = s[i] == -INFINITY ? 0.f : exp2f(s[i] - mnew);
            if (writer) {
                lpart = (i == 0 ? lpart * f : lpart) + e;
                ew[(i * KPW + kk) * 4 + hh] = e;
            }
        }
        // heads' rescale factors from the lanes holding them (lane 2h holds head h)
        float fh[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) fh[h] = __shfl_sync(0xffffffffu, f, 2 * h);
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) o[h][dd] *= fh[h];
        __syncwarp();
        // values: every key of the block, in pass order, for the lane's DPL dims. A
        // pass's KPW rows sit in one fill (a stage holds a multiple of KPW keys), so
        // its row address is found once per pass.
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            const int j0 = (p0 + i * kConsumerWarps) * KPW;
            const uint16_t* vb = attn_row<HD>(R, m, j0 < nc ? j0 : 0) + vofs;
#pragma unroll
            for (int k2 = 0; k2 < KPW; ++k2) {
                const int j = j0 + k2;
                const uint16_t* vr = j < nc ? vb + (size_t)k2 * HD : R.vnew;  // stand-in, masked
                float v[DPL];
                if constexpr (DPL == 2) {
                    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(vr + lane * 2);
                    v[0] = bf_lo(w2);
                    v[1] = bf_hi(w2);
                } else {
                    const uint2 w4 = *reinterpret_cast<const uint2*>(vr + lane * 4);
                    v[0] = bf_lo(w4.x);
                    v[1] = bf_hi(w4.x);
                    v[2] = bf_lo(w4.y);
                    v[3] = bf_hi(w4.y);
                }
                const float4 e4 = *reinterpret_cast<const float4*>(ew + (i * KPW + k2) * 4);
                const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
                    for (int dd = 0; dd < DPL; ++dd) o[h][dd] = fmaf(ev[h], v[dd], o[h][dd]);
            }
        }
    }
    // the warp's l per head: its writer lanes' shares, added over lane bits 3, 4
    lpart += __shfl_xor_sync(0xffffffffu, lpart, 8);
    lpart += __shfl_xor_sync(0xffffffffu, lpart, 16);
    __syncwarp();  // the last block's weights have been read
    if (lane < 8 && (lane & 1) == 0) {
        sc[SC::kWM + 4 * warp + hh] = hh < G ? mrun : -INFINITY;
        sc[SC::kWL + 4 * warp + hh] = hh < G ? lpart : 0.f;
    }
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
        if (h < G)
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) ew[h * HD + lane * DPL + dd] = o[h][dd];
    mark(0);
    if (!bar()) return false;
    mark(1);
    // merge the warps in warp order
#pragma unroll 1
    for (int u = t; u < G * HD; u += NT) {
        const int h = u / HD, d = u % HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sc[SC::kWM + 4 * w + h]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float fw = exp_rel(sc[SC::kWM + 4 * w + h], M);
            L = fmaf(fw, sc[SC::kWL + 4 * w + h], L);
            O = fmaf(fw, sc[(size_t)w * SC::kWarp + h * HD + d], O);
        }
        emit(h, d, O, M, L);
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
        w[i] = (lane < P && h0 + i * hstep < h_end) ? exp2f(w[i] - M) : 0.f;  // empty: 2^-inf = 0
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
