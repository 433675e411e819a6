// The persistent decode megakernel: one CTA per SM runs the whole decode step.
//
// Structure (after the megakernel write-ups: "Look Ma, No Bubbles" summaries,
// sections "Fusing Operations with an On-GPU Interpreter", "Efficient Shared
// Memory Management", "Custom Synchronization Mechanism"; and the Cohere decode
// megakernel, sections on the host task list, weight prefetch ahead of
// activation waits, and static warp-specialised pipelines instead of paging):
//
//  * The host writes one instruction list per SM; the CTA runs it in order, one
//    job at a time for all compute warps (a down-projection instruction is four
//    jobs, one per MLP chunk).
//  * Warp 8 (the loader) streams, in list order, every byte the instructions
//    read from HBM that is final at launch -- weight tiles and the cached KV
//    slots -- into a ring of shared-memory stages with bulk async copies
//    (cp.async.bulk, completion counted on an mbarrier, L2 evict-first). It
//    never waits on a dependency, so the next instructions' weights arrive
//    while the step still waits for their activations.
//  * Activations cross SMs as 64-bit tagged words (value | step, layer, kind)
//    written with relaxed stores: a consumer polls the words themselves until
//    every tag is current, so no release fence (which would wait for the SM's
//    bulk copies in flight) sits on the data path. Counters remain as relaxed
//    completion counts.
//  * Warps 0..7 (compute) build each job's input themselves from the tagged
//    words (RMSNorm for QKV, gate/up and the LM head; the attention output and
//    the residual rows for the O-projection; q and the new key/value for an
//    attention item), split the job's tiles (tile t goes to warp t mod 8) and
//    write the outputs with fused epilogues.
//  * Warp 9 (the activation warp) runs ahead of the compute warps through the
//    same jobs: it stages the RoPE rows of QKV jobs and, at batch 1, the h
//    chunks of the first down-projection jobs, which gate/up completes chunk by
//    chunk while it still streams (the compute warps load the last ones).
//  * Attention items finish their own heads: with one key partition per
//    (sequence, KV group) the item writes o / l; with several, each stores its
//    partial and the one that completes the pair's arrival count merges the
//    pair in partition order, so no other SM waits on a merge.
//  * Counters only grow and tags carry the step's epoch: the last CTA to finish
//    advances the epoch, so no reset kernel is needed.
//  * Every wait is bounded by a time budget; on expiry the step records
//    MK_ERR_TIMEOUT, raises an abort flag that every other wait polls, drains
//    its own copies in flight and returns. No trap, no unbounded spin.
//
// This file is compiled twice: as is, and with MK_TRACE=1 (megakernel_trace.cu)
// into a second namespace whose kernels also record per-job timestamps. The
// timestamps stay out of the production kernels altogether: the code a kernel
// carries is what every SM re-fetches as it moves between ops.
#include <cuda_runtime.h>

#include "mk_device.cuh"

#ifndef MK_TRACE
#define MK_TRACE 0
#endif

namespace mk {
#if MK_TRACE
namespace traced {
#else
namespace plain {
#endif

// Each sequence's position, read once per step by thread 0 (constant during
// the step) so the warps do not reload it from global memory.
__shared__ int g_pos[kMaxBatch];

constexpr int kPairGroups = kConsumerWarps / 2;  // batch > 1: tiles in work at once (two warps each)
// Batch 1: the activation warp stages the h chunks of down-projection chunks
// c < kDownStaged ahead (they complete while gate/up still streams); the last
// chunk, which completes only as gate/up ends, is loaded by all compute warps
// (1B step, same box: staging 1 / 2 / 3 chunks ahead 627 / 611 / 594 us).
constexpr int kDownStaged = 3;

struct Ring {
    uint8_t* base;
    uint64_t* full;
    uint64_t* empty;
    // Fill number the loader last armed on each stage. The mover warps and (for
    // an attention item's cached KV) the compute warps may look for a fill several
    // laps ahead; an mbarrier parity alone only tells phases one lap
    // apart, so a warp first waits until its stage holds its fill, then waits on
    // the parity.
    volatile uint32_t* armed;
    uint32_t stage_bytes;
    uint32_t S;
    __device__ __forceinline__ uint8_t* stage(uint32_t seq) const {
        return base + (size_t)(seq % S) * stage_bytes;
    }
};

// ------------------------------------------------------------------ Tensor Memory
//
// The SM's 256 KB of Tensor Memory hold weight tiles that have landed in the
// ring, so the ring's stages are free again for the next fills as soon as a
// tile is moved: the SM then keeps stages + Tensor Memory slots worth of weights
// on chip while its compute warps wait on the step's dependency chain. A warp
// may only address the 32 lanes of its quarter (its warp index mod 4); slot k
// lies in quarter k mod 4, columns (k / 4) * cols .. +cols, and holds the tile of
// fill seq with seq mod n = k. The mover warp of that quarter stores it, the
// compute warp seq mod 8 (two at batch > 1, seq mod 4 and seq mod 4 + 4) reads it.

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Lane i of the warp stores r[0..15] into lane (quarter base + i), columns
// ta .. ta + 15.
__device__ __forceinline__ void tmem_st16(uint32_t ta, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};" ::"r"(ta),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// The reverse of tmem_st16. The registers are valid only after tmem_wait_ld,
// which names them as operands so the compiler reads none of them earlier.
__device__ __forceinline__ void tmem_ld16(uint32_t ta, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

struct Tmem {
    uint32_t base;              // address of the allocation (lane 0, its first column)
    uint64_t* full;             // [n] the mover arrives when a slot holds its fill
    uint64_t* empty;            // [n] the compute warp(s) arrive when done with it
    volatile uint32_t* armed;   // [n] the fill a slot holds (or last held)
    uint32_t n;                 // slots (a multiple of 4)
    uint32_t cols;              // columns of one slot
    // the slot of fill seq, addressed by `warp` (which must be in the slot's quarter)
    __device__ __forceinline__ uint32_t addr(uint32_t seq, int warp) const {
        const uint32_t k = seq % n;
        return base + ((32u * (uint32_t)(warp & 3)) << 16) + (k / 4u) * cols;
    }
};

// ------------------------------------------------------------------ tensor-core MMA (batch > 1)
//
// On the tensor-core path Tensor Memory holds fp32 accumulators instead of weight
// tiles: segment accumulator a is columns a * 64 .. +63 of all 128 lanes, four
// partial sums u of 16 columns; lane m is the segment's row m, column u * 16 + n
// the input row n (sequence n's high bf16 part for n < 8, sequence n - 8's low
// part above).

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle
// (8-row atoms of 128-byte rows, atoms 1024 bytes apart): start address >> 4
// (bits 0-13), leading offset 1 (unused by this layout, bits 16-29), stride
// 1024 >> 4 between atoms (bits 32-45), descriptor version 1 (bits 46-47),
// layout 2 = 128-byte swizzle (bits 61-63). K advances by 16 elements inside an
// atom by adding 32 bytes to the start address.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 and 10-12 = 1), both K-major, N = 16 (bits 17-22 = N / 8),
// M = 128 (bits 24-28 = M / 16).
constexpr uint32_t kMmaIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((kMmaRows >> 4) << 24);

// D[tmem] (+)= A * B^T for one K = 16 step, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kMmaIdesc), "r"(accumulate)
        : "memory");
}
// One arrival on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// The slot barriers complete one phase per matvec job in the slot (attention jobs,
// which use slots too, pass them by): the issuer and the compute warps each keep
// the slots' phase bits as they walk the same job sequence.
struct MmaBars {
    uint64_t* opnd;    // [NS] each compute warp arrives once the job's operand is written
    uint64_t* mdone;   // [NS] the issuer's commit: the job's MMAs are done with its slot
    uint64_t* afull;   // [kMaxAcc] the issuer's commit: a segment's accumulator is final
    uint64_t* aempty;  // [kMaxAcc] each compute warp arrives once it has read it out
    uint64_t* fin;     // the issuer's last commit
};

struct Slots {
    uint8_t* base;
    uint64_t* full;    // the job's preparer (activation or stage warp) arrives when its input is ready
    // The job each slot was last prepared for. Several warps prepare jobs, so the
    // preparer of job j first waits until its slot was prepared for job j - NS, and
    // only then on the empty parity (which tells phases one lap apart only).
    volatile uint32_t* job;
    uint64_t* empty;   // each compute warp arrives when it is done with the job
    uint32_t* done;    // compute warps finished with the job (the last one signals)
    uint32_t bytes;
    uint32_t NS;
    __device__ __forceinline__ uint8_t* slot(uint32_t job) const {
        return base + (size_t)(job % NS) * bytes;
    }
};

// Tile t of a gate/up instruction: chunk-major, the same slice of each chunk.
__device__ __forceinline__ uint32_t gu_tile(const Params& p, const mk_instr& in, uint32_t t) {
    const uint32_t c = t / in.aux0;
    return c * (uint32_t)(p.F / 8) + in.first + (t - c * in.aux0);
}

// ------------------------------------------------------------------ errors and waits

__device__ __noinline__ void record_error(const Params& p, uint32_t code, uint32_t a, uint32_t b, uint32_t c,
                             uint32_t d, uint32_t e) {
    if (atomicCAS(&p.ctl->status, 0u, code) == 0u) {
        p.ctl->info[0] = blockIdx.x;
        p.ctl->info[1] = a;
        p.ctl->info[2] = b;
        p.ctl->info[3] = c;
        p.ctl->info[4] = d;
        p.ctl->info[5] = e;
        __threadfence();
    }
    atomicExch(&p.ctl->abort, 1u);
}

__device__ __forceinline__ bool aborted(const Params& p) {
    return ld_volatile_u32(&p.ctl->abort) != 0u;
}



// All lanes wait for phase `parity` of an mbarrier; warp-uniform exit. With
// `armed`, first wait until the ring stage holds fill `seq`. Waiting threads
// sleep in the barrier (suspend hint) or back off, so they do not compete for
// issue slots with the warps that compute. Out of line: the inline wait_bar
// below tries once first.
__device__ __noinline__ bool wait_bar_slow(const Params& p, uint64_t* bar, uint32_t parity,
                                           const volatile uint32_t* armed, uint32_t seq, uint32_t site, int lane,
                                           uint32_t sleep_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        bool done;
        if (armed != nullptr && *armed != seq) {
            __nanosleep(64);
            done = false;
        } else {
            done = mbar_wait_sleep(bar, parity, sleep_ns);
        }
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 15u) == 15u) {
            int bad = 0;
            if (lane == 0) {
                if (t0 == 0) t0 = global_timer_ns();
                if (aborted(p)) bad = 1;
                else if (global_timer_ns() - t0 > p.timeout_ns) {
                    record_error(p, MK_ERR_TIMEOUT, seq, 0xfffffff0u + site, 0, parity, site);
                    bad = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) return false;
        }
    }
}

// The sleep hint bounds how long a waiting thread stays suspended; a phase that
// completes by a thread's arrival or a copy's bytes wakes it at once.
constexpr uint32_t kSleepNs = 20000u;
// Phases completed by tcgen05.commit: waiters poll with a short hint instead.
constexpr uint32_t kCommitSleepNs = 256u;

__device__ __forceinline__ bool wait_bar(const Params& p, uint64_t* bar, uint32_t parity, const volatile uint32_t* armed,
                                         uint32_t seq, uint32_t site, int lane, uint32_t sleep_ns = kSleepNs) {
    const bool ready = (armed == nullptr || *armed == seq) && mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ready)) return true;
    return wait_bar_slow(p, bar, parity, armed, seq, site, lane, sleep_ns);
}

__device__ __forceinline__ bool wait_fill(const Params& p, const Ring& r, uint32_t seq, int lane) {
    const uint32_t s = seq % r.S;
    return wait_bar(p, r.full + s, (seq / r.S) & 1u, r.armed + s, seq, 2, lane);
}

__device__ __forceinline__ void release_fill(const Ring& r, uint32_t seq, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(r.empty + seq % r.S);
}

// A compute warp waits until the Tensor Memory slot of fill seq holds it (the
// slot's fill number first: a warp may look several laps ahead of the mover).
__device__ __forceinline__ bool wait_tile(const Params& p, const Tmem& tm, uint32_t seq, int lane) {
    const uint32_t k = seq % tm.n;
    if (!wait_bar(p, tm.full + k, (seq / tm.n) & 1u, tm.armed + k, seq, 6, lane)) return false;
    tmem_fence_after();
    return true;
}

// After the warp's reads of the slot have completed (tmem_wait_ld).
__device__ __forceinline__ void release_tile(const Tmem& tm, uint32_t seq, int lane) {
    tmem_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tm.empty + seq % tm.n);
}

// Barrier of the 8 compute warps (an mbarrier of count 8; bounded, abort-aware,
// so a warp that left on an error cannot leave the others waiting forever).
// `uses` counts this warp's passes; all compute warps pass it in the same jobs.
// The wait is a short spin on the non-blocking probe: the warps arrive within a
// few hundred cycles of each other, and a sleeping waiter would add its wake-up
// latency to every pass.
__device__ __noinline__ bool compute_barrier_wait(const Params& p, uint64_t* cbar, uint32_t uses, uint32_t parity,
                                                  int lane) {
    uint64_t t0 = 0;
    for (uint32_t it = 0; !__all_sync(0xffffffffu, mbar_test_wait(cbar, parity)); ++it) {
        if ((it & 1023u) == 1023u) {
            int bad = 0;
            if (lane == 0) {
                if (t0 == 0) t0 = global_timer_ns();
                if (aborted(p)) bad = 1;
                else if (global_timer_ns() - t0 > p.timeout_ns) {
                    record_error(p, MK_ERR_TIMEOUT, uses, 0xfffffff5u, 0, parity, 5);
                    bad = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) return false;
        }
    }
    return true;
}

__device__ __forceinline__ bool compute_barrier(const Params& p, uint64_t* cbar, uint32_t& uses, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    const uint32_t parity = uses & 1u;
    ++uses;
    if (__all_sync(0xffffffffu, mbar_test_wait(cbar, parity))) return true;
    return compute_barrier_wait(p, cbar, uses, parity, lane);
}

// ------------------------------------------------------------------ activation warp

// The down-projection's chunk-c target (chunks may have different job counts).
__device__ __forceinline__ uint32_t down_chunk_target(const mk_instr& in, int c) {
    return c == 0 ? in.wait_n : c == 1 ? (in.aux0 & 0xffffu) : c == 2 ? (in.aux0 >> 16) : in.aux1;
}

// Element e of an XSmem<KC> vector stored at `v`.
__device__ __forceinline__ void xs_store(float* v, int KC, int e, float x) {
    const int g8 = e >> 3, i = e & 7;
    float* arr = (i < 4) ? v : v + KC * 128;
    arr[g8 * 4 + (i & 3)] = x;
}

// Per-job timestamps (see TraceWord), in the traced build only.
#if MK_TRACE
__device__ __forceinline__ void trace(const Params& p, uint32_t job, int word, uint64_t v) {
    if (p.trace != nullptr && job < (uint32_t)p.trace_jobs)
        p.trace[((size_t)blockIdx.x * p.trace_jobs + job) * kTraceWords + word] = v;
}
__device__ __forceinline__ void trace(const Params& p, uint32_t job, int word) {
    trace(p, job, word, global_timer_ns());
}
#else
__device__ __forceinline__ void trace(const Params&, uint32_t, int, uint64_t) {}
__device__ __forceinline__ void trace(const Params&, uint32_t, int) {}
#endif


// Pause between polls of tagged words that have not arrived yet, bounded by
// the wait budget and the abort flag (lane 0 decides for the warp).
__device__ __forceinline__ bool tag_backoff(const Params& p, uint32_t it, uint64_t& t0, uint32_t where,
                                            int lane) {
    __nanosleep(64);
    if ((it & 15u) != 15u) return true;
    int bad = 0;
    if (lane == 0) {
        if (t0 == 0) t0 = global_timer_ns();
        if (aborted(p)) bad = 1;
        else if (global_timer_ns() - t0 > p.timeout_ns) {
            record_error(p, MK_ERR_TIMEOUT, where, 0xfffffff6u, 0, 0, 7);
            bad = 1;
        }
    }
    return __shfl_sync(0xffffffffu, bad, 0) == 0;
}

// A job's input vector from the tagged activations, by all compute warps (the
// thread's pairs, all loads in flight at once, retried until every tag is the
// expected one); RMSNorm with the bf16 norm weights w when w is given. Ends
// with a compute barrier. Out of line: one copy for every job that needs it.
template <bool MMAOP = false>
__device__ __noinline__ bool block_input_tagged(const Params& p, const uint64_t* src, uint32_t tag, const uint16_t* w, int n,
                                   float* xs, float* red, int t, int warp, int lane, uint64_t* cbar,
                                   uint32_t& cuses, int orow = 0) {
    const int np = n / 2;
    uint32_t wv[kMaxPairs];
    float v0[kMaxPairs], v1[kMaxPairs];
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int j = i * kNT + t;
        wv[i] = (w != nullptr && j < np) ? ld_cg_u32(w + 2 * j) : 0u;
    }
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint64_t a[kMaxPairs], b[kMaxPairs];
#pragma unroll
        for (int i = 0; i < kMaxPairs; ++i) {
            const int j = i * kNT + t;
            a[i] = b[i] = 0ull;
            if (j < np) ld_tagged2(src + 2 * j, a[i], b[i]);
        }
        bool ok = true;
#pragma unroll
        for (int i = 0; i < kMaxPairs; ++i) {
            const int j = i * kNT + t;
            v0[i] = tag_val(a[i]);
            v1[i] = tag_val(b[i]);
            if (j < np) ok = ok & tag_ok(a[i], tag) & tag_ok(b[i], tag);
        }
        if (__all_sync(0xffffffffu, ok)) break;
        if (!tag_backoff(p, it, t0, 1, lane)) return false;
    }
    auto bar = [&]() { return compute_barrier(p, cbar, cuses, lane); };
    return block_store_input<MMAOP>(v0, v1, wv, w != nullptr, p.eps, n, xs, red, t, warp, lane, bar, orow);
}

// Batch > 1: the input vectors of two sequences at once (xs0 / operand row orow,
// xs1 / row orow + 1), all their loads in flight together and one barrier for both
// norms, so a job's inputs take half the rounds. Each vector's arithmetic is
// block_input_tagged's exactly (the same pairs per thread, sums in the same order).
// PP: pairs per thread of one vector (n / 2 / threads, rounded up).
template <int PP, bool MMAOP>
__device__ __noinline__ bool block_input_tagged2(const Params& p, const uint64_t* src0, const uint64_t* src1,
                                                 uint32_t tag, const uint16_t* w, int n, float* xs0, float* xs1,
                                                 float* red, int t, int warp, int lane, uint64_t* cbar,
                                                 uint32_t& cuses, int orow) {
    static_assert(2 * kConsumerWarps <= 32, "two vectors' warp sums fit the reduction words");
    const int np = n / 2;
    uint32_t wv[PP];
#pragma unroll
    for (int i = 0; i < PP; ++i) {
        const int j = i * kNT + t;
        wv[i] = (w != nullptr && j < np) ? ld_cg_u32(w + 2 * j) : 0u;
    }
    float v0[2][PP], v1[2][PP];
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint64_t a[2][PP], b[2][PP];
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int i = 0; i < PP; ++i) {
                const int j = i * kNT + t;
                a[k][i] = b[k][i] = 0ull;
                if (j < np) ld_tagged2((k ? src1 : src0) + 2 * j, a[k][i], b[k][i]);
            }
        bool ok = true;
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int i = 0; i < PP; ++i) {
                const int j = i * kNT + t;
                v0[k][i] = tag_val(a[k][i]);
                v1[k][i] = tag_val(b[k][i]);
                if (j < np) ok = ok & tag_ok(a[k][i], tag) & tag_ok(b[k][i], tag);
            }
        if (__all_sync(0xffffffffu, ok)) break;
        if (!tag_backoff(p, it, t0, 1, lane)) return false;
    }
    float r[2] = {1.f, 1.f};
    if (w != nullptr) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < PP; ++i)
                if (i * kNT + t < np) {
                    ss = fmaf(v0[k][i], v0[k][i], ss);
                    ss = fmaf(v1[k][i], v1[k][i], ss);
                }
            ss = warp_sum(ss);
            if (lane == 0) red[k * kConsumerWarps + warp] = ss;
        }
        if (!compute_barrier(p, cbar, cuses, lane)) return false;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            float tot = 0.f;
#pragma unroll
            for (int ww = 0; ww < kConsumerWarps; ++ww) tot += red[k * kConsumerWarps + ww];
            r[k] = 1.0f / sqrtf(tot / (float)n + p.eps);
        }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int i = 0; i < PP; ++i) {
            const int j = i * kNT + t;
            if (j < np) {
                float x0 = v0[k][i], x1 = v1[k][i];
                if (w != nullptr) {
                    x0 = __fmul_rn(__fmul_rn(x0, r[k]), bf_lo(wv[i]));
                    x1 = __fmul_rn(__fmul_rn(x1, r[k]), bf_hi(wv[i]));
                }
                if constexpr (MMAOP) mma_opnd_store(xs0, orow + k, 2 * j, x0, x1);
                else *reinterpret_cast<float2*>((k ? xs1 : xs0) + xs_index(n, 2 * j)) = make_float2(x0, x1);
            }
        }
    return compute_barrier(p, cbar, cuses, lane);
}

// `rows` (<= kMaxResidRows) consecutive tagged words into dst, by the threads
// t < rows (whole warps; the others return at once). No barrier.
__device__ bool rows_tagged(const Params& p, const uint64_t* src, uint32_t tag, int rows, float* dst, int t,
                            int lane) {
    if (t >= ((rows + 31) & ~31)) return true;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const uint64_t w = t < rows ? ld_tagged(src + t) : 0ull;
        if (__all_sync(0xffffffffu, t >= rows || tag_ok(w, tag))) {
            if (t < rows) dst[t] = tag_val(w);
            return true;
        }
        if (!tag_backoff(p, it, t0, 3, lane)) return false;
    }
}

// Where a job's residual rows sit in its slot (per sequence, kMaxResidRows).
__device__ __forceinline__ float* slot_resid(const Params& p, float* sv, int b) {
    return sv + (size_t)p.xs_aux_floats + (size_t)p.B * (p.d + 4) + (size_t)b * kMaxResidRows;
}

// The input of a matvec job, built by the compute warps (they poll the tagged
// words themselves): RMSNorm of x (tagged) or of the embedding row (QKV of
// layer 0) for QKV, gate/up and the LM head; the attention output and the
// residual rows (x before the O-projection, or the embedding row) for the
// O-projection. (The down-projection's inputs: down_input_batch / prep_job.) On the
// tensor-core path (MMA) every sequence's vector goes into the slot's MMA
// operand, row b (mma_opnd_store).
template <bool BATCHED, bool MMA = false, int PPH = 1, int PPQ = 1>
__device__ bool job_input(const Params& p, const mk_instr& in, int c, float* sv, float* red, int warp, int lane,
                          uint64_t* cbar, uint32_t& cuses, uint32_t epoch) {
    const int t = warp * 32 + lane, l = in.layer;
    auto bar = [&]() { return compute_barrier(p, cbar, cuses, lane); };
    const int B = BATCHED ? p.B : 1;
    // at batch > 1 two sequences at a time (block_input_tagged2) where the input is tagged
    const bool pairs = BATCHED && !(in.op == MK_OP_QKV && l == 0);
    for (int b = 0; b < B;) {
        const bool two = pairs && b + 1 < B;
        float* xs = MMA ? sv : sv + (size_t)b * p.xs_vec_floats;
        float* xs1 = MMA ? sv : sv + (size_t)(b + 1) * p.xs_vec_floats;
        switch (in.op) {
            case MK_OP_QKV:
            case MK_OP_GATEUP:
            case MK_OP_LMHEAD: {
                const size_t nrm = in.op == MK_OP_QKV ? (size_t)(2 * l) : in.op == MK_OP_GATEUP
                                                                     ? (size_t)(2 * l + 1)
                                                                     : (size_t)(2 * p.L);
                const uint16_t* w = norm_ptr(p, p.off_norms + nrm * p.H * 2);
                if (in.op == MK_OP_QKV && l == 0) {
                    if (!block_input_plain<MMA>(nullptr, embed_row(p, b), w, p.eps, p.H, xs, red, t, warp, lane, bar,
                                                b))
                        return false;
                } else {
                    // x after the previous layer's MLP (QKV, LM head) or after this layer's attention
                    const uint32_t tag = in.op == MK_OP_GATEUP
                                             ? act_tag(epoch, l, kTagXAttn)
                                             : act_tag(epoch, in.op == MK_OP_QKV ? l - 1 : l, kTagXMlp);
                    const uint64_t* src = p.x_t + (size_t)b * p.H;
                    if (BATCHED && two) {
                        if (!block_input_tagged2<PPH, MMA>(p, src, src + p.H, tag, w, p.H, xs, xs1, red, t, warp,
                                                           lane, cbar, cuses, b))
                            return false;
                    } else if (!block_input_tagged<MMA>(p, src, tag, w, p.H, xs, red, t, warp, lane, cbar, cuses,
                                                        b)) {
                        return false;
                    }
                }
                break;
            }
            case MK_OP_OPROJ: {
                const int rows = (int)in.count * 4;
                for (int k = 0; k < (two ? 2 : 1); ++k) {
                    float* xr = slot_resid(p, sv, b + k);
                    if (l == 0) {
                        if (t < rows) xr[t] = bf2f(embed_row(p, b + k)[(size_t)in.first * 4 + t]);
                    } else if (!rows_tagged(p, p.x_t + (size_t)(b + k) * p.H + (size_t)in.first * 4,
                                            act_tag(epoch, l - 1, kTagXMlp), rows, xr, t, lane)) {
                        return false;
                    }
                }
                const uint64_t* src = p.attn_t + (size_t)b * p.Q;
                const uint32_t tag = act_tag(epoch, l, kTagAttn);
                if (BATCHED && two) {
                    if (!block_input_tagged2<PPQ, MMA>(p, src, src + p.Q, tag, nullptr, p.Q, xs, xs1, red, t, warp,
                                                       lane, cbar, cuses, b))
                        return false;
                } else if (!block_input_tagged<MMA>(p, src, tag, nullptr, p.Q, xs, red, t, warp, lane, cbar, cuses,
                                                    b)) {
                    return false;
                }
                break;
            }
        }
        b += two ? 2 : 1;
    }
    return true;
}

// A down-projection chunk's inputs, by all compute warps: h chunk c of every
// sequence, two at a time, and, with the last chunk, the residual rows (x after
// attention). At batch 1 the stage and activation warps stage chunks c <
// kDownStaged ahead instead (one warp moves one sequence's early chunk in time;
// eight sequences' it does not, nor the chunks that complete only as gate/up ends).
template <bool MMA = false, int PPF = 1>
__device__ __forceinline__ bool down_input_batch(const Params& p, const mk_instr& in, int c, float* sv, float* red,
                                              int warp, int lane, uint64_t* cbar, uint32_t& cuses,
                                              uint32_t epoch) {
    const int t = warp * 32 + lane, l = in.layer;
    const uint32_t tag = act_tag(epoch, l, kTagH);
    for (int b = 0; b < p.B;) {
        const bool two = b + 1 < p.B;
        for (int k = 0; k < (two ? 2 : 1); ++k)
            if (c == 3 && !rows_tagged(p, p.x_t + (size_t)(b + k) * p.H + (size_t)in.first * 4,
                                       act_tag(epoch, l, kTagXAttn), (int)in.count * 4, slot_resid(p, sv, b + k), t,
                                       lane))
                return false;
        const uint64_t* src = p.h_t + (size_t)b * p.F + (size_t)c * (p.F / 4);
        float* xs = MMA ? sv : sv + (size_t)b * p.xs_vec_floats;
        if (two) {
            if (!block_input_tagged2<PPF, MMA>(p, src, src + p.F, tag, nullptr, p.F / 4, xs,
                                               MMA ? sv : sv + (size_t)(b + 1) * p.xs_vec_floats, red, t, warp, lane,
                                               cbar, cuses, b))
                return false;
        } else if (!block_input_tagged<MMA>(p, src, tag, nullptr, p.F / 4, xs, red, t, warp, lane, cbar, cuses, b)) {
            return false;
        }
        b += two ? 2 : 1;
    }
    return true;
}

// An attention item's inputs, by the compute warps: q of the group's heads
// (fp32) and the step's new key and value (bf16) into the slot. Ends with a
// compute barrier.
template <int HD>
__device__ bool attn_input(const Params& p, const mk_instr& in, uint8_t* slot, int warp, int lane, uint64_t* cbar,
                           uint32_t& cuses, uint32_t epoch) {
    const int t = warp * 32 + lane;
    const uint32_t tag = act_tag(epoch, in.layer, kTagQKV);
    const int nq = p.group * HD;
    const uint64_t* qsrc = p.q_t + (size_t)in.batch * p.Q + (size_t)in.group * nq;
    const uint64_t* kvsrc = p.kv_t + (size_t)(in.batch * p.nkv + in.group) * 2 * HD;
    float* qdst = reinterpret_cast<float*>(slot);
    uint16_t* kv = reinterpret_cast<uint16_t*>(slot + (size_t)nq * 4);
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        bool ok = true;
        for (int e = t; e < nq + 2 * HD; e += kNT) {
            const uint64_t w = ld_tagged(e < nq ? qsrc + e : kvsrc + (e - nq));
            ok = ok & tag_ok(w, tag);
            if (e < nq) qdst[e] = tag_val(w);
            else kv[e - nq] = f2bf(tag_val(w));  // exact: the values are bf16
        }
        if (__all_sync(0xffffffffu, ok)) break;
        if (!tag_backoff(p, it, t0, 5, lane)) return false;
    }
    return compute_barrier(p, cbar, cuses, lane);
}

// Waits (lane 0 polls, the warp follows) until the tagged word at `w` carries
// `tag`: a cheap sign that a vector's producers have written it, before the
// warp reads the whole vector (whose every tag is still checked).
__device__ __forceinline__ bool poll_tagged(const Params& p, const uint64_t* w, uint32_t tag, uint32_t where,
                                            int lane) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const int ok = lane == 0 ? (int)tag_ok(ld_tagged(w), tag) : 1;
        if (__shfl_sync(0xffffffffu, ok, 0)) return true;
        if (!tag_backoff(p, it, t0, where, lane)) return false;
    }
}

// A tagged vector of n elements into the XSmem vector at dst, by one warp,
// sixteen pairs per lane in flight; retried until every tag is current.
__device__ bool warp_load_tagged(const Params& p, const uint64_t* src, uint32_t tag, int n, float* dst,
                                 uint32_t where, int lane) {
    const int np = n / 2;
    constexpr int D = 16;
    if (!poll_tagged(p, src + n - 1, tag, where, lane)) return false;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        bool ok = true;
        for (int j0 = 0; j0 < np; j0 += 32 * D) {
            uint64_t a[D], b[D];
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int j = j0 + i * 32 + lane;
                a[i] = b[i] = 0ull;
                if (j < np) ld_tagged2(src + 2 * j, a[i], b[i]);
            }
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int j = j0 + i * 32 + lane;
                if (j < np) {
                    ok = ok & tag_ok(a[i], tag) & tag_ok(b[i], tag);
                    *reinterpret_cast<float2*>(dst + xs_index(n, 2 * j)) = make_float2(tag_val(a[i]), tag_val(b[i]));
                }
            }
        }
        if (__all_sync(0xffffffffu, ok)) return true;
        if (!tag_backoff(p, it, t0, where, lane)) return false;
    }
}

// The activation warp's part of a job: for QKV jobs, stage the RoPE row of each
// sequence's position (constant during the step) in the slot. It waits on no
// dependency: the compute warps poll the tagged inputs themselves, which saves
// the round trip of a counter read on every hop.
template <int HD, bool BATCHED>
__device__ bool prep_job(const Params& p, const mk_instr* ins, int c, uint8_t* slot, int lane, uint32_t epoch,
                         uint32_t job) {
    const mk_instr& in = ins[0];
    float* sv = reinterpret_cast<float*>(slot);
    if (lane == 0) trace(p, job, kTrCtrDone);
    if (!BATCHED && in.op == MK_OP_DOWN && c < kDownStaged) {
        // down chunk c: h chunk c (gate/up runs chunk-major, so chunks complete one
        // after another while gate/up still streams) and, with the last chunk, the
        // residual rows (x after attention), staged ahead of the compute warps
        for (int b = 0; b < (BATCHED ? p.B : 1); ++b) {
            if (!warp_load_tagged(p, p.h_t + (size_t)b * p.F + (size_t)c * (p.F / 4), act_tag(epoch, in.layer, kTagH),
                                  p.F / 4, sv + (size_t)b * p.xs_vec_floats, 8, lane))
                return false;
            if (kDownStaged > 3 && c == 3) {
                const int rows = (int)in.count * 4;
                const uint64_t* xs = p.x_t + (size_t)b * p.H + (size_t)in.first * 4;
                const uint32_t tag = act_tag(epoch, in.layer, kTagXAttn);
                float* xr = slot_resid(p, sv, b);
                for (int r0 = 0; r0 < rows; r0 += 32) {
                    const int r = r0 + lane;
                    uint64_t t0 = 0;
                    for (uint32_t it = 0;; ++it) {
                        const uint64_t w = r < rows ? ld_tagged(xs + r) : 0ull;
                        if (__all_sync(0xffffffffu, r >= rows || tag_ok(w, tag))) {
                            if (r < rows) xr[r] = tag_val(w);
                            break;
                        }
                        if (!tag_backoff(p, it, t0, 4, lane)) return false;
                    }
                }
            }
        }
    }
    if (in.op == MK_OP_QKV) {
        float* aux = sv + (size_t)p.xs_aux_floats;
        for (int b = 0; b < (BATCHED ? p.B : 1); ++b) {
            const int pos = g_pos[b];
            float* row = aux + (size_t)b * (HD + 4);
            for (int i = lane; i < HD / 2; i += 32) {
                row[i] = p.rope_cos[(size_t)pos * (HD / 2) + i];
                row[HD / 2 + i] = p.rope_sin[(size_t)pos * (HD / 2) + i];
            }
            if (lane == 0) reinterpret_cast<int*>(row)[HD] = pos;
        }
    }
    return true;
}

// The preparer of `job`: -1 is the activation warp, h >= 0 stage warp h (at batch
// 1, the down-projection chunk-h jobs, h < kStageWarps and h < kDownStaged).
template <bool BATCHED>
__device__ __forceinline__ int preparer(uint32_t op, int c) {
    return (!BATCHED && op == MK_OP_DOWN && c < kStageWarps && c < kDownStaged) ? c : -1;
}

// The activation warp (role -1) or stage warp h (role h) walks the SM's jobs and
// prepares its own: it waits for the job's slot (prepared for job j - NS, then
// released by the compute warps), stages what the job needs ahead (prep_job),
// records the job in the slot and arrives on the slot's full barrier.
template <int KH, int KO, int KF, int HD, bool BATCHED>
__device__ void activation_warp(const Params& p, const Slots& sl, int i0, int i1, int lane, uint32_t epoch,
                                int role) {
    uint32_t j = 0;
    for (int i = i0; i < i1;) {
        const mk_instr* ins = p.instrs + i;
        const uint32_t op = ins[0].op;
        const int njobs = (op == MK_OP_DOWN) ? 4 : 1;
        for (int c = 0; c < njobs; ++c, ++j) {
            if (preparer<BATCHED>(op, c) != role) continue;
            const uint32_t s = j % sl.NS, use = j / sl.NS;
            if (lane == 0) {
                trace(p, j, kTrSlotWait);
                trace(p, j, kTrMeta, op | ((uint32_t)ins[0].layer << 8) | ((uint32_t)c << 24));
            }
            if (use > 0 && !wait_bar(p, sl.empty + s, (use - 1) & 1u, sl.job + s, j - sl.NS, 3, lane)) return;
            if (lane == 0) trace(p, j, kTrCtrWait);
            if (!prep_job<HD, BATCHED>(p, ins, c, sl.slot(j), lane, epoch, j)) return;
            __syncwarp();
            if (lane == 0) {
                trace(p, j, kTrReady);
                sl.job[s] = j;             // published by the release of the arrive below
                mbar_arrive(sl.full + s);  // release: the slot's contents
            }
        }
        ++i;
    }
}

// ------------------------------------------------------------------ compute warps

// Greedy selection: (value, index) pairs, the larger value first, the lower index
// among equal values; a NaN value is never chosen (an all-NaN row gives index 0).
struct Best {
    float v;
    uint32_t i;
};
__device__ __forceinline__ Best best_none() { return {__int_as_float(0x7fffffff), 0xffffffffu}; }
__device__ __forceinline__ bool best_before(float v, uint32_t i, const Best& b) {
    if (v != v) return false;          // NaN: never
    if (b.v != b.v) return true;       // anything beats nothing
    return v > b.v || (v == b.v && i < b.i);
}
__device__ __forceinline__ void best_take(Best& b, float v, uint32_t i) {
    if (best_before(v, i, b)) b = {v, i};
}
// Over the lanes whose bits under `mask` differ (an xor butterfly).
__device__ __forceinline__ Best best_reduce(Best b, uint32_t masks_from, uint32_t masks_to) {
    for (uint32_t m = masks_from; m >= masks_to && m > 0; m >>= 1) {
        const float v = __shfl_xor_sync(0xffffffffu, b.v, (int)m);
        const uint32_t i = __shfl_xor_sync(0xffffffffu, b.i, (int)m);
        best_take(b, v, i);
    }
    return b;
}

// One 4-row tile, read from the warp's Tensor Memory slot at `ta`, against an
// input vector in shared memory: the same lane mapping and order of arithmetic as
// dot4 (lane ln holds the 16-byte pieces (row r, kc*32 + ln); the mover stored
// row r's piece kc at columns kc*16 + 4r .. +3), so the totals equal dot4's bit
// for bit. A single copy of the code per input width, shared by every op (the
// kernel's instruction footprint is what each SM re-fetches for every layer).
template <int KC>
__device__ __noinline__ float4 tile_dot(uint32_t ta, const float* v, int lane) {
    static_assert(KC % 2 == 0, "pieces are read in pairs");
    const XSmem<KC> x{reinterpret_cast<float4*>(const_cast<float*>(v)),
                      reinterpret_cast<float4*>(const_cast<float*>(v)) + KC * 32};
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto use = [&](const uint32_t (&r)[16], int kc) {
        float e[8];
        x.get(kc, lane, e);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
            fma8(acc[rr], make_uint4(r[4 * rr], r[4 * rr + 1], r[4 * rr + 2], r[4 * rr + 3]), e);
    };
    // the next piece's load is in flight while the current one is used
    uint32_t a[16], b[16];
    tmem_ld16(ta, a);
    tmem_wait_ld(a);
#pragma unroll 1
    for (int kc = 0; kc < KC; kc += 2) {
        tmem_ld16(ta + (uint32_t)(kc + 1) * 16u, b);
        use(a, kc);
        tmem_wait_ld(b);
        if (kc + 2 < KC) tmem_ld16(ta + (uint32_t)(kc + 2) * 16u, a);
        use(b, kc + 1);
        if (kc + 2 < KC) tmem_wait_ld(a);
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) acc[rr] = warp_sum(acc[rr]);
    return make_float4(acc[0], acc[1], acc[2], acc[3]);
}

// Batch 1 (batch > 1 runs compute_tiles_pair). Tile t of the job is the SM's fill
// seq = in.seq + t; compute warp seq mod 8 takes it (its Tensor Memory quarter,
// seq mod 4, is the one the mover stored it in).
template <int KC, int HD>
__device__ bool compute_tiles(const Params& p, const Tmem& tm, const mk_instr& in,
                              const float* sv, int warp, int lane, uint32_t job, uint32_t epoch, uint2* selp) {
    // a dropped instruction (the failure-detection hook) computes but publishes nothing
    const bool pub = in.signal_ctr != MK_NO_COUNTER;
    const bool sel = in.op == MK_OP_LMHEAD && p.next_tokens != nullptr;
    Best best = best_none();  // the lane's LM-head row (lanes 0..3)
    int k = 0;  // trace: warp 0's first tiles (fill wait start, fill ready, dot done)
    auto stamp = [&](int w) {
        if (warp == 0 && lane == 0 && w < 8) trace(p, job, kTrSub0 + w);
    };
    for (uint32_t t = (uint32_t)(warp - (int)in.seq) & 7u; t < in.count; t += kConsumerWarps) {
        const uint32_t seq = in.seq + t;
        if (k < 2) stamp(3 * k);
        if (!wait_tile(p, tm, seq, lane)) return false;
        if (t == 0 && lane == 0) trace(p, job, kTrFill);
        if (k < 2) stamp(3 * k + 1);
        {
            constexpr int b = 0;  // batch 1: every lane holds the 4 totals
            const int el = lane;
            float acc[4];
            {
                const float4 a4 = tile_dot<KC>(tm.addr(seq, warp), sv, lane);
                acc[0] = a4.x; acc[1] = a4.y; acc[2] = a4.z; acc[3] = a4.w;
            }
            release_tile(tm, seq, lane);
            if (k < 2) stamp(3 * k + 2);
            const uint32_t tl = in.op == MK_OP_GATEUP ? gu_tile(p, in, t) : in.first + t;
            switch (in.op) {
                case MK_OP_QKV: {
                    const float* row = sv + (size_t)p.xs_aux_floats + (size_t)b * (HD + 4);
                    const RopeRow rr{row, row + HD / 2, reinterpret_cast<const int*>(row)[HD]};
                    if (pub) qkv_epilogue<HD, true>(p, in.layer, b, tl, acc, el, rr, act_tag(epoch, in.layer, kTagQKV));
                    break;
                }
                case MK_OP_GATEUP:
                    if (pub) gateup_epilogue<true>(p, b, tl, acc, el, act_tag(epoch, in.layer, kTagH));
                    break;
                case MK_OP_OPROJ:
                    // x = x_in + W_o attn for the tile's rows; x_in waits in the slot
                    if (pub && el < 4) {
                        const float xin = slot_resid(p, const_cast<float*>(sv), b)[(tl - in.first) * 4 + el];
                        st_tagged(p.x_t + (size_t)b * p.H + tl * 4 + el, __fadd_rn(xin, pick4(acc, el)),
                                  act_tag(epoch, in.layer, kTagXAttn));
                    }
                    break;
                default:
                    logits_epilogue(p, b, tl, acc, el);
                    if (sel && el < 4) best_take(best, pick4(acc, el), tl * 4 + el);
                    break;
            }
        }
        if (k == 1) stamp(6);
        ++k;
    }
    if (sel) {  // the warp's best of the job, for the job's last warp (publish_best)
        best = best_reduce(best, 16, 1);
        if (lane == 0) selp[warp * kMaxBatch] = make_uint2(__float_as_uint(best.v), best.i);
    }
    return true;
}

// Batch > 1: two compute warps share each tile by sequences -- the warps w with
// w mod 4 = seq mod 4 (the tile's Tensor Memory quarter), sequences [b0, b0 + nb)
// with b0 = (w / 4) * ceil(B / 2) -- so a tile is held for half the batched
// arithmetic. Each (sequence, row) total is dot4's for that sequence, bit for bit
// (the arithmetic of dot4_batch4 on the pieces read from Tensor Memory); both
// warps release the slot (its empty barrier counts two arrivals).
template <int KC>
__device__ __noinline__ float tile_dot_batch4(uint32_t ta, const float* xs, uint32_t vec_floats, int B4,
                                              int lane) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
#pragma unroll 1
    for (int kc = 0; kc < KC; ++kc) {
        uint32_t r[16];
        tmem_ld16(ta + (uint32_t)kc * 16u, r);
        tmem_wait_ld(r);
        float w[4][8];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
            unpack8(make_uint4(r[4 * rr], r[4 * rr + 1], r[4 * rr + 2], r[4 * rr + 3]), w[rr]);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (b < B4) {
                const float4* x = reinterpret_cast<const float4*>(xs + (size_t)b * vec_floats);
                const float4 lo = x[kc * 32 + lane], hi = x[KC * 32 + kc * 32 + lane];
                const float e[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[b * 4 + rr] = fmaf(w[rr][i], e[i], v[b * 4 + rr]);
            }
        }
    }
    return reduce_batch4(v, lane);
}

struct PairSeqs {
    int b0, nb;  // this warp's sequences
    __device__ PairSeqs(int B, int warp) {
        const int per = (B + 1) / 2;
        b0 = (warp / kPairGroups) * per;
        nb = min(per, B - b0);
    }
};

template <int KC, int HD>
__device__ bool compute_tiles_pair(const Params& p, const Tmem& tm, const mk_instr& in, const float* sv, int warp,
                                   int lane, uint32_t job, uint32_t epoch, uint2* selp) {
    const bool pub = in.signal_ctr != MK_NO_COUNTER;
    const bool sel = in.op == MK_OP_LMHEAD && p.next_tokens != nullptr;
    Best best = best_none();  // the lane's row of its sequence (active lanes)
    const PairSeqs ps(p.B, warp);
    const int sl = lane >> 3;                         // the sequence (of this warp's) the lane holds
    const bool act = sl < ps.nb && (lane & 1) == 0;   // lanes l and l ^ 1 hold the same total
    const int b = ps.b0 + (sl < ps.nb ? sl : 0);
    const int el = act ? ((lane >> 1) & 3) : 32;      // acts as lane `el` of a 4-row epilogue
    for (uint32_t t = (uint32_t)(warp - (int)in.seq) & 3u; t < in.count; t += kPairGroups) {
        const uint32_t seq = in.seq + t;
        if (!wait_tile(p, tm, seq, lane)) return false;
        if (t == 0 && lane == 0 && warp < kPairGroups) trace(p, job, kTrFill);
        const float tb = tile_dot_batch4<KC>(tm.addr(seq, warp), sv + (size_t)ps.b0 * p.xs_vec_floats,
                                             p.xs_vec_floats, ps.nb, lane);
        release_tile(tm, seq, lane);
        float acc[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[r] = __shfl_sync(0xffffffffu, tb, (lane & ~7) + 2 * r);
        const uint32_t tl = in.op == MK_OP_GATEUP ? gu_tile(p, in, t) : in.first + t;
        switch (in.op) {
            case MK_OP_QKV: {
                const float* row = sv + (size_t)p.xs_aux_floats + (size_t)b * (HD + 4);
                const RopeRow rr{row, row + HD / 2, reinterpret_cast<const int*>(row)[HD]};
                if (pub) qkv_epilogue<HD, true>(p, in.layer, b, tl, acc, el, rr, act_tag(epoch, in.layer, kTagQKV));
                break;
            }
            case MK_OP_GATEUP:
                if (pub) gateup_epilogue<true>(p, b, tl, acc, el, act_tag(epoch, in.layer, kTagH));
                break;
            case MK_OP_OPROJ:
                if (pub && el < 4) {
                    const float xin = slot_resid(p, const_cast<float*>(sv), b)[(tl - in.first) * 4 + el];
                    st_tagged(p.x_t + (size_t)b * p.H + tl * 4 + el, __fadd_rn(xin, pick4(acc, el)),
                              act_tag(epoch, in.layer, kTagXAttn));
                }
                break;
            default:
                logits_epilogue(p, b, tl, acc, el);
                if (sel && el < 4) best_take(best, pick4(acc, el), tl * 4 + el);
                break;
        }
    }
    if (sel) {
        // lanes 8 s' .. 8 s' + 7 hold the warp's sequence b0 + s' (the active ones)
        best = best_reduce(best, 4, 1);
        for (int s2 = 0; s2 < 4; ++s2) {
            const float v = __shfl_sync(0xffffffffu, best.v, 8 * s2);
            const uint32_t i = __shfl_sync(0xffffffffu, best.i, 8 * s2);
            if (lane == 0 && s2 < ps.nb) selp[warp * kMaxBatch + ps.b0 + s2] = make_uint2(__float_as_uint(v), i);
        }
    }
    return true;
}

// Every chunk job at batch > 1 starts with the compute warps' input barrier
// (down_input_batch), so a running sum that another warp added to in the previous
// chunk is complete before this chunk adds to it.
template <int KF>
__device__ bool compute_down_pair(const Params& p, const Tmem& tm, const mk_instr& in, int c, const float* sv,
                                  float* tot, int warp, int lane, uint32_t job, uint32_t epoch) {
    const PairSeqs ps(p.B, warp);
    const int sl = lane >> 3;
    const bool act = sl < ps.nb && (lane & 1) == 0;
    const int b = ps.b0 + (sl < ps.nb ? sl : 0);
    const int row = (lane >> 1) & 3;
    const uint32_t base = in.seq + (uint32_t)c * in.count;
    for (uint32_t r = (uint32_t)(warp - (int)base) & 3u; r < in.count; r += kPairGroups) {
        const uint32_t seq = base + r;
        if (!wait_tile(p, tm, seq, lane)) return false;
        if (r == 0 && lane == 0 && warp < kPairGroups) trace(p, job, kTrFill);
        const float y = tile_dot_batch4<KF>(tm.addr(seq, warp), sv + (size_t)ps.b0 * p.xs_vec_floats,
                                            p.xs_vec_floats, ps.nb, lane);
        release_tile(tm, seq, lane);
        if (act) {
            float* t = tot + ((size_t)r * p.B + b) * 4 + row;
            *t = (c == 0) ? y : *t + y;
            if (c == 3 && in.signal_ctr != MK_NO_COUNTER) {  // x = x_in + W_d h; x_in waits in the slot
                const float xin = slot_resid(p, const_cast<float*>(sv), b)[r * 4 + row];
                st_tagged(p.x_t + (size_t)b * p.H + (in.first + r) * 4 + row, __fadd_rn(xin, *t),
                          act_tag(epoch, in.layer, kTagXMlp));
            }
        }
    }
    return true;
}

// Down-projection at batch 1 (batch > 1 runs compute_down_pair), chunk c: row
// block r's tile of chunk c is fill seq = in.seq + c * count + r, taken by compute
// warp seq mod 8 -- a different warp in each chunk -- so chunks 0..2 store their
// totals y_c apart, and chunk 3, whose inputs the compute warps load behind a
// barrier of all of them (kDownStaged <= 3), adds ((y_0 + y_1) + y_2) + y_3 and the
// residual.
static_assert(kDownStaged <= 3, "chunk 3 must start with the compute warps' input barrier");
template <int KF>
__device__ bool compute_down(const Params& p, const Tmem& tm, const mk_instr& in, int c,
                             const float* sv, float* tot, int warp, int lane, uint32_t job, uint32_t epoch) {
    const uint32_t base = in.seq + (uint32_t)c * in.count;
    for (uint32_t r = (uint32_t)(warp - (int)base) & 7u; r < in.count; r += kConsumerWarps) {
        const uint32_t seq = base + r;
        if (!wait_tile(p, tm, seq, lane)) return false;
        if (r == 0 && lane == 0) trace(p, job, kTrFill);
        float y;
        {
            const float4 a4 = tile_dot<KF>(tm.addr(seq, warp), sv, lane);
            const float acc[4] = {a4.x, a4.y, a4.z, a4.w};
            y = pick4(acc, lane & 3);
        }
        release_tile(tm, seq, lane);
        if (lane < 4) {
            float* yc = tot + r * 4 + lane;  // y_c at yc[c * kMaxDownRows * 4]
            if (c < 3) {
                yc[c * kMaxDownRows * 4] = y;
            } else if (in.signal_ctr != MK_NO_COUNTER) {  // x = x_in + W_d h; x_in waits in the slot
                const float sum = ((yc[0] + yc[kMaxDownRows * 4]) + yc[2 * kMaxDownRows * 4]) + y;
                const float xin = slot_resid(p, const_cast<float*>(sv), 0)[r * 4 + lane];
                st_tagged(p.x_t + (in.first + r) * 4 + lane, __fadd_rn(xin, sum), act_tag(epoch, in.layer, kTagXMlp));
            }
        }
    }
    return true;
}

// Tensor-core path: the outputs of one segment row of sequence b, as the fused
// epilogues of the CUDA-core path take them (a tile's 4 rows in acc, this lane
// its row `el`). Returns the row's value (the LM head's greedy selection).
template <int HD>
__device__ __noinline__ void mma_epilogue(const Params& p, const mk_instr& in, int b, uint32_t tl,
                                          const float (&acc)[4], int el, const float* sv, uint32_t epoch) {
    const bool pub = in.signal_ctr != MK_NO_COUNTER;  // a dropped instruction publishes nothing
    switch (in.op) {
        case MK_OP_QKV: {
            const float* row = sv + (size_t)p.xs_aux_floats + (size_t)b * (HD + 4);
            const RopeRow rr{row, row + HD / 2, reinterpret_cast<const int*>(row)[HD]};
            if (pub) qkv_epilogue<HD, true>(p, in.layer, b, tl, acc, el, rr, act_tag(epoch, in.layer, kTagQKV));
            break;
        }
        case MK_OP_GATEUP:
            if (pub) gateup_epilogue<true>(p, b, tl, acc, el, act_tag(epoch, in.layer, kTagH));
            break;
        case MK_OP_OPROJ:
        case MK_OP_DOWN:
            // x = x_in + W y for the instruction's rows; x_in waits in the slot
            if (pub) {
                const float xin = slot_resid(p, const_cast<float*>(sv), b)[(tl - in.first) * 4 + el];
                st_tagged(p.x_t + (size_t)b * p.H + tl * 4 + el, __fadd_rn(xin, pick4(acc, el)),
                          act_tag(epoch, in.layer, in.op == MK_OP_OPROJ ? kTagXAttn : kTagXMlp));
            }
            break;
        default:
            logits_epilogue(p, b, tl, acc, el);
            break;
    }
}

// Tensor-core path, a matvec job of the compute warps once its operand is in the
// slot: for each of the instruction's segments (the down-projection's only after
// its last chunk), wait for the accumulator, read this warp's lane quarter (rows
// 32 q .. 32 q + 31 of the segment, q = warp mod 4) and release it, then run the
// epilogues of the warp's sequences (the first half of the batch for warps 0-3,
// the second for 4-7, as on the CUDA-core path): y = high + low column. `sg` is
// the SM's number of the instruction's first segment (the issuer counts alike).
template <int HD>
__device__ bool mma_job(const Params& p, const MmaBars& mb, uint32_t tbase, const mk_instr& in, int c, uint32_t sg,
                        const float* sv, int warp, int lane, uint32_t job, uint32_t epoch, uint2* selp) {
    const MmaGeom g = mma_geom(in.op, in.count, in.aux0, p.H, p.Q, p.F, p.stage_bytes);
    if (c + 1 < (int)g.jobs) return true;  // down chunks 0-2 only accumulate
    const bool sel = in.op == MK_OP_LMHEAD && p.next_tokens != nullptr;
    const uint32_t q = (uint32_t)warp & 3u;
    const PairSeqs ps(p.B, warp);
    const int el = lane & 3;
    Best best[4] = {best_none(), best_none(), best_none(), best_none()};
    for (uint32_t rg = 0; rg < g.nrange; ++rg) {
        for (uint32_t sgi = 0; sgi < g.segs; ++sgi) {
            const uint32_t sn = sg + rg * g.segs + sgi, a = sn % (uint32_t)kMaxAcc;
            if (!wait_bar(p, mb.afull + a, (sn / (uint32_t)kMaxAcc) & 1u, nullptr, sn, 13, lane, kCommitSleepNs))
                return false;
            if (rg == 0 && sgi == 0 && warp == 0 && lane == 0) trace(p, job, kTrFill);
            tmem_fence_after();
            // the warp's sequences' high and low sums over the partial sums, in order
            float shi[4] = {0.f, 0.f, 0.f, 0.f}, slo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (uint32_t u = 0; u < kSubAcc; ++u) {
                uint32_t d[16];
                tmem_ld16(tbase + ((32u * q) << 16) + (a * kSubAcc + u) * kAccCols, d);
                tmem_wait_ld(d);
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    float hi = 0.f, lo = 0.f;
#pragma unroll
                    for (int b = 0; b < kMaxBatch; ++b)
                        if (b == ps.b0 + bb) {
                            hi = __uint_as_float(d[b]);
                            lo = __uint_as_float(d[kMaxBatch + b]);
                        }
                    shi[bb] = __fadd_rn(shi[bb], hi);
                    slo[bb] = __fadd_rn(slo[bb], lo);
                }
            }
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(mb.aempty + a);
            const uint32_t left = g.rows - sgi * kMmaRows;
            const uint32_t rows = left < kMmaRows ? left : kMmaRows;
            const uint32_t m = 32u * q + (uint32_t)lane;  // the lane's row of the segment
            const uint32_t first = in.op == MK_OP_GATEUP ? rg * (uint32_t)(p.F / 8) + in.first : in.first;
            const uint32_t tl = first + sgi * (kMmaRows / 4) + (m >> 2);
            // the warp's sequences' totals, high + low (register indices fixed at compile time)
            float y[4];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) y[bb] = __fadd_rn(shi[bb], slo[bb]);
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                if (bb < ps.nb) {  // warp-uniform
                    float acc[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[r] = __shfl_sync(0xffffffffu, y[bb], (lane & ~3) | r);
                    if (m < rows) {
                        mma_epilogue<HD>(p, in, ps.b0 + bb, tl, acc, el, sv, epoch);
                        if (sel) best_take(best[bb], y[bb], tl * 4 + el);
                    }
                }
            }
        }
    }
    if (sel) {  // the warp's best row of each of its sequences (publish_best)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
            const Best r = best_reduce(best[bb], 16, 1);
            if (lane == 0 && bb < ps.nb)
                selp[warp * kMaxBatch + ps.b0 + bb] = make_uint2(__float_as_uint(r.v), r.i);
        }
    }
    return true;
}

// One attention item as one job of all compute warps (see attn_item_block). Every
// fill of the item must have landed first: each warp reads all of them. With a
// single partition per (sequence, group) the item writes o / l for its heads;
// otherwise it stores its partial, counts its heads on the pair's arrival
// counter, and the item that completes the count merges the pair's partitions
// in partition order. Either way the group's heads are signalled on the
// attention counter once their output is written.
template <int HD, bool BATCHED>
__device__ bool compute_attn_job(const Params& p, const Ring& ring, const mk_instr& a, uint8_t* slot, int warp,
                                 int lane, uint64_t* cbar, uint32_t& cuses, uint32_t job, uint32_t epoch) {
    const int G = p.group, b = a.batch, g = a.group;
    // the item's scratch follows its q and new key/value in the job's slot
    float* sc = reinterpret_cast<float*>(slot + attn_item_bytes(G, HD));
    const int pos = g_pos[b];
    for (uint32_t f = 0; f < a.nfill; ++f)
        if (!wait_fill(p, ring, a.seq + f, lane)) return false;
    if (warp == 0 && lane == 0) trace(p, job, kTrFill);
    const float* qs = reinterpret_cast<const float*>(slot);
    const uint16_t* knew = reinterpret_cast<const uint16_t*>(slot + (size_t)G * HD * 4);
    const int jn = pos - (int)a.first;
    const AttnRows<HD> R{ring.base, ring.stage_bytes, (int)ring.S, (int)(a.seq % ring.S), p.keys_per_stage,
                         min((int)a.count, jn + 1), (jn >= 0 && jn < (int)a.count) ? jn : -1, knew, knew + HD};
    auto bar = [&]() { return compute_barrier(p, cbar, cuses, lane); };
    // trace: warp 0 at the end of each phase and after each barrier
    auto mark = [&](int k) {
        if (warp == 0 && lane == 0) trace(p, job, kTrSub0 + k);
    };
    const int t = warp * 32 + lane;
    uint32_t* sig = p.counters + (size_t)a.signal_ctr * kCounterStride;
    {
        // one instance of the item's code for both outputs (the kernel's code size
        // is what every SM re-fetches): o / l with one partition, else the partial
        uint64_t* out = p.attn_t + (size_t)b * p.Q + (size_t)g * G * HD;
        const uint32_t tag = act_tag(epoch, a.layer, kTagAttn);
        const bool pub = a.signal_ctr != MK_NO_COUNTER;  // a dropped item publishes nothing
        const bool single = p.n_parts == 1;
        const int part = (int)(a.first / (uint32_t)p.part_keys);
        if (!attn_item_block<HD>(R, qs, G, sc, warp, lane, bar, mark, [&](int h, int d, float o, float m, float l) {
                if (single) {
                    if (pub) st_tagged(out + h * HD + d, __fdiv_rn(o, l), tag);
                    return;
                }
                const size_t hp = ((size_t)b * p.nq + (size_t)(g * G + h)) * p.n_parts + part;
                p.part_o[hp * HD + d] = o;
                if (d == 0) {
                    p.part_ml[hp * 2] = m;
                    p.part_ml[hp * 2 + 1] = l;
                }
            }))
            return false;
    }
    // every warp has passed the barrier after its last read of the fills
    if (warp == kConsumerWarps - 1 && lane == 0)
        for (uint32_t f = 0; f < a.nfill; ++f)  // (the tensor-core path counts one per issuer)
            for (int r = 0; r < (p.mma ? kIssuers : 1); ++r) mbar_arrive(ring.empty + (a.seq + f) % ring.S);
    if (!bar()) return false;  // every output of the item is stored
    if (p.n_parts == 1) {
        if (t == 0 && a.signal_ctr != MK_NO_COUNTER) red_relaxed_add(sig, (uint32_t)G);
        mark(6);
        return true;
    }
    uint32_t* flag = reinterpret_cast<uint32_t*>(sc + AttnScratch<HD>::kFlag);
    if (t == 0) {
        uint32_t last = 0;
        if (a.signal_ctr != MK_NO_COUNTER) {  // a dropped item (failure injection) never arrives
            const uint32_t target = (epoch + 1u) * (uint32_t)(p.n_parts * G);
            const uint32_t old = atom_acq_rel_add(p.counters + (size_t)a.aux0 * kCounterStride, (uint32_t)G);
            last = old + (uint32_t)G == target;
        }
        *flag = last;
    }
    if (!bar()) return false;
    if (*reinterpret_cast<volatile uint32_t*>(flag) == 0u) return true;
    if (warp < G) {
        uint64_t* out = p.attn_t + (size_t)b * p.Q;
        const uint32_t tag = act_tag(epoch, a.layer, kTagAttn);
        const int head = g * G + warp;
        attn_merge_heads<HD, 1>(p, b, head, 1, head + 1, lane, [&](int e, float x) { st_tagged(out + e, x, tag); });
    }
    if (!bar()) return false;
    if (t == 0) red_relaxed_add(sig, (uint32_t)G);
    return true;
}

// The LM-head job's last compute warp (all lanes): the SM's best row of each
// sequence from its warps' bests (at batch > 1 a sequence's tiles were shared by
// the warps w with w / 4 = its half), stored at the job's ordinal in.aux0; then
// one acquire-release increment of the LM-head counter. The job that completes the
// step's count (epoch + 1) * n_lm_jobs reduces every job's best, one lane per
// job, and writes each sequence's next token, its next position, and the token
// into the generated list. Every step writes every entry before it counts, so no
// stale entry is read.
__device__ __noinline__ void publish_best(const Params& p, const mk_instr& in, const uint2* selp, int lane,
                                          uint32_t epoch) {
    const int per = (p.B + 1) / 2;
    if (lane < p.B) {
        const int b = lane;
        const int w0 = p.B > 1 ? (b < per ? 0 : kPairGroups) : 0;
        const int w1 = p.B > 1 ? w0 + kPairGroups : kConsumerWarps;
        Best bb = best_none();
        for (int w = w0; w < w1; ++w) {
            const uint2 e = selp[w * kMaxBatch + b];
            best_take(bb, __uint_as_float(e.x), e.y);
        }
        __stcg(reinterpret_cast<uint2*>(p.sel_best) + (size_t)b * p.n_lm_jobs + in.aux0,
               make_uint2(__float_as_uint(bb.v), bb.i));
    }
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        const uint32_t old = atom_acq_rel_add(p.counters + (size_t)in.signal_ctr * kCounterStride, 1u);
        last = old + 1u == (epoch + 1u) * (uint32_t)p.n_lm_jobs;
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    for (int b = 0; b < p.B; ++b) {
        Best bb = best_none();
        for (int k = lane; k < p.n_lm_jobs; k += 32) {
            const uint2 e = __ldcg(reinterpret_cast<const uint2*>(p.sel_best) + (size_t)b * p.n_lm_jobs + k);
            best_take(bb, __uint_as_float(e.x), e.y);
        }
        bb = best_reduce(bb, 16, 1);
        if (lane == 0) {
            const int32_t tok = bb.i == 0xffffffffu ? 0 : (int32_t)bb.i;  // all NaN: 0
            p.next_tokens[b] = tok;
            if (p.next_positions) p.next_positions[b] = g_pos[b] + 1;
            if (p.gen_tokens) p.gen_tokens[b] = tok;
        }
    }
}

template <int KH, int KO, int KF, int HD, bool BATCHED, bool MMA>
__device__ void compute_warp(const Params& p, const Ring& ring, const Tmem& tm, const Slots& sl, const MmaBars& mb,
                             float* tot, float* red, uint64_t* cbar, uint2* selp, int i0, int i1, int warp,
                             int lane, uint32_t epoch) {
    uint32_t j = 0, cuses = 0;
    uint32_t sg = 0;  // tensor-core path: the SM's segments so far (mma_issuer counts alike)
    uint32_t ph = 0;  // tensor-core path: bit s, the phase of slot s's operand / MMA-done barriers
    for (int i = i0; i < i1;) {
        const mk_instr in = p.instrs[i];
        const int njobs = (in.op == MK_OP_DOWN) ? 4 : 1;
        for (int c = 0; c < njobs; ++c, ++j) {
            const uint32_t s = j % sl.NS;
            if (!wait_bar(p, sl.full + s, (j / sl.NS) & 1u, nullptr, j, 4, lane)) return;
            if (warp == 0 && lane == 0) trace(p, j, kTrStart);
            float* sv = reinterpret_cast<float*>(sl.slot(j));
            // inputs: the attention item's q/k/v and every matvec input but the
            // early down-projection chunks at batch 1 (staged by the activation
            // warp) are loaded here
            bool ok = in.op == MK_OP_ATTN   ? attn_input<HD>(p, in, sl.slot(j), warp, lane, cbar, cuses, epoch)
                      : in.op == MK_OP_DOWN ? ((!BATCHED && c < kDownStaged) ||
                                                     down_input_batch<MMA, (KF + 1) / 2>(p, in, c, sv, red, warp,
                                                                                         lane, cbar, cuses, epoch))
                                            : job_input<BATCHED, MMA, (KH + 1) / 2, (KO + 1) / 2>(
                                                  p, in, c, sv, red, warp, lane, cbar, cuses, epoch);
            if (!ok) return;
            if (warp == 0 && lane == 0) trace(p, j, kTrSub0 + 7);
            // one call site per routine: the kernel's code is what every SM re-fetches
            // from L2 as it moves between ops, so nothing is inlined twice
            if (in.op == MK_OP_ATTN) {
                ok = compute_attn_job<HD, BATCHED>(p, ring, in, sl.slot(j), warp, lane, cbar, cuses, j,
                                                   epoch);
            } else if constexpr (MMA) {
                // the operand is complete (the input's last barrier): hand it to the
                // tensor cores (async proxy), then read the accumulators; the slot is
                // free once the job's MMAs are done
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(mb.opnd + s);
                ok = mma_job<HD>(p, mb, tm.base, in, c, sg, sv, warp, lane, j, epoch, selp) &&
                     wait_bar(p, mb.mdone + s, (ph >> s) & 1u, nullptr, j, 12, lane, kCommitSleepNs);
                ph ^= 1u << s;
            } else if (in.op == MK_OP_DOWN) {
                if constexpr (BATCHED) ok = compute_down_pair<KF>(p, tm, in, c, sv, tot, warp, lane, j, epoch);
                else ok = compute_down<KF>(p, tm, in, c, sv, tot, warp, lane, j, epoch);
            } else if (KO != KH && in.op == MK_OP_OPROJ) {
                if constexpr (KO != KH) {
                    if constexpr (BATCHED) ok = compute_tiles_pair<KO, HD>(p, tm, in, sv, warp, lane, j, epoch, selp);
                    else ok = compute_tiles<KO, HD>(p, tm, in, sv, warp, lane, j, epoch, selp);
                }
            } else {  // QKV, gate/up, the LM head (and the O-projection when its width is the hidden size)
                if constexpr (BATCHED) ok = compute_tiles_pair<KH, HD>(p, tm, in, sv, warp, lane, j, epoch, selp);
                else ok = compute_tiles<KH, HD>(p, tm, in, sv, warp, lane, j, epoch, selp);
            }
            if (!ok) return;
            // job done for this warp; the last of the 8 counts the job's completion
            // (acquire-release at CTA scope on the shared count, then a relaxed
            // increment: consumers read the tagged outputs, not the counter)
            __syncwarp();
            int last_warp = 0;
            if (lane == 0) {
                const uint32_t old = atom_shared_acq_rel_add(sl.done + s, 1u);
                last_warp = old == kConsumerWarps - 1;
            }
            last_warp = __shfl_sync(0xffffffffu, last_warp, 0);
            // greedy selection: the LM-head job's last warp publishes the SM's best;
            // the SM that completes the step's count picks the next tokens
            if (last_warp && in.op == MK_OP_LMHEAD && p.next_tokens != nullptr && in.signal_ctr != MK_NO_COUNTER)
                publish_best(p, in, selp, lane, epoch);
            if (lane == 0) {
                if (last_warp) {
                    sl.done[s] = 0;
                    trace(p, j, kTrDone);
                    // attention items signal their heads themselves (compute_attn_job)
                    const bool last_chunk = (in.op != MK_OP_DOWN || c == 3) && in.op != MK_OP_ATTN &&
                                            !(in.op == MK_OP_LMHEAD && p.next_tokens != nullptr);
                    if (last_chunk && in.signal_ctr != MK_NO_COUNTER) {
                        // QKV / gate-up: one increment on each KV group / MLP chunk counter
                        // the job's tiles touched
                        const uint32_t span =
                            (in.op == MK_OP_QKV || in.op == MK_OP_GATEUP) && in.aux1 > 1 ? in.aux1 : 1u;
                        for (uint32_t k = 0; k < span; ++k)
                            red_relaxed_add(p.counters + (size_t)(in.signal_ctr + k) * kCounterStride, 1u);
                    }
                }
                mbar_arrive(sl.empty + s);
            }
        }
        if constexpr (MMA) {
            if (in.op != MK_OP_ATTN) {
                const MmaGeom g = mma_geom(in.op, in.count, in.aux0, p.H, p.Q, p.F, p.stage_bytes);
                sg += g.nrange * g.segs;
            }
        }
        ++i;
    }
}

// ------------------------------------------------------------------ the loader and the mover warps

// Global source of ring fill t of instruction `in`: one range (weights), or two
// ranges of `bytes` each for attention (the cached keys and values < pos).
struct FillSrc {
    const uint8_t* a;
    const uint8_t* b;
    uint32_t bytes;
};

__device__ __forceinline__ FillSrc fill_source(const Params& p, const mk_instr& in, uint32_t t) {
    const size_t lbase = p.off_layer0 + (size_t)in.layer * p.layer_stride;
    switch (in.op) {
        case MK_OP_ATTN: {
            const int pos = g_pos[in.batch];
            const int ka = (int)in.first + (int)t * p.keys_per_stage;
            const int kend = min(ka + p.keys_per_stage, (int)(in.first + in.count));
            const int np = max(0, min(kend, pos) - ka);  // cached keys (< pos)
            const size_t off = kv_off(p, in.layer, in.batch, in.group, ka);
            return {reinterpret_cast<const uint8_t*>(p.kc + off),
                    reinterpret_cast<const uint8_t*>(p.vc + off), (uint32_t)np * p.d * 2};
        }
        case MK_OP_QKV:
            return {p.packed + lbase + p.rel_qkv + (size_t)(in.first + t) * p.tile_h, nullptr, p.tile_h};
        case MK_OP_OPROJ:
            return {p.packed + lbase + p.rel_o + (size_t)(in.first + t) * p.tile_o, nullptr, p.tile_o};
        case MK_OP_GATEUP:
            return {p.packed + lbase + p.rel_gu + (size_t)gu_tile(p, in, t) * p.tile_h, nullptr, p.tile_h};
        case MK_OP_DOWN: {
            const uint32_t c = t / in.count, r = t % in.count;  // chunk-major
            return {p.packed + lbase + p.rel_down + ((size_t)(in.first + r) * 4 + c) * p.tile_f, nullptr,
                    p.tile_f};
        }
        default:  // LM head: rows of the (tied) embedding table
            return {p.packed + (size_t)(in.first + t) * p.tile_h, nullptr, p.tile_h};
    }
}

// Position of fill `seq` in the SM's list: the instruction holding it (an SM's
// fills are numbered consecutively, instruction by instruction).
struct FillCur {
    int i;
    uint32_t seq;
};

__device__ __forceinline__ void fill_seek(const Params& p, FillCur& c, int i1) {
    while (c.i < i1 && c.seq >= p.instrs[c.i].seq + p.instrs[c.i].nfill) ++c.i;
}

// Tensor-core path: the segments of a matvec instruction in fill order -- job
// (the down-projection's chunk), range, segment -- each with its rows, its first
// row in the matrix's packed row order, its boxes per fill, fills and tensor map.
// The loader and the issuer walk the same sequence.
struct MmaSeg {
    uint32_t rows, row0, nb, fps;
    const void* map;
};
__device__ __forceinline__ MmaSeg mma_seg(const Params& p, const mk_instr& in, const MmaGeom& g, uint32_t c,
                                          uint32_t rg, uint32_t sgi) {
    MmaSeg m;
    const bool last = sgi + 1 == g.segs;
    m.rows = last ? g.rows_l : kMmaRows;
    m.nb = last ? g.nb_l : g.nb_f;
    m.fps = last ? g.fps_l : g.fps_f;
    const uint32_t hk = m.rows / 8u - 1u;
    int idx;
    switch (in.op) {
        case MK_OP_QKV: idx = kTmQKV * kTmPerKind; m.row0 = 4u * in.first; break;
        case MK_OP_OPROJ: idx = kTmO * kTmPerKind; m.row0 = 4u * in.first; break;
        case MK_OP_GATEUP: idx = kTmGU * kTmPerKind; m.row0 = 4u * (rg * (uint32_t)(p.F / 8) + in.first); break;
        case MK_OP_DOWN: idx = kTmDown0 + (int)c * 8; m.row0 = 4u * in.first; break;
        default: idx = kTmLM * kTmPerKind; m.row0 = 4u * in.first; break;
    }
    m.row0 += sgi * kMmaRows;
    m.map = static_cast<const uint8_t*>(p.tmaps) + (size_t)(idx + (int)hk) * kTmBytes;
    return m;
}

// One fill of a segment: a single TMA copy of nb 64-column boxes from K-box kb0
// (past the end of K the boxes read zeros, never used), landing as nb boxes of
// the segment's rows side by side at dst.
__device__ __forceinline__ void issue_mma_fill(const Params& p, const mk_instr& in, const MmaSeg& m, uint32_t kb0,
                                               uint8_t* dst, uint64_t* bar, uint64_t pol) {
    mbar_arrive_expect_tx(bar, m.nb * m.rows * 128u);
    if (in.op == MK_OP_DOWN)  // {column, row in block, row block, K-box, layer}
        tma_load_5d(dst, m.map, 0, 0, (int)(m.row0 / 4u), (int)kb0, (int)in.layer, bar, pol);
    else if (in.op == MK_OP_LMHEAD)
        tma_load_3d(dst, m.map, 0, (int)m.row0, (int)kb0, bar, pol);
    else
        tma_load_4d(dst, m.map, 0, (int)m.row0, (int)kb0, (int)in.layer, bar, pol);
}

// One thread (the loader warp's lane 0) streams the SM's fills into the ring, in
// list order: weight tiles and the cached KV of attention items, all final at
// launch. It never waits on a dependency counter, only for a stage to be free
// again: moved to Tensor Memory by a mover warp (weights), read by the tensor
// cores (weights, tensor-core path) or read by its attention item (KV). So the
// next instructions' weights arrive while the step still waits for their
// activations. It issues nothing else, so a freed stage is refilled at once.
template <bool MMA>
__device__ void loader(const Params& p, const Ring& ring, int i0, int i1) {
    const uint64_t pol = l2_evict_first_policy();
    uint32_t issued = 0;  // fills issued so far (they are numbered 0, 1, 2, ...)
    uint32_t job0 = 0;    // the instruction's first job (trace)
    // Waits until stage seq mod S is free for fill seq and arms it (bounded).
    auto acquire = [&](uint32_t seq) {
        const uint32_t s = seq % ring.S, use = seq / ring.S;
        if (use > 0) {
            uint64_t t0 = 0;
            for (uint32_t it = 0; !mbar_wait_sleep(ring.empty + s, (use - 1) & 1u, MMA ? kCommitSleepNs : kSleepNs);
                 ++it) {
                if ((it & 15u) == 15u) {
                    if (t0 == 0) t0 = global_timer_ns();
                    if (aborted(p)) return false;
                    if (global_timer_ns() - t0 > p.timeout_ns) {
                        record_error(p, MK_ERR_TIMEOUT, seq, 0xfffffffdu, 0, use, 3);
                        return false;
                    }
                }
            }
        }
        ring.armed[s] = seq;  // published by the release of the fill's arrive
        return true;
    };
    for (int i = i0; i < i1; job0 += p.instrs[i].op == MK_OP_DOWN ? 4u : 1u, ++i) {
        const mk_instr in = p.instrs[i];
        if (MMA && in.op != MK_OP_ATTN) {
            const MmaGeom g = mma_geom(in.op, in.count, in.aux0, p.H, p.Q, p.F, p.stage_bytes);
            uint32_t seq = in.seq;
            for (uint32_t c = 0; c < g.jobs; ++c) {
                if (MK_TRACE) trace(p, job0 + c, kTrSub0 + 0);  // the job's first fill is issued next
                for (uint32_t rg = 0; rg < g.nrange; ++rg)
                    for (uint32_t sgi = 0; sgi < g.segs; ++sgi) {
                        const MmaSeg m = mma_seg(p, in, g, c, rg, sgi);
                        for (uint32_t kf = 0; kf < m.fps; ++kf, ++seq) {
                            if (!acquire(seq)) goto drain;
                            const uint32_t s = seq % ring.S;
                            issue_mma_fill(p, in, m, kf * m.nb, ring.base + (size_t)s * ring.stage_bytes,
                                           ring.full + s, pol);
                            issued = seq + 1;
                        }
                    }
                if (MK_TRACE) trace(p, job0 + c, kTrSub0 + 1);  // the job's last fill is issued
            }
            continue;
        }
        for (uint32_t t = 0; t < in.nfill; ++t) {
            const uint32_t seq = in.seq + t;
            if (!acquire(seq)) goto drain;
            const uint32_t s = seq % ring.S;
            uint8_t* dst = ring.base + (size_t)s * ring.stage_bytes;
            uint64_t* bar = ring.full + s;
            const FillSrc f = fill_source(p, in, t);
            if (f.b != nullptr) {  // attention: keys, then values half a stage later
                mbar_arrive_expect_tx(bar, 2 * f.bytes);
                if (f.bytes) {
                    bulk_g2s(dst, f.a, f.bytes, bar, pol);
                    bulk_g2s(dst + (size_t)p.keys_per_stage * p.d * 2, f.b, f.bytes, bar, pol);
                }
            } else {
                mbar_arrive_expect_tx(bar, f.bytes);
                bulk_g2s(dst, f.a, f.bytes, bar, pol);
            }
            issued = seq + 1;
        }
    }
drain:
    // Every copy issued must land before the CTA may exit: wait for the last
    // fill of each stage used (earlier fills of a stage completed before it
    // could be refilled).
    for (uint32_t s = 0; s < ring.S && s < issued; ++s) {
        const uint32_t last_seq = s + ((issued - 1 - s) / ring.S) * ring.S;
        const uint32_t par = (last_seq / ring.S) & 1u;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_wait_sleep(ring.full + s, par, 20000u)) {
            if (global_timer_ns() - t0 > p.timeout_ns) {
                record_error(p, MK_ERR_TIMEOUT, last_seq, 0xfffffffcu, 0, par, 4);
                break;
            }
        }
    }
}

// Tensor-core path: issuer u (warps 8-11, the mover warps' places; converged, lane
// 0 issues) walks the SM's jobs in order. For a matvec job it waits until the
// compute warps have written the job's operand into its slot, then for each fill:
// that its segment's accumulator has been read out since its previous use (first
// fill of the segment), that the fill has landed; it issues its K step of every
// box of the fill (K = 16 at byte 32 u of the box's 128-byte rows) into partial
// sum u of the segment's accumulator (the segment's first overwrites it) and
// commits them to the stage's empty barrier, which completes once all four
// issuers' MMAs have read the stage. A segment's last fill also commits to its
// accumulator's full barrier, a job's last to the slot's MMA-done barrier (each
// counts the four issuers). Before it returns, on every way out, it waits until
// the MMAs of all four have completed (the CTA then releases Tensor Memory). Every
// wait is bounded.
__device__ void mma_issuer(const Params& p, const Ring& ring, const MmaBars& mb, const Slots& sl, uint32_t tbase,
                           int i0, int i1, int u, int lane) {
    uint32_t j = 0, sg = 0;
    uint32_t ph = 0;  // bit s: phase of slot s's operand / MMA-done barriers (matvec jobs only)
    for (int i = i0; i < i1; ++i) {
        const mk_instr in = p.instrs[i];
        if (in.op == MK_OP_ATTN) {
            ++j;
            continue;
        }
        const MmaGeom g = mma_geom(in.op, in.count, in.aux0, p.H, p.Q, p.F, p.stage_bytes);
        uint32_t seq = in.seq;
        for (uint32_t c = 0; c < g.jobs; ++c, ++j) {
            const uint32_t s = j % sl.NS;
            if (!wait_bar(p, mb.opnd + s, (ph >> s) & 1u, nullptr, j, 10, lane)) goto out;
            ph ^= 1u << s;
            if (lane == 0 && u == 0) trace(p, j, kTrSub0 + 2);  // the operand is in the slot
            {
                const uint32_t opnd = smem_addr(sl.slot(j));
                for (uint32_t rg = 0; rg < g.nrange; ++rg)
                    for (uint32_t sgi = 0; sgi < g.segs; ++sgi) {
                        const MmaSeg m = mma_seg(p, in, g, c, rg, sgi);
                        const uint32_t sn = sg + rg * g.segs + sgi;
                        const uint32_t a = sn % (uint32_t)kMaxAcc, use = sn / (uint32_t)kMaxAcc;
                        if (c == 0 && use > 0 && !wait_bar(p, mb.aempty + a, (use - 1u) & 1u, nullptr, sn, 11, lane))
                            goto out;
                        const uint32_t ta = tbase + a * (kAccCols * kSubAcc);
                        for (uint32_t kf = 0; kf < m.fps; ++kf, ++seq) {
                            if (!wait_bar(p, ring.full + seq % ring.S, (seq / ring.S) & 1u, ring.armed + seq % ring.S,
                                          seq, 2, lane, kCommitSleepNs))
                                goto out;
                            tmem_fence_after();
                            if (lane == 0) {
                                const uint32_t b0 = kf * m.nb, nbx = min(m.nb, g.k64 - b0);
                                // descriptors advance by adding to their start-address field
                                // (addresses stay below 256 KB, so the field never carries):
                                // a box further is rows * 128 bytes in the stage and 2048 in
                                // the operand, a K step 32 bytes in both
                                // this issuer's K step of every box: 32 bytes into the box
                                uint64_t da = sw128_desc(smem_addr(ring.stage(seq)) + 32u * (uint32_t)u);
                                uint64_t db = sw128_desc(opnd + b0 * 2048u + 32u * (uint32_t)u);
                                const uint64_t astep = (uint64_t)(m.rows * 128u) >> 4;
                                const uint32_t tu = ta + (uint32_t)u * kAccCols;
                                // K step (b0 + bx) * 4 + u goes to partial sum u; the first box
                                // of the segment's first job starts it
                                uint32_t acc = (c | kf) != 0u;
#pragma unroll 4
                                for (uint32_t bx = 0; bx < nbx; ++bx) {
                                    mma_bf16(tu, da, db, acc);
                                    da += astep;
                                    db += 2048u >> 4;
                                    acc = 1u;
                                }
                                mma_commit(ring.empty + seq % ring.S);
                                if (c + 1 == g.jobs && kf + 1 == m.fps) mma_commit(mb.afull + a);
                            }
                            __syncwarp();
                        }
                    }
            }
            if (lane == 0) {
                mma_commit(mb.mdone + s);
                if (u == 0) trace(p, j, kTrSub0 + 5);  // every MMA of the job issued
            }
            __syncwarp();
        }
        sg += g.nrange * g.segs;
    }
out:
    if (lane == 0) {  // a commit with nothing issued arrives at once
        mma_commit(mb.fin);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_wait_sleep(mb.fin, 0u, kCommitSleepNs)) {
            if (global_timer_ns() - t0 > p.timeout_ns) {
                record_error(p, MK_ERR_TIMEOUT, j, 0xfffffff9u, 0, 0, 14);
                break;
            }
        }
    }
    __syncwarp();
}

// Mover warp q (its lanes converged throughout; its warp index mod 4 is q, the
// Tensor Memory lane quarter it may address) takes the SM's fills seq = q (mod 4)
// in list order. A landed weight tile goes into Tensor Memory slot seq mod n once
// the compute warp has released that slot's previous tile; its ring stage is then
// free for the loader. A cached-KV fill stays in the ring for its attention item
// (which frees the stage); its slot is passed over (marked and released at once).
// The waits block, bounded: the slot's previous tile is an earlier fill and every
// earlier fill has been issued, so the compute warps can reach it; the fill itself
// is issued in order by the loader.
template <bool BATCHED>
__device__ void mover(const Params& p, const Ring& ring, const Tmem& tm, int i0, int i1, int q, int lane) {
    const uint32_t S = ring.S;
    FillCur mov{i0, (uint32_t)q};
    fill_seek(p, mov, i1);
    while (mov.i < i1) {
        const mk_instr& in = p.instrs[mov.i];
        const uint32_t seq = mov.seq, s = seq % S, k = seq % tm.n;
        const bool kv = in.op == MK_OP_ATTN;
        if (seq >= tm.n && !wait_bar(p, tm.empty + k, (seq / tm.n - 1u) & 1u, nullptr, seq, 8, lane)) return;
        if (!kv) {
            if (!wait_bar(p, ring.full + s, (seq / S) & 1u, ring.armed + s, seq, 9, lane)) return;
            tmem_fence_after();
            const uint32_t bytes = in.op == MK_OP_OPROJ ? p.tile_o : in.op == MK_OP_DOWN ? p.tile_f : p.tile_h;
            const int KC = (int)(bytes / 2048u);  // even for every supported width
            const uint4* src = reinterpret_cast<const uint4*>(ring.stage(seq)) + lane;
            const uint32_t ta = tm.addr(seq, q);
#pragma unroll 1
            for (int kc = 0; kc < KC; kc += 2) {
                uint32_t r0[16], r1[16];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const uint4 v0 = lds_v4(src + (rr * KC + kc) * 32);
                    const uint4 v1 = lds_v4(src + (rr * KC + kc + 1) * 32);
                    r0[4 * rr] = v0.x; r0[4 * rr + 1] = v0.y; r0[4 * rr + 2] = v0.z; r0[4 * rr + 3] = v0.w;
                    r1[4 * rr] = v1.x; r1[4 * rr + 1] = v1.y; r1[4 * rr + 2] = v1.z; r1[4 * rr + 3] = v1.w;
                }
                tmem_st16(ta + (uint32_t)kc * 16u, r0);
                tmem_st16(ta + (uint32_t)(kc + 1) * 16u, r1);
            }
            tmem_wait_st();
            tmem_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
            tm.armed[k] = seq;  // published by the release of the arrive below
            mbar_arrive(tm.full + k);
            if (kv) {
                for (int j = 0; j < (BATCHED ? 2 : 1); ++j) mbar_arrive(tm.empty + k);
            } else {
                mbar_arrive(ring.empty + s);  // the stage is free for the next fill
            }
        }
        mov.seq += kMoveWarps;
        fill_seek(p, mov, i1);
    }
}

// ------------------------------------------------------------------ the kernel

template <int KH, int KO, int KF, int HD, bool BATCHED, bool MMA>
__global__ void __launch_bounds__(kThreads, 1) megakernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_epoch, s_skip;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemLayout m = smem_layout(p.n_stages, p.stage_bytes, p.xs_slots, p.xs_slot_bytes, MMA);
    Ring ring;
    ring.base = smem + m.ring;
    ring.full = reinterpret_cast<uint64_t*>(smem + m.full);
    ring.empty = reinterpret_cast<uint64_t*>(smem + m.empty);
    ring.armed = reinterpret_cast<volatile uint32_t*>(smem + m.armed);
    ring.stage_bytes = p.stage_bytes;
    ring.S = (uint32_t)p.n_stages;
    Slots sl;
    sl.base = smem + m.xs;
    sl.full = reinterpret_cast<uint64_t*>(smem + m.xs_full);
    sl.empty = reinterpret_cast<uint64_t*>(smem + m.xs_empty);
    sl.done = reinterpret_cast<uint32_t*>(smem + m.xs_done);
    sl.job = reinterpret_cast<volatile uint32_t*>(smem + m.xs_job);
    sl.bytes = p.xs_slot_bytes;
    sl.NS = (uint32_t)p.xs_slots;
    Tmem tm;
    tm.full = reinterpret_cast<uint64_t*>(smem + m.tfull);
    tm.empty = reinterpret_cast<uint64_t*>(smem + m.tempty);
    tm.armed = reinterpret_cast<volatile uint32_t*>(smem + m.tarmed);
    tm.n = (uint32_t)p.n_tslots;
    tm.cols = p.tslot_cols;
    uint32_t* tbase = reinterpret_cast<uint32_t*>(smem + m.tbase);
    MmaBars mb;
    mb.opnd = reinterpret_cast<uint64_t*>(smem + m.opnd);
    mb.mdone = reinterpret_cast<uint64_t*>(smem + m.mdone);
    mb.afull = reinterpret_cast<uint64_t*>(smem + m.afull);
    mb.aempty = reinterpret_cast<uint64_t*>(smem + m.aempty);
    mb.fin = reinterpret_cast<uint64_t*>(smem + m.fin);

    // All of the SM's Tensor Memory for this CTA (one CTA per SM; the previous
    // step's CTA released it before exiting). Warp 0, converged.
    if (warp == 0) {
        tmem_alloc(tbase, kTmemCols);
        tmem_relinquish();
        tmem_fence_before();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.n_stages; ++s) {
            mbar_init(ring.full + s, 1);
            // released by a mover (weights) or the attention item (KV); on the tensor-core
            // path by each issuer's commit (weights) or kIssuers arrivals of the item (KV)
            mbar_init(ring.empty + s, MMA ? kIssuers : 1);
            ring.armed[s] = 0xffffffffu;
        }
        for (int k = 0; k < p.n_tslots; ++k) {
            mbar_init(tm.full + k, 1);
            mbar_init(tm.empty + k, BATCHED ? 2 : 1);  // batch > 1: two warps share each tile
            tm.armed[k] = 0xffffffffu;
        }
        for (int s = 0; s < p.xs_slots; ++s) {
            mbar_init(sl.full + s, 1);
            mbar_init(sl.empty + s, kConsumerWarps);
            sl.done[s] = 0;
            sl.job[s] = 0xffffffffu;
        }
        mbar_init(reinterpret_cast<uint64_t*>(smem + m.cbar), kConsumerWarps);
        if (MMA) {
            for (int s = 0; s < p.xs_slots; ++s) {
                mbar_init(mb.opnd + s, kConsumerWarps);
                mbar_init(mb.mdone + s, kIssuers);
            }
            for (int a = 0; a < kMaxAcc; ++a) {
                mbar_init(mb.afull + a, kIssuers);
                mbar_init(mb.aempty + a, kConsumerWarps);
            }
            mbar_init(mb.fin, kIssuers);
        }
        fence_mbar_init();
        s_epoch = ld_volatile_u32(&p.ctl->epoch);
        uint32_t skip = ld_volatile_u32(&p.ctl->status) != 0u;
        // the tensor-core path's swizzled operands need 1024-byte-aligned slots and stages
        if (!skip && MMA && ((smem_addr(smem) | smem_addr(smem + m.xs)) & 1023u) != 0u) {
            skip = 1;
            if (blockIdx.x == 0) record_error(p, MK_ERR_UNSUPPORTED, smem_addr(smem), smem_addr(smem + m.xs), 0, 0, 15);
        }
        if (!skip) {
            for (int b = 0; b < p.B; ++b) {
                const int tok = p.tokens[b], pos = p.positions[b];
                g_pos[b] = pos;
                uint32_t code = 0;
                if (tok < 0 || tok >= p.V) code = MK_ERR_BAD_TOKEN;
                else if (pos < 0 || pos >= p.max_seq || pos + 1 > p.max_ctx) code = MK_ERR_BAD_POSITION;
                if (code) {
                    skip = 1;
                    if (blockIdx.x == 0) record_error(p, code, b, (uint32_t)tok, (uint32_t)pos, 0, 5);
                    break;
                }
            }
        }
        s_skip = skip;
    }
    __syncthreads();
    tmem_fence_after();
    tm.base = *reinterpret_cast<volatile uint32_t*>(tbase);

    if (!s_skip) {
        const int i0 = p.sm_off[blockIdx.x], i1 = p.sm_off[blockIdx.x + 1];
        if (warp >= kConsumerWarps && warp < kConsumerWarps + kMoveWarps) {
            if constexpr (MMA) {
                mma_issuer(p, ring, mb, sl, tm.base, i0, i1, warp - kConsumerWarps, lane);
            } else {
                mover<BATCHED>(p, ring, tm, i0, i1, warp & 3, lane);
            }
        } else if (warp == kLoaderWarp) {
            if (lane == 0) loader<MMA>(p, ring, i0, i1);
        } else if (warp == kPrepWarp || warp >= kStageWarp0) {
            // one call site: the stage warps have jobs at batch 1 only
            if (warp == kPrepWarp || !BATCHED)
                activation_warp<KH, KO, KF, HD, BATCHED>(p, sl, i0, i1, lane, s_epoch,
                                                         warp == kPrepWarp ? -1 : warp - kStageWarp0);
        } else {
            compute_warp<KH, KO, KF, HD, BATCHED, MMA>(p, ring, tm, sl, mb, reinterpret_cast<float*>(smem + m.tot),
                                                  reinterpret_cast<float*>(smem + m.red),
                                                  reinterpret_cast<uint64_t*>(smem + m.cbar),
                                                  reinterpret_cast<uint2*>(smem + m.sel), i0, i1, warp, lane,
                                                  s_epoch);
        }
    }
    // every warp's Tensor Memory reads and writes have completed (waited for)
    tmem_fence_before();
    __syncthreads();
    if (warp == 0) {
        tmem_fence_after();
        tmem_dealloc(tm.base, kTmemCols);
    }

    // The last CTA to finish closes the step: it advances the epoch, or, after a
    // failed step, clears the counters and every tagged word (so no stale tag can
    // match the restarted epochs) and restarts the epoch at 0.
    __shared__ uint32_t s_close;  // 0: not last, 1: last, 2: last after a failure
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t old = atom_acq_rel_add(&p.ctl->done, 1u);
        s_close = old == gridDim.x - 1 ? (ld_volatile_u32(&p.ctl->status) != 0u ? 2u : 1u) : 0u;
    }
    __syncthreads();
    if (s_close == 2u) {
        for (size_t i = threadIdx.x; i < p.tagged_words; i += blockDim.x) p.x_t[i] = 0ull;
        for (int c = threadIdx.x; c < p.n_counters; c += blockDim.x) p.counters[(size_t)c * kCounterStride] = 0u;
        __syncthreads();
    }
    if (threadIdx.x == 0 && s_close != 0u) {
        if (s_close == 2u) {
            p.ctl->epoch = 0u;
            p.ctl->abort = 0u;
        } else {
            p.ctl->epoch = s_epoch + 1u;
        }
        p.ctl->done = 0u;
        __threadfence();
    }
}

// ------------------------------------------------------------------ host-side launch

size_t smem_bytes(const Params& p) {
    return smem_layout(p.n_stages, p.stage_bytes, p.xs_slots, p.xs_slot_bytes, p.mma != 0).total;
}

using KernelFn = void (*)(Params);

// One kernel per shape and per batch class: only the batch > 1 kernel carries the
// compute warps' down-chunk loads (at batch 1 they would change the batch-1
// kernel's register allocation and cost it a few microseconds per step).
template <bool BATCHED, bool MMA>
static KernelFn pick_b(int KH, int KO, int KF, int HD) {
    if (KH == 2 && KO == 2 && KF == 2 && HD == 64) return megakernel<2, 2, 2, 64, BATCHED, MMA>;
    if (KH == 8 && KO == 8 && KF == 8 && HD == 64) return megakernel<8, 8, 8, 64, BATCHED, MMA>;
    if (KH == 12 && KO == 12 && KF == 8 && HD == 128) return megakernel<12, 12, 8, 128, BATCHED, MMA>;
    return nullptr;
}

// Batch > 1: the CUDA-core kernel or the tensor-core one (p.mma).
static KernelFn pick(int KH, int KO, int KF, int HD, int B, bool mma) {
    if (B <= 1) return pick_b<false, false>(KH, KO, KF, HD);
    return mma ? pick_b<true, true>(KH, KO, KF, HD) : pick_b<true, false>(KH, KO, KF, HD);
}

static KernelFn pick(const Params& p) { return pick(p.H / 256, p.Q / 256, p.F / 1024, p.d, p.B, p.mma != 0); }

bool supported(int H, int Q, int F, int d) {
    if (H % 256 || Q % 256 || F % 1024) return false;
    return pick(H / 256, Q / 256, F / 1024, d, 1, false) != nullptr;
}

cudaError_t prepare(const Params& p) {
    KernelFn fn = pick(p);
    if (!fn) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(p));
}

cudaError_t occupancy(const Params& p, int* blocks_per_sm) {
    KernelFn fn = pick(p);
    if (!fn) return cudaErrorInvalidValue;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fn, kThreads, smem_bytes(p));
}

cudaError_t launch(const Params& p, cudaStream_t stream) {
    KernelFn fn = pick(p);
    if (!fn) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_sm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes(p);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace plain / traced

#if !MK_TRACE
// The library's entry points: the traced kernels when the schedule records
// timestamps (p.trace set), else the plain ones.
namespace traced {
cudaError_t prepare(const Params& p);
cudaError_t occupancy(const Params& p, int* blocks_per_sm);
cudaError_t launch(const Params& p, cudaStream_t stream);
}  // namespace traced

size_t megakernel_smem_bytes(const Params& p) { return plain::smem_bytes(p); }
bool megakernel_supported(int H, int Q, int F, int d) { return plain::supported(H, Q, F, d); }
cudaError_t megakernel_prepare(const Params& p) { return p.trace ? traced::prepare(p) : plain::prepare(p); }
cudaError_t megakernel_occupancy(const Params& p, int* blocks_per_sm) {
    return p.trace ? traced::occupancy(p, blocks_per_sm) : plain::occupancy(p, blocks_per_sm);
}
cudaError_t megakernel_launch(const Params& p, cudaStream_t stream) {
    return p.trace ? traced::launch(p, stream) : plain::launch(p, stream);
}
#endif

}  // namespace mk
