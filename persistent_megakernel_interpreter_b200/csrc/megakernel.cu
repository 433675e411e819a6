// The persistent decode megakernel: one CTA per SM runs the whole decode step.
//
// Structure (after the megakernel write-ups: "Look Ma, No Bubbles" summaries,
// sections "Fusing Operations with an On-GPU Interpreter", "Efficient Shared
// Memory Management", "Custom Synchronization Mechanism"; and the Cohere decode
// megakernel, sections on the host task list, weight prefetch ahead of
// activation waits, and static per-opcode pipelines instead of paging):
//
//  * The host writes one instruction list per SM. Every CTA walks its list.
//  * Warp 8 (the loader) streams, in list order, every byte the instructions
//    will read from HBM that is already final at launch -- weight tiles and the
//    cached KV slots -- into a ring of shared-memory stages with bulk async
//    copies (cp.async.bulk, completion counted on an mbarrier, L2 evict-first).
//    It never waits on a dependency counter, so weights for the next
//    instructions arrive while the consumers still wait for activations.
//  * Warps 0..7 (consumers) take instructions round-robin. Each waits for its
//    input counter (acquire load, bounded spin), reads its small activation
//    vector from L2, consumes its ring stages, writes its outputs and
//    increments its output counter (release).
//  * Counters only grow: a step waits for (epoch + 1) * n increments, and the
//    last CTA to finish advances the epoch, so no reset kernel is needed.
//  * Every wait is bounded by a time budget; on expiry the step records
//    MK_ERR_TIMEOUT, raises an abort flag that every other wait polls, drains
//    its own copies in flight and returns. No trap, no unbounded spin.
#include <cuda_runtime.h>

#include "mk_device.cuh"

namespace mk {


struct Ring {
    uint8_t* base;
    uint64_t* full;
    uint64_t* empty;
    // Fill number the loader last armed on each stage. Consumer warps take
    // instructions out of order and may look for a fill up to several laps ahead;
    // an mbarrier parity alone only tells phases one lap apart, so a consumer
    // first waits until its stage holds its fill, then waits on the parity.
    volatile uint32_t* armed;
    uint32_t stage_bytes;
    uint32_t S;
    __device__ __forceinline__ uint8_t* stage(uint32_t seq) const {
        return base + (size_t)(seq % S) * stage_bytes;
    }
};

// ------------------------------------------------------------------ errors and waits

__device__ void record_error(const Params& p, uint32_t code, uint32_t a, uint32_t b, uint32_t c,
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

// Lane 0 spins until counter `ctr` reaches `target` (wrap-safe); the result is
// broadcast to the warp. False on abort or timeout.
__device__ bool wait_counter(const Params& p, uint32_t ctr, uint32_t target, uint32_t where,
                             int lane) {
    int ok = 1;
    if (lane == 0) {
        const uint32_t* c = p.counters + (size_t)ctr * kCounterStride;
        uint32_t v = ld_acquire_u32(c);
        if ((int32_t)(v - target) < 0) {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t it = 1;; ++it) {
                v = ld_acquire_u32(c);
                if ((int32_t)(v - target) >= 0) break;
                if ((it & 31u) == 0u) {
                    if (aborted(p)) { ok = 0; break; }
                    if (global_timer_ns() - t0 > p.timeout_ns) {
                        record_error(p, MK_ERR_TIMEOUT, where, ctr, v, target, 1);
                        ok = 0;
                        break;
                    }
                }
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// All lanes wait for ring fill `seq` to land; warp-uniform exit.
__device__ bool wait_full(const Params& p, const Ring& r, uint32_t seq, int lane) {
    const uint32_t s = seq % r.S;
    uint64_t* bar = r.full + s;
    const uint32_t par = (seq / r.S) & 1u;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool done = r.armed[s] == seq && mbar_try_wait(bar, par);
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 15u) == 15u) {
            int bad = 0;
            if (lane == 0) {
                if (t0 == 0) t0 = global_timer_ns();
                if (aborted(p)) bad = 1;
                else if (global_timer_ns() - t0 > p.timeout_ns) {
                    record_error(p, MK_ERR_TIMEOUT, seq, 0xfffffffeu, r.armed[s], par, 2);
                    bad = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) return false;
        }
    }
}

__device__ __forceinline__ void release_stage(const Ring& r, uint32_t seq, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(r.empty + seq % r.S);
}

__device__ __forceinline__ void signal(const Params& p, uint32_t ctr, int lane) {
    __syncwarp();
    if (lane == 0 && ctr != MK_NO_COUNTER) red_release_add(p.counters + (size_t)ctr * kCounterStride, 1u);
}

__device__ __forceinline__ uint32_t target_of(uint32_t epoch, uint32_t n) { return (epoch + 1u) * n; }

// ------------------------------------------------------------------ instruction bodies

template <int OP, int KC, int HD>
__device__ bool exec_tiles(const Params& p, const Ring& ring, const mk_instr& in, int lane,
                           uint64_t pol, uint32_t epoch, float* slot) {
    if (in.wait_ctr != MK_NO_COUNTER &&
        !wait_counter(p, in.wait_ctr, target_of(epoch, in.wait_n), in.seq, lane))
        return false;
    const int l = in.layer;
    XSmem<KC> x{reinterpret_cast<float4*>(slot), reinterpret_cast<float4*>(slot) + KC * 32};
    if (p.B == 1) prep_input<OP, KC>(p, l, 0, x, lane);
    for (uint32_t t = 0; t < in.count; ++t) {
        const uint32_t seq = in.seq + t;
        if (!wait_full(p, ring, seq, lane)) return false;
        const uint8_t* tile = ring.stage(seq);
        for (int b = 0; b < p.B; ++b) {
            if (p.B > 1) prep_input<OP, KC>(p, l, b, x, lane);
            float acc[4];
            dot4<KC, true>(tile, x, acc, lane, pol);
            tile_epilogue<OP, HD>(p, l, b, in.first + t, acc, lane);
        }
        release_stage(ring, seq, lane);
    }
    signal(p, in.signal_ctr, lane);
    return true;
}

// Down-projection: row block(s) over the 4 chunks of h, each chunk waited for
// separately (the per-chunk MLP counters of the 1B megakernel); partial sums
// added in chunk order, then the residual [R6]. With one sequence an
// instruction may hold several row blocks (fills ordered chunk-major); with
// more sequences it holds one. Running sums live in the warp's scratch.
template <int KF>
__device__ bool exec_down(const Params& p, const Ring& ring, const mk_instr& in, int lane,
                          uint64_t pol, uint32_t epoch, float* slot) {
    const int nslot = (p.B > 1) ? p.B : (int)in.count;
    XSmem<KF> x{reinterpret_cast<float4*>(slot), reinterpret_cast<float4*>(slot) + KF * 32};
    float* tot = slot + KF * 256;  // running sums, [nslot][4]
    for (int c = 0; c < 4; ++c) {
        if (!wait_counter(p, in.wait_ctr + c, target_of(epoch, in.wait_n), in.seq, lane)) return false;
        if (p.B == 1) load_vec<KF>(p.hbuf + (size_t)c * (p.F / 4), x, lane);
        for (int i = 0; i < nslot; ++i) {
            const int b = (p.B > 1) ? i : 0, r = (p.B > 1) ? 0 : i;
            const uint32_t seq = in.seq + (uint32_t)c * in.count + r;
            if (!wait_full(p, ring, seq, lane)) return false;
            if (p.B > 1) load_vec<KF>(p.hbuf + (size_t)b * p.F + (size_t)c * (p.F / 4), x, lane);
            float acc[4];
            dot4<KF, true>(ring.stage(seq), x, acc, lane, pol);
            if (lane < 4) {
                const float v = pick4(acc, lane);
                tot[i * 4 + lane] = (c == 0) ? v : tot[i * 4 + lane] + v;
            }
            if (p.B == 1 || i == nslot - 1) release_stage(ring, seq, lane);
        }
    }
    __syncwarp();
    for (int i = 0; i < nslot; ++i) {
        const int b = (p.B > 1) ? i : 0, r = (p.B > 1) ? 0 : i;
        if (lane < 4) residual_one(p, false, b, (in.first + r) * 4 + lane, tot[i * 4 + lane]);
    }
    __syncwarp();
    signal(p, in.signal_ctr, lane);
    return true;
}

template <int HD>
__device__ bool exec_attn(const Params& p, const Ring& ring, const mk_instr& in, int lane,
                          uint32_t epoch, float* sbuf) {
    if (!wait_counter(p, in.wait_ctr, target_of(epoch, in.wait_n), in.seq, lane)) return false;
    const int l = in.layer, b = in.batch, g = in.group;
    const int pos = p.positions[b];
    const int kps = p.keys_per_stage;
    AttnState<HD> st;
    attn_init<HD>(p, b, g, st, lane);
    const uint16_t* Kpos = p.kc + kv_off(p, l, b, g, pos);
    const uint16_t* Vpos = p.vc + kv_off(p, l, b, g, pos);
    for (uint32_t ci = 0; ci < in.nfill; ++ci) {
        const uint32_t seq = in.seq + ci;
        if (!wait_full(p, ring, seq, lane)) return false;
        const int ka = (int)in.first + (int)ci * kps;
        int kend = min(ka + kps, (int)(in.first + in.count));
        kend = min(kend, pos + 1);
        if (ka < kend) {
            const uint16_t* Ks = reinterpret_cast<const uint16_t*>(ring.stage(seq));
            const uint16_t* Vs = Ks + (size_t)kps * HD;
            attn_chunk<HD, true>(p, st, Ks, Vs, Kpos, Vpos, ka, kend, pos, sbuf, kps, lane);
        }
        release_stage(ring, seq, lane);
    }
    attn_store_partial<HD>(p, st, b, g, (int)(in.first / (uint32_t)p.part_keys), lane);
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        const uint32_t old = atom_acq_rel_add(p.counters + (size_t)in.signal_ctr * kCounterStride, 1u);
        last = (old == epoch * in.aux_n + in.aux_n - 1u);
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    if (last) {
        attn_merge<HD>(p, b, g, lane);
        signal(p, in.aux_ctr, lane);
    }
    return true;
}

// ------------------------------------------------------------------ the loader warp

__device__ void loader(const Params& p, const Ring& ring, int i0, int i1) {
    const uint64_t pol = l2_evict_first_policy();
    uint32_t issued = 0;  // fills issued so far (they are numbered 0, 1, 2, ...)
    for (int i = i0; i < i1; ++i) {
        const mk_instr in = p.instrs[i];
        const size_t lbase = p.off_layer0 + (size_t)in.layer * p.layer_stride;
        for (uint32_t t = 0; t < in.nfill; ++t) {
            const uint32_t seq = in.seq + t;
            const uint32_t s = seq % ring.S, use = seq / ring.S;
            if (use > 0) {
                // wait for the consumers to release the previous fill of this stage
                uint64_t t0 = 0;
                bool ok = true;
                for (uint32_t it = 0; !mbar_try_wait(ring.empty + s, (use - 1) & 1u); ++it) {
                    if ((it & 15u) == 15u) {
                        if (t0 == 0) t0 = global_timer_ns();
                        if (aborted(p)) { ok = false; break; }
                        if (global_timer_ns() - t0 > p.timeout_ns) {
                            record_error(p, MK_ERR_TIMEOUT, seq, 0xfffffffdu, 0, use, 3);
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) goto drain;
            }
            {
                uint8_t* dst = ring.base + (size_t)s * ring.stage_bytes;
                uint64_t* bar = ring.full + s;
                ring.armed[s] = seq;  // published by the release of the arrive below
                if (in.op == MK_OP_ATTN) {
                    const int pos = p.positions[in.batch];
                    const int ka = (int)in.first + (int)t * p.keys_per_stage;
                    const int kend = min(ka + p.keys_per_stage, (int)(in.first + in.count));
                    const int np = max(0, min(kend, pos) - ka);  // cached keys (< pos)
                    const uint32_t bytes = (uint32_t)np * p.d * 2;
                    mbar_arrive_expect_tx(bar, 2 * bytes);
                    if (np > 0) {
                        const size_t off = kv_off(p, in.layer, in.batch, in.group, ka);
                        bulk_g2s(dst, p.kc + off, bytes, bar, pol);
                        bulk_g2s(dst + (size_t)p.keys_per_stage * p.d * 2, p.vc + off, bytes, bar, pol);
                    }
                } else {
                    const uint8_t* src;
                    uint32_t bytes;
                    switch (in.op) {
                        case MK_OP_QKV:
                            src = p.packed + lbase + p.rel_qkv + (size_t)(in.first + t) * p.tile_h;
                            bytes = p.tile_h;
                            break;
                        case MK_OP_OPROJ:
                            src = p.packed + lbase + p.rel_o + (size_t)(in.first + t) * p.tile_o;
                            bytes = p.tile_o;
                            break;
                        case MK_OP_GATEUP:
                            src = p.packed + lbase + p.rel_gu + (size_t)(in.first + t) * p.tile_h;
                            bytes = p.tile_h;
                            break;
                        case MK_OP_DOWN: {
                            const uint32_t c = t / in.count, r = t % in.count;
                            src = p.packed + lbase + p.rel_down +
                                  ((size_t)(in.first + r) * 4 + c) * p.tile_f;
                            bytes = p.tile_f;
                            break;
                        }
                        default:  // LM head: rows of the (tied) embedding table
                            src = p.packed + (size_t)(in.first + t) * p.tile_h;
                            bytes = p.tile_h;
                            break;
                    }
                    mbar_arrive_expect_tx(bar, bytes);
                    bulk_g2s(dst, src, bytes, bar, pol);
                }
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
        while (!mbar_try_wait(ring.full + s, par)) {
            if (global_timer_ns() - t0 > p.timeout_ns) {
                record_error(p, MK_ERR_TIMEOUT, last_seq, 0xfffffffcu, 0, par, 4);
                break;
            }
        }
    }
}

// ------------------------------------------------------------------ the kernel

template <int KH, int KO, int KF, int HD>
__global__ void __launch_bounds__(kThreads, 1) megakernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_epoch, s_skip;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Ring ring;
    ring.base = smem;
    ring.stage_bytes = p.stage_bytes;
    ring.S = (uint32_t)p.n_stages;
    ring.full = reinterpret_cast<uint64_t*>(smem + (size_t)p.n_stages * p.stage_bytes);
    ring.empty = ring.full + p.n_stages;
    ring.armed = reinterpret_cast<volatile uint32_t*>(ring.empty + p.n_stages);
    // each consumer warp's scratch slot: its matvec input vector, its attention
    // scores, or its down-projection running sums (one instruction at a time)
    float* warp_scratch = reinterpret_cast<float*>(
        reinterpret_cast<uintptr_t>(ring.armed + p.n_stages + 3) & ~uintptr_t(15));

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.n_stages; ++s) {
            mbar_init(ring.full + s, 1);
            mbar_init(ring.empty + s, 1);
            ring.armed[s] = 0xffffffffu;
        }
        fence_mbar_init();
        s_epoch = ld_volatile_u32(&p.ctl->epoch);
        uint32_t skip = ld_volatile_u32(&p.ctl->status) != 0u;
        if (!skip) {
            for (int b = 0; b < p.B; ++b) {
                const int tok = p.tokens[b], pos = p.positions[b];
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

    if (!s_skip) {
        const int i0 = p.sm_off[blockIdx.x], i1 = p.sm_off[blockIdx.x + 1];
        if (warp == kConsumerWarps) {
            if (lane == 0) loader(p, ring, i0, i1);
        } else {
            const uint64_t pol = l2_evict_first_policy();
            const uint32_t epoch = s_epoch;
            float* slot = warp_scratch + (size_t)warp * p.warp_scratch_floats;
            for (int i = i0 + warp; i < i1; i += kConsumerWarps) {
                const mk_instr in = p.instrs[i];
                bool ok;
                switch (in.op) {
                    case MK_OP_QKV: ok = exec_tiles<MK_OP_QKV, KH, HD>(p, ring, in, lane, pol, epoch, slot); break;
                    case MK_OP_ATTN: ok = exec_attn<HD>(p, ring, in, lane, epoch, slot); break;
                    case MK_OP_OPROJ: ok = exec_tiles<MK_OP_OPROJ, KO, HD>(p, ring, in, lane, pol, epoch, slot); break;
                    case MK_OP_GATEUP: ok = exec_tiles<MK_OP_GATEUP, KH, HD>(p, ring, in, lane, pol, epoch, slot); break;
                    case MK_OP_DOWN: ok = exec_down<KF>(p, ring, in, lane, pol, epoch, slot); break;
                    default: ok = exec_tiles<MK_OP_LMHEAD, KH, HD>(p, ring, in, lane, pol, epoch, slot); break;
                }
                if (!ok) break;
            }
        }
    }
    __syncthreads();

    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t old = atom_acq_rel_add(&p.ctl->done, 1u);
        if (old == gridDim.x - 1) {  // last CTA of the step
            if (ld_volatile_u32(&p.ctl->status) != 0u) {
                for (int c = 0; c < p.n_counters; ++c) p.counters[(size_t)c * kCounterStride] = 0u;
                p.ctl->epoch = 0u;
                p.ctl->abort = 0u;
            } else {
                p.ctl->epoch = s_epoch + 1u;
            }
            p.ctl->done = 0u;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------------ host-side launch

size_t megakernel_smem_bytes(const Params& p) {
    return (size_t)p.n_stages * p.stage_bytes + (size_t)p.n_stages * 20 + 16 +
           (size_t)kConsumerWarps * p.warp_scratch_floats * sizeof(float);
}

using KernelFn = void (*)(Params);

static KernelFn pick(int KH, int KO, int KF, int HD) {
    if (KH == 2 && KO == 2 && KF == 2 && HD == 64) return megakernel<2, 2, 2, 64>;
    if (KH == 8 && KO == 8 && KF == 8 && HD == 64) return megakernel<8, 8, 8, 64>;
    if (KH == 12 && KO == 12 && KF == 8 && HD == 128) return megakernel<12, 12, 8, 128>;
    return nullptr;
}

bool megakernel_supported(int H, int Q, int F, int d) {
    if (H % 256 || Q % 256 || F % 1024) return false;
    return pick(H / 256, Q / 256, F / 1024, d) != nullptr;
}

cudaError_t megakernel_prepare(const Params& p) {
    KernelFn fn = pick(p.H / 256, p.Q / 256, p.F / 1024, p.d);
    if (!fn) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)megakernel_smem_bytes(p));
}

cudaError_t megakernel_occupancy(const Params& p, int* blocks_per_sm) {
    KernelFn fn = pick(p.H / 256, p.Q / 256, p.F / 1024, p.d);
    if (!fn) return cudaErrorInvalidValue;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fn, kThreads,
                                                         megakernel_smem_bytes(p));
}

cudaError_t megakernel_launch(const Params& p, cudaStream_t stream) {
    KernelFn fn = pick(p.H / 256, p.Q / 256, p.F / 1024, p.d);
    if (!fn) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_sm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = megakernel_smem_bytes(p);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace mk
