// Host-side packer and schedule builder interfaces (internal to libmk.so).
#pragma once

#include <vector>

#include "mk_internal.h"

namespace mk {

struct Segment {
    size_t dst;          // byte offset in the packed buffer
    const void* src;     // source bytes (device pointer for mk_create, host for the host packer)
    uint32_t bytes;
    uint32_t pad;
};

std::vector<Segment> pack_segments(const Layout& L, const mk_weights& w);
bool weights_complete(const Layout& L, const mk_weights& w);

struct Plan {
    std::vector<mk_instr> instrs;   // SM lists, concatenated
    std::vector<int32_t> sm_off;    // n_sm + 1 offsets into instrs
    mk_schedule_info info;
};

// Ring stage size the kernel uses for this shape.
uint32_t default_stage_bytes(const Layout& L, bool mma = false);

// Shared-memory budget split: activation slots and ring stages.
struct SlotPlan {
    int keys_per_stage;
    uint32_t vec_floats;   // one sequence's input vector inside a slot
    uint32_t item_bytes;   // an attention item's q and new key/value inside a slot
    uint32_t aux_floats;   // where the RoPE rows and residual rows start inside a slot
    uint32_t slot_bytes;
    int xs_slots;
    int stages;
    uint32_t smem_bytes;
};
SlotPlan slot_plan(const Layout& L, int batch, uint32_t stage_bytes, bool mma = false);
// Whether a schedule for `batch` with these options runs the projections on the
// tensor cores.
bool use_mma(const Layout& L, int batch, const mk_schedule_opts* opts);

// The tensor-core path's tensor maps for ring stages of stage_bytes (mk_tmap_spec).
std::vector<mk_tmap_spec> tmap_specs(const Layout& L, uint32_t stage_bytes);

mk_status plan_schedule(const Layout& L, int batch, int max_ctx, int n_sm,
                        const mk_schedule_opts* opts, uint32_t stage_bytes, Plan* out);

}  // namespace mk
