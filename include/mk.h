/*
 * mk.h -- C ABI of the persistent decode megakernel library (libmk.so).
 *
 * One decode step of a Llama-style decoder (batch 1 or a few sequences) runs as
 * ONE persistent sm_100a kernel: one CTA per SM, each working through a
 * host-built list of instructions, with dependencies between instructions
 * resolved inside the kernel rather than by kernel boundaries. This is the design
 * of the "Look Ma, No Bubbles" Llama-3.2-1B megakernel (summaries: sections
 * "Fusing Operations with an On-GPU Interpreter" and "Custom Synchronization
 * Mechanism") and of the Cohere decode megakernel (section "Megakernel 是什么": a
 * resident block per SM reading a host-written task list of tile-sized work
 * items). Those designs wait on atomic-increment counters; here the activations
 * that cross SMs carry their own validity (64-bit words tagged with the step,
 * layer and producer), the consumer polls the words themselves, and counters
 * remain as completion counts (see mk_read_counters).
 *
 * Conventions for every entry point:
 *   - Pointers documented as "device" must be CUDA device memory of the handle's
 *     device; "host" pointers are ordinary host memory.
 *   - bf16 tensors are arrays of uint16 bit patterns (IEEE bfloat16), row-major.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - No entry point throws; each returns an mk_status. Host-checkable errors are
 *     returned before anything is enqueued. Errors found by the GPU during a step
 *     are recorded on the device and reported by mk_get_status().
 *   - A handle is not thread-safe; distinct handles are independent.
 *   - Calls that enqueue GPU work for a handle (the decode steps) run on the calling
 *     thread's current device and are refused with MK_ERR_INVALID_ARG when that is
 *     not the handle's device. The synchronous calls (create, schedule, status,
 *     readers, destroy) switch to the handle's device themselves and give the
 *     caller's current device back before they return.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mk_status {
    MK_OK = 0,
    MK_ERR_INVALID_ARG = 1,   /* null pointer, bad size, batch > schedule batch ... */
    MK_ERR_CUDA = 2,          /* a CUDA runtime call failed (message via mk_get_status) */
    MK_ERR_UNSUPPORTED = 3,   /* shape this build has no kernel for, or the device cannot
                                 keep one CTA resident on every SM */
    MK_ERR_NO_SCHEDULE = 4,   /* mk_decode_step before mk_build_schedule */
    MK_ERR_TIMEOUT = 5,       /* device: a counter or barrier wait ran past its budget */
    MK_ERR_BAD_TOKEN = 6,     /* device: token outside [0, vocab) */
    MK_ERR_BAD_POSITION = 7,  /* device: position outside [0, min(max_seq, max_ctx)) */
    MK_ERR_OUT_OF_MEMORY = 8
} mk_status;

/* Model shape. The decoder is Llama-style: RMSNorm (eps inside the root),
 * rotate-half RoPE with inv_freq_i = rope_theta^(-2i/head_dim), grouped-query
 * attention (query head h reads KV head h / (n_heads / n_kv_heads)), SiLU-gated
 * MLP, tied embeddings (the embedding table is also the LM head). */
typedef struct mk_config {
    int32_t n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
    float rms_eps;
    double rope_theta;
    int32_t max_batch;   /* batch dimension of the KV cache and largest schedulable batch */
    int32_t max_seq;     /* slot dimension of the KV cache */
} mk_config;
/* Accepted ranges (else MK_ERR_UNSUPPORTED from mk_create, 0 from mk_packed_bytes):
 * 1..64 layers; hidden a multiple of 256 up to 65536; head_dim 64 or 128; at most 32
 * query heads and 4 per KV head; n_heads*head_dim a multiple of 256; ffn a multiple
 * of 1024 up to 262144; vocab a multiple of 4 up to 2^24; max_batch 1..8; max_seq
 * 1..2^20. mk_create further needs a shape the kernels are instantiated for. */

/* Weight pointers for mk_create. Matrices are bf16 row-major [out][in]:
 *   wq [n_heads*head_dim][hidden], wk/wv [n_kv_heads*head_dim][hidden],
 *   wo [hidden][n_heads*head_dim], wgate/wup [ffn][hidden], wdown [hidden][ffn],
 *   embed [vocab][hidden]; norm vectors bf16 [hidden].
 * Per-layer fields are HOST arrays of n_layers pointers. With mk_create the
 * pointed-to tensors are device memory; with mk_pack_weights_host they are host
 * memory. The library copies what it needs: the caller may free them after the
 * call returns. */
typedef struct mk_weights {
    const void* embed;
    const void* const* attn_norm;
    const void* const* wq;
    const void* const* wk;
    const void* const* wv;
    const void* const* wo;
    const void* const* mlp_norm;
    const void* const* wgate;
    const void* const* wup;
    const void* const* wdown;
    const void* final_norm;
} mk_weights;

typedef struct mk_handle mk_handle;

/* Create a handle on `device`: validates the shape, packs the weights into one
 * library-owned device buffer (layout: see mk_pack_weights_host), builds the RoPE
 * table (angles in double, cos/sin stored as float) and allocates the scratch
 * (activations, attention partials, counters). Synchronous. On error *out is NULL.
 * Defining passage: the Cohere decode megakernel page ("Cohere 开源 Megakernel 推理
 * 系统"), section "Megakernel 是什么": one resident thread block per SM for the
 * whole decode step, working from host-prepared tile-sized tasks; the handle
 * holds what those tasks read, laid out once before any step (weights as
 * contiguous tiles, the RoPE table, the counters and scratch in global memory). */
mk_status mk_create(const mk_config* cfg, const mk_weights* w, int device, mk_handle** out);

/* Options for mk_build_schedule; pass NULL for defaults. Zero fields mean "auto". */
typedef struct mk_schedule_opts {
    int32_t n_sm;            /* SMs to use (<= device SMs); 0 = all */
    int32_t part_keys;       /* keys per attention partition (a multiple of 8 up to the
                                ring's keys-per-stage, else a multiple of it); 0 = one
                                partition per (sequence, KV group) up to 320 keys, beyond
                                that as many as leave one item per SM (each of at most
                                512 keys and what the ring holds) */
    int32_t rowblocks_down;  /* 4-row blocks per down-projection instruction at most
                                (1..16); 0 = 16 */
    uint32_t seed;           /* 0 = plain greedy placement; else ties are broken by a
                                seeded shuffle (for robustness tests) */
    int32_t wait_timeout_ms; /* budget of every device wait; 0 = 2000 ms */
    int32_t test_drop_item;  /* failure-detection test hook: 1-based index, in the list
                                order, of one instruction that computes but never publishes
                                its outputs or its completion (its consumers then end the
                                step with MK_ERR_TIMEOUT); 0 = none */
    int32_t trace;           /* nonzero: every step records per-job timestamps (see
                                mk_read_trace) */
    int32_t proj;            /* the projections' arithmetic at batch > 1: MK_PROJ_AUTO
                                (the tensor cores), MK_PROJ_CUDA_CORES or
                                MK_PROJ_TENSOR_CORES (batch 1 always runs on the CUDA
                                cores) */
} mk_schedule_opts;

/* mk_schedule_opts.proj. Tensor cores: each instruction's weight rows stream as
 * 64-column TMA boxes (128-byte swizzle) and one thread issues tcgen05.mma
 * (M = 128 weight rows, N = 16: the batch's fp32 inputs split into bf16 high and
 * low parts, K = 16 per instruction) into an fp32 accumulator in Tensor Memory,
 * read back by the compute warps for the same fused epilogues; four warps issue
 * the MMAs, one per K step of each box. CUDA cores: each 4-row tile's batched fp32
 * dot product, as at batch 1. AUTO picks the tensor cores: measured on the
 * 3B-style shape at batch 8 and 2048 positions (one B200) the step takes 6.30 ms
 * against 6.63 ms. The two differ only in the order and form of the fp32
 * accumulation. The tensor-core path needs a vocabulary that is a multiple of 8
 * (else the CUDA cores run). */
#define MK_PROJ_AUTO 0
#define MK_PROJ_CUDA_CORES 1
#define MK_PROJ_TENSOR_CORES 2

/* Build the per-SM instruction lists for `batch` sequences (1 <= batch <= max_batch)
 * whose steps use at most `max_ctx` keys (position + 1 <= max_ctx <= max_seq), and
 * upload them. Replaces any earlier schedule. Synchronous.
 * Defining passages: the "Look Ma, No Bubbles" summary, section "Fusing Operations
 * with an On-GPU Interpreter" (each SM executes a sequence of instructions such as
 * fused RMSNorm + QKV + RoPE, attention, ...), and the Stanford write-up
 * ("斯坦福团队新作：Llama-1B实现毫秒级推理获Andrej Karpathy盛赞"), section
 * "Megakernel：从零设计的融合思路" (an execution plan per SM, dependencies between
 * instructions arranged statically before the run); the Cohere page, section
 * "Megakernel 是什么" (the host writes the task list into global memory).
 * The attention of a (sequence, KV group) is split into at most 32 key partitions,
 * each holding at most what the SM's weight ring holds at once (and 512 keys), so
 * max_ctx has a ceiling that depends on the shape and batch: 16384 keys for the
 * Llama-3.2-1B shape; for head_dim 128 with 24 query and 8 KV heads, 12288 at
 * batch 1 and 7168 at batch 2-8 (on the CUDA-core path 12288 at batch 2 and 6144 at
 * 3-8). A larger max_ctx
 * (or a part_keys that needs more than 32 partitions) returns MK_ERR_INVALID_ARG. */
mk_status mk_build_schedule(mk_handle* h, int batch, int max_ctx, const mk_schedule_opts* opts);

/* One decode step of the persistent megakernel, asynchronous on `stream`.
 * Defining passage: the "Look Ma, No Bubbles" summary, section "Megakernel: The
 * Core Solution" (the whole Llama-1B forward pass as one kernel, so loads and
 * compute continue across what would be kernel boundaries), with section "Custom
 * Synchronization Mechanism" (dependencies inside the kernel; the MLP's
 * intermediate state in four chunks so the down-projection starts early).
 *   tokens, positions : device int32 [batch]
 *   k_cache, v_cache  : device bf16 [n_layers][max_batch][n_kv_heads][max_seq][head_dim],
 *                       caller-owned; sequence b reads slots 0..positions[b] and writes
 *                       slot positions[b] (its RoPE'd key and its value)
 *   logits            : device fp32 [batch][vocab]
 * Enqueues exactly one cooperative kernel launch; no host synchronisation, no
 * allocation. A step with a bad token or position writes no KV slot and leaves the
 * logits unspecified; the error is reported by mk_get_status. Returns
 * MK_ERR_INVALID_ARG (nothing enqueued) for a NULL pointer, a KV cache that is not
 * 16-byte aligned, or a calling thread whose current device is not the handle's;
 * MK_ERR_NO_SCHEDULE before mk_build_schedule. */
mk_status mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions,
                         void* k_cache, void* v_cache, float* logits, void* stream);

/* n_steps greedy decode steps back to back, asynchronous on `stream`, with no host
 * work between them: each is mk_decode_step with the greedy choice fused into its
 * LM head. Each LM-head instruction reduces its rows to the best (largest logit,
 * lowest index among equal ones, NaN never chosen; an all-NaN row gives 0) per
 * sequence; the SM that completes the step's LM head picks each sequence's next
 * token from those and writes it over tokens[b], writes positions[b] + 1 over
 * positions[b], and, when `generated` (device int32 [n_steps][batch]) is given,
 * stores it at generated[step][b]. The next launch then decodes it. The tokens
 * equal mk_greedy_select's on the same logits, bit for bit; `logits` holds the
 * last step's. Arguments as for mk_decode_step (tokens and positions are read and
 * written); n_steps >= 1 launches are enqueued. The caller keeps the positions
 * below max_ctx: a step past it is skipped and reported (MK_ERR_BAD_POSITION), as
 * are the steps after it. Defining passage: the "Look Ma, No Bubbles" summary,
 * section "Megakernel: The Core Solution" (no kernel boundaries inside a forward
 * pass): here the token choice, too, stays inside the step's kernel. */
mk_status mk_decode_steps_greedy(mk_handle* h, int32_t* tokens, int32_t* positions, void* k_cache,
                                 void* v_cache, float* logits, int32_t* generated, int n_steps, void* stream);

/* The same step as a sequence of ordinary kernels (one per op and layer), the
 * multi-kernel "bubble" baseline; identical arguments, identical arithmetic, so
 * its results equal mk_decode_step's bit for bit. Capturable in a CUDA graph. */
mk_status mk_baseline_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions,
                                  void* k_cache, void* v_cache, float* logits, void* stream);

/* End-to-end step from HOST buffers: copies tokens and positions (host int32
 * [batch], preferably pinned) to the device, runs mk_decode_step, copies the
 * logits back to `logits_host` (fp32 [batch][vocab]) and synchronises `stream`.
 * Uses handle-owned device staging (no allocation per call). Returns the
 * host-side status; device-detected errors are reported by mk_get_status. */
mk_status mk_decode_step_host(mk_handle* h, const int32_t* tokens_host,
                              const int32_t* positions_host, void* k_cache, void* v_cache,
                              float* logits_host, void* stream);

/* Synchronises the device, then reports and clears the device-side error state.
 * *device_status receives the first error recorded since the last call (MK_OK if
 * none); msg (may be NULL) receives a one-line description. After an error every
 * step is skipped until this call clears it. Returns MK_ERR_CUDA if the sync fails. */
mk_status mk_get_status(mk_handle* h, mk_status* device_status, char* msg, size_t msg_len);

/* Frees everything the handle owns. NULL is allowed. */
void mk_destroy(mk_handle* h);

const char* mk_status_str(mk_status s);

/* Greedy selection between decode steps: next_tokens[b] = the index v in [0, vocab)
 * of the largest logits[b][v], the lowest such index where several are equal (the
 * greedy decoding rule of the decoder's generation loop). NaN entries are never
 * selected; a row of NaNs gives 0.
 *   logits       device fp32 [batch][vocab], rows contiguous (mk_decode_step's output)
 *   batch, vocab >= 1
 *   next_tokens  device int32 [batch]; may be the tokens buffer of the next
 *                mk_decode_step, so a decode loop needs no host round trip
 *   positions    device int32 [batch] or NULL: when given, each positions[b] is
 *                incremented by one in the same launch
 *   stream       the CUDA stream the selection is enqueued on
 * Enqueues one kernel launch (one CTA per sequence) on the calling thread's current
 * device, which must own the buffers and the stream; no synchronisation, no
 * allocation, capturable in a CUDA graph. Returns MK_ERR_INVALID_ARG for a NULL
 * logits or next_tokens pointer or a size below 1, MK_ERR_CUDA if the launch fails. */
mk_status mk_greedy_select(const float* logits, int batch, int vocab, int32_t* next_tokens,
                           int32_t* positions, void* stream);

/* ------------------------------------------------------------------ inspection */

/* One instruction of the per-SM lists (48 bytes). An SM's CTA runs its list in
 * order; each instruction is one "job" for all of the CTA's compute warps (a
 * down-projection is four jobs, one per MLP chunk; up to eight consecutive
 * attention items form one job, one item per warp). The kinds: */
enum {
    MK_OP_QKV = 1,     /* RMSNorm + QKV matvec + RoPE; writes q and the KV slot */
    MK_OP_ATTN = 2,    /* GQA attention over one key partition of a (sequence, KV group)
                          pair; the pair's last partition to finish merges the pair */
    MK_OP_OPROJ = 3,   /* O-projection + residual */
    MK_OP_GATEUP = 4,  /* RMSNorm + gate/up matvec + SiLU-gated product */
    MK_OP_DOWN = 5,    /* down-projection over the 4 MLP chunks + residual */
    MK_OP_LMHEAD = 6   /* final RMSNorm + LM head */
};
#define MK_NO_COUNTER 0xffffffffu

typedef struct mk_instr {
    uint16_t op, layer;
    uint16_t batch;      /* sequence (MK_OP_ATTN), else 0 */
    uint16_t group;      /* KV group (QKV, ATTN), else 0 */
    uint32_t first;      /* first 4-row tile / row block (DOWN) / first key (ATTN);
                            GATEUP: first tile of the SM's slice of each MLP chunk */
    uint32_t count;      /* tiles / row blocks / keys */
    uint32_t seq;        /* index of its first ring stage fill in this SM's stream */
    uint32_t nfill;      /* ring stage fills it consumes */
    uint32_t wait_ctr;   /* counter waited on (MK_NO_COUNTER: none); DOWN waits on the
                            4 consecutive chunk counters wait_ctr .. wait_ctr+3 */
    uint32_t wait_n;     /* increments that counter receives per step (DOWN: chunk 0) */
    uint32_t signal_ctr; /* counter incremented by one when the instruction is done;
                            ATTN: the layer's attention counter, incremented once per
                            query head when that head's output is final */
    uint32_t job_items;  /* 1: every instruction (an attention item included) is one
                            job of the SM's compute warps (DOWN: four, one per chunk) */
    uint32_t aux0, aux1; /* DOWN: per-step increments of chunk counters 1, 2 (low and
                            high 16 bits of aux0) and 3 (aux1). ATTN: aux0 = the pair's
                            arrival counter (heads whose partial is stored). LMHEAD:
                            aux0 = its ordinal among the step's LM-head instructions. GATEUP:
                            aux0 = tiles per chunk; the instruction's tile i is tile
                            (i / aux0) * (ffn / 8) + first + i % aux0 (chunk-major). QKV and
                            GATEUP: aux1 = how many consecutive counters from signal_ctr
                            the instruction increments by one each (the KV groups / MLP
                            chunks its tiles touch; 0 reads as 1). Else 0 */
} mk_instr;

typedef struct mk_schedule_info {
    int32_t n_sm, batch, max_ctx, part_keys, n_parts, keys_per_stage;
    int32_t stage_bytes, n_stages, n_counters, n_instr;
    uint64_t bytes_per_step;    /* weight + KV bytes one step streams */
    uint64_t max_sm_bytes;      /* largest per-SM share of those bytes */
    uint64_t min_sm_bytes;
    int32_t proj;               /* the projections' path: MK_PROJ_CUDA_CORES or _TENSOR_CORES */
    int32_t reserved0;
} mk_schedule_info;

/* Plans a schedule on the host only (no device, no handle): writes up to
 * `cap` instructions to instr_out (may be NULL to query), n_sm+1 list offsets to
 * sm_offsets (may be NULL) and the summary to info. `stage_bytes` is the ring
 * stage size the kernel would use (0 = the library's choice for this shape).
 * Returns MK_ERR_INVALID_ARG if cap is too small (info->n_instr says how many). */
mk_status mk_plan_schedule_host(const mk_config* cfg, int batch, int max_ctx, int n_sm,
                                const mk_schedule_opts* opts, mk_instr* instr_out, size_t cap,
                                int32_t* sm_offsets, mk_schedule_info* info);

/* One tensor map of the tensor-core path (mk_schedule_opts.proj): a view of the
 * packed weights (mk_pack_weights_host's layout) as bf16 elements. Element
 * (c_0, ..., c_{rank-1}) sits at byte base_offset + 2 * c_0 + sum_{i >= 1} c_i *
 * strides[i - 1] of the packed buffer; box is the block one TMA copy reads (one
 * fill: 64 columns x rows x boxes of 64 columns). index is the map's place in the
 * kernel's table. */
typedef struct mk_tmap_spec {
    int32_t index, rank;
    uint64_t base_offset;
    uint64_t dims[5];
    uint64_t strides[4];
    uint32_t box[5];
} mk_tmap_spec;

/* The tensor maps a schedule with ring stages of `stage_bytes` uses (host only, for
 * inspection and tests): writes up to `cap` specs to out (may be NULL to query)
 * and their count to *n. MK_ERR_UNSUPPORTED for a shape the kernels do not take. */
mk_status mk_tensor_map_specs_host(const mk_config* cfg, uint32_t stage_bytes, mk_tmap_spec* out, size_t cap,
                                   size_t* n);

/* Summary of the handle's current schedule. */
mk_status mk_get_schedule_info(mk_handle* h, mk_schedule_info* info);

/* Copies the handle's step counters (uint32 each) to host memory: the
 * dependency counters, then epoch, then the end-of-step arrival count.
 * *n_total receives how many exist; at most n are copied. Synchronous. */
mk_status mk_read_counters(mk_handle* h, uint32_t* host, size_t n, size_t* n_total);

/* Per-job timestamps of the last traced step (schedule built with opts.trace):
 * uint64 [n_sm][jobs][16] globaltimer nanoseconds -- 0 activation warp starts
 * waiting for a free input slot, 1 slot free, 2 the activation warp starts its
 * part of the job, 3 its part is ready (the slot is handed to the compute
 * warps), 4 compute warp 0 starts (it then builds the job's input from the
 * producers' tagged words), 5 the job's last compute warp finished, 6 op |
 * layer << 8 | chunk << 24, 7 compute warp 0 has its first ring fill of the job
 * (0 if it had none), 8..15 finer op-specific points of compute warp 0 (15: the
 * job's input built; 0 where unused).
 * *jobs receives the per-SM job capacity; at most `bytes` are copied.
 * Synchronous. */
mk_status mk_read_trace(mk_handle* h, uint64_t* host, size_t bytes, int32_t* jobs);

/* Bytes of the packed weight buffer for `cfg`. */
size_t mk_packed_bytes(const mk_config* cfg);

/* Packs host weights into `dst` (host, mk_packed_bytes(cfg) bytes) with the same
 * layout mk_create builds on the device, 256-byte aligned regions in this order:
 *   embed      [vocab][hidden] unchanged (it is also the LM head);
 *   per layer:
 *     QKV      4-row tiles of [4][hidden]; KV group g holds, in order, its
 *              n_heads/n_kv_heads query heads, key head g, value head g; a query or
 *              key head's tile j holds rows {2j, 2j+d/2, 2j+1, 2j+1+d/2} (the two
 *              RoPE pairs), a value head's tile j rows {4j..4j+3};
 *     O        wo unchanged [hidden][n_heads*head_dim];
 *     gate/up  tile j = rows {gate 2j, up 2j, gate 2j+1, up 2j+1} of [4][hidden];
 *     down     for row block r (rows 4r..4r+3), chunk c (columns c*ffn/4 ..): a
 *              [4][ffn/4] tile, ordered [r][c];
 *   norms      attn_norm[l], mlp_norm[l] for each layer, then final_norm.
 * Bit copy only. */
mk_status mk_pack_weights_host(const mk_config* cfg, const mk_weights* w, void* dst,
                               size_t dst_bytes);

/* The multi-kernel decode step (as mk_baseline_decode_step) for callers that
 * cannot allocate device memory -- an engine whose device memory is all handed
 * out by its own arena, or code running where cudaMalloc is not allowed. It
 * needs no handle and allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library call); the web pages describe no such entry point, it has
 * no counterpart there. The caller owns every input and output:
 *   cfg               the model (as for mk_create)
 *   packed            device, mk_packed_bytes(cfg) bytes in the mk_pack_weights_host
 *                     layout (e.g. packed on the host and copied by the caller)
 *   tokens, positions device int32 [batch]
 *   k_cache, v_cache  device bf16 [n_layers][max_batch][n_kv_heads][max_seq][head_dim]
 *                     (as for mk_decode_step: reads slots 0..positions[b], writes
 *                     slot positions[b])
 *   logits            device fp32 [batch][vocab]
 *   batch, max_ctx    1 <= batch <= cfg->max_batch; positions[b] + 1 <= max_ctx <=
 *                     cfg->max_seq
 *   status_out        device int32 or NULL: receives the step's device status
 *                     (MK_OK, MK_ERR_BAD_TOKEN, MK_ERR_BAD_POSITION)
 *   stream            the CUDA stream the step is enqueued on
 * Scratch (activations, attention partials, the RoPE table, the error word) lives
 * in one 4 MiB device array of the library, per device, held until the process
 * exits. Its layout does not depend on max_ctx: the RoPE table holds a fixed
 * number of positions per head_dim (8192 at 64, 4096 at 128) in a 2 MiB region,
 * the activations follow at a fixed offset. The first call on a device (with that
 * device current) looks up the array's device address, and a call whose
 * rope_theta or head_dim differs from the table in the array uploads a new table
 * from the stack: make those calls before any stream capture (during a capture
 * such a call returns MK_ERR_INVALID_ARG), and do not replay a graph captured
 * before a change of rope_theta or head_dim. Every call shares the array and
 * leaves its contents for the next; the error word is cleared by each call. Calls
 * that overlap on the GPU (on different streams, or from different host threads)
 * race on it.
 * Returns MK_ERR_INVALID_ARG for bad arguments, for max_ctx beyond the RoPE
 * table's positions, and for a step whose activations and attention partials
 * exceed the array's other 2 MiB (more than 32 attention partitions of 320 keys
 * are refused too). */
mk_status mk_baseline_decode_step_noalloc(const mk_config* cfg, const void* packed, const int32_t* tokens,
                                          const int32_t* positions, void* k_cache, void* v_cache, float* logits,
                                          int batch, int max_ctx, int32_t* status_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
