// Greedy token selection on the device, between two decode steps.
//
// Greedy decoding takes as the next token the index of the largest logit of the
// step, the lowest index among equal maxima. Doing that on the device keeps a
// multi-step decode loop free of host round trips: the selected ids are written
// straight into the token buffer the next mk_decode_step reads, and the
// positions can be advanced by the same launch.
//
// One CTA of 1024 threads per sequence. A row is 128256 fp32 logits (501 KB) for
// the Llama-3.2 vocabulary, just written by the step's LM head and so still in
// L2; each thread scans a strided slice (16-byte loads where the row allows),
// then the CTA reduces (value, index) pairs through warp shuffles and shared
// memory. The comparison is total over non-NaN values, so the result does not
// depend on the scan or reduction order.
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>

#include "mk.h"

namespace {

constexpr int kThreads = 1024;

struct Best {
    float v;
    int i;  // INT32_MAX: nothing seen yet
};

// (v, i) replaces a when v is larger, or equal with a lower index; a NaN v never does
__device__ __forceinline__ void take(Best& a, float v, int i) {
    if (v > a.v || (v == a.v && i < a.i)) {
        a.v = v;
        a.i = i;
    }
}

__global__ void __launch_bounds__(kThreads) greedy_select_kernel(const float* __restrict__ logits, int vocab,
                                                                  int32_t* __restrict__ next_tokens,
                                                                  int32_t* __restrict__ positions) {
    __shared__ Best warp_best[kThreads / 32];
    const int b = blockIdx.x, tid = threadIdx.x;
    const float* row = logits + (size_t)b * vocab;
    Best best{-INFINITY, INT32_MAX};
    // the aligned body in float4 loads, the rest one element at a time
    const int head = (int)(((16u - ((uintptr_t)row & 15u)) & 15u) / 4u);
    const int lead = head < vocab ? head : vocab;
    const int n4 = (vocab - lead) / 4;
    if (tid < lead) take(best, row[tid], tid);
    const float4* body = reinterpret_cast<const float4*>(row + lead);
#pragma unroll 4
    for (int j = tid; j < n4; j += kThreads) {
        const float4 q = body[j];
        const int i = lead + 4 * j;
        take(best, q.x, i);
        take(best, q.y, i + 1);
        take(best, q.z, i + 2);
        take(best, q.w, i + 3);
    }
    for (int i = lead + 4 * n4 + tid; i < vocab; i += kThreads) take(best, row[i], i);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
        const float v = __shfl_xor_sync(0xffffffffu, best.v, m);
        const int i = __shfl_xor_sync(0xffffffffu, best.i, m);
        take(best, v, i);
    }
    if ((tid & 31) == 0) warp_best[tid >> 5] = best;
    __syncthreads();
    if (tid < 32) {
        best = warp_best[tid];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            const float v = __shfl_xor_sync(0xffffffffu, best.v, m);
            const int i = __shfl_xor_sync(0xffffffffu, best.i, m);
            take(best, v, i);
        }
        if (tid == 0) {
            next_tokens[b] = best.i == INT32_MAX ? 0 : best.i;
            if (positions) positions[b] += 1;
        }
    }
}

}  // namespace

extern "C" mk_status mk_greedy_select(const float* logits, int batch, int vocab, int32_t* next_tokens,
                                      int32_t* positions, void* stream) {
    if (!logits || !next_tokens || batch < 1 || vocab < 1) return MK_ERR_INVALID_ARG;
    greedy_select_kernel<<<batch, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(logits, vocab, next_tokens,
                                                                                    positions);
    return cudaGetLastError() == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}
