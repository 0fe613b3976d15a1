// kv_append.cuh -- KV-cache append: after a block is decoded the encoder absorbs it and each
// layer's cache grows by that block ("Encoder-Decoder Diffusion Language Models for Efficient
// Training and Inference", paper notes, sec. 3).  A pure copy, HBM-bound: 16-byte vector
// loads and stores, grid-stride over the rows of K (blockIdx.y == 0) and V (blockIdx.y == 1).
// Every entry appends at the same length P, or (ragged) at its own length read from the device.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace e2d2 {

struct AppendParams {
    uint4* cache[2];      // K, V caches [B*Hkv][capacity][D]
    const uint4* src[2];  // new rows [B*Hkv][S_new][D]
    int capacity, P, S_new, vec_per_row, units;
    // ragged: entry b appends at its own length P_dev[b] (device array, clamped to [0, capacity]);
    // rows that would land at or past capacity are not written.  Null: every entry at P.
    const int* P_dev;
    int kv_heads;
};

__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams a) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();  // the previous kernel may still read the cache or write the new rows
    const int which = blockIdx.y;
    uint4* __restrict__ dst = a.cache[which];
    const uint4* __restrict__ src = a.src[which];
    const long long per_unit = static_cast<long long>(a.S_new) * a.vec_per_row;
    const long long total = per_unit * a.units;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long unit = i / per_unit;
        const long long rem = i - unit * per_unit;  // (row, vec) inside the unit
        long long P = a.P;
        if (a.P_dev != nullptr) {
            const int pb = __ldg(a.P_dev + unit / a.kv_heads);
            P = pb < 0 ? 0 : (pb > a.capacity ? a.capacity : pb);
            if (P + rem / a.vec_per_row >= a.capacity) continue;
        }
        const long long d = (unit * a.capacity + P) * a.vec_per_row + rem;
        dst[d] = __ldg(src + i);
    }
}

}  // namespace e2d2
