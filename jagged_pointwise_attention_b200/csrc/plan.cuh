// plan.cuh -- longest-first work list for the jagged attention.
//
// A work unit is one 128-row query tile of one sequence: rows [q0, q_end),
// keys from the sequence start k0, nk = t + 1 key tiles for query tile t
// (tiles after the diagonal are skipped by causality). Units are listed by
// descending nk, so the block scheduler hands out the longest units first
// (greedy longest-processing-time order); heads are expanded by the kernel.
#pragma once

#include "common.cuh"

namespace hstu {

// One block. Shared memory: 3 * max_tiles ints.
__global__ void __launch_bounds__(1024)
plan_kernel(const int64_t* __restrict__ seq_offsets, int B, int max_seqlen, int max_tiles,
            int max_units, int4* __restrict__ units, int* __restrict__ unit_count) {
    extern __shared__ int plan_smem[];
    int* hist = plan_smem;               // units with query tile t
    int* start = hist + max_tiles;       // first list slot of tile t
    int* fill = start + max_tiles;       // slots of tile t used so far
    for (int t = threadIdx.x; t < max_tiles; t += blockDim.x) {
        hist[t] = 0;
        fill[t] = 0;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        int64_t n = seq_offsets[b + 1] - seq_offsets[b];
        if (n < 0 || n > max_seqlen) {
            raise_error(kErrBadInput);
            n = n < 0 ? 0 : max_seqlen;
        }
        const int nt = static_cast<int>((n + kTile - 1) / kTile);
        for (int t = 0; t < nt; ++t) atomicAdd(&hist[t], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int t = max_tiles - 1; t >= 0; --t) {
            start[t] = acc;
            acc += hist[t];
        }
        *unit_count = acc < max_units ? acc : max_units;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int64_t o = seq_offsets[b];
        int64_t n = seq_offsets[b + 1] - o;
        n = n < 0 ? 0 : (n > max_seqlen ? max_seqlen : n);
        const int nt = static_cast<int>((n + kTile - 1) / kTile);
        for (int t = 0; t < nt; ++t) {
            const int slot = start[t] + atomicAdd(&fill[t], 1);
            if (slot < max_units) {
                const int64_t q0 = o + static_cast<int64_t>(t) * kTile;
                const int64_t qe = q0 + kTile < o + n ? q0 + kTile : o + n;
                units[slot] = make_int4(static_cast<int>(q0), static_cast<int>(qe),
                                        static_cast<int>(o), t + 1);
            }
        }
    }
}

}  // namespace hstu
