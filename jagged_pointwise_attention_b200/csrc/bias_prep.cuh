// bias_prep.cuh -- per-launch bias tables of the bf16 attention.
//
// The attention stages two things per key tile, and both depend on less than
// the (query tile, key tile) pair:
//  * the relative-position window of the tile, bf16 pos/2 in the sliding-
//    window layout of BiasStage::wb, depends only on the head h and the
//    tile's diagonal offset dd = (q0 - kt0) / 128. Offsets dd >= DD - 1 see
//    only the last table entry (the whole window clamps to P - 1), so DD
//    tables per head cover every tile;
//  * the key timestamps of the tile relative to its first key, with per
//    32-key chunk minimum, maximum and exactness flags, depend only on the
//    key tile, i.e. on the unit whose rows are those keys.
// This kernel builds both once per launch, in the workspace; the attention
// copies them into shared memory per tile with two bulk copies.
#pragma once

#include "attn_tc.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

// Diagonal offsets whose windows differ: the window of offset dd reads
// pos[clamp(128 dd + 127 - k)], k = 0..254, which is all pos[P - 1] once
// 128 dd - 127 >= P - 1.
__host__ __device__ inline int window_tables(int P, int max_tiles) {
    const int dc = (P + 126 + 127) / 128;          // first fully clamped offset
    const int dd = dc + 1;
    return dd < max_tiles ? dd : (max_tiles > 0 ? max_tiles : 1);
}

struct BiasPrepArgs {
    const float* pos;           // [H, P] or null (tables of zeros)
    int P, H, DD;
    uint4* ptab;                // [H][DD][kWinEntries]
    const int4* units;          // plan's units and count
    const int* unit_count;
    int max_units;
    const int64_t* ts;          // [T] or null (no key summaries)
    int64_t T;
    KeySummary* ksum;           // [max_units]
    int table_blocks;           // blocks [0, table_blocks) build tables, the rest one unit each
};

// Programmatic launch chain plan -> bias prep -> attention. The attention
// waits (griddepcontrol.wait) only for this grid, its direct prerequisite, so
// this grid must not complete before the plan has: every block of it executes
// griddepcontrol.wait before it exits, including the blocks that never read
// the plan's output. The table blocks wait after writing their entries, so
// that work still overlaps the plan.
__global__ void __launch_bounds__(128) bias_prep_kernel(const BiasPrepArgs a) {
    // let the attention that follows start its set-up (it waits for this grid)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x;
    if (static_cast<int>(blockIdx.x) < a.table_blocks) {
        // entry s of table (h, dd) holds R[s..s+7]: words (R[s+2i], R[s+2i+1])
        const int64_t e = static_cast<int64_t>(blockIdx.x) * 128 + tid;
        if (e < static_cast<int64_t>(a.H) * a.DD * kWinEntries)
            a.ptab[e] = window_entry(a.pos, a.P, a.DD, e);
        asm volatile("griddepcontrol.wait;" ::: "memory");   // complete only after the plan
        return;
    }
    // key summary of unit u: its 128 rows as keys
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the plan's units
    if (a.ts == nullptr) return;
    const int u = static_cast<int>(blockIdx.x) - a.table_blocks;
    const int n_units = min(*a.unit_count, a.max_units);
    if (u >= n_units) return;
    const int4 d = a.units[u];
    const int lane = tid & 31, c = tid >> 5;
    const int64_t kt0 = d.x;
    const int64_t key = kt0 + tid;
    const bool kvalid = key < d.y;
    const int64_t kv = __ldg(a.ts + (key < a.T ? key : a.T - 1));
    const int64_t base = __ldg(a.ts + kt0);
    const int64_t dk = kv - base;
    KeySummary& ks = a.ksum[u];
    ks.kt32[tid] = static_cast<int32_t>(dk);
    const bool near = dk > -(1ll << 30) && dk < (1ll << 30);
    const int dmin = __reduce_min_sync(0xffffffffu, (kvalid && near) ? static_cast<int>(dk) : INT_MAX);
    const int dmax = __reduce_max_sync(0xffffffffu, (kvalid && near) ? static_cast<int>(dk) : INT_MIN);
    const bool all_near = __all_sync(0xffffffffu, !kvalid || near);
    if (lane == 0) {
        ks.cmin[c] = dmin;
        ks.cmax[c] = dmax;
        ks.ok[c] = all_near ? 1 : 0;
    }
    if (tid == 0) {
        ks.base = base;
        ks.pad[0] = ks.pad[1] = 0;
    }
}

}  // namespace hstu
