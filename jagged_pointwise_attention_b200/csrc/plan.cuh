// plan.cuh -- work list of the jagged attention.
//
// A work unit is a tile of at most 128 query rows with the key range it needs:
// (q0, q_end, k0, nk | nt << 11 | packed << 31), nt = the number of units of
// its sequence (1 for packed units). Two kinds:
//  * aligned: query tile t of a sequence longer than 128 tokens: rows
//    [o + 128t, min(o + 128t + 128, o + n)), keys from the sequence start
//    k0 = o, nk = t + 1 key tiles (tiles past the diagonal are causally empty).
//  * packed: several whole sequences of at most 128 tokens each, consecutive in
//    the batch, sharing one tile: rows [q0, q_end) = keys, nk = 1 (k0 = q0).
//    starts[u] marks the rows of the tile where a sequence begins (bit r of
//    the 128-bit mask = row q0 + r), from which the kernel finds each row's
//    own sequence start to mask pairs that cross a sequence boundary. Packing
//    is greedy inside each 128-token bucket of sequence start positions, so
//    buckets are packed in parallel, each in one pass by one thread.
// Aligned units are listed sequence by sequence, longest sequence first, and
// inside a sequence by descending query tile (descending nk); packed units
// follow. The attention kernel hands out work items (unit, head) in the order
// sequence, head, tile, so the CTAs running at any time share the keys and
// values of one or two (sequence, head) pairs, which stay in L2, while items
// still come longest first within each pair.
//
// Aligned units are placed without per-unit atomics: sequences are counting-
// sorted by their tile count nt (descending); a sequence of rank rho in the
// bucket of count v starts at unit cum[v] + (rho - base[v]) * v, cum[v]
// counting the units of all longer buckets.
//
// On request (order_tab non-null) the plan also writes the table from which
// the attention backward orders its work items by cost: for v = 1 ..
// max_tiles, in four rows of max_tiles + 2 ints, the number of sequences
// with nt >= v; the number of items (order_h per unit, one per head) of
// aligned units with nk >= v; cum[v]; base[v]. Entry max_tiles + 1 of the
// first two rows is 0.
#pragma once

#include "common.cuh"

namespace hstu {

constexpr int kPlanSmemOffsets = 4096;    // offsets cached in shared memory below this B

// One block of 1024 threads. Dynamic shared memory: 3 * (max_tiles + 1) ints,
// then (B + 1) int64 offsets when B < kPlanSmemOffsets. The body is compiled
// once for offsets in shared memory (kCache) and once for offsets read from
// global memory: a pointer that may be either makes every offset load a
// generic load, which then waits behind the thread's global stores.
template <bool kCache>
__device__ __forceinline__ void plan_body(const int64_t* __restrict__ seq_offsets, int B, int64_t T,
                                          int max_seqlen, int max_tiles, int max_units,
                                          int4* __restrict__ units, uint4* __restrict__ starts,
                                          int* __restrict__ unit_count,
                                          int* __restrict__ item_counter, int* plan_smem,
                                          int order_h, int* __restrict__ order_tab) {
    const int NT = max_tiles + 1;        // tile counts 0..max_tiles
    int* cnt = plan_smem;                // sequences with nt == v
    int* base = cnt + NT;                // first rank of nt == v in the descending order
    int* cum = base + NT;                // first unit of the sequences with nt == v
    __shared__ int n_aligned, n_packed;
    int64_t* off_s = reinterpret_cast<int64_t*>(plan_smem + ((3 * NT + 1) & ~1));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int v = tid; v < NT; v += blockDim.x) cnt[v] = 0;
    if (kCache)
        for (int b = tid; b <= B; b += blockDim.x) off_s[b] = seq_offsets[b];
    if (tid == 0) {
        n_packed = 0;
        item_counter[0] = 0;   // next work item to hand out
        item_counter[1] = 0;   // CTAs finished
    }
    __syncthreads();
    const int64_t* __restrict__ off = kCache ? off_s : seq_offsets;
    auto length = [&](int b) -> int64_t {
        int64_t n = off[b + 1] - off[b];
        if (n < 0 || n > max_seqlen) {
            raise_error(kErrBadInput);
            n = n < 0 ? 0 : max_seqlen;
        }
        return n;
    };
    auto tiles_of = [&](int64_t n) -> int {
        return n > kTile ? static_cast<int>((n + kTile - 1) / kTile) : 0;   // 0: packed
    };
    // histogram of tile counts of the long sequences
    for (int b = tid; b < B; b += blockDim.x) {
        const int nt = tiles_of(length(b));
        if (nt > 0) atomicAdd(&cnt[nt], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int rank = 0, slots = 0;
        for (int v = max_tiles; v >= 1; --v) {
            base[v] = rank;
            cum[v] = slots;
            rank += cnt[v];
            slots += cnt[v] * v;
        }
        n_aligned = slots;
        for (int v = 0; v < NT; ++v) cnt[v] = 0;   // reused as fill counters
    }
    __syncthreads();
    // aligned units: one rank per sequence, then its nt consecutive slots,
    // tile nt-1 first
    for (int b = tid; b < B; b += blockDim.x) {
        const int64_t n = length(b);
        const int nt = tiles_of(n);
        if (nt == 0) continue;
        const int ubase = cum[nt] + atomicAdd(&cnt[nt], 1) * nt;
        const int64_t o = off[b];
        for (int k = 0; k < nt; ++k) {
            const int t = nt - 1 - k;
            const int slot = ubase + k;
            if (slot < max_units) {
                const int64_t q0 = o + static_cast<int64_t>(t) * kTile;
                const int64_t qe = q0 + kTile < o + n ? q0 + kTile : o + n;
                units[slot] = make_int4(static_cast<int>(q0), static_cast<int>(qe),
                                        static_cast<int>(o), (t + 1) | (nt << 11));
            }
        }
    }
    // packed units. The first non-empty short sequence of each 128-token start
    // bucket packs the short sequences of its bucket greedily in one pass;
    // each unit takes its slot with a shared-memory atomic as it closes.
    for (int b0 = warp * 32; b0 < B; b0 += nwarps * 32) {
        const int b = b0 + lane;
        bool first = false;
        int64_t bucket = 0;
        if (b < B) {
            const int64_t n = length(b);
            if (n > 0 && n <= kTile) {
                bucket = off[b] / kTile;
                first = true;
                for (int c = b - 1; c >= 0; --c) {   // nearest earlier non-empty sequence
                    if (off[c + 1] - off[c] == 0) continue;
                    first = (off[c] / kTile) != bucket || (off[c + 1] - off[c]) > kTile;
                    break;
                }
            }
        }
        if (!first) continue;
        // the open unit: tokens [ts0, te), sequence-start mask m
        int64_t ts0 = -1, te = -1;
        uint32_t m0 = 0u, m1 = 0u, m2 = 0u, m3 = 0u;
        auto close = [&]() {
            const int slot = n_aligned + atomicAdd(&n_packed, 1);
            if (slot < max_units) {
                units[slot] = make_int4(static_cast<int>(ts0), static_cast<int>(te),
                                        static_cast<int>(ts0), static_cast<int>(0x80000801u));
                starts[slot] = make_uint4(m0, m1, m2, m3);
            }
        };
        for (int c = b; c < B && off[c] / kTile == bucket; ++c) {
            const int64_t nc = length(c);
            if (nc == 0) continue;
            if (nc > kTile) break;                   // a long sequence ends the run
            const int64_t oc = off[c];
            if (ts0 >= 0 && oc + nc - ts0 > kTile) {
                close();
                ts0 = -1;
            }
            if (ts0 < 0) {
                ts0 = oc;
                m0 = m1 = m2 = m3 = 0u;
            }
            te = oc + nc;
            const int r = static_cast<int>(oc - ts0);
            const uint32_t bit = 1u << (r & 31);
            m0 |= (r >> 5) == 0 ? bit : 0u;
            m1 |= (r >> 5) == 1 ? bit : 0u;
            m2 |= (r >> 5) == 2 ? bit : 0u;
            m3 |= (r >> 5) == 3 ? bit : 0u;
        }
        if (ts0 >= 0) close();
    }
    __syncthreads();
    if (tid == 0) {
        const int total = n_aligned + n_packed;
        *unit_count = total < max_units ? total : max_units;
    }
    if (order_tab != nullptr && tid == 0) {
        // cnt[v] counts the sequences placed in bucket v again
        const int stride = max_tiles + 2;
        int items = 0;
        order_tab[max_tiles + 1] = 0;
        order_tab[stride + max_tiles + 1] = 0;
        for (int v = max_tiles; v >= 1; --v) {
            const int seqs = base[v] + cnt[v];
            items += order_h * seqs;
            order_tab[v] = seqs;
            order_tab[stride + v] = items;
            order_tab[2 * stride + v] = cum[v];
            order_tab[3 * stride + v] = base[v];
        }
        order_tab[0] = order_tab[1];
        order_tab[stride] = items;
        order_tab[2 * stride] = n_aligned;
        order_tab[3 * stride] = order_tab[1];
    }
}

__global__ void __launch_bounds__(1024)
plan_kernel(const int64_t* __restrict__ seq_offsets, int B, int64_t T, int max_seqlen,
            int max_tiles, int max_units, int4* __restrict__ units, uint4* __restrict__ starts,
            int* __restrict__ unit_count, int* __restrict__ item_counter, int order_h,
            int* __restrict__ order_tab) {
    extern __shared__ int plan_smem[];
    // let the attention kernel that follows start its set-up now (it waits
    // for this grid to complete before it reads the work list)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (B < kPlanSmemOffsets)
        plan_body<true>(seq_offsets, B, T, max_seqlen, max_tiles, max_units, units, starts,
                        unit_count, item_counter, plan_smem, order_h, order_tab);
    else
        plan_body<false>(seq_offsets, B, T, max_seqlen, max_tiles, max_units, units, starts,
                         unit_count, item_counter, plan_smem, order_h, order_tab);
}

}  // namespace hstu
