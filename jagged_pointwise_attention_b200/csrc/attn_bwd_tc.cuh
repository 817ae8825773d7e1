// attn_bwd_tc.cuh -- bf16 HSTU jagged causal attention backward on tcgen05.
//
// The gradients of out_i = (1/N) sum_{j<=i} silu(s_ij) v_j with
// s_ij = q_i.k_j + pos + time (the forward of the generative-recommenders
// HSTU attention; its README, "HSTU Ultra attention benchmark", names forward
// and backward kernels):
//     dv_j = sum_i p_ij dout_i                  p_ij  = silu(s_ij) / N
//     ds_ij = (dout_i . v_j) silu'(s_ij) / N    silu'(s) = sg (1 + s (1 - sg)), sg = sigmoid(s)
//     dq_i = sum_j ds_ij k_j,  dk_j = sum_i ds_ij q_i
//     dpos[min(i - j, P - 1)] and dtime[bucket(ts_i - ts_j)] sum the ds of their pairs.
//
// Persistent kernel over work items (key tile j, head h): the plan unit of
// query tile t (t + 1 key tiles) maps to key tile nt - 1 - t, whose item walks
// t + 1 query tiles. The items are sorted by that count, most first, and dealt
// to the CTAs in a snake (the order of turns reverses every round), which
// leaves every CTA within about one item of the mean; a plain round robin
// over the plan's list, where each sequence's items fall from nt steps to 1,
// gave some CTAs half again the mean on long batches. Key tile K_j and V_j stay
// in shared memory while the item walks its query tiles i = j .. nt - 1; Q_i
// streams through a two-stage TMA ring, dO_i through a two-stage ring (d = 64)
// or a single buffer (d = 128, for shared memory), reloaded as soon as its
// step's dV has been computed. Per step, with keys as TMEM lanes throughout:
//     S^T  = K_j Q_i^T      SS   -> TMEM cols [0, 128)
//     dP^T = V_j dO_i^T     SS   -> TMEM cols [128, 256)
//     pointwise: P^T (bf16) back into the S^T columns (the forward's in-place
//                packing), dS^T (bf16) into shared memory (128-byte swizzle)
//     dV_j += P^T dO_i      TS   (A from TMEM, dO_i MN-major) -> TMEM [256, 256 + D)
//     dK_j += dS^T Q_i      SS   (dS^T K-major, Q_i MN-major)  -> TMEM [256 + D, 256 + 2D)
//     dQ_i  = dS K_j        SS   (dS^T read MN-major, K_j MN-major) -> TMEM [128, 128 + D)
// and the pointwise warps read dQ_i out of TMEM (which frees its columns for
// the next dP^T) and add it into the fp32 dq with bulk tensor reductions,
// staged through the dS^T buffer (free once dQ_i is computed; the next step's
// dS^T stores wait until those stages have been read); after the item's last
// step they store dK_j and dV_j (fp32).
//
// Warp roles: 0-15 pointwise (four warps per TMEM lane quarter, one 32-column
// chunk of queries each: with four warps per scheduler one warp's TMEM, SFU
// and shared-memory latencies hide behind the others' arithmetic), 16 TMA
// producer, 17 MMA issuer and TMEM owner, 18 table warp (bias staging and
// table-gradient flushes, off the pointwise warps' path).
//
// Pointwise arithmetic per pair in fp32: s = S + pos + time; one tanh gives
// sg = 1/2 + tanh(s/2)/2, then p and ds without the factor 1/N, which is
// applied once to every gradient as it leaves the kernel. Two steps ahead the table warp
// stages a step's bias data in shared memory: the 255 position-table values
// the tile's diagonals read, the 128 query timestamps with each 32-column
// chunk's smallest and largest, and the head's time-table row. The time
// bucket is floor(log2(max(1, dt))) clamped to NB - 1 from a count of leading
// zeros; when every row of a warp sees one bucket at the chunk's smallest and
// largest query timestamp, the bucket is constant over the chunk (it is
// monotone in dt) and the per-pair bucket work is skipped.
// Table gradients without shared-memory atomics per pair: a warp sums ds
// along the diagonals of its 32 x 32 chunk by passing a running sum one lane
// down per column (lane l adds the pair (l, e) to the sum lane l - 1 held for
// (l - 1, e - 1)), so each diagonal's sum leaves through lane 31 or stays in
// the last column's lanes, into the warp's own diagonal buffer; the time
// gradient sums ds per row over runs of one bucket and adds the runs into the
// warp's own bucket slots, merging lanes with equal buckets first. Once every
// pointwise warp is done with a step, the table warp sums the sixteen warps'
// buffers per tile diagonal and per bucket and adds them to the global tables
// with atomics. Bias data and sums have two buffers, by step parity, so the
// table warp works on step m (and stages step m + 2) while step m + 1 runs.
//
// Every wait is bounded; a wait that runs out raises kErrTimeout, the other
// roles notice through a shared abort flag, and the CTA drains its own copies
// and MMAs before it frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

struct BwdArgs {
    const int4* units;          // plan: (q0, q_end, k0, nk | nt << 11 | packed << 31)
    const int* unit_count;
    int max_units;
    const uint4* starts;        // plan: per packed unit, rows where a sequence begins
    int H;
    int64_t T;
    const int64_t* ts;          // [T], or null without the time term
    const float* pos;           // [H, P] or null
    int P;
    const float* tb;            // [H, NB], or null without the time term
    int NB;
    float inv_n;
    float* dq;                  // [T, H, D] fp32: zeroed before, accumulated
    float* dk;                  // [T, H, D] fp32: written
    float* dv;                  // [T, H, D] fp32: written
    float* dpos;                // [H, P]: zeroed before, accumulated (with pos)
    float* dtime;               // [H, NB]: zeroed before, accumulated (with the time term)
    const int* order;           // plan: item-order table, four rows of max_tiles + 2 ints
    int max_tiles;
};

template <int D>
struct BwdCfg {
    static_assert(D == 64 || D == 128, "head dimension");
    static constexpr int kKB = D / 64;                      // 64-column blocks of a tile
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kPointwiseWarps = 16;
    static constexpr int kPointwiseThreads = 32 * kPointwiseWarps;
    static constexpr int kWarpTMA = kPointwiseWarps, kWarpMMA = kPointwiseWarps + 1;
    static constexpr int kWarpTable = kPointwiseWarps + 2;
    // 19 warps: at most five per scheduler, the same 96-register cap as 18
    static constexpr int kThreads = 32 * (kPointwiseWarps + 3);
    static constexpr uint32_t kColS = 0, kColP = 128, kColV = 256, kColK = 256 + D;
};

template <int D>
struct BwdSmem {
    using C = BwdCfg<D>;
    static constexpr int kDOStages = D == 128 ? 1 : 2;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + C::kTileBytes;
    static constexpr int kOffQ = kOffV + C::kTileBytes;            // [2 stages]
    static constexpr int kOffDO = kOffQ + 2 * C::kTileBytes;       // [kDOStages]
    static constexpr int kOffDS = kOffDO + kDOStages * C::kTileBytes;  // dS^T: 2 blocks of 64 queries
    // a step's bias data and table sums, two buffers by step parity
    static constexpr int kOffPosW = kOffDS + 2 * 16384;            // [2][256] floats: pos of the tile diagonals
    static constexpr int kOffQts = kOffPosW + 2 * 1024;            // [2][128] query timestamps
    static constexpr int kOffCmm = kOffQts + 2 * 1024;             // [2][4 chunks]: min, max timestamp
    static constexpr int kOffTb = kOffCmm + 2 * 64;                // [2][64] floats: the head's time table
    static constexpr int kOffDiag = kOffTb + 2 * 256;              // [2][16 warps][64] diagonal sums
    static constexpr int kOffTslot = kOffDiag + 2 * 16 * 64 * 4;   // [2][16 warps][64] bucket sums
    static constexpr int kOffBar = kOffTslot + 2 * 16 * 64 * 4;
    static constexpr int kNumBars = 21;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;                   // 1 KB alignment slack
    static_assert(kAlloc <= 227 * 1024, "shared memory per block");
};

enum {
    kBwKVFull = 0,      // K_j and V_j landed
    kBwKVFree = 1,      // MMA commit after the item's last MMA that reads K_j or V_j
    kBwQFull = 2,       // +stage: Q_i landed
    kBwQFree = 4,       // +stage: MMA commit after dK_i (the last MMA that reads Q_i)
    kBwDOFull = 6,      // +stage: dO_i landed
    kBwDOFree = 8,      // +stage: MMA commit after dV_i (the last MMA that reads dO_i)
    kBwSFull = 10,      // MMA commit: S^T and dP^T of the step are in TMEM
    kBwPFull = 11,      // the pointwise threads: P^T in TMEM, dS^T in shared memory
    kBwDQFull = 12,     // MMA commit after dQ (dV and dK before it have completed too)
    kBwDQFree = 13,     // the pointwise threads have read dQ out of TMEM
    kBwAccFree = 14,    // the pointwise threads have read dK_j and dV_j out of TMEM
    kBwDSFree = 15,     // the pointwise threads' dQ staging in the dS^T buffer has been read
    kBwPwDone = 16,     // +parity of the step: the pointwise threads' table sums are complete
    kBwReady = 18,      // +parity of the step: the table warp staged its bias data, cleared its sums
    kBwDrain = 20,      // the MMA issuer's last commit
};

// A work item of the backward: key tile [kt0, key_end) of head h; its query
// tiles start at qt0 + 128 s for s < nq, queries end at q_end.
struct BwdItem {
    int kt0, key_end, qt0, q_end, nq, h, u;
    bool packed;
};

// Item w. The plan lists a sequence's units consecutively, tile nt - 1
// first (nk = nt - k for the k-th); items run sequence by sequence, then
// head, then unit, as in the forward.
__device__ __forceinline__ BwdItem bwd_item(const BwdArgs& a, int w) {
    const int u1 = w / a.H;
    const int4 d1 = a.units[u1];
    const int nk1 = d1.w & 0x7ff, nt = (d1.w >> 11) & 0x7ff;
    const int ubase = u1 - (nt - nk1);
    const int r = w - a.H * ubase;
    const int h = r / nt;
    const int u = ubase + (r - h * nt);
    const int4 wu = u == u1 ? d1 : a.units[u];
    BwdItem it;
    it.h = h;
    it.u = u;
    it.packed = (wu.w >> 31) & 1;
    if (it.packed) {
        it.kt0 = wu.x;
        it.key_end = wu.y;
        it.qt0 = wu.x;
        it.q_end = wu.y;
        it.nq = 1;
    } else {
        const int nk = wu.w & 0x7ff;
        const int seq_end = a.units[ubase].y;        // the last query tile's end
        it.kt0 = wu.z + kTile * (nt - nk);
        it.key_end = min(it.kt0 + kTile, seq_end);
        it.qt0 = it.kt0;
        it.q_end = seq_end;
        it.nq = nk;
    }
    return it;
}

// The item of a CTA's k-th turn, or -1 past the last. Items are taken in
// order of cost, most steps first (nq = nk of the unit: c steps for the
// aligned items of cost c, ranked by sequence, then head; then the packed
// items, one step each, in list order), and dealt to the CTAs in a snake:
// turn k takes position k G + b for even k, k G + G - 1 - b for odd k. The
// plan's table gives, per cost v, the sequences with nt >= v (sge), the
// aligned items of cost >= v (ige), the first unit (cum) and rank (base) of
// the sequences with nt == v.
__device__ __forceinline__ int bwd_item_index(const BwdArgs& a, int k, int n_items) {
    const int G = gridDim.x, b = blockIdx.x;
    const int64_t p64 = static_cast<int64_t>(k) * G + ((k & 1) ? G - 1 - b : b);
    if (p64 >= n_items) return -1;
    const int p = static_cast<int>(p64);
    const int stride = a.max_tiles + 2;
    const int* sge = a.order;
    const int* ige = a.order + stride;
    const int* cum = a.order + 2 * stride;
    const int* base = a.order + 3 * stride;
    if (p >= __ldg(ige + 1)) return p;               // packed: list order
    // cost c: ige[c] > p >= ige[c + 1]
    int lo = 1, hi = a.max_tiles;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(ige + mid) > p) lo = mid;
        else hi = mid - 1;
    }
    const int c = lo;
    const int idx = p - __ldg(ige + c + 1);
    const int rho = idx / a.H, h = idx - rho * a.H;
    // tile count v of the sequence of rank rho: sge[v] > rho >= sge[v + 1]
    lo = c;
    hi = a.max_tiles;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(sge + mid) > rho) lo = mid;
        else hi = mid - 1;
    }
    const int v = lo;
    const int ubase = __ldg(cum + v) + (rho - __ldg(base + v)) * v;
    const int w = a.H * ubase + h * v + (v - c);     // the unit with nk = c, head h
    return w < n_items ? w : -1;
}

// Smallest row p > r of a packed tile at which a sequence begins (bit p of
// the 128-bit mask m), or `len` if none.
__device__ __forceinline__ int next_start_after(const uint4 m, int r, int len) {
    const uint32_t w[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int lo = 32 * k;
        if (r + 1 > lo + 31) continue;
        uint32_t bits = w[k];
        if (r + 1 > lo) bits &= ~0u << (r + 1 - lo);
        if (bits) return min(lo + __ffs(bits) - 1, len);
    }
    return len;
}

__device__ __forceinline__ int time_bucket_of(long long dt, int NB) {
    const unsigned long long x = dt < 1 ? 1ull : static_cast<unsigned long long>(dt);
    return min(63 - __clzll(x), NB - 1);
}

// Sum of v over the lanes of a warp (every lane gets it).
__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Add every lane's (bucket b, value v) with has set into the warp's own
// bucket slots: lanes with equal buckets are summed first, one slot update
// per distinct bucket (warp-uniform; every lane must call it).
__device__ __forceinline__ void warp_bucket_add(float* slots, bool has, int b, float v) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    unsigned pend = __ballot_sync(0xffffffffu, has);
    while (pend) {
        const int leader = __ffs(pend) - 1;
        const int bb = __shfl_sync(0xffffffffu, b, leader);
        const bool mine = ((pend >> lane) & 1u) && b == bb;
        const float x = warp_allsum(mine ? v : 0.f);
        if (lane == leader) slots[bb] += x;
        pend &= ~__ballot_sync(0xffffffffu, mine);
    }
    __syncwarp();
}

// warp_bucket_add as a call, for the rare per-pair flushes of TM 2 (keeps the
// unrolled pair loop small).
__device__ __noinline__ void warp_bucket_add_call(float* slots, bool has, int b, float v) {
    warp_bucket_add(slots, has, b, v);
}

// Shared-memory store by lane 31 only, as a predicated instruction (no branch
// in the straight-line pair loop).
__device__ __forceinline__ void st_shared_if_lane31(float* p, float v, int lane) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.eq.u32 q, %2, 31;\n\t@q st.shared.f32 [%0], %1;\n\t}" ::"r"(
            smem_u32(p)),
        "f"(v), "r"(lane));
}

// The pointwise work of one 32-column chunk for one key row (lane), in two
// halves of 16 columns: s, p = silu(s) and ds = dp silu'(s), both without
// the 1/N (applied to the sums at the end); P^T packed as bf16 pairs back
// into TMEM in place of the chunk's S^T columns (c0 .. c0 + 15) and dS^T
// into the 128-byte swizzled row `ds_row` of the chunk's 64-query block
// (16-byte units u0 .. u0 + 3); the chunk's diagonal sums of ds into the
// warp's area `diag` (entry 31 + e - lane for pair (lane, e); entry 63 is
// scratch); the time gradient by bucket into the warp's slots. Rows see
// buckets b0 .. b0 + nbk - 1 over the chunk, at most `most` for any row of
// the warp. TM 0: one bucket per row (most == 1); TM 1: up to four (summed in
// registers in the pair loop); TM 2: any, as runs of one bucket per row over
// the kept pairs (the bucket is monotone in the query timestamp, so a row
// sees few runs), each run added into the warp's slots when any lane's run
// ends. Straight-line code over the pairs for TM 0 and 1. Before its first
// dS^T store the warp waits for phase `ds_parity` of `ds_free` (the previous
// step's dQ staging in the same buffer has been read), unless ds_parity < 0;
// returns false if that wait gave up.
template <int TM>
__device__ __forceinline__ bool bwd_chunk(uint32_t tS_c, uint32_t tP_c, uint8_t* ds_row, int u0,
                                          int c0, int r, int lo, int span, const float* s_posw,
                                          const long long* s_qts, const float* s_tb, long long tk,
                                          int NB, bool has_time, int b0, int nbk, int most,
                                          float* diag, float* tslot, uint64_t* ds_free,
                                          int ds_parity, volatile int* abort_flag) {
    const int lane = threadIdx.x & 31;
    bool ok = true;
    const float tb0 = has_time ? s_tb[b0] : 0.f;
    float dsum = 0.f;                       // running diagonal sum, passed one lane down
    float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;   // TM 0 / 1: buckets b0 .. b0 + 3
    float run = 0.f;                        // TM 2: the row's current bucket run
    int run_b = -1;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t sv[16], pv[16], pk_p[8], pk_ds[8];
        tmem_ld16x2(tS_c + 16 * h2, tP_c + 16 * h2, sv, pv);
        float pe = 0.f, de = 0.f;
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
            const int e = 16 * h2 + e2;
            const int c = c0 + e;
            const bool keep = static_cast<unsigned>(c - lo) < static_cast<unsigned>(span);
            float sc = __uint_as_float(sv[e2]) + s_posw[c - r + 127];
            int j = 0;
            if (TM == 0) {
                sc += tb0;
            } else {
                const int bk = time_bucket_of(s_qts[c] - tk, NB);
                sc += s_tb[bk];
                j = bk - b0;
            }
            const float sg = fmaf(0.5f, tanh_approx(0.5f * sc), 0.5f);
            const float p = keep ? sc * sg : 0.f;
            const float g = fmaf(sg * sc, 1.f - sg, sg);
            const float ds = keep ? __uint_as_float(pv[e2]) * g : 0.f;
            // the diagonal through (lane, e) continues from (lane - 1, e - 1);
            // it leaves the chunk at lane 31 (entry e) or at column 31 (below)
            const float up = __shfl_up_sync(0xffffffffu, dsum, 1);
            dsum = (lane == 0 ? 0.f : up) + ds;
            st_shared_if_lane31(diag + e, dsum, lane);
            if (TM == 0) {
                t0 += ds;
            } else if (TM == 1) {
                if (j == 0) t0 += ds;
                if (j == 1) t1 += ds;
                if (j == 2) t2 += ds;
                if (j == 3) t3 += ds;
            } else {
                const int bk = j + b0;
                const bool ends = keep && bk != run_b && run_b >= 0;
                if (__any_sync(0xffffffffu, ends)) warp_bucket_add_call(tslot, ends, run_b, run);
                const bool starts = keep && bk != run_b;
                run = starts ? ds : run + ds;
                run_b = starts ? bk : run_b;
            }
            if (e2 & 1) {
                pk_p[e2 >> 1] = pack_bf16x2(pe, p);
                pk_ds[e2 >> 1] = pack_bf16x2(de, ds);
            } else {
                pe = p;
                de = ds;
            }
        }
        // the half's P^T words over S^T columns this warp has already read
        tmem_st8_async(tS_c + 8 * h2, pk_p);
        if (h2 == 0 && ds_parity >= 0)
            ok = warp_wait(ds_free, static_cast<uint32_t>(ds_parity), abort_flag);
#pragma unroll
        for (int j = 0; j < 2; ++j)
            *reinterpret_cast<uint4*>(ds_row + (((u0 + 2 * h2 + j) ^ (r & 7)) << 4)) =
                make_uint4(pk_ds[4 * j], pk_ds[4 * j + 1], pk_ds[4 * j + 2], pk_ds[4 * j + 3]);
    }
    diag[lane < 31 ? 62 - lane : 63] = dsum;
    __syncwarp();
    if (has_time) {
        if (TM == 0) {
            warp_bucket_add(tslot, true, b0, t0);
        } else if (TM == 1) {
            warp_bucket_add(tslot, true, b0, t0);
            warp_bucket_add(tslot, nbk > 1, b0 + 1, t1);
            warp_bucket_add(tslot, nbk > 2, b0 + 2, t2);
            warp_bucket_add(tslot, nbk > 3, b0 + 3, t3);
        } else {
            warp_bucket_add(tslot, run_b >= 0, run_b, run);
        }
    }
    return ok;
}

// A step of the backward: query tile q0 of key tile kt0, head h.
struct BwdStep {
    int q0, kt0, h;
    bool valid;
};

// Walks a CTA's steps in order: the items of its turns k = 0, 1, ..., each
// over its query tiles.
struct BwdCursor {
    int k, s;
    BwdItem I;
    bool valid;
    __device__ __forceinline__ void start(const BwdArgs& a, int k0, int n_items) {
        k = k0;
        s = 0;
        const int w = bwd_item_index(a, k, n_items);
        valid = w >= 0;
        if (valid) I = bwd_item(a, w);
    }
    __device__ __forceinline__ void next(const BwdArgs& a, int n_items) {
        if (!valid) return;
        if (++s < I.nq) return;
        start(a, k + 1, n_items);
    }
    __device__ __forceinline__ BwdStep step() const {
        return BwdStep{valid ? I.qt0 + s * kTile : 0, valid ? I.kt0 : 0, valid ? I.h : 0, valid};
    }
};

// Bias data of step st into one buffer, by one warp: the position table at
// the tile's 255 diagonals (zero without the position term), the 128 query
// timestamps with each 32-query chunk's smallest and largest, and the head's
// time-table row.
__device__ __forceinline__ void bwd_stage_tables(const BwdArgs& a, const BwdStep& st, float* posw,
                                                 long long* qts, long long* cmm, float* tbrow,
                                                 bool has_pos, bool has_time) {
    if (!st.valid) return;
    const int lane = threadIdx.x & 31;
    float pv[8], tv[2];
    long long tsv[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = lane + 32 * k;
        const int rel = st.q0 - st.kt0 - 127 + i;
        pv[k] = (has_pos && i < 255)
                    ? __ldg(a.pos + static_cast<int64_t>(st.h) * a.P + min(max(rel, 0), a.P - 1))
                    : 0.f;
    }
    if (has_time) {
#pragma unroll
        for (int k = 0; k < 2; ++k)
            tv[k] = __ldg(a.tb + static_cast<int64_t>(st.h) * a.NB + min(lane + 32 * k, a.NB - 1));
#pragma unroll
        for (int k = 0; k < 4; ++k)
            tsv[k] = __ldg(a.ts + min(static_cast<int64_t>(st.q0) + lane + 32 * k, a.T - 1));
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (lane + 32 * k < 255) posw[lane + 32 * k] = pv[k];
    if (has_time) {
#pragma unroll
        for (int k = 0; k < 2; ++k) tbrow[lane + 32 * k] = tv[k];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            qts[lane + 32 * k] = tsv[k];
            long long mn = tsv[k], mx = tsv[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            if (lane == 0) {
                cmm[2 * k] = mn;
                cmm[2 * k + 1] = mx;
            }
        }
    }
}

// Step st's table sums from one buffer into the global tables, by one warp:
// each tile diagonal (c - r + 127) collects the diagonal sums of the warps
// whose 32 x 32 chunk it crosses (warp 4 cq + qd holds diagonal
// 32 cq - 32 qd + 96 + i at entry i, i = 0 .. 62); each bucket sums the
// warps' slots, which are cleared for the buffer's next step.
__device__ __forceinline__ void bwd_flush_tables(const BwdArgs& a, const BwdStep& st, const float* diag,
                                                 float* tslot, bool has_pos, bool has_time) {
    if (!st.valid) return;
    const int lane = threadIdx.x & 31;
    if (has_pos) {
#pragma unroll 2
        for (int k = 0; k < 8; ++k) {
            const int t = lane + 32 * k;
            if (t >= 255) continue;
            float v = 0.f;
#pragma unroll
            for (int ww = 0; ww < 16; ++ww) {
                const int i = t - ((ww >> 2) * 32 - (ww & 3) * 32 + 96);
                if (i >= 0 && i <= 62) v += diag[ww * 64 + i];
            }
            if (v != 0.f) {
                const int rel = st.q0 - st.kt0 + t - 127;
                atomicAdd(a.dpos + static_cast<int64_t>(st.h) * a.P + min(max(rel, 0), a.P - 1),
                          v * a.inv_n);
            }
        }
    }
    if (has_time) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int bk = lane + 32 * k;
            float v = 0.f;
#pragma unroll
            for (int ww = 0; ww < 16; ++ww) {
                v += tslot[ww * 64 + bk];
                tslot[ww * 64 + bk] = 0.f;
            }
            if (v != 0.f && bk < a.NB)
                atomicAdd(a.dtime + static_cast<int64_t>(st.h) * a.NB + bk, v * a.inv_n);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
attn_bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
    using C = BwdCfg<D>;
    using L = BwdSmem<D>;
    constexpr int SD = L::kDOStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
    float* s_posw = reinterpret_cast<float*>(smem + L::kOffPosW);
    long long* s_qts = reinterpret_cast<long long*>(smem + L::kOffQts);
    long long* s_cmm = reinterpret_cast<long long*>(smem + L::kOffCmm);   // [4][2]
    float* s_tb = reinterpret_cast<float*>(smem + L::kOffTb);
    float* s_diag = reinterpret_cast<float*>(smem + L::kOffDiag);
    float* s_tslot = reinterpret_cast<float*>(smem + L::kOffTslot);
    const int n_items = min(*a.unit_count, a.max_units) * a.H;
    const bool has_pos = a.pos != nullptr;
    const bool has_time = a.ts != nullptr && a.tb != nullptr;

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(&bars[kBwKVFull], 1);
        mbar_init(&bars[kBwKVFree], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBwQFull + s], 1);
            mbar_init(&bars[kBwQFree + s], 1);
            mbar_init(&bars[kBwDOFull + s], 1);
            mbar_init(&bars[kBwDOFree + s], 1);
        }
        mbar_init(&bars[kBwSFull], 1);
        mbar_init(&bars[kBwPFull], C::kPointwiseThreads);
        mbar_init(&bars[kBwDQFull], 1);
        mbar_init(&bars[kBwDQFree], C::kPointwiseThreads);
        mbar_init(&bars[kBwAccFree], C::kPointwiseThreads);
        mbar_init(&bars[kBwDSFree], C::kPointwiseThreads);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[kBwPwDone + b], C::kPointwiseThreads);
            mbar_init(&bars[kBwReady + b], 32);
        }
        mbar_init(&bars[kBwDrain], 1);
        mbar_fence_init();
    }
    for (int i = tid; i < 2 * 16 * 64; i += blockDim.x) s_diag[i] = 0.f;
    for (int i = tid; i < 2 * 16 * 64; i += blockDim.x) s_tslot[i] = 0.f;
    if (warp == C::kWarpMMA) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::kWarpTMA) {
        // ------------------------------------------------------------ TMA producer
        int kv_loads = 0, n = 0, nd = 0;   // K/V loads; Q loads; dO loads issued
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            bool ok = true;
            for (int k = 0, w; ok && (w = bwd_item_index(a, k, n_items)) >= 0; ++k) {
                const BwdItem I = bwd_item(a, w);
                if (kv_loads > 0 && !mbar_wait(&bars[kBwKVFree], (kv_loads - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars[kBwKVFull], 2 * C::kTileBytes);
#pragma unroll
                for (int kb = 0; kb < C::kKB; ++kb) {
                    tma_load_2d(smem + L::kOffK + kb * 16384, &tmK, &bars[kBwKVFull],
                                I.h * D + kb * 64, I.kt0);
                    tma_load_2d(smem + L::kOffV + kb * 16384, &tmV, &bars[kBwKVFull],
                                I.h * D + kb * 64, I.kt0);
                }
                ++kv_loads;
                for (int s = 0; s < I.nq; ++s) {
                    const int q0 = I.qt0 + s * kTile;
                    const int st = n & 1;
                    if (n >= 2 && !mbar_wait(&bars[kBwQFree + st], ((n >> 1) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[kBwQFull + st], C::kTileBytes);
#pragma unroll
                    for (int kb = 0; kb < C::kKB; ++kb)
                        tma_load_2d(smem + L::kOffQ + st * C::kTileBytes + kb * 16384, &tmQ,
                                    &bars[kBwQFull + st], I.h * D + kb * 64, q0);
                    ++n;
                    const int sd = nd % SD;
                    if (nd >= SD && !mbar_wait(&bars[kBwDOFree + sd], ((nd / SD) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[kBwDOFull + sd], C::kTileBytes);
#pragma unroll
                    for (int kb = 0; kb < C::kKB; ++kb)
                        tma_load_2d(smem + L::kOffDO + sd * C::kTileBytes + kb * 16384, &tmDO,
                                    &bars[kBwDOFull + sd], I.h * D + kb * 64, q0);
                    ++nd;
                }
            }
            // drain: every copy this thread started has landed before the CTA ends
            if (kv_loads > 0 && !mbar_wait(&bars[kBwKVFull], (kv_loads - 1) & 1, nullptr))
                raise_error(kErrTimeout);
            for (int st = 0; st < 2; ++st) {
                const int c = n > st ? (n - st + 1) / 2 : 0;
                if (c > 0 && !mbar_wait(&bars[kBwQFull + st], (c - 1) & 1, nullptr))
                    raise_error(kErrTimeout);
            }
            for (int sd = 0; sd < SD; ++sd) {
                const int c = nd > sd ? (nd - sd + SD - 1) / SD : 0;
                if (c > 0 && !mbar_wait(&bars[kBwDOFull + sd], (c - 1) & 1, nullptr))
                    raise_error(kErrTimeout);
            }
        }
        __syncwarp();
    } else if (warp == C::kWarpMMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // K-major x K-major
            constexpr uint32_t idesc_kb = idesc_bf16_f32(128, D, 0, 1);    // A K-major, B MN-major
            constexpr uint32_t idesc_q = idesc_bf16_f32(128, D, 1, 1);     // both MN-major
            constexpr uint32_t kStageDesc = static_cast<uint32_t>(C::kTileBytes) >> 4;
            const uint32_t sK = smem_u32(smem + L::kOffK), sV = smem_u32(smem + L::kOffV);
            const uint32_t sQ = smem_u32(smem + L::kOffQ), sDO = smem_u32(smem + L::kOffDO);
            const uint32_t sDS = smem_u32(smem + L::kOffDS);
            const uint64_t dK_k = desc_kmajor_sw128(sK), dV_k = desc_kmajor_sw128(sV);
            const uint64_t dK_mn = desc_mnmajor_sw128(sK, 16384);
            const uint64_t dS_k = desc_kmajor_sw128(sDS), dS_mn = desc_mnmajor_sw128(sDS, 16384);
            int nitem = 0, n = 0;
            bool ok = true;
            for (int w; ok && (w = bwd_item_index(a, nitem, n_items)) >= 0; ++nitem) {
                const BwdItem I = bwd_item(a, w);
                if (!mbar_wait(&bars[kBwKVFull], nitem & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                for (int s = 0; s < I.nq; ++s, ++n) {
                    const int st = n & 1, sd = n % SD;
                    const uint64_t qs = static_cast<uint64_t>(st * kStageDesc);
                    const uint64_t ds = static_cast<uint64_t>(sd * kStageDesc);
                    const uint64_t dQ_k = desc_kmajor_sw128(sQ) + qs;
                    const uint64_t dQ_mn = desc_mnmajor_sw128(sQ, 16384) + qs;
                    const uint64_t dO_k = desc_kmajor_sw128(sDO) + ds;
                    const uint64_t dO_mn = desc_mnmajor_sw128(sDO, 16384) + ds;
                    // S^T into its columns once the previous step's dV (which
                    // read P^T there) has completed
                    if (!mbar_wait(&bars[kBwQFull + st], (n >> 1) & 1, abort_flag) ||
                        (n > 0 && !mbar_wait(&bars[kBwDQFull], (n - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        umma_bf16_ss(tmem + C::kColS, dK_k + off, dQ_k + off, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    // dP^T into its columns once dO_i has landed and the
                    // previous step's dQ was read out
                    if (!mbar_wait(&bars[kBwDOFull + sd], (n / SD) & 1, abort_flag) ||
                        (n > 0 && !mbar_wait(&bars[kBwDQFree], (n - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        umma_bf16_ss(tmem + C::kColP, dV_k + off, dO_k + off, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&bars[kBwSFull]);
                    if (!mbar_wait(&bars[kBwPFull], n & 1, abort_flag) ||
                        (s == 0 && nitem > 0 &&
                         !mbar_wait(&bars[kBwAccFree], (nitem - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // dV_j += P^T dO_i: queries 16kk..16kk+15 at P^T columns
                    // 32 (kk / 2) + 8 (kk % 2)
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        umma_bf16_ts(tmem + C::kColV, tmem + C::kColS + (kk >> 1) * 32 + (kk & 1) * 8,
                                     dO_mn + static_cast<uint64_t>((kk * 2048) >> 4), idesc_kb,
                                     (s == 0 && kk == 0) ? 0u : 1u);
                    umma_commit(&bars[kBwDOFree + sd]);
                    // dK_j += dS^T Q_i
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        umma_bf16_ss(tmem + C::kColK, dS_k + off,
                                     dQ_mn + static_cast<uint64_t>((kk * 2048) >> 4), idesc_kb,
                                     (s == 0 && kk == 0) ? 0u : 1u);
                    }
                    umma_commit(&bars[kBwQFree + st]);
                    // dQ_i = dS K_j (keys 16kk..16kk+15 are rows of dS^T and of K_j)
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        umma_bf16_ss(tmem + C::kColP, dS_mn + static_cast<uint64_t>((kk * 2048) >> 4),
                                     dK_mn + static_cast<uint64_t>((kk * 2048) >> 4), idesc_q,
                                     kk > 0 ? 1u : 0u);
                    umma_commit(&bars[kBwDQFull]);
                    if (s == I.nq - 1) umma_commit(&bars[kBwKVFree]);
                }
            }
            umma_commit(&bars[kBwDrain]);
            if (!mbar_wait(&bars[kBwDrain], 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if (warp == C::kWarpTable) {
        // ------------------------------------------------------------ table warp
        // Step m uses buffer m & 1. The first two steps are staged up front;
        // once the pointwise threads are done with step m, its sums go into
        // the global tables and step m + 2 is staged into the same buffer.
        BwdCursor st, fl;
        st.start(a, 0, n_items);
        fl = st;
        for (int b = 0; b < 2; ++b) {
            bwd_stage_tables(a, st.step(), s_posw + b * 256, s_qts + b * 128, s_cmm + b * 8,
                             s_tb + b * 64, has_pos, has_time);
            mbar_arrive(&bars[kBwReady + b]);
            st.next(a, n_items);
        }
        for (int m = 0; fl.valid; ++m) {
            const int b = m & 1;
            if (!warp_wait(&bars[kBwPwDone + b], (m >> 1) & 1, abort_flag)) break;
            bwd_flush_tables(a, fl.step(), s_diag + b * 1024, s_tslot + b * 1024, has_pos, has_time);
            bwd_stage_tables(a, st.step(), s_posw + b * 256, s_qts + b * 128, s_cmm + b * 8,
                             s_tb + b * 64, has_pos, has_time);
            mbar_arrive(&bars[kBwReady + b]);
            st.next(a, n_items);
            fl.next(a, n_items);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ pointwise stage
        const int qd = warp & 3, cq = warp >> 2;            // TMEM lane quarter, column chunk
        const int r = qd * 32 + lane;                       // key row (S^T) / query row (dQ)
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::kColS, tP = tmem + lane_base + C::kColP;
        const uint32_t tV = tmem + lane_base + C::kColV, tK = tmem + lane_base + C::kColK;
        uint8_t* ds_row = smem + L::kOffDS + r * 128;

        int n = 0;
        bool ok = true;
        for (int k = 0, w; ok && (w = bwd_item_index(a, k, n_items)) >= 0; ++k) {
            const BwdItem I = bwd_item(a, w);
            const int ktok = I.kt0 + r;
            const bool kvalid = ktok < I.key_end;
            // end (exclusive) of the sequence of key row r
            const int kend = I.packed ? I.kt0 + next_start_after(a.starts[I.u], r, I.key_end - I.kt0)
                                      : I.q_end;
            const long long tk = (has_time && kvalid) ? __ldg(a.ts + ktok) : 0ll;
            for (int s = 0; s < I.nq; ++s, ++n) {
                const int q0 = I.qt0 + s * kTile;
                const int lo = ktok - q0;                    // first kept query column
                const int span = kvalid ? max(kend - q0 - lo, 0) : 0;   // kept: lo <= c < lo + span
                const int b = n & 1;                         // the step's table buffers
                if (!warp_wait(&bars[kBwReady + b], (n >> 1) & 1, abort_flag) ||
                    !warp_wait(&bars[kBwSFull], n & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    const float* posw = s_posw + b * 256;
                    const long long* qts = s_qts + b * 128;
                    const long long* cmm = s_cmm + b * 8;
                    const float* tbrow = s_tb + b * 64;
                    // the chunk's diagonal sums: entry i is tile diagonal (c - r + 127)
                    // 32 cq - 32 qd + 96 + i, i = 0 .. 62
                    float* my_diag = s_diag + b * 1024 + warp * 64;
                    float* my_tslot = s_tslot + b * 1024 + warp * 64;
                    const int ds_par = n > 0 ? (n - 1) & 1 : -1;
                    const int c0 = cq * 32;
                    // buckets each row sees over the chunk: b0 .. b0 + nbk - 1
                    int b0 = 0, nbk = 1;
                    if (has_time) {
                        b0 = time_bucket_of(cmm[2 * cq] - tk, a.NB);
                        nbk = time_bucket_of(cmm[2 * cq + 1] - tk, a.NB) - b0 + 1;
                    }
                    const int most = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(nbk));
                    uint8_t* dsr = ds_row + (c0 >> 6) * 16384;
                    const int u0 = (c0 & 63) >> 3;
                    bool chunk_ok;
                    if (most == 1)
                        chunk_ok = bwd_chunk<0>(tS + c0, tP + c0, dsr, u0, c0, r, lo, span, posw, qts,
                                                tbrow, tk, a.NB, has_time, b0, nbk, most, my_diag,
                                                my_tslot, &bars[kBwDSFree], ds_par, abort_flag);
                    else if (most <= 4)
                        chunk_ok = bwd_chunk<1>(tS + c0, tP + c0, dsr, u0, c0, r, lo, span, posw, qts,
                                                tbrow, tk, a.NB, has_time, b0, nbk, most, my_diag,
                                                my_tslot, &bars[kBwDSFree], ds_par, abort_flag);
                    else
                        chunk_ok = bwd_chunk<2>(tS + c0, tP + c0, dsr, u0, c0, r, lo, span, posw, qts,
                                                tbrow, tk, a.NB, has_time, b0, nbk, most, my_diag,
                                                my_tslot, &bars[kBwDSFree], ds_par, abort_flag);
                    if (!chunk_ok) {
                        ok = false;
                        break;
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                fence_proxy_async_smem();
                mbar_arrive(&bars[kBwPFull]);
                mbar_arrive(&bars[kBwPwDone + b]);
                // dQ_i of the step into dq
                if (!warp_wait(&bars[kBwDQFull], n & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    // this warp's D/4 columns of dQ_i leave TMEM first, so the
                    // next dP^T can be computed there; then they go through the
                    // dS^T buffer (its MMAs have completed) as 32 x 16 fp32
                    // blocks (64-byte swizzle), added into dq with bulk tensor
                    // reductions; rows of queries outside the sequence are zero
                    // (every ds of theirs is)
                    uint32_t v[D / 64][16];
                    if constexpr (D == 128)
                        tmem_ld16x2(tP + cq * 32, tP + cq * 32 + 16, v[0], v[1]);
                    else
                        tmem_ld16(tP + cq * 16, v[0]);
                    tc_fence_before();
                    mbar_arrive(&bars[kBwDQFree]);
                    uint8_t* buf = smem + L::kOffDS + warp * 2048;
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb) {
                        if (cb > 0) {
                            if (lane == 0) bulk_wait_group_read<0>();
                            __syncwarp();
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            *reinterpret_cast<float4*>(buf + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
                                make_float4(__uint_as_float(v[cb][4 * u]) * a.inv_n,
                                            __uint_as_float(v[cb][4 * u + 1]) * a.inv_n,
                                            __uint_as_float(v[cb][4 * u + 2]) * a.inv_n,
                                            __uint_as_float(v[cb][4 * u + 3]) * a.inv_n);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_reduce_add_2d(&tmDQ, buf, I.h * D + cq * (D / 4) + cb * 16, q0 + qd * 32);
                            bulk_commit_group();
                        }
                    }
                    if (lane == 0) bulk_wait_group_read<0>();
                    __syncwarp();
                    mbar_arrive(&bars[kBwDSFree]);
                }
                if (s == I.nq - 1) {
                    // the item's dV_j and dK_j (their MMAs completed before dQ's)
                    const int64_t row = (static_cast<int64_t>(ktok) * a.H + I.h) * D + cq * (D / 4);
#pragma unroll 1
                    for (int cb = 0; cb < D / 64; ++cb) {
                        uint32_t v[16];
                        tmem_ld16(tV + cq * (D / 4) + cb * 16, v);
                        if (kvalid) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<float4*>(a.dv + row + cb * 16 + 4 * j) =
                                    make_float4(__uint_as_float(v[4 * j]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 1]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 2]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 3]) * a.inv_n);
                        }
                        tmem_ld16(tK + cq * (D / 4) + cb * 16, v);
                        if (kvalid) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<float4*>(a.dk + row + cb * 16 + 4 * j) =
                                    make_float4(__uint_as_float(v[4 * j]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 1]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 2]) * a.inv_n,
                                                __uint_as_float(v[4 * j + 3]) * a.inv_n);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bars[kBwAccFree]);
                }
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) raise_error(kErrTimeout);
    if (warp == C::kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace hstu
