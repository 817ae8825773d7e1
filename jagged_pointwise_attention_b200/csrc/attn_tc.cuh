// attn_tc.cuh -- bf16 HSTU jagged causal attention forward on tcgen05.
//
// Persistent kernel: one CTA per SM takes work items (a work unit from the plan
// times one head) from a global counter over a longest-first list -- greedy
// longest-processing-time scheduling -- and streams their key tiles through one
// continuous pipeline, so loads, tensor-core work and pointwise work of
// consecutive items overlap. The K producer fetches items ahead of time and
// publishes them to every other role through a ring in shared memory. For every key tile j:
//     S_j  = Q K_j^T                         tcgen05.mma, SMEM x SMEM -> TMEM (fp32)
//     P_j  = silu(S_j + pos + time) * mask   TMEM -> registers -> bf16 TMEM
//     O   += P_j V_j                          tcgen05.mma, TMEM x SMEM -> TMEM (fp32)
// and at the item's last tile out = O / max_seqlen (bf16). There is no
// softmax: no running max, no rescale, no row sum, so O accumulates untouched
// across key tiles and the per-element budget goes to the bias gathers and SiLU.
//
// Warp roles ((4G + 3) warps for G pointwise groups). Every role that blocks
// on a barrier has a warp of its own: a lane suspended in a barrier wait holds
// up the other lanes of its warp.
//   warps 0..4G-1  pointwise stage in G groups of 4 warps. Counting the tiles a
//              CTA processes as n = 0, 1, 2, ..., group g handles n = g (mod G)
//              in its own S buffer, so the G warps that share an SM
//              sub-partition work on different tiles and hide each other's
//              TMEM, MUFU and barrier latencies. Warp w owns TMEM lanes
//              32*(w%4).. (one query row per thread) and all 128 columns. The
//              group that handles an item's last tile also writes its output.
//              Each group stages the bias data of its own tiles (below).
//   warp 4G    item scheduler and TMA producer of Q tiles and the K ring
//   warp 4G+1  TMA producer of the V ring
//   warp 4G+2  MMA issuer (one thread) and TMEM owner
// TMEM (512 columns): S buffers at 128g, then one or two O accumulators.
// P_j overwrites the S_j buffer it came from, chunk by chunk: after a thread
// has read S columns 32c..32c+31 of its row it writes their 32 bf16 results
// into columns 32c..32c+15 (two per 32-bit column). The MMA issues PV_n and
// only then S_n+G into the same buffer.
//
// Bias staging. Per key tile a group needs the tile's window of the
// relative-position table and its key timestamps. The group's 128 threads
// stage them into one of two stages of its own while the tile's S is still
// being computed: right after finishing its previous tile, so the global loads
// overlap the wait for S, and spread over 128 threads, so no single warp has
// to keep up with every tile of the SM. Two stages per group suffice: a thread
// refills a stage only after S of the group's previous tile was ready, which
// the MMA issues only after every thread of the group finished the tile
// before it (the stage's last reader). Per-row values (the row's timestamp,
// its sequence start, the head's time-bias table) are loaded once per item.
//
// Masking: pair (i, j) is kept iff start(i) <= j <= i, with start(i) the first
// token of row i's sequence (the unit's k0 for aligned units, a per-row value
// for packed units of several short sequences). Warps whose 32 rows are all
// past the unit's end skip the tile: their P rows only feed O rows that are
// never stored.
//
// Pointwise arithmetic per score, with h = x/2 folded into the bias adds:
//   h = s/2 + pos/2 + time/2;  silu(x) = h + h*tanh(h)  (packed bf16x2, one
//   tanh.approx.bf16x2 per two scores). The time bucket floor(log2(max(1,
//   dt))) comes from a count of leading zeros, and the bucket's bias from a
//   32-entry register table via a shuffle. The
//   bucket is monotone in dt, so when every row of a warp sees one bucket at
//   the smallest and the largest key timestamp of a 32-key chunk, the bucket
//   is constant over the chunk and the per-score bucket work is skipped.
//
// Head dimension d = 32 is staged as 64-column tiles (the next head's columns,
// or zeros past the last head): S uses only the first 32 columns of Q and K,
// and PV computes 64 output columns of which the first 32 are stored.
//
// Batches of short sequences take attn_short.cuh instead: one launch, no plan.
//
// Every wait is bounded; a wait that runs out raises kErrTimeout, the other
// roles notice through a shared abort flag, and the CTA drains its own copies
// and MMAs before it frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

struct KeySummary;

struct AttnArgs {
    const int4* units;          // plan: (q0, q_end, k0, nk | nt << 11 | packed << 31)
    const int* unit_count;
    int max_units;              // capacity of the work list (the count is clamped to it)
    int* item_counter;          // plan: zeroed; next work item to hand out
    const uint4* starts;        // plan: per packed unit, rows where a sequence begins
    const uint4* ptab;          // bias prep: [H][DD][248] window tables (see BiasStage)
    int DD;                     // window tables per head (diagonal offsets 0..DD-1)
    const KeySummary* ksum;     // bias prep: per unit, its 128 tokens as keys; null without time
    int H;
    int64_t T;
    const int64_t* ts;          // [T] or null
    const float* pos;           // [H, P] or null
    int P;
    const float* tb;            // [H, NB] or null
    int NB;
    float inv_n;
    __nv_bfloat16* out;
    int64_t out_stride;         // elements per token
};

constexpr int kAttnGroups = 3;          // pointwise groups (S buffers)
constexpr int kItemRing = 8;            // work items published ahead of the pipeline
constexpr uint32_t kTmemCols = 512;

template <int D, int G>
struct AttnCfg {
    static constexpr int DT = D < 64 ? 64 : D;                         // staged tile width
    static constexpr int kPointwiseWarps = 4 * G;
    static constexpr int kWarpK = 4 * G, kWarpV = 4 * G + 1, kWarpMMA = 4 * G + 2,
                         kWarpPV = 4 * G + 3;
    static constexpr int kThreads = (4 * G + 4) * 32;
    static constexpr int kStages = DT == 64 ? 3 : 2;                    // Q, K and V rings
    static constexpr int kOBufs = 128 * G + 2 * DT <= static_cast<int>(kTmemCols) ? 2 : 1;
    static constexpr uint32_t kTmemO = 128 * G;
};

// Staged bias data of one key tile. The relative-position bias of the tile is
// a 255-value window (pair (r, c) reads offset 127 + r - c). It is kept as
// bf16 pos/2 in a sliding-window table: with R[k] = window offset 254 - k,
// entry s of wb holds R[s..s+7], so row r reads the 32 values of columns
// c0..c0+31 as entries k0, k0+8, k0+16, k0+24 (k0 = 127 - r + c0), four
// 16-byte loads whose word p packs columns (c0+2p, c0+2p+1). Entry s lies in
// 16-byte bank slot s mod 8, so the eight consecutive k0 of a quarter warp
// never conflict. The window depends only on the head and on the tile's
// diagonal offset (q0 - kt0) / 128, so the tables are built once per launch
// (bias_prep_kernel, or per CTA in shared memory by the short-batch kernel)
// and copied in per tile.
// Key timestamps are kept relative to `base` (the tile's first key) in 32
// bits, exact whenever every timestamp involved lies within 2^30 of base:
// ok[c] says so for the keys of chunk c, and cmin/cmax are the chunk's
// smallest and largest key timestamp minus base. They depend only on the
// key tile, i.e. on the unit whose rows are those keys, and are also built
// once per launch.
constexpr int kWinEntries = 248;
constexpr int kWinBytes = kWinEntries * 16;

struct alignas(16) KeySummary {
    int32_t kt32[128];     // key timestamps minus base (exact when ok[] holds)
    int64_t base;          // timestamp of the tile's first key
    int32_t cmin[4], cmax[4], ok[4];
    int32_t pad[2];
};
static_assert(sizeof(KeySummary) == 576, "key summary copy size");

struct alignas(16) BiasStage {
    uint4 wb[kWinEntries]; // sliding-window table of bf16 pos/2
    KeySummary keys;
};
static_assert(sizeof(BiasStage) == kWinBytes + sizeof(KeySummary), "stage layout");

// R[k] pair as the attention stages it: word m = (R[2m], R[2m+1]) with
// R[k] = bf16(pos[clamp(base - k)]) / 2 for k <= 254 and R[255] = 0. `row(a)`
// returns pos[clamp(a, 0, P - 1)] of the head's table.
template <typename Row>
__device__ __forceinline__ uint32_t window_word(Row row, int rel0, int m) {
    const int a = rel0 - 2 * m;
    const float v0 = row(a);
    const float v1 = m < 127 ? row(a - 1) : 0.f;
    uint32_t wd;
    // bf16(v) / 2 is exactly bf16(v / 2) (a power-of-two scale)
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(wd) : "r"(pack_bf16x2(v0, v1)), "r"(0x3f003f00u));
    return wd;
}

// Entry s of the window table of diagonal offset dd: R[s..s+7] as words
// (R[s+2i], R[s+2i+1]).
template <typename Row>
__device__ __forceinline__ uint4 window_entry_of(Row row, int dd, int s) {
    const int rel0 = 128 * dd + 127;                 // window offset of R[0]
    const uint32_t sel = (s & 1) ? 0x5432u : 0x3210u;
    uint32_t x[5];
#pragma unroll
    for (int k = 0; k < 5; ++k) x[k] = window_word(row, rel0, (s >> 1) + k);
    return make_uint4(__byte_perm(x[0], x[1], sel), __byte_perm(x[1], x[2], sel),
                      __byte_perm(x[2], x[3], sel), __byte_perm(x[3], x[4], sel));
}

// Entry e of the window tables [H][DD][248], read from the position table in
// global memory (pos null: the position term is absent, all zeros).
__device__ __forceinline__ uint4 window_entry(const float* pos, int P, int DD, int64_t e) {
    const int s = static_cast<int>(e % kWinEntries);
    const int hd = static_cast<int>(e / kWinEntries);
    const int h = hd / DD, dd = hd % DD;
    if (pos == nullptr) return make_uint4(0u, 0u, 0u, 0u);
    const float* prow = pos + static_cast<int64_t>(h) * P;
    return window_entry_of([&](int a) { return __ldg(prow + min(max(a, 0), P - 1)); }, dd, s);
}

template <int D, int G>
struct AttnSmem {
    using C = AttnCfg<D, G>;
    static constexpr int kTileBytes = kTile * C::DT * 2;                // one Q, K or V tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + C::kStages * kTileBytes;
    static constexpr int kOffV = kOffK + C::kStages * kTileBytes;
    static constexpr int kOffStage = kOffV + C::kStages * kTileBytes;   // BiasStage[2G]
    static constexpr int kOffItems = kOffStage + 2 * G * static_cast<int>(sizeof(BiasStage));
    static constexpr int kOffBar = kOffItems + kItemRing * 32;                // int[8] per slot
    static constexpr int kNumBars = 64;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;                        // 1 KB alignment slack
    static_assert(kAlloc <= 227 * 1024, "shared memory per block");
};

// barrier slots (rings of up to 3 stages, up to 3 S buffers, up to 2 O buffers)
enum {
    kBarQFull = 0,      // +stage
    kBarQFree = 3,      // +stage
    kBarKFull = 6,      // +stage
    kBarKFree = 9,      // +stage
    kBarVFull = 12,     // +stage
    kBarVFree = 15,     // +stage
    kBarSFull = 18,     // +buffer: MMA commit
    kBarPFull = 21,     // +buffer: the 128 threads of the buffer's group
    kBarOFull = 24,     // +group: MMA commit after the last PV of an item whose output
                        // that group writes (one barrier per group, so every barrier
                        // is waited by one group in its own order and a waiter can
                        // never be two phases ahead of it)
    kBarOFree = 27,     // +O buffer: the 128 threads that stored the item's output
    kBarDrain = 29,     // the S issuer's last commit
    kBarItemFull = 30,  // +slot (8): scheduler published an item
    kBarItemFree = 38,  // +slot (8): every consumer has read it
    kBarStage = 46,     // +2g+s (up to 6): the copies into stage s of group g landed
    kBarPVDone = 52,    // +buffer (up to 3): PV of the buffer's tile has completed
    kBarDrainPV = 55,   // the PV issuer's last commit
    kBarStageFree = 56, // +2g+s (up to 6): the four warps of group g are done with stage s
    kBarCount = 64,
};
static_assert(kBarCount == AttnSmem<64, kAttnGroups>::kNumBars, "barrier slots");

// A work item as the scheduler publishes it; nk == 0 ends the stream. s0: the
// unit index (packed tiles look up their sequence starts with it).
struct Item {
    int q0, q_end, k0, nk, h, s0;
    int kb;   // unit whose rows are key tile 0 (key tile j: unit kb - j)
    bool packed;
};

// Work item w. Items run sequence by sequence, then head, then unit: the
// units of a sequence are consecutive (nt of them, nt stored in each), so the
// item block of a sequence starting at unit ubase covers items
// [H*ubase, H*(ubase + nt)), and unit w / H lies in that sequence.
__device__ __forceinline__ Item load_item(const AttnArgs& a, int w) {
    const int u1 = w / a.H;
    const int4 d1 = a.units[u1];
    const int nk1 = d1.w & 0x7ff, nt = (d1.w >> 11) & 0x7ff;
    const int ubase = u1 - (nt - nk1);               // units hold tiles nt-1 .. 0
    const int r = w - a.H * ubase;
    const int h = r / nt;
    const int u = ubase + (r - h * nt);
    const int4 wu = u == u1 ? d1 : a.units[u];
    Item it;
    it.q0 = wu.x;
    it.q_end = wu.y;
    it.packed = (wu.w >> 31) & 1;
    it.k0 = wu.z;
    it.s0 = u;
    it.nk = wu.w & 0x7ff;
    it.h = h;
    it.kb = ubase + nt - 1;   // units hold tiles nt-1 .. 0
    return it;
}

__device__ __forceinline__ Item read_item(const volatile int* slot) {
    Item it;
    it.q0 = slot[0];
    it.q_end = slot[1];
    it.k0 = slot[2];
    it.nk = slot[3];
    it.h = slot[4];
    it.packed = slot[5] != 0;
    it.s0 = slot[6];
    it.kb = slot[7];
    return it;
}


// Per-chunk pointwise paths. sv: 32 fp32 scores of columns c0..c0+31 of this
// thread's row; wbk: this row's entry k0 of the pos/2 window table (entries
// wbk[0], wbk[8], wbk[16], wbk[24] cover the chunk); pk: 16 packed bf16x2
// outputs, word p = columns (c0+2p, c0+2p+1).
//
// Every path computes a pair the same way, in packed bf16x2:
//   h = bf16(s) * 0.5 + pos/2  (one rounding),  h = h + bf16(time/2),
//   p = h + h * tanh(h)        (one MUFU op per pair)
// and differs only in how it finds time/2, so which path a warp takes (a
// choice made over all of its 32 rows) never changes a row's bits.

// The half-score pair plus its bias pair.
__device__ __forceinline__ uint32_t half_arg_bf16x2(uint32_t s0, uint32_t s1, uint32_t w2,
                                                    uint32_t t2) {
    const uint32_t s2 = pack_bf16x2(__uint_as_float(s0), __uint_as_float(s1));
    uint32_t h, hb;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(h) : "r"(s2), "r"(0x3f003f00u), "r"(w2));
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(hb) : "r"(h), "r"(t2));
    return hb;
}

// silu(2h) = h + h * tanh(h) on a packed pair.
__device__ __forceinline__ uint32_t silu_of_half_bf16x2(uint32_t hb) {
    uint32_t t, y;
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(hb));
    asm("fma.rn.bf16x2 %0, %1, %2, %1;" : "=r"(y) : "r"(hb), "r"(t));
    return y;
}

// Keep-mask of the pair (c, c+1): pair (i, j) is kept iff lo <= j <= hi.
__device__ __forceinline__ uint32_t pair_mask(int c, int lo, int hi) {
    return ((c >= lo && c <= hi) ? 0x0000ffffu : 0u) | ((c + 1 >= lo && c + 1 <= hi) ? 0xffff0000u : 0u);
}

// Constant time bucket over an unmasked chunk (t2 = time/2 in both halves).
__device__ __forceinline__ void pw_const(const uint32_t* sv, const uint4* wbk, uint32_t t2,
                                         uint32_t* pk) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 W = wbk[8 * q];
        const uint32_t wv[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = 4 * q + u;
            pk[p] = silu_of_half_bf16x2(half_arg_bf16x2(sv[2 * p], sv[2 * p + 1], wv[u], t2));
        }
    }
}

// Two time buckets over an unmasked chunk: scores whose time difference is
// at least a power of two thr take th, the others tl; with key timestamps
// relative to base (ktr) and the row's tib = ti - base that is
// ktr <= kthr = tib - thr. The same bits as a bucket per score whenever every
// score's bucket is one of the two.
__device__ __forceinline__ void pw_two(const uint32_t* sv, int c0, const uint4* wbk,
                                       const int32_t* __restrict__ ktr, int32_t kthr,
                                       float tl, float th, uint32_t* pk) {
    const int4* k4 = reinterpret_cast<const int4*>(ktr + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 W = wbk[8 * q];
        const uint32_t wv[4] = {W.x, W.y, W.z, W.w};
        const int4 ka = k4[2 * q], kb = k4[2 * q + 1];
        const int32_t kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float tv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) tv[e] = kv[2 * u + e] <= kthr ? th : tl;
            const int p = 4 * q + u;
            pk[p] = silu_of_half_bf16x2(
                half_arg_bf16x2(sv[2 * p], sv[2 * p + 1], wv[u], pack_bf16x2(tv[0], tv[1])));
        }
    }
}

// Bucket per score, differences exact in 32 bits (tib - ktr, both relative
// to base). tbr: this lane's entry of the register table (lane L holds
// time/2 of bucket min((L+1) mod 32, NB-1)).
template <bool kMask>
__device__ __forceinline__ void pw_fast(const uint32_t* sv, int c0, const uint4* wbk,
                                        const int32_t* __restrict__ ktr, int32_t tib, float tbr,
                                        int lo, int hi, uint32_t* pk) {
    const int4* k4 = reinterpret_cast<const int4*>(ktr + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 W = wbk[8 * q];
        const uint32_t wv[4] = {W.x, W.y, W.z, W.w};
        const int4 ka = k4[2 * q], kb = k4[2 * q + 1];
        const int32_t kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float tv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int32_t dt = tib - kv[2 * u + e];
                const uint32_t ef = log2_exponent_field(static_cast<uint32_t>(max(dt, 1)));
                tv[e] = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef));
            }
            const int p = 4 * q + u;
            uint32_t hb = half_arg_bf16x2(sv[2 * p], sv[2 * p + 1], wv[u], pack_bf16x2(tv[0], tv[1]));
            if (kMask) hb &= pair_mask(c0 + 2 * p, lo, hi);
            pk[p] = silu_of_half_bf16x2(hb);
        }
    }
}

// Any int64 timestamps: 64-bit bucket from the key timestamps in global
// memory (kts = timestamps of the tile's keys, column c read at min(c, lastc)
// so a tile past the end of the batch stays in bounds), table row of this
// head read through the read-only cache (tbh = time_bias + h * NB, or null).
template <bool kMask>
__device__ __forceinline__ void pw_slow(const uint32_t* sv, int c0, const uint4* wbk,
                                        const int64_t* __restrict__ kts, int lastc, int64_t ti,
                                        const float* __restrict__ tbh, int nbm1, int lo, int hi,
                                        uint32_t* pk) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 W = wbk[8 * q];
        const uint32_t wv[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = 4 * q + u;
            const int c = c0 + 2 * p;
            float tv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
                tv[e] = tbh ? 0.5f * __ldg(tbh + time_bucket64(ti - __ldg(kts + min(c + e, lastc)), nbm1))
                            : 0.f;
            uint32_t hb = half_arg_bf16x2(sv[2 * p], sv[2 * p + 1], wv[u], pack_bf16x2(tv[0], tv[1]));
            if (kMask) hb &= pair_mask(c, lo, hi);
            pk[p] = silu_of_half_bf16x2(hb);
        }
    }
}

// First token of row q0 + r's sequence in a packed tile: the highest marked
// row <= r of the tile's sequence-start mask (row 0 is always marked). Rows
// past the tile's end get a start past every key.
__device__ __forceinline__ int packed_row_start(const AttnArgs& a, const Item& I, int r) {
    if (I.q0 + r >= I.q_end) return 0x7fffffff;
    const uint4 m4 = __ldg(a.starts + I.s0);
    const uint32_t m[4] = {m4.x, m4.y, m4.z, m4.w};
    int w = r >> 5;
    uint32_t x = m[w] & (0xffffffffu >> (31 - (r & 31)));   // marks at rows <= r of word w
#pragma unroll
    for (int k = 0; k < 3; ++k)
        if (x == 0u && w > 0) x = m[--w];
    return I.q0 + 32 * w + 31 - __clz(x);
}

template <int D, int G>
__global__ void __launch_bounds__(AttnCfg<D, G>::kThreads, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
    using C = AttnCfg<D, G>;
    using L = AttnSmem<D, G>;
    constexpr int DT = C::DT;
    constexpr int S = C::kStages;
    constexpr int OB = C::kOBufs;
    constexpr int kKB = DT / 64;   // 64-element (128-byte) column blocks per row
    constexpr int kTileBytes = L::kTileBytes;
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(G >= 1 && G <= 3 && S <= 3 && OB <= 2, "barrier map");
    static_assert(128 * G + OB * DT <= static_cast<int>(kTmemCols), "TMEM budget");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
    BiasStage* stages = reinterpret_cast<BiasStage*>(smem + L::kOffStage);
    volatile int* items = reinterpret_cast<volatile int*>(smem + L::kOffItems);
    constexpr int kConsumers = 3 + C::kPointwiseWarps;   // V, both MMA issuers, pointwise
    const bool use_time = args.ts != nullptr && args.tb != nullptr && args.NB > 0;
    const int nbm1 = use_time ? args.NB - 1 : 0;

    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&bars[kBarQFull + s], 1);
            mbar_init(&bars[kBarQFree + s], 1);
            mbar_init(&bars[kBarKFull + s], 1);
            mbar_init(&bars[kBarKFree + s], 1);
            mbar_init(&bars[kBarVFull + s], 1);
            mbar_init(&bars[kBarVFree + s], 1);
        }
        for (int b = 0; b < G; ++b) {
            mbar_init(&bars[kBarSFull + b], 1);
            mbar_init(&bars[kBarPFull + b], 128);
            mbar_init(&bars[kBarStage + 2 * b], 1);
            mbar_init(&bars[kBarStage + 2 * b + 1], 1);
            mbar_init(&bars[kBarStageFree + 2 * b], 4);
            mbar_init(&bars[kBarStageFree + 2 * b + 1], 4);
        }
        for (int b = 0; b < G; ++b) mbar_init(&bars[kBarOFull + b], 1);
        for (int o = 0; o < OB; ++o) mbar_init(&bars[kBarOFree + o], 128);
        for (int q = 0; q < kItemRing; ++q) {
            mbar_init(&bars[kBarItemFull + q], 1);
            mbar_init(&bars[kBarItemFree + q], kConsumers);
        }
        mbar_init(&bars[kBarDrain], 1);
        mbar_init(&bars[kBarDrainPV], 1);
        for (int b = 0; b < G; ++b) mbar_init(&bars[kBarPVDone + b], 1);
        mbar_fence_init();
    }
    if (warp == C::kWarpMMA) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // The work list comes from the plan kernel launched just before: the set-up
    // above overlaps its tail (programmatic dependent launch); wait for it to
    // complete, with its writes visible, before reading the list.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = min(*args.unit_count, args.max_units) * args.H;

    const uint32_t sQ = smem_u32(smem + L::kOffQ);
    const uint32_t sK = smem_u32(smem + L::kOffK);
    const uint32_t sV = smem_u32(smem + L::kOffV);
    // Consumer side of the item ring: wait for item k, copy it, release the slot.
    auto take_item = [&](int k, bool warp_level, Item& I) -> bool {
        const int slot = k % kItemRing;
        const uint32_t par = (k / kItemRing) & 1;
        const bool got = warp_level ? warp_wait(&bars[kBarItemFull + slot], par, abort_flag)
                                    : mbar_wait(&bars[kBarItemFull + slot], par, abort_flag);
        if (!got) return false;
        I = read_item(items + slot * 8);
        if (warp_level) __syncwarp();
        if (!warp_level || lane == 0) mbar_arrive(&bars[kBarItemFree + slot]);
        return true;
    };

    if (warp == C::kWarpK || warp == C::kWarpV) {
        // ------------------------------------------------------------ TMA producers
        if (lane == 0) {
            const bool is_k = warp == C::kWarpK;
            const CUtensorMap* tm = is_k ? &tmK : &tmV;
            const int ring = is_k ? L::kOffK : L::kOffV;
            uint64_t* full = &bars[is_k ? kBarKFull : kBarVFull];
            uint64_t* freeb = &bars[is_k ? kBarKFree : kBarVFree];
            tma_prefetch_desc(tm);
            if (is_k) tma_prefetch_desc(&tmQ);
            int n = 0, it = 0;
            bool ok = true;
            for (;; ++it) {
                Item I;
                if (is_k) {
                    // item scheduler: greedy dynamic assignment from the global counter,
                    // published to the other roles through the ring
                    const int slot = it % kItemRing;
                    if (it >= kItemRing &&
                        !mbar_wait(&bars[kBarItemFree + slot], ((it / kItemRing) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int w = atomicAdd(args.item_counter, 1);
                    if (w < n_items) {
                        I = load_item(args, w);
                    } else {
                        I.q0 = I.q_end = I.k0 = I.h = I.s0 = I.kb = 0;
                        I.nk = 0;
                        I.packed = false;
                    }
                    volatile int* e = items + slot * 8;
                    e[0] = I.q0;
                    e[1] = I.q_end;
                    e[2] = I.k0;
                    e[3] = I.nk;
                    e[4] = I.h;
                    e[5] = I.packed ? 1 : 0;
                    e[6] = I.s0;
                    e[7] = I.kb;
                    mbar_arrive(&bars[kBarItemFull + slot]);
                } else if (!take_item(it, false, I)) {
                    ok = false;
                    break;
                }
                if (I.nk == 0) break;
                if (is_k) {
                    const int qs = it % S;
                    if (it >= S && !mbar_wait(&bars[kBarQFree + qs], ((it / S) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes);
#pragma unroll
                    for (int kb = 0; kb < kKB; ++kb)
                        tma_load_2d(smem + L::kOffQ + qs * kTileBytes + kb * 16384, &tmQ,
                                    &bars[kBarQFull + qs], I.h * D + kb * 64, I.q0);
                }
                for (int j = 0; j < I.nk; ++j, ++n) {
                    const int ks = n % S;
                    // with K: the tile's bias data goes into stage (n / G) & 1 of group
                    // n % G, once the group is done with that stage's previous tile
                    const int sidx = 2 * (n % G) + ((n / G) & 1);
                    const int use = n / (2 * G);
                    if ((n >= S && !mbar_wait(&freeb[ks], ((n / S) - 1) & 1, abort_flag)) ||
                        (is_k && use > 0 &&
                         !mbar_wait(&bars[kBarStageFree + sidx], (use - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[ks], kTileBytes);
#pragma unroll
                    for (int kb = 0; kb < kKB; ++kb)
                        tma_load_2d(smem + ring + ks * kTileBytes + kb * 16384, tm, &full[ks],
                                    I.h * D + kb * 64, I.k0 + j * kTile);
                    if (is_k) {
                        BiasStage& st = stages[sidx];
                        const int dd = min(I.nk - 1 - j, args.DD - 1);     // diagonal offset
                        mbar_arrive_expect_tx(&bars[kBarStage + sidx],
                                              kWinBytes + (args.ksum ? sizeof(KeySummary) : 0));
                        bulk_load(st.wb, args.ptab + (static_cast<int64_t>(I.h) * args.DD + dd) * kWinEntries,
                                  kWinBytes, &bars[kBarStage + sidx]);
                        if (args.ksum)
                            bulk_load(&st.keys, args.ksum + (I.kb - j), sizeof(KeySummary),
                                      &bars[kBarStage + sidx]);
                    }
                }
                if (!ok) {
                    ++it;   // this item's Q load was issued
                    break;
                }
            }
            // drain: every copy this thread started has landed before the CTA ends
            // (stage s of a ring that took N loads took ceil((N - s) / S) of them)
            for (int s = 0; s < S; ++s) {
                const int cq = it > s ? (it - s + S - 1) / S : 0;
                const int ck = n > s ? (n - s + S - 1) / S : 0;
                if (is_k && cq > 0 && !mbar_wait(&bars[kBarQFull + s], (cq - 1) & 1, nullptr))
                    raise_error(kErrTimeout);
                if (ck > 0 && !mbar_wait(&full[s], (ck - 1) & 1, nullptr)) raise_error(kErrTimeout);
            }
            // stage (g, b) took the tiles g + G k, k even (b = 0) or odd (b = 1), k < K_g
            for (int g = 0; is_k && g < G; ++g) {
                const int kg = n > g ? (n - g + G - 1) / G : 0;
                for (int b = 0; b < 2; ++b) {
                    const int c = kg > b ? (kg - b + 1) / 2 : 0;
                    if (c > 0 && !mbar_wait(&bars[kBarStage + 2 * g + b], (c - 1) & 1, nullptr))
                        raise_error(kErrTimeout);
                }
            }
        }
        __syncwarp();
    } else if (warp == C::kWarpMMA || warp == C::kWarpPV) {
        // ------------------------------------------------------------ MMA issuers
        // The MMA unit queues hardly more than one instruction, so while the
        // issuing thread tests a barrier (a few hundred cycles for any shared
        // memory access after an MMA) the tensor pipe runs dry. S and PV are
        // therefore issued by two warps: while one waits, the other issues.
        // S_n+G overwrites the buffer PV_n reads, so the S issuer waits for
        // PV_n to complete (pv_done of the buffer) before issuing S_n+G.
        if (lane == 0) {
            constexpr uint32_t kStageDesc = kTileBytes >> 4;      // stage stride, descriptor units
            bool ok = true;
            int n = 0;
            if (warp == C::kWarpMMA) {
                // ---- S_n = Q K_n^T into buffer n % G
                constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
                const uint64_t dq0 = desc_kmajor_sw128(sQ);
                const uint64_t dk0 = desc_kmajor_sw128(sK);
                for (int it = 0; ok; ++it) {
                    Item I;
                    if (!take_item(it, false, I)) {
                        ok = false;
                        break;
                    }
                    if (I.nk == 0) break;
                    const int qs = it % S;
                    if (!mbar_wait(&bars[kBarQFull + qs], (it / S) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint64_t dq = dq0 + static_cast<uint64_t>(qs * kStageDesc);
                    for (int j = 0; j < I.nk; ++j, ++n) {
                        const int ks = n % S, b = n % G;
                        if (!mbar_wait(&bars[kBarKFull + ks], (n / S) & 1, abort_flag) ||
                            (n >= G && !mbar_wait(&bars[kBarPVDone + b], ((n / G) - 1) & 1, abort_flag))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t dk = dk0 + static_cast<uint64_t>(ks * kStageDesc);
                        const uint32_t dst = tmem + b * 128;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                            umma_bf16_ss(dst, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars[kBarSFull + b]);
                        umma_commit(&bars[kBarKFree + ks]);
                    }
                    if (!ok) break;
                    umma_commit(&bars[kBarQFree + qs]);
                }
                umma_commit(&bars[kBarDrain]);
                if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) raise_error(kErrTimeout);
            } else {
                // ---- PV_n: O += P V, A operand (P) from TMEM
                constexpr uint32_t idesc_pv = idesc_bf16_f32(128, DT, 0, 1);
                const uint64_t dv0 = desc_mnmajor_sw128(sV, 16384);
                for (int it = 0; ok; ++it) {
                    Item I;
                    if (!take_item(it, false, I)) {
                        ok = false;
                        break;
                    }
                    if (I.nk == 0) break;
                    const int ob = it % OB;
                    for (int j = 0; j < I.nk; ++j, ++n) {
                        const int b = n % G, vs = n % S;
                        const bool first = j == 0;
                        // resources first, right after the previous PV was issued, so
                        // these tests overlap MMAs already in the pipe; then P_n
                        if (!mbar_wait(&bars[kBarVFull + vs], (n / S) & 1, abort_flag) ||
                            (first && it >= OB &&
                             !mbar_wait(&bars[kBarOFree + ob], ((it / OB) - 1) & 1, abort_flag)) ||
                            !mbar_wait(&bars[kBarPFull + b], (n / G) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t dv = dv0 + static_cast<uint64_t>(vs * kStageDesc);
                        const uint32_t pb = tmem + b * 128;
                        const uint32_t dst = tmem + C::kTmemO + ob * DT;
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            // keys 16kk..16kk+15: columns 32*(kk/2) + 8*(kk%2) of the P buffer
                            umma_bf16_ts(dst, pb + (kk >> 1) * 32 + (kk & 1) * 8,
                                         dv + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                                         (first && kk == 0) ? 0u : 1u);
                        }
                        umma_commit(&bars[kBarVFree + vs]);
                        umma_commit(&bars[kBarPVDone + b]);
                        if (j == I.nk - 1) umma_commit(&bars[kBarOFull + b]);   // group b writes this item
                    }
                }
                umma_commit(&bars[kBarDrainPV]);
                if (!mbar_wait(&bars[kBarDrainPV], 0, nullptr)) raise_error(kErrTimeout);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ pointwise stage
        const int g = warp >> 2;                            // group: tiles n = g (mod G)
        const int qd = warp & 3;                            // TMEM lane quarter
        const int r = qd * 32 + lane;                       // query row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const uint32_t s_col = tmem + lane_base + static_cast<uint32_t>(g * 128);

        bool ok = true;
        int n = 0, it = 0, ep = 0;   // ep: outputs this group has written
        int nt = 0;                  // tiles this group has processed (stage nt % 2)
        for (; ok; ++it) {
            Item I;
            if (!take_item(it, true, I)) {
                ok = false;
                break;
            }
            if (I.nk == 0) break;
            const int64_t i = static_cast<int64_t>(I.q0) + r;
            const bool row_valid = i < I.q_end;
            const bool warp_live = __any_sync(0xffffffffu, row_valid);
            // per-row values of the item: timestamp, first token of the row's
            // sequence, and this lane's entry of the head's register time table
            // (lane L holds time/2 of bucket min((L + 1) mod 32, NB - 1))
            const int64_t ti = (use_time && row_valid) ? __ldg(args.ts + i) : 0;
            const int rs = I.packed ? packed_row_start(args, I, r) : I.k0;
            const float tbr = use_time ? 0.5f * __ldg(args.tb + static_cast<int64_t>(I.h) * args.NB +
                                                      min((lane + 1) & 31, nbm1))
                                       : 0.f;
            const float* tbh = use_time ? args.tb + static_cast<int64_t>(I.h) * args.NB : nullptr;
            for (int j = 0; j < I.nk; ++j, ++n) {
                if (n % G != g) continue;
                const int kt0 = I.k0 + j * kTile;
                const int sb = nt & 1;
                const BiasStage& st = stages[2 * g + sb];   // copied in by the K producer
                if (!warp_wait(&bars[kBarStage + 2 * g + sb], (nt >> 1) & 1, abort_flag) ||
                    !warp_wait(&bars[kBarSFull + g], (n / G) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ++nt;
                tc_fence_after();
                if (warp_live) {
                    const int lo = rs - kt0;                // first key of row i's sequence
                    const int hi = row_valid ? static_cast<int>(i - kt0) : -1;
                    bool fast = true;
                    int32_t tib = 0;                        // ti - base, when fast
                    if (use_time) {
                        const int64_t db = ti - st.keys.base;
                        fast = st.keys.ok[0] && st.keys.ok[1] && st.keys.ok[2] && st.keys.ok[3] &&
                               (!row_valid || (db > -(1ll << 30) && db < (1ll << 30)));
                        tib = static_cast<int32_t>(db);
                    }
                    const bool fast_w = __all_sync(0xffffffffu, fast);
                    const uint4* wbr = st.wb + (127 - r);        // entry k0 of chunk 0
                    // no pair of the tile masked for any row of the warp (every tile
                    // but the diagonal one of an aligned unit): no per-chunk tests
                    const bool tile_full = __all_sync(0xffffffffu, lo <= 0 && hi >= 127);
                    // one time bucket over the whole unmasked tile for every row of the
                    // warp (most tiles away from the diagonal): no per-chunk decisions
                    bool tile_const = tile_full && fast_w;
                    float t_tile = 0.f;
                    if (tile_const && use_time) {
                        const int kmin = min(min(st.keys.cmin[0], st.keys.cmin[1]), min(st.keys.cmin[2], st.keys.cmin[3]));
                        const int kmax = max(max(st.keys.cmax[0], st.keys.cmax[1]), max(st.keys.cmax[2], st.keys.cmax[3]));
                        const uint32_t ef_hi = log2_exponent_field(static_cast<uint32_t>(max(tib - kmin, 1)));
                        const uint32_t ef_lo = log2_exponent_field(static_cast<uint32_t>(max(tib - kmax, 1)));
                        t_tile = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef_lo));
                        tile_const = __all_sync(0xffffffffu, ef_hi == ef_lo);
                    }
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        const int c0 = 32 * q;
                        uint32_t pk[16];
                        const bool live = tile_full ||
                                          __any_sync(0xffffffffu, row_valid && hi >= c0 &&
                                                                      lo <= c0 + 31 && lo <= hi);
                        if (!live) {                        // every pair of the chunk is masked
#pragma unroll
                            for (int e = 0; e < 16; ++e) pk[e] = 0u;
                            tmem_st16_async(s_col + c0, pk);
                            continue;
                        }
                        uint32_t sv[32];
                        __syncwarp();
                        tmem_ld32(s_col + c0, sv);
                        const bool full = tile_full || __all_sync(0xffffffffu, lo <= c0 && hi >= c0 + 31);
                        if (!fast_w) {
                            const int lastc = static_cast<int>(args.T - 1 - kt0);
                            if (full) pw_slow<false>(sv, c0, wbr + c0, args.ts + kt0, lastc, ti, tbh, nbm1, lo, hi, pk);
                            else pw_slow<true>(sv, c0, wbr + c0, args.ts + kt0, lastc, ti, tbh, nbm1, lo, hi, pk);
                        } else {
                            // an unmasked chunk sees one or two buckets over its key range
                            // in most rows (tested at its largest and smallest dt); the
                            // rest take a bucket per score
                            int path = 2;
                            float tl = 0.f, th = 0.f;
                            int32_t kthr = INT_MIN;                 // no key below it
                            if (full) {
                                path = 0;
                                tl = t_tile;
                                if (use_time && !tile_const) {
                                    const uint32_t ef_hi = log2_exponent_field(static_cast<uint32_t>(max(tib - st.keys.cmin[q], 1)));
                                    const uint32_t ef_lo = log2_exponent_field(static_cast<uint32_t>(max(tib - st.keys.cmax[q], 1)));
                                    tl = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef_lo));
                                    th = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef_hi));
                                    // bucket ef_hi iff dt >= 2^(ef_hi - 1023) (>= 2 when ef_hi > ef_lo)
                                    if (ef_hi > ef_lo) kthr = tib - (1 << (ef_hi - 1023u));
                                    path = __all_sync(0xffffffffu, ef_hi == ef_lo) ? 0
                                           : __all_sync(0xffffffffu, ef_hi - ef_lo <= 1u) ? 1 : 2;
                                }
                            }
                            if (path == 0) pw_const(sv, wbr + c0, pack_bf16x2(tl, tl), pk);
                            else if (path == 1) pw_two(sv, c0, wbr + c0, st.keys.kt32, kthr, tl, th, pk);
                            else pw_fast<true>(sv, c0, wbr + c0, st.keys.kt32, tib, tbr, lo, hi, pk);
                        }
                        // 32 bf16 results -> columns 32q..32q+15 of the S buffer just read
                        tmem_st16_async(s_col + c0, pk);
                    }
                }
                tmem_wait_st();     // every P store of the tile has landed
                tc_fence_before();
                mbar_arrive(&bars[kBarPFull + g]);
                __syncwarp();       // the warp's last read of the stage is behind it
                if (lane == 0) mbar_arrive(&bars[kBarStageFree + 2 * g + sb]);
                if (j == I.nk - 1) {
                    // this group handled the item's last tile: store its output
                    const int ob = it % OB;
                    if (!warp_wait(&bars[kBarOFull + g], ep & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++ep;
                    tc_fence_after();
                    if (warp_live) {
                        __nv_bfloat16* orow =
                            args.out + i * args.out_stride + static_cast<int64_t>(I.h) * D;
#pragma unroll
                        for (int ch = 0; ch < D / 32; ++ch) {
                            uint32_t ov[32];
                            __syncwarp();
                            tmem_ld32(tmem + lane_base + C::kTmemO + ob * DT + ch * 32, ov);
                            if (row_valid) {
                                uint32_t wv[16];
#pragma unroll
                                for (int e = 0; e < 16; ++e)
                                    wv[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * args.inv_n,
                                                        __uint_as_float(ov[2 * e + 1]) * args.inv_n);
                                uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq)
                                    dst[qq] = make_uint4(wv[4 * qq], wv[4 * qq + 1], wv[4 * qq + 2],
                                                         wv[4 * qq + 3]);
                            }
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bars[kBarOFree + ob]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (*abort_flag) raise_error(kErrTimeout);
        // the last CTA to finish re-arms the item counter, so a plan can be run again
        __threadfence();
        if (atomicAdd(args.item_counter + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            atomicExch(args.item_counter, 0);
            atomicExch(args.item_counter + 1, 0);
            __threadfence();
        }
    }
    if (warp == C::kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace hstu
