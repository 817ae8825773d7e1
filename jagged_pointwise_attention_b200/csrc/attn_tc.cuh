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
// Warp roles ((4G + 4) warps for G pointwise groups). Every role that blocks
// on a barrier has a warp of its own: a lane suspended in a barrier wait holds
// up the other lanes of its warp.
//   warps 0..4G-1  pointwise stage in G groups of 4 warps. Counting the tiles a
//              CTA processes as n = 0, 1, 2, ..., group g handles n = g (mod G)
//              in its own S buffer, so the G warps that share an SM
//              sub-partition work on different tiles and hide each other's
//              TMEM, MUFU and barrier latencies. Warp w owns TMEM lanes
//              32*(w%4).. (one query row per thread) and all 128 columns. The
//              group that handles an item's last tile also writes its output.
//   warp 4G    item scheduler and TMA producer of Q tiles and the K ring
//   warp 4G+1  TMA producer of the V ring
//   warp 4G+2  MMA issuer (one thread) and TMEM owner
//   warp 4G+3  bias staging: per key tile, key timestamps (int64 and low 32
//              bits), their min/max and monotonicity, the window of the
//              relative-position table, and the query rows' timestamps and
//              sequence starts; one stage per S buffer. Software-pipelined: the
//              global loads of the next tile are in flight while the current
//              tile waits for its stage and is stored.
// TMEM (512 columns): S buffers at 128g, then one or two O accumulators.
// P_j overwrites the S_j buffer it came from, chunk by chunk: after a thread
// has read S columns 32c..32c+31 of its row it writes their 32 bf16 results
// into columns 32c..32c+15 (two per 32-bit column). The MMA issues PV_n and
// only then S_n+G into the same buffer.
//
// Masking: pair (i, j) is kept iff start(i) <= j <= i, with start(i) the first
// token of row i's sequence (the unit's k0 for aligned units, a per-row value
// for packed units of several short sequences). Warps whose 32 rows are all
// past the unit's end skip the tile: their P rows only feed O rows that are
// never stored.
//
// Pointwise arithmetic per score, with h = x/2 folded into the bias adds:
//   h = s/2 + pos/2 + time/2;  silu(x) = h + h*tanh(h)  (packed bf16x2, one
//   MUFU op per two scores). The time bucket floor(log2(max(1, dt))) is the
//   exponent field of dt converted exactly to double (no bit-find unit), and
//   the bucket's bias comes from a 32-entry register table via a shuffle. When
//   the key timestamps of a 32-key chunk are non-decreasing and every row of
//   the warp sees one bucket at both ends of the chunk, the bucket is constant
//   over the chunk and the per-score bucket work is skipped.
//
// Every wait is bounded; a wait that runs out raises kErrTimeout, the other
// roles notice through a shared abort flag, and the CTA drains its own copies
// and MMAs before it frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

struct AttnArgs {
    const int4* units;          // plan: (q0, q_end, k0, nk | packed << 31)
    const int* unit_count;
    int* item_counter;          // plan: zeroed; next work item to hand out
    const int* row_start;       // plan: first token of each packed row's sequence
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
constexpr int kMaxHeadsTable = 64;      // heads whose register time table is kept in SMEM
constexpr uint32_t kTmemCols = 512;

template <int D, int G>
struct AttnCfg {
    static constexpr int kPointwiseWarps = 4 * G;
    // One bias-staging warp: it must wait each stage's p_full phases in order
    // (a second warp staging alternate tiles could wait a phase two steps ahead
    // of the barrier, which the parity test cannot tell from the one before).
    static constexpr int kMetaWarps = 1;
    static constexpr int kWarpK = 4 * G, kWarpV = 4 * G + 1, kWarpMMA = 4 * G + 2,
                         kWarpMeta = 4 * G + 3;
    static constexpr int kThreads = (4 * G + 3 + kMetaWarps) * 32;
    static constexpr int kStages = D == 64 ? 3 : 2;                     // Q, K and V rings
    static constexpr int kOBufs = 128 * G + 2 * D <= static_cast<int>(kTmemCols) ? 2 : 1;
    static constexpr uint32_t kTmemO = 128 * G;
};

// One stage of staged bias data for one key tile.
struct MetaStage {
    float w[256];          // w[m] = pos[h][clamp(q0 - kt0 - 127 + m, 0, P-1)] / 2
    int32_t kt32[128];     // low 32 bits of the key timestamps
    int64_t kt64[128];     // key timestamps
    int64_t rts[128];      // query-row timestamps
    int32_t rstart[128];   // query-row sequence starts
    int64_t tmin, tmax;    // over keys of the unit (< q_end)
    int32_t mono;          // keys non-decreasing over the tile (keys < q_end)
    int32_t pad[3];
};

template <int D, int G>
struct AttnSmem {
    using C = AttnCfg<D, G>;
    static constexpr int kTileBytes = kTile * D * 2;                    // one Q, K or V tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + C::kStages * kTileBytes;
    static constexpr int kOffV = kOffK + C::kStages * kTileBytes;
    static constexpr int kOffTB = kOffV + C::kStages * kTileBytes;      // float[kMaxHeadsTable][32]
    static constexpr int kOffMeta = kOffTB + kMaxHeadsTable * 32 * 4;   // MetaStage[G]
    static constexpr int kOffItems = kOffMeta + G * static_cast<int>(sizeof(MetaStage));
    static constexpr int kOffBar = kOffItems + kItemRing * 32;                // int[8] per slot
    static constexpr int kNumBars = 48;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;                        // 1 KB alignment slack
};

// barrier slots (rings of up to 3 stages, up to 3 S buffers, up to 2 O buffers)
enum {
    kBarQFull = 0,      // +stage
    kBarQFree = 3,      // +stage
    kBarKFull = 6,      // +stage
    kBarKFree = 9,      // +stage
    kBarVFull = 12,     // +stage
    kBarVFree = 15,     // +stage
    kBarSFull = 18,     // +buffer: MMA commit + 32 bias-staging lanes
    kBarPFull = 21,     // +buffer: the 128 threads of the buffer's group
    kBarOFull = 24,     // +group: MMA commit after the last PV of an item whose output
                        // that group writes (one barrier per group, so every barrier
                        // is waited by one group in its own order and a waiter can
                        // never be two phases ahead of it)
    kBarOFree = 27,     // +O buffer: the 128 threads that stored the item's output
    kBarDrain = 29,
    kBarItemFull = 30,  // +slot (8): scheduler published an item
    kBarItemFree = 38,  // +slot (8): every consumer has read it
};

// A work item as the scheduler publishes it; nk == 0 ends the stream.
struct Item {
    int q0, q_end, k0, nk, h;
    bool packed;
};

__device__ __forceinline__ Item load_item(const AttnArgs& a, int w) {
    const int u = w / a.H;
    const int4 wu = a.units[u];
    Item it;
    it.q0 = wu.x;
    it.q_end = wu.y;
    it.k0 = wu.z;
    it.nk = wu.w & 0x7fffffff;
    it.packed = (wu.w >> 31) & 1;
    it.h = w - u * a.H;
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
    return it;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

// silu of a packed pair of half-scores: h + h * tanh(h), bf16x2.
__device__ __forceinline__ uint32_t silu_half_bf16x2(float h0, float h1) {
    const uint32_t hp = pack_bf16x2(h0, h1);
    uint32_t t, y;
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(hp));
    asm("fma.rn.bf16x2 %0, %1, %2, %1;" : "=r"(y) : "r"(hp), "r"(t));
    return y;
}

// Per-chunk pointwise paths. sv: 32 fp32 scores of columns c0..c0+31 of this
// thread's row; wrow[-c] = pos/2 of column c; pk: 16 packed bf16x2 outputs.

// Constant time bucket over the chunk: tconst = time/2 for every column.
template <bool kMask>
__device__ __forceinline__ void pw_const(const uint32_t* sv, int c0,
                                         const float* __restrict__ wrow, float tconst, int lo,
                                         int hi, uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float h[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = c0 + e + u;
            float v = fmaf(__uint_as_float(sv[e + u]), 0.5f, wrow[-c]) + tconst;
            if (kMask) v = (c >= lo && c <= hi) ? v : 0.0f;
            h[u] = v;
        }
        pk[e >> 1] = silu_half_bf16x2(h[0], h[1]);
    }
}

// Bucket per score, differences exact in 32 bits. tbr: this lane's entry of
// the register table (lane L holds time/2 of bucket min((L+1) mod 32, NB-1)).
template <bool kMask>
__device__ __forceinline__ void pw_fast(const uint32_t* sv, int c0,
                                        const float* __restrict__ wrow,
                                        const int32_t* __restrict__ kt32, int32_t ti32, float tbr,
                                        int lo, int hi, uint32_t* pk) {
    const int4* k4 = reinterpret_cast<const int4*>(kt32 + c0);
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        const int4 kk = k4[e >> 2];
        const int32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
        float h[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = c0 + e + u;
            const int32_t dt = static_cast<int32_t>(static_cast<uint32_t>(ti32) -
                                                    static_cast<uint32_t>(kv[u]));
            const uint32_t ef = log2_exponent_field(static_cast<uint32_t>(max(dt, 1)));
            const float tv = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef));
            float v = fmaf(__uint_as_float(sv[e + u]), 0.5f, wrow[-c]) + tv;
            if (kMask) v = (c >= lo && c <= hi) ? v : 0.0f;
            h[u] = v;
        }
        pk[e >> 1] = silu_half_bf16x2(h[0], h[1]);
        pk[(e >> 1) + 1] = silu_half_bf16x2(h[2], h[3]);
    }
}

// Any int64 timestamps: 64-bit bucket, table row of this head read through
// the read-only cache (tbh = time_bias + h * NB, or null).
template <bool kMask>
__device__ __forceinline__ void pw_slow(const uint32_t* sv, int c0,
                                        const float* __restrict__ wrow,
                                        const int64_t* __restrict__ kt64, int64_t ti,
                                        const float* __restrict__ tbh, int nbm1, int lo, int hi,
                                        uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float h[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = c0 + e + u;
            const float tv = tbh ? 0.5f * __ldg(tbh + time_bucket64(ti - kt64[c], nbm1)) : 0.f;
            float v = fmaf(__uint_as_float(sv[e + u]), 0.5f, wrow[-c]) + tv;
            if (kMask) v = (c >= lo && c <= hi) ? v : 0.0f;
            h[u] = v;
        }
        pk[e >> 1] = silu_half_bf16x2(h[0], h[1]);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(AttnCfg<D, G>::kThreads, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
    using C = AttnCfg<D, G>;
    using L = AttnSmem<D, G>;
    constexpr int S = C::kStages;
    constexpr int OB = C::kOBufs;
    constexpr int kKB = D / 64;   // 64-element (128-byte) column blocks per row
    constexpr int kTileBytes = L::kTileBytes;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(G >= 1 && G <= 3 && S <= 3 && OB <= 2, "barrier map");
    static_assert(128 * G + OB * D <= static_cast<int>(kTmemCols), "TMEM budget");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int n_items = *args.unit_count * args.H;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
    float* tbh_s = reinterpret_cast<float*>(smem + L::kOffTB);
    MetaStage* meta = reinterpret_cast<MetaStage*>(smem + L::kOffMeta);
    volatile int* items = reinterpret_cast<volatile int*>(smem + L::kOffItems);
    constexpr int kConsumers = 2 + C::kMetaWarps + C::kPointwiseWarps;   // V, MMA, bias, pointwise
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
            mbar_init(&bars[kBarSFull + b], 1 + 32);
            mbar_init(&bars[kBarPFull + b], 128);
        }
        for (int b = 0; b < G; ++b) mbar_init(&bars[kBarOFull + b], 1);
        for (int o = 0; o < OB; ++o) mbar_init(&bars[kBarOFree + o], 128);
        for (int q = 0; q < kItemRing; ++q) {
            mbar_init(&bars[kBarItemFull + q], 1);
            mbar_init(&bars[kBarItemFree + q], kConsumers);
        }
        mbar_init(&bars[kBarDrain], 1);
        mbar_fence_init();
    }
    if (warp == C::kWarpMMA) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp < C::kPointwiseWarps) {
        // register-table source: [h][L] = time/2 of bucket min((L + 1) mod 32, NB - 1)
        for (int idx = tid; idx < args.H * 32; idx += 32 * C::kPointwiseWarps) {
            const int hh = idx >> 5, ll = idx & 31;
            tbh_s[idx] = use_time ? 0.5f * args.tb[static_cast<int64_t>(hh) * args.NB +
                                                   min((ll + 1) & 31, nbm1)]
                                  : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

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
                        I.q0 = I.q_end = I.k0 = I.h = 0;
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
                    if (n >= S && !mbar_wait(&freeb[ks], ((n / S) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[ks], kTileBytes);
#pragma unroll
                    for (int kb = 0; kb < kKB; ++kb)
                        tma_load_2d(smem + ring + ks * kTileBytes + kb * 16384, tm, &full[ks],
                                    I.h * D + kb * 64, I.k0 + j * kTile);
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
        }
        __syncwarp();
    } else if (warp == C::kWarpMMA) {
        // ------------------------------------------------------------ MMA issuer
        // Two cursors over the item stream: S runs G-1 tiles ahead of PV (PV_n
        // is issued before S_n+G reuses buffer n % G). The S cursor takes items
        // from the ring without releasing them; the PV cursor re-reads the same
        // slot and releases it once the item's last PV is issued, so the slot
        // stays valid in between.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            constexpr uint32_t kStageDesc = kTileBytes >> 4;      // stage stride, descriptor units
            const uint64_t dq0 = desc_kmajor_sw128(sQ);
            const uint64_t dk0 = desc_kmajor_sw128(sK);
            const uint64_t dv0 = desc_mnmajor_sw128(sV, 16384);
            auto wait_item = [&](int k, Item& I) -> bool {
                const int slot = k % kItemRing;
                if (!mbar_wait(&bars[kBarItemFull + slot], (k / kItemRing) & 1, abort_flag)) return false;
                I = read_item(items + slot * 8);
                return true;
            };
            bool ok = true;
            // S cursor
            int s_it = 0, s_j = 0, ns = 0;
            Item si;
            si.nk = -1;
            bool s_live = wait_item(0, si) && si.nk > 0;
            if (si.nk < 0) ok = false;                                        // aborted
            // PV cursor
            int p_it = 0, p_j = 0, np = 0;
            Item pi = si;
            while (ok && (s_live || np < ns)) {
                if (s_live && ns - np < G) {
                    // ---- S_ns = Q K^T into buffer ns % G
                    const int qs = s_it % S, ks = ns % S, b = ns % G;
                    if (s_j == 0 && !mbar_wait(&bars[kBarQFull + qs], (s_it / S) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&bars[kBarKFull + ks], (ns / S) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dq = dq0 + static_cast<uint64_t>(qs * kStageDesc);
                    const uint64_t dk = dk0 + static_cast<uint64_t>(ks * kStageDesc);
                    const uint32_t dst = tmem + b * 128;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        umma_bf16_ss(dst, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&bars[kBarSFull + b]);
                    umma_commit(&bars[kBarKFree + ks]);
                    ++ns;
                    if (++s_j == si.nk) {
                        umma_commit(&bars[kBarQFree + qs]);
                        s_j = 0;
                        ++s_it;
                        si.nk = -1;
                        s_live = wait_item(s_it, si) && si.nk > 0;
                        if (si.nk < 0) {               // aborted while waiting for an item
                            ok = false;
                            break;
                        }
                    }
                } else {
                    // ---- PV_np: O += P V, A operand from TMEM
                    const int b = np % G, vs = np % S, ob = p_it % OB;
                    if (p_j == 0 && np > 0) {
                        // the PV cursor enters item p_it: same ring slot the S cursor read
                        pi = read_item(items + (p_it % kItemRing) * 8);
                    }
                    const bool first = p_j == 0, last = p_j == pi.nk - 1;
                    if (!mbar_wait(&bars[kBarPFull + b], (np / G) & 1, abort_flag) ||
                        !mbar_wait(&bars[kBarVFull + vs], (np / S) & 1, abort_flag) ||
                        (first && p_it >= OB &&
                         !mbar_wait(&bars[kBarOFree + ob], ((p_it / OB) - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dv = dv0 + static_cast<uint64_t>(vs * kStageDesc);
                    const uint32_t pb = tmem + b * 128;
                    const uint32_t dst = tmem + C::kTmemO + ob * D;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        // keys 16kk..16kk+15: columns 32*(kk/2) + 8*(kk%2) of the P buffer
                        umma_bf16_ts(dst, pb + (kk >> 1) * 32 + (kk & 1) * 8,
                                     dv + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                                     (first && kk == 0) ? 0u : 1u);
                    }
                    umma_commit(&bars[kBarVFree + vs]);
                    ++np;
                    if (last) {
                        umma_commit(&bars[kBarOFull + b]);   // group b writes this item
                        mbar_arrive(&bars[kBarItemFree + p_it % kItemRing]);
                        p_j = 0;
                        ++p_it;
                    } else {
                        ++p_j;
                    }
                }
            }
            // (the end-of-stream slot is never reused, so it is not released)
            umma_commit(&bars[kBarDrain]);
            if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if (warp == C::kWarpMeta) {
        // ------------------------------------------------------------ bias staging
        // Per-tile values this lane stages: pos window (8), key timestamps (4),
        // query-row timestamps (4) and sequence starts (4).
        struct Staged {
            float w[8];
            int64_t kt[4], rt[4];
            int32_t rs[4];
        };
        auto load_tile = [&](const Item& I, int j, Staged& d) {
            const int kt0 = I.k0 + j * kTile;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int mm = lane + 32 * u;
                d.w[u] = 0.f;
                if (args.pos && mm < 255) {
                    int64_t dd = static_cast<int64_t>(I.q0) - kt0 - 127 + mm;
                    dd = dd < 0 ? 0 : (dd > args.P - 1 ? args.P - 1 : dd);
                    d.w[u] = args.pos[static_cast<int64_t>(I.h) * args.P + dd];
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t key = static_cast<int64_t>(kt0) + lane + 32 * u;
                d.kt[u] = use_time ? args.ts[key < args.T ? key : args.T - 1] : 0;
                const int64_t i = static_cast<int64_t>(I.q0) + lane + 32 * u;
                const bool v = i < I.q_end;
                d.rt[u] = (use_time && v) ? args.ts[i < args.T ? i : args.T - 1] : 0;
                d.rs[u] = (I.packed && v) ? args.row_start[i] : I.k0;
            }
        };
        Item cur;
        int it = 0, j = 0, n = 0;
        bool have = take_item(it++, true, cur) && cur.nk > 0;
        Staged st;
        if (have) load_tile(cur, 0, st);
        while (have) {
            // the following tile: its loads fly while this tile is stored
            Item nxt = cur;
            int nj = j + 1;
            bool nhave = true;
            if (nj >= cur.nk) {
                nj = 0;
                nhave = take_item(it++, true, nxt) && nxt.nk > 0;
            }
            Staged sn;
            if (nhave) load_tile(nxt, nj, sn);
            const int b = n % G;
            // stage b last served tile n-G; P_n-G written means it has been read
            if (n >= G && !warp_wait(&bars[kBarPFull + b], ((n / G) - 1) & 1, abort_flag)) break;
            MetaStage& ms = meta[b];
            const int kt0 = cur.k0 + j * kTile;
#pragma unroll
            for (int u = 0; u < 8; ++u) ms.w[lane + 32 * u] = 0.5f * st.w[u];
            int64_t tmin = INT64_MAX, tmax = INT64_MIN;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int mm = lane + 32 * u;
                ms.kt64[mm] = st.kt[u];
                ms.kt32[mm] = static_cast<int32_t>(static_cast<uint64_t>(st.kt[u]));
                ms.rts[mm] = st.rt[u];
                ms.rstart[mm] = st.rs[u];
                if (kt0 + mm < cur.q_end) {
                    tmin = st.kt[u] < tmin ? st.kt[u] : tmin;
                    tmax = st.kt[u] > tmax ? st.kt[u] : tmax;
                }
            }
            __syncwarp();
            bool mono = true;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int mm = lane + 32 * u;
                if (mm < 127 && kt0 + mm + 1 < cur.q_end)
                    mono = mono && (ms.kt64[mm] <= ms.kt64[mm + 1]);
            }
            mono = __all_sync(0xffffffffu, mono);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const int64_t a = __shfl_xor_sync(0xffffffffu, tmin, o);
                const int64_t c = __shfl_xor_sync(0xffffffffu, tmax, o);
                tmin = a < tmin ? a : tmin;
                tmax = c > tmax ? c : tmax;
            }
            if (lane == 0) {
                ms.tmin = tmin;
                ms.tmax = tmax;
                ms.mono = mono ? 1 : 0;
            }
            __syncwarp();
            mbar_arrive(&bars[kBarSFull + b]);
            cur = nxt;
            j = nj;
            have = nhave;
            st = sn;
            ++n;
        }
    } else {
        // ------------------------------------------------------------ pointwise stage
        const int g = warp >> 2;                            // group: tiles n = g (mod G)
        const int qd = warp & 3;                            // TMEM lane quarter
        const int r = qd * 32 + lane;                       // query row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const MetaStage& ms = meta[g];
        const uint32_t s_col = tmem + lane_base + static_cast<uint32_t>(g * 128);
        bool ok = true;
        int n = 0, it = 0, ep = 0;   // ep: outputs this group has written
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
            const float tbr = tbh_s[I.h * 32 + lane];
            const float* tbh = use_time ? args.tb + static_cast<int64_t>(I.h) * args.NB : nullptr;
            for (int j = 0; j < I.nk; ++j, ++n) {
                if (n % G != g) continue;
                if (!warp_wait(&bars[kBarSFull + g], (n / G) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (warp_live) {
                    const int kt0 = I.k0 + j * kTile;
                    const int lo = ms.rstart[r] - kt0;      // first key of row i's sequence
                    const int hi = row_valid ? static_cast<int>(i - kt0) : -1;
                    const int64_t ti = ms.rts[r];
                    const int32_t ti32 = static_cast<int32_t>(static_cast<uint64_t>(ti));
                    bool fast = true;
                    if (row_valid && use_time) {
                        const int64_t lo_t = ti < ms.tmin ? ti : ms.tmin;
                        const int64_t hi_t = ti > ms.tmax ? ti : ms.tmax;
                        fast = static_cast<uint64_t>(hi_t) - static_cast<uint64_t>(lo_t) < (1ull << 31);
                    }
                    const bool fast_w = __all_sync(0xffffffffu, fast);
                    const bool mono = ms.mono != 0;
                    const float* wrow = ms.w + 127 + r;
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        const int c0 = 32 * q;
                        uint32_t pk[16];
                        const bool live = __any_sync(0xffffffffu, row_valid && hi >= c0 &&
                                                                      lo <= c0 + 31 && lo <= hi);
                        if (!live) {                        // every pair of the chunk is masked
#pragma unroll
                            for (int e = 0; e < 16; ++e) pk[e] = 0u;
                            tmem_st16(s_col + c0, pk);
                            continue;
                        }
                        uint32_t sv[32];
                        __syncwarp();
                        tmem_ld32(s_col + c0, sv);
                        const bool full = __all_sync(0xffffffffu, lo <= c0 && hi >= c0 + 31);
                        bool done = false;
                        if (!fast_w) {
                            if (full) pw_slow<false>(sv, c0, wrow, ms.kt64, ti, tbh, nbm1, lo, hi, pk);
                            else pw_slow<true>(sv, c0, wrow, ms.kt64, ti, tbh, nbm1, lo, hi, pk);
                            done = true;
                        } else if (full && mono) {
                            const uint32_t ef0 = log2_exponent_field(static_cast<uint32_t>(max(
                                static_cast<int32_t>(static_cast<uint32_t>(ti32) - static_cast<uint32_t>(ms.kt32[c0])), 1)));
                            const uint32_t ef1 = log2_exponent_field(static_cast<uint32_t>(max(
                                static_cast<int32_t>(static_cast<uint32_t>(ti32) - static_cast<uint32_t>(ms.kt32[c0 + 31])), 1)));
                            const float tconst = __shfl_sync(0xffffffffu, tbr, static_cast<int>(ef0));
                            if (__all_sync(0xffffffffu, ef0 == ef1)) {
                                pw_const<false>(sv, c0, wrow, tconst, lo, hi, pk);
                                done = true;
                            }
                        }
                        if (!done) {
                            if (full) pw_fast<false>(sv, c0, wrow, ms.kt32, ti32, tbr, lo, hi, pk);
                            else pw_fast<true>(sv, c0, wrow, ms.kt32, ti32, tbr, lo, hi, pk);
                        }
                        // 32 bf16 results -> columns 32q..32q+15 of the S buffer just read
                        tmem_st16(s_col + c0, pk);
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars[kBarPFull + g]);
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
                            tmem_ld32(tmem + lane_base + C::kTmemO + ob * D + ch * 32, ov);
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
