// attn_tc.cuh -- bf16 HSTU jagged causal attention forward on tcgen05.
//
// One CTA computes one (128-row query tile, head) work unit. For every key
// tile j of the unit (causal tiles only):
//     S_j  = Q K_j^T                         tcgen05.mma, SMEM x SMEM -> TMEM (fp32)
//     P_j  = silu(S_j + pos + time) * mask   TMEM -> registers -> bf16 TMEM
//     O   += P_j V_j                          tcgen05.mma, TMEM x SMEM -> TMEM (fp32)
// and finally out = O / max_seqlen (bf16). There is no softmax: no running
// max, no rescale, no row sum, so O accumulates untouched across key tiles
// and the whole per-element budget goes to the bias gathers and the SiLU.
//
// Warp roles ((4G + 3) warps for G pointwise groups):
//   warps 0..4G-1  pointwise stage in G groups of 4 warps. Group g handles the
//              key tiles j = g (mod G) in its own S buffer, so the G warps that
//              share an SM sub-partition work on different tiles and hide each
//              other's TMEM, MUFU and barrier latencies. Warp w owns TMEM lanes
//              32*(w%4).. (one query row per thread) and all 128 columns.
//   warp 4G    TMA producers: lane 0 loads Q and the K ring, lane 1 the V ring
//              (2 stages each; K_j+2 is fetched as soon as S_j is done, V_j+2
//              as soon as PV_j is done)
//   warp 4G+1  MMA issuer (one thread) and TMEM owner
//   warp 4G+2  bias staging: per key tile, key timestamps (int64 and their low
//              32 bits), tile min/max and monotonicity, and the window of the
//              relative-position table the tile needs, one stage per S buffer
// TMEM (512 columns): S buffers at 128g, O at 128G. P_j overwrites the S_j
// buffer it came from, chunk by chunk: after a thread has read S columns
// 32c..32c+31 of its row it writes their 32 bf16 results into columns
// 32c..32c+15 (two per 32-bit column).
//
// Per key tile a group waits once (S_j and its bias stage ready) and arrives
// once (P_j written); the MMA issues PV_j and later S_j+G into the same
// buffer, in order.
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
    const int4* units;          // plan: (q0, q_end, k0, nk)
    const int* unit_count;
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
constexpr uint32_t kTmemCols = 512;

template <int G>
struct AttnRoles {
    static constexpr int kPointwiseWarps = 4 * G;
    static constexpr int kWarpTMA = 4 * G, kWarpMMA = 4 * G + 1, kWarpMeta = 4 * G + 2;
    static constexpr int kThreads = (4 * G + 3) * 32;
    static constexpr uint32_t kTmemO = 128 * G;
};

// One stage of staged bias data for one key tile.
struct MetaStage {
    float w[256];          // w[m] = pos[h][clamp(q0 - kt0 - 127 + m, 0, P-1)] / 2
    int32_t kt32[128];     // low 32 bits of the key timestamps
    int64_t kt64[128];     // key timestamps
    int64_t tmin, tmax;    // over keys of the unit (< q_end)
    int32_t mono;          // keys non-decreasing over the tile (keys < q_end)
    int32_t pad[3];
};

template <int D, int G>
struct AttnSmem {
    static constexpr int kQBytes = kTile * D * 2;       // Q tile, D/64 swizzled 16 KB blocks
    static constexpr int kKVBytes = kTile * D * 2;      // one K (or V) stage
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + 2 * kKVBytes;
    static constexpr int kOffTB = kOffV + 2 * kKVBytes;                 // float[kMaxTimeBuckets]
    static constexpr int kOffMeta = kOffTB + kMaxTimeBuckets * 4;       // MetaStage[G]
    static constexpr int kOffBar = kOffMeta + G * static_cast<int>(sizeof(MetaStage));
    static constexpr int kNumBars = 32;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;                        // 1 KB alignment slack
};

// barrier slots
enum {
    kBarQFull = 0,
    kBarKFull = 1,      // +stage (2)
    kBarKFree = 3,      // +stage (2)
    kBarVFull = 5,      // +stage (2)
    kBarVFree = 7,      // +stage (2)
    kBarSFull = 9,      // +buffer (G <= 3): MMA commit + 32 bias-staging lanes
    kBarPFull = 12,     // +buffer (G <= 3): the 128 threads of the buffer's group
    kBarOFull = 15,
    kBarDrain = 16,
};

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

// Any int64 timestamps: 64-bit bucket, table read from shared memory.
template <bool kMask>
__device__ __forceinline__ void pw_slow(const uint32_t* sv, int c0,
                                        const float* __restrict__ wrow,
                                        const int64_t* __restrict__ kt64, int64_t ti,
                                        const float* __restrict__ tb_s, int nbm1, int lo, int hi,
                                        uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float h[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = c0 + e + u;
            const float tv = tb_s[time_bucket64(ti - kt64[c], nbm1)];
            float v = fmaf(__uint_as_float(sv[e + u]), 0.5f, wrow[-c]) + tv;
            if (kMask) v = (c >= lo && c <= hi) ? v : 0.0f;
            h[u] = v;
        }
        pk[e >> 1] = silu_half_bf16x2(h[0], h[1]);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(AttnRoles<G>::kThreads, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
    using L = AttnSmem<D, G>;
    using R = AttnRoles<G>;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(G >= 1 && G <= 3 && 128 * G + D <= static_cast<int>(kTmemCols), "TMEM budget");
    constexpr int kKB = D / 64;   // 64-element (128-byte) column blocks per row
    constexpr uint32_t kTmemO = R::kTmemO;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int H = args.H;
    const int unit = blockIdx.x / H;
    const int h = blockIdx.x - unit * H;
    if (unit >= *args.unit_count) return;   // whole CTA, before any barrier or TMEM use
    const int4 wu = args.units[unit];
    const int q0 = wu.x, q_end = wu.y, k0 = wu.z, nk = wu.w;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
    float* tb_s = reinterpret_cast<float*>(smem + L::kOffTB);
    MetaStage* meta = reinterpret_cast<MetaStage*>(smem + L::kOffMeta);
    const bool use_time = args.ts != nullptr && args.tb != nullptr && args.NB > 0;
    const int nbm1 = use_time ? args.NB - 1 : 0;

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(&bars[kBarQFull], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBarKFull + s], 1);
            mbar_init(&bars[kBarKFree + s], 1);
            mbar_init(&bars[kBarVFull + s], 1);
            mbar_init(&bars[kBarVFree + s], 1);
        }
        for (int b = 0; b < G; ++b) {
            mbar_init(&bars[kBarSFull + b], 1 + 32);
            mbar_init(&bars[kBarPFull + b], 128);
        }
        mbar_init(&bars[kBarOFull], 1);
        mbar_init(&bars[kBarDrain], 1);
        mbar_fence_init();
    }
    if (warp == R::kWarpMMA) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp < R::kPointwiseWarps) {
        for (int b = tid; b < kMaxTimeBuckets; b += 32 * R::kPointwiseWarps)
            tb_s[b] = (use_time && b < args.NB) ? 0.5f * args.tb[static_cast<int64_t>(h) * args.NB + b] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t sQ = smem_u32(smem + L::kOffQ);
    const uint32_t sK = smem_u32(smem + L::kOffK);
    const uint32_t sV = smem_u32(smem + L::kOffV);

    if (warp == R::kWarpTMA) {
        // ------------------------------------------------------------ TMA producers
        if (lane < 2) {
            const bool is_k = lane == 0;
            const CUtensorMap* tm = is_k ? &tmK : &tmV;
            const int ring = is_k ? L::kOffK : L::kOffV;
            uint64_t* full = &bars[is_k ? kBarKFull : kBarVFull];
            uint64_t* freeb = &bars[is_k ? kBarKFree : kBarVFree];
            tma_prefetch_desc(tm);
            if (is_k) {
                tma_prefetch_desc(&tmQ);
                mbar_arrive_expect_tx(&bars[kBarQFull], L::kQBytes);
#pragma unroll
                for (int kb = 0; kb < kKB; ++kb)
                    tma_load_2d(smem + L::kOffQ + kb * 16384, &tmQ, &bars[kBarQFull], h * D + kb * 64, q0);
            }
            int issued0 = 0, issued1 = 0;
            for (int j = 0; j < nk; ++j) {
                const int s = j & 1;
                if (j >= 2 && !mbar_wait(&freeb[s], ((j >> 1) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], L::kKVBytes);
                const int kt0 = k0 + j * kTile;
#pragma unroll
                for (int kb = 0; kb < kKB; ++kb)
                    tma_load_2d(smem + ring + s * L::kKVBytes + kb * 16384, tm, &full[s],
                                h * D + kb * 64, kt0);
                if (s == 0) ++issued0; else ++issued1;
            }
            // drain: every copy this thread started has landed before the CTA ends
            if (is_k && !mbar_wait(&bars[kBarQFull], 0, nullptr)) raise_error(kErrTimeout);
            if (issued0 > 0 && !mbar_wait(&full[0], (issued0 - 1) & 1, nullptr)) raise_error(kErrTimeout);
            if (issued1 > 0 && !mbar_wait(&full[1], (issued1 - 1) & 1, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if (warp == R::kWarpMMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            auto issue_pv = [&](int jj) -> bool {
                const int b = jj % G;
                const int sv = jj & 1;
                if (!mbar_wait(&bars[kBarPFull + b], (jj / G) & 1, abort_flag)) return false;
                if (!mbar_wait(&bars[kBarVFull + sv], (jj >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vb = sV + sv * L::kKVBytes;
                const uint32_t pb = tmem + b * 128;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    // keys 16kk..16kk+15: columns 32*(kk/2) + 8*(kk%2) of the P buffer
                    const uint32_t a = pb + (kk >> 1) * 32 + (kk & 1) * 8;
                    const uint64_t bd = desc_mnmajor_sw128(vb + kk * 2048, 16384);
                    umma_bf16_ts(tmem + kTmemO, a, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[kBarVFree + sv]);
                return true;
            };
            bool ok = mbar_wait(&bars[kBarQFull], 0, abort_flag);
            int pv_next = 0;
            for (int j = 0; ok && j < nk; ++j) {
                const int s = j & 1;
                // buffer j%G last held P_j-G, read by PV_j-G, issued earlier by this thread
                ok = mbar_wait(&bars[kBarKFull + s], (j >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb_base = sK + s * L::kKVBytes;
                const uint32_t sb = tmem + (j % G) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_bf16_ss(sb, desc_kmajor_sw128(sQ + off), desc_kmajor_sw128(kb_base + off),
                                 idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[kBarSFull + j % G]);
                umma_commit(&bars[kBarKFree + s]);
                if (j >= G - 1) {
                    ok = issue_pv(pv_next);
                    ++pv_next;
                }
            }
            while (ok && pv_next < nk) {
                ok = issue_pv(pv_next);
                ++pv_next;
            }
            if (ok) umma_commit(&bars[kBarOFull]);
            umma_commit(&bars[kBarDrain]);
            if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if (warp == R::kWarpMeta) {
        // ------------------------------------------------------------ bias staging
        for (int j = 0; j < nk; ++j) {
            const int b = j % G;
            // stage b last served tile j-G; P_j-G written means it has been read
            if (j >= G && !warp_wait(&bars[kBarPFull + b], ((j / G) - 1) & 1, abort_flag)) break;
            MetaStage& ms = meta[b];
            const int kt0 = k0 + j * kTile;
            // relative-position window, pre-halved (8 + 4 independent loads per lane)
            float wv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int mm = lane + 32 * u;
                wv[u] = 0.f;
                if (args.pos && mm < 255) {
                    int64_t dd = static_cast<int64_t>(q0) - kt0 - 127 + mm;
                    dd = dd < 0 ? 0 : (dd > args.P - 1 ? args.P - 1 : dd);
                    wv[u] = args.pos[static_cast<int64_t>(h) * args.P + dd];
                }
            }
            int64_t tv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t key = static_cast<int64_t>(kt0) + lane + 32 * u;
                tv[u] = use_time ? args.ts[key < args.T ? key : args.T - 1] : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) ms.w[lane + 32 * u] = 0.5f * wv[u];
            int64_t tmin = INT64_MAX, tmax = INT64_MIN;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int mm = lane + 32 * u;
                ms.kt64[mm] = tv[u];
                ms.kt32[mm] = static_cast<int32_t>(static_cast<uint64_t>(tv[u]));
                if (kt0 + mm < q_end) {
                    tmin = tv[u] < tmin ? tv[u] : tmin;
                    tmax = tv[u] > tmax ? tv[u] : tmax;
                }
            }
            __syncwarp();
            bool mono = true;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int mm = lane + 32 * u;
                if (mm < 127 && kt0 + mm + 1 < q_end) mono = mono && (ms.kt64[mm] <= ms.kt64[mm + 1]);
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
        }
    } else {
        // ------------------------------------------------------------ pointwise stage
        const int g = warp >> 2;                            // group: tiles j = g (mod G)
        const int qd = warp & 3;                            // TMEM lane quarter
        const int r = qd * 32 + lane;                       // query row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const int64_t i = static_cast<int64_t>(q0) + r;
        const bool row_valid = i < q_end;
        const int64_t ti = (use_time && row_valid) ? args.ts[i < args.T ? i : args.T - 1] : 0;
        const int32_t ti32 = static_cast<int32_t>(static_cast<uint64_t>(ti));
        // register table: lane L holds time/2 of bucket min((L + 1) mod 32, NB - 1)
        const float tbr = tb_s[min((lane + 1) & 31, nbm1)];
        const MetaStage& ms = meta[g];
        const uint32_t s_col = tmem + lane_base + static_cast<uint32_t>(g * 128);
        bool ok = true;
        for (int j = g; j < nk; j += G) {
            ok = warp_wait(&bars[kBarSFull + g], (j / G) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const int kt0 = k0 + j * kTile;
            const int lo = k0 - kt0;                        // first key of the sequence
            const int hi = row_valid ? static_cast<int>(i - kt0) : -1;
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
                uint32_t sv[32];
                uint32_t pk[16];
                __syncwarp();
                tmem_ld32(s_col + c0, sv);
                const bool full = __all_sync(0xffffffffu, lo <= c0 && hi >= c0 + 31);
                bool done = false;
                if (!fast_w) {
                    if (full) pw_slow<false>(sv, c0, wrow, ms.kt64, ti, tb_s, nbm1, lo, hi, pk);
                    else pw_slow<true>(sv, c0, wrow, ms.kt64, ti, tb_s, nbm1, lo, hi, pk);
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
            tc_fence_before();
            mbar_arrive(&bars[kBarPFull + g]);
        }
        if (g < 2 && ok && warp_wait(&bars[kBarOFull], 0, abort_flag)) {
            tc_fence_after();
            __nv_bfloat16* orow = args.out + i * args.out_stride + static_cast<int64_t>(h) * D;
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
                const int col = g * (D / 2) + ch * 32;
                uint32_t ov[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + kTmemO + col, ov);
                if (row_valid) {
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * args.inv_n,
                                            __uint_as_float(ov[2 * e + 1]) * args.inv_n);
                    uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(wv[4 * q], wv[4 * q + 1], wv[4 * q + 2], wv[4 * q + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) raise_error(kErrTimeout);
    if (warp == R::kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace hstu
