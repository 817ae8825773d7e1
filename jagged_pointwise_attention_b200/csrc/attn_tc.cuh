// attn_tc.cuh -- bf16 HSTU jagged causal attention forward on tcgen05.
//
// One CTA computes one (128-row query tile, head) work unit. For every key
// tile j of the unit (causal tiles only):
//     S_j  = Q K_j^T                         tcgen05.mma, SMEM x SMEM -> TMEM (fp32)
//     P_j  = silu(S_j + pos + time) * mask   TMEM -> registers -> bf16 SMEM
//     O   += P_j V_j                          tcgen05.mma, SMEM x SMEM -> TMEM (fp32)
// and finally out = O / max_seqlen (bf16). There is no softmax: no running
// max, no rescale, no row sum, so O accumulates untouched across key tiles.
//
// Warp roles (224 threads):
//   warps 0-3  pointwise stage: one query row (TMEM lane) per thread
//   warp 4     TMA producer: Q once, K/V tiles into a 2-stage ring
//   warp 5     MMA issuer (one thread) and TMEM owner
//   warp 6     bias staging: key timestamps and the relative-position window
// TMEM (512 columns): S double buffer at 0 and 128, O at 256.
// Every wait is bounded; a wait that runs out raises kErrTimeout, the other
// roles notice through a shared abort flag, and the CTA drains its own
// copies and MMAs before it frees TMEM and exits.
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

template <int D>
struct AttnSmem {
    static constexpr int kQBytes = kTile * D * 2;       // Q tile, D/64 swizzled 16 KB blocks
    static constexpr int kKVBytes = kTile * D * 2;      // one K (or V) stage
    static constexpr int kPBytes = kTile * kTile * 2;   // P tile, 2 swizzled 16 KB blocks
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + 2 * kKVBytes;
    static constexpr int kOffP = kOffV + 2 * kKVBytes;
    static constexpr int kOffTB = kOffP + kPBytes;                  // float[kMaxTimeBuckets]
    static constexpr int kOffW = kOffTB + kMaxTimeBuckets * 4;      // float[2][256]
    static constexpr int kOffKT64 = kOffW + 2 * 256 * 4;            // int64[2][128]
    static constexpr int kOffKT32 = kOffKT64 + 2 * 128 * 8;         // int32[2][128]
    static constexpr int kOffTMinMax = kOffKT32 + 2 * 128 * 4;      // int64[2][2]
    static constexpr int kOffBar = kOffTMinMax + 64;
    static constexpr int kNumBars = 16;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;                    // 1 KB alignment slack
};

constexpr int kAttnThreads = 224;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

// barrier slots
enum {
    kBarQFull = 0,
    kBarKVFull = 1,    // +stage
    kBarKVFree = 3,    // +stage
    kBarSFull = 5,     // +buffer
    kBarSFree = 7,     // +buffer
    kBarPFull = 9,
    kBarPFree = 10,
    kBarOFull = 11,
    kBarDrain = 12,
    kBarMeta = 13,     // +buffer
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t bfind_u32(uint32_t x) {
    uint32_t r;
    asm("bfind.u32 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

// Pointwise stage for one 32-column chunk of S. kFast: every valid pair of
// this warp has |t_i - t_j| < 2^31, so 32-bit differences are exact.
// kMask: some pair of this warp's rows lies outside [lo, hi] (causal/sequence).
template <bool kFast, bool kMask>
__device__ __forceinline__ void pointwise_chunk(const uint32_t (&sv)[32], int c_base,
                                                const float* __restrict__ wrow,
                                                const float* __restrict__ tb_s,
                                                const int32_t* __restrict__ kt32,
                                                const int64_t* __restrict__ kt64, int32_t ti32,
                                                int64_t ti, int nbm1, int lo, int hi,
                                                uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float p[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = c_base + e + u;
            float x = __uint_as_float(sv[e + u]) + wrow[-c];
            int bkt;
            if (kFast) {
                const int32_t dt = static_cast<int32_t>(static_cast<uint32_t>(ti32) -
                                                        static_cast<uint32_t>(kt32[c]));
                bkt = min(static_cast<int>(bfind_u32(static_cast<uint32_t>(max(dt, 1)))), nbm1);
            } else {
                bkt = time_bucket64(ti - kt64[c], nbm1);
            }
            x += tb_s[bkt];
            float y = silu_tanh(x);
            if (kMask) y = (c >= lo && c <= hi) ? y : 0.0f;
            p[u] = y;
        }
        pk[e >> 1] = pack_bf16x2(p[0], p[1]);
    }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
    using L = AttnSmem<D>;
    static_assert(D == 64 || D == 128, "head dim");
    constexpr int kKB = D / 64;   // 64-element (128-byte) column blocks per row

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
    float* w_s = reinterpret_cast<float*>(smem + L::kOffW);
    int64_t* kt64_s = reinterpret_cast<int64_t*>(smem + L::kOffKT64);
    int32_t* kt32_s = reinterpret_cast<int32_t*>(smem + L::kOffKT32);
    int64_t* tmm_s = reinterpret_cast<int64_t*>(smem + L::kOffTMinMax);

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(&bars[kBarQFull], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBarKVFull + s], 1);
            mbar_init(&bars[kBarKVFree + s], 1);
            mbar_init(&bars[kBarSFull + s], 1);
            mbar_init(&bars[kBarSFree + s], 128);
            mbar_init(&bars[kBarMeta + s], 32);
        }
        mbar_init(&bars[kBarPFull], 128);
        mbar_init(&bars[kBarPFree], 1);
        mbar_init(&bars[kBarOFull], 1);
        mbar_init(&bars[kBarDrain], 1);
        mbar_fence_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid < 128) {
        for (int b = tid; b < args.NB; b += 128) tb_s[b] = args.tb ? args.tb[h * args.NB + b] : 0.f;
        if (args.NB <= 0 && tid == 0) tb_s[0] = 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t sQ = smem_u32(smem + L::kOffQ);
    const uint32_t sK = smem_u32(smem + L::kOffK);
    const uint32_t sV = smem_u32(smem + L::kOffV);
    const uint32_t sP = smem_u32(smem + L::kOffP);

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bars[kBarQFull], L::kQBytes);
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb)
                tma_load_2d(smem + L::kOffQ + kb * 16384, &tmQ, &bars[kBarQFull], h * D + kb * 64, q0);
            int issued[2] = {0, 0};
            for (int j = 0; j < nk; ++j) {
                const int s = j & 1;
                if (j >= 2 && !mbar_wait(&bars[kBarKVFree + s], ((j >> 1) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&bars[kBarKVFull + s], 2 * L::kKVBytes);
                const int kt0 = k0 + j * kTile;
#pragma unroll
                for (int kb = 0; kb < kKB; ++kb) {
                    tma_load_2d(smem + L::kOffK + s * L::kKVBytes + kb * 16384, &tmK,
                                &bars[kBarKVFull + s], h * D + kb * 64, kt0);
                    tma_load_2d(smem + L::kOffV + s * L::kKVBytes + kb * 16384, &tmV,
                                &bars[kBarKVFull + s], h * D + kb * 64, kt0);
                }
                ++issued[s];
            }
            // drain: every copy this thread started has landed before the CTA ends
            if (!mbar_wait(&bars[kBarQFull], 0, nullptr)) raise_error(kErrTimeout);
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0 && !mbar_wait(&bars[kBarKVFull + s], (issued[s] - 1) & 1, nullptr))
                    raise_error(kErrTimeout);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            auto issue_pv = [&](int jj) -> bool {
                if (!mbar_wait(&bars[kBarPFull], jj & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vb = sV + (jj & 1) * L::kKVBytes;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t a = desc_kmajor_sw128(sP + (kk >> 2) * 16384 + (kk & 3) * 32);
                    const uint64_t b = desc_mnmajor_sw128(vb + kk * 2048, 16384);
                    umma_bf16_ss(tmem + kTmemO, a, b, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[kBarPFree]);
                umma_commit(&bars[kBarKVFree + (jj & 1)]);
                return true;
            };
            bool ok = mbar_wait(&bars[kBarQFull], 0, abort_flag);
            for (int j = 0; ok && j < nk; ++j) {
                const int s = j & 1;
                ok = mbar_wait(&bars[kBarKVFull + s], (j >> 1) & 1, abort_flag);
                if (ok && j >= 2) ok = mbar_wait(&bars[kBarSFree + s], ((j >> 1) - 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb_base = sK + s * L::kKVBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_bf16_ss(tmem + s * 128, desc_kmajor_sw128(sQ + off),
                                 desc_kmajor_sw128(kb_base + off), idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[kBarSFull + s]);
                if (j >= 1) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(nk - 1);
            if (ok) umma_commit(&bars[kBarOFull]);
            umma_commit(&bars[kBarDrain]);
            if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if (warp == 6) {
        // ------------------------------------------------------------ bias staging
        for (int j = 0; j < nk; ++j) {
            const int s = j & 1;
            if (j >= 2 && !warp_wait(&bars[kBarSFree + s], ((j >> 1) - 1) & 1, abort_flag)) break;
            const int kt0 = k0 + j * kTile;
            int64_t tmin = INT64_MAX, tmax = INT64_MIN;
            for (int m = lane; m < kTile; m += 32) {
                const int64_t key = static_cast<int64_t>(kt0) + m;
                int64_t t = 0;
                if (args.ts) {
                    t = args.ts[key < args.T ? key : args.T - 1];
                    if (key < q_end) {
                        tmin = t < tmin ? t : tmin;
                        tmax = t > tmax ? t : tmax;
                    }
                }
                kt64_s[s * 128 + m] = t;
                kt32_s[s * 128 + m] = static_cast<int32_t>(static_cast<uint64_t>(t));
            }
            // window w[m] = pos[h][clamp(q0 - kt0 - 127 + m, 0, P-1)], m = 127 + r - c
            for (int m = lane; m < 256; m += 32) {
                float wv = 0.f;
                if (args.pos && m < 255) {
                    int64_t dd = static_cast<int64_t>(q0) - kt0 - 127 + m;
                    dd = dd < 0 ? 0 : (dd > args.P - 1 ? args.P - 1 : dd);
                    wv = args.pos[static_cast<int64_t>(h) * args.P + dd];
                }
                w_s[s * 256 + m] = wv;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const int64_t a = __shfl_xor_sync(0xffffffffu, tmin, o);
                const int64_t b = __shfl_xor_sync(0xffffffffu, tmax, o);
                tmin = a < tmin ? a : tmin;
                tmax = b > tmax ? b : tmax;
            }
            if (lane == 0) {
                tmm_s[s * 2 + 0] = tmin;
                tmm_s[s * 2 + 1] = tmax;
            }
            __syncwarp();
            mbar_arrive(&bars[kBarMeta + s]);
        }
    } else {
        // ------------------------------------------------------------ pointwise stage
        const int r = tid;                                  // query row = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const int64_t i = static_cast<int64_t>(q0) + r;
        const bool row_valid = i < q_end;
        const int64_t ti = (args.ts && row_valid) ? args.ts[i < args.T ? i : args.T - 1] : 0;
        const int32_t ti32 = static_cast<int32_t>(static_cast<uint64_t>(ti));
        const int nbm1 = args.NB > 0 ? args.NB - 1 : 0;
        uint32_t pk[64];
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const int s = j & 1;
            ok = warp_wait(&bars[kBarMeta + s], (j >> 1) & 1, abort_flag);
            if (ok) ok = warp_wait(&bars[kBarSFull + s], (j >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const int kt0 = k0 + j * kTile;
            const int lo = k0 - kt0;                        // first key of the sequence
            const int hi = row_valid ? static_cast<int>(i - kt0) : -1;
            const int64_t tmin = tmm_s[s * 2 + 0], tmax = tmm_s[s * 2 + 1];
            bool fast = true;
            if (row_valid && args.ts && tmin <= tmax) {
                const int64_t lo_t = ti < tmin ? ti : tmin;
                const int64_t hi_t = ti > tmax ? ti : tmax;
                fast = static_cast<uint64_t>(hi_t) - static_cast<uint64_t>(lo_t) < (1ull << 31);
            }
            const bool fast_w = __all_sync(0xffffffffu, fast);
            const bool full_w = __all_sync(0xffffffffu, lo <= 0 && hi >= kTile - 1);
            const float* wrow = w_s + s * 256 + 127 + r;
            const int32_t* kt32 = kt32_s + s * 128;
            const int64_t* kt64 = kt64_s + s * 128;
            const uint32_t s_col = tmem + lane_base + static_cast<uint32_t>(s * 128);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t sv[32];
                __syncwarp();
                tmem_ld32(s_col + ch * 32, sv);
                uint32_t* pkc = pk + ch * 16;
                if (fast_w) {
                    if (full_w)
                        pointwise_chunk<true, false>(sv, ch * 32, wrow, tb_s, kt32, kt64, ti32, ti, nbm1, lo, hi, pkc);
                    else
                        pointwise_chunk<true, true>(sv, ch * 32, wrow, tb_s, kt32, kt64, ti32, ti, nbm1, lo, hi, pkc);
                } else {
                    if (full_w)
                        pointwise_chunk<false, false>(sv, ch * 32, wrow, tb_s, kt32, kt64, ti32, ti, nbm1, lo, hi, pkc);
                    else
                        pointwise_chunk<false, true>(sv, ch * 32, wrow, tb_s, kt32, kt64, ti32, ti, nbm1, lo, hi, pkc);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[kBarSFree + s]);
            if (j >= 1 && !warp_wait(&bars[kBarPFree], (j - 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            // P row r -> two 128 B-swizzled K-major blocks (keys 0-63, 64-127)
            const uint32_t prow = sP + r * 128;
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) {
                const uint32_t addr = prow + (c16 >> 3) * 16384 + (((c16 & 7) ^ (r & 7)) << 4);
                st_shared_v4(addr, pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars[kBarPFull]);
        }
        if (ok && warp_wait(&bars[kBarOFull], 0, abort_flag)) {
            tc_fence_after();
            __nv_bfloat16* orow = args.out + i * args.out_stride + static_cast<int64_t>(h) * D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ov[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + kTmemO + ch * 32, ov);
                if (row_valid) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * args.inv_n,
                                           __uint_as_float(ov[2 * e + 1]) * args.inv_n);
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) raise_error(kErrTimeout);
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace hstu
