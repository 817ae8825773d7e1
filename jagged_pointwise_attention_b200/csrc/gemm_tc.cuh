// gemm_tc.cuh -- y = epilogue(x W^T + b) on tcgen05 for the HSTU layer's two
// projections (UVQK with SiLU, output projection with the residual add).
//
// Tile 128 x 128 per CTA, K in 64-element (128-byte swizzled) blocks through a
// 3-stage TMA ring; the fp32 accumulator lives in 128 TMEM columns. About
// 97 KB of shared memory, so two CTAs share an SM and one CTA's epilogue
// overlaps the other's main loop. Warp roles: 0-3 epilogue (one output row
// per thread), 4 TMA producer, 5 MMA issuer and TMEM owner.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 192;
constexpr int kGemmStageBytes = 2 * 128 * 64 * 2;   // A + B block, 32 KB

struct GemmArgs {
    int64_t M;
    int N, K;
    const float* bias;              // [N] or null
    const __nv_bfloat16* residual;  // [M, N] (ldr) or null
    int64_t ldr;
    __nv_bfloat16* y;
    int64_t ldy;
};

struct GemmSmem {
    static constexpr int kOffA = 0;                                   // [stage] 16 KB
    static constexpr int kOffB = kOffA + kGemmStages * 16384;         // [stage] 16 KB
    static constexpr int kOffBar = kOffB + kGemmStages * 16384;
    static constexpr int kOffTmem = kOffBar + 16 * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;
};

template <int EPI>   // hstu_epilogue_t: 0 none, 1 silu, 2 residual
__global__ void __launch_bounds__(kGemmThreads)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs g) {
    using L = GemmSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * 128;
    const int n0 = blockIdx.y * 128;
    const int nkb = g.K / 64;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* empty = full + kGemmStages;
    uint64_t* acc_full = empty + kGemmStages;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        mbar_fence_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sA = smem_u32(smem + L::kOffA);
    const uint32_t sB = smem_u32(smem + L::kOffB);

    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int issued[kGemmStages] = {0, 0, 0};
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kGemmStages;
                const int round = kb / kGemmStages;
                if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], kGemmStageBytes);
                tma_load_2d(smem + L::kOffA + s * 16384, &tmA, &full[s], kb * 64, m0);
                tma_load_2d(smem + L::kOffB + s * 16384, &tmB, &full[s], kb * 64, n0);
                ++issued[s];
            }
            for (int s = 0; s < kGemmStages; ++s)
                if (issued[s] > 0 && !mbar_wait(&full[s], (issued[s] - 1) & 1, nullptr))
                    raise_error(kErrTimeout);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kGemmStages;
                if (!mbar_wait(&full[s], (kb / kGemmStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_ss(tmem, desc_kmajor_sw128(sA + s * 16384 + kk * 32),
                                 desc_kmajor_sw128(sB + s * 16384 + kk * 32), idesc,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            if (ok) umma_commit(acc_full);
            umma_commit(drain);
            if (!mbar_wait(drain, 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else {
        const int r = tid;
        const int64_t row = static_cast<int64_t>(m0) + r;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag));
        if (ok) {
            tc_fence_after();
            const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t v[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + ch * 32, v);
                if (row < g.M) {
                    const int col0 = n0 + ch * 32;
                    float f[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        f[e] = __uint_as_float(v[e]);
                        if (g.bias) f[e] += g.bias[col0 + e];
                        if (EPI == 1) f[e] = __fdividef(f[e], 1.0f + __expf(-f[e]));
                    }
                    if (EPI == 2) {
                        const uint4* rp =
                            reinterpret_cast<const uint4*>(g.residual + row * g.ldr + col0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 w = rp[q];
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                f[8 * q + 2 * t] += __uint_as_float(ww[t] << 16);
                                f[8 * q + 2 * t + 1] += __uint_as_float(ww[t] & 0xffff0000u);
                            }
                        }
                    }
                    uint4* dst = reinterpret_cast<uint4*>(g.y + row * g.ldy + col0);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pack_bf16x2(f[8 * q], f[8 * q + 1]),
                                            pack_bf16x2(f[8 * q + 2], f[8 * q + 3]),
                                            pack_bf16x2(f[8 * q + 4], f[8 * q + 5]),
                                            pack_bf16x2(f[8 * q + 6], f[8 * q + 7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) raise_error(kErrTimeout);
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace hstu
