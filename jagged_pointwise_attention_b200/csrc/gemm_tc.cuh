// gemm_tc.cuh -- y = epilogue(x W^T + b) on tcgen05 for the HSTU layer's two
// projections (UVQK with SiLU, output projection with the residual add), in
// bf16 or with row-wise E4M3 operands (FP8: y = epilogue((xq wq^T) * sx[m] *
// sw[n] + b), generative-recommenders README, "FP8 linear reference and
// benchmark").
//
// Persistent: one CTA per SM walks output tiles of 128 x BN (BN = 256 when N
// allows, else 128) in row-block-major order, so the CTAs running together
// share each 128-row block of x in L2 while W (at most a few MB) stays there.
// K streams in 128-byte swizzled blocks (64 bf16 or 128 E4M3 elements)
// through a 4-stage TMA ring; the fp32 accumulator of a tile lives in TMEM,
// two buffers of BN columns, so the epilogue of one tile overlaps the main
// loop of the next, and a buffer is handed back as soon as its last columns
// are in registers.
//
// Warp roles: EW epilogue warps (EW/4 per TMEM lane quarter, one row per
// thread, 4 BN / EW columns each), then the TMA producer, then the MMA issuer
// and TMEM owner. EW = 8 where the tensor pipe or the operand feed bounds a
// tile (bf16 projections, the residual epilogue); EW = 16 for the FP8 SiLU
// projection, whose tile the epilogue bounds: with four warps per scheduler
// the SFU (one tanh per output) stays busy while other warps wait on TMEM or
// memory. The epilogue writes each 32 x 32 block of results into shared
// memory (64-byte swizzle, conflict-free) and one lane stores it with a TMA
// bulk store (two staging buffers per warp with EW = 8, one with EW = 16);
// the store clips rows past M. With the residual epilogue the block's
// residual is first loaded into the same buffer by TMA, one block ahead.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

constexpr int kGemmStages = 4;

// epilogue warps of a projection: 16 for the FP8 SiLU projection, else 8
template <int EPI, bool FP8>
struct GemmEpiWarps {
    static constexpr int value = (FP8 && EPI == 1) ? 16 : 8;
};

struct GemmArgs {
    int64_t M;
    int N, K;
    const float* sx;                // FP8: [M] row scales of x
    const float* sw;                // FP8: [N] row scales of W
    const float* bias;              // [N] or null
    const __nv_bfloat16* residual;  // [M, N] (ldr) or null
    int64_t ldr;
    __nv_bfloat16* y;
    int64_t ldy;
};

template <int BN, int EW>
struct GemmSmem {
    static constexpr int kOutBufs = EW == 8 ? 2 : 1;                  // staging buffers per warp
    static constexpr int kBBytes = BN * 128;                          // B block: BN rows x 64
    static constexpr int kStageBytes = 16384 + kBBytes;
    static constexpr int kOffA = 0;                                   // [stage] 16 KB
    static constexpr int kOffB = kOffA + kGemmStages * 16384;         // [stage] BN x 128 B
    static constexpr int kOffOut = kOffB + kGemmStages * kBBytes;     // [warp][buf] 32 x 64 B
    static constexpr int kOffBar = kOffOut + EW * kOutBufs * 2048;
    static constexpr int kOffTmem = kOffBar + 32 * 8;
    static constexpr int kOffAbort = kOffTmem + 8;
    static constexpr int kBytes = kOffAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory per block");
};

// FP8 dequantization of one thread's 32 accumulators of row m, columns
// col0..col0+31: f *= sx[m] * sw[col] (16-byte loads of sw when aligned).
__device__ __forceinline__ void scale_fp8(float (&f)[32], const GemmArgs& g, int64_t m, int col0) {
    const float rs = __ldg(g.sx + min(m, g.M - 1));
    if ((reinterpret_cast<uintptr_t>(g.sw) & 15) == 0) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const float4 w = __ldg(reinterpret_cast<const float4*>(g.sw + col0) + e4);
            f[4 * e4] *= rs * w.x;
            f[4 * e4 + 1] *= rs * w.y;
            f[4 * e4 + 2] *= rs * w.z;
            f[4 * e4 + 3] *= rs * w.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] *= rs * __ldg(g.sw + col0 + e);
    }
}

// EPI: hstu_epilogue_t (0 none, 1 silu, 2 residual)
template <int EPI, int BN, bool FP8 = false, int EW = GemmEpiWarps<EPI, FP8>::value>
__global__ void __launch_bounds__((EW + 2) * 32, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmR,
                 const GemmArgs g) {
    using L = GemmSmem<BN, EW>;
    constexpr int S = kGemmStages;
    constexpr int kWarpTMA = EW, kWarpMMA = EW + 1;
    static_assert(BN == 128 || BN == 256, "tile width");
    static_assert(EW == 8 || (EW == 16 && EPI != 2), "the residual epilogue runs with 8 warps");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kKBlock = FP8 ? 128 : 64;   // elements per 128-byte k-block
    const int nkb = g.K / kKBlock;
    const int tiles_n = g.N / BN;
    const int tiles = static_cast<int>((g.M + 127) / 128) * tiles_n;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;      // [2]
    uint64_t* acc_empty = acc_full + 2;  // [2]
    uint64_t* drain = acc_empty + 2;
    uint64_t* res_full = drain + 1;      // [epilogue warp][2]: residual block landed (EW = 8)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 32 * EW);
        }
        mbar_init(drain, 1);
        if (EPI == 2)
            for (int b = 0; b < 2 * EW; ++b) mbar_init(&res_full[b], 1);
        mbar_fence_init();
    }
    if (warp == kWarpMMA) {
        tmem_alloc(tmem_slot, 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sA = smem_u32(smem + L::kOffA);
    const uint32_t sB = smem_u32(smem + L::kOffB);

    if (warp == kWarpTMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int it = 0;          // k-blocks loaded, over all tiles
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const int m0 = (t / tiles_n) * 128, n0 = (t % tiles_n) * BN;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], L::kStageBytes);
                    tma_load_2d(smem + L::kOffA + s * 16384, &tmA, &full[s], kb * kKBlock, m0);
                    tma_load_2d(smem + L::kOffB + s * L::kBBytes, &tmB, &full[s], kb * kKBlock, n0);
                }
            }
            // drain: stage s took ceil((it - s) / S) loads
            for (int s = 0; s < S; ++s) {
                const int c = it > s ? (it - s + S - 1) / S : 0;
                if (c > 0 && !mbar_wait(&full[s], (c - 1) & 1, nullptr)) raise_error(kErrTimeout);
            }
        }
        __syncwarp();
    } else if (warp == kWarpMMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = FP8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN, 0, 0);
            int it = 0, tl = 0;  // k-blocks consumed; tiles of this CTA
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tl) {
                const int buf = tl & 1;
                if (tl >= 2 && !mbar_wait(&acc_empty[buf], ((tl >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&full[s], (it / S) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // four MMAs of 32 bytes of K each (K = 16 bf16 or 32 E4M3)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t da = desc_kmajor_sw128(sA + s * 16384 + kk * 32);
                        const uint64_t db = desc_kmajor_sw128(sB + s * L::kBBytes + kk * 32);
                        if (FP8) umma_f8_ss(acc, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        else umma_bf16_ss(acc, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&acc_full[buf]);
            }
            umma_commit(drain);
            if (!mbar_wait(drain, 0, nullptr)) raise_error(kErrTimeout);
        }
        __syncwarp();
    } else if constexpr (EW == 8) {
        // ------------------------------------------------------------ epilogue, 8 warps
        const int q = warp & 3, h = warp >> 2;          // lane quarter, column half
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint8_t* stage_out = smem + L::kOffOut + warp * 2 * 2048;
        uint64_t* rbar = res_full + 2 * warp;
        constexpr int kBlocks = BN / 64;                // 32-column blocks per warp and tile
        // residual block ch of tile t into staging buffer b (lane 0)
        auto load_res = [&](int t, int ch, int b) {
            mbar_arrive_expect_tx(&rbar[b], 2048);
            tma_load_2d(stage_out + b * 2048, &tmR, &rbar[b],
                        (t % tiles_n) * BN + h * (BN / 2) + ch * 32, (t / tiles_n) * 128 + q * 32);
        };
        if (lane == 0) {
            tma_prefetch_desc(&tmY);
            if (EPI == 2) {
                tma_prefetch_desc(&tmR);
                if (static_cast<int>(blockIdx.x) < tiles) load_res(blockIdx.x, 0, 0);
            }
        }
        int nst = 0;                                    // blocks this warp has stored
        int nres = EPI == 2 && static_cast<int>(blockIdx.x) < tiles ? 1 : 0;  // residual loads issued
        bool eok = true;
        int tl = 0;
        for (int t = blockIdx.x; eok && t < tiles; t += gridDim.x, ++tl) {
            const int buf = tl & 1;
            const int m0 = (t / tiles_n) * 128, n0 = (t % tiles_n) * BN;
            if (!warp_wait(&acc_full[buf], (tl >> 1) & 1, abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < BN / 64; ++ch, ++nst) {
                const int c = h * (BN / 2) + ch * 32;   // column within the tile
                const int col0 = n0 + c;
                uint32_t v[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * BN + c), v);
                if (ch == kBlocks - 1) {
                    // the whole accumulator is in registers: hand the buffer back
                    tc_fence_before();
                    mbar_arrive(&acc_empty[buf]);
                }
                uint8_t* sb = stage_out + (nst & 1) * 2048;
                if (EPI == 2) {
                    // this block's residual (loaded one block ahead)
                    if (!warp_wait(&rbar[nst & 1], (nst >> 1) & 1, abort_flag)) {
                        eok = false;
                        break;
                    }
                } else {
                    // the store that last read this staging buffer is done with it
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                }
                {
                    float f[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
                    if (FP8) scale_fp8(f, g, m0 + q * 32 + lane, col0);
                    if (g.bias) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) f[e] += __ldg(g.bias + col0 + e);
                    }
                    if (EPI == 1) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) f[e] = silu_tanh(f[e]);
                    }
                    if (EPI == 2) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            const uint4 w = *reinterpret_cast<const uint4*>(
                                sb + lane * 64 + ((qq ^ ((lane >> 1) & 3)) << 4));
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                f[8 * qq + 2 * u] += __uint_as_float(ww[u] << 16);
                                f[8 * qq + 2 * u + 1] += __uint_as_float(ww[u] & 0xffff0000u);
                            }
                        }
                    }
                    // row `lane` of the block: 16-byte unit qq at qq ^ ((lane >> 1) & 3)
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        *reinterpret_cast<uint4*>(sb + lane * 64 + ((qq ^ ((lane >> 1) & 3)) << 4)) =
                            make_uint4(pack_bf16x2(f[8 * qq], f[8 * qq + 1]),
                                       pack_bf16x2(f[8 * qq + 2], f[8 * qq + 3]),
                                       pack_bf16x2(f[8 * qq + 4], f[8 * qq + 5]),
                                       pack_bf16x2(f[8 * qq + 6], f[8 * qq + 7]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, sb, col0, m0 + q * 32);
                    bulk_commit_group();
                    if (EPI == 2) {
                        // the next block's residual into the other buffer, once the
                        // store that last read it is done
                        const int nt = ch + 1 < kBlocks ? t : t + static_cast<int>(gridDim.x);
                        if (nt < tiles) {
                            bulk_wait_group_read<1>();
                            load_res(nt, ch + 1 < kBlocks ? ch + 1 : 0, (nst + 1) & 1);
                            ++nres;
                        }
                    }
                }
            }
            if (!eok) break;
        }
        if (lane == 0) {
            bulk_wait_group_all();
            // a residual load issued for a block never reached (an early exit)
            if (nres > nst && !mbar_wait(&rbar[nst & 1], (nst >> 1) & 1, nullptr))
                raise_error(kErrTimeout);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue, 16 warps
        const int q = warp & 3, hq = warp >> 2;         // lane quarter, column quarter
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint8_t* sb = smem + L::kOffOut + warp * 2048;
        constexpr int kChunks = BN / 128;               // 32-column blocks per warp and tile
        if (lane == 0) tma_prefetch_desc(&tmY);
        int tl = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
            const int buf = tl & 1;
            const int m0 = (t / tiles_n) * 128, n0 = (t % tiles_n) * BN;
            if (!warp_wait(&acc_full[buf], (tl >> 1) & 1, abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < kChunks; ++ch) {
                const int c = hq * (BN / 4) + ch * 32;  // column within the tile
                const int col0 = n0 + c;
                uint32_t v[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * BN + c), v);
                if (ch == kChunks - 1) {
                    // the whole accumulator is in registers: hand the buffer back
                    tc_fence_before();
                    mbar_arrive(&acc_empty[buf]);
                }
                float f[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
                if (FP8) scale_fp8(f, g, m0 + q * 32 + lane, col0);
                if (g.bias) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) f[e] += __ldg(g.bias + col0 + e);
                }
                if (EPI == 1) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) f[e] = silu_tanh(f[e]);
                }
                // the store that last read the staging buffer is done with it
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
                // row `lane` of the block: 16-byte unit qq at qq ^ ((lane >> 1) & 3)
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    *reinterpret_cast<uint4*>(sb + lane * 64 + ((qq ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(pack_bf16x2(f[8 * qq], f[8 * qq + 1]),
                                   pack_bf16x2(f[8 * qq + 2], f[8 * qq + 3]),
                                   pack_bf16x2(f[8 * qq + 4], f[8 * qq + 5]),
                                   pack_bf16x2(f[8 * qq + 6], f[8 * qq + 7]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, sb, col0, m0 + q * 32);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) raise_error(kErrTimeout);
    if (warp == kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BN);
    }
}

}  // namespace hstu
