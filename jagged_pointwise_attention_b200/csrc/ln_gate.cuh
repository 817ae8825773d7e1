// ln_gate.cuh -- Y = LayerNorm(A) * U (GATE) or Y = LayerNorm(A), one warp per
// token row; the block's eight warps stride over the rows, gamma and beta are
// staged in shared memory once per block.
//
// Each lane holds 8 contiguous features per 256-feature block (16-byte
// loads). Mean first, then the biased variance of the centred values (two
// passes over registers, so no cancellation), rsqrt(var + eps), affine, gate.
// With QUANT the bf16 result row is not stored but quantized row-wise to
// E4M3 (exactly as quant_rows_e4m3_kernel would quantize it): with the gate
// the fused output-normalization-to-FP8 step of the FP8 projections, without
// it the fused input-LayerNorm-to-FP8 step of the UVQK projection
// (generative-recommenders README, "FP8 linear reference and benchmark" and
// "HSTU Ultra attention benchmark").
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "quant_fp8.cuh"

namespace hstu {

struct LnGateArgs {
    const __nv_bfloat16* a;
    int64_t lda;
    const __nv_bfloat16* u;
    int64_t ldu;
    int64_t M;
    const float* gamma;
    const float* beta;
    float eps;
    __nv_bfloat16* y;
    int64_t ldy;
    uint8_t* yq;        // QUANT: E4M3 codes [M, F] (row stride ldyq) and row scales
    int64_t ldyq;
    float* ys;
};

__device__ __forceinline__ void unpack8(const uint4 w, float (&f)[8]) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(ww[q] << 16);
        f[2 * q + 1] = __uint_as_float(ww[q] & 0xffff0000u);
    }
}

template <int NV, bool QUANT = false, bool GATE = true>   // F = 256 * NV features
__global__ void __launch_bounds__(256) ln_gate_kernel(const LnGateArgs a) {
    constexpr int F = 256 * NV;
    // gamma and beta (identity where absent), staged once per block: every
    // warp reads them for each of its rows
    __shared__ __align__(16) float s_g[F];
    __shared__ __align__(16) float s_b[F];
    for (int c = threadIdx.x; c < F; c += blockDim.x) {
        s_g[c] = a.gamma ? a.gamma[c] : 1.f;
        s_b[c] = a.beta ? a.beta[c] : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t m = static_cast<int64_t>(blockIdx.x) * 8 + warp; m < a.M;
         m += static_cast<int64_t>(gridDim.x) * 8) {
        float x[NV][8];
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const uint4 w = *reinterpret_cast<const uint4*>(a.a + m * a.lda + k * 256 + lane * 8);
            unpack8(w, x[k]);
#pragma unroll
            for (int e = 0; e < 8; ++e) sum += x[k][e];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float mean = sum * (1.0f / F);
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float dlt = x[k][e] - mean;
                sq = fmaf(dlt, dlt, sq);
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        const float rstd = rsqrtf(sq * (1.0f / F) + a.eps);
        uint4 yrow[QUANT ? NV : 1];     // QUANT: the row's bf16 results, for the row amax
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int col = k * 256 + lane * 8;
            float uf[8];
            if (GATE) {
                unpack8(*reinterpret_cast<const uint4*>(a.u + m * a.ldu + col), uf);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) uf[e] = 1.f;
            }
            const float4 g0 = *reinterpret_cast<const float4*>(s_g + col);
            const float4 g1 = *reinterpret_cast<const float4*>(s_g + col + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(s_b + col);
            const float4 b1 = *reinterpret_cast<const float4*>(s_b + col + 4);
            const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float bt[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            uint32_t out[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float y0 = fmaf((x[k][2 * q] - mean) * rstd, g[2 * q], bt[2 * q]) * uf[2 * q];
                const float y1 = fmaf((x[k][2 * q + 1] - mean) * rstd, g[2 * q + 1], bt[2 * q + 1]) *
                                 uf[2 * q + 1];
                __nv_bfloat162 v2 = __floats2bfloat162_rn(y0, y1);
                out[q] = *reinterpret_cast<uint32_t*>(&v2);
            }
            if (QUANT) yrow[QUANT ? k : 0] = make_uint4(out[0], out[1], out[2], out[3]);
            else *reinterpret_cast<uint4*>(a.y + m * a.ldy + col) = make_uint4(out[0], out[1], out[2], out[3]);
        }
        if (QUANT) {
            uint32_t amax_bits = 0u;
#pragma unroll
            for (int k = 0; k < NV; ++k) amax_bits = amax_bits8(yrow[QUANT ? k : 0], amax_bits);
            amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
            const float amax = __uint_as_float(amax_bits);
            const float2 f = e4m3_row_factors(amax);
            const float inv = f.x;
#pragma unroll
            for (int k = 0; k < NV; ++k)
                *reinterpret_cast<uint2*>(a.yq + m * a.ldyq + k * 256 + lane * 8) =
                    e4m3_codes8(yrow[QUANT ? k : 0], inv);
            if (lane == 0) a.ys[m] = f.y;
        }
    }
}

}  // namespace hstu
