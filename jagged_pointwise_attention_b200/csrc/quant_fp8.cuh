// quant_fp8.cuh -- row-wise E4M3 quantization of a bf16 matrix (the operands
// of the FP8 projections; generative-recommenders README, "FP8 linear
// reference and benchmark").
//
// Per row r: amax = max |x[r, :]|, inv = 448 / amax and scale = amax / 448
// (fp32, rounded to nearest), and code = E4M3(x * inv) with the product
// rounded to fp32 and the conversion rounding to nearest, ties to even,
// saturating at +-448. A row whose inv is not a finite fp32 number (all
// zeros, or amax below 448 / FLT_MAX) takes inv 0 and scale 1: zero codes.
// One warp per row; each lane reads 8 bf16 (16 bytes) per step and writes 8
// codes.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

struct QuantArgs {
    const __nv_bfloat16* x;
    int64_t ldx;
    int64_t M;
    int K;                  // multiple of 8
    uint8_t* q;
    int64_t ldq;
    float* scales;
};

// The codes of 8 consecutive values (one 16-byte load) at row offset c.
__device__ __forceinline__ uint2 e4m3_codes8(const uint4 v, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __fmul_rn(__uint_as_float(w[i] << 16), inv);
        const float hi = __fmul_rn(__uint_as_float(w[i] & 0xffff0000u), inv);
        // x of the pair goes to the lower byte
        const uint32_t pair = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE,
                                                       __NV_E4M3);
        if (i & 1) out[i >> 1] |= pair << 16;
        else out[i >> 1] = pair;
    }
    return make_uint2(out[0], out[1]);
}

// |x| of a bf16 is its fp32 bit pattern without the sign, and for finite
// values the unsigned order of those patterns is the order of the values.
__device__ __forceinline__ uint32_t amax_bits8(const uint4 v, uint32_t m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = max(m, (w[i] << 16) & 0x7fffffffu);
        m = max(m, w[i] & 0x7fff0000u);
    }
    return m;
}

// The row's (inv, scale) from its amax, as described above.
__device__ __forceinline__ float2 e4m3_row_factors(float amax) {
    const float q = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    const bool finite = amax > 0.f && q <= 3.402823466e38f;
    return make_float2(finite ? q : 0.f, finite ? __fdiv_rn(amax, 448.f) : 1.f);
}

// Rows of up to kQuantCached * 256 values are read once, into registers (all loads
// of a lane in flight together); longer rows are read twice.
constexpr int kQuantCached = 4;

__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const QuantArgs a) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.M) return;
    const __nv_bfloat16* xr = a.x + row * a.ldx;
    uint8_t* qr = a.q + row * a.ldq;
    const bool cached = a.K <= kQuantCached * 256;
    uint4 buf[kQuantCached];
    uint32_t amax_bits = 0u;
    if (cached) {
#pragma unroll
        for (int i = 0; i < kQuantCached; ++i) {
            const int c = lane * 8 + i * 256;
            buf[i] = c < a.K ? *reinterpret_cast<const uint4*>(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kQuantCached; ++i) amax_bits = amax_bits8(buf[i], amax_bits);
    } else {
        for (int c = lane * 8; c < a.K; c += 256)
            amax_bits = amax_bits8(*reinterpret_cast<const uint4*>(xr + c), amax_bits);
    }
    amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
    const float amax = __uint_as_float(amax_bits);
    const float2 f = e4m3_row_factors(amax);
    const float inv = f.x, scale = f.y;
    if (cached) {
#pragma unroll
        for (int i = 0; i < kQuantCached; ++i) {
            const int c = lane * 8 + i * 256;
            if (c < a.K) *reinterpret_cast<uint2*>(qr + c) = e4m3_codes8(buf[i], inv);
        }
    } else {
        for (int c = lane * 8; c < a.K; c += 256)
            *reinterpret_cast<uint2*>(qr + c) = e4m3_codes8(*reinterpret_cast<const uint4*>(xr + c), inv);
    }
    if (lane == 0) a.scales[row] = scale;
}

}  // namespace hstu
