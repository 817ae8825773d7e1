// quant_fp8.cuh -- row-wise E4M3 quantization of a bf16 matrix (the operands
// of the FP8 projections; generative-recommenders README, "FP8 linear
// reference and benchmark").
//
// Per row r: amax = max |x[r, :]|, inv = 448 / amax and scale = amax / 448
// (fp32, rounded to nearest; an all-zero row takes inv 0, scale 1), and
// code = E4M3(x * inv) with the product rounded to fp32 and the conversion
// rounding to nearest, ties to even, saturating at +-448. One warp per row;
// each lane reads 8 bf16 (16 bytes) per step and writes 8 codes.
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

__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const QuantArgs a) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.M) return;
    const __nv_bfloat16* xr = a.x + row * a.ldx;
    // |x| of a bf16 is its fp32 bit pattern without the sign, and for finite
    // values the unsigned order of those patterns is the order of the values
    uint32_t amax_bits = 0u;
    for (int c = lane * 8; c < a.K; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax_bits = max(amax_bits, (w[i] << 16) & 0x7fffffffu);
            amax_bits = max(amax_bits, w[i] & 0x7fff0000u);
        }
    }
    amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
    const float amax = __uint_as_float(amax_bits);
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint8_t* qr = a.q + row * a.ldq;
    for (int c = lane * 8; c < a.K; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
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
        *reinterpret_cast<uint2*>(qr + c) = make_uint2(out[0], out[1]);
    }
    if (lane == 0) a.scales[row] = scale;
}

}  // namespace hstu
