// common.cuh -- device error word and the integer bias-index functions shared
// by the attention kernels and the bias-index test hook.
#pragma once

#include <cstdint>

namespace hstu {

// Per-device error word. Bits: kErrTimeout (a bounded wait gave up),
// kErrBadInput (offsets decrease or a sequence is longer than max_seqlen).
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;
constexpr unsigned int kErrBadInput = 2u;

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

constexpr int kTile = 128;          // query rows and keys per tile
constexpr int kMaxTimeBuckets = 1024;
constexpr int kMaxSeqlen = 131072;  // 1024 query tiles per sequence

// Log-time bucket, 64-bit path: clamp(floor(log2(max(1, dt))), 0, nb - 1).
// floor(log2) of a positive integer is the index of its most significant set
// bit, taken with the hardware bit-find on the high or the low word.
__device__ __forceinline__ int time_bucket64(int64_t dt, int nb_minus_1) {
    if (dt < 1) dt = 1;
    const uint32_t hi = static_cast<uint32_t>(static_cast<uint64_t>(dt) >> 32);
    const uint32_t lo = static_cast<uint32_t>(dt);
    const int msb = hi ? 32 + (31 - __clz(hi)) : (31 - __clz(lo));
    return min(msb, nb_minus_1);
}

// 1023 + floor(log2(x)) for 1 <= x < 2^32 (the biased exponent x would have
// as a double), from a count of leading zeros. The time-bias register table
// is indexed by this value modulo 32. (An earlier form built the double
// 2^52 + x and subtracted 2^52 on the FP64 pipe; on B200 that chain sat on
// the critical path of every 32-key chunk and cost about 9% of the kernel.)
__device__ __forceinline__ uint32_t log2_exponent_field(uint32_t x) {
    return 1054u - static_cast<uint32_t>(__clz(x));
}

// Same bucket for a difference already known to fit in int32.
__device__ __forceinline__ int time_bucket32(int32_t dt, int nb_minus_1) {
    const int k = static_cast<int>(log2_exponent_field(static_cast<uint32_t>(max(dt, 1)))) - 1023;
    return min(k, nb_minus_1);
}

// Relative-position index min(i - j, P - 1), clamped at 0 for pairs that the
// causal mask removes anyway (keeps every table read in bounds).
__device__ __forceinline__ int pos_index(int64_t i, int64_t j, int num_pos) {
    int64_t r = i - j;
    r = r < 0 ? 0 : r;
    return static_cast<int>(r > num_pos - 1 ? num_pos - 1 : r);
}

}  // namespace hstu
