// debug.cuh -- test hooks: the bias indices the attention kernel computes, and
// a bounded wait that is made to run out.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

// One block per sequence. Entry e of the output is the pair (i, j <= i) of
// sequence b in row-major order, after the pairs of sequences 0..b-1.
// The bucket follows the attention kernel's choice: the 32-bit function when
// the difference fits in int32, the 64-bit one otherwise.
__global__ void __launch_bounds__(256)
bias_indices_kernel(const int64_t* __restrict__ seq_offsets, int B, const int64_t* __restrict__ ts,
                    int P, int NB, int* __restrict__ pos_out, int* __restrict__ bkt_out) {
    const int b = blockIdx.x;
    __shared__ long long base_s;
    if (threadIdx.x == 0) {
        long long base = 0;
        for (int c = 0; c < b; ++c) {
            const long long n = seq_offsets[c + 1] - seq_offsets[c];
            base += n * (n + 1) / 2;
        }
        base_s = base;
    }
    __syncthreads();
    const int64_t o = seq_offsets[b];
    const int64_t n = seq_offsets[b + 1] - o;
    for (int64_t i = 0; i < n; ++i) {
        const long long row = base_s + i * (i + 1) / 2;
        for (int64_t j = threadIdx.x; j <= i; j += blockDim.x) {
            if (pos_out) pos_out[row + j] = pos_index(i, j, P);
            if (bkt_out) {
                const int64_t dt = ts[o + i] - ts[o + j];
                int bk;
                if (dt >= INT32_MIN && dt <= INT32_MAX) {
                    const int32_t d32 = static_cast<int32_t>(static_cast<uint32_t>(ts[o + i]) -
                                                             static_cast<uint32_t>(ts[o + j]));
                    bk = time_bucket32(d32, NB - 1);
                } else {
                    bk = time_bucket64(dt, NB - 1);
                }
                bkt_out[row + j] = bk;
            }
        }
    }
}

// Waits on a barrier that nothing signals, for at most `limit` cycles, then
// records a timeout in the device error word and returns.
__global__ void wait_timeout_kernel(long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit)) raise_error(kErrTimeout);
}

}  // namespace hstu
