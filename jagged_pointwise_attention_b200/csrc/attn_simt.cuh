// attn_simt.cuh -- fp32 HSTU jagged causal attention on CUDA cores.
//
// One thread per (query token, head): the thread walks the keys of its own
// sequence up to the diagonal, accumulating silu(s_ij) v_j in fp32 registers.
// SiLU uses the accurate expf so the path stays within fp32 rounding of the
// definition. Intended for small fp32 problems; the bf16 path is the fast one.
#pragma once

#include "common.cuh"

namespace hstu {

struct AttnF32Args {
    const float* q;
    int64_t q_stride;
    const float* k;
    int64_t k_stride;
    const float* v;
    int64_t v_stride;
    const int64_t* seq_offsets;
    int B;
    int64_t T;
    int H, dqk, dv;
    const int64_t* ts;
    const float* pos;
    int P;
    const float* tb;
    int NB;
    float inv_n;
    float* out;
    int64_t out_stride;
};

// largest b with seq_offsets[b] <= t (offsets non-decreasing)
__device__ __forceinline__ int find_sequence(const int64_t* __restrict__ off, int B, int64_t t) {
    int lo = 0, hi = B;   // invariant: off[lo] <= t < off[hi] (off[B] = T > t)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

template <int DMAX>
__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(const AttnF32Args a) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int h = blockIdx.y;
    if (i >= a.T) return;
    const int b = find_sequence(a.seq_offsets, a.B, i);
    const int64_t o = a.seq_offsets[b];
    float qi[DMAX];
    float acc[DMAX];
#pragma unroll
    for (int c = 0; c < DMAX; ++c) {
        qi[c] = c < a.dqk ? a.q[i * a.q_stride + h * a.dqk + c] : 0.f;
        acc[c] = 0.f;
    }
    const int64_t ti = a.ts ? a.ts[i] : 0;
    const int nbm1 = a.NB - 1;
    for (int64_t j = o; j <= i; ++j) {
        const float* kj = a.k + j * a.k_stride + h * a.dqk;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < DMAX; ++c)
            if (c < a.dqk) s = fmaf(qi[c], kj[c], s);
        if (a.pos) s += a.pos[static_cast<int64_t>(h) * a.P + pos_index(i, j, a.P)];
        if (a.ts && a.tb) s += a.tb[static_cast<int64_t>(h) * a.NB + time_bucket64(ti - a.ts[j], nbm1)];
        const float p = s / (1.0f + expf(-s));
        const float* vj = a.v + j * a.v_stride + h * a.dv;
#pragma unroll
        for (int c = 0; c < DMAX; ++c)
            if (c < a.dv) acc[c] = fmaf(p, vj[c], acc[c]);
    }
    float* orow = a.out + i * a.out_stride + h * a.dv;
#pragma unroll
    for (int c = 0; c < DMAX; ++c)
        if (c < a.dv) orow[c] = acc[c] * a.inv_n;
}

}  // namespace hstu
