// attn_bwd_simt.cuh -- backward of the HSTU jagged causal attention, fp32 on
// CUDA cores (the pages' reference implementation has forward and backward
// attention kernels; generative-recommenders README, "HSTU Ultra attention
// benchmark"). With s_ij = q_i.k_j + pos + time, p_ij = silu(s_ij) / N and
// out_i = sum_j p_ij v_j, for an upstream gradient dout:
//   ds_ij = (dout_i . v_j) silu'(s_ij) / N, silu'(s) = sig(s)(1 + s(1 - sig(s)))
//   dq_i = sum_{j<=i} ds_ij k_j                      (query pass)
//   dk_j = sum_{i>=j} ds_ij q_i, dv_j = sum_{i>=j} p_ij dout_i   (key pass)
//   dpos[h][min(i-j, P-1)] += ds_ij, dtime[h][bucket] += ds_ij   (query pass)
// Two passes, one thread per (token, head) each, scores recomputed in both,
// so no gradient of q, k or v needs an atomic; the table gradients collect in
// shared memory per block and then in global memory with atomics. A first
// correct version: the contractions belong on the tensor cores next.
#pragma once

#include "attn_simt.cuh"
#include "common.cuh"

namespace hstu {

struct AttnBwdArgs {
    const float* q;             // [T, H, dqk] contiguous
    const float* k;
    const float* v;             // [T, H, dv]
    const float* dout;          // [T, H, dv]
    const int64_t* seq_offsets;
    int B;
    int64_t T;
    int H, dqk, dv;
    const int64_t* ts;          // [T] or null
    const float* pos;           // [H, P] or null
    int P;
    const float* tb;            // [H, NB] or null
    int NB;
    float inv_n;
    float* dq;                  // [T, H, dqk]
    float* dk;
    float* dvv;                 // [T, H, dv]
    float* dpos;                // [H, P] (zeroed before) or null
    float* dtime;               // [H, NB] (zeroed before) or null
};

__device__ __forceinline__ float score_ij(const AttnBwdArgs& a, const float* qi, const float* kj,
                                          int h, int64_t i, int64_t j, int64_t o, int* pidx,
                                          int* bkt) {
    float s = 0.f;
    for (int c = 0; c < a.dqk; ++c) s = fmaf(qi[c], kj[c], s);
    *pidx = -1;
    *bkt = -1;
    if (a.pos) {
        *pidx = pos_index(i - o, j - o, a.P);
        s += a.pos[static_cast<int64_t>(h) * a.P + *pidx];
    }
    if (a.ts && a.tb) {
        *bkt = time_bucket64(a.ts[i] - a.ts[j], a.NB - 1);
        s += a.tb[static_cast<int64_t>(h) * a.NB + *bkt];
    }
    return s;
}

__device__ __forceinline__ float silu_grad_f(float s) {
    const float sg = 1.0f / (1.0f + expf(-s));
    return sg * (1.0f + s * (1.0f - sg));
}

// Query pass: dq_i and the table gradients. Dynamic shared memory: P + NB
// floats (the block's partial table gradients for head blockIdx.y).
template <int DMAX>
__global__ void __launch_bounds__(128) attn_bwd_q_kernel(const AttnBwdArgs a) {
    extern __shared__ float tabs[];
    float* spos = tabs;
    float* stime = tabs + (a.pos ? a.P : 0);
    const int h = blockIdx.y;
    const int ntab = (a.pos ? a.P : 0) + ((a.ts && a.tb) ? a.NB : 0);
    for (int e = threadIdx.x; e < ntab; e += blockDim.x) tabs[e] = 0.f;
    __syncthreads();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < a.T) {
        const int b = find_sequence(a.seq_offsets, a.B, i);
        const int64_t o = a.seq_offsets[b];
        const float* qi = a.q + (i * a.H + h) * a.dqk;
        const float* gi = a.dout + (i * a.H + h) * a.dv;
        float dq[DMAX];
#pragma unroll
        for (int c = 0; c < DMAX; ++c) dq[c] = 0.f;
        for (int64_t j = o; j <= i; ++j) {
            const float* kj = a.k + (j * a.H + h) * a.dqk;
            const float* vj = a.v + (j * a.H + h) * a.dv;
            int pidx, bkt;
            const float s = score_ij(a, qi, kj, h, i, j, o, &pidx, &bkt);
            float dp = 0.f;
            for (int c = 0; c < a.dv; ++c) dp = fmaf(gi[c], vj[c], dp);
            const float ds = dp * silu_grad_f(s) * a.inv_n;
#pragma unroll
            for (int c = 0; c < DMAX; ++c)
                if (c < a.dqk) dq[c] = fmaf(ds, kj[c], dq[c]);
            if (pidx >= 0) atomicAdd(&spos[pidx], ds);
            if (bkt >= 0) atomicAdd(&stime[bkt], ds);
        }
        float* dqi = a.dq + (i * a.H + h) * a.dqk;
#pragma unroll
        for (int c = 0; c < DMAX; ++c)
            if (c < a.dqk) dqi[c] = dq[c];
    }
    __syncthreads();
    if (a.dpos)
        for (int e = threadIdx.x; e < a.P; e += blockDim.x)
            if (spos[e] != 0.f) atomicAdd(&a.dpos[static_cast<int64_t>(h) * a.P + e], spos[e]);
    if (a.dtime)
        for (int e = threadIdx.x; e < a.NB; e += blockDim.x)
            if (stime[e] != 0.f) atomicAdd(&a.dtime[static_cast<int64_t>(h) * a.NB + e], stime[e]);
}

// Key pass: dk_j and dv_j.
template <int DMAX>
__global__ void __launch_bounds__(128) attn_bwd_kv_kernel(const AttnBwdArgs a) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int h = blockIdx.y;
    if (j >= a.T) return;
    const int b = find_sequence(a.seq_offsets, a.B, j);
    const int64_t o = a.seq_offsets[b], end = a.seq_offsets[b + 1];
    const float* kj = a.k + (j * a.H + h) * a.dqk;
    const float* vj = a.v + (j * a.H + h) * a.dv;
    float dk[DMAX], dv[DMAX];
#pragma unroll
    for (int c = 0; c < DMAX; ++c) dk[c] = dv[c] = 0.f;
    for (int64_t i = j; i < end; ++i) {
        const float* qi = a.q + (i * a.H + h) * a.dqk;
        const float* gi = a.dout + (i * a.H + h) * a.dv;
        int pidx, bkt;
        const float s = score_ij(a, qi, kj, h, i, j, o, &pidx, &bkt);
        const float p = s / (1.0f + expf(-s)) * a.inv_n;
        float dp = 0.f;
        for (int c = 0; c < a.dv; ++c) dp = fmaf(gi[c], vj[c], dp);
        const float ds = dp * silu_grad_f(s) * a.inv_n;
#pragma unroll
        for (int c = 0; c < DMAX; ++c) {
            if (c < a.dqk) dk[c] = fmaf(ds, qi[c], dk[c]);
            if (c < a.dv) dv[c] = fmaf(p, gi[c], dv[c]);
        }
    }
    float* dkj = a.dk + (j * a.H + h) * a.dqk;
    float* dvj = a.dvv + (j * a.H + h) * a.dv;
#pragma unroll
    for (int c = 0; c < DMAX; ++c) {
        if (c < a.dqk) dkj[c] = dk[c];
        if (c < a.dv) dvj[c] = dv[c];
    }
}

}  // namespace hstu
