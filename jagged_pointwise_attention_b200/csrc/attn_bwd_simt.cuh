// attn_bwd_simt.cuh -- backward of the HSTU jagged causal attention, fp32 on
// CUDA cores (the pages' reference implementation has forward and backward
// attention kernels; generative-recommenders README, "HSTU Ultra attention
// benchmark"). With s_ij = q_i.k_j + pos + time, p_ij = silu(s_ij) / N and
// out_i = sum_j p_ij v_j, for an upstream gradient dout:
//   ds_ij = (dout_i . v_j) silu'(s_ij) / N, silu'(s) = sig(s)(1 + s(1 - sig(s)))
//   dq_i = sum_{j<=i} ds_ij k_j                      (query pass)
//   dk_j = sum_{i>=j} ds_ij q_i, dv_j = sum_{i>=j} p_ij dout_i   (key pass)
//   dpos[h][min(i-j, P-1)] += ds_ij, dtime[h][bucket] += ds_ij   (query pass)
// Two passes, one warp per (token, head) each (lanes split the head
// dimension, dot products reduced by shuffles), scores recomputed in both, so
// no gradient of q, k or v needs an atomic; the table gradients collect in
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

__device__ __forceinline__ float silu_grad_f(float s) {
    const float sg = 1.0f / (1.0f + expf(-s));
    return sg * (1.0f + s * (1.0f - sg));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Bias of pair (i, j) (sequence start o): adds pos and time to s and returns
// their table indices (-1 when the term is absent). Lane-uniform.
__device__ __forceinline__ float pair_bias(const AttnBwdArgs& a, int h, int64_t i, int64_t j,
                                           int* pidx, int* bkt) {
    float bias = 0.f;
    *pidx = -1;
    *bkt = -1;
    if (a.pos) {
        *pidx = pos_index(i, j, a.P);
        bias += __ldg(a.pos + static_cast<int64_t>(h) * a.P + *pidx);
    }
    if (a.ts && a.tb) {
        *bkt = time_bucket64(__ldg(a.ts + i) - __ldg(a.ts + j), a.NB - 1);
        bias += __ldg(a.tb + static_cast<int64_t>(h) * a.NB + *bkt);
    }
    return bias;
}

// Query pass: one warp per (query row i, head), lane l holding elements l,
// l + 32, ... of q_i, dout_i and dq_i; dq_i and the table gradients.
// Dynamic shared memory: P + NB floats, the block's partial table gradients
// for head blockIdx.y. The time-table gradient of consecutive keys (which
// mostly share a bucket) is summed in a register and added once per run.
template <int DMAX>
__global__ void __launch_bounds__(128) attn_bwd_q_kernel(const AttnBwdArgs a) {
    constexpr int NE = DMAX / 32;
    extern __shared__ float tabs[];
    float* spos = tabs;
    float* stime = tabs + (a.pos ? a.P : 0);
    const int h = blockIdx.y, lane = threadIdx.x & 31;
    const int ntab = (a.pos ? a.P : 0) + ((a.ts && a.tb) ? a.NB : 0);
    for (int e = threadIdx.x; e < ntab; e += blockDim.x) tabs[e] = 0.f;
    __syncthreads();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (i < a.T) {
        const int b = find_sequence(a.seq_offsets, a.B, i);
        const int64_t o = a.seq_offsets[b];
        float qi[NE], gi[NE], dq[NE];
#pragma unroll
        for (int t = 0; t < NE; ++t) {
            const int c = lane + 32 * t;
            qi[t] = c < a.dqk ? a.q[(i * a.H + h) * a.dqk + c] : 0.f;
            gi[t] = c < a.dv ? a.dout[(i * a.H + h) * a.dv + c] : 0.f;
            dq[t] = 0.f;
        }
        int run_bkt = -1;
        float run = 0.f;
        // U keys per step: their shuffle reductions are independent
        constexpr int U = 4;
        for (int64_t j0 = o; j0 <= i; j0 += U) {
            const int nu = static_cast<int>(i - j0 + 1 < U ? i - j0 + 1 : U);
            float kk[U][NE], sp[U], dpp[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                sp[u] = dpp[u] = 0.f;
                const int64_t j = j0 + (u < nu ? u : 0);
                const float* kj = a.k + (j * a.H + h) * a.dqk;
                const float* vj = a.v + (j * a.H + h) * a.dv;
#pragma unroll
                for (int t = 0; t < NE; ++t) {
                    const int c = lane + 32 * t;
                    kk[u][t] = c < a.dqk ? kj[c] : 0.f;
                    sp[u] = fmaf(qi[t], kk[u][t], sp[u]);
                    if (c < a.dv) dpp[u] = fmaf(gi[t], vj[c], dpp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                sp[u] = warp_sum(sp[u]);
                dpp[u] = warp_sum(dpp[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (u >= nu) break;
                int pidx, bkt;
                const float s = sp[u] + pair_bias(a, h, i, j0 + u, &pidx, &bkt);
                const float ds = dpp[u] * silu_grad_f(s) * a.inv_n;
#pragma unroll
                for (int t = 0; t < NE; ++t) dq[t] = fmaf(ds, kk[u][t], dq[t]);
                if (lane == 0) {
                    if (pidx >= 0) atomicAdd(&spos[pidx], ds);
                    if (bkt >= 0) {
                        if (bkt != run_bkt) {
                            if (run_bkt >= 0) atomicAdd(&stime[run_bkt], run);
                            run_bkt = bkt;
                            run = 0.f;
                        }
                        run += ds;
                    }
                }
            }
        }
        if (lane == 0 && run_bkt >= 0) atomicAdd(&stime[run_bkt], run);
#pragma unroll
        for (int t = 0; t < NE; ++t) {
            const int c = lane + 32 * t;
            if (c < a.dqk) a.dq[(i * a.H + h) * a.dqk + c] = dq[t];
        }
    }
    __syncthreads();
    if (a.dpos)
        for (int e = threadIdx.x; e < a.P; e += blockDim.x)
            if (spos[e] != 0.f) atomicAdd(&a.dpos[static_cast<int64_t>(h) * a.P + e], spos[e]);
    if (a.dtime)
        for (int e = threadIdx.x; e < a.NB; e += blockDim.x)
            if (stime[e] != 0.f) atomicAdd(&a.dtime[static_cast<int64_t>(h) * a.NB + e], stime[e]);
}

// Key pass: one warp per (key row j, head), lanes over the elements as in the
// query pass; dk_j and dv_j.
template <int DMAX>
__global__ void __launch_bounds__(128) attn_bwd_kv_kernel(const AttnBwdArgs a) {
    constexpr int NE = DMAX / 32;
    const int h = blockIdx.y, lane = threadIdx.x & 31;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (j >= a.T) return;
    const int b = find_sequence(a.seq_offsets, a.B, j);
    const int64_t end = a.seq_offsets[b + 1];
    float kj[NE], vj[NE], dk[NE], dv[NE];
#pragma unroll
    for (int t = 0; t < NE; ++t) {
        const int c = lane + 32 * t;
        kj[t] = c < a.dqk ? a.k[(j * a.H + h) * a.dqk + c] : 0.f;
        vj[t] = c < a.dv ? a.v[(j * a.H + h) * a.dv + c] : 0.f;
        dk[t] = dv[t] = 0.f;
    }
    // U queries per step: their shuffle reductions are independent
    constexpr int U = 4;
    for (int64_t i0 = j; i0 < end; i0 += U) {
        const int nu = static_cast<int>(end - i0 < U ? end - i0 : U);
        float qq[U][NE], gg[U][NE], sp[U], dpp[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            sp[u] = dpp[u] = 0.f;
            const int64_t i = i0 + (u < nu ? u : 0);
            const float* qi = a.q + (i * a.H + h) * a.dqk;
            const float* gi = a.dout + (i * a.H + h) * a.dv;
#pragma unroll
            for (int t = 0; t < NE; ++t) {
                const int c = lane + 32 * t;
                qq[u][t] = c < a.dqk ? qi[c] : 0.f;
                gg[u][t] = c < a.dv ? gi[c] : 0.f;
                sp[u] = fmaf(qq[u][t], kj[t], sp[u]);
                dpp[u] = fmaf(gg[u][t], vj[t], dpp[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            sp[u] = warp_sum(sp[u]);
            dpp[u] = warp_sum(dpp[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (u >= nu) break;
            int pidx, bkt;
            const float s = sp[u] + pair_bias(a, h, i0 + u, j, &pidx, &bkt);
            const float p = s / (1.0f + expf(-s)) * a.inv_n;
            const float ds = dpp[u] * silu_grad_f(s) * a.inv_n;
#pragma unroll
            for (int t = 0; t < NE; ++t) {
                dk[t] = fmaf(ds, qq[u][t], dk[t]);
                dv[t] = fmaf(p, gg[u][t], dv[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NE; ++t) {
        const int c = lane + 32 * t;
        if (c < a.dqk) a.dk[(j * a.H + h) * a.dqk + c] = dk[t];
        if (c < a.dv) a.dvv[(j * a.H + h) * a.dv + c] = dv[t];
    }
}

}  // namespace hstu
