// Device bodies shared by the standalone router / permutation kernels and the
// fused decode front kernel (each translation unit gets its own copy).
#pragma once

#include "common.cuh"

namespace moe {

// a ranks above b: larger logit; ties -> lower index; NaN below everything.
__device__ __forceinline__ bool ranks_above(float a, int ia, float b, int ib)
{
    bool na = isnan(a), nb = isnan(b);
    if (na != nb) return nb;
    if (na) return ia < ib;
    if (a != b) return a > b;
    return ia < ib;
}

// Top-k of one token's logits (row lt of E) by one warp, with the logits in
// registers (EPL per lane, expert lane + 32 i in slot i; E <= 32 EPL): k rounds
// of arg-max over the experts not yet taken, then exp(l - lmax) renormalised
// over the k chosen.  Lane j < k writes choice j to idx[j], w[j].
template <int EPL>
__device__ __forceinline__ void topk_token(const float* __restrict__ lt, int E, int k, int lane,
                                           int32_t* __restrict__ idx, float* __restrict__ w)
{
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; i++) v[i] = (lane + 32 * i < E) ? lt[lane + 32 * i] : 0.0f;
    uint32_t avail = 0;   // bit i: expert lane + 32 i exists and is not taken
#pragma unroll
    for (int i = 0; i < EPL; i++)
        if (lane + 32 * i < E) avail |= 1u << i;
    float my_l = 0.0f;
    int my_i = 0;
    for (int r = 0; r < k; r++) {
        float bv = 0.0f;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < EPL; i++)
            if (((avail >> i) & 1) && (bi < 0 || ranks_above(v[i], lane + 32 * i, bv, bi))) {
                bv = v[i];
                bi = lane + 32 * i;
            }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (oi >= 0 && (bi < 0 || ranks_above(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) avail &= ~(1u << (bi >> 5));
        if (lane == r) { my_l = bv; my_i = bi; }
    }
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    float p = (lane < k) ? expf(my_l - lmax) : 0.0f;
    float z = p;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
        idx[lane] = my_i;
        w[lane] = p / z;
    }
}

constexpr int kSmallA = 1024;   // assignments the one-CTA permutation handles
constexpr int kSmallE = 1024;   // experts the one-CTA permutation handles

struct PermSmem {
    int idx[kSmallA];
    int cnt[kSmallE];
    int warp[32];
    int tot;
};

// The permutation of A <= kSmallA assignments over E <= kSmallE experts by one
// 1024-thread CTA: per-expert counts, their exclusive scan (offsets), and each
// assignment's row = its expert's offset + its rank among earlier assignments
// to the same expert.  Every thread of the CTA calls it.
__device__ __forceinline__ void perm_small_body(const int32_t* __restrict__ idx, int A, int E,
                                                int32_t* __restrict__ offsets, int32_t* __restrict__ row_of,
                                                int32_t* __restrict__ assign_of, PermSmem& S)
{
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    for (int e = tid; e < E; e += blockDim.x) S.cnt[e] = 0;
    __syncthreads();
    for (int a = tid; a < A; a += blockDim.x) {
        int e = idx[a];
        if (e < 0 || e >= E) e = -1;          // out-of-range experts get no row
        S.idx[a] = e;
        if (e >= 0) atomicAdd(&S.cnt[e], 1);  // integer counts: order-independent
    }
    __syncthreads();
    // offsets: exclusive scan of the counts (E <= blockDim.x)
    const int v = (tid < E) ? S.cnt[tid] : 0;
    int inc = v;
    for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) S.warp[w] = inc;
    __syncthreads();
    if (w == 0) {
        int x = (lane < (int)(blockDim.x >> 5)) ? S.warp[lane] : 0;
        int xi = x;
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, xi, off);
            if (lane >= off) xi += o;
        }
        S.warp[lane] = xi - x;
        if (lane == 31) S.tot = xi;
    }
    __syncthreads();
    const int excl = S.warp[w] + inc - v;
    __syncthreads();
    if (tid < E) {
        offsets[tid] = excl;
        S.cnt[tid] = excl;                    // reuse as the base row of each expert
    }
    if (tid == 0) offsets[E] = S.tot;
    __syncthreads();
    for (int a = tid; a < A; a += blockDim.x) {
        const int e = S.idx[a];
        if (e < 0) {
            row_of[a] = -1;
            continue;
        }
        int rank = 0;
        for (int b = 0; b < a; b++) rank += (S.idx[b] == e);
        const int row = S.cnt[e] + rank;
        row_of[a] = row;
        assign_of[row] = a;
    }
}

}  // namespace moe
