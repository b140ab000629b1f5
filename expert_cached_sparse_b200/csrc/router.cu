// Router: logits in a fixed fp32 order, then top-k and renormalised softmax
// weights.  Each token goes to a few of the layer's experts ("FreeToken
// linux", section "Como gestiona FreeToken la memoria MoE").
//
// The logit order is part of the contract (it decides integer outputs):
// for one (token, expert) pair, 32 lanes; lane l owns the 8-element chunks
// l, l+32, ... of the hidden dimension and accumulates them with fused
// multiply-adds in ascending order; an xor butterfly (16, 8, 4, 2, 1)
// then sums the lanes, leaving the same value in all of them.
#include "common.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

// 8 activations of chunk c of token row xrow, widened exactly to fp32.
template <bool XF32>
__device__ __forceinline__ void load_x8(const void* xrow, int c, float v[8])
{
    if (XF32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(xrow) + 8 * c);
        float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(xrow) + 8 * c));
        uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

// Warp per (token group of TB, expert group of EB).  TB tokens share each
// gate-row load, EB experts each activation load.  U chunks of every lane
// are loaded before their multiply-adds, so U loads per operand are in
// flight; the multiply-adds still run in the lane's ascending chunk order.
template <bool XF32, int TB, int EB, int U>
__global__ void __launch_bounds__(256) router_logits_kernel(const void* __restrict__ x,
                                                            const uint16_t* __restrict__ wg,
                                                            const float* __restrict__ bias, int n,
                                                            int H, int E, float* __restrict__ logits)
{
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int egroups = (E + EB - 1) / EB;
    const int tgroups = (n + TB - 1) / TB;
    const int chunks = H / 8;
    const size_t xrow_bytes = (size_t)H * (XF32 ? 4 : 2);
    for (int wi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wi < egroups * tgroups;
         wi += warps_total) {
        const int eg = wi % egroups, tg = wi / egroups;
        float acc[TB][EB];
#pragma unroll
        for (int a = 0; a < TB; a++)
#pragma unroll
            for (int b = 0; b < EB; b++) acc[a][b] = 0.0f;
        for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
            float xv[U][TB][8];
            uint4 wq[U][EB];
#pragma unroll
            for (int uu = 0; uu < U; uu++) {
                const int c = c0 + 32 * uu;
#pragma unroll
                for (int a = 0; a < TB; a++) {
                    int t = tg * TB + a;
                    if (c < chunks && t < n)
                        load_x8<XF32>(static_cast<const char*>(x) + (size_t)t * xrow_bytes, c, xv[uu][a]);
                    else
#pragma unroll
                        for (int i = 0; i < 8; i++) xv[uu][a][i] = 0.0f;
                }
#pragma unroll
                for (int b = 0; b < EB; b++) {
                    int e = eg * EB + b;
                    wq[uu][b] = (c < chunks && e < E)
                                    ? __ldg(reinterpret_cast<const uint4*>(wg + (size_t)e * H + 8 * c))
                                    : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int uu = 0; uu < U; uu++) {
                if (c0 + 32 * uu >= chunks) break;
#pragma unroll
                for (int b = 0; b < EB; b++) {
                    const uint32_t w4[4] = {wq[uu][b].x, wq[uu][b].y, wq[uu][b].z, wq[uu][b].w};
                    float wv[8];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        wv[2 * i] = __uint_as_float(w4[i] << 16);
                        wv[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
                    }
#pragma unroll
                    for (int a = 0; a < TB; a++)
#pragma unroll
                        for (int i = 0; i < 8; i++) acc[a][b] = __fmaf_rn(xv[uu][a][i], wv[i], acc[a][b]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < TB; a++)
#pragma unroll
            for (int b = 0; b < EB; b++)
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1)
                    acc[a][b] = __fadd_rn(acc[a][b], __shfl_xor_sync(0xffffffffu, acc[a][b], off));
        if (lane == 0) {
#pragma unroll
            for (int a = 0; a < TB; a++) {
                int t = tg * TB + a;
                if (t >= n) break;
#pragma unroll
                for (int b = 0; b < EB; b++) {
                    int e = eg * EB + b;
                    if (e >= E) break;
                    logits[(size_t)t * E + e] = bias ? __fadd_rn(acc[a][b], __ldg(bias + e)) : acc[a][b];
                }
            }
        }
    }
}

// Many tokens (prefill): a CTA computes a 32-token x 16-expert block of logits
// with both operand slices staged in shared memory as fp32.  K is walked in
// slices of 256 elements = 32 chunks of 8, so lane l of every warp owns chunk
// l of each slice: the per-(token, expert) order is the same fixed order as
// above (lane chunks ascending, then the xor butterfly).  Warp w owns tokens
// 4w..4w+3 and all 16 experts (64 accumulators per lane).  A staged row keeps
// the first four elements of every chunk, then the last four, so a warp's
// 16-byte reads of one half are 512 contiguous bytes (no bank conflicts).
constexpr int RT_TOK = 32, RT_EXP = 16, RT_K = 256;

template <bool XF32>
__global__ void __launch_bounds__(256) router_logits_tiled_kernel(const void* __restrict__ x,
                                                                  const uint16_t* __restrict__ wg,
                                                                  const float* __restrict__ bias, int n, int H,
                                                                  int E, float* __restrict__ logits)
{
    __shared__ __align__(16) float xs[RT_TOK][RT_K];
    __shared__ __align__(16) float ws[RT_EXP][RT_K];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int t0 = blockIdx.x * RT_TOK, e0 = blockIdx.y * RT_EXP;
    float acc[4][RT_EXP];
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < RT_EXP; b++) acc[a][b] = 0.0f;
    for (int k0 = 0; k0 < H; k0 += RT_K) {
        // stage: x slice (32 x 256) and gate slice (16 x 256) as fp32
        for (int i = tid; i < RT_TOK * RT_K / 8; i += 256) {
            const int r = i / (RT_K / 8), c = i % (RT_K / 8);
            const int t = t0 + r, k = k0 + 8 * c;
            float v[8];
            if (t < n && k < H) {
                if (XF32) {
                    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * H + k);
                    float4 a = __ldg(p), b = __ldg(p + 1);
                    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
                } else {
                    uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)t * H + k));
                    const uint32_t u4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        v[2 * j] = __uint_as_float(u4[j] << 16);
                        v[2 * j + 1] = __uint_as_float(u4[j] & 0xFFFF0000u);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; j++) v[j] = 0.0f;
            }
            *reinterpret_cast<float4*>(&xs[r][4 * c]) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(&xs[r][RT_K / 2 + 4 * c]) = make_float4(v[4], v[5], v[6], v[7]);
        }
        for (int i = tid; i < RT_EXP * RT_K / 8; i += 256) {
            const int r = i / (RT_K / 8), c = i % (RT_K / 8);
            const int e = e0 + r, k = k0 + 8 * c;
            float v[8];
            if (e < E && k < H) {
                uint4 q = __ldg(reinterpret_cast<const uint4*>(wg + (size_t)e * H + k));
                const uint32_t u4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    v[2 * j] = __uint_as_float(u4[j] << 16);
                    v[2 * j + 1] = __uint_as_float(u4[j] & 0xFFFF0000u);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; j++) v[j] = 0.0f;
            }
            *reinterpret_cast<float4*>(&ws[r][4 * c]) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(&ws[r][RT_K / 2 + 4 * c]) = make_float4(v[4], v[5], v[6], v[7]);
        }
        __syncthreads();
        if (k0 + 8 * lane < H) {   // lane's chunk exists in this slice
            float xv[4][8];
#pragma unroll
            for (int a = 0; a < 4; a++) {
                const float4 q0 = *reinterpret_cast<const float4*>(&xs[4 * w + a][4 * lane]);
                const float4 q1 = *reinterpret_cast<const float4*>(&xs[4 * w + a][RT_K / 2 + 4 * lane]);
                xv[a][0] = q0.x; xv[a][1] = q0.y; xv[a][2] = q0.z; xv[a][3] = q0.w;
                xv[a][4] = q1.x; xv[a][5] = q1.y; xv[a][6] = q1.z; xv[a][7] = q1.w;
            }
#pragma unroll
            for (int b = 0; b < RT_EXP; b++) {
                const float4 q0 = *reinterpret_cast<const float4*>(&ws[b][4 * lane]);
                const float4 q1 = *reinterpret_cast<const float4*>(&ws[b][RT_K / 2 + 4 * lane]);
                const float wv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                for (int a = 0; a < 4; a++)
#pragma unroll
                    for (int i = 0; i < 8; i++) acc[a][b] = __fmaf_rn(xv[a][i], wv[i], acc[a][b]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < RT_EXP; b++)
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                acc[a][b] = __fadd_rn(acc[a][b], __shfl_xor_sync(0xffffffffu, acc[a][b], off));
    // lane b of the warp writes expert e0+b for the warp's 4 tokens
#pragma unroll
    for (int a = 0; a < 4; a++) {
        const int t = t0 + 4 * w + a;
#pragma unroll
        for (int b = 0; b < RT_EXP; b++)
            if (lane == b && t < n && e0 + b < E)
                logits[(size_t)t * E + e0 + b] = bias ? __fadd_rn(acc[a][b], __ldg(bias + e0 + b)) : acc[a][b];
    }
}

// The same block of logits for bf16 x, with the operand slices copied
// raw (bf16) by cp.async into two buffers: the copies of slice s+1 are in
// flight while slice s is multiplied, and each lane widens its own x and
// gate chunks exactly when it reads them.  Lane l still owns chunk l of
// every slice and multiplies its 8 elements in order, so every logit is
// the same fp32 value as above.  Rows past n (or E) and chunks past H are
// zero-filled by the copy itself (source size 0).
__device__ __forceinline__ void cp_async16(void* smem, const void* src, uint32_t bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void widen8(uint4 q, float v[8])
{
    const uint32_t u4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        v[2 * j] = __uint_as_float(u4[j] << 16);
        v[2 * j + 1] = __uint_as_float(u4[j] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(256, 2) router_logits_pipe_kernel(const uint16_t* __restrict__ x,
                                                                    const uint16_t* __restrict__ wg,
                                                                    const float* __restrict__ bias, int n, int H,
                                                                    int E, float* __restrict__ logits)
{
    __shared__ __align__(16) uint16_t xs[2][RT_TOK][RT_K];
    __shared__ __align__(16) uint16_t ws[2][RT_EXP][RT_K];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int t0 = blockIdx.x * RT_TOK, e0 = blockIdx.y * RT_EXP;
    const int nsl = (H + RT_K - 1) / RT_K;
    auto stage = [&](int buf, int k0) {
        for (int i = tid; i < RT_TOK * RT_K / 8; i += 256) {
            const int r = i / (RT_K / 8), c = i % (RT_K / 8), t = t0 + r, k = k0 + 8 * c;
            const bool ok = t < n && k < H;
            cp_async16(&xs[buf][r][8 * c], ok ? x + (size_t)t * H + k : x, ok ? 16u : 0u);
        }
        for (int i = tid; i < RT_EXP * RT_K / 8; i += 256) {
            const int r = i / (RT_K / 8), c = i % (RT_K / 8), e = e0 + r, k = k0 + 8 * c;
            const bool ok = e < E && k < H;
            cp_async16(&ws[buf][r][8 * c], ok ? wg + (size_t)e * H + k : wg, ok ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    float acc[4][RT_EXP];
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < RT_EXP; b++) acc[a][b] = 0.0f;
    stage(0, 0);
    for (int s = 0; s < nsl; s++) {
        const int buf = s & 1, k0 = s * RT_K;
        if (s + 1 < nsl) {
            stage(buf ^ 1, k0 + RT_K);
            asm volatile("cp.async.wait_group 1;" ::: "memory");   // slice s has landed
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        if (k0 + 8 * lane < H) {   // lane's chunk exists in this slice
            float xv[4][8];
#pragma unroll
            for (int a = 0; a < 4; a++) widen8(*reinterpret_cast<const uint4*>(&xs[buf][4 * w + a][8 * lane]), xv[a]);
#pragma unroll
            for (int b = 0; b < RT_EXP; b++) {
                float wv[8];
                widen8(*reinterpret_cast<const uint4*>(&ws[buf][b][8 * lane]), wv);
#pragma unroll
                for (int a = 0; a < 4; a++)
#pragma unroll
                    for (int i = 0; i < 8; i++) acc[a][b] = __fmaf_rn(xv[a][i], wv[i], acc[a][b]);
            }
        }
        __syncthreads();   // buffer `buf` is refilled by the next iteration's copies
    }
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < RT_EXP; b++)
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                acc[a][b] = __fadd_rn(acc[a][b], __shfl_xor_sync(0xffffffffu, acc[a][b], off));
#pragma unroll
    for (int a = 0; a < 4; a++) {
        const int t = t0 + 4 * w + a;
#pragma unroll
        for (int b = 0; b < RT_EXP; b++)
            if (lane == b && t < n && e0 + b < E)
                logits[(size_t)t * E + e0 + b] = bias ? __fadd_rn(acc[a][b], __ldg(bias + e0 + b)) : acc[a][b];
    }
}

// Warp per token: k rounds of arg-max, then exp(l - lmax) renormalised.
__global__ void __launch_bounds__(128) router_topk_kernel(const float* __restrict__ logits, int n,
                                                          int E, int k, int32_t* __restrict__ idx,
                                                          float* __restrict__ w)
{
    extern __shared__ unsigned char s_taken[];  // [warps][E]
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    unsigned char* taken = s_taken + (size_t)wib * E;
    const int t = blockIdx.x * (blockDim.x >> 5) + wib;
    if (t >= n) return;
    const float* lt = logits + (size_t)t * E;
    for (int e = lane; e < E; e += 32) taken[e] = 0;
    __syncwarp();
    float my_l = 0.0f;
    int my_i = 0;
    for (int r = 0; r < k; r++) {
        float bv = 0.0f;
        int bi = -1;
        for (int e = lane; e < E; e += 32) {
            if (taken[e]) continue;
            float v = __ldg(lt + e);
            if (bi < 0 || ranks_above(v, e, bv, bi)) { bv = v; bi = e; }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (oi >= 0 && (bi < 0 || ranks_above(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        if (lane == 0) taken[bi] = 1;
        if (lane == r) { my_l = bv; my_i = bi; }
        __syncwarp();
    }
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    float p = (lane < k) ? expf(my_l - lmax) : 0.0f;
    float z = p;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_i;
        w[(size_t)t * k + lane] = p / z;
    }
}

// Warp per token with the token's logits in registers (topk_token).
template <int EPL>
__global__ void __launch_bounds__(128) router_topk_reg_kernel(const float* __restrict__ logits, int n, int E, int k,
                                                              int32_t* __restrict__ idx, float* __restrict__ w)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= n) return;
    topk_token<EPL>(logits + (size_t)t * E, E, k, lane, idx + (size_t)t * k, w + (size_t)t * k);
}

template <bool XF32>
int launch_logits(const void* x, const uint16_t* wg, const float* bias, int n, int H, int E,
                  float* logits, cudaStream_t st)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256, wpb = threads / 32;
    if (n >= 64) {
        dim3 grid((n + RT_TOK - 1) / RT_TOK, (E + RT_EXP - 1) / RT_EXP);
        if constexpr (XF32)
            router_logits_tiled_kernel<XF32><<<grid, 256, 0, st>>>(x, wg, bias, n, H, E, logits);
        else
            router_logits_pipe_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), wg, bias, n, H, E,
                                                             logits);
    } else {
        // from 8 tokens a warp takes 2 tokens x 2 experts: each gate-row load
        // serves two tokens and each activation load two experts (measured 2.6 us
        // faster per 16-token call; 2.4 us slower at 1-4 tokens, which keep a warp
        // per pair).  The per-lane order, and so every logit, is the same.
        auto grid_for = [&](int TB, int EB) {
            const long units = (long)((E + EB - 1) / EB) * ((n + TB - 1) / TB);
            const int g = (int)((units + wpb - 1) / wpb);
            return g > sms * 8 ? sms * 8 : g;
        };
        if (n >= 8)
            router_logits_kernel<XF32, 2, 2, 4><<<grid_for(2, 2), threads, 0, st>>>(x, wg, bias, n, H, E, logits);
        else
            router_logits_kernel<XF32, 1, 1, 8><<<grid_for(1, 1), threads, 0, st>>>(x, wg, bias, n, H, E, logits);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace

// The logits kernel alone (the decode front kernel takes the top-k).
int launch_router_logits(const void* x, int x_dtype, const uint16_t* wg, const float* bias, int n, int H, int E,
                         float* logits, cudaStream_t st)
{
    if (n == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_ROUTER, st);
    prof_count(MOE_PROF_ROUTER, 1);
    return (x_dtype == MOE_DT_F32) ? launch_logits<true>(x, wg, bias, n, H, E, logits, st)
                                   : launch_logits<false>(x, wg, bias, n, H, E, logits, st);
}

int launch_router(const void* x, int x_dtype, const uint16_t* wg, const float* bias, int n, int H,
                  int E, int k, float* logits, int32_t* idx, float* w, cudaStream_t st)
{
    if (n == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_ROUTER, st);
    prof_count(MOE_PROF_ROUTER, 2);
    int rc = (x_dtype == MOE_DT_F32) ? launch_logits<true>(x, wg, bias, n, H, E, logits, st)
                                     : launch_logits<false>(x, wg, bias, n, H, E, logits, st);
    if (rc) return rc;
    const int wpb = 4;
    const int blocks = (n + wpb - 1) / wpb;
    if (E <= 256)
        router_topk_reg_kernel<8><<<blocks, wpb * 32, 0, st>>>(logits, n, E, k, idx, w);
    else if (E <= 1024)
        router_topk_reg_kernel<32><<<blocks, wpb * 32, 0, st>>>(logits, n, E, k, idx, w);
    else
        router_topk_kernel<<<blocks, wpb * 32, (size_t)wpb * E, st>>>(logits, n, E, k, idx, w);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

extern "C" int moe_router_topk(const void* d_x, int32_t x_dtype, const uint16_t* d_wg,
                               const float* d_bias, int32_t n, int32_t hidden, int32_t experts,
                               int32_t k, float* d_logits, int32_t* d_topk_idx, float* d_topk_w,
                               void* stream)
{
    if (n < 0 || hidden <= 0 || hidden % 8 || experts <= 0 || experts > moe::kMaxExperts || k <= 0 ||
        k > experts || k > moe::kMaxTopK)
        return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_x || !d_wg || !d_logits || !d_topk_idx || !d_topk_w)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_x | (uintptr_t)d_wg) & 15) return MOE_ERR_INVALID_ARG;
    return moe::launch_router(d_x, x_dtype, d_wg, d_bias, n, hidden, experts, k, d_logits,
                              d_topk_idx, d_topk_w, moe::as_stream(stream));
}
