// Gate-weighted combine: out[t] = sum_j w[t][j] * y_perm[row_of[t*k+j]],
// j ascending, fp32 accumulation, no atomics (bitwise reproducible).
#include "common.cuh"

namespace moe {
namespace {

template <bool OUTF32>
__global__ void combine_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ row_of,
                               const float* __restrict__ w, int n, int k, int H, void* __restrict__ out)
{
    const int chunks = H / 8;
    const long total = (long)n * chunks;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const int t = (int)(i / chunks), c = (int)(i % chunks);
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; q++) acc[q] = 0.0f;
        for (int j = 0; j < k; j++) {
            const float wj = __ldg(w + (size_t)t * k + j);
            const int r = __ldg(row_of + (size_t)t * k + j);
            if (r < 0 || r >= n * k) continue;      // not a row of this call
            uint4 v = __ldg(reinterpret_cast<const uint4*>(y + (size_t)r * H) + c);
            uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
                acc[2 * q] = __fmaf_rn(wj, bf16_bits_to_f32(u[q] & 0xFFFFu), acc[2 * q]);
                acc[2 * q + 1] = __fmaf_rn(wj, bf16_bits_to_f32(u[q] >> 16), acc[2 * q + 1]);
            }
        }
        if (OUTF32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)t * H) + 2 * c;
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
            uint4 o;
            o.x = f32_to_bf16_bits(acc[0]) | ((uint32_t)f32_to_bf16_bits(acc[1]) << 16);
            o.y = f32_to_bf16_bits(acc[2]) | ((uint32_t)f32_to_bf16_bits(acc[3]) << 16);
            o.z = f32_to_bf16_bits(acc[4]) | ((uint32_t)f32_to_bf16_bits(acc[5]) << 16);
            o.w = f32_to_bf16_bits(acc[6]) | ((uint32_t)f32_to_bf16_bits(acc[7]) << 16);
            reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + (size_t)t * H)[c] = o;
        }
    }
}

}  // namespace

int launch_combine(const uint16_t* y_perm, const int32_t* row_of, const float* w, int n, int k, int H, void* out,
                   int out_dtype, cudaStream_t st)
{
    if (n == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_COMBINE, st);
    prof_count(MOE_PROF_COMBINE, 1);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long total = (long)n * (H / 8);
    int grid = (int)((total + 255) / 256);
    if (grid > sms * 8) grid = sms * 8;
    if (out_dtype == MOE_DT_F32)
        combine_kernel<true><<<grid, 256, 0, st>>>(y_perm, row_of, w, n, k, H, out);
    else
        combine_kernel<false><<<grid, 256, 0, st>>>(y_perm, row_of, w, n, k, H, out);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

extern "C" int moe_combine(const uint16_t* d_y_perm, const int32_t* d_row_of, const float* d_topk_w, int32_t n,
                           int32_t k, int32_t hidden, void* d_out, int32_t out_dtype, void* stream)
{
    if (n < 0 || k <= 0 || hidden <= 0 || hidden % 8) return MOE_ERR_INVALID_ARG;
    if (out_dtype != MOE_DT_F32 && out_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_y_perm || !d_row_of || !d_topk_w || !d_out)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_y_perm | (uintptr_t)d_out) & 15) return MOE_ERR_INVALID_ARG;
    return moe::launch_combine(d_y_perm, d_row_of, d_topk_w, n, k, hidden, d_out, out_dtype, moe::as_stream(stream));
}
