// Token -> expert permutation: per-expert counts, exclusive offsets, a stable
// scatter of the assignments and the gather of activation rows, so that each
// expert's rows are contiguous for the grouped FFN.  Stable means row order
// inside an expert follows the assignment index a = t*k + j.
//
// Atomic-free and deterministic.  Chunks of 32*W assignments (W warps of a
// CTA); inside a warp __match_any_sync gives each assignment its rank among
// equal experts; warp counts are combined per expert in shared memory; chunk
// counts are scanned per expert across chunks; offsets come from a block
// scan of the totals.
#include "common.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

constexpr int kPermThreads = 1024;

static int warps_per_chunk(int E)
{
    int w = 8192 / E;               // warp histograms of E ints within 32 KB
    if (w > 32) w = 32;
    if (w < 1) w = 1;
    return w;
}

struct PermWs {
    int32_t* chunk_hist;   // [chunks][E]: counts, then exclusive base per chunk
    int32_t* rank;         // [A] rank of the assignment among its expert inside its chunk
};

static size_t ws_layout(int A, int E, PermWs* p, void* base)
{
    int W = warps_per_chunk(E);
    int chunk = 32 * W;
    size_t chunks = (A + chunk - 1) / chunk;
    size_t off_hist = 0;
    size_t off_rank = align_up(sizeof(int32_t) * chunks * E, 256);
    size_t total = off_rank + align_up(sizeof(int32_t) * (size_t)A, 256);
    if (p) {
        char* b = static_cast<char*>(base);
        p->chunk_hist = reinterpret_cast<int32_t*>(b + off_hist);
        p->rank = reinterpret_cast<int32_t*>(b + off_rank);
    }
    return total < 256 ? 256 : total;
}

// One CTA of W warps per chunk.  Writes chunk_hist[chunk][e] (counts) and
// rank[a] (rank inside the chunk among assignments of the same expert).
__global__ void perm_hist_kernel(const int32_t* __restrict__ idx, int A, int E, int W,
                                 int32_t* __restrict__ chunk_hist, int32_t* __restrict__ rank)
{
    extern __shared__ int wh[];       // [W][E]
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int a = (blockIdx.x * W + w) * 32 + lane;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) wh[i] = 0;
    __syncthreads();
    int e = (a < A) ? idx[a] : -1;
    if (e >= E) e = -1;                 // out-of-range experts get no row
    unsigned peers = __match_any_sync(0xffffffffu, e);
    int r_in_warp = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && r_in_warp == 0) wh[w * E + e] = __popc(peers);
    __syncthreads();
    // exclusive scan over warps, per expert
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
        int run = 0;
        for (int ww = 0; ww < W; ww++) {
            int v = wh[ww * E + x];
            wh[ww * E + x] = run;
            run += v;
        }
        chunk_hist[(size_t)blockIdx.x * E + x] = run;
    }
    __syncthreads();
    if (e >= 0) rank[a] = wh[w * E + e] + r_in_warp;
}

// Single CTA: per expert, exclusive scan of the chunk counts (in place), then
// offsets = exclusive scan of the totals.
__global__ void __launch_bounds__(kPermThreads) perm_scan_kernel(int32_t* __restrict__ chunk_hist,
                                                                 int chunks, int E,
                                                                 int32_t* __restrict__ offsets)
{
    __shared__ int s_warp[32];
    __shared__ int s_tot;
    __shared__ int s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        int e = e0 + threadIdx.x;
        int run = 0;
        if (e < E) {
            for (int c = 0; c < chunks; c++) {
                int v = chunk_hist[(size_t)c * E + e];
                chunk_hist[(size_t)c * E + e] = run;
                run += v;
            }
        }
        // block exclusive scan of `run`
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        int inc = run;
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) s_warp[w] = inc;
        __syncthreads();
        if (w == 0) {
            int x = (lane < (blockDim.x >> 5)) ? s_warp[lane] : 0;
            int xi = x;
            for (int off = 1; off < 32; off <<= 1) {
                int o = __shfl_up_sync(0xffffffffu, xi, off);
                if (lane >= off) xi += o;
            }
            s_warp[lane] = xi - x;
            if (lane == 31) s_tot = xi;
        }
        __syncthreads();
        if (e < E) offsets[e] = s_carry + s_warp[w] + inc - run;
        __syncthreads();
        if (threadIdx.x == 0) s_carry += s_tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[E] = s_carry;
}

// row_of / assign_of, then one warp per assignment copies its token's row.
template <bool XF32>
__global__ void perm_scatter_gather_kernel(const int32_t* __restrict__ idx, int A, int E, int k, int W,
                                           const int32_t* __restrict__ offsets,
                                           const int32_t* __restrict__ chunk_base,
                                           const int32_t* __restrict__ rank, const void* __restrict__ x,
                                           int H, int32_t* __restrict__ row_of,
                                           int32_t* __restrict__ assign_of, uint16_t* __restrict__ x_perm)
{
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int chunk = 32 * W;
    for (int a = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); a < A; a += warps_total) {
        int e = idx[a];
        if (e < 0 || e >= E) {
            if (lane == 0) row_of[a] = -1;
            continue;
        }
        int row = offsets[e] + chunk_base[(size_t)(a / chunk) * E + e] + rank[a];
        if (lane == 0) {
            row_of[a] = row;
            assign_of[row] = a;
        }
        if (!x_perm) continue;
        const int t = a / k;
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * H);
        if (XF32) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * H);
            for (int c = lane; c < H / 8; c += 32) {
                float4 p = __ldg(src + 2 * c), q = __ldg(src + 2 * c + 1);
                uint4 o;
                o.x = (uint32_t)f32_to_bf16_bits(p.x) | ((uint32_t)f32_to_bf16_bits(p.y) << 16);
                o.y = (uint32_t)f32_to_bf16_bits(p.z) | ((uint32_t)f32_to_bf16_bits(p.w) << 16);
                o.z = (uint32_t)f32_to_bf16_bits(q.x) | ((uint32_t)f32_to_bf16_bits(q.y) << 16);
                o.w = (uint32_t)f32_to_bf16_bits(q.z) | ((uint32_t)f32_to_bf16_bits(q.w) << 16);
                dst[c] = o;
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)t * H);
            for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
        }
    }
}

// Small calls (decode): one CTA does the whole index work.  Per-expert
// counts, an exclusive block scan for the offsets, and for every assignment
// its rank among earlier assignments to the same expert (a scan over the
// call's indices held in shared memory).
__global__ void __launch_bounds__(1024) perm_small_kernel(const int32_t* __restrict__ idx, int A, int E,
                                                          int32_t* __restrict__ offsets, int32_t* __restrict__ row_of,
                                                          int32_t* __restrict__ assign_of)
{
    __shared__ PermSmem S;
    perm_small_body(idx, A, E, offsets, row_of, assign_of, S);
}

// x_perm[row] = bf16(x[assign_of[row] / k]): one warp per row.
template <bool XF32>
__global__ void perm_gather_kernel(const int32_t* __restrict__ assign_of, const int32_t* __restrict__ offsets, int E,
                                   int k, const void* __restrict__ x, int H, uint16_t* __restrict__ x_perm)
{
    const int lane = threadIdx.x & 31;
    const int rows = offsets[E];
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps_total) {
        const int t = assign_of[r] / k;
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * H);
        if (XF32) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * H);
            for (int c = lane; c < H / 8; c += 32) {
                float4 p = __ldg(src + 2 * c), q = __ldg(src + 2 * c + 1);
                uint4 o;
                o.x = (uint32_t)f32_to_bf16_bits(p.x) | ((uint32_t)f32_to_bf16_bits(p.y) << 16);
                o.y = (uint32_t)f32_to_bf16_bits(p.z) | ((uint32_t)f32_to_bf16_bits(p.w) << 16);
                o.z = (uint32_t)f32_to_bf16_bits(q.x) | ((uint32_t)f32_to_bf16_bits(q.y) << 16);
                o.w = (uint32_t)f32_to_bf16_bits(q.z) | ((uint32_t)f32_to_bf16_bits(q.w) << 16);
                dst[c] = o;
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)t * H);
            for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
        }
    }
}

}  // namespace

size_t permute_ws_bytes(int n, int E, int k) { return ws_layout(n * k, E, nullptr, nullptr); }

int launch_permute(const int32_t* idx, int n, int E, int k, const void* x, int x_dtype, int H,
                   int32_t* offsets, int32_t* row_of, int32_t* assign_of, uint16_t* x_perm, void* ws,
                   cudaStream_t st)
{
    const int A = n * k;
    if (A == 0) {
        MOE_CUDA_TRY(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st));
        return MOE_OK;
    }
    ProfScope ps(MOE_PROF_PERMUTE, st);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (A <= kSmallA && E <= kSmallE) {
        perm_small_kernel<<<1, 1024, 0, st>>>(idx, A, E, offsets, row_of, assign_of);
        MOE_LAUNCH_CHECK();
        prof_count(MOE_PROF_PERMUTE, x_perm ? 2 : 1);
        if (!x_perm) return MOE_OK;
        int grid = (A + 7) / 8;
        if (grid > sms * 8) grid = sms * 8;
        if (x_dtype == MOE_DT_F32)
            perm_gather_kernel<true><<<grid, 256, 0, st>>>(assign_of, offsets, E, k, x, H, x_perm);
        else
            perm_gather_kernel<false><<<grid, 256, 0, st>>>(assign_of, offsets, E, k, x, H, x_perm);
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
    prof_count(MOE_PROF_PERMUTE, 3);
    PermWs p;
    ws_layout(A, E, &p, ws);
    const int W = warps_per_chunk(E);
    const int chunks = (A + 32 * W - 1) / (32 * W);
    perm_hist_kernel<<<chunks, 32 * W, sizeof(int) * W * E, st>>>(idx, A, E, W, p.chunk_hist, p.rank);
    MOE_LAUNCH_CHECK();
    perm_scan_kernel<<<1, kPermThreads, 0, st>>>(p.chunk_hist, chunks, E, offsets);
    MOE_LAUNCH_CHECK();
    int grid = (A + 7) / 8;
    if (grid > sms * 8) grid = sms * 8;
    if (x_dtype == MOE_DT_F32)
        perm_scatter_gather_kernel<true><<<grid, 256, 0, st>>>(idx, A, E, k, W, offsets, p.chunk_hist,
                                                               p.rank, x, H, row_of, assign_of, x_perm);
    else
        perm_scatter_gather_kernel<false><<<grid, 256, 0, st>>>(idx, A, E, k, W, offsets, p.chunk_hist,
                                                                p.rank, x, H, row_of, assign_of, x_perm);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

extern "C" size_t moe_permute_workspace_bytes(int32_t n, int32_t experts, int32_t top_k)
{
    if (n < 0 || experts <= 0 || experts > moe::kMaxExperts || top_k <= 0) return 0;
    return moe::permute_ws_bytes(n, experts, top_k);
}

extern "C" int moe_permute(const int32_t* d_topk_idx, int32_t n, int32_t experts, int32_t k, const void* d_x,
                           int32_t x_dtype, int32_t hidden, int32_t* d_expert_offsets, int32_t* d_row_of,
                           int32_t* d_assign_of, uint16_t* d_x_perm, void* d_ws, size_t ws_bytes,
                           void* stream)
{
    if (n < 0 || experts <= 0 || experts > moe::kMaxExperts || k <= 0 || hidden <= 0 || hidden % 8)
        return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (!d_expert_offsets) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_topk_idx || !d_x || !d_row_of || !d_assign_of || !d_x_perm || !d_ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe::permute_ws_bytes(n, experts, k)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_x | (uintptr_t)d_x_perm) & 15) return MOE_ERR_INVALID_ARG;
    return moe::launch_permute(d_topk_idx, n, experts, k, d_x, x_dtype, hidden, d_expert_offsets, d_row_of,
                               d_assign_of, d_x_perm, d_ws, moe::as_stream(stream));
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the same permutation for callers that must not
// allocate device memory themselves (see include/moe.h).  Its scratch lives
// in one file-scope device array that every GPU loading this library holds
// until the process exits.  Host code cannot pass the array's name to a
// kernel (on the host it is only a stand-in symbol), so the device address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on it.
#include <mutex>

namespace {

constexpr size_t kPermuteStaticScratch = MOE_PERMUTE_NOALLOC_MAX_SCRATCH;
static __device__ __align__(256) unsigned char g_permute_scratch[kPermuteStaticScratch];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];   // device address of g_permute_scratch per device

// Device address of the static scratch on the current device (nullptr on failure).
void* permute_static_scratch()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int moe_permute_noalloc(const int32_t* d_topk_idx, int32_t n, int32_t experts, int32_t k,
                                   const void* d_x, int32_t x_dtype, int32_t hidden, int32_t* d_expert_offsets,
                                   int32_t* d_row_of, int32_t* d_assign_of, uint16_t* d_x_perm, void* stream)
{
    if (n < 0 || experts <= 0 || experts > moe::kMaxExperts || k <= 0 || hidden <= 0 || hidden % 8)
        return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (!d_expert_offsets) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_topk_idx || !d_x || !d_row_of || !d_assign_of || !d_x_perm)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_x | (uintptr_t)d_x_perm) & 15) return MOE_ERR_INVALID_ARG;
    if ((long long)n * k > (1ll << 30)) return MOE_ERR_UNSUPPORTED;
    if (moe::permute_ws_bytes(n, experts, k) > kPermuteStaticScratch) return MOE_ERR_UNSUPPORTED;
    void* scratch = permute_static_scratch();
    if (!scratch) return MOE_ERR_CUDA;
    // Every scratch entry the kernels read is written earlier in the same call,
    // so the previous call's contents need no clearing.
    return moe::launch_permute(d_topk_idx, n, experts, k, d_x, x_dtype, hidden, d_expert_offsets, d_row_of,
                               d_assign_of, d_x_perm, scratch, moe::as_stream(stream));
}
