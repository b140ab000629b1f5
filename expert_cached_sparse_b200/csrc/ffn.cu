// Grouped SwiGLU expert FFN over permuted rows, weights streamed from the
// expert slots.  "A cache hit runs on the GPU" ("FreeToken quantization",
// section "Como se desplazan los pesos MoE cuantizados por la memoria").
//
// Weight-streaming design (decode is bound by HBM: each touched expert's
// weights are read once per pass):
//  - the unit of work is one warp x one 16-row tile of W13 (or W2) x up to
//    32 rows (tokens) of one expert; units run in a persistent grid;
//  - A (weights) is the mma.sync m16n8k16 row operand, fed straight from
//    registers: each lane's 16-byte load of a packed tile holds exactly its
//    fragment elements (rows g and g+8, 16 consecutive k); E2M1 codes become
//    f16 with cvt.rn.f16x2.e2m1x2, are re-biased into bf16 (x 2^-112, exact)
//    and multiplied by (block scale x 2^112) in bf16, which is exact because
//    e2m1 x scale has at most 6 significant bits;
//  - B (tokens) is bf16 from x_perm (phase 1) or h (phase 2); the k order
//    inside each 64-column tile is permuted identically for A and B, so a
//    lane's B data is 16 consecutive elements (two 16-byte loads);
//  - phase 1 tiles pair 8 gate rows with the 8 matching up rows, so the
//    SwiGLU epilogue is lane-local: h = silu(gate) * up, rounded to bf16;
//  - phase 2 writes y rows in bf16; the NVFP4 tensor scales multiply the
//    fp32 accumulators.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kFfnThreads = 128;
constexpr int kRowsPerUnit = 32;   // 4 n-tiles of 8 tokens

struct FfnArgs {
    const char* pool;
    size_t slot_bytes;
    size_t w_off;      // tile base of the matrix inside the blob
    size_t s_off;      // scale-tile base
    size_t ts_off;     // NVFP4 tensor scales
    int R, K;          // matrix rows / columns (2F x H for phase 1, H x F for phase 2)
    int E;
    const int32_t* slot_of;
    const int32_t* offsets;
    int pool_slots;    // slots >= pool_slots (or < 0) are skipped
    int rows;          // rows of in/out; row ranges are clipped to it
    const uint16_t* in;    // [rows][K] bf16
    uint16_t* out;         // [rows][R/2] (phase 1, h) or [rows][R] (phase 2, y)
};

__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& f0, uint32_t& f1, uint32_t& f2,
                                                uint32_t& f3)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(f0), "=r"(f1), "=r"(f2), "=r"(f3)
        : "r"(w));
}

// f16x2 holding E2M1 values -> bf16x2 of (value * 2^-112), exact, then
// times the bf16x2 multiplier m2 = (scale * 2^112, scale * 2^112).
__device__ __forceinline__ uint32_t f16x2_e2m1_to_bf16x2(uint32_t f, uint32_t m2)
{
    uint32_t b = ((f & 0x7FFF7FFFu) >> 3) | (f & 0x80008000u);
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(b), "r"(m2));
    return r;
}

__device__ __forceinline__ void mma_bf16(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 bits of value(code) * 2^112 for the block-scale codes of the format.
__device__ uint16_t scale_mult_bits(int wfmt, int c)
{
    if (wfmt == MOE_W_MXFP4) {
        int e = c + 112;             // 2^(c-127) * 2^112 = 2^(c-15); codes outside [2,142] rejected at pack
        if (e < 1) e = 1;
        if (e > 254) e = 254;
        return (uint16_t)(e << 7);
    }
    // E4M3: sign, 4-bit exponent (bias 7), 3-bit mantissa; subnormals m*2^-9
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    float v = (e == 0) ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    v = ldexpf(v, 112);
    if (s) v = -v;
    return f32_to_bf16_bits(v);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

template <int WFMT, int PHASE>
__global__ void __launch_bounds__(kFfnThreads) ffn_kernel(FfnArgs a)
{
    extern __shared__ int s_prefix[];          // [E+1] unit prefix per expert
    __shared__ uint16_t s_mult[256];
    __shared__ int s_warp[kFfnThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int RT = a.R / 16, KT = a.K / 64;
    const int E = a.E;

    if (WFMT != MOE_W_BF16)
        for (int c = tid; c < 256; c += kFfnThreads) s_mult[c] = scale_mult_bits(WFMT, c);
    // per-expert unit counts -> exclusive prefix (contiguous experts per thread)
    const int EPT = (E + kFfnThreads - 1) / kFfnThreads;
    int loc = 0;
    for (int e = tid * EPT; e < tid * EPT + EPT && e < E; e++) {
        int cnt = a.offsets[e + 1] - a.offsets[e];
        int sl = a.slot_of[e];
        int u = (cnt > 0 && sl >= 0 && sl < a.pool_slots) ? ((cnt + kRowsPerUnit - 1) / kRowsPerUnit) * RT : 0;
        s_prefix[e] = u;
        loc += u;
    }
    {
        int inc = loc;
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) s_warp[tid >> 5] = inc;
        __syncthreads();
        int wbase = 0;
        for (int w = 0; w < (tid >> 5); w++) wbase += s_warp[w];
        int run = wbase + inc - loc;
        for (int e = tid * EPT; e < tid * EPT + EPT && e < E; e++) {
            int u = s_prefix[e];
            s_prefix[e] = run;
            run += u;
        }
        if (tid == kFfnThreads - 1) s_prefix[E] = run;
    }
    __syncthreads();
    const int total = s_prefix[E];
    const int warps_total = gridDim.x * (kFfnThreads / 32);

    for (int u = blockIdx.x * (kFfnThreads / 32) + (tid >> 5); u < total; u += warps_total) {
        // expert of unit u: largest e with s_prefix[e] <= u
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const int local = u - s_prefix[e];
        const int tg = local / RT, rt = local % RT;
        const int row0 = a.offsets[e] + tg * kRowsPerUnit;
        const int row_end = min(min(a.offsets[e + 1], row0 + kRowsPerUnit), a.rows);
        if (row0 < 0 || row0 >= row_end) continue;
        const int nq = (row_end - row0 + 7) >> 3;
        const char* blob = a.pool + (size_t)a.slot_of[e] * a.slot_bytes;
        float tsc = 1.0f;
        if (WFMT == MOE_W_NVFP4) tsc = reinterpret_cast<const float*>(blob + a.ts_off)[PHASE - 1];

        float acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; q++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[q][i] = 0.0f;

        constexpr int PF = (WFMT == MOE_W_BF16) ? 2 : 8;      // tiles in flight
        constexpr int TILE = (WFMT == MOE_W_BF16) ? 2048 : 512;
        constexpr int STILE = (WFMT == MOE_W_MXFP4) ? 32 : 64;
        constexpr int NV = (WFMT == MOE_W_BF16) ? 4 : 1;     // uint4 per lane per tile
        const char* wt = blob + a.w_off + (size_t)rt * KT * TILE;
        const char* st = blob + a.s_off + (size_t)rt * KT * STILE;

        uint4 abuf[PF][NV];
        uint2 sbuf[PF];
#pragma unroll
        for (int i = 0; i < PF; i++) {
            if (i < KT) {
#pragma unroll
                for (int v = 0; v < NV; v++)
                    abuf[i][v] = __ldg(reinterpret_cast<const uint4*>(wt + (size_t)i * TILE + v * 512 + 16 * lane));
                if (WFMT == MOE_W_MXFP4)
                    sbuf[i].x = __ldg(reinterpret_cast<const uint32_t*>(st + (size_t)i * STILE + 4 * g));
                if (WFMT == MOE_W_NVFP4)
                    sbuf[i] = __ldg(reinterpret_cast<const uint2*>(st + (size_t)i * STILE + 8 * g));
            }
        }
        for (int kt0 = 0; kt0 < KT; kt0 += PF) {
#pragma unroll
            for (int i = 0; i < PF; i++) {
                const int kt = kt0 + i;
                if (kt >= KT) break;
                uint4 cur[NV];
#pragma unroll
                for (int v = 0; v < NV; v++) cur[v] = abuf[i][v];
                uint2 cs = sbuf[i];
                if (kt + PF < KT) {
#pragma unroll
                    for (int v = 0; v < NV; v++)
                        abuf[i][v] = __ldg(reinterpret_cast<const uint4*>(wt + (size_t)(kt + PF) * TILE + v * 512 +
                                                                          16 * lane));
                    if (WFMT == MOE_W_MXFP4)
                        sbuf[i].x = __ldg(reinterpret_cast<const uint32_t*>(st + (size_t)(kt + PF) * STILE + 4 * g));
                    if (WFMT == MOE_W_NVFP4)
                        sbuf[i] = __ldg(reinterpret_cast<const uint2*>(st + (size_t)(kt + PF) * STILE + 8 * g));
                }
                // A fragments for the 4 k16 steps of this tile: A[j][0..3] = a0,a1,a2,a3
                uint32_t A[4][4];
                if (WFMT == MOE_W_BF16) {
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        A[j][0] = cur[j].x;  // row g   k 16t+4j, +1
                        A[j][2] = cur[j].y;  // row g   k 16t+4j+2, +3
                        A[j][1] = cur[j].z;  // row g+8
                        A[j][3] = cur[j].w;
                    }
                } else {
                    uint32_t sg, sg8;
                    if (WFMT == MOE_W_MXFP4) {
                        sg = (cs.x >> (8 * (t >> 1))) & 0xFF;
                        sg8 = (cs.x >> (8 * (2 + (t >> 1)))) & 0xFF;
                    } else {
                        sg = (cs.x >> (8 * t)) & 0xFF;
                        sg8 = (cs.y >> (8 * t)) & 0xFF;
                    }
                    uint32_t mg = s_mult[sg], mg8 = s_mult[sg8];
                    mg |= mg << 16;
                    mg8 |= mg8 << 16;
                    uint32_t f[4];
                    // row g: bytes 0..7 -> steps (byte 2j -> a0, byte 2j+1 -> a2)
                    e2m1x8_to_f16x2(cur[0].x, f[0], f[1], f[2], f[3]);
                    A[0][0] = f16x2_e2m1_to_bf16x2(f[0], mg);
                    A[0][2] = f16x2_e2m1_to_bf16x2(f[1], mg);
                    A[1][0] = f16x2_e2m1_to_bf16x2(f[2], mg);
                    A[1][2] = f16x2_e2m1_to_bf16x2(f[3], mg);
                    e2m1x8_to_f16x2(cur[0].y, f[0], f[1], f[2], f[3]);
                    A[2][0] = f16x2_e2m1_to_bf16x2(f[0], mg);
                    A[2][2] = f16x2_e2m1_to_bf16x2(f[1], mg);
                    A[3][0] = f16x2_e2m1_to_bf16x2(f[2], mg);
                    A[3][2] = f16x2_e2m1_to_bf16x2(f[3], mg);
                    e2m1x8_to_f16x2(cur[0].z, f[0], f[1], f[2], f[3]);
                    A[0][1] = f16x2_e2m1_to_bf16x2(f[0], mg8);
                    A[0][3] = f16x2_e2m1_to_bf16x2(f[1], mg8);
                    A[1][1] = f16x2_e2m1_to_bf16x2(f[2], mg8);
                    A[1][3] = f16x2_e2m1_to_bf16x2(f[3], mg8);
                    e2m1x8_to_f16x2(cur[0].w, f[0], f[1], f[2], f[3]);
                    A[2][1] = f16x2_e2m1_to_bf16x2(f[0], mg8);
                    A[2][3] = f16x2_e2m1_to_bf16x2(f[1], mg8);
                    A[3][1] = f16x2_e2m1_to_bf16x2(f[2], mg8);
                    A[3][3] = f16x2_e2m1_to_bf16x2(f[3], mg8);
                }
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    if (q >= nq) break;
                    const int r = row0 + q * 8 + g;
                    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                    if (r < row_end) {
                        const uint4* xp = reinterpret_cast<const uint4*>(a.in + (size_t)r * a.K + kt * 64 + 16 * t);
                        x0 = __ldg(xp);
                        x1 = __ldg(xp + 1);
                    }
                    mma_bf16(acc[q], A[0][0], A[0][1], A[0][2], A[0][3], x0.x, x0.y);
                    mma_bf16(acc[q], A[1][0], A[1][1], A[1][2], A[1][3], x0.z, x0.w);
                    mma_bf16(acc[q], A[2][0], A[2][1], A[2][2], A[2][3], x1.x, x1.y);
                    mma_bf16(acc[q], A[3][0], A[3][1], A[3][2], A[3][3], x1.z, x1.w);
                }
            }
        }
        // epilogue
#pragma unroll
        for (int q = 0; q < 4; q++) {
            if (q >= nq) break;
            const int r0 = row0 + q * 8 + 2 * t, r1 = r0 + 1;
            if (PHASE == 1) {
                const int F = a.R / 2;
                const int f = 8 * rt + g;
                float g0 = acc[q][0] * tsc, g1 = acc[q][1] * tsc, u0 = acc[q][2] * tsc, u1 = acc[q][3] * tsc;
                if (r0 < row_end) a.out[(size_t)r0 * F + f] = f32_to_bf16_bits(silu(g0) * u0);
                if (r1 < row_end) a.out[(size_t)r1 * F + f] = f32_to_bf16_bits(silu(g1) * u1);
            } else {
                const int Ho = a.R;
                const int o = 16 * rt + g;
                if (r0 < row_end) {
                    a.out[(size_t)r0 * Ho + o] = f32_to_bf16_bits(acc[q][0] * tsc);
                    a.out[(size_t)r0 * Ho + o + 8] = f32_to_bf16_bits(acc[q][2] * tsc);
                }
                if (r1 < row_end) {
                    a.out[(size_t)r1 * Ho + o] = f32_to_bf16_bits(acc[q][1] * tsc);
                    a.out[(size_t)r1 * Ho + o + 8] = f32_to_bf16_bits(acc[q][3] * tsc);
                }
            }
        }
    }
}

template <int WFMT>
int launch_ffn_fmt(const moe_shape* s, const BlobLayout& bl, FfnArgs a1, FfnArgs a2, int rows, int sms,
                   cudaStream_t st)
{
    const int E = s->experts;
    size_t smem = sizeof(int) * (E + 1);
    auto grid_for = [&](int R) {
        long max_units = (long)((rows + kRowsPerUnit - 1) / kRowsPerUnit + (rows < E ? rows : E)) * (R / 16);
        long g = (max_units + 3) / 4;
        long cap = (long)sms * 8;
        return (int)(g < 1 ? 1 : (g > cap ? cap : g));
    };
    ffn_kernel<WFMT, 1><<<grid_for(a1.R), kFfnThreads, smem, st>>>(a1);
    MOE_LAUNCH_CHECK();
    ffn_kernel<WFMT, 2><<<grid_for(a2.R), kFfnThreads, smem, st>>>(a2);
    MOE_LAUNCH_CHECK();
    (void)bl;
    return MOE_OK;
}

}  // namespace

// Grouped GEMM on tcgen05 when groups are large (prefill: rows >= 4 per
// expert on average) and the weights are FP4; the weight-streaming mma.sync
// kernel otherwise.  MOE_FFN_PATH=mma|tc overrides the choice.
static bool use_tc_path(const moe_shape* s, int rows)
{
    if (!ffn_tc_supported(s)) return false;
    const char* force = getenv("MOE_FFN_PATH");
    if (force && !strcmp(force, "mma")) return false;
    if (force && !strcmp(force, "tc")) return true;
    return rows >= 4 * s->experts;
}

size_t ffn_ws_bytes(const moe_shape* s, int rows) { return align_up((size_t)rows * s->ffn * 2, 256) + 256; }

int launch_ffn(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
               const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm, void* ws,
               cudaStream_t st)
{
    if (rows == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_FFN, st);
    prof_count(MOE_PROF_FFN, 2);
    BlobLayout bl = blob_layout(s);
    uint16_t* h = static_cast<uint16_t*>(ws);
    FfnArgs a1{};
    a1.pool = static_cast<const char*>(pool);
    a1.slot_bytes = slot_bytes;
    a1.w_off = bl.w13;
    a1.s_off = bl.s13;
    a1.ts_off = bl.ts;
    a1.R = 2 * s->ffn;
    a1.K = s->hidden;
    a1.E = s->experts;
    a1.slot_of = slot_of;
    a1.offsets = offsets;
    a1.pool_slots = pool_slots;
    a1.rows = rows;
    a1.in = x_perm;
    a1.out = h;
    FfnArgs a2 = a1;
    a2.w_off = bl.w2;
    a2.s_off = bl.s2;
    a2.R = s->hidden;
    a2.K = s->ffn;
    a2.in = h;
    a2.out = y_perm;
    if (use_tc_path(s, rows))
        return launch_ffn_tc(s, pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows, y_perm, h, st);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    switch (s->wfmt) {
    case MOE_W_BF16: return launch_ffn_fmt<MOE_W_BF16>(s, bl, a1, a2, rows, sms, st);
    case MOE_W_MXFP4: return launch_ffn_fmt<MOE_W_MXFP4>(s, bl, a1, a2, rows, sms, st);
    case MOE_W_NVFP4: return launch_ffn_fmt<MOE_W_NVFP4>(s, bl, a1, a2, rows, sms, st);
    }
    return MOE_ERR_INVALID_ARG;
}

}  // namespace moe

extern "C" size_t moe_ffn_workspace_bytes(const moe_shape* shape, int32_t rows)
{
    if (!moe::shape_ok(shape) || rows < 0) return 0;
    return moe::ffn_ws_bytes(shape, rows);
}

extern "C" int moe_grouped_ffn(const moe_shape* shape, const void* d_slot_pool, int32_t pool_slots,
                               const int32_t* d_slot_of_expert, const int32_t* d_expert_offsets,
                               const uint16_t* d_x_perm, int32_t rows, uint16_t* d_y_perm, void* d_ws,
                               size_t ws_bytes, void* stream)
{
    if (!moe::shape_ok(shape) || rows < 0 || pool_slots < 0) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!d_slot_pool || !d_slot_of_expert || !d_expert_offsets || !d_x_perm || !d_y_perm || !d_ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe::ffn_ws_bytes(shape, rows)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_slot_pool | (uintptr_t)d_x_perm | (uintptr_t)d_ws) & 15) return MOE_ERR_INVALID_ARG;
    size_t sb = moe::blob_layout(shape).bytes;
    return moe::launch_ffn(shape, d_slot_pool, sb, pool_slots, d_slot_of_expert, d_expert_offsets, d_x_perm, rows,
                           d_y_perm, d_ws, moe::as_stream(stream));
}
