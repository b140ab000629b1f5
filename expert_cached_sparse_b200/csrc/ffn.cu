// Grouped SwiGLU expert FFN over permuted rows, weights streamed from the
// expert slots: the decode path.  Experts found in the GPU cache are executed
// on the GPU ("FreeToken quantization", section "Como se desplazan los pesos
// MoE cuantizados por la memoria").
//
// Decode is bound by HBM: each touched expert's weights are read once per
// pass and every token row is reused across all of them.  Design:
//  - work unit = (token group of up to 16 rows of one expert, 128-row block
//    of W13 or W2), over the whole K; a persistent grid of three CTAs per SM
//    walks the units (round-robin, or stream-K ranges when there are fewer
//    units than CTAs, see the kernel);
//  - per CTA, one lane streams the units through a shared-memory ring with
//    1-D bulk copies (TMA engine) completed on mbarriers: a stage is four
//    64-column chunks of the block (one contiguous copy of eight 512-byte
//    tiles per chunk run), their scales and the group's activation rows;
//    eight compute warps each own one 16-row tile of the block;
//  - weights are the mma.sync m16n8k16 row operand: a lane's 16 bytes of a
//    packed tile are exactly its fragment bytes for four k16 steps; E2M1
//    pairs become f16 pairs with one cvt.rn.f16x2.e2m1x2 (exact);
//  - the activations (x gathered by token, then h) are first rewritten once
//    per call into an operand copy: f16 scaled by a power of two per row (the
//    row's largest magnitude lands in [2^14, 2^15): exact for bf16 rows,
//    11-bit for fp32 h), stored column-block-major ([64-column block][row])
//    so any 8 consecutive rows of a block are one contiguous 1 KB copy, and
//    permuted / swizzled inside each 128-byte row so a lane's fragment data
//    for four k16 steps is two conflict-free 16-byte reads;
//  - block scales are applied to fp32 partial sums: the MMA accumulates one
//    scale block (32 columns MXFP4, 16 NVFP4) from zero, then one FFMA per
//    accumulator element folds it in with the row's scale; the activation
//    row's power of two and the NVFP4 tensor scale come off in the epilogue;
//  - phase 1 tiles pair 8 gate rows with the 8 matching up rows, so the
//    SwiGLU epilogue is lane-local: h = silu(gate) * up in fp32.
// BF16 weights use the same units with bf16 fragments and a bf16 operand copy.
#include <stdlib.h>
#include <string.h>

#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {

__device__ int g_ffn_error;   // first device-side error of the decode FFN (0: none)

namespace {

constexpr int kRowsPerUnit = 16;   // 2 n-tiles of 8 tokens
constexpr int kPrepThreads = 256;
constexpr int kRowPad = 16;        // operand copies carry 16 spare rows (whole 8-row reads past the end)
constexpr long long kWaitCycles = 4000000000ll;   // ~2 s before a wait gives up

// Programmatic dependent launch: the kernels of one FFN call are launched so
// that each may start while the previous one drains; every kernel waits for
// its predecessor's results (griddepcontrol.wait, a no-op for a normal
// launch) before reading them, and lets its successor launch once all its
// CTAs are running.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ workspace
struct FfnWs {
    uint16_t* xb;     // [H/64][rows+16][64] operand copy of the input rows
    int32_t* xe;      // [rows] row exponent of xb
    float* h32;       // [rows][F] h in fp32
    uint16_t* hb;     // [F/64][rows+16][64] operand copy of h
    int32_t* he;      // [rows]
    int32_t* groups;  // [E+1] exclusive prefix of token groups per expert
    int32_t* cnt;     // [ncnt] pieces finished per unit of a unit split across CTAs
    int ncnt;
    float* pieces;    // [kMaxDecCtas][2][kPieceFloats] partial sums of split units
};

constexpr int kCW = 8;                               // compute warps of the streaming kernel
constexpr int kMaxDecCtas = 1024;                    // CTAs of one streaming launch, at most
constexpr int kPieceFloats = kCW * 2 * 32 * 4;       // one CTA's partial tile set [warp][q][lane][4]

// Units (token group x 128-row block) of a layer call, at most: token groups
// number at most rows/16 + (experts with rows) per expert, blocks max(2F, H)/128.
long dec_units_max(const moe_shape* s, int rows)
{
    const long R = 2 * s->ffn > s->hidden ? 2 * s->ffn : s->hidden;
    const long RB = (R / 16 + 7) / 8;
    const long groups = (rows + kRowsPerUnit - 1) / kRowsPerUnit + (rows < s->experts ? rows : s->experts);
    return groups * RB;
}

size_t ffn_ws_layout(const moe_shape* s, int rows, void* base, FfnWs* w)
{
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align_up(o + b, 256); return at; };
    const size_t R = rows > 0 ? rows : 1, RP = R + kRowPad;
    size_t oxb = take(2 * RP * s->hidden);
    size_t oxe = take(4 * R);
    size_t oh = take(4 * R * s->ffn);
    size_t ohb = take(2 * RP * s->ffn);
    size_t ohe = take(4 * R);
    size_t og = take(4 * (size_t)(s->experts + 1));
    const long ncnt = dec_units_max(s, (int)R);
    size_t oc = take(4 * (size_t)ncnt);
    size_t op = take(4 * (size_t)kMaxDecCtas * 2 * kPieceFloats);
    if (w) {
        char* b = static_cast<char*>(base);
        w->xb = reinterpret_cast<uint16_t*>(b + oxb);
        w->xe = reinterpret_cast<int32_t*>(b + oxe);
        w->h32 = reinterpret_cast<float*>(b + oh);
        w->hb = reinterpret_cast<uint16_t*>(b + ohb);
        w->he = reinterpret_cast<int32_t*>(b + ohe);
        w->groups = reinterpret_cast<int32_t*>(b + og);
        w->cnt = reinterpret_cast<int32_t*>(b + oc);
        w->ncnt = (int)ncnt;
        w->pieces = reinterpret_cast<float*>(b + op);
    }
    return o;
}

// Operand copy layout (the MMA B fragments of the streaming kernel): block
// kt = k/64 is [RP][64] elements.  Inside a row's block, quad lane t reads
// positions 16t..16t+15, where k16 step j's two column pairs sit at 16t+4j
// (columns 16j+2t, +1) and 16t+4j+2 (columns 16j+8+2t, +1); the eight 16-byte
// chunks of row r are stored XOR-swizzled by r&7.

// ------------------------------------------------------------------ prep
// Operand copy (+ row exponent) of a bf16 or fp32 row
// (read directly, or token gather[r]/gk of the source).  With `groups` set,
// the last CTA writes the per-expert token-group prefix and clears `zero`.  ROWMAJOR writes a
// plain [rows][K] f16 copy (the tensor-core path's TMA source) instead of the
// column-block-major fragment layout.
template <bool IN_F32, bool OUT_F16, bool ROWMAJOR = false>
__global__ void __launch_bounds__(kPrepThreads) ffn_prep_kernel(const void* __restrict__ in, int rows, int K,
                                                                uint16_t* __restrict__ out, int32_t* __restrict__ ex,
                                                                const int32_t* __restrict__ offsets,
                                                                const int32_t* __restrict__ slot_of, int E,
                                                                int pool_slots, int32_t* __restrict__ groups,
                                                                const int32_t* __restrict__ gather, int gk,
                                                                int32_t* __restrict__ zero, int nzero)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    if (groups && blockIdx.x == gridDim.x - 1) {
        for (int i = threadIdx.x; i < nzero; i += kPrepThreads) zero[i] = 0;
        __shared__ int s_warp[kPrepThreads / 32];
        const int EPT = (E + kPrepThreads - 1) / kPrepThreads;   // <= 16 for E <= 4096
        int loc = 0, cnts[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            int e = threadIdx.x * EPT + i, gcount = 0;
            if (i < EPT && e < E) {
                int m = offsets[e + 1] - offsets[e];
                int sl = slot_of[e];
                bool ok = m > 0 && sl >= 0 && sl < pool_slots && offsets[e] >= 0 && offsets[e + 1] <= rows;
                gcount = ok ? (m + kRowsPerUnit - 1) / kRowsPerUnit : 0;
            }
            cnts[i] = gcount;
            loc += gcount;
        }
        int inc = loc;
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) s_warp[threadIdx.x >> 5] = inc;
        __syncthreads();
        int run = inc - loc;
        for (int w = 0; w < (int)(threadIdx.x >> 5); w++) run += s_warp[w];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            int e = threadIdx.x * EPT + i;
            if (i < EPT && e < E) groups[e] = run;
            run += cnts[i];
        }
        if (threadIdx.x == kPrepThreads - 1) groups[E] = run;
        return;
    }
    // one CTA per row: pass 1 finds the row's largest magnitude (f16 copies
    // are scaled by a power of two), pass 2 writes 16-byte output chunks
    __shared__ float s_max[kPrepThreads / 32 + 1];
    const int RP = rows + kRowPad;
    const int nblocks = gridDim.x - (groups ? 1 : 0);
    const int nch = K / 8;   // 8-element chunks per row
    const int wid = threadIdx.x >> 5;
    for (int r = blockIdx.x; r < rows; r += nblocks) {
        const size_t sr = gather ? (size_t)(__ldg(gather + r) / gk) : (size_t)r;   // source row
        const float* inf = static_cast<const float*>(in) + sr * K;
        const uint16_t* inb = static_cast<const uint16_t*>(in) + sr * K;
        int p = 0;
        if (OUT_F16) {
            float mx = 0.0f;
            for (int c = threadIdx.x; c < nch; c += kPrepThreads) {
                if (IN_F32) {
                    const float4 a = __ldg(reinterpret_cast<const float4*>(inf + 8 * c));
                    const float4 b = __ldg(reinterpret_cast<const float4*>(inf + 8 * c) + 1);
                    mx = fmaxf(mx, fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))),
                                         fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w)))));
                } else {
                    const uint4 q = __ldg(reinterpret_cast<const uint4*>(inb + 8 * c));
                    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        mx = fmaxf(mx, fmaxf(fabsf(bf16_bits_to_f32(u[i] & 0xFFFF)), fabsf(bf16_bits_to_f32(u[i] >> 16))));
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) s_max[wid] = mx;
            __syncthreads();
            if (threadIdx.x == 0) {
                float m = 0.0f;
                for (int i = 0; i < kPrepThreads / 32; i++) m = fmaxf(m, s_max[i]);
                s_max[kPrepThreads / 32] = m;
            }
            __syncthreads();
            mx = s_max[kPrepThreads / 32];
            if (mx > 0.0f && mx <= 3.4e38f) {
                int e2;
                frexpf(mx, &e2);          // mx = m * 2^e2, m in [0.5, 1)
                p = 15 - e2;              // mx * 2^p in [2^14, 2^15)
                p = p < -100 ? -100 : (p > 100 ? 100 : p);
            }
            if (threadIdx.x == 0) ex[r] = p;
        }
        const float sc = ldexpf(1.0f, p);
        auto cvt2 = [&](float v0, float v1) -> uint32_t {
            if (OUT_F16) {
                const __half2 h = __floats2half2_rn(v0 * sc, v1 * sc);
                return *reinterpret_cast<const uint32_t*>(&h);
            }
            return (uint32_t)f32_to_bf16_bits(v0) | ((uint32_t)f32_to_bf16_bits(v1) << 16);
        };
        // two adjacent source columns (col even)
        auto pair = [&](int col) -> uint32_t {
            if (IN_F32) {
                const float2 v = __ldg(reinterpret_cast<const float2*>(inf + col));
                return cvt2(v.x, v.y);
            }
            const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(inb + col));
            return cvt2(bf16_bits_to_f32(q & 0xFFFF), bf16_bits_to_f32(q >> 16));
        };
        for (int c = threadIdx.x; c < nch; c += kPrepThreads) {
            uint4 o;
            if (ROWMAJOR) {
                o = make_uint4(pair(8 * c), pair(8 * c + 2), pair(8 * c + 4), pair(8 * c + 6));
                *reinterpret_cast<uint4*>(out + (size_t)r * K + 8 * c) = o;
            } else {
                // output chunk cc of 64-column block kt holds, for j = 2(cc&1) + jj
                // and t = cc/2, the pairs at columns 16j + 8h + 2t (element 4jj + 2h)
                const int kt = c >> 3, cc = c & 7, t = cc >> 1, jb = 2 * (cc & 1);
                const int base = 64 * kt + 16 * jb + 2 * t;
                o = make_uint4(pair(base), pair(base + 8), pair(base + 16), pair(base + 24));
                *reinterpret_cast<uint4*>(out + ((size_t)kt * RP + r) * 64 + (size_t)((cc ^ (r & 7)) * 8)) = o;
            }
        }
        if (OUT_F16) __syncthreads();   // s_max is reused by the next row
    }
}

// ------------------------------------------------------------------ GEMM units
struct FfnArgs {
    const char* pool;
    size_t slot_bytes;
    size_t w_off, s_off, ts_off;
    int R, K, E;
    const int32_t* slot_of;
    const int32_t* offsets;
    const int32_t* groups;
    int rows;
    const uint16_t* in;     // operand copy [K/64][rows+16][64]
    const int32_t* in_ex;   // [rows] its exponents (FP4 formats)
    float* out_h;           // phase 1: h [rows][R/2] fp32
    uint16_t* out_y;        // phase 2: y [rows][R] bf16
    int32_t* cnt;           // per unit: pieces finished (units split across CTAs)
    float* pieces;          // [gridDim.x][2][kPieceFloats]
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the thread for up to kSuspendNs
// while the phase is incomplete (it resumes when the phase completes), so
// waiting warps do not take issue slots from working ones.
constexpr uint32_t kSuspendNs = 20000;

__device__ __forceinline__ bool mbar_try_suspend(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity), "n"(kSuspendNs)
                 : "memory");
    return ok != 0;
}

// Bounded wait (about 2 s of clock), false on timeout.  With `abort` set the
// wait also gives up as soon as another warp of the CTA has raised it, and
// raises it itself on a timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort = nullptr)
{
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_suspend(bar, parity)) return true;
        if (abort && *abort) return false;
        if (clock64() - t0 > kWaitCycles) {
            if (abort) *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void e2m1x4_to_f16x2(uint32_t w, uint32_t& f0, uint32_t& f1, uint32_t& f2, uint32_t& f3)
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

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    if (F16)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%0,%1,%2,%3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%0,%1,%2,%3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// E8M0 code -> 2^(c-127) (codes 114..140 only reach the kernels)
__device__ __forceinline__ float mx_scale(uint32_t c) { return __uint_as_float(c << 23); }

// E4M3 code -> value (subnormals m * 2^-9; NaN codes are rejected at packing)
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    const uint32_t s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    float v = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return s ? -v : v;
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// ---- CTA-cooperative weight streaming -------------------------------------
// Work is a list of units (token group of one expert, 128-row block of W),
// each KP = ceil(K/128) stages of two 64-column chunks long.  With at least
// as many units as CTAs, CTAs take whole units round-robin.  Otherwise the
// concatenated stage list is cut into equal ranges over the CTAs (stream-K):
// a CTA runs whole units where its range covers them and pieces of the units
// at its range ends.  A piece's partial sums go to a per-CTA buffer; the CTA that
// finishes a unit's last piece adds all pieces in CTA order (deterministic)
// and writes the result.
// Inside a CTA, warp 8 (one lane) fills a ring stage with bulk copies: the
// block's FP4 (or bf16) tiles of KC consecutive chunks (contiguous in the
// slot), their scales, and the token group's 8 or 16 activation rows of each
// chunk.  Warps 0..7 each multiply the 16-row tile they own in every chunk of
// the stage and then release it on an mbarrier.
constexpr int kDecThreads = 32 * (kCW + 1);   // + one copy-issue warp

template <int WFMT>
struct DecCfg {
    static constexpr bool FP4 = WFMT != MOE_W_BF16;
    static constexpr int TILE = FP4 ? 512 : 2048;
    static constexpr int KC = FP4 ? 4 : 1;                       // 64-column chunks per stage
    static constexpr int STILE = (WFMT == MOE_W_MXFP4) ? 32 : (WFMT == MOE_W_NVFP4 ? 64 : 0);
    static constexpr int D = FP4 ? 2 : 4;                        // ring stages
    static constexpr int A_BYTES = KC * kCW * TILE;
    static constexpr int S_BYTES = KC * kCW * STILE;
    static constexpr int X_CHUNK = 2 * 1024;                     // up to 16 rows x 128 bytes
    static constexpr int STAGE = A_BYTES + S_BYTES + KC * X_CHUNK;
};

template <int WFMT>
size_t dec_smem_bytes(int E)
{
    return 1024 + (size_t)DecCfg<WFMT>::D * DecCfg<WFMT>::STAGE + 4 * (size_t)(E + 1);
}

struct DecUnit {
    int e, G, ng, row0, row_end, nq, k0, k1;
    const char* blob;
};

// Unit u, column chunks [k0, k1).
__device__ __forceinline__ DecUnit dec_unit(const FfnArgs& a, const int* s_groups, int u, int RT, int RB, int k0,
                                            int k1)
{
    DecUnit U;
    U.G = u % RB;
    const int gi = u / RB;
    int lo = 0, hi = a.E - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (s_groups[mid] <= gi) lo = mid;
        else hi = mid - 1;
    }
    U.e = lo;
    U.row0 = a.offsets[lo] + (gi - s_groups[lo]) * kRowsPerUnit;
    U.row_end = min(min(a.offsets[lo + 1], U.row0 + kRowsPerUnit), a.rows);
    U.nq = (U.row_end - U.row0 + 7) >> 3;
    U.ng = min(8, RT - 8 * U.G);
    U.k0 = k0;
    U.k1 = k1;
    U.blob = a.pool + (size_t)a.slot_of[lo] * a.slot_bytes;
    return U;
}

// Stage-list ranges: CTA c owns [bound(c), bound(c+1)).
__device__ __forceinline__ long dec_bound(long W, int c, int grid) { return W * c / grid; }

__device__ __forceinline__ int dec_cta_of(long W, long idx, int grid)
{
    int c = (int)(idx * grid / W);
    while (c + 1 < grid && dec_bound(W, c + 1, grid) <= idx) c++;
    while (c > 0 && dec_bound(W, c, grid) > idx) c--;
    return c;
}

// Operands of one 16-row x 64-column tile in registers.
template <int WFMT, int NQ>
struct TileRegs {
    uint4 w[WFMT == MOE_W_BF16 ? 4 : 1];
    uint2 sc;
    uint4 x[NQ][2];
};

template <int WFMT, int NQ>
__device__ __forceinline__ void load_tile(TileRegs<WFMT, NQ>& T, const unsigned char* sg, int c, int ng, int w,
                                          int lane, int g, int t, int sw)
{
    using CFG = DecCfg<WFMT>;
    const unsigned char* wt = sg + (c * ng + w) * CFG::TILE + 16 * lane;
#pragma unroll
    for (int v = 0; v < (CFG::FP4 ? 1 : 4); v++) T.w[v] = *reinterpret_cast<const uint4*>(wt + v * 512);
    const unsigned char* st = sg + CFG::A_BYTES + (c * ng + w) * CFG::STILE;
    if (WFMT == MOE_W_MXFP4) T.sc.x = *reinterpret_cast<const uint32_t*>(st + 4 * g);
    if (WFMT == MOE_W_NVFP4) T.sc = *reinterpret_cast<const uint2*>(st + 8 * g);
#pragma unroll
    for (int q = 0; q < NQ; q++) {
        const unsigned char* xrow = sg + CFG::A_BYTES + CFG::S_BYTES + c * CFG::X_CHUNK + q * 1024 + g * 128;
        T.x[q][0] = *reinterpret_cast<const uint4*>(xrow + (((2 * t) ^ sw) << 4));
        T.x[q][1] = *reinterpret_cast<const uint4*>(xrow + (((2 * t + 1) ^ sw) << 4));
    }
}

// Multiply-accumulate of one tile.  FP4: the MMAs of one scale block sum
// into a zeroed fp32 block result that is then scaled into the accumulator
// (two independent chains per tile for MXFP4, four for NVFP4).
template <int WFMT, int NQ>
__device__ __forceinline__ void mma_tile(float (&acc)[2][4], const TileRegs<WFMT, NQ>& T)
{
    if (WFMT == MOE_W_BF16) {
        // bf16 fragments: w[j] = {a0, a2, a1, a3} of step j
#pragma unroll
        for (int q = 0; q < NQ; q++) {
            const uint32_t X[8] = {T.x[q][0].x, T.x[q][0].y, T.x[q][0].z, T.x[q][0].w,
                                   T.x[q][1].x, T.x[q][1].y, T.x[q][1].z, T.x[q][1].w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                mma16816<false>(acc[q], T.w[j].x, T.w[j].z, T.w[j].y, T.w[j].w, X[2 * j], X[2 * j + 1]);
        }
        return;
    }
    // f16 fragments from E2M1 bytes: row g bytes in .x/.y, row g+8 in .z/.w;
    // byte 2j -> a0 (a1) of step j, byte 2j+1 -> a2 (a3)
    uint32_t A[4][4];
    uint32_t f0, f1, f2, f3;
    e2m1x4_to_f16x2(T.w[0].x, f0, f1, f2, f3);
    A[0][0] = f0; A[0][2] = f1; A[1][0] = f2; A[1][2] = f3;
    e2m1x4_to_f16x2(T.w[0].y, f0, f1, f2, f3);
    A[2][0] = f0; A[2][2] = f1; A[3][0] = f2; A[3][2] = f3;
    e2m1x4_to_f16x2(T.w[0].z, f0, f1, f2, f3);
    A[0][1] = f0; A[0][3] = f1; A[1][1] = f2; A[1][3] = f3;
    e2m1x4_to_f16x2(T.w[0].w, f0, f1, f2, f3);
    A[2][1] = f0; A[2][3] = f1; A[3][1] = f2; A[3][3] = f3;
    float sg4[4], s84[4];   // scale of k16 steps 0..3 for rows g and g+8
    if (WFMT == MOE_W_MXFP4) {
        sg4[0] = sg4[1] = mx_scale(T.sc.x & 0xFF);
        sg4[2] = sg4[3] = mx_scale((T.sc.x >> 8) & 0xFF);
        s84[0] = s84[1] = mx_scale((T.sc.x >> 16) & 0xFF);
        s84[2] = s84[3] = mx_scale(T.sc.x >> 24);
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            sg4[j] = e4m3_value((T.sc.x >> (8 * j)) & 0xFF);
            s84[j] = e4m3_value((T.sc.y >> (8 * j)) & 0xFF);
        }
    }
    constexpr int SPB = (WFMT == MOE_W_MXFP4) ? 2 : 1;   // k16 steps per scale block
#pragma unroll
    for (int q = 0; q < NQ; q++) {
        const uint32_t X[8] = {T.x[q][0].x, T.x[q][0].y, T.x[q][0].z, T.x[q][0].w,
                               T.x[q][1].x, T.x[q][1].y, T.x[q][1].z, T.x[q][1].w};
#pragma unroll
        for (int j0 = 0; j0 < 4; j0 += SPB) {
            float tmp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = j0; j < j0 + SPB; j++)
                mma16816<true>(tmp, A[j][0], A[j][1], A[j][2], A[j][3], X[2 * j], X[2 * j + 1]);
            acc[q][0] = __fmaf_rn(tmp[0], sg4[j0], acc[q][0]);
            acc[q][1] = __fmaf_rn(tmp[1], sg4[j0], acc[q][1]);
            acc[q][2] = __fmaf_rn(tmp[2], s84[j0], acc[q][2]);
            acc[q][3] = __fmaf_rn(tmp[3], s84[j0], acc[q][3]);
        }
    }
}

// Ring position shared by the compute warps.
struct Ring {
    int st;
    uint32_t ph;
    __device__ __forceinline__ void next(int D)
    {
        if (++st == D) { st = 0; ph ^= 1; }
    }
};

// One unit's stages for a compute warp: wait, multiply its tile of both
// chunks, release.  Returns false when a wait gave up.
template <int WFMT, int NQ>
__device__ __forceinline__ bool run_unit(float (&acc)[2][4], const DecUnit& U, bool act, Ring& R,
                                         unsigned char* ring, uint64_t* full, uint64_t* empty, int w, int lane,
                                         volatile int* abort)
{
    using CFG = DecCfg<WFMT>;
    const int g = lane >> 2, t = lane & 3, sw = (U.row0 + g) & 7;
    for (int kt = U.k0; kt < U.k1; kt += CFG::KC) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&full[R.st]), R.ph, abort))) return false;
        const unsigned char* sg = ring + (size_t)R.st * CFG::STAGE;
        if (act) {
            // one tile's operands live at a time; the stage is released after both
            TileRegs<WFMT, NQ> T;
#pragma unroll
            for (int cc = 0; cc < CFG::KC; cc++) {
                if (kt + cc < U.k1) {
                    load_tile<WFMT, NQ>(T, sg, cc, U.ng, w, lane, g, t, sw);
                    mma_tile<WFMT, NQ>(acc, T);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[R.st]));
        R.next(CFG::D);
    }
    return true;
}

// Final values of a warp's tile: undo the activation row exponents, apply
// the NVFP4 tensor scale, then h = silu(gate) * up (phase 1) or y in bf16.
template <int WFMT, int PHASE>
__device__ __forceinline__ void write_tile(const FfnArgs& a, const DecUnit& U, int rt, const float (&acc)[2][4],
                                           int g, int t)
{
    float tsc = 1.0f;
    if (WFMT == MOE_W_NVFP4) tsc = reinterpret_cast<const float*>(U.blob + a.ts_off)[PHASE - 1];
#pragma unroll
    for (int q = 0; q < 2; q++) {
        if (q >= U.nq) break;
        const int r0 = U.row0 + q * 8 + 2 * t, r1 = r0 + 1;
        float u0 = tsc, u1 = tsc;
        if (WFMT != MOE_W_BF16) {
            if (r0 < U.row_end) u0 = tsc * pow2i(-__ldg(a.in_ex + r0));
            if (r1 < U.row_end) u1 = tsc * pow2i(-__ldg(a.in_ex + r1));
        }
        if (PHASE == 1) {
            const int F = a.R / 2;
            const int f = 8 * rt + g;
            if (r0 < U.row_end) a.out_h[(size_t)r0 * F + f] = silu(acc[q][0] * u0) * (acc[q][2] * u0);
            if (r1 < U.row_end) a.out_h[(size_t)r1 * F + f] = silu(acc[q][1] * u1) * (acc[q][3] * u1);
        } else {
            const int Ho = a.R;
            const int o = 16 * rt + g;
            if (r0 < U.row_end) {
                a.out_y[(size_t)r0 * Ho + o] = f32_to_bf16_bits(acc[q][0] * u0);
                a.out_y[(size_t)r0 * Ho + o + 8] = f32_to_bf16_bits(acc[q][2] * u0);
            }
            if (r1 < U.row_end) {
                a.out_y[(size_t)r1 * Ho + o] = f32_to_bf16_bits(acc[q][1] * u1);
                a.out_y[(size_t)r1 * Ho + o + 8] = f32_to_bf16_bits(acc[q][3] * u1);
            }
        }
    }
}

// Segments of one CTA: whole units u = blockIdx.x + i * gridDim.x, or the
// stream-K pieces of its stage range [pos, end): unit u, stages [p0, p1).
struct Seg {
    long pos;     // next unit (whole) or next stage (stream-K)
    long start;   // first stage of the current segment (stream-K)
    int u, p0, p1;
    __device__ __forceinline__ bool next(bool whole, int NU, int KP, long end)
    {
        if (whole) {
            if (pos >= NU) return false;
            u = (int)pos;
            p0 = 0;
            p1 = KP;
            pos += gridDim.x;
            return true;
        }
        if (pos >= end) return false;
        start = pos;
        u = (int)(pos / KP);
        p0 = (int)(pos % KP);
        p1 = (int)min((long)KP, p0 + (end - pos));
        pos += p1 - p0;
        return true;
    }
};

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kCW) : "memory"); }

template <int WFMT, int PHASE>
__global__ void __launch_bounds__(kDecThreads, 3) ffn_kernel(FfnArgs a)
{
    using CFG = DecCfg<WFMT>;
    constexpr int TILE = CFG::TILE, STILE = CFG::STILE, D = CFG::D, STAGE = CFG::STAGE;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);            // [D]
    uint64_t* empty = full + D;                                     // [D]
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + 512);
    volatile int* s_last = reinterpret_cast<volatile int*>(smem + 516);
    unsigned char* ring = smem + 1024;
    int* s_groups = reinterpret_cast<int*>(ring + (size_t)D * STAGE);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
    const int RT = a.R / 16, RB = (RT + 7) / 8, KT = a.K / 64, KP = (KT + CFG::KC - 1) / CFG::KC, RP = a.rows + kRowPad;
    pdl_wait();
    for (int i = tid; i <= a.E; i += kDecThreads) s_groups[i] = a.groups[i];
    if (tid == 0) {
        for (int i = 0; i < D; i++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&full[i])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&empty[i])), "r"(kCW) : "memory");
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    pdl_trigger();
    // With at least one unit per CTA, whole units go round-robin (an SM's
    // CTAs share its issue slots, so uneven unit counts per CTA even out per
    // SM); with fewer units than CTAs, the units' stages are cut into equal
    // ranges over the CTAs (stream-K).
    const int NU = s_groups[a.E] * RB;
    const bool whole = NU >= (int)gridDim.x;
    const long W = whole ? 0 : (long)NU * KP;     // stream-K stages
    // CTAs in the stream-K part: no more than stages, so that no range is empty
    const int grid = (int)(W < (long)gridDim.x ? W : (long)gridDim.x);
    const bool in_use = (int)blockIdx.x < grid;
    const long b0 = in_use ? dec_bound(W, blockIdx.x, grid) : 0, b1 = in_use ? dec_bound(W, blockIdx.x + 1, grid) : 0;

    if (w == kCW) {
        // ------------------------------------------------ copy issue (one lane)
        if (lane == 0) {
            int st = 0;
            uint32_t ph = 0;
            long issued = 0;
            bool ok = true;
            auto issue = [&](const DecUnit& U) {
                for (int kt = U.k0; kt < U.k1 && ok; kt += CFG::KC) {
                    const int nc = min(CFG::KC, U.k1 - kt);
                    if (!(ok = mbar_wait_bounded(smem_u32(&empty[st]), ph ^ 1, s_abort))) break;
                    const uint32_t bar = smem_u32(&full[st]);
                    unsigned char* sg = ring + (size_t)st * STAGE;
                    const size_t ti = tile_index(8 * U.G, kt, RT, KT);   // chunks kt, kt+1 are adjacent
                    const uint32_t bytes = nc * (U.ng * (TILE + STILE) + U.nq * 1024);
                    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                                 : "memory");
                    bulk_copy(smem_u32(sg), U.blob + a.w_off + ti * TILE, nc * U.ng * TILE, bar);
                    if (STILE)
                        bulk_copy(smem_u32(sg + CFG::A_BYTES), U.blob + a.s_off + ti * STILE, nc * U.ng * STILE, bar);
                    for (int c = 0; c < nc; c++)
                        bulk_copy(smem_u32(sg + CFG::A_BYTES + CFG::S_BYTES + c * CFG::X_CHUNK),
                                  a.in + ((size_t)(kt + c) * RP + U.row0) * 64, U.nq * 1024, bar);
                    issued++;
                    if (++st == D) { st = 0; ph ^= 1; }
                }
            };
            Seg sg{whole ? (long)blockIdx.x : b0};
            while (ok && sg.next(whole, NU, KP, b1))
                issue(dec_unit(a, s_groups, sg.u, RT, RB, CFG::KC * sg.p0, min(KT, CFG::KC * sg.p1)));
            if (!ok) atomicCAS(&g_ffn_error, 0, (int)MOE_ERR_TIMEOUT);
            // let the last copies land before the CTA exits (stage i was last
            // filled in this pass if i < st, else in the previous one)
            for (int i = 0; i < D && i < issued; i++)
                mbar_wait_bounded(smem_u32(&full[i]), i < st ? ph : (ph ^ 1));
        }
        return;
    }

    // ------------------------------------------------ compute warps
    // Every compute warp walks the same segments and meets the same named
    // barriers; after a failed wait a warp keeps walking without waiting.
    Ring R{0, 0};
    bool ok = true;
    auto multiply = [&](const DecUnit& U, float (&acc)[2][4]) {
#pragma unroll
        for (int q = 0; q < 2; q++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[q][i] = 0.0f;
        if (ok)
            ok = U.nq == 1 ? run_unit<WFMT, 1>(acc, U, w < U.ng, R, ring, full, empty, w, lane, s_abort)
                           : run_unit<WFMT, 2>(acc, U, w < U.ng, R, ring, full, empty, w, lane, s_abort);
    };
    Seg sg{whole ? (long)blockIdx.x : b0};
    while (sg.next(whole, NU, KP, b1)) {
        const int u = sg.u, p0 = sg.p0, p1 = sg.p1;
        const long idx = sg.start;
        const DecUnit U = dec_unit(a, s_groups, u, RT, RB, CFG::KC * p0, min(KT, CFG::KC * p1));
        const bool act = w < U.ng;          // this warp has a row tile in the block
        const int rt = 8 * U.G + w;
        float acc[2][4];
        multiply(U, acc);
        if (p0 == 0 && p1 == KP) {
            if (ok && act) write_tile<WFMT, PHASE>(a, U, rt, acc, g, t);
        } else {
            // a piece: publish the partial sums, count the piece, and let the
            // CTA that completes the unit add all pieces up in CTA order
            const int slot = idx == b0 ? 0 : 1;
            float* mine = a.pieces + ((size_t)blockIdx.x * 2 + slot) * kPieceFloats;
            if (ok && act)
#pragma unroll
                for (int q = 0; q < 2; q++)
                    if (q < U.nq)
                        *reinterpret_cast<float4*>(mine + ((w * 2 + q) * 32 + lane) * 4) =
                            make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
            __threadfence();
            compute_bar();
            const long u_lo = (long)u * KP, u_hi = u_lo + KP - 1;
            const int c_lo = dec_cta_of(W, u_lo, grid), c_hi = dec_cta_of(W, u_hi, grid);
            if (tid == 0) {
                int last = 0;
                if (!*s_abort) last = atomicAdd(a.cnt + u, 1) == c_hi - c_lo;
                *s_last = last;
            }
            compute_bar();
            if (*s_last) {
                __threadfence();
                if (ok && act) {
                    float sum[2][4];
#pragma unroll
                    for (int q = 0; q < 2; q++)
#pragma unroll
                        for (int i = 0; i < 4; i++) sum[q][i] = 0.0f;
                    for (int c = c_lo; c <= c_hi; c++) {
                        const int sl = dec_bound(W, c, grid) >= u_lo ? 0 : 1;
                        const float* pc = a.pieces + ((size_t)c * 2 + sl) * kPieceFloats;
#pragma unroll
                        for (int q = 0; q < 2; q++)
                            if (q < U.nq) {
                                const float4 v = __ldcg(reinterpret_cast<const float4*>(pc + ((w * 2 + q) * 32 + lane) * 4));
                                sum[q][0] += v.x; sum[q][1] += v.y; sum[q][2] += v.z; sum[q][3] += v.w;
                            }
                    }
                    write_tile<WFMT, PHASE>(a, U, rt, sum, g, t);
                }
                if (tid == 0) a.cnt[u] = 0;
            }
        }
    }
    if (!ok && lane == 0) atomicCAS(&g_ffn_error, 0, (int)MOE_ERR_TIMEOUT);
}

template <int WFMT>
int launch_decode(const moe_shape* s, const BlobLayout& bl, const void* pool, size_t slot_bytes, int pool_slots,
                  const int32_t* slot_of, const int32_t* offsets, const uint16_t* x_perm, int rows,
                  uint16_t* y_perm, const FfnWs& w, int sms, cudaStream_t st, const RowSource* gather)
{
    constexpr bool FP4 = WFMT != MOE_W_BF16;
    const int E = s->experts, H = s->hidden, F = s->ffn;
    int prep_blocks = rows < sms * 8 ? rows : sms * 8;   // a CTA per row
    const void* src = gather ? gather->x : static_cast<const void*>(x_perm);
    const int32_t* gidx = gather ? gather->assign_of : nullptr;
    const int gk = gather ? gather->k : 1;
    if (gather && gather->x_dtype == MOE_DT_F32)
        MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<true, FP4>, prep_blocks + 1, kPrepThreads, 0, st, src, rows, H, w.xb,
                                w.xe, offsets, slot_of, E, pool_slots, w.groups, gidx, gk, w.cnt, w.ncnt));
    else
        MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<false, FP4>, prep_blocks + 1, kPrepThreads, 0, st, src, rows, H, w.xb,
                                w.xe, offsets, slot_of, E, pool_slots, w.groups, gidx, gk, w.cnt, w.ncnt));
    FfnArgs a{};
    a.pool = static_cast<const char*>(pool);
    a.slot_bytes = slot_bytes;
    a.ts_off = bl.ts;
    a.E = E;
    a.slot_of = slot_of;
    a.offsets = offsets;
    a.groups = w.groups;
    a.rows = rows;
    a.cnt = w.cnt;
    a.pieces = w.pieces;
    const size_t smem = dec_smem_bytes<WFMT>(E);
    // persistent grid: as many CTAs as fit at once (recomputed when the
    // shared-memory size, which grows with E, changes)
    // function attributes and occupancy are per device (context)
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    static size_t attr_smem_dev[kMaxDevices], occ_smem_dev[kMaxDevices];
    static int resident_dev[kMaxDevices];
    size_t& attr_smem = attr_smem_dev[dev];
    size_t& occ_smem = occ_smem_dev[dev];
    int& resident = resident_dev[dev];
    if (smem > attr_smem) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<WFMT, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<WFMT, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        // several CTAs share an SM: take the largest shared-memory split
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<WFMT, 1>, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<WFMT, 2>, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        attr_smem = smem;
    }
    if (smem != occ_smem) {
        MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, ffn_kernel<WFMT, 1>, kDecThreads, smem));
        if (resident < 1) resident = 1;
        occ_smem = smem;
    }
    long grid = (long)sms * resident;
    if (grid > kMaxDecCtas) grid = kMaxDecCtas;
    // no more CTAs than stages (upper bound of the stage count: every unit possible)
    auto grid_for = [&](int R, int K) {
        const long RB = (R / 16 + 7) / 8, KP = (K / 64 + DecCfg<WFMT>::KC - 1) / DecCfg<WFMT>::KC;
        const long groups = (rows + kRowsPerUnit - 1) / kRowsPerUnit + (rows < E ? rows : E);
        const long wmax = groups * RB * KP;
        return (int)(wmax < grid ? (wmax < 1 ? 1 : wmax) : grid);
    };
    a.w_off = bl.w13;
    a.s_off = bl.s13;
    a.R = 2 * F;
    a.K = H;
    a.in = w.xb;
    a.in_ex = w.xe;
    a.out_h = w.h32;
    MOE_CUDA_TRY(launch_pdl(ffn_kernel<WFMT, 1>, grid_for(2 * F, H), kDecThreads, smem, st, a));
    MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<true, FP4>, prep_blocks, kPrepThreads, 0, st,
                            static_cast<const void*>(w.h32), rows, F, w.hb, w.he, nullptr, nullptr, E, 0, nullptr,
                            nullptr, 1, nullptr, 0));
    FfnArgs b = a;
    b.w_off = bl.w2;
    b.s_off = bl.s2;
    b.R = H;
    b.K = F;
    b.in = w.hb;
    b.in_ex = w.he;
    b.out_h = nullptr;
    b.out_y = y_perm;
    MOE_CUDA_TRY(launch_pdl(ffn_kernel<WFMT, 2>, grid_for(H, F), kDecThreads, smem, st, b));
    return MOE_OK;
}

// Grouped GEMM on tcgen05 when groups are large (prefill: rows >= 4 per
// expert on average) and the weights are FP4; the weight-streaming mma.sync
// kernels otherwise.  MOE_FFN_PATH=mma|tc overrides the choice.
bool use_tc_path(const moe_shape* s, int rows)
{
    if (!ffn_tc_supported(s)) return false;
    const char* force = getenv("MOE_FFN_PATH");
    if (force && !strcmp(force, "mma")) return false;
    if (force && !strcmp(force, "tc")) return true;
    return rows >= 4 * s->experts;
}

}  // namespace

size_t ffn_ws_bytes(const moe_shape* s, int rows) { return ffn_ws_layout(s, rows, nullptr, nullptr) + 256; }

int ffn_device_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_ffn_error, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    if (clear && v) {
        int z = 0;
        if (cudaMemcpyToSymbol(g_ffn_error, &z, sizeof z) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return v;
}

int launch_ffn(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
               const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm, void* ws,
               cudaStream_t st, const RowSource* gather)
{
    if (rows == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_FFN, st);
    FfnWs w;
    ffn_ws_layout(s, rows, ws, &w);
    int dev0 = 0, sms0 = 148;
    cudaGetDevice(&dev0);
    cudaDeviceGetAttribute(&sms0, cudaDevAttrMultiProcessorCount, dev0);
    if (use_tc_path(s, rows)) {
        // tensor-core path: f16 operand rows (x, then h), each scaled by a power of two
        prof_count(MOE_PROF_FFN, 4);
        const int pb = rows < sms0 * 8 ? rows : sms0 * 8;   // a CTA per row
        if (gather && gather->x_dtype == MOE_DT_F32)   // token rows gathered straight from x
            ffn_prep_kernel<true, true, true><<<pb, kPrepThreads, 0, st>>>(gather->x, rows, s->hidden, w.xb, w.xe,
                                                                            nullptr, nullptr, s->experts, 0, nullptr,
                                                                            gather->assign_of, gather->k, nullptr, 0);
        else
            ffn_prep_kernel<false, true, true><<<pb, kPrepThreads, 0, st>>>(
                gather ? gather->x : static_cast<const void*>(x_perm), rows, s->hidden, w.xb, w.xe, nullptr, nullptr,
                s->experts, 0, nullptr, gather ? gather->assign_of : nullptr, gather ? gather->k : 1, nullptr, 0);
        MOE_LAUNCH_CHECK();
        TcOperands op{w.xb, w.xe, w.h32, w.hb, w.he};
        return launch_ffn_tc(s, pool, slot_bytes, pool_slots, slot_of, offsets, rows, y_perm, op, st, [&]() -> int {
            ffn_prep_kernel<true, true, true><<<pb, kPrepThreads, 0, st>>>(w.h32, rows, s->ffn, w.hb, w.he, nullptr,
                                                                            nullptr, s->experts, 0, nullptr, nullptr, 1,
                                                                            nullptr, 0);
            MOE_LAUNCH_CHECK();
            return MOE_OK;
        });
    }
    prof_count(MOE_PROF_FFN, 4);
    BlobLayout bl = blob_layout(s);
    const int sms = sms0;
    switch (s->wfmt) {
    case MOE_W_BF16:
        return launch_decode<MOE_W_BF16>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows, y_perm,
                                         w, sms, st, gather);
    case MOE_W_MXFP4:
        return launch_decode<MOE_W_MXFP4>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows,
                                          y_perm, w, sms, st, gather);
    case MOE_W_NVFP4:
        return launch_decode<MOE_W_NVFP4>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows,
                                          y_perm, w, sms, st, gather);
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
