// Grouped SwiGLU expert FFN for FP4 expert weights (MXFP4, NVFP4) on the
// block-scaled fifth-generation tensor cores: the experts found in the GPU
// cache execute on the GPU ("FreeToken quantization", section "Como se
// desplazan los pesos MoE cuantizados por la memoria"; "FreeToken 290b
// model", section "Como gestiona FreeToken el prellenado y la
// decodificacion").
//
// Design for sm_100a:
//  - the weights stay E2M1 with their block scales all the way into the
//    tensor core: tcgen05.mma kind::mxf4 (E8M0 scale per 32 columns, MXFP4)
//    or kind::mxf4nvf4 block16 (unsigned E4M3 scale per 16 columns, NVFP4)
//    multiplies them as they sit in shared memory, with the scale factors in
//    tensor memory.  No SM instruction touches a weight byte;
//  - the slot blob stores every 128-row x 256-column block of a matrix as the
//    exact shared-memory image the MMA reads (rows of 128 bytes in the
//    128-byte swizzle) followed by its scale-factor images (the layout one
//    tcgen05.cp 32x128b.warpx4 moves to tensor memory), so one bulk copy per
//    pipeline stage brings weights and scales in (see common.cuh);
//  - the activations (x rows, then h rows) are rewritten once per call as a
//    short sum of E2M1 terms, each with its own block scale of the weights'
//    scale type: term t+1 encodes what terms 0..t left over, so T terms carry
//    about 3.3 T bits of each block (T = 4 for decode, 3 for prefill: about
//    2e-4 and 2e-3 relative error).  The terms of a token are consecutive
//    rows of the MMA's N operand and are summed in the epilogue;
//  - swap-AB tiles: 128 weight rows are M, (terms x tokens) are N (up to 64
//    for decode, 192 for prefill), K advances 64 columns per MMA, 256 per
//    pipeline stage;
//  - one persistent CTA per SM: warp 0 issues the bulk copies, warp 1 the
//    scale-factor copies and MMAs (one thread each), warps 2-5 read the
//    double-buffered accumulator back with tcgen05.ld and apply SwiGLU (gate
//    and up rows 16 lanes apart) or the NVFP4 tensor scale;
//  - decode cuts the concatenated K stages of all units into equal ranges
//    per CTA (stream-K); the CTA finishing a unit sums its pieces in CTA
//    order, so results are deterministic.  Prefill deals whole units.
// Every wait is bounded (the limit is a kernel argument, about 2 s unless a
// test shortens it); a timeout records MOE_ERR_TIMEOUT, raises the CTA's
// abort flag so the other roles drain, and the kernel returns.
#include <algorithm>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

namespace moe {

__device__ int g_fp4_error;   // first device-side error of this file's kernels (0: none)

namespace {

constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
// Epilogue warps of the separate GEMM kernel: with prefill tiles (64 tokens
// per unit) reading back and finishing a unit takes longer than its MMAs, so
// two warps share each tensor-memory lane quarter, one per half of the
// unit's 8-token chunks.
template <class CFG>
struct SepCfg {
    static constexpr int EW = CFG::SPLIT ? kEpiWarps : 2 * kEpiWarps;
    static constexpr int THREADS = 32 * (2 + EW);
};
constexpr int kQuantThreads = 256;
constexpr long long kWaitCycles = 4000000000ll;   // ~2 s: drains, and waits unless a test sets a limit
constexpr int kMaxCtas = 160;                      // persistent grid: one CTA per SM at most
constexpr int kSmemBudget = 227 * 1024;

// Tile configurations: decode (few tokens per expert, stream-K) and prefill.
template <int NMAX_, int T_, bool SPLIT_>
struct TileCfg {
    static constexpr int NMAX = NMAX_;   // MMA N per tile (terms x tokens), multiple of 8 T
    static constexpr int T = T_;         // E2M1 terms per activation value
    static constexpr int NT = NMAX_ / T_;  // tokens per tile
    static constexpr bool SPLIT = SPLIT_;
    static_assert(NMAX_ % (8 * T_) == 0, "token groups of 8 per epilogue step");
};
using DecodeCfg = TileCfg<64, 4, true>;
using PrefillCfg = TileCfg<192, 3, false>;

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Issued by one elected lane of a converged warp (the copy warps walk their
// loops warp-uniformly; see tc_commit).
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
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
// try_wait that lets the hardware suspend the thread while the phase is
// incomplete, so waiting warps leave issue slots to working ones.
__device__ __forceinline__ bool mbar_try_suspend(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity), "n"(20000)
                 : "memory");
    return ok != 0;
}
// Bounded wait: gives up when another role raised the abort flag, or after
// `limit` cycles, in which case it records MOE_ERR_TIMEOUT and raises the flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, long long limit)
{
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_suspend(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) break;
    }
    *abort_flag = 1;
    atomicCAS(&g_fp4_error, 0, (int)MOE_ERR_TIMEOUT);
    return false;
}

// Drain wait for this CTA's own asynchronous work (copies, MMAs) before it
// exits or frees tensor memory: bounded by time only, not by the abort flag.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_suspend(bar, parity))
        if (clock64() - t0 > kWaitCycles) {
            atomicCAS(&g_fp4_error, 0, (int)MOE_ERR_TIMEOUT);
            return;
        }
}

// One elected lane of a converged warp issues the copy.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// L2 prefetch of a weight chunk the CTA streams a little later (one elected lane).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e cp.async.bulk.prefetch.L2.global [%0], %1;\n\t}" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// The MMA warps issue tcgen05 operations from warp-uniform code: every lane
// computes the operands, one lane elected by elect.sync issues (keeping the
// operands warp-uniform roughly halves the issue cost of a chunk against a
// lane-0-only branch).  Callers are converged warps.
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
                 : "memory");
}

// Shared-memory descriptor of a K-major operand in the 128-byte swizzle:
// 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Descriptor of one scale-factor image: 32 rows of 16 bytes, no swizzle.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// One 512-byte scale image (descriptor d) -> 4 tensor-memory columns of all
// 128 lanes (the 32-lane pattern is replicated into the four lane quarters).
__device__ __forceinline__ void tc_cp_sf_d(uint32_t taddr, uint64_t desc)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr), "l"(desc));
}

// D[tmem] (+)= A[smem] * B[smem], E2M1 operands with block scales from tensor memory.
template <int WFMT>
__device__ __forceinline__ void tc_mma_fp4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                           uint32_t sfa, uint32_t sfb)
{
    if (WFMT == MOE_W_MXFP4)
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    else
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
}

// Instruction descriptor (block-scaled kinds): E2M1 A and B, K-major, M = 128,
// N = n, scale type E8M0 (MXFP4) or E4M3 (NVFP4), scale-factor byte `id`
// inside each tensor-memory word for A and B.
template <int WFMT>
__device__ __forceinline__ uint32_t idesc_fp4(int n, uint32_t id)
{
    const uint32_t sfmt = WFMT == MOE_W_MXFP4 ? 1u : 0u;
    return (id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (sfmt << 23) | (8u << 24) | (id << 29);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* v)
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// E4M3 code -> value (no NaN codes reach here)
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    const uint32_t e = (c >> 3) & 15, m = c & 7;
    const float v = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (c & 0x80) ? -v : v;
}

// ------------------------------------------------------------------ activation terms
// Scale of one term of a block whose largest remaining magnitude is m: the
// smallest scale of the format with m / scale <= 6 (E2M1's largest value).
template <int WFMT>
__device__ __forceinline__ uint32_t term_scale(float m, float& sval)
{
    if (!(m > 0.0f)) {   // zero block (or NaN): any scale, all codes 0
        sval = 1.0f;
        return WFMT == MOE_W_MXFP4 ? 127u : 0x38u;
    }
    if (WFMT == MOE_W_MXFP4) {
        // m = f 2^E with f in [0.5, 1): E = biased exponent - 126, f > 0.75
        // exactly when the mantissa exceeds 2^22; 6 * 2^(code-127) >= m is
        // then minimal for code = E - 2 (f > 0.75) or E - 3, plus 127
        const uint32_t b = __float_as_uint(m);
        int code = (int)(b >> 23) + ((b & 0x7FFFFF) > 0x400000 ? -1 : -2);
        code = code < 1 ? 1 : (code > 254 ? 254 : code);
        sval = __uint_as_float((uint32_t)code << 23);
        return (uint32_t)code;
    }
    const float s = __fdiv_rn(m, 6.0f);
    uint32_t code;
    if (s < 0.015625f) {                               // below 2^-6: subnormal steps of 2^-9
        const float k = ceilf(s * 512.0f);
        code = (uint32_t)k;                            // 1..8 (8 is 2^-6, the first normal code)
    } else {
        const uint32_t b = __float_as_uint(s);
        int e = (int)(b >> 23) - 127;
        uint32_t m3 = (b >> 20) & 7;
        if (b & 0xFFFFF) m3++;                         // round up
        if (m3 == 8) { m3 = 0; e++; }
        code = e > 8 ? 0x7Eu : ((uint32_t)(e + 7) << 3) | m3;
        if (code > 0x7E) code = 0x7E;                  // 448
    }
    sval = e4m3_value(code);
    return code;
}

// Nearest E2M1 codes of 8 values |x| <= 6, ties to the even code (the
// hardware's round-to-nearest-even conversion to E2M1, which is that rule),
// NaN taken as 0 and a zero magnitude with the + sign (code 0); column i in
// bits 4i..4i+3 of the result, the codes' values in q[].
__device__ __forceinline__ uint32_t e2m1x8_round(const float (&x)[8], float (&q)[8])
{
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; i++) y[i] = x[i] == x[i] ? x[i] : 0.0f;
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    const uint32_t m = w & 0x77777777u;
    w = m | (w & ((m + 0x77777777u) & 0x88888888u));   // -0 -> +0: sign kept only on a nonzero magnitude
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t"
        ".reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %8;\n\t"
        "cvt.rn.f16x2.e2m1x2 h0, b0;\n\tcvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h2, b2;\n\tcvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
        "mov.b32 {l0, u0}, h0;\n\tmov.b32 {l1, u1}, h1;\n\tmov.b32 {l2, u2}, h2;\n\tmov.b32 {l3, u3}, h3;\n\t"
        "cvt.f32.f16 %0, l0;\n\tcvt.f32.f16 %1, u0;\n\tcvt.f32.f16 %2, l1;\n\tcvt.f32.f16 %3, u1;\n\t"
        "cvt.f32.f16 %4, l2;\n\tcvt.f32.f16 %5, u2;\n\tcvt.f32.f16 %6, l3;\n\tcvt.f32.f16 %7, u3;\n\t}"
        : "=f"(q[0]), "=f"(q[1]), "=f"(q[2]), "=f"(q[3]), "=f"(q[4]), "=f"(q[5]), "=f"(q[6]), "=f"(q[7])
        : "r"(w));
    return w;
}

// The E4M3-scaled (NVFP4) counterpart without the division: the nearest
// E2M1 code of v / s from |v| against the midpoints between neighbouring
// E2M1 magnitudes times s (mid[], at most 7 significant bits: exact
// products).  > at the midpoints whose lower neighbour has the even code
// (0.25, 1.25, 2.5, 5), >= at the others (0.75, 1.75, 3.5): exact ties go to
// the even code.  The same code as the nearest one to the IEEE quotient:
// rounding is monotone, and for fp32 v other than m s, |v - m s| >= ulp(m s)
// (when m s is not a power of two; else s is one and the quotient is exact)
// with s < 2^(e+1) (s = sigma 2^e) keeps |v/s - m| above half an ulp of m,
// so no quotient rounds onto a midpoint.  NaN -> 0.
__device__ __forceinline__ uint32_t e2m1_round_scaled(float v, const float (&mid)[7], float* q)
{
    const float a = fabsf(v);
    const uint32_t k = (uint32_t)(a > mid[0]) + (uint32_t)(a >= mid[1]) + (uint32_t)(a > mid[2]) +
                       (uint32_t)(a >= mid[3]) + (uint32_t)(a > mid[4]) + (uint32_t)(a >= mid[5]) +
                       (uint32_t)(a > mid[6]);
    const float mag = k < 4 ? 0.5f * (float)k : (k == 7 ? 6.0f : (float)(k - 2));
    *q = copysignf(mag, v);
    return (v < 0.0f && k) ? (k | 8u) : k;
}

__device__ __forceinline__ void e2m1_midpoints(float s, float (&mid)[7])
{
    mid[0] = __fmul_rn(0.25f, s);
    mid[1] = __fmul_rn(0.75f, s);
    mid[2] = __fmul_rn(1.25f, s);
    mid[3] = __fmul_rn(1.75f, s);
    mid[4] = __fmul_rn(2.5f, s);
    mid[5] = __fmul_rn(3.5f, s);
    mid[6] = __fmul_rn(5.0f, s);
}



// Per-chunk bytes of a token group's operand image with n rows (n multiple of 8).
__host__ __device__ __forceinline__ int b_chunk_bytes(int n, int nsub)
{
    return n * 128 + nsub * ((n + 127) / 128) * 512;
}

template <int WFMT>
struct Fmt {
    static constexpr int VS = WFMT == MOE_W_MXFP4 ? 32 : 16;   // columns per block scale
    static constexpr int NSUB = 256 / VS / 4;                    // scale images per 256-column chunk
    static constexpr int CB = 16384 + 512 * NSUB;                // blob bytes per 128 x 256 chunk
};

// The plan of one call: for every expert e with rows and a slot in the pool,
// its token groups (of NT rows) are numbered from gpre[e]; the per-chunk
// bytes of their operand images are summed in boffc (in expert order); and
// group g's entry gtab[g] = {first row, rows, slot, per-chunk byte offset of
// its operand image} lets the GEMM find a unit with one load.
__global__ void __launch_bounds__(256) fp4_plan_kernel(const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ slot_of, int E, int rows,
                                                       int pool_slots, int NT, int T, int nsub,
                                                       int32_t* __restrict__ gpre, int32_t* __restrict__ boffc,
                                                       int4* __restrict__ gtab,
                                                       int32_t* __restrict__ zero, int nzero)
{
    pdl_wait();
    for (int i = threadIdx.x; i < nzero; i += 256) zero[i] = 0;
    __shared__ int s_g[8], s_b[8];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int EPT = (E + 255) / 256;   // <= 16 for E <= 4096
    int gl = 0, bl = 0, gc[16], bc[16];
    const int nfull = ((T * NT + 7) / 8) * 8;
    for (int i = 0; i < 16; i++) {
        const int e = threadIdx.x * EPT + i;
        int g = 0, b = 0;
        if (i < EPT && e < E) {
            const int m = offsets[e + 1] - offsets[e], sl = slot_of[e];
            if (m > 0 && sl >= 0 && sl < pool_slots && offsets[e] >= 0 && offsets[e + 1] <= rows) {
                g = (m + NT - 1) / NT;
                const int last = m - (g - 1) * NT;
                b = (g - 1) * b_chunk_bytes(nfull, nsub) + b_chunk_bytes(((T * last + 7) / 8) * 8, nsub);
            }
        }
        gc[i] = g;
        bc[i] = b;
        gl += g;
        bl += b;
    }
    int gi = gl, bi = bl;
    for (int off = 1; off < 32; off <<= 1) {
        const int go = __shfl_up_sync(0xffffffffu, gi, off), bo = __shfl_up_sync(0xffffffffu, bi, off);
        if (lane >= off) { gi += go; bi += bo; }
    }
    if (lane == 31) { s_g[wid] = gi; s_b[wid] = bi; }
    __syncthreads();
    int gr = gi - gl, br = bi - bl;
    for (int w = 0; w < wid; w++) { gr += s_g[w]; br += s_b[w]; }
    const int bfull = b_chunk_bytes(nfull, nsub);
    for (int i = 0; i < 16; i++) {
        const int e = threadIdx.x * EPT + i;
        if (i < EPT && e < E) {
            gpre[e] = gr;
            boffc[e] = br;
            const int m = offsets[e + 1] - offsets[e], sl = slot_of[e];
            for (int g = 0; g < gc[i]; g++)
                gtab[gr + g] = make_int4(offsets[e] + g * NT, min(NT, m - g * NT), sl, br + g * bfull);
        }
        gr += gc[i];
        br += bc[i];
    }
    if (threadIdx.x == 255) { gpre[E] = gr; boffc[E] = br; }
}

// T E2M1 terms of 8 consecutive columns (a lane's share of a scale block of
// 8 LPB columns; the LPB lanes of a block are adjacent and all active): for
// each term the block's largest remaining magnitude (shuffles across the
// block's lanes), its scale code, the 8 codes as one 32-bit word (column i in
// bits 4i..4i+3) and the residual left for the next term.
template <int WFMT, int LPB>
__device__ __noinline__ uint32_t term8(float* v, uint32_t* scode);

template <int WFMT, int T, int LPB>
__device__ __forceinline__ void terms8(float (&v)[8], uint32_t (&word)[T], uint32_t (&scode)[T])
{
#pragma unroll
    for (int t = 0; t < T; t++) {
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
        for (int off = 1; off < LPB; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float sval;
        scode[t] = term_scale<WFMT>(mx, sval);
        // MXFP4 scales are powers of two: multiplying by the exact reciprocal is the division
        const float inv = WFMT == MOE_W_MXFP4 ? __uint_as_float((254u - scode[t]) << 23) : 0.0f;
        uint32_t w = 0;
        if (WFMT == MOE_W_MXFP4) {
            float x[8], q[8];
#pragma unroll
            for (int i = 0; i < 8; i++) x[i] = __fmul_rn(v[i], inv);
            w = e2m1x8_round(x, q);
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = __fsub_rn(v[i], __fmul_rn(q[i], sval));
        } else {
            float mid[7];
            e2m1_midpoints(sval, mid);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                float q;
                w |= e2m1_round_scaled(v[i], mid, &q) << (4 * i);
                v[i] = __fsub_rn(v[i], __fmul_rn(q, sval));
            }
        }
        word[t] = w;
    }
}

// One term of terms8 as a called function (one copy of the code for all
// callers; the fused decode kernel runs it only a few times per launch, so
// code size, not issue rate, decides its cost: measured, two items'
// terms inlined and interleaved ran no faster at batch 16 and 6 us slower
// per call at batch 1).
template <int WFMT, int LPB>
__device__ __noinline__ uint32_t term8(float* v, uint32_t* scode)
{
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
    for (int off = 1; off < LPB; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sval;
    *scode = term_scale<WFMT>(mx, sval);
    const float inv = WFMT == MOE_W_MXFP4 ? __uint_as_float((254u - *scode) << 23) : 0.0f;
    uint32_t w = 0;
    if (WFMT == MOE_W_MXFP4) {
        float x[8], q[8];
#pragma unroll
        for (int i = 0; i < 8; i++) x[i] = __fmul_rn(v[i], inv);
        w = e2m1x8_round(x, q);
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = __fsub_rn(v[i], __fmul_rn(q[i], sval));
    } else {
        float mid[7];
        e2m1_midpoints(sval, mid);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float q;
            w |= e2m1_round_scaled(v[i], mid, &q) << (4 * i);
            v[i] = __fsub_rn(v[i], __fmul_rn(q, sval));
        }
    }
    return w;
}

// 8 activation values of a row (bf16 bits or fp32) as floats.  fp32 rows
// may have been written earlier in the same kernel (h in the fused decode
// kernel), so they are read through L2, not the read-only cache.
template <bool IN_F32>
__device__ __forceinline__ void load8(const void* row, int k, float (&v)[8])
{
    if (IN_F32) {
        const float* f = static_cast<const float*>(row) + k;
        const float4 a = __ldcg(reinterpret_cast<const float4*>(f));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(f) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(row) + k));
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; h++) {
            v[2 * h] = bf16_bits_to_f32(u[h] & 0xFFFF);
            v[2 * h + 1] = bf16_bits_to_f32(u[h] >> 16);
        }
    }
}

// Power-of-two exponent p of an NVFP4 activation row: 2^p times its largest
// magnitude lands in [2^10, 2^11) (p = 0 for a zero or non-finite maximum).
__device__ __forceinline__ int row_exponent(float mx)
{
    int p = 0;
    if (mx > 0.0f && mx <= 3.4e38f) {
        int e2;
        frexpf(mx, &e2);          // mx = f 2^e2, f in [0.5, 1)
        p = 11 - e2;
        p = p < -100 ? -100 : (p > 100 ? 100 : p);
    }
    return p;
}

// Where a term row of a token group's operand image chunk keeps the codes of
// columns [kin, kin+8) (kin = column inside the 256-column chunk) and the
// scale of their block: byte offsets inside the chunk image of n rows.
__device__ __forceinline__ int img_code_off(int row, int kin)
{
    return 1024 * (row >> 3) + 128 * (row & 7) + 16 * ((kin / 32) ^ (row & 7)) + (kin % 32) / 2;
}
template <int VS>
__device__ __forceinline__ int img_scale_off(int n, int row, int kin)
{
    const int blk = kin / VS, nh = (n + 127) / 128;
    return n * 128 + 512 * (nh * (blk / 4) + (row >> 7)) + 16 * (row & 31) + 4 * ((row & 127) >> 5) + (blk % 4);
}

// Activation rows (x gathered by token, or h) -> their T E2M1 terms and block
// scales in the token group's operand image, and (NVFP4) the power-of-two
// exponent p the row was scaled by, 2^p times its largest magnitude lying in
// [2^10, 2^11) so every term scale stays inside the E4M3 range.  Rows of
// experts without a slot are skipped.  A CTA covers kSegCols columns of one
// row (blockIdx.x = row * segments + segment); each thread owns 8 consecutive
// columns, so a 32-column block is 4 lanes (16 columns: 2 lanes) that share
// their block maximum through shuffles, and a thread's 8 codes are one
// 32-bit word of the image row.
// CANON: no groups; row r's codes go to ccodes [rows][T][K] (one per byte),
// its scale codes to cscales [rows][T][K / vs] and p to rex[r].
constexpr int kSegCols = 8 * kQuantThreads;

template <int WFMT, int T, bool IN_F32, bool CANON = false>
__global__ void __launch_bounds__(kQuantThreads) fp4_terms_kernel(
    const void* __restrict__ in, int rows, int K, const int32_t* __restrict__ gather, int gk,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ slot_of, int E, int pool_slots,
    const int32_t* __restrict__ boffc, int NT, char* __restrict__ bimg, int32_t* __restrict__ rex,
    uint8_t* __restrict__ ccodes = nullptr, uint8_t* __restrict__ cscales = nullptr)
{
    using FM = Fmt<WFMT>;
    constexpr int VS = FM::VS, NSUB = FM::NSUB, LPB = VS / 8;   // lanes per scale block
    pdl_wait();
    pdl_trigger();
    __shared__ float s_max[kQuantThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, KC = K / 256;
    const int nseg = (K + kSegCols - 1) / kSegCols;
    const int nfull = ((T * NT + 7) / 8) * 8;
    for (int item = blockIdx.x; item < rows * nseg; item += gridDim.x) {
        const int r = item / nseg, seg = item % nseg;
        int j = 0, N = 0, BB = 0;
        char* base = nullptr;
        if (!CANON) {
            int lo = 0, hi = E - 1;   // expert of row r: the largest e with offsets[e] <= r
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (__ldg(offsets + mid) <= r) lo = mid;
                else hi = mid - 1;
            }
            const int e = lo, sl = __ldg(slot_of + e), m = __ldg(offsets + e + 1) - __ldg(offsets + e);
            if (!(m > 0 && sl >= 0 && sl < pool_slots && __ldg(offsets + e) >= 0 && __ldg(offsets + e + 1) <= rows))
                continue;
            const int loc = r - __ldg(offsets + e), gi = loc / NT, nt = min(NT, m - gi * NT);
            j = loc % NT;
            N = ((T * nt + 7) / 8) * 8;
            BB = b_chunk_bytes(N, NSUB);
            base = bimg + (size_t)KC * ((size_t)__ldg(boffc + e) + (size_t)gi * b_chunk_bytes(nfull, NSUB));
        }
        const size_t sr = gather ? (size_t)(__ldg(gather + r) / gk) : (size_t)r;
        const void* row = IN_F32 ? static_cast<const void*>(static_cast<const float*>(in) + sr * K)
                                 : static_cast<const void*>(static_cast<const uint16_t*>(in) + sr * K);
        int p = 0;
        if (WFMT == MOE_W_NVFP4) {   // row maximum (every segment's CTA reads the whole row)
            float mx = 0.0f;
            for (int k = tid * 8; k < K; k += kQuantThreads * 8) {
                float v[8];
                load8<IN_F32>(row, k, v);
#pragma unroll
                for (int i = 0; i < 8; i++) mx = fmaxf(mx, fabsf(v[i]));
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) s_max[tid >> 5] = mx;
            __syncthreads();
            mx = s_max[0];
#pragma unroll
            for (int w = 1; w < kQuantThreads / 32; w++) mx = fmaxf(mx, s_max[w]);
            __syncthreads();   // s_max is reused by the next item
            p = row_exponent(mx);
        }
        if (seg == 0 && tid == 0 && (WFMT == MOE_W_NVFP4 || CANON)) rex[r] = p;
        const float sc = ldexpf(1.0f, p);
        const int k0 = seg * kSegCols + tid * 8;
        if (k0 >= K) continue;          // whole scale blocks: every lane of a block is active together
        float v[8];
        load8<IN_F32>(row, k0, v);
        if (WFMT == MOE_W_NVFP4)
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = __fmul_rn(v[i], sc);
        uint32_t word[T], scode[T];
        terms8<WFMT, T, LPB>(v, word, scode);
        const int c = k0 / 256, kin = k0 % 256;   // chunk, column inside it
#pragma unroll
        for (int t = 0; t < T; t++) {
            if (CANON) {
                uint8_t* cr = ccodes + ((size_t)r * T + t) * K + k0;
                const uint32_t w = word[t];
                uint2 o;
                o.x = (w & 0xF) | ((w >> 4 & 0xF) << 8) | ((w >> 8 & 0xF) << 16) | ((w >> 12 & 0xF) << 24);
                o.y = (w >> 16 & 0xF) | ((w >> 20 & 0xF) << 8) | ((w >> 24 & 0xF) << 16) | ((w >> 28) << 24);
                *reinterpret_cast<uint2*>(cr) = o;
                if ((tid % LPB) == 0) cscales[((size_t)r * T + t) * (K / VS) + k0 / VS] = (uint8_t)scode[t];
                continue;
            }
            char* cb = base + (size_t)c * BB;
            const int n = j * T + t;
            *reinterpret_cast<uint32_t*>(cb + img_code_off(n, kin)) = word[t];
            if ((tid % LPB) == 0) cb[img_scale_off<VS>(N, n, kin)] = (char)scode[t];
        }
    }
}

// ------------------------------------------------------------------ grouped GEMM
struct Fp4Args {
    const char* pool;
    size_t slot_bytes;
    size_t w_off;       // matrix offset inside a blob
    size_t ts_off;      // NVFP4 tensor scales
    int R, K, E, rows, pool_slots;
    const int32_t* slot_of;
    const int32_t* offsets;
    const int32_t* gpre;
    const int4* gtab;       // per token group: first row, rows, slot, per-chunk image offset
    const char* bimg;       // operand images of this phase's activations
    const int32_t* rex;     // per-row exponents of the activations (NVFP4), else null
    float* out_h;           // phase 1: h [rows][R/2] fp32
    uint16_t* out_y;        // phase 2: y [rows][R] bf16
    int32_t* cnt;           // per unit: pieces finished (stream-K)
    float* pieces;          // [gridDim.x][2][128 * NMAX] partial accumulators (stream-K)
    long long wait;         // limit of every bounded wait, in SM clock cycles
    int withhold;           // testing: CTA 0 leaves its first ring stage unfilled
};

template <int WFMT, class CFG>
struct KCfg {
    using FM = Fmt<WFMT>;
    static constexpr int NH = (CFG::NMAX + 127) / 128;
    static constexpr int A_BYTES = FM::CB;                                // 1024-multiple
    static constexpr int B_BYTES = CFG::NMAX * 128 + FM::NSUB * NH * 512;  // 1024-multiple
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int D = (kSmemBudget - 2048) / STAGE > 8 ? 8 : (kSmemBudget - 2048) / STAGE;
    static constexpr int SMEM = 1024 + 1024 + D * STAGE;   // barriers, alignment slack, ring
    // tensor memory: two accumulators, then two scale-factor sets
    static constexpr int SF_A = 4 * FM::NSUB, SF_B = 4 * FM::NSUB * NH;
    static constexpr int SF_COL = 2 * CFG::NMAX;
    static constexpr int SF_SET = SF_A + SF_B;
    static constexpr int COLS_USED = SF_COL + 2 * SF_SET;
    static constexpr uint32_t TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                          : COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "tensor memory");
    static_assert(STAGE % 1024 == 0, "1024-byte aligned stages");
};

// The scale-factor copies and four MMAs of one 256-column chunk whose ring
// stage starts at shared address sa (weight image, its scale images, then
// the token group's image with n rows and its scale images).  Descriptors of
// the later K steps and operands are offsets of the first one: the address
// field counts 16-byte units and the ring lies below 256 KB, so no carry.
template <int WFMT, int A_BYTES>
__device__ __forceinline__ void issue_chunk(uint32_t sa, int n, int nh, uint32_t dcol, uint32_t sfa, uint32_t sfb,
                                            uint32_t id0, uint32_t id1, bool first)
{
    using FM = Fmt<WFMT>;
    const uint64_t da = desc_sw128(sa), db = da + (A_BYTES >> 4);
    const uint64_t dsa = desc_sf(sa + 16384), dsb = dsa + (uint64_t)((A_BYTES - 16384 + n * 128) >> 4);
#pragma unroll
    for (int s = 0; s < FM::NSUB; s++) tc_cp_sf_d(sfa + 4 * s, dsa + (uint64_t)(32 * s));
    for (int s = 0; s < FM::NSUB * nh; s++) tc_cp_sf_d(sfb + 4 * s, dsb + (uint64_t)(32 * s));
#pragma unroll
    for (int k = 0; k < 4; k++) {
        // MXFP4: two 32-column scales per MMA, bytes 0-1 or 2-3 of a word;
        // NVFP4: four 16-column scales per MMA, one image each
        const int s = WFMT == MOE_W_MXFP4 ? (k >> 1) : k;
        tc_mma_fp4<WFMT>(dcol, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k),
                         (WFMT == MOE_W_MXFP4 && (k & 1)) ? id1 : id0, (!first || k > 0) ? 1u : 0u, sfa + 4 * s,
                         sfb + 4 * nh * s);
    }
}

// A unit: (token group of one expert, 128-row block of the weight matrix).
struct Unit {
    int G, row0, nt, n;      // n: MMA N (terms x tokens, multiple of 8)
    const char* blob;        // the expert's slot
    const char* a;           // chunk 0 of the weight block
    const char* b;           // chunk 0 of the token group's operand image
    int bb;                  // bytes per chunk of that image
};

template <int WFMT, class CFG>
__device__ __forceinline__ Unit unit_of(const Fp4Args& a, int u, int RB, int KC, int4 g)
{
    using FM = Fmt<WFMT>;
    Unit U;
    U.G = u % RB;
    U.row0 = g.x;
    U.nt = g.y;
    U.n = ((CFG::T * U.nt + 7) / 8) * 8;
    U.bb = b_chunk_bytes(U.n, FM::NSUB);
    U.blob = a.pool + (size_t)g.z * a.slot_bytes;
    U.a = U.blob + a.w_off + (size_t)U.G * KC * FM::CB;
    U.b = a.bimg + (size_t)KC * (size_t)g.w;
    return U;
}

__device__ __forceinline__ int4 group_of(const Fp4Args& a, int u, int RB) { return __ldg(a.gtab + u / RB); }

// Segments of one CTA: whole units u = blockIdx.x + i * gridDim.x, or the
// stream-K pieces of its stage range [pos, end): unit u, chunks [p0, p1).
struct Seg {
    long pos, start;
    int u, p0, p1;
    __device__ __forceinline__ bool next(bool whole, int NU, int KC, long end)
    {
        if (whole) {
            if (pos >= NU) return false;
            u = (int)pos;
            p0 = 0;
            p1 = KC;
            pos += gridDim.x;
            return true;
        }
        if (pos >= end) return false;
        start = pos;
        u = (int)(pos / KC);
        p0 = (int)(pos % KC);
        p1 = (int)min((long)KC, p0 + (end - pos));
        pos += p1 - p0;
        return true;
    }
};

__device__ __forceinline__ long sk_bound(long W, int c, int grid) { return W * c / grid; }
__device__ __forceinline__ int sk_cta_of(long W, long idx, int grid)
{
    int c = (int)(idx * grid / W);
    while (c + 1 < grid && sk_bound(W, c + 1, grid) <= idx) c++;
    while (c > 0 && sk_bound(W, c, grid) > idx) c--;
    return c;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory"); }

// Final values of 8 tokens of a unit from their 8 T accumulator columns d:
// sum of the terms, the row exponents undone, then SwiGLU into h (phase 1,
// lanes 0-15 gate rows, 16-31 the matching up rows) or y in bf16.
template <int WFMT, int PHASE, int T>
__device__ __forceinline__ void finish8(const Fp4Args& a, const Unit& U, int q, int lane, int ch, const float* d,
                                        float tsc)
{
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const int tok = 8 * ch + j;
        float v = 0.0f;
#pragma unroll
        for (int t = 0; t < T; t++) v += d[j * T + t];
        const bool live = tok < U.nt;
        const int row = U.row0 + tok;
        float u = tsc;
        if (WFMT == MOE_W_NVFP4 && live) u = tsc * pow2i(-__ldcg(a.rex + row));   // written in this grid (fused)
        v *= u;
        if (PHASE == 1) {
            const float up = __shfl_down_sync(0xffffffffu, v, 16);
            if (live && lane < 16) {
                const int F = a.R / 2;
                a.out_h[(size_t)row * F + 64 * U.G + 16 * q + lane] = silu(v) * up;
            }
        } else if (live) {
            a.out_y[(size_t)row * a.R + 128 * U.G + 32 * q + lane] = f32_to_bf16_bits(v);
        }
    }
}

template <int WFMT, int PHASE, class CFG>
__global__ void __launch_bounds__(SepCfg<CFG>::THREADS, 1) ffn_fp4_kernel(Fp4Args a)
{
    using FM = Fmt<WFMT>;
    using KC_ = KCfg<WFMT, CFG>;
    constexpr int D = KC_::D, STAGE = KC_::STAGE, T = CFG::T;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // [D]
    uint64_t* empty = full + D;                           // [D]
    uint64_t* acc_full = empty + D;                       // [2]
    uint64_t* acc_empty = acc_full + 2;                   // [2]
    uint64_t* fin = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    int* s_last = abort_flag + 1;
    unsigned char* ring = smem + 1024;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int RB = a.R / 128, KC = a.K / 256;

    if (tid == 0) {
        for (int i = 0; i < D; i++) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 32 * SepCfg<CFG>::EW);
        }
        mbar_init(smem_u32(fin), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(KC_::TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int* abort_v = abort_flag;
    // The plan (token groups, their table) was written by a kernel that had
    // completed before this grid's predecessor started, so it may be read
    // before griddepcontrol.wait; the activation images, row exponents and
    // the outputs belong to the predecessor and are touched only after it.
    pdl_trigger();

    // work: whole units round-robin (prefill), or the units' K chunks cut into
    // equal ranges over the CTAs (decode)
    const int NU = __ldg(a.gpre + a.E) * RB;
    const bool whole = !CFG::SPLIT;
    const long W = whole ? 0 : (long)NU * KC;
    const int grid = whole ? (int)gridDim.x : (int)(W < (long)gridDim.x ? W : (long)gridDim.x);
    const bool in_use = whole || (int)blockIdx.x < grid;
    const long b0 = (!whole && in_use) ? sk_bound(W, blockIdx.x, grid) : 0;
    const long b1 = (!whole && in_use) ? sk_bound(W, blockIdx.x + 1, grid) : 0;
    const long first = whole ? (long)blockIdx.x : b0;

    if (warp == 0) {
        // ============ bulk copies: weight chunk image + token group image chunk
        // (the whole warp walks the loop, one elected lane issues).  The first
        // D stages' weight copies are issued before waiting for the
        // predecessor grid (weights do not depend on it); their activation
        // copies follow once it has completed.
        if (in_use) {
            int st = 0;
            uint32_t ph = 0;
            long issued = 0;
            bool ok = true, waited = false;
            int withheld = -1;   // testing: the stage left unfilled
            const char* pend_src[D];
            uint32_t pend_bytes[D];
            int npend = 0;
            auto release_pending = [&]() {
                pdl_wait();
                waited = true;
                for (int i = 0; i < npend; i++) {
                    if (pend_bytes[i])
                        bulk_g2s(smem_u32(ring + (size_t)i * STAGE + KC_::A_BYTES), pend_src[i], pend_bytes[i],
                                 smem_u32(&full[i]));
                }
                npend = 0;
            };
            Seg sg{first};
            bool have = sg.next(whole, NU, KC, b1);
            int4 g = have ? group_of(a, sg.u, RB) : make_int4(0, 0, 0, 0);
            while (ok && have) {
                const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, g);
                Seg nx = sg;   // look one unit ahead: its table entry loads during this unit's copies
                const bool have_nx = nx.next(whole, NU, KC, b1);
                const int4 gn = have_nx ? group_of(a, nx.u, RB) : g;
                for (int c = sg.p0; c < sg.p1; c++) {
                    if (!(ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&empty[st]), ph ^ 1, abort_v, a.wait))))
                        break;
                    const uint32_t bar = smem_u32(&full[st]);
                    unsigned char* sp = ring + (size_t)st * STAGE;
                    if (a.withhold && blockIdx.x == 0 && issued == 0) {
                        // testing: never filled, so the wait for it runs out
                        withheld = st;
                        pend_src[npend] = nullptr;
                        pend_bytes[npend++] = 0;
                    } else {
                        mbar_expect_tx(bar, (uint32_t)(FM::CB + U.bb));
                        bulk_g2s(smem_u32(sp), U.a + (size_t)c * FM::CB, FM::CB, bar);
                        if (waited) {
                            bulk_g2s(smem_u32(sp + KC_::A_BYTES), U.b + (size_t)c * U.bb, (uint32_t)U.bb, bar);
                        } else {   // first pass over the ring: stage st == issued
                            pend_src[npend] = U.b + (size_t)c * U.bb;
                            pend_bytes[npend++] = (uint32_t)U.bb;
                        }
                    }
                    issued++;
                    if (++st == D) { st = 0; ph ^= 1; }
                    if (!waited && issued == D) release_pending();
                }
                sg = nx;
                have = have_nx;
                g = gn;
            }
            if (!waited) release_pending();
            // every issued copy lands before the CTA exits (stage i was last
            // filled in this pass if i < st, else in the previous one; a
            // withheld stage is never refilled: its consumer gives up first)
            for (int i = 0; i < D && i < issued; i++)
                if (i != withheld) mbar_drain(smem_u32(&full[i]), i < st ? ph : (ph ^ 1));
        } else {
            pdl_wait();
        }
    } else if (warp == 1) {
        // ============ scale-factor copies and MMAs (the whole warp walks the
        // loop, one elected lane issues)
        const uint32_t ring_s = smem_u32(ring);
        if (in_use) {
            int st = 0, it = 0;
            uint32_t ph = 0;
            long cc = 0;
            bool ok = true;
            Seg sg{first};
            bool have = sg.next(whole, NU, KC, b1);
            int4 g = have ? group_of(a, sg.u, RB) : make_int4(0, 0, 0, 0);
            while (ok && have) {
                const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, g);
                Seg nx = sg;
                const bool have_nx = nx.next(whole, NU, KC, b1);
                const int4 gn = have_nx ? group_of(a, nx.u, RB) : g;
                const int ab = it & 1, nh = (U.n + 127) / 128;
                const uint32_t id0 = idesc_fp4<WFMT>(U.n, 0), id1 = idesc_fp4<WFMT>(U.n, 2);
                if (it >= 2) {   // the epilogue has read this accumulator's previous unit
                    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_empty[ab]), ((it >> 1) - 1) & 1, abort_v, a.wait));
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t dcol = tmem + (uint32_t)(ab * CFG::NMAX);
                for (int c = sg.p0; c < sg.p1; c++, cc++) {
                    if (!(ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), ph, abort_v, a.wait)))) break;
                    tc_fence_after();
                    const uint32_t sfa = tmem + KC_::SF_COL + (uint32_t)((cc & 1) * KC_::SF_SET);
                    issue_chunk<WFMT, KC_::A_BYTES>(ring_s + (uint32_t)(st * STAGE), U.n, nh, dcol, sfa,
                                                    sfa + KC_::SF_A, id0, id1, c == sg.p0);
                    tc_commit(smem_u32(&empty[st]));   // the stage is free once these MMAs have read it
                    if (++st == D) { st = 0; ph ^= 1; }
                }
                if (!ok) break;
                tc_commit(smem_u32(&acc_full[ab]));
                it++;
                sg = nx;
                have = have_nx;
                g = gn;
            }
            // every MMA issued here completes before tensor memory is released
            tc_commit(smem_u32(fin));
            mbar_drain(smem_u32(fin), 0);
        }
    } else if (in_use) {
        // ============ epilogue: warps 2.., tensor-memory lane quarter q = warp % 4;
        // with 8 epilogue warps, warp w takes the unit's chunks ch = (w - 2) / 4 mod 2.
        // All four warps walk the same segments and meet the same named
        // barriers; after a failed wait a warp keeps walking without waiting
        // or touching tensor memory, so the barriers still match.
        const int q = warp & 3;
        const int etid = tid - 64;   // 0..127
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        pdl_wait();
        int it = 0;
        bool ok = true;
        Seg sg{first};
        while (sg.next(whole, NU, KC, b1)) {
            const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, group_of(a, sg.u, RB));
            const int ab = it & 1;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[ab]), (it >> 1) & 1, abort_v, a.wait));
            if (ok) tc_fence_after();
            float tsc = 1.0f;
            if (WFMT == MOE_W_NVFP4) tsc = __ldg(reinterpret_cast<const float*>(U.blob + a.ts_off) + PHASE - 1);
            const uint32_t dcol = tmem + lane_base + (uint32_t)(ab * CFG::NMAX);
            const int nch = (U.nt + 7) / 8;
            if (whole || (sg.p0 == 0 && sg.p1 == KC)) {
                if (ok) {
                    constexpr int EH = SepCfg<CFG>::EW / 4;
                    for (int ch = (warp - 2) / 4; ch < nch; ch += EH) {
                        uint32_t d[8 * T];
#pragma unroll
                        for (int t = 0; t < T; t++) tmem_ld8(dcol + 8 * T * ch + 8 * t, d + 8 * t);
                        tmem_wait_ld();
                        finish8<WFMT, PHASE, T>(a, U, q, lane, ch, reinterpret_cast<const float*>(d), tsc);
                    }
                    tc_fence_before();
                    mbar_arrive(smem_u32(&acc_empty[ab]));
                }
            } else {
                // a piece: publish the partial sums, count the piece; the CTA
                // completing the unit adds all pieces in CTA order
                const int slot = sg.start == b0 ? 0 : 1;
                float* mine = a.pieces + ((size_t)blockIdx.x * 2 + slot) * (128 * CFG::NMAX);
                if (ok) {
                    for (int ch = 0; ch < nch; ch++) {
                        uint32_t d[8 * T];
#pragma unroll
                        for (int t = 0; t < T; t++) tmem_ld8(dcol + 8 * T * ch + 8 * t, d + 8 * t);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8 * T; i++)
                            mine[(size_t)(8 * T * ch + i) * 128 + etid] = __uint_as_float(d[i]);
                    }
                    tc_fence_before();
                    mbar_arrive(smem_u32(&acc_empty[ab]));
                }
                __threadfence();
                epi_bar();
                const long u_lo = (long)sg.u * KC, u_hi = u_lo + KC - 1;
                const int c_lo = sk_cta_of(W, u_lo, grid), c_hi = sk_cta_of(W, u_hi, grid);
                // a warp that failed its wait has raised the abort flag before this barrier
                if (etid == 0) *s_last = (ok && !*abort_v && atomicAdd(a.cnt + sg.u, 1) == c_hi - c_lo) ? 1 : 0;
                epi_bar();
                if (*s_last) {
                    __threadfence();
                    for (int ch = 0; ch < nch; ch++) {
                        float d[8 * T];
#pragma unroll
                        for (int i = 0; i < 8 * T; i++) d[i] = 0.0f;
                        for (int c = c_lo; c <= c_hi; c++) {
                            const int sl = sk_bound(W, c, grid) >= u_lo ? 0 : 1;
                            const float* pc = a.pieces + ((size_t)c * 2 + sl) * (128 * CFG::NMAX);
#pragma unroll
                            for (int i = 0; i < 8 * T; i++)
                                d[i] += __ldcg(pc + (size_t)(8 * T * ch + i) * 128 + etid);
                        }
                        finish8<WFMT, PHASE, T>(a, U, q, lane, ch, d, tsc);
                    }
                    if (etid == 0) a.cnt[sg.u] = 0;
                }
                epi_bar();   // s_last is rewritten by the next piece
            }
            it++;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(KC_::TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------ fused decode FFN
// Decode calls are too small to pay one kernel boundary per step (each costs
// several microseconds on the GPU timeline), so with decode tiles the whole
// FFN call is one cooperative persistent kernel, one CTA per SM:
//   plan (every CTA computes the token groups of the call for itself, in
//   shared memory) -> x terms -> grid barrier -> gate-up GEMM -> barrier ->
//   h terms -> barrier -> down GEMM.
// The quantisation steps run on the four epilogue warps; the copy warp keeps
// streaming weights across the barriers and holds back only the activation
// copies until the barrier that publishes them has passed.
// Grid barriers count arrivals on one 64-bit counter that only grows: a
// launch whose CTAs all finish adds (barriers x CTAs) to it.  Each CTA rounds
// the counter down to a multiple of the grid when it starts (the first
// barrier cannot complete before every CTA has arrived, so every CTA finds
// the same value) and barrier k completes when the counter reaches that value
// plus (k + 1) x grid.  Arrival is one release add, waiting is acquire loads;
// every wait is bounded.  Clearing the error word resets the counter.
// Grid-barrier arrivals since the last clear, one counter per grid size: a
// launch finds its base by rounding its counter down to a multiple of its
// grid, which holds only if every earlier launch on that counter had the
// same grid (a one-expert pass runs on fewer CTAs than a full one).
__device__ unsigned long long g_gb_count[kMaxCtas + 1];
__device__ int g_gb_abort;                  // set when a CTA gave up; cleared with the error word

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

constexpr int kFusedMaxE = 512;
constexpr int kPfUnit = 8;     // weight chunks of the current unit prefetched into L2 ahead of its copies

struct FusedArgs {
    Fp4Args p1, p2;                 // the two GEMM phases (gpre / gtab unused)
    const void* x;                  // input rows: token gather[r] / gk of x (row r when gather is null)
    int x_f32;
    const int32_t* gather;
    int gk;
    char* bx;                       // operand images of x and of h
    char* bh;
    int32_t* rex_x;
    int32_t* rex_h;
    int32_t* cnt2;                  // phase-2 piece counters (phase 1 uses p1.cnt)
    int ncnt;
};

template <int WFMT>
struct FusedCfg {
    using K = KCfg<WFMT, DecodeCfg>;
    static constexpr int STAGE = K::STAGE;
    // offsets, group prefix, image offsets, slots; padded so the ring stays
    // 1024-byte aligned (the 128-byte swizzle of the operand images needs it)
    static constexpr int PLAN = (4 * 4 * (kFusedMaxE + 1) + 1023) / 1024 * 1024;
    static constexpr int D = (kSmemBudget - 2048 - PLAN) / STAGE > 8 ? 8 : (kSmemBudget - 2048 - PLAN) / STAGE;
    static constexpr int SMEM = 1024 + 1024 + PLAN + D * STAGE;
    static_assert(PLAN % 1024 == 0 && STAGE % 1024 == 0, "1024-byte aligned ring");
};

// The arrival count this CTA's first grid barrier completes at (epilogue
// thread 0, before its first arrival).
__device__ __forceinline__ unsigned long long grid_bar_first()
{
    const unsigned long long c = ld_acquire_u64(&g_gb_count[gridDim.x]);
    return c - c % gridDim.x + gridDim.x;
}

// Bounded grid barrier for the four epilogue warps of every CTA.  Their
// global writes before it are visible to every CTA after it (generic and
// async proxy: operand images are read by bulk copies).  `next` (meaningful
// in epilogue thread 0) is the count this barrier completes at; it moves on
// to the next barrier's.
__device__ __forceinline__ bool grid_sync_epi(int etid, volatile int* s_flag, long long limit,
                                              unsigned long long& next)
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    epi_bar();
    if (etid == 0) {
        bool ok = !*reinterpret_cast<volatile int*>(&g_gb_abort);
        red_release_add_u64(&g_gb_count[gridDim.x], 1ull);
        const long long t0 = clock64();
        while (ld_acquire_u64(&g_gb_count[gridDim.x]) < next) {
            if (*reinterpret_cast<volatile int*>(&g_gb_abort)) { ok = false; break; }
            if (clock64() - t0 > limit) {
                ok = false;
                atomicExch(&g_gb_abort, 1);
                atomicCAS(&g_fp4_error, 0, (int)MOE_ERR_TIMEOUT);
                break;
            }
        }
        *s_flag = ok ? 1 : 0;
    }
    next += gridDim.x;
    epi_bar();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return *s_flag != 0;
}

// The call's plan in shared memory, computed by every CTA.
struct Plan {
    int* off;    // [E+1] row offsets
    int* gpre;   // [E+1] first token group of each expert (experts with rows and a slot have groups)
    int* boff;   // [E+1] per-chunk image byte offset of its first group
    int* slot;   // [E]   slot, -1 when the expert is skipped
    int E;
};

__device__ __forceinline__ int4 plan_group(const Plan& P, int gi, int NT, int bfull)
{
    int lo = 0, hi = P.E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.gpre[mid] <= gi) lo = mid;
        else hi = mid - 1;
    }
    const int i = gi - P.gpre[lo], m = P.off[lo + 1] - P.off[lo];
    return make_int4(P.off[lo] + i * NT, min(NT, m - i * NT), P.slot[lo], P.boff[lo] + i * bfull);
}

// One quantisation item of one epilogue warp: row r, 256-column chunk c of
// its K, into the operand image of its token group (32 lanes x 8 columns).
// qitem_load finds the item's place and loads its 8 values per lane (a warp
// loads two items before computing, so their global-memory latencies
// overlap); fused_quant_items computes the terms and writes them.
struct QItem {
    char* cb;          // the item's chunk of its group's operand image (null: skipped row)
    const void* row;   // the source row
    int r, c, n0, N;   // row, chunk, first term row (j T), image rows
    float v[8];
};

template <int WFMT, int T, bool IN_F32>
__device__ __forceinline__ void qitem_load(QItem& it, const Plan& P, const void* in, int K, const int32_t* gather,
                                           int gk, int r, int c, char* bimg, int lane)
{
    using FM = Fmt<WFMT>;
    constexpr int NT = DecodeCfg::NT;
    it.cb = nullptr;
    it.r = r;
    it.c = c;
    int lo = 0, hi = P.E - 1;   // expert of row r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.off[mid] <= r) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo;
    if (P.slot[e] < 0) return;   // the same for the whole warp
    const int m = P.off[e + 1] - P.off[e], loc = r - P.off[e], gi = loc / NT, j = loc % NT;
    const int nt = min(NT, m - gi * NT);
    it.N = ((T * nt + 7) / 8) * 8;
    it.n0 = j * T;
    const int KC = K / 256;
    it.cb = bimg + (size_t)KC * ((size_t)P.boff[e] + (size_t)gi * b_chunk_bytes(DecodeCfg::NMAX, FM::NSUB)) +
            (size_t)c * b_chunk_bytes(it.N, FM::NSUB);
    const size_t sr = gather ? (size_t)(__ldg(gather + r) / gk) : (size_t)r;
    it.row = IN_F32 ? static_cast<const void*>(static_cast<const float*>(in) + sr * K)
                    : static_cast<const void*>(static_cast<const uint16_t*>(in) + sr * K);
    load8<IN_F32>(it.row, c * 256 + lane * 8, it.v);
}

// Largest magnitude of a row of K activations, by one warp (8 loads per
// lane in flight).
template <bool IN_F32>
__device__ __forceinline__ float row_absmax(const void* row, int K, int lane)
{
    float mx = 0.0f;
#pragma unroll 8
    for (int k = lane * 8; k < K; k += 256) {
        float u[8];
        load8<IN_F32>(row, k, u);
#pragma unroll
        for (int i = 0; i < 8; i++) mx = fmaxf(mx, fabsf(u[i]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    return mx;
}

// The quantisation items first, first + step, ... (below end) of one
// epilogue warp, two at a time: both items' loads first, then their terms.
// An NVFP4 row's scale 2^p comes from its largest magnitude, taken once per
// source row the warp meets (NVFP4 warps take consecutive items: chunks of
// a row, then of the next; MXFP4 warps every step-th).  After the first loads are issued, lane 0 arrives on
// `loaded` (when not null): the copy warp holds its weight prefetch until
// then, so these few loads do not queue behind megabytes of bulk copies.
template <int WFMT, int T, bool IN_F32>
__device__ __forceinline__ void fused_quant_items(const Plan& P, const void* in, int K, const int32_t* gather, int gk,
                                                  char* bimg, int32_t* rex, long first, long step, long end,
                                                  int lane, uint64_t* loaded)
{
    using FM = Fmt<WFMT>;
    constexpr int VS = FM::VS, LPB = VS / 8;
    const int KC = K / 256, kin = lane * 8;
    const void* p_row = nullptr;   // NVFP4: the source row whose exponent is p (scale sc)
    int p = 0;
    float sc = 1.0f;
    for (long i0 = first; i0 < end; i0 += 2 * step) {
        QItem q[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const long i = i0 + k * step;
            q[k].cb = nullptr;
            if (i < end) qitem_load<WFMT, T, IN_F32>(q[k], P, in, K, gather, gk, (int)(i / KC), (int)(i % KC), bimg, lane);
        }
        if (loaded && i0 == first) {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(loaded));
            loaded = nullptr;
        }
        if (WFMT == MOE_W_NVFP4) {
#pragma unroll
            for (int k = 0; k < 2; k++) {
                if (!q[k].cb) continue;   // the same for the whole warp
                if (q[k].row != p_row) {
                    p = row_exponent(row_absmax<IN_F32>(q[k].row, K, lane));
                    sc = ldexpf(1.0f, p);
                    p_row = q[k].row;
                }
                if (q[k].c == 0 && lane == 0) rex[q[k].r] = p;
#pragma unroll
                for (int j = 0; j < 8; j++) q[k].v[j] = __fmul_rn(q[k].v[j], sc);
            }
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            if (!q[k].cb) continue;
#pragma unroll 1
            for (int t = 0; t < T; t++) {
                uint32_t scode;
                const uint32_t word = term8<WFMT, LPB>(q[k].v, &scode);
                const int n = q[k].n0 + t;
                *reinterpret_cast<uint32_t*>(q[k].cb + img_code_off(n, kin)) = word;
                if ((lane % LPB) == 0) q[k].cb[img_scale_off<VS>(q[k].N, n, kin)] = (char)scode;
            }
        }
    }
    if (loaded && lane == 0) mbar_arrive(smem_u32(loaded));   // no items
}

template <int WFMT>
__global__ void __launch_bounds__(kThreads, 1) ffn_fp4_fused_kernel(FusedArgs f)
{
    using FM = Fmt<WFMT>;
    using CFG = DecodeCfg;
    using KC_ = KCfg<WFMT, CFG>;
    using FC = FusedCfg<WFMT>;
    constexpr int D = FC::D, STAGE = FC::STAGE, T = CFG::T, NT = CFG::NT;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ int s_g[kThreads / 32], s_b[kThreads / 32];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // [D]
    uint64_t* empty = full + D;                           // [D]
    uint64_t* acc_full = empty + D;                       // [2]
    uint64_t* acc_empty = acc_full + 2;                   // [2]
    uint64_t* fin = acc_empty + 2;
    uint64_t* gate = fin + 1;                             // [2]: x terms published, h terms published
    uint64_t* xloaded = gate + 2;                         // the epilogue warps' first x loads are issued
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xloaded + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    int* s_last = abort_flag + 1;
    int* s_flag = s_last + 1;
    Plan P;
    P.E = f.p1.E;
    P.off = reinterpret_cast<int*>(smem + 1024);
    P.gpre = P.off + (kFusedMaxE + 1);
    P.boff = P.gpre + (kFusedMaxE + 1);
    P.slot = P.boff + (kFusedMaxE + 1);
    unsigned char* ring = smem + 1024 + FC::PLAN;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = P.E, rows = f.p1.rows;
    const int bfull = b_chunk_bytes(CFG::NMAX, FM::NSUB);

    if (tid == 0) {
        for (int i = 0; i < D; i++) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 32 * kEpiWarps);
            mbar_init(smem_u32(&gate[i]), 1);
        }
        mbar_init(smem_u32(fin), 1);
        mbar_init(smem_u32(xloaded), kEpiWarps);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(KC_::TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    // ---- plan: the call's token groups (the same in every CTA)
    {
        const int EPT = (E + kThreads - 1) / kThreads;   // <= 3 for E <= 512
        int gl = 0, bl = 0;
        for (int i = 0; i < EPT; i++) {
            const int e = tid * EPT + i;
            if (e < E) {
                const int o0 = __ldg(f.p1.offsets + e), o1 = __ldg(f.p1.offsets + e + 1);
                const int sl = __ldg(f.p1.slot_of + e);
                const bool ok = o1 > o0 && sl >= 0 && sl < f.p1.pool_slots && o0 >= 0 && o1 <= rows;
                P.off[e] = o0;
                P.slot[e] = ok ? sl : -1;
                if (e == E - 1) P.off[E] = o1;
                if (ok) {
                    const int g = (o1 - o0 + NT - 1) / NT, last = o1 - o0 - (g - 1) * NT;
                    gl += g;
                    bl += (g - 1) * bfull + b_chunk_bytes(((T * last + 7) / 8) * 8, FM::NSUB);
                }
            }
        }
        int gi = gl, bi = bl;   // inclusive scan over the warp, then over the warps
        for (int o = 1; o < 32; o <<= 1) {
            const int go = __shfl_up_sync(0xffffffffu, gi, o), bo = __shfl_up_sync(0xffffffffu, bi, o);
            if (lane >= o) { gi += go; bi += bo; }
        }
        if (lane == 31) { s_g[warp] = gi; s_b[warp] = bi; }
        __syncthreads();   // also publishes P.off / P.slot
        int gr = gi - gl, br = bi - bl;
        for (int w = 0; w < warp; w++) { gr += s_g[w]; br += s_b[w]; }
        for (int i = 0; i < EPT; i++) {
            const int e = tid * EPT + i;
            if (e < E) {
                P.gpre[e] = gr;
                P.boff[e] = br;
                if (P.slot[e] >= 0) {
                    const int m = P.off[e + 1] - P.off[e];
                    const int g = (m + NT - 1) / NT, last = m - (g - 1) * NT;
                    gr += g;
                    br += (g - 1) * bfull + b_chunk_bytes(((T * last + 7) / 8) * 8, FM::NSUB);
                }
            }
        }
        if (tid == kThreads - 1) { P.gpre[E] = gr; P.boff[E] = br; }
    }
    // the piece counters of both phases start at zero (published by the first grid barrier)
    for (int i = blockIdx.x * kThreads + tid; i < f.ncnt; i += gridDim.x * kThreads) {
        f.p1.cnt[i] = 0;
        f.cnt2[i] = 0;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int* abort_v = abort_flag;
    const int grid = gridDim.x;
    const int NG = P.gpre[E];
    if (NG == 0) {
        // no expert with rows has a slot (an empty miss-group pass): every
        // CTA sees the same plan and leaves before the first grid barrier
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(KC_::TMEM_COLS)
                         : "memory");
        }
        return;
    }

    if (warp == 0) {
        // ============ bulk copies of both phases: the whole warp walks the
        // chunk sequence, one elected lane issues.  A phase's activation copies
        // wait for its gate (the grid barrier that publishes the images); the
        // weight copies do not, up to a ring full of held-back stages.
        int st = 0;
        uint32_t ph = 0;
        long issued = 0;
        bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(xloaded), 0, abort_v, f.p1.wait));   // x loads first
        int withheld = -1;   // testing: the stage left unfilled
        int pend_st[D];
        const char* pend_src[D];
        uint32_t pend_bytes[D];
        for (int phase = 0; phase < 2 && ok; phase++) {
            const Fp4Args& a = phase ? f.p2 : f.p1;
            const int RB = a.R / 128, KC = a.K / 256, NU = NG * RB;
            const long W = (long)NU * KC;
            const int gridp = (int)(W < (long)grid ? W : (long)grid);
            if ((int)blockIdx.x >= gridp) continue;
            int npend = 0;
            bool open = false;   // this phase's activation images are published
            auto issue_pending = [&]() {
                for (int i = 0; i < npend; i++)
                    bulk_g2s(smem_u32(ring + (size_t)pend_st[i] * STAGE + KC_::A_BYTES), pend_src[i], pend_bytes[i],
                             smem_u32(&full[pend_st[i]]));
                npend = 0;
            };
            auto release = [&]() -> bool {
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&gate[phase]), 0, abort_v, f.p1.wait))) return false;
                asm volatile("fence.proxy.async.global;" ::: "memory");
                issue_pending();
                open = true;
                return true;
            };
            Seg sg{sk_bound(W, blockIdx.x, gridp)};
            const long b1 = sk_bound(W, blockIdx.x + 1, gridp);
            while (ok && sg.next(false, NU, KC, b1)) {
                const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, plan_group(P, sg.u / RB, NT, bfull));
                for (int c = sg.p0; c < sg.p1; c++) {
                    // a ring full of held-back stages: wait for the gate before reusing one
                    if (!open && npend == D && !(ok = release())) break;
                    if (!(ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&empty[st]), ph ^ 1, abort_v, f.p1.wait))))
                        break;
                    const uint32_t bar = smem_u32(&full[st]);
                    unsigned char* sp = ring + (size_t)st * STAGE;
                    if (f.p1.withhold && blockIdx.x == 0 && issued == 0) {
                        withheld = st;   // testing: never filled, so the wait for it runs out
                    } else {
                        mbar_expect_tx(bar, (uint32_t)(FM::CB + U.bb));
                        bulk_g2s(smem_u32(sp), U.a + (size_t)c * FM::CB, FM::CB, bar);
                        // the unit's chunks kPfUnit ahead go to L2 meanwhile
                        if (c == sg.p0)
                            for (int j = 1; j < kPfUnit && c + j < sg.p1; j++)
                                prefetch_l2(U.a + (size_t)(c + j) * FM::CB, FM::CB);
                        if (c + kPfUnit < sg.p1) prefetch_l2(U.a + (size_t)(c + kPfUnit) * FM::CB, FM::CB);
                        // (once the gate has passed, release() cannot fail)
                        if (!open && __any_sync(0xffffffffu, mbar_try(smem_u32(&gate[phase]), 0))) release();
                        if (open) {
                            bulk_g2s(smem_u32(sp + KC_::A_BYTES), U.b + (size_t)c * U.bb, (uint32_t)U.bb, bar);
                        } else {
                            pend_st[npend] = st;
                            pend_src[npend] = U.b + (size_t)c * U.bb;
                            pend_bytes[npend++] = (uint32_t)U.bb;
                        }
                    }
                    issued++;
                    if (++st == D) { st = 0; ph ^= 1; }
                }
            }
            if (ok && !open && npend > 0) ok = release();
            // after an abort the held-back activation copies are issued anyway
            // (their data is not used), so that every stage whose weight copy
            // went out completes its phase before the drain
            if (!ok) issue_pending();
        }
        // every issued copy lands before the CTA exits (a withheld stage is
        // never refilled: its consumer gives up first)
        for (int i = 0; i < D && i < issued; i++)
            if (i != withheld) mbar_drain(smem_u32(&full[i]), i < st ? ph : (ph ^ 1));
    } else if (warp == 1) {
        // ============ scale-factor copies and MMAs of both phases (the whole
        // warp walks the loop, one elected lane issues)
        const uint32_t ring_s = smem_u32(ring);
        {
            int st = 0, it = 0;
            uint32_t ph = 0;
            long cc = 0;
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; phase++) {
                const Fp4Args& a = phase ? f.p2 : f.p1;
                const int RB = a.R / 128, KC = a.K / 256, NU = NG * RB;
                const long W = (long)NU * KC;
                const int gridp = (int)(W < (long)grid ? W : (long)grid);
                if ((int)blockIdx.x >= gridp) continue;
                Seg sg{sk_bound(W, blockIdx.x, gridp)};
                const long b1 = sk_bound(W, blockIdx.x + 1, gridp);
                while (ok && sg.next(false, NU, KC, b1)) {
                    const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, plan_group(P, sg.u / RB, NT, bfull));
                    const int ab = it & 1, nh = (U.n + 127) / 128;
                    const uint32_t id0 = idesc_fp4<WFMT>(U.n, 0), id1 = idesc_fp4<WFMT>(U.n, 2);
                    if (it >= 2) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(smem_u32(&acc_empty[ab]), ((it >> 1) - 1) & 1, abort_v, f.p1.wait));
                        if (!ok) break;
                        tc_fence_after();
                    }
                    const uint32_t dcol = tmem + (uint32_t)(ab * CFG::NMAX);
                    for (int c = sg.p0; c < sg.p1; c++, cc++) {
                        if (!(ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), ph, abort_v, f.p1.wait))))
                            break;
                        tc_fence_after();
                        const uint32_t sfa = tmem + KC_::SF_COL + (uint32_t)((cc & 1) * KC_::SF_SET);
                        issue_chunk<WFMT, KC_::A_BYTES>(ring_s + (uint32_t)(st * STAGE), U.n, nh, dcol, sfa,
                                                        sfa + KC_::SF_A, id0, id1, c == sg.p0);
                        tc_commit(smem_u32(&empty[st]));
                        if (++st == D) { st = 0; ph ^= 1; }
                    }
                    if (!ok) break;
                    tc_commit(smem_u32(&acc_full[ab]));
                    it++;
                }
            }
            tc_commit(smem_u32(fin));
            mbar_drain(smem_u32(fin), 0);
        }
    } else {
        // ============ epilogue warps: terms of x, phase-1 epilogue, terms of h, phase-2 epilogue.
        // All four warps walk the same items and segments and meet the same
        // barriers; after a failed wait they keep walking without waiting.
        const int q = warp & 3;
        const int etid = tid - 64;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int it = 0;
        bool ok = true;
        unsigned long long gb_next = etid == 0 ? grid_bar_first() : 0ull;
        for (int phase = 0; phase < 2; phase++) {
            const Fp4Args& a = phase ? f.p2 : f.p1;
            {   // the activation terms of this phase's input rows: (row, chunk) items; NVFP4
                // warps take equal ranges of consecutive items, MXFP4 warps every nw-th
                const long items = (long)rows * (a.K / 256), nw = (long)grid * kEpiWarps;
                const long w_ = (long)blockIdx.x * kEpiWarps + (warp - 2), per = (items + nw - 1) / nw;
                long first = w_, step = nw, end = items;
                if (WFMT == MOE_W_NVFP4) {
                    first = w_ * per < items ? w_ * per : items;
                    step = 1;
                    end = first + per < items ? first + per : items;
                }
                if (phase == 1)
                    fused_quant_items<WFMT, T, true>(P, f.p1.out_h, a.K, nullptr, 1, f.bh, f.rex_h, first, step, end,
                                                     lane, nullptr);
                else if (f.x_f32)
                    fused_quant_items<WFMT, T, true>(P, f.x, a.K, f.gather, f.gk, f.bx, f.rex_x, first, step, end,
                                                     lane, xloaded);
                else
                    fused_quant_items<WFMT, T, false>(P, f.x, a.K, f.gather, f.gk, f.bx, f.rex_x, first, step, end,
                                                      lane, xloaded);
            }
            ok = grid_sync_epi(etid, s_flag, f.p1.wait, gb_next) && ok;   // terms published (phase 0: counters zero)
            if (etid == 0) mbar_arrive(smem_u32(&gate[phase]));
            const int RB = a.R / 128, KC = a.K / 256, NU = NG * RB;
            const long W = (long)NU * KC;
            const int gridp = (int)(W < (long)grid ? W : (long)grid);
            if ((int)blockIdx.x < gridp) {
                const long b0 = sk_bound(W, blockIdx.x, gridp), b1 = sk_bound(W, blockIdx.x + 1, gridp);
                Seg sg{b0};
                while (sg.next(false, NU, KC, b1)) {
                    const Unit U = unit_of<WFMT, CFG>(a, sg.u, RB, KC, plan_group(P, sg.u / RB, NT, bfull));
                    const int ab = it & 1;
                    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[ab]), (it >> 1) & 1, abort_v, f.p1.wait));
                    if (ok) tc_fence_after();
                    float tsc = 1.0f;
                    if (WFMT == MOE_W_NVFP4) tsc = __ldg(reinterpret_cast<const float*>(U.blob + a.ts_off) + phase);
                    const uint32_t dcol = tmem + lane_base + (uint32_t)(ab * CFG::NMAX);
                    const int nch = (U.nt + 7) / 8;
                    if (sg.p0 == 0 && sg.p1 == KC) {
                        if (ok) {
                            for (int ch = 0; ch < nch; ch++) {
                                uint32_t d[8 * T];
#pragma unroll
                                for (int t = 0; t < T; t++) tmem_ld8(dcol + 8 * T * ch + 8 * t, d + 8 * t);
                                tmem_wait_ld();
                                if (phase == 0)
                                    finish8<WFMT, 1, T>(a, U, q, lane, ch, reinterpret_cast<const float*>(d), tsc);
                                else
                                    finish8<WFMT, 2, T>(a, U, q, lane, ch, reinterpret_cast<const float*>(d), tsc);
                            }
                            tc_fence_before();
                            mbar_arrive(smem_u32(&acc_empty[ab]));
                        }
                    } else {
                        const int slot = sg.start == b0 ? 0 : 1;
                        float* mine = a.pieces + ((size_t)blockIdx.x * 2 + slot) * (128 * CFG::NMAX);
                        if (ok) {
                            for (int ch = 0; ch < nch; ch++) {
                                uint32_t d[8 * T];
#pragma unroll
                                for (int t = 0; t < T; t++) tmem_ld8(dcol + 8 * T * ch + 8 * t, d + 8 * t);
                                tmem_wait_ld();
#pragma unroll
                                for (int i = 0; i < 8 * T; i++)
                                    mine[(size_t)(8 * T * ch + i) * 128 + etid] = __uint_as_float(d[i]);
                            }
                            tc_fence_before();
                            mbar_arrive(smem_u32(&acc_empty[ab]));
                        }
                        __threadfence();
                        epi_bar();
                        const long u_lo = (long)sg.u * KC, u_hi = u_lo + KC - 1;
                        const int c_lo = sk_cta_of(W, u_lo, gridp), c_hi = sk_cta_of(W, u_hi, gridp);
                        if (etid == 0) *s_last = (ok && !*abort_v && atomicAdd(a.cnt + sg.u, 1) == c_hi - c_lo) ? 1 : 0;
                        epi_bar();
                        if (*s_last) {
                            __threadfence();
                            for (int ch = 0; ch < nch; ch++) {
                                float d[8 * T];
#pragma unroll
                                for (int i = 0; i < 8 * T; i++) d[i] = 0.0f;
                                for (int c = c_lo; c <= c_hi; c++) {
                                    const int sl = sk_bound(W, c, gridp) >= u_lo ? 0 : 1;
                                    const float* pc = a.pieces + ((size_t)c * 2 + sl) * (128 * CFG::NMAX);
#pragma unroll
                                    for (int i = 0; i < 8 * T; i++)
                                        d[i] += __ldcg(pc + (size_t)(8 * T * ch + i) * 128 + etid);
                                }
                                if (phase == 0) finish8<WFMT, 1, T>(a, U, q, lane, ch, d, tsc);
                                else finish8<WFMT, 2, T>(a, U, q, lane, ch, d, tsc);
                            }
                            if (etid == 0) a.cnt[sg.u] = 0;
                        }
                        epi_bar();   // s_last is rewritten by the next piece
                    }
                    it++;
                }
            }
            if (phase == 0) ok = grid_sync_epi(etid, s_flag, f.p1.wait, gb_next) && ok;   // h complete before its terms are taken
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(KC_::TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host side
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

struct Fp4Ws {
    int32_t* gpre;
    int32_t* boffc;
    int4* gtab;
    int32_t* rex_x;
    int32_t* rex_h;
    char* bx;
    char* bh;
    float* h32;
    int32_t* cnt;
    int32_t* cnt2;   // second counter set (the fused decode kernel's down projection)
    int ncnt;
    float* pieces;
};

// Upper bound of the per-chunk bytes of all token-group images of a call.
template <class CFG>
size_t group_chunk_bound(int rows, int E, int nsub)
{
    const size_t G = (size_t)(rows + CFG::NT - 1) / CFG::NT + (size_t)(rows < E ? rows : E);
    const size_t n = (size_t)CFG::T * rows + 7 * G;          // image rows
    return 128 * n + (size_t)nsub * 512 * (G + n / 128 + 1);
}

size_t fp4_ws_layout(const moe_shape* s, int rows, void* base, Fp4Ws* w)
{
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align_up(o + b, 256); return at; };
    const int R = rows > 0 ? rows : 1, E = s->experts, nsub = s->wfmt == MOE_W_MXFP4 ? 2 : 4;
    const size_t per_chunk =
        group_chunk_bound<DecodeCfg>(R, E, nsub) > group_chunk_bound<PrefillCfg>(R, E, nsub)
            ? group_chunk_bound<DecodeCfg>(R, E, nsub)
            : group_chunk_bound<PrefillCfg>(R, E, nsub);
    const size_t ogp = take(4 * (size_t)(E + 1));
    const size_t obo = take(4 * (size_t)(E + 1));
    const size_t Gmax = (size_t)(R + DecodeCfg::NT - 1) / DecodeCfg::NT + (size_t)(R < E ? R : E);
    const size_t ogt = take(16 * Gmax);
    const size_t orx = take(4 * (size_t)R);
    const size_t orh = take(4 * (size_t)R);
    const size_t obx = take(per_chunk * (s->hidden / 256));
    const size_t obh = take(per_chunk * (s->ffn / 256));
    const size_t oh = take(4 * (size_t)R * s->ffn);
    const long RBmax = (2 * s->ffn > s->hidden ? 2 * s->ffn : s->hidden) / 128;
    const long ncnt = ((long)(R + DecodeCfg::NT - 1) / DecodeCfg::NT + (R < E ? R : E)) * RBmax;
    const size_t oc = take(4 * (size_t)ncnt);
    const size_t oc2 = take(4 * (size_t)ncnt);
    const size_t op = take(4 * (size_t)kMaxCtas * 2 * 128 * DecodeCfg::NMAX);
    if (w) {
        char* b = static_cast<char*>(base);
        w->gpre = reinterpret_cast<int32_t*>(b + ogp);
        w->boffc = reinterpret_cast<int32_t*>(b + obo);
        w->gtab = reinterpret_cast<int4*>(b + ogt);
        w->rex_x = reinterpret_cast<int32_t*>(b + orx);
        w->rex_h = reinterpret_cast<int32_t*>(b + orh);
        w->bx = b + obx;
        w->bh = b + obh;
        w->h32 = reinterpret_cast<float*>(b + oh);
        w->cnt = reinterpret_cast<int32_t*>(b + oc);
        w->cnt2 = reinterpret_cast<int32_t*>(b + oc2);
        w->ncnt = (int)ncnt;
        w->pieces = reinterpret_cast<float*>(b + op);
    }
    return o;
}

template <int WFMT, int PHASE, class CFG>
int set_smem_attr()
{
    constexpr int smem = KCfg<WFMT, CFG>::SMEM;
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    static bool done[kMaxDevices];
    if (!done[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_fp4_kernel<WFMT, PHASE, CFG>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        done[dev] = true;
    }
    return MOE_OK;
}

constexpr uint8_t* kNoCanon = nullptr;

template <int WFMT, class CFG>
int run_fp4(const moe_shape* s, const BlobLayout& bl, const void* pool, size_t slot_bytes, int pool_slots,
            const int32_t* slot_of, const int32_t* offsets, int rows, uint16_t* y_perm, const Fp4Ws& w,
            const RowSource& src, int sms, cudaStream_t st)
{
    using FM = Fmt<WFMT>;
    const int E = s->experts, H = s->hidden, F = s->ffn;
    // per-chunk image offsets must stay 32-bit
    if (group_chunk_bound<CFG>(rows, E, FM::NSUB) >= (size_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    int rc;
    if ((rc = set_smem_attr<WFMT, 1, CFG>())) return rc;
    if ((rc = set_smem_attr<WFMT, 2, CFG>())) return rc;
    MOE_CUDA_TRY(launch_pdl(fp4_plan_kernel, 1, 256, 0, st, offsets, slot_of, E, rows, pool_slots, CFG::NT, CFG::T,
                            FM::NSUB, w.gpre, w.boffc, w.gtab, w.cnt, w.ncnt));
    auto qgrid_for = [&](int K) {
        const long items = (long)rows * ((K + kSegCols - 1) / kSegCols);
        return (int)(items < (long)sms * 8 ? items : (long)sms * 8);
    };
    const int qgrid = qgrid_for(H);
    if (src.x_dtype == MOE_DT_F32)
        MOE_CUDA_TRY(launch_pdl(fp4_terms_kernel<WFMT, CFG::T, true>, qgrid, kQuantThreads, 0, st, src.x, rows, H,
                                src.assign_of, src.k, offsets, slot_of, E, pool_slots, w.boffc, CFG::NT, w.bx, w.rex_x,
                                kNoCanon, kNoCanon));
    else
        MOE_CUDA_TRY(launch_pdl(fp4_terms_kernel<WFMT, CFG::T, false>, qgrid, kQuantThreads, 0, st, src.x, rows, H,
                                src.assign_of, src.k, offsets, slot_of, E, pool_slots, w.boffc, CFG::NT, w.bx, w.rex_x,
                                kNoCanon, kNoCanon));
    Fp4Args a{};
    a.pool = static_cast<const char*>(pool);
    a.slot_bytes = slot_bytes;
    a.ts_off = bl.ts;
    a.E = E;
    a.rows = rows;
    a.pool_slots = pool_slots;
    a.slot_of = slot_of;
    a.offsets = offsets;
    a.gpre = w.gpre;
    a.gtab = w.gtab;
    a.cnt = w.cnt;
    a.pieces = w.pieces;
    a.wait = test_wait_cycles(kWaitCycles);
    a.withhold = test_withhold();
    const int grid = sms < kMaxCtas ? sms : kMaxCtas;
    constexpr int smem = KCfg<WFMT, CFG>::SMEM;
    a.w_off = bl.w13;
    a.R = 2 * F;
    a.K = H;
    a.bimg = w.bx;
    a.rex = WFMT == MOE_W_NVFP4 ? w.rex_x : nullptr;
    a.out_h = w.h32;
    MOE_CUDA_TRY(launch_pdl(ffn_fp4_kernel<WFMT, 1, CFG>, grid, SepCfg<CFG>::THREADS, smem, st, a));
    MOE_CUDA_TRY(launch_pdl(fp4_terms_kernel<WFMT, CFG::T, true>, qgrid_for(F), kQuantThreads, 0, st,
                            static_cast<const void*>(w.h32), rows, F, static_cast<const int32_t*>(nullptr), 1,
                            offsets, slot_of, E, pool_slots, w.boffc, CFG::NT, w.bh, w.rex_h, kNoCanon, kNoCanon));
    Fp4Args b = a;
    b.w_off = bl.w2;
    b.R = H;
    b.K = F;
    b.bimg = w.bh;
    b.rex = WFMT == MOE_W_NVFP4 ? w.rex_h : nullptr;
    b.out_h = nullptr;
    b.out_y = y_perm;
    MOE_CUDA_TRY(launch_pdl(ffn_fp4_kernel<WFMT, 2, CFG>, grid, SepCfg<CFG>::THREADS, smem, st, b));
    return MOE_OK;
}

// The whole decode-tile FFN call as one cooperative launch (one CTA per SM).
// Returns MOE_ERR_UNSUPPORTED when the device cannot run it that way, so the
// caller falls back to one launch per step.
template <int WFMT>
int run_fp4_fused(const moe_shape* s, const BlobLayout& bl, const void* pool, size_t slot_bytes, int pool_slots,
                  const int32_t* slot_of, const int32_t* offsets, int rows, uint16_t* y_perm, const Fp4Ws& w,
                  const RowSource& src, int sms, cudaStream_t st)
{
    using FC = FusedCfg<WFMT>;
    const int E = s->experts, H = s->hidden, F = s->ffn;
    if (E > kFusedMaxE) return MOE_ERR_UNSUPPORTED;
    if (group_chunk_bound<DecodeCfg>(rows, E, Fmt<WFMT>::NSUB) >= (size_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
    int dev = 0, coop = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
    if (!coop) return MOE_ERR_UNSUPPORTED;
    static int resident[kMaxDevices];   // 0 unknown, 1 one CTA per SM fits, -1 it does not
    if (!resident[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_fp4_fused_kernel<WFMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          FC::SMEM));
        int nb = 0;
        MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, ffn_fp4_fused_kernel<WFMT>, kThreads, FC::SMEM));
        resident[dev] = nb >= 1 ? 1 : -1;
    }
    if (resident[dev] < 0) return MOE_ERR_UNSUPPORTED;
    FusedArgs f{};
    Fp4Args& a = f.p1;
    a.pool = static_cast<const char*>(pool);
    a.slot_bytes = slot_bytes;
    a.ts_off = bl.ts;
    a.E = E;
    a.rows = rows;
    a.pool_slots = pool_slots;
    a.slot_of = slot_of;
    a.offsets = offsets;
    a.pieces = w.pieces;
    a.w_off = bl.w13;
    a.R = 2 * F;
    a.K = H;
    a.bimg = w.bx;
    a.rex = WFMT == MOE_W_NVFP4 ? w.rex_x : nullptr;
    a.out_h = w.h32;
    a.cnt = w.cnt;
    a.wait = test_wait_cycles(kWaitCycles);
    a.withhold = test_withhold();
    Fp4Args& b = f.p2;
    b = a;
    b.w_off = bl.w2;
    b.R = H;
    b.K = F;
    b.bimg = w.bh;
    b.rex = WFMT == MOE_W_NVFP4 ? w.rex_h : nullptr;
    b.out_h = nullptr;
    b.out_y = y_perm;
    b.cnt = w.cnt2;
    f.x = src.x;
    f.x_f32 = src.x_dtype == MOE_DT_F32;
    f.gather = src.assign_of;
    f.gk = src.k;
    f.bx = w.bx;
    f.bh = w.bh;
    f.rex_x = w.rex_x;
    f.rex_h = w.rex_h;
    f.cnt2 = w.cnt2;
    f.ncnt = w.ncnt;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms < kMaxCtas ? sms : kMaxCtas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = FC::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, ffn_fp4_fused_kernel<WFMT>, f));
    return MOE_OK;
}

// Prefill tiles once groups are large (four rows per expert on average);
// MOE_FFN_TILE=decode|prefill overrides the choice.
bool use_prefill_tiles(const moe_shape* s, int rows)
{
    const char* force = getenv("MOE_FFN_TILE");
    if (force && !strcmp(force, "decode")) return false;
    if (force && !strcmp(force, "prefill")) return true;
    return rows >= 4 * s->experts;
}

}  // namespace

size_t ffn_fp4_ws_bytes(const moe_shape* s, int rows) { return fp4_ws_layout(s, rows, nullptr, nullptr) + 256; }

int ffn_fp4_device_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_fp4_error, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    if (clear && v) {
        // the kernels are not running: put the grid barrier back in its idle state too
        const int z = 0;
        const unsigned long long zu[kMaxCtas + 1] = {};
        if (cudaMemcpyToSymbol(g_fp4_error, &z, sizeof z) != cudaSuccess ||
            cudaMemcpyToSymbol(g_gb_abort, &z, sizeof z) != cudaSuccess ||
            cudaMemcpyToSymbol(g_gb_count, zu, sizeof zu) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return v;
}

int launch_ffn_fp4(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
                   const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm, void* ws,
                   cudaStream_t st, const RowSource* gather, bool one_expert)
{
    Fp4Ws w;
    fp4_ws_layout(s, rows, ws, &w);
    int dev = 0, sms = 148;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const RowSource src = gather ? *gather : RowSource{x_perm, MOE_DT_BF16, nullptr, 1};
    const BlobLayout bl = blob_layout(s);
    const bool pre = use_prefill_tiles(s, rows);
    if (one_expert && !pre) {
        // One expert's decode pass is latency-bound: about 16 gate-up chunks
        // per CTA (32 CTAs for H = 4096, F = 2048) beat one chunk-sliver per SM
        // (measured, one expert and two rows: 45 us on 148 CTAs, 37 on 64, 31.5
        // on 32).  The stream-K split, and so the bits, follow the grid.
        const int cap = (2 * s->ffn / 128) * (s->hidden / 256) / 16;
        sms = std::min(sms, std::max(8, cap));
    }
    if (!pre && !getenv("MOE_FFN_UNFUSED")) {
        const int rc = s->wfmt == MOE_W_MXFP4
                           ? run_fp4_fused<MOE_W_MXFP4>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                        y_perm, w, src, sms, st)
                           : run_fp4_fused<MOE_W_NVFP4>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                        y_perm, w, src, sms, st);
        if (rc != MOE_ERR_UNSUPPORTED) {
            if (rc == MOE_OK) prof_count(MOE_PROF_FFN, 1);
            return rc;
        }
    }
    prof_count(MOE_PROF_FFN, 5);
    if (s->wfmt == MOE_W_MXFP4)
        return pre ? run_fp4<MOE_W_MXFP4, PrefillCfg>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                      y_perm, w, src, sms, st)
                   : run_fp4<MOE_W_MXFP4, DecodeCfg>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                     y_perm, w, src, sms, st);
    if (s->wfmt == MOE_W_NVFP4)
        return pre ? run_fp4<MOE_W_NVFP4, PrefillCfg>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                      y_perm, w, src, sms, st)
                   : run_fp4<MOE_W_NVFP4, DecodeCfg>(s, bl, pool, slot_bytes, pool_slots, slot_of, offsets, rows,
                                                     y_perm, w, src, sms, st);
    return MOE_ERR_INVALID_ARG;
}

}  // namespace moe

extern "C" int moe_act_terms(const void* d_x, int32_t x_dtype, int32_t rows, int32_t K, int32_t wfmt,
                             int32_t terms, uint8_t* d_codes, uint8_t* d_scales, int32_t* d_row_exp, void* stream)
{
    using namespace moe;
    if (rows < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (wfmt != MOE_W_MXFP4 && wfmt != MOE_W_NVFP4) return MOE_ERR_INVALID_ARG;
    if (terms != 3 && terms != 4) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!d_x || !d_codes || !d_scales || !d_row_exp || ((uintptr_t)d_x & 15)) return MOE_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const long items = (long)rows * ((K + kSegCols - 1) / kSegCols);
    const int grid = (int)(items < (long)sms * 8 ? items : (long)sms * 8);
    cudaStream_t st = as_stream(stream);
    const bool f32 = x_dtype == MOE_DT_F32;
#define MOE_TERMS_LAUNCH(W, TT, F)                                                                                 \
    fp4_terms_kernel<W, TT, F, true><<<grid, kQuantThreads, 0, st>>>(d_x, rows, K, nullptr, 1, nullptr, nullptr, 0, \
                                                                      0, nullptr, 1, nullptr, d_row_exp, d_codes,  \
                                                                      d_scales)
    if (wfmt == MOE_W_MXFP4) {
        if (terms == 3) { if (f32) MOE_TERMS_LAUNCH(MOE_W_MXFP4, 3, true); else MOE_TERMS_LAUNCH(MOE_W_MXFP4, 3, false); }
        else { if (f32) MOE_TERMS_LAUNCH(MOE_W_MXFP4, 4, true); else MOE_TERMS_LAUNCH(MOE_W_MXFP4, 4, false); }
    } else {
        if (terms == 3) { if (f32) MOE_TERMS_LAUNCH(MOE_W_NVFP4, 3, true); else MOE_TERMS_LAUNCH(MOE_W_NVFP4, 3, false); }
        else { if (f32) MOE_TERMS_LAUNCH(MOE_W_NVFP4, 4, true); else MOE_TERMS_LAUNCH(MOE_W_NVFP4, 4, false); }
    }
#undef MOE_TERMS_LAUNCH
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
