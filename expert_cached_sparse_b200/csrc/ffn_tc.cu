// Prefill grouped SwiGLU GEMM on the fifth-generation tensor cores (tcgen05).
//
// Prefill touches nearly every expert with tens to hundreds of rows each, so
// the expert FFN becomes a grouped GEMM ("FreeToken 290b model", section
// "Como gestiona FreeToken el prellenado y la decodificacion": prefill runs
// whole layers; the pages' own design streams the next layer's experts over
// PCIe, here every expert is already resident).  Design for sm_100a:
//  - swap-AB: the expert's weight rows are the MMA's M side (128 rows per
//    tile), tokens the N side (up to 192 per tile), K in chunks of 64;
//  - weights stay packed FP4 in HBM; a bulk copy brings each 128 x 64 FP4
//    chunk (4 KB + scales) to shared memory, eight warps expand it exactly to
//    f16 (E2M1 x block scale is exact in f16 for the accepted scale codes)
//    and write it with tcgen05.st straight into tensor memory, where the MMA
//    reads its A operand; no f16 weight tile ever touches shared memory;
//  - tokens (x_perm, or h for the down projection) arrive by TMA in 16- to
//    128-row boxes with the 128-byte swizzle the MMA's shared-memory
//    descriptor expects, as many 64-column chunks per 32 KB stage as fit, so
//    small token blocks keep more chunks in flight; rows past the expert's
//    block are loaded but never stored;
//  - two accumulators live in tensor memory (128 lanes x up to 192 fp32
//    columns each); four epilogue warps read one back with tcgen05.ld while
//    the MMA fills the other: SwiGLU (gate and up rows are 8 lanes apart, one
//    shuffle) into h, or the NVFP4 tensor scale into y;
//  - warp 0 issues the weight copies, the last warp the token copies, warp 1
//    the MMAs (one thread each); mbarriers chain the roles; every wait is
//    bounded and a timeout sets an error word and drains the CTA instead of
//    hanging.
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {

__device__ int g_tc_error;   // first device-side error of the tensor-core FFN (0: none)

namespace {

constexpr int BM = 128;
constexpr int BN_MAX = 192;       // token rows per tile (two accumulators fit tensor memory)
constexpr int BK = 64;
constexpr int SA = 16;             // FP4 A stages (one 64-column chunk each)
constexpr int SB = 4;              // token (B) stages: as many 64-column chunks as fit 32 KB
constexpr int NABUF = 4;           // tensor-memory A buffers
constexpr int NXG = 1;             // expanding groups: group g expands chunks g, g+NXG, ...
constexpr int NXW = 8 * NXG;       // expanding warps: two per tensor-memory lane quarter and group
constexpr int NEPI = 4;            // epilogue warps, one per tensor-memory lane quarter
constexpr int BWARP = 2 + NXW + NEPI;           // token (B) copy issue
constexpr int THREADS = 32 * (BWARP + 1);         // warp 0 weight copies, warp 1 MMA, expand, epilogue, B copies
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;      // two accumulators: columns [0, 192) and [192, 384)
constexpr uint32_t A_COL = 384;    // A buffers: 32 columns each (4 buffers: 384..511)
constexpr uint32_t B_STAGE_BYTES = 32 * 1024;
constexpr uint32_t A_STAGE_BYTES = 8 * 512;
constexpr uint32_t S_STAGE_BYTES = 8 * 64;
constexpr long long WAIT_CYCLES = 4000000000ll;   // ~2 s at 2 GHz before a wait gives up

struct TcArgs {
    const char* pool;
    size_t slot_bytes;
    size_t w_off, s_off, ts_off;
    int R, K, E;
    const int32_t* slot_of;
    const int32_t* offsets;
    int pool_slots, rows;
    const int32_t* in_ex;   // power-of-two exponent of each B row (token)
    float* out_h;           // phase 1: h [rows][R/2] fp32
    uint16_t* out_y;        // phase 2: y [rows][R] bf16
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
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

// Bounded wait: suspending try_wait in a loop; after every try it checks the
// CTA's abort flag and the clock, and after WAIT_CYCLES it records
// MOE_ERR_TIMEOUT and raises the abort flag so the other roles drain too.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag)
{
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_suspend(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_CYCLES) break;
    }
    *abort_flag = 1;
    atomicCAS(&g_tc_error, 0, (int)MOE_ERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
                 ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0),
                 "r"(0)
                 : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                 "%12, %13, %14, %15, %16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                 "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                 "r"(v[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                 "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
                 "[%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                   "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                   "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                   "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                   "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: kind::f16, f16 A and B (K-major), fp32 D, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16(int n)
{
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void e2m1x4_to_f16x2(uint32_t w, uint32_t (&f)[4])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(f[0]), "=r"(f[1]), "=r"(f[2]), "=r"(f[3])
        : "r"(w));
}

// f16x2 of E2M1 values times the f16x2 block scale m2: exact, since E2M1 x
// scale has at most 6 significant bits and stays in the f16 normal range
// (MXFP4 scale codes 114..140, any finite E4M3 scale).
__device__ __forceinline__ uint32_t to_f16x2_scaled(uint32_t f, uint32_t m2)
{
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(f), "r"(m2));
    return r;
}

// f16 bits of the block scale of code c.
__device__ uint16_t scale_mult(int wfmt, int c)
{
    if (wfmt == MOE_W_MXFP4) {
        int e = c - 112;                       // 2^(c-127) as f16: exponent field c-127+15
        e = e < 1 ? 1 : (e > 30 ? 30 : e);     // codes outside 114..140 are rejected at packing
        return (uint16_t)(e << 10);
    }
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    float v = (e == 0) ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    __half h = __float2half_rn(s ? -v : v);
    return *reinterpret_cast<uint16_t*>(&h);
}

struct Tile {
    int e, rb, row0, nrows, bn;
    int ncps;   // 64-column chunks of the token block per B stage
};

__device__ __forceinline__ Tile tile_of(int u, const int* prefix, int E, int RB, const int32_t* offsets)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    Tile t;
    t.e = lo;
    int local = u - prefix[lo];
    int tb = local / RB;
    t.rb = local % RB;
    int m = offsets[lo + 1] - offsets[lo];
    int nblk = (m + BN_MAX - 1) / BN_MAX;
    int bs = (((m + nblk - 1) / nblk) + 15) & ~15;
    t.row0 = offsets[lo] + tb * bs;
    t.nrows = max(0, min(bs, m - tb * bs));
    t.bn = max(16, (t.nrows + 15) & ~15);
    t.ncps = min(8, (int)(B_STAGE_BYTES / (t.bn * 128)));
    return t;
}

// Token-row tensor maps with boxes of 16, 32, 64 and 128 rows (64 columns):
// a block of bn rows is loaded with at most four boxes.
struct RowMaps {
    CUtensorMap m[4];
};

template <int WFMT, int PHASE>
__global__ void __launch_bounds__(THREADS, 1)
    ffn_tc_kernel(TcArgs a, const __grid_constant__ RowMaps maps)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sB = smem;                                   // SB x 32 KB, 1024-aligned
    unsigned char* sA = sB + SB * B_STAGE_BYTES;                // SA x 4 KB
    unsigned char* sS = sA + SA * A_STAGE_BYTES;                // SA x 512 B
    uint64_t* bars = reinterpret_cast<uint64_t*>(sS + SA * S_STAGE_BYTES);
    uint64_t* full_a = bars;
    uint64_t* empty_a = full_a + SA;
    uint64_t* full_b = empty_a + SA;
    uint64_t* empty_b = full_b + SB;
    uint64_t* a_ready = empty_b + SB;
    uint64_t* a_free = a_ready + NABUF;
    uint64_t* d_full = a_free + NABUF;   // [2]
    uint64_t* d_empty = d_full + 2;      // [2]
    uint64_t* fin = d_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    uint16_t* s_mult = reinterpret_cast<uint16_t*>(abort_flag + 1);   // [256]
    int* prefix = reinterpret_cast<int*>(s_mult + 256);              // [E+1]
    __shared__ int s_warp[THREADS / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, RB = a.R / BM, KT = a.K / BK;
    constexpr int STILE = (WFMT == MOE_W_MXFP4) ? 32 : 64;

    // ---- set-up: tables, barriers, tensor memory
    for (int c = tid; c < 256; c += THREADS) s_mult[c] = scale_mult(WFMT, c);
    {
        const int EPT = (E + THREADS - 1) / THREADS;
        int loc = 0;
        for (int e = tid * EPT; e < tid * EPT + EPT && e < E; e++) {
            int m = a.offsets[e + 1] - a.offsets[e];
            int sl = a.slot_of[e];
            bool ok = m > 0 && sl >= 0 && sl < a.pool_slots && a.offsets[e] >= 0 && a.offsets[e + 1] <= a.rows;
            int u = ok ? RB * ((m + BN_MAX - 1) / BN_MAX) : 0;
            prefix[e] = u;
            loc += u;
        }
        int inc = loc;
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) s_warp[warp] = inc;
        __syncthreads();
        int run = inc - loc;
        for (int w = 0; w < warp; w++) run += s_warp[w];
        for (int e = tid * EPT; e < tid * EPT + EPT && e < E; e++) {
            int u = prefix[e];
            prefix[e] = run;
            run += u;
        }
        if (tid == THREADS - 1) prefix[E] = run;
    }
    if (tid == 0) {
        for (int i = 0; i < SA; i++) {
            mbar_init(smem_u32(&full_a[i]), 1);
            mbar_init(smem_u32(&empty_a[i]), NXW / NXG);
        }
        for (int i = 0; i < SB; i++) {
            mbar_init(smem_u32(&full_b[i]), 1);
            mbar_init(smem_u32(&empty_b[i]), 1);
        }
        for (int i = 0; i < NABUF; i++) {
            mbar_init(smem_u32(&a_ready[i]), 32 * NXW / NXG);
            mbar_init(smem_u32(&a_free[i]), 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(smem_u32(&d_full[i]), 1);
            mbar_init(smem_u32(&d_empty[i]), 32 * NEPI);
        }
        mbar_init(smem_u32(fin), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = prefix[E];
    volatile int* abort_v = abort_flag;

    if (warp == 0) {
        // ================= weight copy issue (one thread) =================
        if (lane == 0) {
            int sa = 0;
            uint32_t pa = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                Tile t = tile_of(u, prefix, E, RB, a.offsets);
                const char* blob = a.pool + (size_t)a.slot_of[t.e] * a.slot_bytes;
                const int RT = a.R / 16;
                for (int c = 0; c < KT && ok; c++) {
                    ok = mbar_wait(smem_u32(&empty_a[sa]), pa ^ 1, abort_v);
                    if (!ok) break;
                    const uint32_t fa = smem_u32(&full_a[sa]);
                    const size_t ti = tile_index(8 * t.rb, c, RT, KT);   // 8 contiguous row tiles
                    mbar_expect_tx(fa, A_STAGE_BYTES + 8 * STILE);
                    bulk_g2s(smem_u32(sA + sa * A_STAGE_BYTES), blob + a.w_off + ti * 512, A_STAGE_BYTES, fa);
                    bulk_g2s(smem_u32(sS + sa * S_STAGE_BYTES), blob + a.s_off + ti * STILE, 8 * STILE, fa);
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                }
            }
            // drain: every stage's most recent fill must land before the CTA exits
            // (stage i was last filled in the current round if i < next stage, else in the
            // previous one; a stage never filled reads as complete for the previous parity)
            for (int i = 0; i < SA; i++) mbar_wait(smem_u32(&full_a[i]), (i < sa) ? pa : (pa ^ 1), abort_v);
        }
    } else if (warp == BWARP) {
        // ================= token copy issue (one thread) =================
        if (lane == 0) {
            int sb = 0;
            uint32_t pb = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                Tile t = tile_of(u, prefix, E, RB, a.offsets);
                for (int c = 0; c < KT && ok; c += t.ncps) {
                    ok = mbar_wait(smem_u32(&empty_b[sb]), pb ^ 1, abort_v);
                    if (!ok) break;
                    const uint32_t fb = smem_u32(&full_b[sb]);
                    const int nch = min(t.ncps, KT - c);
                    mbar_expect_tx(fb, (uint32_t)(nch * t.bn * 128));
                    for (int j = 0; j < nch; j++) {
                        const uint32_t dst = smem_u32(sB + sb * B_STAGE_BYTES + j * t.bn * 128);
                        int done = 0;
#pragma unroll
                        for (int mi = 3; mi >= 0; mi--) {
                            const int box = 16 << mi;
                            while (t.bn - done >= box) {
                                tma_load_2d(dst + done * 128, &maps.m[mi], (c + j) * BK, t.row0 + done, fb);
                                done += box;
                            }
                        }
                    }
                    if (++sb == SB) { sb = 0; pb ^= 1; }
                }
            }
            for (int i = 0; i < SB; i++) mbar_wait(smem_u32(&full_b[i]), (i < sb) ? pb : (pb ^ 1), abort_v);
        }
    } else if (warp == 1) {
        // ================= MMA issue (one thread) =================
        if (lane == 0) {
            int sb = 0, ab = 0, it = 0;
            uint32_t pb = 0, pab = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x, it++) {
                Tile t = tile_of(u, prefix, E, RB, a.offsets);
                const int db = it & 1;   // accumulator of this tile
                if (it >= 2) {           // its previous tile's epilogue is done
                    ok = mbar_wait(smem_u32(&d_empty[db]), ((it >> 1) - 1) & 1, abort_v);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t idesc = idesc_f16(t.bn);
                for (int c = 0; c < KT && ok; c++) {
                    const int j = c % t.ncps;   // chunk inside the B stage
                    if (j == 0) ok = mbar_wait(smem_u32(&full_b[sb]), pb, abort_v);
                    ok = ok && mbar_wait(smem_u32(&a_ready[ab]), pab, abort_v);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t bbase = smem_u32(sB + sb * B_STAGE_BYTES + j * t.bn * 128);
#pragma unroll
                    for (int k = 0; k < BK / 16; k++)
                        tc_mma_ts(tmem + D_COL + BN_MAX * db, tmem + A_COL + 32 * ab + 8 * k, smem_desc_sw128(bbase + 32 * k), idesc,
                                  (c | k) != 0);
                    tc_commit(smem_u32(&a_free[ab]));
                    if (j == t.ncps - 1 || c == KT - 1) {   // the stage's last chunk
                        tc_commit(smem_u32(&empty_b[sb]));
                        if (++sb == SB) { sb = 0; pb ^= 1; }
                    }
                    if (++ab == NABUF) { ab = 0; pab ^= 1; }
                }
                if (ok) tc_commit(smem_u32(&d_full[db]));
            }
            // every MMA issued by this thread completes before tensor memory is released
            tc_commit(smem_u32(fin));
            mbar_wait(smem_u32(fin), 0, abort_v);
        }
    } else if (warp < 2 + NXW) {
        // ================= expand FP4 -> tensor memory =================
        // Per group, two warps per tensor-memory lane quarter: set 0 expands
        // bytes 0..3 of each lane segment (columns 0..15 of the chunk), set 1
        // bytes 4..7 (columns 16..31).  Group g takes the chunks whose running
        // index is g mod NXG.
        const int xw = warp - 2;
        const int q = warp & 3;                 // tensor-memory lane quarter of this warp
        const int set = (xw >> 2) & 1;          // 0 or 1
        const int grp = xw >> 3;                // 0 .. NXG-1
        const int r = 32 * q + lane;            // weight row inside the 128-row block
        const int rtl = r >> 4, rr = r & 15, g = rr & 7, half = rr >> 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int pend = -1;           // buffer whose tensor-memory store is in flight
        long ci = 0;             // running chunk index over this CTA's tiles
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            for (int c = 0; c < KT && ok; c++, ci++) {
                if ((int)(ci % NXG) != grp) continue;
                const int sa = (int)(ci % SA), ab = (int)(ci % NABUF);
                const uint32_t pa = (uint32_t)(ci / SA) & 1, pab = (uint32_t)(ci / NABUF) & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full_a[sa]), pa, abort_v));
                if (!ok) break;
                const unsigned char* arow = sA + sa * A_STAGE_BYTES + rtl * 512 + 64 * g + 8 * half + 4 * set;
                const unsigned char* srow = sS + sa * S_STAGE_BYTES + rtl * STILE;
                uint32_t q4[4];
#pragma unroll
                for (int tt = 0; tt < 4; tt++) q4[tt] = *reinterpret_cast<const uint32_t*>(arow + 16 * tt);
                // byte p of lane segment tt is the row's byte 4p+tt (tensor-memory column 4p+tt):
                // MXFP4 block = column/16 (= set), NVFP4 block = column/8 (= 2*set + p/2)
                uint32_t m0, m1;
                if (WFMT == MOE_W_MXFP4) {
                    m0 = s_mult[srow[4 * g + 2 * half + set]];
                    m1 = m0;
                } else {
                    m0 = s_mult[srow[8 * g + 4 * half + 2 * set]];
                    m1 = s_mult[srow[8 * g + 4 * half + 2 * set + 1]];
                }
                m0 |= m0 << 16;
                m1 |= m1 << 16;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_a[sa]));
                uint32_t v[16];
#pragma unroll
                for (int tt = 0; tt < 4; tt++) {
                    uint32_t f[4];
                    e2m1x4_to_f16x2(q4[tt], f);
#pragma unroll
                    for (int b = 0; b < 4; b++) v[4 * b + tt] = to_f16x2_scaled(f[b], b < 2 ? m0 : m1);
                }
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&a_free[ab]), pab ^ 1, abort_v));
                if (!ok) break;
                // the previous chunk's store has run while this chunk was expanded:
                // complete it and hand that buffer to the MMA
                if (pend >= 0) {
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(smem_u32(&a_ready[pend]));
                }
                tc_fence_after();
                tmem_st16(tmem + lane_base + A_COL + 32 * ab + 16 * set, v);
                pend = ab;
            }
            if (pend >= 0) {   // the tile's last chunk
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&a_ready[pend]));
                pend = -1;
            }
        }
    } else if (warp < BWARP) {
        // ================= epilogue: accumulator -> h or y =================
        // One warp per tensor-memory lane quarter; tile `it` used accumulator
        // it & 1, so this runs while the next tile is multiplied.
        const int q = warp & 3;
        const int r = 32 * q + lane;            // weight row inside the 128-row block
        const int rtl = r >> 4, rr = r & 15, g = rr & 7, half = rr >> 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int it = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x, it++) {
            const Tile t = tile_of(u, prefix, E, RB, a.offsets);
            const int db = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&d_full[db]), (it >> 1) & 1, abort_v))) break;
            tc_fence_after();
            const char* blob = a.pool + (size_t)a.slot_of[t.e] * a.slot_bytes;
            float tsc = 1.0f;
            if (WFMT == MOE_W_NVFP4) tsc = reinterpret_cast<const float*>(blob + a.ts_off)[PHASE - 1];
            for (int c0 = 0; c0 < t.bn; c0 += 32) {
                uint32_t d[32];
                tmem_ld32(tmem + lane_base + D_COL + BN_MAX * db + c0, d);
                // lane j holds the scale of token column c0 + j (row exponent, NVFP4 tensor scale)
                const int nl = c0 + lane;
                const float ul = (nl < t.nrows) ? tsc * pow2i(-__ldg(a.in_ex + t.row0 + nl)) : 0.0f;
                tmem_wait_ld();
                if (PHASE == 1) {
                    const int F = a.R / 2;
                    const int f = 64 * t.rb + 8 * rtl + g;
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int n = c0 + j;
                        const float x = __uint_as_float(d[j]) * __shfl_sync(0xffffffffu, ul, j);
                        const float up = __shfl_down_sync(0xffffffffu, x, 8);
                        if (half == 0 && n < t.nrows)
                            a.out_h[(size_t)(t.row0 + n) * F + f] = x / (1.0f + __expf(-x)) * up;
                    }
                } else {
                    const int Ho = a.R;
                    const int o = BM * t.rb + r;
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int n = c0 + j;
                        const float u = __shfl_sync(0xffffffffu, ul, j);
                        if (n < t.nrows)
                            a.out_y[(size_t)(t.row0 + n) * Ho + o] = f32_to_bf16_bits(__uint_as_float(d[j]) * u);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&d_empty[db]));
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows][cols] f16, boxes of box_rows rows x 64 columns, 128-byte swizzle.
int make_rows_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MOE_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

int make_row_maps(RowMaps* rm, const void* base, int rows, int cols)
{
    for (int i = 0; i < 4; i++) {
        int rc = make_rows_map(&rm->m[i], base, rows, cols, 16 << i);
        if (rc) return rc;
    }
    return MOE_OK;
}

size_t tc_smem_bytes(int E)
{
    return 1024 + SB * B_STAGE_BYTES + SA * A_STAGE_BYTES + SA * S_STAGE_BYTES + 8 * (2 * SA + 2 * SB + 2 * NABUF + 5) +
           8 + 2 * 256 + 4 * (size_t)(E + 1) + 64;
}

template <int WFMT, int PHASE>
int launch_one(const TcArgs& a, const RowMaps& map, int rows, int sms, cudaStream_t st)
{
    size_t smem = tc_smem_bytes(a.E);
    int dev = 0;   // the attribute is per device (context)
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    static size_t attr_smem_dev[kMaxDevices];
    size_t& attr_smem = attr_smem_dev[dev];
    if (smem > attr_smem) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_tc_kernel<WFMT, PHASE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem));
        attr_smem = smem;
    }
    long RB = a.R / BM;
    long active = rows < a.E ? rows : a.E;
    long bound = RB * (active + rows / BN_MAX + 1);
    int grid = (int)(bound < sms ? bound : sms);
    if (grid < 1) grid = 1;
    ffn_tc_kernel<WFMT, PHASE><<<grid, THREADS, smem, st>>>(a, map);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace

bool ffn_tc_supported(const moe_shape* s)
{
    return (s->wfmt == MOE_W_MXFP4 || s->wfmt == MOE_W_NVFP4) && (2 * s->ffn) % BM == 0 && s->hidden % BM == 0 &&
           tc_smem_bytes(s->experts) <= 227 * 1024;
}

int launch_ffn_tc(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
                  const int32_t* offsets, int rows, uint16_t* y_perm, const TcOperands& op, cudaStream_t st,
                  const std::function<int()>& between)
{
    BlobLayout bl = blob_layout(s);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    RowMaps mx, mh;
    int rc;
    if ((rc = make_row_maps(&mx, op.x16, rows, s->hidden))) return rc;
    if ((rc = make_row_maps(&mh, op.h16, rows, s->ffn))) return rc;
    TcArgs a1{};
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
    a1.in_ex = op.xe;
    a1.out_h = op.h32;
    TcArgs a2 = a1;
    a2.w_off = bl.w2;
    a2.s_off = bl.s2;
    a2.R = s->hidden;
    a2.K = s->ffn;
    a2.in_ex = op.he;
    a2.out_h = nullptr;
    a2.out_y = y_perm;
    if (s->wfmt == MOE_W_MXFP4) {
        if ((rc = launch_one<MOE_W_MXFP4, 1>(a1, mx, rows, sms, st))) return rc;
        if ((rc = between())) return rc;
        return launch_one<MOE_W_MXFP4, 2>(a2, mh, rows, sms, st);
    }
    if ((rc = launch_one<MOE_W_NVFP4, 1>(a1, mx, rows, sms, st))) return rc;
    if ((rc = between())) return rc;
    return launch_one<MOE_W_NVFP4, 2>(a2, mh, rows, sms, st);
}

}  // namespace moe

extern "C" int moe_get_device_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, moe::g_tc_error, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    if (clear && v) {
        int z = 0;
        if (cudaMemcpyToSymbol(moe::g_tc_error, &z, sizeof z) != cudaSuccess) return MOE_ERR_CUDA;
    }
    const int d = moe::ffn_device_error(clear);
    return v ? v : d;
}
