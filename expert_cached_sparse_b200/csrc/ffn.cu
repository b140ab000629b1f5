// Grouped SwiGLU expert FFN over permuted rows for BF16 expert weights,
// streamed from the expert slots.  Experts found in the GPU cache are
// executed on the GPU ("FreeToken quantization", section "Como se desplazan
// los pesos MoE cuantizados por la memoria").  FP4 weights (MXFP4, NVFP4) go
// to the block-scaled tensor-core kernels of ffn_fp4.cu.
//
// The BF16 layers are bound by HBM: each touched expert's weights are read
// once per pass and every token row is reused across all of them.  Design:
//  - work unit = (token group of up to 16 rows of one expert, 128-row block
//    of W13 or W2), over the whole K; a persistent grid of three CTAs per SM
//    walks the units (round-robin, or stream-K ranges when there are fewer
//    units than CTAs, see the kernel);
//  - per CTA, one lane streams the units through a shared-memory ring with
//    1-D bulk copies (TMA engine) completed on mbarriers: a stage is one
//    64-column chunk of the block (eight 2 KB tiles, contiguous in the slot)
//    and the group's activation rows of that chunk; eight compute warps each
//    own one 16-row tile of the block;
//  - weights are the mma.sync m16n8k16 row operand: a lane's 16 bytes of a
//    packed tile per k16 step are exactly its fragment words;
//  - the activations (x gathered by token, then h) are first rewritten once
//    per call into a bf16 operand copy stored column-block-major
//    ([64-column block][row]) so any 8 consecutive rows of a block are one
//    contiguous 1 KB copy, permuted and swizzled inside each 128-byte row so
//    a lane's fragment data for four k16 steps is two conflict-free 16-byte
//    reads;
//  - phase 1 tiles pair 8 gate rows with the 8 matching up rows, so the
//    SwiGLU epilogue is lane-local: h = silu(gate) * up in fp32.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

namespace moe {

__device__ int g_ffn_error;   // first device-side error of the BF16 streaming FFN (0: none)

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
    float* h32;       // [rows][F] h in fp32
    uint16_t* hb;     // [F/64][rows+16][64] operand copy of h
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
    size_t oh = take(4 * R * s->ffn);
    size_t ohb = take(2 * RP * s->ffn);
    size_t og = take(4 * (size_t)(s->experts + 1));
    const long ncnt = dec_units_max(s, (int)R);
    size_t oc = take(4 * (size_t)ncnt);
    size_t op = take(4 * (size_t)kMaxDecCtas * 2 * kPieceFloats);
    if (w) {
        char* b = static_cast<char*>(base);
        w->xb = reinterpret_cast<uint16_t*>(b + oxb);
        w->h32 = reinterpret_cast<float*>(b + oh);
        w->hb = reinterpret_cast<uint16_t*>(b + ohb);
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
// bf16 operand copy of a bf16 or fp32 row (read directly, or token
// gather[r]/gk of the source).  With `groups` set, the last CTA writes the
// per-expert token-group prefix and clears `zero`.
template <bool IN_F32>
__global__ void __launch_bounds__(kPrepThreads) ffn_prep_kernel(const void* __restrict__ in, int rows, int K,
                                                                uint16_t* __restrict__ out,
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
    const int RP = rows + kRowPad;
    const int nblocks = gridDim.x - (groups ? 1 : 0);
    const int nch = K / 8;   // 8-element chunks per row
    for (int r = blockIdx.x; r < rows; r += nblocks) {
        const size_t sr = gather ? (size_t)(__ldg(gather + r) / gk) : (size_t)r;   // source row
        const float* inf = static_cast<const float*>(in) + sr * K;
        const uint16_t* inb = static_cast<const uint16_t*>(in) + sr * K;
        // two adjacent source columns (col even) as a bf16 pair
        auto pair = [&](int col) -> uint32_t {
            if (IN_F32) {
                const float2 v = __ldg(reinterpret_cast<const float2*>(inf + col));
                return (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
            }
            return __ldg(reinterpret_cast<const uint32_t*>(inb + col));
        };
        for (int c = threadIdx.x; c < nch; c += kPrepThreads) {
            // output chunk cc of 64-column block kt holds, for j = 2(cc&1) + jj
            // and t = cc/2, the pairs at columns 16j + 8h + 2t (element 4jj + 2h)
            const int kt = c >> 3, cc = c & 7, t = cc >> 1, jb = 2 * (cc & 1);
            const int base = 64 * kt + 16 * jb + 2 * t;
            const uint4 o = make_uint4(pair(base), pair(base + 8), pair(base + 16), pair(base + 24));
            *reinterpret_cast<uint4*>(out + ((size_t)kt * RP + r) * 64 + (size_t)((cc ^ (r & 7)) * 8)) = o;
        }
    }
}

// ------------------------------------------------------------------ GEMM units
struct FfnArgs {
    const char* pool;
    size_t slot_bytes;
    size_t w_off;
    int R, K, E;
    const int32_t* slot_of;
    const int32_t* offsets;
    const int32_t* groups;
    int rows;
    const uint16_t* in;     // operand copy [K/64][rows+16][64]
    float* out_h;           // phase 1: h [rows][R/2] fp32
    uint16_t* out_y;        // phase 2: y [rows][R] bf16
    int32_t* cnt;           // per unit: pieces finished (units split across CTAs)
    float* pieces;          // [gridDim.x][2][kPieceFloats]
    long long wait;         // limit of the bounded waits of the copy lane and the compute warps
    int withhold;           // testing: CTA 0 leaves its first ring stage unfilled
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

// Bounded wait (`limit` cycles, about 2 s by default), false on timeout.
// With `abort` set the wait also gives up as soon as another warp of the CTA
// has raised it, and raises it itself on a timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort = nullptr,
                                                  long long limit = kWaitCycles)
{
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_suspend(bar, parity)) return true;
        if (abort && *abort) return false;
        if (clock64() - t0 > limit) {
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

__device__ __forceinline__ void mma16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// ---- CTA-cooperative weight streaming -------------------------------------
// Work is a list of units (token group of one expert, 128-row block of W),
// each KP = K/64 stages of one 64-column chunk long.  With at least as many
// units as CTAs, CTAs take whole units round-robin.  Otherwise the
// concatenated stage list is cut into equal ranges over the CTAs (stream-K):
// a CTA runs whole units where its range covers them and pieces of the units
// at its range ends.  A piece's partial sums go to a per-CTA buffer; the CTA
// that finishes a unit's last piece adds all pieces in CTA order
// (deterministic) and writes the result.
// Inside a CTA, warp 8 (one lane) fills a ring stage with bulk copies: the
// block's bf16 tiles of the chunk (contiguous in the slot) and the token
// group's 8 or 16 activation rows of the chunk.  Warps 0..7 each multiply the
// 16-row tile they own and then release the stage on an mbarrier.
constexpr int kDecThreads = 32 * (kCW + 1);   // + one copy-issue warp
constexpr int kTile = 2048;                   // 16 x 64 bf16
constexpr int kRing = 4;                      // ring stages
constexpr int kABytes = kCW * kTile;
constexpr int kXChunk = 2 * 1024;             // up to 16 rows x 128 bytes
constexpr int kStage = kABytes + kXChunk;

size_t dec_smem_bytes(int E) { return 1024 + (size_t)kRing * kStage + 4 * (size_t)(E + 1); }

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

// Multiply-accumulate of one 16-row x 64-column tile: w[j] = {a0, a2, a1, a3}
// of k16 step j; X = the token rows' fragment words of the four steps.
template <int NQ>
__device__ __forceinline__ void mma_tile(float (&acc)[2][4], const unsigned char* sg, int ng, int w, int lane,
                                         int g, int t, int sw)
{
    uint4 wv[4];
    const unsigned char* wt = sg + w * kTile + 16 * lane;
#pragma unroll
    for (int v = 0; v < 4; v++) wv[v] = *reinterpret_cast<const uint4*>(wt + v * 512);
#pragma unroll
    for (int q = 0; q < NQ; q++) {
        const unsigned char* xrow = sg + kABytes + q * 1024 + g * 128;
        const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + (((2 * t) ^ sw) << 4));
        const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + (((2 * t + 1) ^ sw) << 4));
        const uint32_t X[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int j = 0; j < 4; j++)
            mma16816_bf16(acc[q], wv[j].x, wv[j].z, wv[j].y, wv[j].w, X[2 * j], X[2 * j + 1]);
    }
}

// Ring position shared by the compute warps.
struct Ring {
    int st;
    uint32_t ph;
    __device__ __forceinline__ void next()
    {
        if (++st == kRing) { st = 0; ph ^= 1; }
    }
};

// One unit's stages for a compute warp: wait, multiply its tile, release.
// Returns false when a wait gave up.
template <int NQ>
__device__ __forceinline__ bool run_unit(float (&acc)[2][4], const DecUnit& U, bool act, Ring& R,
                                         unsigned char* ring, uint64_t* full, uint64_t* empty, int w, int lane,
                                         volatile int* abort, long long limit)
{
    const int g = lane >> 2, t = lane & 3, sw = (U.row0 + g) & 7;
    for (int kt = U.k0; kt < U.k1; kt++) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&full[R.st]), R.ph, abort, limit))) return false;
        const unsigned char* sg = ring + (size_t)R.st * kStage;
        if (act) mma_tile<NQ>(acc, sg, U.ng, w, lane, g, t, sw);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[R.st]));
        R.next();
    }
    return true;
}

// Final values of a warp's tile: h = silu(gate) * up (phase 1) or y in bf16.
template <int PHASE>
__device__ __forceinline__ void write_tile(const FfnArgs& a, const DecUnit& U, int rt, const float (&acc)[2][4],
                                           int g, int t)
{
#pragma unroll
    for (int q = 0; q < 2; q++) {
        if (q >= U.nq) break;
        const int r0 = U.row0 + q * 8 + 2 * t, r1 = r0 + 1;
        if (PHASE == 1) {
            const int F = a.R / 2;
            const int f = 8 * rt + g;
            if (r0 < U.row_end) a.out_h[(size_t)r0 * F + f] = silu(acc[q][0]) * acc[q][2];
            if (r1 < U.row_end) a.out_h[(size_t)r1 * F + f] = silu(acc[q][1]) * acc[q][3];
        } else {
            const int Ho = a.R;
            const int o = 16 * rt + g;
            if (r0 < U.row_end) {
                a.out_y[(size_t)r0 * Ho + o] = f32_to_bf16_bits(acc[q][0]);
                a.out_y[(size_t)r0 * Ho + o + 8] = f32_to_bf16_bits(acc[q][2]);
            }
            if (r1 < U.row_end) {
                a.out_y[(size_t)r1 * Ho + o] = f32_to_bf16_bits(acc[q][1]);
                a.out_y[(size_t)r1 * Ho + o + 8] = f32_to_bf16_bits(acc[q][3]);
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

template <int PHASE>
__global__ void __launch_bounds__(kDecThreads, 3) ffn_kernel(FfnArgs a)
{
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);            // [kRing]
    uint64_t* empty = full + kRing;                                 // [kRing]
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + 512);
    volatile int* s_last = reinterpret_cast<volatile int*>(smem + 516);
    unsigned char* ring = smem + 1024;
    int* s_groups = reinterpret_cast<int*>(ring + (size_t)kRing * kStage);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
    const int RT = a.R / 16, RB = (RT + 7) / 8, KP = a.K / 64, RP = a.rows + kRowPad;
    pdl_wait();
    for (int i = tid; i <= a.E; i += kDecThreads) s_groups[i] = a.groups[i];
    if (tid == 0) {
        for (int i = 0; i < kRing; i++) {
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
            int withheld = -1;   // testing: the stage left unfilled
            auto issue = [&](const DecUnit& U) {
                for (int kt = U.k0; kt < U.k1 && ok; kt++) {
                    if (!(ok = mbar_wait_bounded(smem_u32(&empty[st]), ph ^ 1, s_abort, a.wait))) break;
                    const uint32_t bar = smem_u32(&full[st]);
                    unsigned char* sg = ring + (size_t)st * kStage;
                    const size_t ti = tile_index(8 * U.G, kt, RT, KP);
                    const uint32_t bytes = U.ng * kTile + U.nq * 1024;
                    if (a.withhold && blockIdx.x == 0 && issued == 0) {
                        withheld = st;   // never filled, so the compute warps' wait for it runs out
                    } else {
                        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                                     : "memory");
                        bulk_copy(smem_u32(sg), U.blob + a.w_off + ti * kTile, U.ng * kTile, bar);
                        bulk_copy(smem_u32(sg + kABytes), a.in + ((size_t)kt * RP + U.row0) * 64, U.nq * 1024, bar);
                    }
                    issued++;
                    if (++st == kRing) { st = 0; ph ^= 1; }
                }
            };
            Seg sg{whole ? (long)blockIdx.x : b0};
            while (ok && sg.next(whole, NU, KP, b1))
                issue(dec_unit(a, s_groups, sg.u, RT, RB, sg.p0, sg.p1));
            if (!ok) atomicCAS(&g_ffn_error, 0, (int)MOE_ERR_TIMEOUT);
            // let the last copies land before the CTA exits (stage i was last
            // filled in this pass if i < st, else in the previous one; a
            // withheld stage is never refilled: its consumers give up first)
            for (int i = 0; i < kRing && i < issued; i++)
                if (i != withheld) mbar_wait_bounded(smem_u32(&full[i]), i < st ? ph : (ph ^ 1));
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
            ok = U.nq == 1 ? run_unit<1>(acc, U, w < U.ng, R, ring, full, empty, w, lane, s_abort, a.wait)
                           : run_unit<2>(acc, U, w < U.ng, R, ring, full, empty, w, lane, s_abort, a.wait);
    };
    Seg sg{whole ? (long)blockIdx.x : b0};
    while (sg.next(whole, NU, KP, b1)) {
        const int u = sg.u, p0 = sg.p0, p1 = sg.p1;
        const long idx = sg.start;
        const DecUnit U = dec_unit(a, s_groups, u, RT, RB, p0, p1);
        const bool act = w < U.ng;          // this warp has a row tile in the block
        const int rt = 8 * U.G + w;
        float acc[2][4];
        multiply(U, acc);
        if (p0 == 0 && p1 == KP) {
            if (ok && act) write_tile<PHASE>(a, U, rt, acc, g, t);
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
                    write_tile<PHASE>(a, U, rt, sum, g, t);
                }
                if (tid == 0) a.cnt[u] = 0;
            }
            compute_bar();   // s_last is rewritten by the next piece
        }
    }
    if (!ok && lane == 0) atomicCAS(&g_ffn_error, 0, (int)MOE_ERR_TIMEOUT);
}

int launch_bf16(const moe_shape* s, const BlobLayout& bl, const void* pool, size_t slot_bytes, int pool_slots,
                const int32_t* slot_of, const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm,
                const FfnWs& w, int sms, cudaStream_t st, const RowSource* gather)
{
    const int E = s->experts, H = s->hidden, F = s->ffn;
    int prep_blocks = rows < sms * 8 ? rows : sms * 8;   // a CTA per row
    const void* src = gather ? gather->x : static_cast<const void*>(x_perm);
    const int32_t* gidx = gather ? gather->assign_of : nullptr;
    const int gk = gather ? gather->k : 1;
    if (gather && gather->x_dtype == MOE_DT_F32)
        MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<true>, prep_blocks + 1, kPrepThreads, 0, st, src, rows, H, w.xb,
                                offsets, slot_of, E, pool_slots, w.groups, gidx, gk, w.cnt, w.ncnt));
    else
        MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<false>, prep_blocks + 1, kPrepThreads, 0, st, src, rows, H, w.xb,
                                offsets, slot_of, E, pool_slots, w.groups, gidx, gk, w.cnt, w.ncnt));
    FfnArgs a{};
    a.pool = static_cast<const char*>(pool);
    a.slot_bytes = slot_bytes;
    a.E = E;
    a.slot_of = slot_of;
    a.offsets = offsets;
    a.groups = w.groups;
    a.rows = rows;
    a.cnt = w.cnt;
    a.pieces = w.pieces;
    a.wait = test_wait_cycles(kWaitCycles);
    a.withhold = test_withhold();
    const size_t smem = dec_smem_bytes(E);
    // persistent grid: as many CTAs as fit at once (recomputed when the
    // shared-memory size, which grows with E, changes); function attributes
    // and occupancy are per device (context)
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    static size_t attr_smem_dev[kMaxDevices], occ_smem_dev[kMaxDevices];
    static int resident_dev[kMaxDevices];
    size_t& attr_smem = attr_smem_dev[dev];
    size_t& occ_smem = occ_smem_dev[dev];
    int& resident = resident_dev[dev];
    if (smem > attr_smem) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        // several CTAs share an SM: take the largest shared-memory split
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<1>, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_kernel<2>, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        attr_smem = smem;
    }
    if (smem != occ_smem) {
        MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, ffn_kernel<1>, kDecThreads, smem));
        if (resident < 1) resident = 1;
        occ_smem = smem;
    }
    long grid = (long)sms * resident;
    if (grid > kMaxDecCtas) grid = kMaxDecCtas;
    // no more CTAs than stages (upper bound of the stage count: every unit possible)
    auto grid_for = [&](int R, int K) {
        const long RB = (R / 16 + 7) / 8, KP = K / 64;
        const long groups = (rows + kRowsPerUnit - 1) / kRowsPerUnit + (rows < E ? rows : E);
        const long wmax = groups * RB * KP;
        return (int)(wmax < grid ? (wmax < 1 ? 1 : wmax) : grid);
    };
    a.w_off = bl.w13;
    a.R = 2 * F;
    a.K = H;
    a.in = w.xb;
    a.out_h = w.h32;
    MOE_CUDA_TRY(launch_pdl(ffn_kernel<1>, grid_for(2 * F, H), kDecThreads, smem, st, a));
    MOE_CUDA_TRY(launch_pdl(ffn_prep_kernel<true>, prep_blocks, kPrepThreads, 0, st,
                            static_cast<const void*>(w.h32), rows, F, w.hb, nullptr, nullptr, E, 0, nullptr, nullptr,
                            1, nullptr, 0));
    FfnArgs b = a;
    b.w_off = bl.w2;
    b.R = H;
    b.K = F;
    b.in = w.hb;
    b.out_h = nullptr;
    b.out_y = y_perm;
    MOE_CUDA_TRY(launch_pdl(ffn_kernel<2>, grid_for(H, F), kDecThreads, smem, st, b));
    return MOE_OK;
}

}  // namespace

size_t ffn_ws_bytes(const moe_shape* s, int rows)
{
    if (s->wfmt != MOE_W_BF16) return ffn_fp4_ws_bytes(s, rows);
    return ffn_ws_layout(s, rows, nullptr, nullptr) + 256;
}

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
               cudaStream_t st, const RowSource* gather, bool one_expert)
{
    if (rows == 0) return MOE_OK;
    ProfScope ps(MOE_PROF_FFN, st);
    if (s->wfmt != MOE_W_BF16)
        return launch_ffn_fp4(s, pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows, y_perm, ws, st, gather,
                              one_expert);
    FfnWs w;
    ffn_ws_layout(s, rows, ws, &w);
    int dev = 0, sms = 148;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    prof_count(MOE_PROF_FFN, 4);
    return launch_bf16(s, blob_layout(s), pool, slot_bytes, pool_slots, slot_of, offsets, x_perm, rows, y_perm, w,
                       sms, st, gather);
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

namespace moe {
namespace {
long long g_test_wait = 0;   // 0: every kernel's default limit
int g_test_withhold = 0;
}  // namespace
long long test_wait_cycles(long long dflt) { return g_test_wait > 0 ? g_test_wait : dflt; }
int test_withhold() { return g_test_withhold; }
}  // namespace moe

extern "C" int moe_test_set_wait(int64_t cycles, int32_t withhold)
{
    if (cycles < 0) return MOE_ERR_INVALID_ARG;
    moe::g_test_wait = cycles;
    moe::g_test_withhold = withhold ? 1 : 0;
    return MOE_OK;
}

extern "C" int moe_get_device_error(int clear)
{
    const int a = moe::ffn_fp4_device_error(clear);
    const int b = moe::ffn_device_error(clear);
    if (a < 0 && a != MOE_ERR_TIMEOUT) return a;   // the read itself failed
    return a ? a : b;
}
