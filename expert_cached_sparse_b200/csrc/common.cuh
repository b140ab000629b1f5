// Internal helpers shared by the libmoe.so translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe.h"

#define MOE_CUDA_TRY(expr)                                  \
    do {                                                    \
        cudaError_t _e = (expr);                            \
        if (_e != cudaSuccess) return MOE_ERR_CUDA;         \
    } while (0)

#define MOE_LAUNCH_CHECK() MOE_CUDA_TRY(cudaGetLastError())

namespace moe {

constexpr int kMaxExperts = 4096;
constexpr int kMaxCapacity = 8192;
constexpr int kMaxTopK = 32;
constexpr int kMaxDevices = 64;   // device ordinals with per-device launch caches

static inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

__host__ __device__ static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static inline bool shape_ok(const moe_shape* s)
{
    if (!s) return false;
    if (s->layers <= 0 || s->experts <= 0 || s->experts > kMaxExperts) return false;
    if ((int64_t)s->layers * s->experts >= 65536) return false;
    if (s->hidden <= 0 || s->hidden % 64 || s->ffn <= 0 || s->ffn % 64) return false;
    if (s->top_k <= 0 || s->top_k > s->experts || s->top_k > kMaxTopK) return false;
    if (s->wfmt < MOE_W_BF16 || s->wfmt > MOE_W_NVFP4) return false;
    // FP4 blobs are stored in 128-row x 256-column chunks
    if (s->wfmt != MOE_W_BF16 && (s->hidden % 256 || s->ffn % 256)) return false;
    return true;
}

// ---------------------------------------------------------------- blob layout
// One packed expert (= one slot); W13 is [2F][H], W2 is [H][F].
//
// BF16 weights: matrices cut into tiles of 16 rows x 64 columns; tile (rt, kt)
// of a [R][K] matrix sits at tile_index(rt, kt).  Inside a tile, lane L = 4g+t
// of a warp owns rows g and g+8: for k16 step j its 16 bytes are the
// mma.sync fragment words {a0, a2, a1, a3} (2048 B per tile).  W13 rows are
// reordered so row tile rt holds gate rows f = 8rt..8rt+7 in its rows 0..7
// and the matching up rows in rows 8..15.  Tiles are stored in row groups of
// 8 row tiles (128 rows): for row group G and column block kt the group's
// tiles are contiguous, so one 128 x 64 block is one contiguous copy.  Index
// of tile (rt, kt) of a matrix with RT row tiles and KT column blocks (the
// last group may hold fewer than 8):
__host__ __device__ static inline size_t tile_index(int rt, int kt, int RT, int KT)
{
    const int G = rt >> 3, w = rt & 7;
    const int ng = (RT - 8 * G) < 8 ? (RT - 8 * G) : 8;
    return (size_t)8 * G * KT + (size_t)kt * ng + w;
}

// FP4 weights (MXFP4: E8M0 scale per 32 columns; NVFP4: E4M3 scale per 16
// columns and one fp32 scale per matrix): each matrix is a sequence of
// chunks, row block G (128 rows) by column chunk c (256 columns), at chunk
// index G * (K / 256) + c, fp4_chunk_bytes apart.  A chunk is
//   16384 B: the 128 rows' 128 bytes of E2M1 codes (two per byte, even
//            column in the low nibble) as the tensor core reads them from
//            shared memory: row r at 1024 (r / 8) + 128 (r % 8), its
//            16-byte piece j stored at piece position j ^ (r % 8);
//   then 256 / 32 / 4 = 2 (MXFP4) or 256 / 16 / 4 = 4 (NVFP4) scale images
//            of 512 B, image i holding scales 4i..4i+3 of each row: scale s
//            of row r at byte 16 (r % 32) + 4 (r / 32) + (s % 4).
// Row r of W2 block G is output row 128 G + r.  Row r of W13 block G, with
// q = r / 32 and i = r % 32, is gate row f = 64 G + 16 q + (i % 16) when
// i < 16 and the matching up row (F + f) otherwise.  NVFP4 scales are stored
// unsigned: a negative block scale is folded into the signs of its 16 codes.
// The two NVFP4 tensor scales {s13, s2} end the blob.
__host__ __device__ static inline int fp4_chunk_bytes(int wfmt) { return wfmt == MOE_W_MXFP4 ? 16384 + 1024 : 16384 + 2048; }

struct BlobLayout {
    size_t w13, w2, ts, bytes;
    int tile_bytes;    // BF16: 2048
    int chunk_bytes;   // FP4: fp4_chunk_bytes
};

static inline BlobLayout blob_layout(const moe_shape* s)
{
    BlobLayout b{};
    size_t H = s->hidden, F = s->ffn;
    if (s->wfmt == MOE_W_BF16) {
        b.tile_bytes = 2048;
        b.w13 = 0;
        b.w2 = 2 * F * H * 2;
        b.ts = b.w2 + H * F * 2;
        b.bytes = align_up(b.ts, 128);
        return b;
    }
    const size_t cb = (size_t)fp4_chunk_bytes(s->wfmt);
    b.chunk_bytes = (int)cb;
    b.w13 = 0;
    b.w2 = (2 * F / 128) * (H / 256) * cb;
    b.ts = b.w2 + (H / 128) * (F / 256) * cb;
    b.bytes = align_up(b.ts + (s->wfmt == MOE_W_NVFP4 ? 8 : 0), 128);
    return b;
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f)
{
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// 2^p for |p| <= 126 (the operand-copy exponents stay within +-100)
__device__ __forceinline__ float pow2i(int p) { return __int_as_float((127 + p) << 23); }

__device__ __forceinline__ uint32_t lane_id()
{
    uint32_t l;
    asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
    return l;
}

}  // namespace moe

// ---------------------------------------------------------------- profiling
namespace moe {
void prof_count(int kind, int launches);
// Brackets the work enqueued on `st` during its lifetime with two events
// when timing is enabled (moe_profile_enable); a no-op otherwise.
class ProfScope {
  public:
    ProfScope(int kind, cudaStream_t st);
    ~ProfScope();
    ProfScope(const ProfScope&) = delete;
    ProfScope& operator=(const ProfScope&) = delete;

  private:
    int kind_;
    cudaStream_t st_;
    cudaEvent_t a_;
};
}  // namespace moe

// ---------------------------------------------------------------- internal launchers
namespace moe {
int launch_router(const void* x, int x_dtype, const uint16_t* wg, const float* bias, int n, int H,
                  int E, int k, float* logits, int32_t* idx, float* w, cudaStream_t st);
int launch_router_logits(const void* x, int x_dtype, const uint16_t* wg, const float* bias, int n, int H, int E,
                         float* logits, cudaStream_t st);
size_t permute_ws_bytes(int n, int E, int k);
int launch_permute(const int32_t* idx, int n, int E, int k, const void* x, int x_dtype, int H,
                   int32_t* offsets, int32_t* row_of, int32_t* assign_of, uint16_t* x_perm, void* ws,
                   cudaStream_t st);
size_t ffn_ws_bytes(const moe_shape* s, int rows);
// Source of the grouped FFN's input rows when x_perm is not materialised:
// row r is token assign_of[r] / k of x (x_dtype).
struct RowSource {
    const void* x;
    int x_dtype;
    const int32_t* assign_of;
    int k;
};
int ffn_device_error(int clear);   // BF16 streaming FFN's device error word (0: none)
// Testing hook (moe_test_set_wait): the wait limit the FFN kernels launched
// next get (dflt unless a test set one), and whether CTA 0 withholds a stage.
long long test_wait_cycles(long long dflt);
int test_withhold();
int ffn_fp4_device_error(int clear);   // FP4 FFN's device error word (0: none)
// one_expert: the pass computes at most one expert (a miss group after the
// first), so the FP4 decode tiles run on a grid sized for one expert's work.
int launch_ffn(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
               const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm, void* ws,
               cudaStream_t st, const RowSource* gather = nullptr, bool one_expert = false);
size_t ffn_fp4_ws_bytes(const moe_shape* s, int rows);
int launch_ffn_fp4(const moe_shape* s, const void* pool, size_t slot_bytes, int pool_slots, const int32_t* slot_of,
                   const int32_t* offsets, const uint16_t* x_perm, int rows, uint16_t* y_perm, void* ws,
                   cudaStream_t st, const RowSource* gather, bool one_expert);
int launch_combine(const uint16_t* y_perm, const int32_t* row_of, const float* w, int n, int k, int H,
                   void* out, int out_dtype, cudaStream_t st);

// ---------------------------------------------------------------- miss groups
// The misses of a decode layer call are filled, and their FFN run, in up to
// kMissGroups groups in miss-list order.  The last groups hold one miss
// each, so only the last miss's FFN waits for the last fill; every earlier
// group computes while later blobs are still being copied.  Groups are
// right-aligned: with nm misses, groups g < kMissGroups - min(nm,
// kMissGroups) are empty, and group g covers misses [*b, *e) of the list.
constexpr int kMissGroups = 4;

__host__ __device__ static inline void miss_group(int nm, int g, int* b, int* e)
{
    const int ng = nm < kMissGroups ? nm : kMissGroups;
    const int j = g - (kMissGroups - ng);   // index among the ng non-empty groups
    if (nm <= 0 || j < 0 || g >= kMissGroups) {
        *b = *e = 0;
        return;
    }
    const int first = nm - ng + 1;           // misses of the first non-empty group
    *b = j == 0 ? 0 : first + j - 1;
    *e = j == 0 ? first : first + j;
}

// ---------------------------------------------------------------- cache internals (cache.cu)
int cache_launch_lookup(moe_cache* c, int layer, const int32_t* idx, int count, int32_t* slot_user, cudaStream_t st);
bool cache_layer_resident(const moe_cache* c, int layer);
const int32_t* cache_slot_all(const moe_cache* c);
const int32_t* cache_slot_hit(const moe_cache* c);
const char* cache_pool(const moe_cache* c);
size_t cache_slot_bytes(const moe_cache* c);
int cache_read_and_fill(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, int* n_miss,
                        cudaEvent_t ev = nullptr, bool groups = false);
int cache_group_fills(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, unsigned* live);
int cache_launch_group_slots(moe_cache* c, int32_t* grp_slots, cudaStream_t st);
cudaEvent_t cache_group_event(const moe_cache* c, int g);
const moe_shape* cache_shape(const moe_cache* c);
int cache_capacity_int(const moe_cache* c);
int cache_fill_mode(const moe_cache* c);
int cache_launch_device_fill(moe_cache* c, int layer, cudaStream_t copy, cudaEvent_t ev = nullptr, int group = -1);
int cache_fill(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, cudaEvent_t ev);
cudaEvent_t cache_prefill_event(const moe_cache* c, int i);
bool cache_front_fits(const moe_cache* c, int n);
int cache_launch_front(moe_cache* c, int layer, const float* logits, int n, int32_t* idx, float* w,
                       int32_t* offsets, int32_t* row_of, int32_t* assign_of, cudaStream_t st);
}  // namespace moe
