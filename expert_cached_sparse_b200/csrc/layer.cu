// The whole routed MoE layer chained on one compute stream, with miss fills
// on a copy stream overlapped with the FFN over the hits.
//
// Pages: during decode the routed experts are checked in the GPU cache, hits
// execute directly on the GPU and misses are brought in ("FreeToken 290b
// model", section "Como gestiona FreeToken el prellenado y la
// decodificacion"); data movement is overlapped with computation instead of
// leaving the GPU idle ("FreeToken linux", mechanism table in section "Como
// gestiona FreeToken la memoria MoE").  Splitting misses between fills and
// CPU execution is not done here: every miss is filled and runs on the GPU.
#include "common.cuh"

namespace moe {
int cache_launch_lookup(moe_cache* c, int layer, const int32_t* idx, int count, int32_t* slot_user, cudaStream_t st);
bool cache_layer_resident(const moe_cache* c, int layer);
const int32_t* cache_slot_all(const moe_cache* c);
const int32_t* cache_slot_hit(const moe_cache* c);
const int32_t* cache_slot_miss(const moe_cache* c);
const char* cache_pool(const moe_cache* c);
size_t cache_slot_bytes(const moe_cache* c);
int cache_read_and_fill(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, int* n_miss);
cudaEvent_t cache_fill_event(const moe_cache* c);
const moe_shape* cache_shape(const moe_cache* c);
int cache_capacity_int(const moe_cache* c);
int cache_fill_mode(const moe_cache* c);
int cache_launch_device_fill(moe_cache* c, int layer, cudaStream_t copy);

struct LayerWs {
    float* logits;
    int32_t* idx;
    float* w;
    int32_t* offsets;
    int32_t* row_of;
    int32_t* assign_of;
    uint16_t* y_perm;
    void* ffn_ws;
    void* perm_ws;
    size_t bytes;
};

static LayerWs layer_ws(const moe_shape* s, int n, void* base)
{
    LayerWs L{};
    const size_t A = (size_t)n * s->top_k, E = s->experts, H = s->hidden;
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align_up(o + b, 256); return at; };
    size_t o_logits = take(4 * (size_t)n * E);
    size_t o_idx = take(4 * A);
    size_t o_w = take(4 * A);
    size_t o_off = take(4 * (E + 1));
    size_t o_row = take(4 * A);
    size_t o_asg = take(4 * A);
    size_t o_yp = take(2 * A * H);
    size_t o_ffn = take(ffn_ws_bytes(s, (int)A));
    size_t o_perm = take(permute_ws_bytes(n, s->experts, s->top_k));
    L.bytes = o;
    if (base) {
        char* b = static_cast<char*>(base);
        L.logits = reinterpret_cast<float*>(b + o_logits);
        L.idx = reinterpret_cast<int32_t*>(b + o_idx);
        L.w = reinterpret_cast<float*>(b + o_w);
        L.offsets = reinterpret_cast<int32_t*>(b + o_off);
        L.row_of = reinterpret_cast<int32_t*>(b + o_row);
        L.assign_of = reinterpret_cast<int32_t*>(b + o_asg);
        L.y_perm = reinterpret_cast<uint16_t*>(b + o_yp);
        L.ffn_ws = b + o_ffn;
        L.perm_ws = b + o_perm;
    }
    return L;
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_layer_workspace_bytes(const moe_shape* shape, int32_t n)
{
    if (!shape_ok(shape) || n < 0) return 0;
    return layer_ws(shape, n, nullptr).bytes;
}

extern "C" int moe_layer_forward(moe_cache* c, int32_t layer, const void* d_x, int32_t x_dtype, const uint16_t* d_wg,
                                 const float* d_bias, int32_t n, void* d_out, void* d_ws, size_t ws_bytes,
                                 void* stream, void* copy_stream, int32_t* d_topk_idx_out, float* d_topk_w_out)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    const moe_shape* s = cache_shape(c);
    if (layer < 0 || layer >= s->layers || n < 0) return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_x || !d_wg || !d_out || !d_ws)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_x | (uintptr_t)d_wg | (uintptr_t)d_out | (uintptr_t)d_ws) & 15) return MOE_ERR_INVALID_ARG;
    LayerWs L = layer_ws(s, n, d_ws);
    if (ws_bytes < L.bytes) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    cudaStream_t st = as_stream(stream), cp = as_stream(copy_stream);
    const int E = s->experts, k = s->top_k, H = s->hidden, A = n * k;
    int32_t* idx = d_topk_idx_out ? d_topk_idx_out : L.idx;
    float* w = d_topk_w_out ? d_topk_w_out : L.w;
    int rc;
    if ((rc = launch_router(d_x, x_dtype, d_wg, d_bias, n, H, E, k, L.logits, idx, w, st))) return rc;
    if ((rc = cache_launch_lookup(c, layer, idx, A, nullptr, st))) return rc;
    // Both FFN paths gather the token rows straight from x into their own
    // operand copies, so the permutation writes no x_perm.
    uint16_t* xp = nullptr;
    if ((rc = launch_permute(idx, n, E, k, d_x, x_dtype, H, L.offsets, L.row_of, L.assign_of, xp, L.perm_ws, st)))
        return rc;
    const RowSource src{d_x, x_dtype, L.assign_of, k};
    const RowSource* gather = &src;
    const char* pool = cache_pool(c);
    const size_t sb = cache_slot_bytes(c);
    const int C = cache_capacity_int(c);
    if (cache_fill_mode(c) == MOE_FILL_DEVICE) {
        // the copy kernel takes the miss list from the lookup on the device:
        // it starts first (it needs few SMs and only PCIe), the hits run
        // beside it, the misses after it.  Nothing is read back.
        if ((rc = cache_launch_device_fill(c, layer, cp))) return rc;
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_hit(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
        MOE_CUDA_TRY(cudaStreamWaitEvent(st, cache_fill_event(c), 0));
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_miss(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
    } else if (cache_layer_resident(c, layer)) {
        // every expert of this layer is resident: no miss is possible, nothing is read back
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_all(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
    } else {
        // hits first, while the host learns the miss list and issues the fills
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_hit(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
        int nm = 0;
        if ((rc = cache_read_and_fill(c, layer, st, cp, &nm))) return rc;
        if (nm > 0) {
            MOE_CUDA_TRY(cudaStreamWaitEvent(st, cache_fill_event(c), 0));
            if ((rc = launch_ffn(s, pool, sb, C, cache_slot_miss(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
                return rc;
        }
    }
    return launch_combine(L.y_perm, L.row_of, w, n, k, H, d_out, x_dtype, st);
}

extern "C" const char* moe_status_str(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_CAPACITY: return "more distinct experts requested than cache slots";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_FILL: return "expert fill failed";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or scale codes";
    case MOE_ERR_STATE: return "cache state error";
    }
    return "unknown status";
}

extern "C" int moe_version(void) { return 100; }
